// jfa_forward_fixed_scratch: the forward pass for callers that cannot
// allocate device memory.
//
// jfa_forward needs a caller-provided workspace (error word, tile schedule,
// dense-bias offsets).  Some callers have no way to obtain one: a plugin
// running inside a host framework that owns every byte of the device memory
// pool and exposes no allocator, or a serving loop whose policy forbids any
// allocation after start-up.  For them this entry point keeps that scratch
// in a file-scope __device__ array of fixed size, which every GPU that loads
// the library holds until the process exits.
//
// The array's name is only a host-side stand-in for the device symbol, so
// the host never passes it to a kernel; the device address is obtained with
// cudaGetSymbolAddress once per device (with that device current) on the
// first call made on that device, and cached.
#include <mutex>

#include "jfa_common.cuh"

namespace {

constexpr size_t kFixedScratchBytes = size_t(8) << 20;  // 8 MiB

__device__ __align__(256) uint8_t g_fixed_scratch[kFixedScratchBytes];

constexpr int kMaxDevices = 64;
void* g_scratch_ptr[kMaxDevices] = {};
std::mutex g_scratch_mu;

}  // namespace

extern "C" jfa_status jfa_forward_fixed_scratch(const jfa_problem* problem, const void* q,
                                                const void* k, const void* v,
                                                const int32_t* q_offsets,
                                                const int32_t* kv_offsets, const void* bias,
                                                jfa_act act, int causal, void* out, float* lse,
                                                jfa_stream_t stream) {
    const size_t need = jfa_workspace_bytes(problem, 0);
    if (need == 0)  // invalid descriptor: let jfa_forward report why
        return jfa_forward(problem, q, k, v, q_offsets, kv_offsets, bias, act, causal, out, lse,
                           nullptr, 0, stream);
    if (need > kFixedScratchBytes)
        return jfa::set_last_error(JFA_ERR_WORKSPACE,
                                   "problem needs %zu bytes of scratch; the fixed array holds %zu "
                                   "(use jfa_forward with a caller workspace)",
                                   need, kFixedScratchBytes);
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess || dev < 0 || dev >= kMaxDevices)
        return jfa::set_last_error(JFA_ERR_CUDA, "cudaGetDevice failed or device id out of range");
    void* scratch = nullptr;
    {
        std::lock_guard<std::mutex> lock(g_scratch_mu);
        if (!g_scratch_ptr[dev]) {
            void* p = nullptr;
            e = cudaGetSymbolAddress(&p, g_fixed_scratch);
            if (e != cudaSuccess || p == nullptr)
                return jfa::set_last_error(JFA_ERR_CUDA, "cudaGetSymbolAddress: %s",
                                           cudaGetErrorString(e));
            g_scratch_ptr[dev] = p;
        }
        scratch = g_scratch_ptr[dev];
    }
    // The schedule kernels rewrite the error word and every count before the
    // attention kernel reads them, so nothing left by an earlier call needs
    // clearing here.
    return jfa_forward(problem, q, k, v, q_offsets, kv_offsets, bias, act, causal, out, lse,
                       scratch, kFixedScratchBytes, stream);
}
