// Bias gradient support: zero the masked pairs of a dense jagged bias
// gradient before a causal or windowed backward.
//
// The backward kernels write ds_ij at every (query, key) pair of the tiles
// they visit, masked pairs of those tiles included (as 0).  Under a causal
// mask or a sliding window a key tile is never visited by the query rows
// that see none of its keys, so those pairs -- all masked -- are zeroed here:
// one warp per (head, query row) of a sequence clears the keys before the
// row's visible range and after it.
#include "jfa_common.cuh"

namespace jfa {
namespace {

template <typename T>
__global__ void __launch_bounds__(256) dbias_zero_masked_kernel(AttnArgs a) {
    if (a.hdr->err != 0) return;
    const int warps = blockDim.x >> 5, w = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int b = blockIdx.x; b < a.B; b += gridDim.x) {
        const int nq = a.q_off[b + 1] - a.q_off[b], nkv = a.kv_off[b + 1] - a.kv_off[b];
        T* blk = reinterpret_cast<T*>(a.dbias) + a.dense_off[b];
        for (int64_t row = w; row < (int64_t)a.H * nq; row += warps) {
            const int i = (int)(row % nq);
            T* dst = blk + row * nkv;
            const int lo = vis_key_lo(a.window, i, nq, nkv);
            const int hi = max(vis_key_hi(a.causal, a.window, i, nq, nkv), lo - 1);
            for (int j = lane; j < lo; j += 32) dst[j] = from_f<T>(0.f);
            for (int j = hi + 1 + lane; j < nkv; j += 32) dst[j] = from_f<T>(0.f);
        }
    }
}

}  // namespace

cudaError_t dbias_zero_masked(const AttnArgs& a, int elem_bytes, cudaStream_t st) {
    const int grid = a.B < 148 * 8 ? (a.B > 0 ? a.B : 1) : 148 * 8;
    prof_begin(st);
    if (elem_bytes == 4) dbias_zero_masked_kernel<float><<<grid, 256, 0, st>>>(a);
    else dbias_zero_masked_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>(a);
    prof_end(st, K_DBIAS_ZERO);
    return cudaGetLastError();
}

}  // namespace jfa
