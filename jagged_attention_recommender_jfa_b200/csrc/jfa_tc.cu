// Dispatch to the tensor-core (tcgen05) kernels: which problems they take and
// how they are launched.
//
// MXFP8 (dtype JFA_MXFP8): Q and K are quantised along d, V along 32-row
// blocks of each sequence (OCP MX: E4M3 elements, one E8M0 scale per 32) into
// the workspace, once, and the forward runs block-scaled E4M3 MMAs on them
// (P quantised per 32 keys inside the kernel); jfa_forward_mxfp8 takes
// operands quantised by their producer and skips that pass.  The backward
// computes bf16 gradients on the dequantised Q/K/V (straight-through
// quantiser).
#include "jfa_common.cuh"

namespace jfa {

cudaError_t tc_forward_launch(const jfa_problem& p, const AttnArgs& a, cudaStream_t st);
cudaError_t tc_backward_launch(const jfa_problem& p, const AttnArgs& a, const AttnArgs& kv,
                               cudaStream_t st);
cudaError_t tc_bwd_pre_launch(const jfa_problem& p, const AttnArgs& a, cudaStream_t st);
cudaError_t tc_backward_sq_launch(const jfa_problem& p, const AttnArgs& a, cudaStream_t st);
bool tc_backward_short_q(const jfa_problem& p);
cudaError_t tc_forward_sq_launch(const jfa_problem& p, const AttnArgs& a, cudaStream_t st);
cudaError_t mx_fake_quant_qkv(const void* q, const void* k, const void* v, const int32_t* kv_off,
                              int64_t total_q, int64_t total_kv, int heads, int d, int batch,
                              int max_kv_len, void* qf, void* kf, void* vf, cudaStream_t st);
cudaError_t quantize_mx(const void* x, int64_t rows, int heads, int d, const int32_t* offsets,
                        int batch, int max_rows_per_seq, int along_rows, uint8_t* codes,
                        uint8_t* scales, void* dequant, cudaStream_t st);
cudaError_t tc_forward_mx_launch(const jfa_problem& p, const AttnArgs& a, const void* q8,
                                 const uint8_t* qs, const void* k8, const uint8_t* ks,
                                 const void* v8, const uint8_t* vs, int64_t n_vblocks,
                                 int32_t* vbase, cudaStream_t st);

// bf16 storage with head_dim 128 (any activation and bias kind); MXFP8 with
// head_dim 128 and softmax.
bool tc_supported(const jfa_problem& p, int act, int backward) {
    (void)backward;
    if (p.head_dim != 128) return false;
    if (p.dtype == JFA_BF16) return true;
    return p.dtype == JFA_MXFP8 && act == JFA_ACT_SOFTMAX;
}

namespace {
struct Extra {
    size_t dq_acc, qf, kf, vf, bias4, total;
    size_t q8, qs, k8, ks, v8, vs, vbase;   // MXFP8 forward: quantised operands
};
int64_t mx_vblocks(const jfa_problem& p) { return p.total_kv / 32 + p.batch; }
// entries per head of the prepared table: the table, and at least the
// 384-entry window the forward stages per key tile
int bias4_stride(const jfa_problem& p) { return p.relpos_len < 384 ? 384 : p.relpos_len; }
Extra extra_layout(const jfa_problem& p, int backward) {
    Extra e{};
    size_t off = 0;
    if (p.bias_kind == JFA_BIAS_RELPOS) {
        e.bias4 = off;
        off = align256(off + sizeof(float4) * (size_t)p.heads * bias4_stride(p));
    }
    if (backward) {
        e.dq_acc = off;
        off = align256(off + sizeof(float) * (size_t)p.total_q * p.heads * p.head_dim);
    }
    if (p.dtype == JFA_MXFP8 && backward) {
        e.qf = off; off = align256(off + 2 * (size_t)p.total_q * p.heads * p.head_dim);
        e.kf = off; off = align256(off + 2 * (size_t)p.total_kv * p.heads * p.head_dim);
        e.vf = off; off = align256(off + 2 * (size_t)p.total_kv * p.heads * p.head_dim);
    }
    if (p.dtype == JFA_MXFP8 && !backward) {
        const size_t hd = (size_t)p.heads * p.head_dim;
        e.q8 = off; off = align256(off + (size_t)p.total_q * hd);
        e.qs = off; off = align256(off + (size_t)p.total_q * hd / 32);
        e.k8 = off; off = align256(off + (size_t)p.total_kv * hd);
        e.ks = off; off = align256(off + (size_t)p.total_kv * hd / 32);
        e.v8 = off; off = align256(off + (size_t)p.total_kv * hd);
        e.vs = off; off = align256(off + (size_t)mx_vblocks(p) * hd);
        e.vbase = off; off = align256(off + sizeof(int32_t) * (size_t)(p.batch > 0 ? p.batch : 1));
    }
    e.total = off;
    return e;
}

cudaError_t fake_quant(const jfa_problem& p, AttnArgs& a, char* ws, const Extra& L, cudaStream_t st) {
    void *qf = ws + L.qf, *kf = ws + L.kf, *vf = ws + L.vf;
    cudaError_t e = mx_fake_quant_qkv(a.q, a.k, a.v, a.kv_off, p.total_q, p.total_kv, p.heads,
                                      p.head_dim, p.batch, p.max_kv_len, qf, kf, vf, st);
    a.q = qf;
    a.k = kf;
    a.v = vf;
    return e;
}
// out[h * stride + t] = log2(e) * (table[h][t], table[h][t+1], table[h][t+2],
// table[h][t+3]), indices clamped to len - 1: entry t is the run of four that
// starts at t, so any run of the table can be read as 16-byte-aligned float4s
__global__ void __launch_bounds__(256) tc_bias_prep(const float* __restrict__ tab, int len, int heads,
                                                    int stride, float4* __restrict__ out) {
    const int64_t n = (int64_t)heads * stride;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int t = (int)(i % stride), h = (int)(i / stride);
        const float* row = tab + (int64_t)h * len;
        const float k = 1.4426950408889634f;
        out[i] = make_float4(row[min(t, len - 1)] * k, row[min(t + 1, len - 1)] * k,
                             row[min(t + 2, len - 1)] * k, row[min(t + 3, len - 1)] * k);
    }
}

cudaError_t prep_bias(const jfa_problem& p, AttnArgs& a, char* ws, const Extra& L, cudaStream_t st) {
    if (p.bias_kind != JFA_BIAS_RELPOS) return cudaSuccess;
    const int stride = bias4_stride(p);
    float* out = reinterpret_cast<float*>(ws + L.bias4);
    const int64_t n = (int64_t)p.heads * stride;
    const int blocks = (int)((n + 255) / 256 < 1024 ? (n + 255) / 256 : 1024);
    prof_begin(st);
    tc_bias_prep<<<blocks, 256, 0, st>>>(reinterpret_cast<const float*>(a.bias), p.relpos_len, p.heads,
                                          stride, reinterpret_cast<float4*>(out));
    prof_end(st, K_TC_BIAS_PREP);
    a.bias4 = out;
    a.bias4_stride = stride;
    return cudaGetLastError();
}
}  // namespace

// The backward keeps an fp32 dQ accumulator [total_q][heads][128] and, for
// MXFP8, the three dequantised operands; the MXFP8 forward keeps the E4M3
// codes and E8M0 scales of Q, K and V; a relative-position bias adds its
// log2(e)-scaled table of runs of four.
size_t tc_workspace_extra(const jfa_problem& p, int backward) {
    return extra_layout(p, backward).total;
}

cudaError_t tc_forward(const jfa_problem& p, const AttnArgs& a, void* ws_extra, cudaStream_t st) {
    AttnArgs aa = a;
    {
        cudaError_t e = prep_bias(p, aa, reinterpret_cast<char*>(ws_extra), extra_layout(p, 0), st);
        if (e != cudaSuccess) return e;
    }
    if (p.dtype == JFA_MXFP8) {
        // quantise Q, K along d and V along 32-key blocks once, then the
        // block-scaled kernel
        char* ws = reinterpret_cast<char*>(ws_extra);
        const Extra L = extra_layout(p, 0);
        uint8_t *q8 = reinterpret_cast<uint8_t*>(ws + L.q8), *k8 = reinterpret_cast<uint8_t*>(ws + L.k8);
        uint8_t *v8 = reinterpret_cast<uint8_t*>(ws + L.v8);
        uint8_t *qs = reinterpret_cast<uint8_t*>(ws + L.qs), *ks = reinterpret_cast<uint8_t*>(ws + L.ks);
        uint8_t *vs = reinterpret_cast<uint8_t*>(ws + L.vs);
        cudaError_t e = quantize_mx(a.q, p.total_q, p.heads, p.head_dim, nullptr, 0, 0, 0, q8, qs, nullptr, st);
        if (e == cudaSuccess)
            e = quantize_mx(a.k, p.total_kv, p.heads, p.head_dim, nullptr, 0, 0, 0, k8, ks, nullptr, st);
        if (e == cudaSuccess)
            e = quantize_mx(a.v, p.total_kv, p.heads, p.head_dim, a.kv_off, p.batch, p.max_kv_len, 1,
                            v8, vs, nullptr, st);
        if (e != cudaSuccess) return e;
        return tc_forward_mx_launch(p, aa, q8, qs, k8, ks, v8, vs, mx_vblocks(p),
                                    reinterpret_cast<int32_t*>(ws + L.vbase), st);
    }
    // short query sequences: two (sequence, head) items per CTA step
    if (tc_backward_short_q(p)) return tc_forward_sq_launch(p, aa, st);
    return tc_forward_launch(p, aa, st);
}

// Forward on operands quantised by their producer (jfa_forward_mxfp8).
cudaError_t tc_forward_mx_prequant(const jfa_problem& p, const AttnArgs& a, const void* q8,
                                   const uint8_t* qs, const void* k8, const uint8_t* ks,
                                   const void* v8, const uint8_t* vs, void* ws_extra,
                                   cudaStream_t st) {
    AttnArgs aa = a;
    const Extra L = extra_layout(p, 0);
    cudaError_t e = prep_bias(p, aa, reinterpret_cast<char*>(ws_extra), L, st);
    if (e != cudaSuccess) return e;
    return tc_forward_mx_launch(p, aa, q8, qs, k8, ks, v8, vs, mx_vblocks(p),
                                reinterpret_cast<int32_t*>(reinterpret_cast<char*>(ws_extra) + L.vbase), st);
}

cudaError_t tc_backward(const jfa_problem& p, const AttnArgs& a, const AttnArgs& kv,
                        void* ws_extra, cudaStream_t st) {
    const Extra L = extra_layout(p, 1);
    char* ws = reinterpret_cast<char*>(ws_extra);
    AttnArgs aq = a, akv = kv;
    aq.dq_acc = reinterpret_cast<float*>(ws + L.dq_acc);
    akv.dq_acc = aq.dq_acc;
    {
        cudaError_t e = prep_bias(p, akv, ws, L, st);
        if (e != cudaSuccess) return e;
        aq.bias4 = akv.bias4;
        aq.bias4_stride = akv.bias4_stride;
    }
    if (p.dtype == JFA_MXFP8) {
        cudaError_t e = fake_quant(p, aq, ws, L, st);
        if (e != cudaSuccess) return e;
        akv.q = aq.q;
        akv.k = aq.k;
        akv.v = aq.v;
    }
    if (tc_backward_short_q(p)) {
        // query-stationary: one CTA per (sequence, head), items from the
        // query-block schedule in `a`
        cudaError_t e = tc_bwd_pre_launch(p, aq, st);
        if (e != cudaSuccess) return e;
        return tc_backward_sq_launch(p, aq, st);
    }
    return tc_backward_launch(p, aq, akv, st);
}

// Short query sequences (every n_q <= 64) take the paired-item forward and
// the query-stationary backward; with a sliding window the general kernels,
// which compute only the key tiles inside the band, run instead.
bool tc_backward_short_q(const jfa_problem& p) { return p.max_q_len <= 64 && p.window == 0; }

int tc_fwd_tile() { return 256; }   // a forward work item is a 256-row query block
int tc_bwd_tile() { return 128; }

}  // namespace jfa
