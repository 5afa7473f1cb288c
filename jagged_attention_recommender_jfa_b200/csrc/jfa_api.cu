// C ABI of libjfa: host-side validation, workspace carve-out and dispatch.
// The operations are defined in include/jfa.h.
#include <math.h>
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include <vector>

#include "jfa_common.cuh"

namespace jfa {
cudaError_t build_schedule(const jfa_problem& pb, const int32_t* q_off, const int32_t* kv_off,
                           int causal, int backward, int tile, WsHeader* hdr, int64_t* dense_off,
                           int2* pair_bt, int64_t* pair_cost, int64_t pairs_cap, int4* items,
                           int32_t* item_count, int32_t* pair_count, int reset_err,
                           int64_t* seq_tmp, int64_t* seq_start, cudaStream_t stream,
                           int wait_limit_us = 0, int cost_tiles = 0);
cudaError_t simt_forward(const AttnArgs& a, int head_dim, bool bf16, int grid, cudaStream_t st);
cudaError_t simt_backward(const AttnArgs& a, const AttnArgs& kv_args, int head_dim, bool bf16,
                          int grid_q, int grid_kv, int64_t rows, cudaStream_t st);
cudaError_t quantize_mx(const void* x, int64_t rows, int heads, int d, const int32_t* offsets,
                        int batch, int max_rows_per_seq, int along_rows, uint8_t* codes,
                        uint8_t* scales, void* dequant, cudaStream_t st);
bool tc_supported(const jfa_problem& p, int act, int backward);
size_t tc_workspace_extra(const jfa_problem& p, int backward);
cudaError_t tc_forward(const jfa_problem& p, const AttnArgs& a, void* ws_extra, cudaStream_t st);
cudaError_t tc_backward(const jfa_problem& p, const AttnArgs& a, const AttnArgs& kv_args,
                        void* ws_extra, cudaStream_t st);
int tc_fwd_tile();
int tc_bwd_tile();
bool tc_backward_short_q(const jfa_problem& p);
cudaError_t dbias_zero_masked(const AttnArgs& a, int elem_bytes, cudaStream_t st);
cudaError_t tc_forward_mx_prequant(const jfa_problem& p, const AttnArgs& a, const void* q8,
                                   const uint8_t* qs, const void* k8, const uint8_t* ks,
                                   const void* v8, const uint8_t* vs, void* ws_extra,
                                   cudaStream_t st);
}  // namespace jfa

using namespace jfa;

// ---------------------------------------------------------------------------
// Launch timing: a per-thread record of (start event, stop event, kernel id).
// ---------------------------------------------------------------------------
namespace {

struct Profiler {
    bool on = false;
    std::vector<cudaEvent_t> pool;
    size_t used = 0;
    std::vector<int> ids;
    ~Profiler() {}
    cudaEvent_t next() {
        if (used == pool.size()) {
            cudaEvent_t e;
            if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
            pool.push_back(e);
        }
        return pool[used++];
    }
};
thread_local Profiler g_prof;
thread_local char g_msg[512] = "";
thread_local int g_test_hook = 0;       // jfa_test_inject: armed for the next forward
constexpr int kTestWaitLimitUs = 5000;  // the injected failure's wait limit

const char* const kKernelNames[K_COUNT] = {
    "sched_prepare", "sched_rank", "simt_fwd", "simt_bwd_pre", "simt_bwd_dq", "simt_bwd_dkdv",
    "mx_along_d", "mx_along_rows", "tc_fwd", "tc_bwd_pre", "tc_bwd", "tc_dq_finalize",
    "tc_fwd_mxfp8", "tc_bias_prep", "dbias_zero_masked", "norm_quantize_mxfp8", "tc_bwd_sq", "tc_fwd_sq"};

}  // namespace

namespace jfa {
jfa_status set_last_error(jfa_status s, const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_msg, sizeof(g_msg), fmt, ap);
    va_end(ap);
    return s;
}

void prof_begin(cudaStream_t st) {
    if (!g_prof.on) return;
    cudaEvent_t e = g_prof.next();
    if (e) cudaEventRecord(e, st);
}
void prof_end(cudaStream_t st, int kernel_id) {
    if (!g_prof.on) return;
    cudaEvent_t e = g_prof.next();
    if (e) cudaEventRecord(e, st);
    g_prof.ids.push_back(kernel_id);
}
}  // namespace jfa

namespace {

jfa_status fail(jfa_status s, const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_msg, sizeof(g_msg), fmt, ap);
    va_end(ap);
    return s;
}

jfa_status cuda_fail(cudaError_t e, const char* where) {
    return fail(JFA_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
}

constexpr int kSimtFwdTile = 64;   // query rows per CUDA-core forward / dQ item
constexpr int kSimtBwdTile = 64;   // key rows per CUDA-core dK/dV item

jfa_status check_problem(const jfa_problem* p) {
    if (!p) return fail(JFA_ERR_INVALID_ARGUMENT, "problem is NULL");
    if (p->batch < 0 || p->heads < 1 || p->max_q_len < 0 || p->max_kv_len < 0 ||
        p->total_q < 0 || p->total_kv < 0)
        return fail(JFA_ERR_INVALID_ARGUMENT, "negative size in problem");
    if (p->total_q >= (int64_t)1 << 31 || p->total_kv >= (int64_t)1 << 31)
        return fail(JFA_ERR_INVALID_ARGUMENT, "total rows must fit int32 offsets");
    if (p->head_dim != 32 && p->head_dim != 64 && p->head_dim != 128)
        return fail(JFA_ERR_UNSUPPORTED, "head_dim %d not in {32, 64, 128}", p->head_dim);
    if (p->dtype != JFA_F32 && p->dtype != JFA_BF16 && p->dtype != JFA_MXFP8)
        return fail(JFA_ERR_INVALID_ARGUMENT, "bad dtype %d", (int)p->dtype);
    if (p->bias_kind != JFA_BIAS_NONE && p->bias_kind != JFA_BIAS_RELPOS &&
        p->bias_kind != JFA_BIAS_DENSE_JAGGED)
        return fail(JFA_ERR_INVALID_ARGUMENT, "bad bias_kind %d", (int)p->bias_kind);
    if (p->bias_kind == JFA_BIAS_RELPOS && (p->relpos_len < 1 || (p->relpos_len & 1) == 0))
        return fail(JFA_ERR_INVALID_ARGUMENT, "relpos_len must be odd and >= 1");
    if (!(p->scale == p->scale)) return fail(JFA_ERR_INVALID_ARGUMENT, "scale is NaN");
    if (p->window < 0) return fail(JFA_ERR_INVALID_ARGUMENT, "negative window %d", p->window);
    return JFA_OK;
}

jfa_status check_act(int act) {
    if (act != JFA_ACT_SOFTMAX && act != JFA_ACT_SILU && act != JFA_ACT_GELU_TANH)
        return fail(JFA_ERR_INVALID_ARGUMENT, "bad act %d", act);
    return JFA_OK;
}

bool use_tc(const jfa_problem& p, int act, int backward) { return tc_supported(p, act, backward); }

size_t workspace_bytes(const jfa_problem& p, int backward) {
    WsLayout L = ws_layout(p, backward != 0, false);
    size_t extra = 0;
    if (use_tc(p, JFA_ACT_SOFTMAX, backward) || use_tc(p, JFA_ACT_SILU, backward))
        extra = tc_workspace_extra(p, backward);
    return L.total + align256(extra);
}

// MXFP8 runs only on the tensor-core path (head_dim 128, softmax).
jfa_status check_mxfp8(const jfa_problem& p, int act) {
    if (p.dtype == JFA_MXFP8 && !use_tc(p, act, 0))
        return fail(JFA_ERR_UNSUPPORTED, "MXFP8 needs head_dim 128 and softmax");
    return JFA_OK;
}

float eff_scale(const jfa_problem& p) {
    return p.scale > 0.f ? p.scale : 1.0f / sqrtf((float)p.head_dim);
}

#define ALIGNED16(ptr) ((((uintptr_t)(ptr)) & 15u) == 0)

}  // namespace

extern "C" {

size_t jfa_workspace_bytes(const jfa_problem* problem, int backward) {
    if (check_problem(problem) != JFA_OK) return 0;
    return workspace_bytes(*problem, backward);
}

const char* jfa_last_error(void) { return g_msg; }

int jfa_path(const jfa_problem* problem, jfa_act act, int backward) {
    if (check_problem(problem) != JFA_OK) return -1;
    return use_tc(*problem, act, backward) ? 1 : 0;
}

}  // extern "C"

namespace {

// MXFP8 operands quantised by their producer (jfa_forward_mxfp8)
struct PreQuant {
    const uint8_t *q8, *qs, *k8, *ks, *v8, *vs;
};

jfa_status forward_impl(const jfa_problem* problem, const void* q, const void* k, const void* v,
                        const int32_t* q_offsets, const int32_t* kv_offsets, const void* bias,
                        jfa_act act, int causal, void* out, float* lse, void* workspace,
                        size_t ws_bytes, jfa_stream_t stream, const PreQuant* pq) {
    jfa_status s = check_problem(problem);
    if (s != JFA_OK) return s;
    if ((s = check_act(act)) != JFA_OK) return s;
    const jfa_problem& p = *problem;
    if ((s = check_mxfp8(p, act)) != JFA_OK) return s;
    if (!q_offsets || !kv_offsets || !workspace) return fail(JFA_ERR_INVALID_ARGUMENT, "NULL offsets or workspace");
    if ((p.total_q > 0 && (!q || !out)) || (p.total_kv > 0 && (!k || !v)))
        return fail(JFA_ERR_INVALID_ARGUMENT, "NULL tensor");
    if (p.bias_kind != JFA_BIAS_NONE && !bias) return fail(JFA_ERR_INVALID_ARGUMENT, "NULL bias");
    if (!ALIGNED16(q) || !ALIGNED16(k) || !ALIGNED16(v) || !ALIGNED16(out) || !ALIGNED16(workspace))
        return fail(JFA_ERR_INVALID_ARGUMENT, "tensors and workspace must be 16-byte aligned");
    if (ws_bytes < workspace_bytes(p, 0)) return fail(JFA_ERR_WORKSPACE, "workspace %zu < %zu bytes", ws_bytes, workspace_bytes(p, 0));
    if (p.batch == 0) return JFA_OK;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    char* ws = reinterpret_cast<char*>(workspace);
    WsLayout L = ws_layout(p, false, false);
    WsHeader* hdr = reinterpret_cast<WsHeader*>(ws);
    const bool tc = use_tc(p, act, 0);
    const int tile = tc ? tc_fwd_tile() : kSimtFwdTile;
    const bool inject = tc && g_test_hook == JFA_TEST_FWD_SKIP_LOAD;
    g_test_hook = 0;
    cudaError_t e = build_schedule(p, q_offsets, kv_offsets, causal, 0, tile, hdr,
                                   reinterpret_cast<int64_t*>(ws + L.dense_off),
                                   reinterpret_cast<int2*>(ws + L.pair_bt),
                                   reinterpret_cast<int64_t*>(ws + L.pair_cost), L.pairs_max_q,
                                   reinterpret_cast<int4*>(ws + L.items), &hdr->item_count,
                                   &hdr->pair_count, 1, nullptr, nullptr, st,
                                   inject ? kTestWaitLimitUs : 0,
                                   (tc && p.dtype != JFA_MXFP8 && tc_backward_short_q(p)) ? 1 : 0);
    if (e != cudaSuccess) return cuda_fail(e, "schedule");
    AttnArgs a{};
    a.q = q; a.k = k; a.v = v; a.q_off = q_offsets; a.kv_off = kv_offsets;
    a.bias = bias; a.dense_off = reinterpret_cast<const int64_t*>(ws + L.dense_off);
    a.bias_kind = p.bias_kind; a.relpos_len = p.relpos_len; a.B = p.batch; a.H = p.heads;
    a.causal = causal ? 1 : 0; a.window = p.window; a.act = act; a.scale = eff_scale(p);
    a.out = out; a.lse = (act == JFA_ACT_SOFTMAX) ? lse : nullptr;
    a.items = reinterpret_cast<const int4*>(ws + L.items); a.item_count = &hdr->item_count;
    a.hdr = hdr;
    a.test_skip_load = inject ? 1 : 0;
    if (pq) {
        e = tc_forward_mx_prequant(p, a, pq->q8, pq->qs, pq->k8, pq->ks, pq->v8, pq->vs,
                                   ws + L.total, st);
    } else if (tc) {
        e = tc_forward(p, a, ws + L.total, st);
    } else {
        int64_t grid = pairs_bound(p.batch, p.max_q_len, p.total_q, tile) * p.heads;
        if (grid > 0x7fffffff) return fail(JFA_ERR_UNSUPPORTED, "too many tiles");
        e = simt_forward(a, p.head_dim, p.dtype != JFA_F32, (int)grid, st);
    }
    if (e != cudaSuccess) return cuda_fail(e, "forward");
    return JFA_OK;
}

}  // namespace

extern "C" {

jfa_status jfa_forward(const jfa_problem* problem, const void* q, const void* k, const void* v,
                       const int32_t* q_offsets, const int32_t* kv_offsets, const void* bias,
                       jfa_act act, int causal, void* out, float* lse, void* workspace,
                       size_t ws_bytes, jfa_stream_t stream) {
    return forward_impl(problem, q, k, v, q_offsets, kv_offsets, bias, act, causal, out, lse,
                        workspace, ws_bytes, stream, nullptr);
}

jfa_status jfa_forward_mxfp8(const jfa_problem* problem, const uint8_t* q8, const uint8_t* q_scales,
                             const uint8_t* k8, const uint8_t* k_scales, const uint8_t* v8,
                             const uint8_t* v_scales, const int32_t* q_offsets,
                             const int32_t* kv_offsets, const void* bias, int causal, void* out,
                             float* lse, void* workspace, size_t ws_bytes, jfa_stream_t stream) {
    jfa_status s = check_problem(problem);
    if (s != JFA_OK) return s;
    if (problem->dtype != JFA_MXFP8 || problem->head_dim != 128)
        return fail(JFA_ERR_UNSUPPORTED, "jfa_forward_mxfp8 needs dtype JFA_MXFP8 and head_dim 128");
    if ((problem->total_q > 0 && (!q8 || !q_scales)) || (problem->total_kv > 0 && (!k8 || !k_scales || !v8 || !v_scales)))
        return fail(JFA_ERR_INVALID_ARGUMENT, "NULL quantised operand or scales");
    const PreQuant pq{q8, q_scales, k8, k_scales, v8, v_scales};
    return forward_impl(problem, q8, k8, v8, q_offsets, kv_offsets, bias, JFA_ACT_SOFTMAX, causal,
                        out, lse, workspace, ws_bytes, stream, &pq);
}

}  // extern "C"

namespace {

jfa_status backward_impl(const jfa_problem* problem, const void* q, const void* k, const void* v,
                         const void* out, const float* lse, const void* dout,
                         const int32_t* q_offsets, const int32_t* kv_offsets, const void* bias,
                         jfa_act act, int causal, void* dq, void* dk, void* dv, void* dbias,
                         void* workspace, size_t ws_bytes, jfa_stream_t stream) {
    jfa_status s = check_problem(problem);
    if (s != JFA_OK) return s;
    if ((s = check_act(act)) != JFA_OK) return s;
    const jfa_problem& p = *problem;
    if ((s = check_mxfp8(p, act)) != JFA_OK) return s;
    if (!q_offsets || !kv_offsets || !workspace) return fail(JFA_ERR_INVALID_ARGUMENT, "NULL offsets or workspace");
    if ((p.total_q > 0 && (!q || !dout || !dq)) || (p.total_kv > 0 && (!k || !v || !dk || !dv)))
        return fail(JFA_ERR_INVALID_ARGUMENT, "NULL tensor");
    if (act == JFA_ACT_SOFTMAX && p.total_q > 0 && (!out || !lse))
        return fail(JFA_ERR_INVALID_ARGUMENT, "softmax backward needs out and lse");
    if (p.bias_kind != JFA_BIAS_NONE && !bias) return fail(JFA_ERR_INVALID_ARGUMENT, "NULL bias");
    if (!ALIGNED16(q) || !ALIGNED16(k) || !ALIGNED16(v) || !ALIGNED16(dout) || !ALIGNED16(dq) ||
        !ALIGNED16(dk) || !ALIGNED16(dv) || !ALIGNED16(workspace) || !ALIGNED16(out))
        return fail(JFA_ERR_INVALID_ARGUMENT, "tensors and workspace must be 16-byte aligned");
    if (ws_bytes < workspace_bytes(p, 1)) return fail(JFA_ERR_WORKSPACE, "workspace %zu < %zu bytes", ws_bytes, workspace_bytes(p, 1));
    if (dbias && p.bias_kind == JFA_BIAS_NONE)
        return fail(JFA_ERR_INVALID_ARGUMENT, "dbias given for a problem without a bias");
    if (dbias && !ALIGNED16(dbias)) return fail(JFA_ERR_INVALID_ARGUMENT, "dbias must be 16-byte aligned");
    if (p.batch == 0) return JFA_OK;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (dbias && p.bias_kind == JFA_BIAS_RELPOS) {
        // the kernels add every pair's score gradient into the table
        cudaError_t e0 = cudaMemsetAsync(dbias, 0, sizeof(float) * (size_t)p.heads * p.relpos_len, st);
        if (e0 != cudaSuccess) return cuda_fail(e0, "dbias zero");
    }
    char* ws = reinterpret_cast<char*>(workspace);
    WsLayout L = ws_layout(p, true, false);
    WsHeader* hdr = reinterpret_cast<WsHeader*>(ws);
    const bool tc = use_tc(p, act, 1);
    // short queries on the tensor cores: one item per (sequence, head)
    const bool sq = tc && tc_backward_short_q(p);
    const int qtile = tc ? tc_fwd_tile() : kSimtFwdTile;
    const int ktile = tc ? tc_bwd_tile() : kSimtBwdTile;
    // the CUDA-core backward walks both schedules, the query-stationary one
    // only the query-block one, the key-stationary one only the key-tile one
    // (the first build resets the error word and, for a dense bias, writes
    // the sequences' bias offsets)
    cudaError_t e = cudaSuccess;
    if (!tc || sq) {
        e = build_schedule(p, q_offsets, kv_offsets, causal, 0, qtile, hdr,
                           reinterpret_cast<int64_t*>(ws + L.dense_off),
                           reinterpret_cast<int2*>(ws + L.pair_bt),
                           reinterpret_cast<int64_t*>(ws + L.pair_cost), L.pairs_max_q,
                           reinterpret_cast<int4*>(ws + L.items), &hdr->item_count,
                           &hdr->pair_count, 1, nullptr, nullptr, st, 0, sq ? 1 : 0);
        if (e != cudaSuccess) return cuda_fail(e, "schedule");
    }
    if (!sq) {
        e = build_schedule(p, q_offsets, kv_offsets, causal, 1, ktile, hdr,
                           tc ? reinterpret_cast<int64_t*>(ws + L.dense_off) : nullptr,
                           reinterpret_cast<int2*>(ws + L.kv_pair_bt),
                           reinterpret_cast<int64_t*>(ws + L.kv_pair_cost), L.pairs_max_kv,
                           reinterpret_cast<int4*>(ws + L.kv_items), &hdr->kv_item_count,
                           &hdr->kv_pair_count, tc ? 1 : 0, reinterpret_cast<int64_t*>(ws + L.kv_seq_tmp),
                           reinterpret_cast<int64_t*>(ws + L.kv_seq_start), st);
        if (e != cudaSuccess) return cuda_fail(e, "schedule");
    }
    AttnArgs a{};
    a.q = q; a.k = k; a.v = v; a.q_off = q_offsets; a.kv_off = kv_offsets;
    a.bias = bias; a.dense_off = reinterpret_cast<const int64_t*>(ws + L.dense_off);
    a.bias_kind = p.bias_kind; a.relpos_len = p.relpos_len; a.B = p.batch; a.H = p.heads;
    a.causal = causal ? 1 : 0; a.window = p.window; a.act = act; a.scale = eff_scale(p);
    a.out = const_cast<void*>(out); a.lse = const_cast<float*>(lse);
    a.items = reinterpret_cast<const int4*>(ws + L.items); a.item_count = &hdr->item_count;
    a.hdr = hdr;
    a.dout = dout; a.dterm = reinterpret_cast<float*>(ws + L.dterm);
    a.dq = dq; a.dk = dk; a.dv = dv;
    a.dbias = dbias;
    if (dbias && p.bias_kind == JFA_BIAS_DENSE_JAGGED && (causal || p.window > 0)) {
        // masked pairs of a causal or windowed block get 0; the kernels write the rest
        e = dbias_zero_masked(a, p.dtype == JFA_F32 ? 4 : 2, st);
        if (e != cudaSuccess) return cuda_fail(e, "dbias zero");
    }
    AttnArgs kv = a;
    kv.items = reinterpret_cast<const int4*>(ws + L.kv_items);
    kv.item_count = &hdr->kv_item_count;
    if (tc) {
        e = tc_backward(p, a, kv, ws + L.total, st);
    } else {
        int64_t gq = pairs_bound(p.batch, p.max_q_len, p.total_q, qtile) * p.heads;
        int64_t gk = pairs_bound(p.batch, p.max_kv_len, p.total_kv, ktile) * p.heads;
        if (gq > 0x7fffffff || gk > 0x7fffffff) return fail(JFA_ERR_UNSUPPORTED, "too many tiles");
        e = simt_backward(a, kv, p.head_dim, p.dtype != JFA_F32, (int)gq, (int)gk,
                          p.total_q * p.heads, st);
    }
    if (e != cudaSuccess) return cuda_fail(e, "backward");
    return JFA_OK;
}

}  // namespace

extern "C" {

jfa_status jfa_backward(const jfa_problem* problem, const void* q, const void* k, const void* v,
                        const void* out, const float* lse, const void* dout,
                        const int32_t* q_offsets, const int32_t* kv_offsets, const void* bias,
                        jfa_act act, int causal, void* dq, void* dk, void* dv, void* workspace,
                        size_t ws_bytes, jfa_stream_t stream) {
    return backward_impl(problem, q, k, v, out, lse, dout, q_offsets, kv_offsets, bias, act,
                         causal, dq, dk, dv, nullptr, workspace, ws_bytes, stream);
}

jfa_status jfa_backward_dbias(const jfa_problem* problem, const void* q, const void* k,
                              const void* v, const void* out, const float* lse, const void* dout,
                              const int32_t* q_offsets, const int32_t* kv_offsets,
                              const void* bias, jfa_act act, int causal, void* dq, void* dk,
                              void* dv, void* dbias, void* workspace, size_t ws_bytes,
                              jfa_stream_t stream) {
    return backward_impl(problem, q, k, v, out, lse, dout, q_offsets, kv_offsets, bias, act,
                         causal, dq, dk, dv, dbias, workspace, ws_bytes, stream);
}

namespace {
jfa_status quantize_entry(const void* x_bf16, int64_t rows, int32_t heads, int32_t d,
                          const int32_t* offsets, int32_t batch, int32_t max_len, int along_rows,
                          uint8_t* codes, uint8_t* scales, void* dequant, jfa_stream_t stream) {
    if (rows < 0 || heads < 1 || d < 32 || (d % 32) != 0)
        return fail(JFA_ERR_INVALID_ARGUMENT, "bad quantiser sizes");
    if (rows > 0 && (!x_bf16 || !codes || !scales)) return fail(JFA_ERR_INVALID_ARGUMENT, "NULL tensor");
    if (!ALIGNED16(x_bf16) || !ALIGNED16(codes) || !ALIGNED16(dequant))
        return fail(JFA_ERR_INVALID_ARGUMENT, "x, codes and dequant must be 16-byte aligned");
    if (along_rows && (!offsets || batch < 0 || max_len < 0))
        return fail(JFA_ERR_INVALID_ARGUMENT, "along_rows needs offsets, batch and max_len");
    cudaError_t e = quantize_mx(x_bf16, rows, heads, d, offsets, batch, max_len, along_rows, codes,
                                scales, dequant, reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "quantize");
    return JFA_OK;
}
}  // namespace

jfa_status jfa_quantize_mxfp8(const void* x_bf16, int64_t rows, int32_t heads, int32_t d,
                              const int32_t* offsets, int32_t batch, int32_t max_len,
                              int along_rows, uint8_t* codes, uint8_t* scales,
                              jfa_stream_t stream) {
    return quantize_entry(x_bf16, rows, heads, d, offsets, batch, max_len, along_rows, codes, scales,
                          nullptr, stream);
}

jfa_status jfa_quantize_mxfp8_dequant(const void* x_bf16, int64_t rows, int32_t heads, int32_t d,
                                      const int32_t* offsets, int32_t batch, int32_t max_len,
                                      int along_rows, uint8_t* codes, uint8_t* scales,
                                      void* dequant_bf16, jfa_stream_t stream) {
    if (rows > 0 && !dequant_bf16) return fail(JFA_ERR_INVALID_ARGUMENT, "NULL dequant");
    return quantize_entry(x_bf16, rows, heads, d, offsets, batch, max_len, along_rows, codes, scales,
                          dequant_bf16, stream);
}

jfa_status jfa_schedule(const jfa_problem* problem, const int32_t* q_offsets,
                        const int32_t* kv_offsets, int causal, int backward, int tile,
                        int32_t* items, int64_t capacity, int32_t* count, void* workspace,
                        size_t ws_bytes, jfa_stream_t stream) {
    jfa_status s = check_problem(problem);
    if (s != JFA_OK) return s;
    const jfa_problem& p = *problem;
    if (!q_offsets || !kv_offsets || !items || !count || !workspace)
        return fail(JFA_ERR_INVALID_ARGUMENT, "NULL pointer");
    if (tile < kMinTile || tile > 256 || (tile % 16) != 0)
        return fail(JFA_ERR_INVALID_ARGUMENT, "tile must be a multiple of 16 in [16, 256]");
    int64_t need = pairs_bound(p.batch, backward ? p.max_kv_len : p.max_q_len,
                               backward ? p.total_kv : p.total_q, tile) * p.heads;
    if (capacity < need) return fail(JFA_ERR_INVALID_ARGUMENT, "capacity %lld < %lld items", (long long)capacity, (long long)need);
    if (ws_bytes < workspace_bytes(p, backward)) return fail(JFA_ERR_WORKSPACE, "workspace too small");
    char* ws = reinterpret_cast<char*>(workspace);
    WsLayout L = ws_layout(p, backward != 0, false);
    WsHeader* hdr = reinterpret_cast<WsHeader*>(ws);
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e = build_schedule(p, q_offsets, kv_offsets, causal, backward, tile, hdr,
                                   reinterpret_cast<int64_t*>(ws + L.dense_off),
                                   reinterpret_cast<int2*>(ws + (backward ? L.kv_pair_bt : L.pair_bt)),
                                   reinterpret_cast<int64_t*>(ws + (backward ? L.kv_pair_cost : L.pair_cost)),
                                   backward ? L.pairs_max_kv : L.pairs_max_q,
                                   reinterpret_cast<int4*>(items), count,
                                   backward ? &hdr->kv_pair_count : &hdr->pair_count, 1,
                                   backward ? reinterpret_cast<int64_t*>(ws + L.kv_seq_tmp) : nullptr,
                                   backward ? reinterpret_cast<int64_t*>(ws + L.kv_seq_start) : nullptr, st);
    if (e != cudaSuccess) return cuda_fail(e, "schedule");
    return JFA_OK;
}

jfa_status jfa_test_inject(int what) {
    if (what != 0 && what != JFA_TEST_FWD_SKIP_LOAD)
        return fail(JFA_ERR_INVALID_ARGUMENT, "unknown test injection %d", what);
    g_test_hook = what;
    return JFA_OK;
}

jfa_status jfa_profile_enable(int enable) {
    if (enable) {
        g_prof.used = 0;
        g_prof.ids.clear();
    }
    g_prof.on = enable != 0;
    return JFA_OK;
}

int jfa_profile_read(float* ms, int32_t* kernel_ids, int32_t capacity) {
    const int n = (int)g_prof.ids.size();
    if (2 * (size_t)n > g_prof.used) return -1;
    for (int i = 0; i < n && i < capacity; ++i) {
        cudaEvent_t a = g_prof.pool[2 * i], b = g_prof.pool[2 * i + 1];
        if (cudaEventSynchronize(b) != cudaSuccess) return -1;
        float t = 0.f;
        if (cudaEventElapsedTime(&t, a, b) != cudaSuccess) return -1;
        if (ms) ms[i] = t;
        if (kernel_ids) kernel_ids[i] = g_prof.ids[i];
    }
    return n;
}

const char* jfa_kernel_name(int32_t kernel_id) {
    if (kernel_id < 0 || kernel_id >= K_COUNT) return "unknown";
    return kKernelNames[kernel_id];
}

jfa_status jfa_check_error(void* workspace, jfa_stream_t stream) {
    if (!workspace) return fail(JFA_ERR_INVALID_ARGUMENT, "NULL workspace");
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return cuda_fail(e, "synchronize");
    int32_t err = 0;
    e = cudaMemcpy(&err, workspace, sizeof(int32_t), cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return cuda_fail(e, "read error word");
    if (err != 0) {
        int32_t zero = 0;
        cudaMemcpy(workspace, &zero, sizeof(int32_t), cudaMemcpyHostToDevice);
        if (err == JFA_ERR_BAD_OFFSETS) return fail(JFA_ERR_BAD_OFFSETS, "offsets failed validation on the device");
        if (err == JFA_ERR_TIMEOUT) return fail(JFA_ERR_TIMEOUT, "a bounded device wait timed out");
        return fail((jfa_status)err, "device error %d", err);
    }
    return JFA_OK;
}

}  // extern "C"
