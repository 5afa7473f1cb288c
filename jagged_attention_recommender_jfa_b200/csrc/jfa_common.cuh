// Shared device-side definitions of libjfa: workspace layout, kernel argument
// block, element conversions and the on-device error word.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "jfa.h"

namespace jfa {

// ---------------------------------------------------------------------------
// Workspace layout.  Everything the passes need between kernels lives in the
// caller's workspace; offsets are 256-byte aligned.
//
//   [header 256 B]  err, item_count, pair_count, queue counters
//   dense_off       int64 [B + 1]    start of sequence b's dense bias block
//   pair_bt         int32 [P_max][2] (sequence, tile) of each schedule pair
//   pair_cost       int64 [P_max]    pairs computed by that tile
//   items           int4  [P_max*H]  {b, h, tile, cost} in execution order
//   (backward)      kv_items, D = rowsum(dO*O) fp32 [total_q*H],
//                   dQ accumulator fp32 [total_q*H*d] (tensor-core path)
// P_max covers the smallest schedule tile (16 rows), so one workspace serves
// every tile height.
// ---------------------------------------------------------------------------
struct WsHeader {
    int32_t err;
    int32_t item_count;
    int32_t pair_count;
    int32_t queue;
    int32_t kv_item_count;
    int32_t kv_pair_count;
    int32_t kv_queue;        // next work item of the persistent key-tile backward
    int32_t wait_limit_us;   // bounded device waits give up after this (0: 1 s)
    int32_t pad[56];
};
static_assert(sizeof(WsHeader) == 256, "header is 256 bytes");

constexpr int kMinTile = 16;

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

struct WsLayout {
    size_t dense_off, pair_bt, pair_cost, items;           // forward schedule
    size_t kv_pair_bt, kv_pair_cost, kv_items;             // backward schedule
    size_t kv_seq_tmp, kv_seq_start;                       // its sequence order
    size_t dterm, dq_acc;                                  // backward rows
    size_t total;
    int64_t pairs_max_q, pairs_max_kv;
};

// Upper bound of sum_b ceil(n(b) / tile) given only host-side sizes.
inline int64_t pairs_bound(int64_t batch, int64_t max_len, int64_t total, int tile) {
    int64_t a = batch * ((max_len + tile - 1) / tile);
    int64_t b = total / tile + batch;
    return a < b ? a : b;
}

inline WsLayout ws_layout(const jfa_problem& p, bool backward, bool need_dq_acc) {
    WsLayout L{};
    size_t off = sizeof(WsHeader);
    L.pairs_max_q = pairs_bound(p.batch, p.max_q_len, p.total_q, kMinTile);
    L.pairs_max_kv = pairs_bound(p.batch, p.max_kv_len, p.total_kv, kMinTile);
    L.dense_off = off;  off = align256(off + sizeof(int64_t) * (size_t)(p.batch + 1));
    L.pair_bt = off;    off = align256(off + sizeof(int32_t) * 2 * (size_t)L.pairs_max_q);
    L.pair_cost = off;  off = align256(off + sizeof(int64_t) * (size_t)L.pairs_max_q);
    L.items = off;      off = align256(off + sizeof(int4) * (size_t)L.pairs_max_q * p.heads);
    if (backward) {
        L.kv_pair_bt = off;   off = align256(off + sizeof(int32_t) * 2 * (size_t)L.pairs_max_kv);
        L.kv_pair_cost = off; off = align256(off + sizeof(int64_t) * (size_t)L.pairs_max_kv);
        L.kv_items = off;     off = align256(off + sizeof(int4) * (size_t)L.pairs_max_kv * p.heads);
        L.kv_seq_tmp = off;   off = align256(off + sizeof(int64_t) * (size_t)p.batch);
        L.kv_seq_start = off; off = align256(off + sizeof(int64_t) * (size_t)p.batch);
        L.dterm = off;        off = align256(off + sizeof(float) * (size_t)p.total_q * p.heads);
        if (need_dq_acc) {
            L.dq_acc = off;
            off = align256(off + sizeof(float) * (size_t)p.total_q * p.heads * p.head_dim);
        }
    }
    L.total = off;
    return L;
}

// ---------------------------------------------------------------------------
// Kernel arguments (one block for every attention kernel).
// ---------------------------------------------------------------------------
struct AttnArgs {
    const void* q;
    const void* k;
    const void* v;
    const int32_t* q_off;
    const int32_t* kv_off;
    const void* bias;
    const int64_t* dense_off;  // int64 [B+1] (dense bias only)
    int bias_kind;
    int relpos_len;
    int B, H;
    int causal;
    int window;   // sliding-window width w (0: none), see vis_key_lo / vis_key_hi
    int act;
    float scale;
    void* out;
    float* lse;
    const int4* items;
    const int32_t* item_count;
    WsHeader* hdr;
    // backward
    const void* dout;
    const float* o_for_d;  // unused placeholder (O is read through `out`)
    float* dterm;          // D = rowsum(dO * O), fp32 [total_q*H]
    void* dq;
    void* dk;
    void* dv;
    float* dq_acc;
    // bias gradient (NULL: not requested).  RELPOS: fp32 [H][relpos_len],
    // zeroed before the backward kernels, which add into it; DENSE_JAGGED:
    // element type, the bias layout, one ds per visited pair
    void* dbias;
    // tensor-core path, relative-position bias: each head's table scaled by
    // log2(e) as runs of four (float4 entry t = entries t .. t+3), so that any
    // run of table entries can be read with 16-byte-aligned vector loads;
    // entry t of head h is bias4[4 * (h * bias4_stride + t) + 0..3]
    const float* bias4;
    int bias4_stride;  // float4 entries per head (at least 384)
    // test hook (jfa_test_inject): CTA 0 of the tensor-core forward skips its
    // first key-tile load, so that the bounded waits run out
    int test_skip_load;
};

// ---------------------------------------------------------------------------
// Element conversions.
// ---------------------------------------------------------------------------
__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T>
__device__ __forceinline__ T from_f(float x);
template <>
__device__ __forceinline__ float from_f<float>(float x) { return x; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }

// Load 4 consecutive elements as float4 (16-byte aligned for float, 8-byte
// for bf16).
__device__ __forceinline__ float4 load4(const float* p) { return *reinterpret_cast<const float4*>(p); }
__device__ __forceinline__ float4 load4(const __nv_bfloat16* p) {
    uint2 u = *reinterpret_cast<const uint2*>(p);
    __nv_bfloat162 a = *reinterpret_cast<__nv_bfloat162*>(&u.x);
    __nv_bfloat162 b = *reinterpret_cast<__nv_bfloat162*>(&u.y);
    float2 fa = __bfloat1622float2(a), fb = __bfloat1622float2(b);
    return make_float4(fa.x, fa.y, fb.x, fb.y);
}
__device__ __forceinline__ void store4(float* p, float4 v) { *reinterpret_cast<float4*>(p) = v; }
__device__ __forceinline__ void store4(__nv_bfloat16* p, float4 v) {
    __nv_bfloat162 a = __floats2bfloat162_rn(v.x, v.y);
    __nv_bfloat162 b = __floats2bfloat162_rn(v.z, v.w);
    uint2 u;
    u.x = *reinterpret_cast<uint32_t*>(&a);
    u.y = *reinterpret_cast<uint32_t*>(&b);
    *reinterpret_cast<uint2*>(p) = u;
}

// ---------------------------------------------------------------------------
// Launch timing (jfa_profile_*): prof_begin / prof_end bracket every launch.
// ---------------------------------------------------------------------------
enum KernelId {
    K_SCHED_PREPARE = 0,
    K_SCHED_RANK,
    K_SIMT_FWD,
    K_SIMT_BWD_PRE,
    K_SIMT_BWD_DQ,
    K_SIMT_BWD_DKDV,
    K_QUANT_ALONG_D,
    K_QUANT_ALONG_ROWS,
    K_TC_FWD,
    K_TC_BWD_PRE,
    K_TC_BWD,
    K_TC_DQ_FINALIZE,
    K_TC_FWD_MXFP8,
    K_TC_BIAS_PREP,
    K_DBIAS_ZERO,
    K_NORM_QUANT,
    K_TC_BWD_SQ,
    K_TC_FWD_SQ,
    K_COUNT
};
void prof_begin(cudaStream_t st);
void prof_end(cudaStream_t st, int kernel_id);

// Records the thread-local message jfa_last_error() returns and passes the
// status through.
jfa_status set_last_error(jfa_status s, const char* fmt, ...);

__device__ __forceinline__ void set_error(WsHeader* hdr, int code) {
    atomicCAS(&hdr->err, 0, code);
}

// Activations of the GDPA variant.
//   SiLU(x) = x * sigmoid(x)
//   GELU_tanh(x) = 0.5 x (1 + tanh(sqrt(2/pi) (x + 0.044715 x^3)))
// Both are x * sigmoid(k(x)): k = x for SiLU and, since 0.5 (1 + tanh z) =
// sigmoid(2 z), k = 2 sqrt(2/pi) (x + 0.044715 x^3) for tanh-GELU.  The
// sigmoid is 1 / (1 + 2^(-k log2 e)) from the hardware base-2 exponential and
// a fast reciprocal (a few ulp; a large negative k gives 0, a large positive 1).
__device__ __forceinline__ float sigmoid_fast(float k) {
    float e;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(e) : "f"(-k * 1.4426950408889634f));
    return __fdividef(1.0f, 1.0f + e);
}

__device__ __forceinline__ float act_arg(int act, float x) {
    return act == JFA_ACT_SILU ? x : 1.5957691216057308f * fmaf(0.044715f * x, x * x, x);
}

__device__ __forceinline__ float act_f(int act, float x) { return x * sigmoid_fast(act_arg(act, x)); }

// The forward's GDPA weight act(s) * c from x = s log2(e) (scores kept in
// log2 units), with one hardware tanh (relative error ~2^-11) instead of an
// exponential and a reciprocal:
//   SiLU(s)      = s/2 (1 + tanh(s / 2))
//   GELU_tanh(s) = s/2 (1 + tanh(sqrt(2/pi) (s + 0.044715 s^3)))
// half_c = c / (2 log2(e)), so that x * half_c = c s / 2.  x = -inf gives NaN:
// callers select 0 for masked keys.
__device__ __forceinline__ float tanh_hw(float z) {
    float t;
    asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(z));
    return t;
}
template <int ACT>
__device__ __forceinline__ float gdpa_weight_log2(float x, float half_c) {
    const float y = x * half_c;
    float z;
    if (ACT == JFA_ACT_SILU) {
        z = x * (0.5f / 1.4426950408889634f);
    } else {
        const float s = x * (1.0f / 1.4426950408889634f);
        z = 0.7978845608028654f * fmaf(0.044715f * s, s * s, s);
    }
    return fmaf(y, tanh_hw(z), y);
}

// Derivatives, from s = sigmoid(k(x)):
//   SiLU'(x)      = s (1 + x (1 - s))
//   GELU_tanh'(x) = 0.5 (1 + t) + 0.5 x (1 - t^2) sqrt(2/pi) (1 + 3 * 0.044715 x^2)
//                 = s + 2 x s (1 - s) sqrt(2/pi) (1 + 3 * 0.044715 x^2)
//   (t = tanh z = 2 s - 1, so 1 + t = 2 s and 1 - t^2 = 4 s (1 - s))
__device__ __forceinline__ float act_grad_from(int act, float x, float s) {
    if (act == JFA_ACT_SILU) return s * fmaf(x, 1.0f - s, 1.0f);
    return fmaf(2.0f * x * s * (1.0f - s), 0.7978845608028654f * fmaf(3.0f * 0.044715f, x * x, 1.0f), s);
}

// Additive bias beta_h(i, j) of sequence b (i, j relative to the sequence).
template <typename T>
__device__ __forceinline__ float bias_at(const AttnArgs& a, int b, int h, int nq, int nkv, int i, int j) {
    if (a.bias_kind == JFA_BIAS_RELPOS) {
        const int C = (a.relpos_len - 1) >> 1;
        int r = i - j;
        r = r < -C ? -C : (r > C ? C : r);
        return __ldg(reinterpret_cast<const float*>(a.bias) + (int64_t)h * a.relpos_len + (r + C));
    }
    if (a.bias_kind == JFA_BIAS_DENSE_JAGGED) {
        const T* base = reinterpret_cast<const T*>(a.bias);
        return to_f(base[a.dense_off[b] + ((int64_t)h * nq + i) * nkv + j]);
    }
    return 0.0f;
}

// Validity with bottom-right alignment: query i sits at key position
// p = i + (n_kv - n_q).  Causal: key j is visible iff j <= p.  Sliding window
// w > 0 (windowed attention, "Meta Enhances GEM Training Efficiency with
// Advanced LLM-Scale Innovations", "Exploring the Customized Kernel Library"
// -> "BlockAttention": windows instead of full attention over long user
// histories): additionally p - j < w, and without the causal rule also
// j - p < w.  The visible keys of a query row and the queries that see a key
// are contiguous ranges, returned clamped to the sequence (empty: lo > hi).
__device__ __forceinline__ int vis_key_lo(int window, int i, int nq, int nkv) {
    if (window <= 0) return 0;
    const int64_t lo = (int64_t)i + (nkv - nq) - window + 1;
    return lo < 0 ? 0 : (int)lo;
}
__device__ __forceinline__ int vis_key_hi(int causal, int window, int i, int nq, int nkv) {
    const int64_t p = (int64_t)i + (nkv - nq);
    const int64_t hi = causal ? p : (window > 0 ? p + window - 1 : (int64_t)nkv - 1);
    return (int)(hi < (int64_t)nkv - 1 ? (hi < -1 ? -1 : hi) : (int64_t)nkv - 1);
}
__device__ __forceinline__ int vis_query_lo(int causal, int window, int j, int nq, int nkv) {
    const int64_t shift = (int64_t)nkv - nq;
    const int64_t lo = causal ? j - shift : (window > 0 ? j - window + 1 - shift : 0);
    return lo < 0 ? 0 : (lo > nq ? nq : (int)lo);
}
__device__ __forceinline__ int vis_query_hi(int window, int j, int nq, int nkv) {
    if (window <= 0) return nq - 1;
    const int64_t hi = (int64_t)j + window - 1 - ((int64_t)nkv - nq);
    return (int)(hi < (int64_t)nq - 1 ? (hi < -1 ? -1 : hi) : (int64_t)nq - 1);
}
__device__ __forceinline__ bool key_visible(int causal, int window, int i, int j, int nq, int nkv) {
    return j >= vis_key_lo(window, i, nq, nkv) && j <= vis_key_hi(causal, window, i, nq, nkv);
}

}  // namespace jfa
