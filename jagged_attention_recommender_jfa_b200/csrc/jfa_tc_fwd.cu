// Tensor-core (tcgen05) jagged attention forward for bf16, head_dim 128.
//
// One CTA per work item (sequence, head, 128-row query tile) of the
// longest-first schedule.  Attention runs directly on the packed jagged
// buffers ("Meta GEM Training Efficiency: Why LLM-Scale Recommenders Need a
// Different Stack", section "Bottleneck move 1"): TMA fetches the query tile
// once and streams 128-row key/value tiles of the same sequence through a
// two-stage ring; rows of a tile that lie past the sequence end belong to the
// neighbouring sequence and are masked out of the scores (and zeroed in the
// value tile) before they can contribute.
//
// Warp roles (192 threads):
//   warp 0      TMA producer (one thread)
//   warp 1      TMEM allocator and MMA issuer (one thread)
//   warps 2..5  softmax / activation and epilogue; warp w owns TMEM lanes
//               32*(w%4) .. +31, i.e. one query row per thread
//
// Per key tile j:  S = Q K_j^T  (tcgen05, 128x128x128, fp32 in TMEM)
//                  softmax warps: scale, bias, mask, online softmax in the
//                  log2 domain (or GDPA act(s)/n_kv), P (bf16) -> shared
//                  memory in the 128B-swizzled K-major layout
//                  O += P V_j   (tcgen05, A = P from smem, B = V MN-major)
// The rescale of O by exp2(m_old - m_new) is lazy: it happens only when a
// row's running maximum grows by more than 8 (a factor 256), otherwise the
// old maximum stays the reference; the final O / l is exact either way.
//
// TMEM: S at columns [0, 128), O at [128, 256).
#include <math_constants.h>

#include "jfa_mx.cuh"
#include "jfa_sm100.cuh"

namespace jfa {

using namespace sm100;

JFA_TRACE_DEFINE(fwd)

namespace {

constexpr int BM = 128, BN = 128, HD = 128;
constexpr int NG = 4;                       // column groups: a softmax thread owns 128/NG columns of a row
constexpr int CW = 128 / NG;                // columns per softmax thread
constexpr int kThreads = 64 + NG * 128;     // warp 0 TMA, warp 1 MMA, the rest softmax
constexpr uint32_t kBox = 128 * 128;        // bytes of one [128 rows][64 bf16] box
constexpr uint32_t kTile = 2 * kBox;        // one 128 x 128 bf16 tile (two boxes)
constexpr uint32_t kOffQ = 0;
constexpr uint32_t kOffK = kOffQ + kTile;        // 2 stages
constexpr uint32_t kOffV = kOffK + 2 * kTile;    // 2 stages
constexpr uint32_t kOffBar = kOffV + 2 * kTile;  // 163840
constexpr uint32_t kOffRed = kOffBar + 512;      // row-max exchange [2][NG][128] + l [2][NG][128]
constexpr uint32_t kSmemBytes = kOffRed + 2 * 2 * NG * 128 * 4 + 1024;  // + alignment slack
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleThreshold = 8.0f;        // log2 units

struct Bars {
    uint64_t q_full, q_free;
    uint64_t k_full[2], k_empty[2];
    uint64_t v_full[2], v_empty[2];
    uint64_t s_full[2];
    uint64_t p_full;
    uint64_t pv_done;
    uint64_t o_free[2];
    uint64_t drain;
    uint32_t tmem_base;
    int abort_flag;
};
static_assert(sizeof(Bars) <= 512, "barrier block");

struct FwdParams {
    CUtensorMap tm_q;
    CUtensorMap tm_k;
    CUtensorMap tm_v;
    AttnArgs a;
};

// K-major operand (Q, K, P) at K-step k (16 elements): box k/4, +32 B per step.
__device__ __forceinline__ uint64_t kmajor_desc(uint32_t tile_base, int k) {
    return smem_desc_sw128(tile_base + (uint32_t)(k >> 2) * kBox + (uint32_t)(k & 3) * 32u, 16u,
                           1024u);
}

// MN-major operand (V: keys x d, d contiguous) at K-step k (16 keys):
// 8-key groups 1024 B apart (SBO), the two 64-column halves kBox apart (LBO).
__device__ __forceinline__ uint64_t mnmajor_desc(uint32_t tile_base, int k) {
    return smem_desc_sw128(tile_base + (uint32_t)k * 2048u, kBox, 1024u);
}

__device__ __forceinline__ void named_sync_softmax() {
    asm volatile("bar.sync 1, %0;" ::"n"(NG * 128) : "memory");
}

// The work item a CTA takes at its r-th turn: items are listed longest
// first and dealt out in snake order (0..G-1, G-1..0, ...), which evens out
// the per-CTA totals of a decreasing cost list.
__device__ __forceinline__ int item_of_turn(int r, int c, int G) {
    return r * G + ((r & 1) ? (G - 1 - c) : c);
}

struct Item {
    int b, h, row0, q0, nq, k0, nkv, n_tiles;
};

__device__ __forceinline__ Item load_item(const AttnArgs& a, int idx) {
    const int4 it = a.items[idx];
    Item w;
    w.b = it.x;
    w.h = it.y;
    w.row0 = it.z * BM;
    w.q0 = a.q_off[w.b];
    w.nq = a.q_off[w.b + 1] - w.q0;
    w.k0 = a.kv_off[w.b];
    w.nkv = a.kv_off[w.b + 1] - w.k0;
    const int rows_hi = min(w.row0 + BM, w.nq);
    int kv_end = a.causal ? min(w.nkv, rows_hi + (w.nkv - w.nq)) : w.nkv;
    kv_end = max(kv_end, 0);
    w.n_tiles = (kv_end + BN - 1) / BN;
    return w;
}

// Persistent forward: one CTA per SM walks its share of the longest-first
// work list.  BIAS: 0 none, 1 relative-position (read through L1), 2 dense
// jagged.  SOFTMAX: softmax (true) or GDPA.  QP: MXFP8 attention -- P is
// quantised to E4M3 with one E8M0 scale per 32 keys (counted from the
// sequence's first key) before P.V; l uses the unquantised weights.
//
// Tensor-core order per item: QK_0, QK_1, then for each tile j: [P_j ready]
// P.V_j, QK_{j+2}.  S is double-buffered in TMEM (columns 0 / 128), O too
// (columns 256 / 384, alternating per item) so that an item's epilogue
// overlaps the next item's score MMAs.  Q is reloaded as soon as the item's
// last QK has retired.  Barrier phases follow per-CTA counters (g: key tiles
// so far, nk: items with keys so far, m: items so far).  Each softmax thread
// owns one query row and one 64-column half of it; the two halves exchange
// partial row maxima through shared memory.
template <int BIAS, bool SOFTMAX, bool QP>
__global__ void __launch_bounds__(kThreads, 1) tc_fwd_kernel(const __grid_constant__ FwdParams P) {
    const AttnArgs& a = P.a;
    const int n_items = *a.item_count;
    if (a.hdr->err != 0 || (int)blockIdx.x >= n_items) return;
    extern __shared__ uint8_t smem_dyn[];
    uint8_t* smem = smem_dyn + ((1024u - (smem_u32(smem_dyn) & 1023u)) & 1023u);
    Bars* bars = reinterpret_cast<Bars*>(smem + kOffBar);
    float* red = reinterpret_cast<float*>(smem + kOffRed);   // [2 parity][NG groups][128 rows]
    float* lred = red + 2 * NG * 128;                          // [2 item parity][NG groups][128 rows]
    const int G = gridDim.x, cta = blockIdx.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    constexpr bool softmax = SOFTMAX;

    if (threadIdx.x == 0) {
        mbar_init(&bars->q_full, 1);
        mbar_init(&bars->q_free, 1);
        for (int s = 0; s < 2; ++s) {
            mbar_init(&bars->k_full[s], 1);
            mbar_init(&bars->k_empty[s], 1);
            mbar_init(&bars->v_full[s], 1);
            mbar_init(&bars->v_empty[s], 1);
            mbar_init(&bars->s_full[s], 1);
            mbar_init(&bars->o_free[s], NG * 4);
        }
        mbar_init(&bars->p_full, NG * 4);
        mbar_init(&bars->pv_done, 1);
        mbar_init(&bars->drain, 1);
        bars->abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(&bars->tmem_base, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bars->tmem_base;
    volatile int* abort_flag = &bars->abort_flag;
    const uint32_t sbase = smem_u32(smem);

    if (warp == 0) {
        // ------------------------------------------------------------ TMA
        if (lane == 0) {
            tma_prefetch_desc(&P.tm_q);
            tma_prefetch_desc(&P.tm_k);
            tma_prefetch_desc(&P.tm_v);
            int g = 0, nk = 0;        // key tiles issued, items with keys
            int kq = 0, kv_i = 0;     // loads issued (for the drain)
            bool ok = true;
            for (int r = 0; ok; ++r) {
                const int idx = item_of_turn(r, cta, G);
                if (idx >= n_items) break;
                const Item w = load_item(a, idx);
                if (w.n_tiles == 0) continue;
                if (nk > 0 && !mbar_wait(&bars->q_free, (nk - 1) & 1, abort_flag, a.hdr)) { ok = false; break; }
                mbar_arrive_expect_tx(&bars->q_full, kTile);
                tma_load_3d(smem + kOffQ, &P.tm_q, &bars->q_full, 0, w.h, w.q0 + w.row0);
                tma_load_3d(smem + kOffQ + kBox, &P.tm_q, &bars->q_full, 64, w.h, w.q0 + w.row0);
                ++nk;
                for (int j = 0; j < w.n_tiles; ++j, ++g) {
                    const int s = g & 1;
                    const uint32_t par = ((g >> 1) - 1) & 1;
                    const int z = w.k0 + j * BN;
                    if (g >= 2 && !mbar_wait(&bars->k_empty[s], par, abort_flag, a.hdr)) { ok = false; break; }
                    JFA_TRACE_EV(fwd, 0, g, 0);
                    mbar_arrive_expect_tx(&bars->k_full[s], kTile);
                    tma_load_3d(smem + kOffK + s * kTile, &P.tm_k, &bars->k_full[s], 0, w.h, z);
                    tma_load_3d(smem + kOffK + s * kTile + kBox, &P.tm_k, &bars->k_full[s], 64, w.h, z);
                    ++kq;
                    if (g >= 2 && !mbar_wait(&bars->v_empty[s], par, abort_flag, a.hdr)) { ok = false; break; }
                    JFA_TRACE_EV(fwd, 0, g, 1);
                    mbar_arrive_expect_tx(&bars->v_full[s], kTile);
                    tma_load_3d(smem + kOffV + s * kTile, &P.tm_v, &bars->v_full[s], 0, w.h, z);
                    tma_load_3d(smem + kOffV + s * kTile + kBox, &P.tm_v, &bars->v_full[s], 64, w.h, z);
                    ++kv_i;
                    if (j + 2 < w.n_tiles) {  // warm L2 for the tiles loaded after the next release
                        tma_prefetch_l2_3d(&P.tm_k, 0, w.h, z + 2 * BN);
                        tma_prefetch_l2_3d(&P.tm_k, 64, w.h, z + 2 * BN);
                        tma_prefetch_l2_3d(&P.tm_v, 0, w.h, z + 2 * BN);
                        tma_prefetch_l2_3d(&P.tm_v, 64, w.h, z + 2 * BN);
                    }
                }
            }
            // never leave the CTA with copies in flight: wait for the last loads
            if (nk > 0) mbar_wait_drain(&bars->q_full, (nk - 1) & 1, a.hdr);
            for (int t = (kq > 2 ? kq - 2 : 0); t < kq; ++t) mbar_wait_drain(&bars->k_full[t & 1], (t >> 1) & 1, a.hdr);
            for (int t = (kv_i > 2 ? kv_i - 2 : 0); t < kv_i; ++t) mbar_wait_drain(&bars->v_full[t & 1], (t >> 1) & 1, a.hdr);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA
        if (lane == 0) {
            constexpr uint32_t idesc_qk = idesc_bf16(BM, BN, 0, 0);
            constexpr uint32_t idesc_pv = idesc_bf16(BM, HD, 0, 1);
            const uint32_t qb = sbase + kOffQ;
            int g = 0, nk = 0, m = 0;
            bool ok = true;
            auto issue_qk = [&](int gg, int n_left_after) -> bool {
                const int s = gg & 1;
                if (!mbar_wait(&bars->k_full[s], (gg >> 1) & 1, abort_flag, a.hdr)) return false;
                JFA_TRACE_EV(fwd, 1, gg, 0);
                tc_fence_after();
                const uint32_t kb = sbase + kOffK + s * kTile;
#pragma unroll
                for (int k = 0; k < HD / 16; ++k)
                    mma_bf16_ss(tmem + s * 128, kmajor_desc(qb, k), kmajor_desc(kb, k), idesc_qk, k > 0 ? 1u : 0u);
                mma_commit(&bars->s_full[s]);
                JFA_TRACE_EV(fwd, 1, gg, 1);
                mma_commit(&bars->k_empty[s]);
                if (n_left_after == 0) mma_commit(&bars->q_free);  // last score MMA of the item
                return true;
            };
            for (int r = 0; ok; ++r, ++m) {
                const int idx = item_of_turn(r, cta, G);
                if (idx >= n_items) break;
                const Item w = load_item(a, idx);
                if (w.n_tiles == 0) continue;
                const int ob = m & 1;
                const uint32_t tO = tmem + 256 + ob * 128;
                if (!mbar_wait(&bars->q_full, nk & 1, abort_flag, a.hdr)) { ok = false; break; }
                ++nk;
                // the epilogue of the item two turns back must be done with this O buffer
                if (m >= 2 && !mbar_wait(&bars->o_free[ob], ((m >> 1) - 1) & 1, abort_flag, a.hdr)) { ok = false; break; }
                const int n = w.n_tiles, g0 = g;
                for (int t = 0; t < 2 && t < n && ok; ++t) ok = issue_qk(g0 + t, n - 1 - t);
                for (int t = 0; ok && t < n; ++t, ++g) {
                    const int s = g & 1;
                    if (!mbar_wait(&bars->p_full, g & 1, abort_flag, a.hdr)) { ok = false; break; }
                    JFA_TRACE_EV(fwd, 1, g, 2);
                    if (!mbar_wait(&bars->v_full[s], (g >> 1) & 1, abort_flag, a.hdr)) { ok = false; break; }
                    JFA_TRACE_EV(fwd, 1, g, 3);
                    tc_fence_after();
                    const uint32_t vb = sbase + kOffV + s * kTile;
                    const uint32_t tP = tmem + s * 128;  // P (bf16 pairs) over columns 0..63 of its S
#pragma unroll
                    for (int k = 0; k < BN / 16; ++k)
                        mma_bf16_ts(tO, tP + k * 8, mnmajor_desc(vb, k), idesc_pv,
                                    (t > 0 || k > 0) ? 1u : 0u);
                    mma_commit(&bars->v_empty[s]);
                    mma_commit(&bars->pv_done);
                    JFA_TRACE_EV(fwd, 1, g, 4);
                    if (t + 2 < n) ok = issue_qk(g + 2, n - 1 - (t + 2));
                }
            }
            // all issued MMAs retire before TMEM is released
            mma_commit(&bars->drain);
            mbar_wait_drain(&bars->drain, 0, a.hdr);
        }
    } else {
        // ------------------------------------------------ softmax warps
        const int wq = warp & 3;                 // TMEM lane quarter
        const int grp = (warp - 2) >> 2;         // column group of S / O
        const int r_ = wq * 32 + lane;           // row within the tile
        const int c0 = grp * CW;                 // first column of this thread's group
        const uint32_t lane_addr = (uint32_t)(wq * 32) << 16;
        const float sc = a.scale * kLog2e;
        const int C = (a.relpos_len - 1) >> 1;
        int g = 0, m = 0;
        bool ok = true;
        const int tslot = (warp == 2 && lane == 0) ? 2 : ((warp == kThreads / 32 - 1 && lane == 0) ? 3 : -1);
#define SM_EV(ev)                                     \
    do {                                              \
        if (tslot >= 0) JFA_TRACE_EV(fwd, tslot, g, ev); \
    } while (0)
        // Every softmax warp runs the same sequence of named barriers: a failed
        // (timed-out) wait only sets the CTA's abort flag, and the loops are left
        // right after a barrier, where all warps read the same flag.
        for (int rr = 0; ok; ++rr, ++m) {
            const int idx = item_of_turn(rr, cta, G);
            if (idx >= n_items) break;
            const Item w = load_item(a, idx);
            const int i = w.row0 + r_;             // query index within the sequence
            const int shift = w.nkv - w.nq;        // causal: key j visible iff j <= i + shift
            const float inv_n = w.nkv > 0 ? 1.0f / (float)w.nkv : 0.f;
            const int jmax_vis = a.causal ? min(w.nkv - 1, i + shift) : w.nkv - 1;
            const float* tab4 = (BIAS == 1) ? a.bias4 + (int64_t)w.h * 4 * a.bias4_stride : nullptr;
            const __nv_bfloat16* dense = reinterpret_cast<const __nv_bfloat16*>(a.bias);
            const int64_t dense_row = (BIAS == 2 && i < w.nq)
                                          ? a.dense_off[w.b] + ((int64_t)w.h * w.nq + i) * w.nkv : 0;
            const uint32_t tO = tmem + lane_addr + 256 + (m & 1) * 128 + c0;
            float m_used = -CUDART_INF_F, l = 0.f;   // l: this group's partial sum
            for (int j = 0; j < w.n_tiles; ++j, ++g) {
                const int s = g & 1;
                SM_EV(0);
                mbar_wait(&bars->s_full[s], (g >> 1) & 1, abort_flag, a.hdr);
                SM_EV(1);
                tc_fence_after();
                const int jc = j * BN + c0;          // key index of this group's column 0
                float x[CW];
                {
                    uint32_t u[32];
                    tmem_ld32(tmem + lane_addr + s * 128 + c0, u);
                    tmem_wait_ld();
#pragma unroll
                    for (int t = 0; t < CW; ++t) x[t] = __uint_as_float(u[t]);
                }
                const int nvis = i < w.nq ? max(0, min(CW, jmax_vis - jc + 1)) : 0;  // visible: [0, nvis)
                if (BIAS == 1) {
                    // bias(i, jc + c) = table[i - jc - c + C] (log2(e)-scaled copy);
                    // within a sequence |i - j| <= C, so only tiles past the rows
                    // need the clamp
                    const int hi = i - jc + C;
                    const float2 sc2 = make_float2(sc, sc);
                    float bb[CW];
                    if (hi - (CW - 1) >= 0 && hi <= 2 * C) {
                        const float* tb = tab4 + hi;   // tb[-c]
#pragma unroll
                        for (int c = 0; c < CW; ++c) bb[c] = __ldg(tb - c);
                    } else {
#pragma unroll
                        for (int c = 0; c < CW; ++c) bb[c] = __ldg(tab4 + min(max(hi - c, 0), 2 * C));
                    }
#pragma unroll
                    for (int c = 0; c < CW; c += 2) {
                        const float2 r2 = fma2(make_float2(x[c], x[c + 1]), sc2, make_float2(bb[c], bb[c + 1]));
                        x[c] = r2.x, x[c + 1] = r2.y;
                    }
                } else if (BIAS == 2) {
#pragma unroll
                    for (int c = 0; c < CW; ++c)
                        x[c] = fmaf(x[c], sc, c < nvis ? __bfloat162float(dense[dense_row + jc + c]) * kLog2e : 0.f);
                } else {
#pragma unroll
                    for (int c = 0; c < CW; c += 2) {
                        const float2 r2 = mul2(make_float2(x[c], x[c + 1]), make_float2(sc, sc));
                        x[c] = r2.x, x[c + 1] = r2.y;
                    }
                }
                const bool masked_tile = __any_sync(0xffffffffu, nvis < CW);
                if (masked_tile) {
#pragma unroll
                    for (int c = 0; c < CW; ++c) x[c] = c < nvis ? x[c] : -CUDART_INF_F;
                }
                float alpha = 1.f;
                bool rescale = false;
                if (softmax) {
                    float pm4[4];
#pragma unroll
                    for (int t = 0; t < 4; ++t) pm4[t] = fmaxf(x[2 * t], x[2 * t + 1]);
#pragma unroll
                    for (int c = 8; c < CW; c += 2) pm4[(c >> 1) & 3] = max3(pm4[(c >> 1) & 3], x[c], x[c + 1]);
                    const float pm = max3(pm4[0], pm4[1], fmaxf(pm4[2], pm4[3]));
                    red[(s * NG + grp) * 128 + r_] = pm;
                    SM_EV(2);
                    named_sync_softmax();
                    SM_EV(3);
                    if (*abort_flag) { ok = false; break; }
                    float tmax = pm;
#pragma unroll
                    for (int q = 0; q < NG; ++q) tmax = fmaxf(tmax, red[(s * NG + q) * 128 + r_]);
                    // lazy rescale: keep the reference unless the row maximum grew by
                    // more than 8 (a factor 2^8).  With MXFP8 P the reference is an
                    // integer (ceil of the maximum, log2 units), so rescales are exact
                    // powers of two and the block quantisation of P does not depend on
                    // it; otherwise the maximum itself, so the largest weight is 1.
                    const bool need = tmax > m_used + kRescaleThreshold;
                    const float m_new = need ? (QP ? ceilf(tmax) : tmax) : m_used;
                    if (need && m_used != -CUDART_INF_F) {
                        alpha = ex2(m_used - m_new);
                        rescale = true;
                    } else if (need) {
                        l = 0.f;  // first visible key of this row
                    }
                    m_used = m_new;
                }
                // a rescale of O needs every earlier P.V of this item retired
                if (softmax && __any_sync(0xffffffffu, rescale)) {
                    if (g > 0) {
                        mbar_wait(&bars->pv_done, (g - 1) & 1, abort_flag, a.hdr);
                        tc_fence_after();
                    }
                    uint32_t u[32];
                    tmem_ld32(tO, u);
                    tmem_wait_ld();
#pragma unroll
                    for (int t = 0; t < 32; ++t) u[t] = __float_as_uint(__uint_as_float(u[t]) * alpha);
                    tmem_st32(tO, u);
                    tmem_wait_st();
                    l *= alpha;
                }
                SM_EV(4);
                if (softmax) {
                    // ex2(-inf) = 0 masks the invisible columns; a row with no visible
                    // key yet uses reference 0 so that -inf - ref stays -inf
                    const float ref = m_used == -CUDART_INF_F ? 0.f : m_used;
                    const float2 ref2 = make_float2(ref, ref);
                    float2 ps[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                                    make_float2(0.f, 0.f)};
#pragma unroll
                    for (int c = 0; c < CW; c += 2) {
                        const float2 y = sub2(make_float2(x[c], x[c + 1]), ref2);
                        x[c] = ex2(y.x);
                        x[c + 1] = ex2(y.y);
                        ps[(c >> 1) & 3] = add2(ps[(c >> 1) & 3], make_float2(x[c], x[c + 1]));
                    }
                    const float2 s01 = add2(ps[0], ps[1]), s23 = add2(ps[2], ps[3]);
                    const float2 s4 = add2(s01, s23);
                    l += s4.x + s4.y;
                    if (QP) mx::fake_quant32(x);  // the group's 32 keys are one MX block
                } else {
#pragma unroll
                    for (int c = 0; c < CW; ++c) {
                        const float s_nat = x[c] * (1.0f / kLog2e);
                        x[c] = c < nvis ? act_f(a.act, s_nat) * inv_n : 0.f;
                    }
                    // P overwrites S columns other groups may still be loading
                    named_sync_softmax();
                }
                // P row part (bf16 pairs) -> TMEM over the first 64 columns of its own
                // S buffer: column c0/2 + t holds keys c0 + 2t (low half) and c0 + 2t + 1.
                // Every group has loaded its S columns (they did so before the barrier
                // above), and the next write to this buffer is QK_{j+2}, issued after
                // P.V_j, which reads it.
                {
                    uint32_t pw[16];
#pragma unroll
                    for (int t = 0; t < 16; ++t) pw[t] = pack_bf16(x[2 * t], x[2 * t + 1]);
                    tmem_st16(tmem + lane_addr + s * 128 + (c0 >> 1), pw);
                    tmem_wait_st();
                }
                // value rows past the sequence end (neighbour data) must not reach P.V
                const int nvalid = w.nkv - j * BN;
                if (nvalid < BN) {  // same for the whole CTA
                    mbar_wait(&bars->v_full[s], (g >> 1) & 1, abort_flag, a.hdr);
                    if (r_ >= nvalid && (grp & 1) == 0) {  // groups 0 and 2 clear the two boxes
                        uint8_t* vrow = smem + kOffV + s * kTile + (grp >> 1) * kBox + r_ * 128;
                        const uint4 z = make_uint4(0, 0, 0, 0);
#pragma unroll
                        for (int ch = 0; ch < 8; ++ch) *reinterpret_cast<uint4*>(vrow + ch * 16) = z;
                    }
                }
                fence_proxy_async_smem();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars->p_full);
                SM_EV(5);
            }
            if (!ok) break;
            // ---------------------------------------------------- epilogue
            if (w.n_tiles > 0) mbar_wait(&bars->pv_done, (g - 1) & 1, abort_flag, a.hdr);
            SM_EV(6);
            lred[((m & 1) * NG + grp) * 128 + r_] = l;
            named_sync_softmax();
            SM_EV(7);
            if (*abort_flag) { ok = false; break; }
            float l_row = 0.f;
#pragma unroll
            for (int q = 0; q < NG; ++q) l_row += lred[((m & 1) * NG + q) * 128 + r_];
            tc_fence_after();
            const float inv = softmax ? (l_row > 0.f ? 1.f / l_row : 0.f) : 1.f;
            __nv_bfloat16* orow = reinterpret_cast<__nv_bfloat16*>(a.out) + ((int64_t)(w.q0 + i) * a.H + w.h) * HD + c0;
            uint32_t u[32];
            if (w.n_tiles > 0) {
                tmem_ld32(tO, u);
                tmem_wait_ld();
            } else {
#pragma unroll
                for (int t = 0; t < 32; ++t) u[t] = 0u;
            }
            // O buffer free for the item two turns ahead
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->o_free[m & 1]);
            if (i < w.nq) {
#pragma unroll
                for (int t = 0; t < 32; t += 8) {
                    uint4 wv;
                    wv.x = pack_bf16(__uint_as_float(u[t + 0]) * inv, __uint_as_float(u[t + 1]) * inv);
                    wv.y = pack_bf16(__uint_as_float(u[t + 2]) * inv, __uint_as_float(u[t + 3]) * inv);
                    wv.z = pack_bf16(__uint_as_float(u[t + 4]) * inv, __uint_as_float(u[t + 5]) * inv);
                    wv.w = pack_bf16(__uint_as_float(u[t + 6]) * inv, __uint_as_float(u[t + 7]) * inv);
                    *reinterpret_cast<uint4*>(orow + t) = wv;
                }
                if (softmax && grp == 0 && a.lse)
                    a.lse[(int64_t)(w.q0 + i) * a.H + w.h] =
                        l_row > 0.f ? m_used * (1.0f / kLog2e) + logf(l_row) : -CUDART_INF_F;
            }
        }
#undef SM_EV
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

}  // namespace

// [rows][heads][128] bf16 viewed as a 3-D tensor (d, head, row); boxes of
// 64 d x 1 head x 128 rows with the 128-byte swizzle.
bool make_tmap_rows_heads_d(CUtensorMap* map, const void* base, int64_t rows, int heads) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {(cuuint64_t)HD, (cuuint64_t)heads, (cuuint64_t)(rows > 0 ? rows : 1)};
    cuuint64_t strides[2] = {(cuuint64_t)HD * 2, (cuuint64_t)heads * HD * 2};
    cuuint32_t box[3] = {64, 1, 128};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides,
                    box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

constexpr int kSmemLimit = 232448;  // 227 KB opt-in per CTA

cudaError_t tc_forward_launch(const jfa_problem& p, const AttnArgs& a, bool quant_p, cudaStream_t st) {
    FwdParams P{};
    if (!make_tmap_rows_heads_d(&P.tm_q, a.q, p.total_q, p.heads) ||
        !make_tmap_rows_heads_d(&P.tm_k, a.k, p.total_kv, p.heads) ||
        !make_tmap_rows_heads_d(&P.tm_v, a.v, p.total_kv, p.heads))
        return cudaErrorInvalidValue;
    P.a = a;
    const int smem = (int)kSmemBytes;
    const int64_t items_bound = pairs_bound(p.batch, p.max_q_len, p.total_q, BM) * p.heads;
    if (items_bound <= 0) return cudaSuccess;
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int grid = (int)(items_bound < sms ? items_bound : sms);
    const int bias = p.bias_kind == JFA_BIAS_RELPOS ? 1 : (p.bias_kind == JFA_BIAS_DENSE_JAGGED ? 2 : 0);
    const bool sm = a.act == JFA_ACT_SOFTMAX;
    void (*kern)(FwdParams) = nullptr;
    if (quant_p) {
        if (!sm) return cudaErrorInvalidValue;
        kern = bias == 0 ? tc_fwd_kernel<0, true, true>
                         : (bias == 1 ? tc_fwd_kernel<1, true, true> : tc_fwd_kernel<2, true, true>);
    } else if (bias == 0) {
        kern = sm ? tc_fwd_kernel<0, true, false> : tc_fwd_kernel<0, false, false>;
    } else if (bias == 1) {
        kern = sm ? tc_fwd_kernel<1, true, false> : tc_fwd_kernel<1, false, false>;
    } else {
        kern = sm ? tc_fwd_kernel<2, true, false> : tc_fwd_kernel<2, false, false>;
    }
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemLimit);
    if (e != cudaSuccess) return e;
    prof_begin(st);
    kern<<<grid, kThreads, smem, st>>>(P);
    prof_end(st, quant_p ? K_TC_FWD_MXFP8 : K_TC_FWD);
    return cudaGetLastError();
}

}  // namespace jfa
