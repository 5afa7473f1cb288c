// Tensor-core jagged attention forward for short query sequences (every
// n_q <= 64; bf16, head_dim 128): two (sequence, head) items per CTA step.
//
// Target-aware cross attention and pooled attention have a few query tokens
// against a long key/value history ("GEM Training: How Meta Doubled the
// Efficiency of Its LLM-Scale Ads Foundation Model", "Challenge 1: Achieving
// High Per-GPU Utilization": such asymmetric shapes make intra-kernel
// pipelining less effective).  The general forward gives a (sequence, head)
// a 256-row query block of two tiles that alternate on the tensor core; with
// <= 64 query rows only one of them has work and nothing overlaps its
// softmax.  Here the two tiles of a CTA step hold two different items (the
// schedule's items 2p and 2p+1, adjacent in the longest-first order, so of
// similar length), each with its own key/value stream (one K and one V buffer
// per tile: K(j+1) loads during the softmax of step j, V(j+1) during the next
// Q K^T), and the tensor core alternates between them:
//   QK_A(0), QK_B(0), then per step j: [P_A(j)] PV_A(j), QK_A(j+1),
//   [P_B(j)] PV_B(j), QK_B(j+1).
// The queries of both items share one 128-row Q tile: item A's <= 64 rows in
// rows 0..63, item B's in rows 64..127.  Both Q K^T run M = 128 on the whole
// tile (each against its own item's keys), so item A's scores are valid in
// TMEM lanes 0..63 of S_A and item B's in lanes 64..127 of S_B (the other
// lanes pair a query with the other item's keys and are never read); P.V
// keeps the same lanes in O_A / O_B.  The softmax work of the two items thus
// falls on all four lane quarters, i.e. on all four SM sub-partitions.
//
// Warps: softmax warps 0, 1, 4, 5 (item A: lane quarters 0, 1) and 2, 3, 6, 7
// (item B: quarters 2, 3), half row (w >> 2) & 1 (64 columns); warp 8 MMA
// issuer and TMEM allocator, warp 9 TMA; warps 10, 11 (item A) and 12, 13
// (item B) stage a dense bias: each lane copies one query row's segment of
// the key tile (the covering 16-byte blocks, one bulk copy) into a per-item
// shared buffer as soon as the softmax warps have read the previous tile's,
// so the bias of a step is on chip when its scores arrive.
// With 448 threads a softmax thread keeps its 64 scores in registers between
// the maximum and the exponentials (one TMEM read per step).
#include <math_constants.h>

#include "jfa_sm100.cuh"

namespace jfa {

using namespace sm100;

bool make_tmap_rows_heads_d(CUtensorMap* map, const void* base, int64_t rows, int heads);
bool make_tmap_rows_heads_d_box(CUtensorMap* map, const void* base, int64_t rows, int heads, int box_rows);

JFA_TRACE_DEFINE(fwdsq)

namespace {

constexpr int BM = 128, BN = 128, HD = 128, BQ = 64;
constexpr int kMmaWarp = 8, kTmaWarp = 9;
constexpr int kThreads = 32 * 14;
constexpr int CW = 64;
constexpr uint32_t kBox = 128 * 128;
constexpr uint32_t kTile = 2 * kBox;
constexpr uint32_t kQHalf = BQ * 128;             // one item's [64 rows][64 bf16] in a box
constexpr uint32_t kOffQ = 0;                     // [Q_A; Q_B]: one 128-row tile
constexpr uint32_t kOffK = kOffQ + kTile;         // K_A, K_B
constexpr uint32_t kOffV = kOffK + 2 * kTile;     // V_A, V_B
constexpr int kWin = 384;
constexpr uint32_t kWinBytes = kWin * 16;
constexpr uint32_t kOffBias = kOffV + 2 * kTile;  // per tile
// dense bias rows of a key tile, per tile: 64 rows x 272 bytes (the 16-byte
// blocks that cover 128 bf16 at any 2-byte alignment)
constexpr uint32_t kDRow = 272;
constexpr uint32_t kOffDense = kOffBias + 2 * kWinBytes;
constexpr uint32_t kOffRed = kOffDense + 2 * BQ * kDRow;  // [parity][tile][half][64] row maxima
constexpr uint32_t kOffLred = kOffRed + 2 * 2 * 2 * 64 * 4;
constexpr uint32_t kOffBar = kOffLred + 2 * 2 * 2 * 64 * 4;
constexpr uint32_t kSmemBytes = kOffBar + 512 + 1024;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleThreshold = 8.0f;

struct Bars {
    uint64_t q_full[2], q_free[2];
    uint64_t k_full[2], k_empty[2];
    uint64_t v_full[2], v_empty[2];
    uint64_t s_full[2], p_full[2], pv_done[2], o_free[2];
    uint64_t bias_full[2];
    uint64_t dense_full[2], dense_empty[2];   // per tile: dense bias rows staged / read
    uint64_t pair[4];     // [tile][lane quarter]
    uint64_t drain;
    uint32_t tmem_base;
    int abort_flag;
};
static_assert(sizeof(Bars) <= 512, "barrier block");

struct FwdSqParams {
    CUtensorMap tm_q;
    CUtensorMap tm_k;
    CUtensorMap tm_v;
    AttnArgs a;
};

constexpr uint32_t kDescHi = sw128_desc_hi(1024u);
__device__ __forceinline__ uint32_t kmajor_lo(uint32_t tile_base) { return sw128_desc_lo(tile_base, 16u); }
__device__ __forceinline__ uint32_t mnmajor_lo(uint32_t tile_base) { return sw128_desc_lo(tile_base, kBox); }
__device__ __forceinline__ uint64_t kmajor_desc(uint32_t lo, int k) {
    return sw128_desc(lo + (uint32_t)(k >> 2) * (kBox >> 4) + (uint32_t)(k & 3) * 2u, kDescHi);
}
__device__ __forceinline__ uint64_t mnmajor_desc(uint32_t lo, int k) {
    return sw128_desc(lo + (uint32_t)k * 128u, kDescHi);
}

__device__ __forceinline__ int pair_of_turn(int r, int c, int G) {
    return r * G + ((r & 1) ? (G - 1 - c) : c);
}

struct Item {
    int b, h, q0, nq, k0, nkv;
    int n;   // key tiles (0: no item, or a sequence without keys)
    bool live;
};

__device__ __forceinline__ Item load_item(const AttnArgs& a, int idx, int n_items) {
    Item w{};
    w.live = idx < n_items;
    if (!w.live) return w;
    const int4 it = a.items[idx];
    w.b = it.x;
    w.h = it.y;
    w.q0 = a.q_off[w.b];
    w.nq = a.q_off[w.b + 1] - w.q0;
    w.k0 = a.kv_off[w.b];
    w.nkv = a.kv_off[w.b + 1] - w.k0;
    const int kv_end = a.causal ? max(0, min(w.nkv, w.nq + (w.nkv - w.nq))) : w.nkv;
    w.n = w.nq > 0 ? (kv_end + BN - 1) / BN : 0;
    return w;
}

__device__ __forceinline__ int bias_window_start(int jc, int C, int stride) {
    return min(max(-jc - (BN - 1) + C, 0), stride - kWin);
}

__device__ __forceinline__ void dense_bias16(const __nv_bfloat16* p, float (&bb)[16]) {
    const uintptr_t addr = reinterpret_cast<uintptr_t>(p);
    const uint4* blk = reinterpret_cast<const uint4*>(addr & ~static_cast<uintptr_t>(15));
    const int e0 = (int)(addr & 15) >> 1;
    const uint4 b0 = __ldg(blk), b1 = __ldg(blk + 1);
    const uint4 b2 = e0 ? __ldg(blk + 2) : make_uint4(0u, 0u, 0u, 0u);
    const uint32_t W[12] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w, b2.x, b2.y, b2.z, b2.w};
    const int s = e0 >> 1, sh = (e0 & 1) * 16;
    uint32_t V1[10], V2[9];
#pragma unroll
    for (int k = 0; k < 10; ++k) V1[k] = (s & 2) ? W[k + 2] : W[k];
#pragma unroll
    for (int k = 0; k < 9; ++k) V2[k] = (s & 1) ? V1[k + 1] : V1[k];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        const uint32_t pr = __funnelshift_r(V2[k], V2[k + 1], sh);
        bb[2 * k] = __uint_as_float(pr << 16);
        bb[2 * k + 1] = __uint_as_float(pr & 0xffff0000u);
    }
}

// 16 consecutive bf16 of a staged bias row as floats: element e of the row
// buffer (its first element at e0 < 8 of the first 16-byte block); the three
// blocks that cover them are in the buffer for every e <= e0 + 112.
__device__ __forceinline__ void staged_bias16(const uint8_t* rowbuf, int e, float (&bb)[16]) {
    const uint4* blk = reinterpret_cast<const uint4*>(rowbuf) + (e >> 3);
    const uint4 b0 = blk[0], b1 = blk[1], b2 = blk[2];
    const uint32_t W[12] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w, b2.x, b2.y, b2.z, b2.w};
    const int e0 = e & 7, s = e0 >> 1, sh = (e0 & 1) * 16;
    uint32_t V1[10], V2[9];
#pragma unroll
    for (int k = 0; k < 10; ++k) V1[k] = (s & 2) ? W[k + 2] : W[k];
#pragma unroll
    for (int k = 0; k < 9; ++k) V2[k] = (s & 1) ? V1[k + 1] : V1[k];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        const uint32_t pr = __funnelshift_r(V2[k], V2[k + 1], sh);
        bb[2 * k] = __uint_as_float(pr << 16);
        bb[2 * k + 1] = __uint_as_float(pr & 0xffff0000u);
    }
}

template <int BIAS, bool SOFTMAX>
__global__ void __launch_bounds__(kThreads, 1) tc_fwd_sq_kernel(const __grid_constant__ FwdSqParams P) {
    const AttnArgs& a = P.a;
    const int n_items = *a.item_count;
    const int n_pairs = (n_items + 1) >> 1;
    if (a.hdr->err != 0 || (int)blockIdx.x >= n_pairs) return;
    const bool out32 = (reinterpret_cast<uintptr_t>(a.out) & 31) == 0;
    extern __shared__ uint8_t smem_dyn[];
    uint8_t* smem = smem_dyn + ((1024u - (smem_u32(smem_dyn) & 1023u)) & 1023u);
    Bars* bars = reinterpret_cast<Bars*>(smem + kOffBar);
    const int G = gridDim.x, cta = blockIdx.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    constexpr bool softmax = SOFTMAX;

    if (threadIdx.x == 0) {
        for (int t = 0; t < 2; ++t) {
            mbar_init(&bars->q_full[t], 1);
            mbar_init(&bars->q_free[t], 1);
            mbar_init(&bars->k_full[t], 1);
            mbar_init(&bars->k_empty[t], 1);
            mbar_init(&bars->v_full[t], 1);
            mbar_init(&bars->v_empty[t], 1);
            mbar_init(&bars->s_full[t], 1);
            mbar_init(&bars->p_full[t], 4);
            mbar_init(&bars->pv_done[t], 1);
            mbar_init(&bars->o_free[t], 4);
            mbar_init(&bars->bias_full[t], 1);
            mbar_init(&bars->dense_full[t], 2);
            mbar_init(&bars->dense_empty[t], 4);
        }
        for (int q = 0; q < 4; ++q) mbar_init(&bars->pair[q], 2);
        mbar_init(&bars->drain, 1);
        bars->abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == kMmaWarp) {
        tmem_alloc(&bars->tmem_base, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bars->tmem_base;
    volatile int* abort_flag = &bars->abort_flag;
    const uint32_t sbase = smem_u32(smem);

    if (warp == kTmaWarp) {
        // ------------------------------------------------------------ TMA
        // lane t loads tile t's operands, in the order its MMAs free them:
        // K(j) once Q K(j-1)^T has run, V(j) once P.V(j-1) has
        if (lane < 2) {
            const int t = lane;
            tma_prefetch_desc(&P.tm_q);
            tma_prefetch_desc(&P.tm_k);
            tma_prefetch_desc(&P.tm_v);
            int qc = 0, kc = 0, vc = 0;   // Q, K and V loads issued for this tile
            bool ok = true;
            for (int r = 0; ok; ++r) {
                const int pr = pair_of_turn(r, cta, G);
                if (pr >= n_pairs) break;
                const Item w = load_item(a, 2 * pr + t, n_items);
                if (w.n == 0) continue;
                if (qc > 0 && !mbar_wait(&bars->q_free[t], (qc - 1) & 1, abort_flag, a.hdr)) { ok = false; break; }
                mbar_arrive_expect_tx(&bars->q_full[t], 2 * kQHalf);
                tma_load_3d(smem + kOffQ + t * kQHalf, &P.tm_q, &bars->q_full[t], 0, w.h, w.q0);
                tma_load_3d(smem + kOffQ + kBox + t * kQHalf, &P.tm_q, &bars->q_full[t], 64, w.h, w.q0);
                ++qc;
                for (int j = 0; j < w.n; ++j) {
                    const int z = w.k0 + j * BN;
                    if (kc > 0 && !mbar_wait(&bars->k_empty[t], (kc - 1) & 1, abort_flag, a.hdr)) { ok = false; break; }
                    mbar_arrive_expect_tx(&bars->k_full[t], kTile);
                    tma_load_3d(smem + kOffK + t * kTile, &P.tm_k, &bars->k_full[t], 0, w.h, z);
                    tma_load_3d(smem + kOffK + t * kTile + kBox, &P.tm_k, &bars->k_full[t], 64, w.h, z);
                    ++kc;
                    if (vc > 0 && !mbar_wait(&bars->v_empty[t], (vc - 1) & 1, abort_flag, a.hdr)) { ok = false; break; }
                    mbar_arrive_expect_tx(&bars->v_full[t], kTile);
                    tma_load_3d(smem + kOffV + t * kTile, &P.tm_v, &bars->v_full[t], 0, w.h, z);
                    tma_load_3d(smem + kOffV + t * kTile + kBox, &P.tm_v, &bars->v_full[t], 64, w.h, z);
                    if (BIAS == 1) {
                        // the previous window of this tile was read before its P.V
                        const int C = (a.relpos_len - 1) >> 1;
                        const int w0 = bias_window_start(j * BN, C, a.bias4_stride);
                        const float* src = a.bias4 + 4 * ((int64_t)w.h * a.bias4_stride + w0);
                        mbar_arrive_expect_tx(&bars->bias_full[t], kWinBytes);
                        bulk_load(smem + kOffBias + t * kWinBytes, src, kWinBytes, &bars->bias_full[t]);
                    }
                    ++vc;
                    if (j + 1 < w.n) {   // warm L2 for the next key tile
                        tma_prefetch_l2_3d(&P.tm_k, 0, w.h, z + BN);
                        tma_prefetch_l2_3d(&P.tm_k, 64, w.h, z + BN);
                        tma_prefetch_l2_3d(&P.tm_v, 0, w.h, z + BN);
                        tma_prefetch_l2_3d(&P.tm_v, 64, w.h, z + BN);
                    }
                }
            }
            // never leave the CTA with copies in flight (the K load of an
            // aborted step may have gone out without its V load)
            if (qc > 0) mbar_wait_drain(&bars->q_full[t], (qc - 1) & 1, a.hdr);
            if (kc > 0) mbar_wait_drain(&bars->k_full[t], (kc - 1) & 1, a.hdr);
            if (vc > 0) {
                mbar_wait_drain(&bars->v_full[t], (vc - 1) & 1, a.hdr);
                if (BIAS == 1) mbar_wait_drain(&bars->bias_full[t], (vc - 1) & 1, a.hdr);
            }
        }
    } else if (warp == kMmaWarp) {
        // ------------------------------------------------------------ MMA
        if (lane == 0) {
            constexpr uint32_t idesc_qk = idesc_bf16(BM, BN, 0, 0);
            constexpr uint32_t idesc_pv = idesc_bf16(BM, HD, 0, 1);
            int qc[2] = {0, 0}, kc[2] = {0, 0}, gt[2] = {0, 0}, mt[2] = {0, 0};
            bool ok = true;
            const uint32_t qK = kmajor_lo(sbase + kOffQ);   // both items' queries
            const uint32_t kK[2] = {kmajor_lo(sbase + kOffK), kmajor_lo(sbase + kOffK + kTile)};
            const uint32_t vM[2] = {mnmajor_lo(sbase + kOffV), mnmajor_lo(sbase + kOffV + kTile)};
            for (int r = 0; ok; ++r) {
                const int pr = pair_of_turn(r, cta, G);
                if (pr >= n_pairs) break;
                Item w[2] = {load_item(a, 2 * pr, n_items), load_item(a, 2 * pr + 1, n_items)};
                // S_T = Q_T K_T(j)^T; K is released after it, Q after the item's last
                auto issue_qk = [&](int t, int j) -> bool {
                    JFA_TRACE_EV(fwdsq, 1, kc[t], 2 * t);
                    if (!mbar_wait(&bars->k_full[t], kc[t] & 1, abort_flag, a.hdr)) return false;
                    JFA_TRACE_EV(fwdsq, 1, kc[t], 2 * t + 1);
                    tc_fence_after();
#pragma unroll
                    for (int k = 0; k < HD / 16; ++k)
                        mma_bf16_ss(tmem + t * 128, kmajor_desc(qK, k), kmajor_desc(kK[t], k), idesc_qk, k > 0 ? 1u : 0u);
                    mma_commit(&bars->s_full[t]);
                    mma_commit(&bars->k_empty[t]);
                    if (j == w[t].n - 1) mma_commit(&bars->q_free[t]);
                    return true;
                };
                for (int t = 0; t < 2 && ok; ++t) {
                    if (w[t].n == 0) continue;
                    if (!mbar_wait(&bars->q_full[t], qc[t] & 1, abort_flag, a.hdr)) { ok = false; break; }
                    ++qc[t];
                    ok = issue_qk(t, 0);
                }
                const int n = max(w[0].n, w[1].n);
                for (int j = 0; ok && j < n; ++j) {
                    for (int t = 0; t < 2 && ok; ++t) {
                        if (j >= w[t].n) continue;
                        if (!mbar_wait(&bars->p_full[t], gt[t] & 1, abort_flag, a.hdr)) { ok = false; break; }
                        if (j == 0 && mt[t] > 0 &&
                            !mbar_wait(&bars->o_free[t], (mt[t] - 1) & 1, abort_flag, a.hdr)) { ok = false; break; }
                        JFA_TRACE_EV(fwdsq, 1, kc[t], 4 + 2 * t);
                        if (!mbar_wait(&bars->v_full[t], kc[t] & 1, abort_flag, a.hdr)) { ok = false; break; }
                        JFA_TRACE_EV(fwdsq, 1, kc[t], 5 + 2 * t);
                        tc_fence_after();
                        const uint32_t tP = tmem + t * 128, tO = tmem + 256 + t * 128;
#pragma unroll
                        for (int k = 0; k < BN / 16; ++k)
                            mma_bf16_ts(tO, tP + k * 8 + (k >= 4 ? 32 : 0), mnmajor_desc(vM[t], k), idesc_pv,
                                        (j > 0 || k > 0) ? 1u : 0u);
                        mma_commit(&bars->pv_done[t]);
                        mma_commit(&bars->v_empty[t]);
                        ++gt[t];
                        ++kc[t];
                        if (j == 0) ++mt[t];
                        if (j + 1 < w[t].n) ok = issue_qk(t, j + 1);
                    }
                }
            }
            mma_commit(&bars->drain);
            mbar_wait_drain(&bars->drain, 0, a.hdr);
        }
    } else if (warp < 8) {
        // ------------------------------------------------ softmax warps
        auto wwait = [&](uint64_t* bar, uint32_t parity) -> bool {
            return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag, a.hdr));
        };
        const int wq = warp & 3;                 // TMEM lane quarter
        const int tt = wq >> 1;                  // item A: quarters 0, 1; item B: 2, 3
        const int hf = (warp >> 2) & 1;
        const int r_ = (wq & 1) * 32 + lane;     // row 0..63 of the item
        const int cb = hf * CW;
        const uint32_t lane_addr = (uint32_t)(wq * 32) << 16;
        const uint32_t tS = tmem + lane_addr + tt * 128;
        const uint32_t tO = tmem + lane_addr + 256 + tt * 128 + cb;
        float* red = reinterpret_cast<float*>(smem + kOffRed);
        float* lred = reinterpret_cast<float*>(smem + kOffLred);
        uint64_t* pair_bar = &bars->pair[tt * 2 + (wq & 1)];
        int n_pair = 0;
        auto pair_sync = [&]() -> bool {
            __syncwarp();
            if (lane == 0) mbar_arrive(pair_bar);
            return wwait(pair_bar, (n_pair++) & 1);
        };
        const float sc = a.scale * kLog2e;
        const float2 sc2 = make_float2(sc, sc);
        const int C = (a.relpos_len - 1) >> 1;
        int gt = 0, mt = 0;
        bool ok = true;
        for (int rr = 0; ok; ++rr) {
            const int pr = pair_of_turn(rr, cta, G);
            if (pr >= n_pairs) break;
            const Item w = load_item(a, 2 * pr + tt, n_items);
            if (!w.live) continue;
            const int n = w.n;
            const int i = r_;
            if (n == 0) {
                if (i < w.nq) {
                    __nv_bfloat16* orow = reinterpret_cast<__nv_bfloat16*>(a.out) + ((int64_t)(w.q0 + i) * a.H + w.h) * HD + cb;
#pragma unroll
                    for (int t = 0; t < CW; t += 8) *reinterpret_cast<uint4*>(orow + t) = make_uint4(0, 0, 0, 0);
                    if (softmax && a.lse && hf == 0) a.lse[(int64_t)(w.q0 + i) * a.H + w.h] = -CUDART_INF_F;
                }
                continue;
            }
            const int shift = w.nkv - w.nq;
            const float inv_n = w.nkv > 0 ? 1.0f / (float)w.nkv : 0.f;
            const float half_c = inv_n * (0.5f / kLog2e);   // GDPA: act(s) / n_kv = x half_c (1 + tanh)
            const int jmax_vis = a.causal ? min(w.nkv - 1, i + shift) : w.nkv - 1;
            const float* tab4 = (BIAS == 1) ? a.bias4 + (int64_t)w.h * 4 * a.bias4_stride : nullptr;
            const __nv_bfloat16* dense = reinterpret_cast<const __nv_bfloat16*>(a.bias);
            const int64_t dense_row = (BIAS == 2 && i < w.nq)
                                          ? a.dense_off[w.b] + ((int64_t)w.h * w.nq + i) * w.nkv : 0;
            // this row's staged bias: element k of key tile j at element e0 + k
            // of the row buffer (e0: the 2-byte offset of the tile's first key
            // in its 16-byte block; a key tile starts 128 elements on, so e0
            // is the same for every tile of the row)
            const uint8_t* drow = smem + kOffDense + (tt * BQ + r_) * kDRow;
            const int e0 = (int)((reinterpret_cast<uintptr_t>(dense + dense_row) & 15) >> 1);
            float m_used = -CUDART_INF_F, l = 0.f;
            const bool tr = lane == 0 && (warp == 0 || warp == 2);
            for (int j = 0; j < n; ++j, ++gt) {
                if (tr) JFA_TRACE_EV(fwdsq, 2 + tt, gt, 0);
                if (!wwait(&bars->s_full[tt], gt & 1)) { ok = false; break; }
                if (tr) JFA_TRACE_EV(fwdsq, 2 + tt, gt, 1);
                tc_fence_after();
                const int jc = j * BN;
                if (BIAS == 1 && !wwait(&bars->bias_full[tt], gt & 1)) { ok = false; break; }
                if (BIAS == 2 && !wwait(&bars->dense_full[tt], gt & 1)) { ok = false; break; }
                if (tr) JFA_TRACE_EV(fwdsq, 2 + tt, gt, 2);
                const int nvis = i < w.nq ? max(0, min(BN, jmax_vis - jc + 1)) : 0;
                const bool masked_half = __any_sync(0xffffffffu, nvis < cb + CW);
                const int lo = i - jc - (BN - 1) + C;
                const int wrel = BIAS == 1 ? lo - bias_window_start(jc, C, a.bias4_stride) : 0;
                const bool win_ok = BIAS == 1 && lo >= 0 && lo + (BN - 1) <= 2 * C && wrel >= 0 && wrel + BN - 4 < kWin;
                const float4* win = reinterpret_cast<const float4*>(smem + kOffBias + tt * kWinBytes) + wrel;
                // ---- this thread's 64 scores, held in registers
                uint32_t xs[CW / 16][16];
#pragma unroll
                for (int c = 0; c < CW / 16; ++c) tmem_ld16(tS + cb + c * 16, xs[c]);
                float pm = -CUDART_INF_F;
                tmem_wait_ld();
#pragma unroll
                for (int c = 0; c < CW / 16; ++c) {
                    const int cc = cb + c * 16;
                    float* x = reinterpret_cast<float*>(xs[c]);
                    if (BIAS == 1) {
                        float bb[16];
                        if (win_ok) {
#pragma unroll
                            for (int q = 0; q < 4; ++q) {
                                const float4 t4 = win[(BN - 4) - cc - 4 * q];
                                bb[4 * q] = t4.w, bb[4 * q + 1] = t4.z, bb[4 * q + 2] = t4.y, bb[4 * q + 3] = t4.x;
                            }
                        } else {
                            const int hi = lo + (BN - 1) - cc;
#pragma unroll
                            for (int v = 0; v < 16; ++v) bb[v] = __ldg(tab4 + 4 * min(max(hi - v, 0), 2 * C));
                        }
#pragma unroll
                        for (int v = 0; v < 16; v += 2) {
                            const float2 r2 = fma2(make_float2(x[v], x[v + 1]), sc2, make_float2(bb[v], bb[v + 1]));
                            x[v] = r2.x, x[v + 1] = r2.y;
                        }
                    } else if (BIAS == 2) {
                        if (cc + 16 <= nvis) {
                            float bb[16];
                            staged_bias16(drow, e0 + cc, bb);
#pragma unroll
                            for (int v = 0; v < 16; v += 2) {
                                const float2 r2 = fma2(make_float2(x[v], x[v + 1]), sc2,
                                                       mul2(make_float2(bb[v], bb[v + 1]), make_float2(kLog2e, kLog2e)));
                                x[v] = r2.x, x[v + 1] = r2.y;
                            }
                        } else {
#pragma unroll
                            for (int v = 0; v < 16; ++v)
                                x[v] = fmaf(x[v], sc,
                                            cc + v < nvis
                                                ? __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(drow)[e0 + cc + v]) * kLog2e
                                                : 0.f);
                        }
                    } else {
#pragma unroll
                        for (int v = 0; v < 16; v += 2) {
                            const float2 r2 = mul2(make_float2(x[v], x[v + 1]), sc2);
                            x[v] = r2.x, x[v + 1] = r2.y;
                        }
                    }
                    if (masked_half) {
#pragma unroll
                        for (int v = 0; v < 16; ++v) x[v] = cc + v < nvis ? x[v] : -CUDART_INF_F;
                    }
                    if (softmax) {
                        const float m0 = max3(x[0], x[1], x[2]), m1 = max3(x[3], x[4], x[5]);
                        const float m2 = max3(x[6], x[7], x[8]), m3 = max3(x[9], x[10], x[11]);
                        const float m4 = max3(x[12], x[13], x[14]);
                        pm = max3(pm, max3(m0, m1, m2), max3(m3, m4, x[15]));
                    }
                }
                if (BIAS == 2) {   // the staged rows of this step are read
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&bars->dense_empty[tt]);
                }
                if (tr) JFA_TRACE_EV(fwdsq, 2 + tt, gt, 3);
                float ref = 0.f;
                if (softmax) {
                    float* rp = red + ((gt & 1) * 4 + tt * 2) * 64;
                    rp[hf * 64 + r_] = pm;
                    if (!pair_sync()) { ok = false; break; }
                    pm = fmaxf(pm, rp[(hf ^ 1) * 64 + r_]);
                    float alpha = 1.f;
                    bool rescale = false;
                    const bool need = pm > m_used + kRescaleThreshold;
                    const float m_new = need ? pm : m_used;
                    if (need && m_used != -CUDART_INF_F) {
                        alpha = ex2(m_used - m_new);
                        rescale = true;
                    } else if (need) {
                        l = 0.f;
                    }
                    m_used = m_new;
                    if (__any_sync(0xffffffffu, rescale)) {
                        if (j > 0) {
                            if (!wwait(&bars->pv_done[tt], (gt - 1) & 1)) { ok = false; break; }
                            tc_fence_after();
#pragma unroll 1
                            for (int c = 0; c < CW / 32; ++c) {
                                uint32_t u[32];
                                tmem_ld32(tO + c * 32, u);
                                tmem_wait_ld();
#pragma unroll
                                for (int t = 0; t < 32; t += 2) {
                                    const float2 r2 = mul2(make_float2(__uint_as_float(u[t]), __uint_as_float(u[t + 1])),
                                                           make_float2(alpha, alpha));
                                    u[t] = __float_as_uint(r2.x), u[t + 1] = __float_as_uint(r2.y);
                                }
                                tmem_st32(tO + c * 32, u);
                            }
                        }
                        l *= alpha;
                    }
                    ref = m_used == -CUDART_INF_F ? 0.f : m_used;
                }
                // ---- P (bf16 pairs) over the first half of this thread's S columns
                {
                    const float2 ref2 = make_float2(ref, ref);
                    float2 ps = make_float2(0.f, 0.f), ps2 = make_float2(0.f, 0.f);
#pragma unroll
                    for (int c = 0; c < CW / 16; ++c) {
                        const int cc = cb + c * 16;
                        float* x = reinterpret_cast<float*>(xs[c]);
                        if (softmax) {
#pragma unroll
                            for (int v = 0; v < 16; v += 2) {
                                const float2 y = sub2(make_float2(x[v], x[v + 1]), ref2);
                                x[v] = ex2(y.x);
                                x[v + 1] = ex2(y.y);
                                if (v & 2) ps2 = add2(ps2, make_float2(x[v], x[v + 1]));
                                else ps = add2(ps, make_float2(x[v], x[v + 1]));
                            }
                        } else if (a.act == JFA_ACT_SILU) {
#pragma unroll
                            for (int v = 0; v < 16; ++v)
                                x[v] = cc + v < nvis ? gdpa_weight_log2<JFA_ACT_SILU>(x[v], half_c) : 0.f;
                        } else {
#pragma unroll
                            for (int v = 0; v < 16; ++v)
                                x[v] = cc + v < nvis ? gdpa_weight_log2<JFA_ACT_GELU_TANH>(x[v], half_c) : 0.f;
                        }
                        uint32_t pw[8];
#pragma unroll
                        for (int t = 0; t < 8; ++t) pw[t] = pack_bf16(x[2 * t], x[2 * t + 1]);
                        tmem_st8(tS + cb + c * 8, pw);
                    }
                    tmem_wait_st();
                    const float2 s4 = add2(ps, ps2);
                    l += s4.x + s4.y;
                }
                // value rows past the sequence end must not reach P.V (rows
                // 64..127 of this thread's warp pair are cleared by the row r_
                // and r_ + 64 threads)
                const int nvalid = w.nkv - jc;
                if (nvalid < BN) {
                    if (!wwait(&bars->v_full[tt], gt & 1)) { ok = false; break; }
                    uint8_t* vt = smem + kOffV + tt * kTile + hf * kBox;
                    const uint4 z = make_uint4(0, 0, 0, 0);
                    for (int rr2 = r_; rr2 < BN; rr2 += BQ)
                        if (rr2 >= nvalid)
#pragma unroll
                            for (int ch = 0; ch < 8; ++ch) *reinterpret_cast<uint4*>(vt + rr2 * 128 + ch * 16) = z;
                }
                fence_proxy_async_smem();
                tc_fence_before();
                __syncwarp();
                if (tr) JFA_TRACE_EV(fwdsq, 2 + tt, gt, 4);
                if (lane == 0) mbar_arrive(&bars->p_full[tt]);
            }
            if (!ok) break;
            // ---------------------------------------------------- epilogue
            if (!wwait(&bars->pv_done[tt], (gt - 1) & 1)) { ok = false; break; }
            tc_fence_after();
            float l_row = l;
            if (softmax) {
                float* lp = lred + ((mt & 1) * 4 + tt * 2) * 64;
                lp[hf * 64 + r_] = l;
                if (!pair_sync()) { ok = false; break; }
                l_row += lp[(hf ^ 1) * 64 + r_];
            }
            ++mt;
            const float inv = softmax ? (l_row > 0.f ? 1.f / l_row : 0.f) : 1.f;
            __nv_bfloat16* orow = reinterpret_cast<__nv_bfloat16*>(a.out) + ((int64_t)(w.q0 + i) * a.H + w.h) * HD + cb;
#pragma unroll 1
            for (int c = 0; c < CW / 32; ++c) {
                uint32_t u[32];
                tmem_ld32(tO + c * 32, u);
                tmem_wait_ld();
                if (i < w.nq) {
#pragma unroll
                    for (int t = 0; t < 32; t += 16) store_bf16x16(orow + c * 32 + t, u + t, inv, out32);
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->o_free[tt]);
            if (softmax && hf == 0 && i < w.nq && a.lse)
                a.lse[(int64_t)(w.q0 + i) * a.H + w.h] =
                    l_row > 0.f ? m_used * (1.0f / kLog2e) + logf(l_row) : -CUDART_INF_F;
        }
    } else if (BIAS == 2 && warp >= 10) {
        // ------------------------------------------------ dense bias stagers
        // warps 10, 11 (item A) and 12, 13 (item B); lane -> query row
        const int tt = (warp - 10) >> 1;
        const int row = (warp & 1) * 32 + lane;
        uint8_t* dst = smem + kOffDense + (tt * BQ + row) * kDRow;
        uint64_t* full = &bars->dense_full[tt];
        const __nv_bfloat16* dense = reinterpret_cast<const __nv_bfloat16*>(a.bias);
        int g = 0;   // steps staged for this tile (the softmax warps' step count)
        bool ok = true;
        for (int rr = 0; ok; ++rr) {
            const int pr = pair_of_turn(rr, cta, G);
            if (pr >= n_pairs) break;
            const Item w = load_item(a, 2 * pr + tt, n_items);
            if (!w.live || w.n == 0) continue;
            const bool has_row = row < w.nq;
            const int64_t row_off = has_row ? a.dense_off[w.b] + ((int64_t)w.h * w.nq + row) * w.nkv : 0;
            for (int j = 0; j < w.n; ++j, ++g) {
                // the buffer is free once the softmax warps have read step g - 1
                if (g > 0 && !__all_sync(0xffffffffu, mbar_wait(&bars->dense_empty[tt], (g - 1) & 1, abort_flag, a.hdr))) {
                    ok = false;
                    break;
                }
                const int jc = j * BN;
                const int nk = min(BN, w.nkv - jc);   // keys of this tile (>= 1)
                // the 16-byte blocks covering the row's nk bias values: every
                // block holds a value of the bias tensor, so the copy stays in
                // its allocation
                uintptr_t src = 0;
                uint32_t bytes = 0;
                if (has_row) {
                    const uintptr_t first = reinterpret_cast<uintptr_t>(dense + row_off + jc);
                    src = first & ~static_cast<uintptr_t>(15);
                    bytes = (uint32_t)(((first + 2u * (uint32_t)nk + 15u) & ~static_cast<uintptr_t>(15)) - src);
                }
                const uint32_t total = __reduce_add_sync(0xffffffffu, bytes);
                if (lane == 0) mbar_arrive_expect_tx(full, total);
                __syncwarp();
                if (bytes) bulk_load(dst, reinterpret_cast<const void*>(src), bytes, full);
                if (has_row && j + 1 < w.n) {   // warm L2 for the next step's rows
                    prefetch_l2(dense + row_off + jc + BN);
                    prefetch_l2(dense + row_off + min(jc + 2 * BN, w.nkv) - 1);
                }
            }
        }
        // never leave the CTA with copies in flight
        if (g > 0 && lane == 0) mbar_wait_drain(full, (g - 1) & 1, a.hdr);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

}  // namespace

constexpr int kSmemLimitFsq = 232448;

// Items: the forward's query-block schedule (one item per (sequence, head)
// when every n_q <= 64), taken two at a time.
cudaError_t tc_forward_sq_launch(const jfa_problem& p, const AttnArgs& a, cudaStream_t st) {
    FwdSqParams P{};
    if (!make_tmap_rows_heads_d_box(&P.tm_q, a.q, p.total_q, p.heads, BQ) ||
        !make_tmap_rows_heads_d(&P.tm_k, a.k, p.total_kv, p.heads) ||
        !make_tmap_rows_heads_d(&P.tm_v, a.v, p.total_kv, p.heads))
        return cudaErrorInvalidValue;
    P.a = a;
    const int64_t items_bound = (int64_t)p.batch * p.heads;
    if (items_bound <= 0) return cudaSuccess;
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t pairs = (items_bound + 1) / 2;
    const int grid = (int)(pairs < sms ? pairs : sms);
    const int bias = p.bias_kind == JFA_BIAS_RELPOS ? 1 : (p.bias_kind == JFA_BIAS_DENSE_JAGGED ? 2 : 0);
    const bool sm = a.act == JFA_ACT_SOFTMAX;
    void (*kern)(FwdSqParams) =
        bias == 0 ? (sm ? tc_fwd_sq_kernel<0, true> : tc_fwd_sq_kernel<0, false>)
                  : (bias == 1 ? (sm ? tc_fwd_sq_kernel<1, true> : tc_fwd_sq_kernel<1, false>)
                               : (sm ? tc_fwd_sq_kernel<2, true> : tc_fwd_sq_kernel<2, false>));
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemLimitFsq);
    if (e != cudaSuccess) return e;
    static_assert(kSmemBytes <= (uint32_t)kSmemLimitFsq, "shared memory");
    prof_begin(st);
    kern<<<grid, kThreads, kSmemBytes, st>>>(P);
    prof_end(st, K_TC_FWD_SQ);
    return cudaGetLastError();
}

}  // namespace jfa
