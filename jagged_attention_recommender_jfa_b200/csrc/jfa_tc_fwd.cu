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

namespace {

constexpr int BM = 128, BN = 128, HD = 128;
constexpr int kThreads = 320;               // warp 0 TMA, warp 1 MMA, warps 2..9 softmax
constexpr uint32_t kBox = 128 * 128;        // bytes of one [128 rows][64 bf16] box
constexpr uint32_t kTile = 2 * kBox;        // one 128 x 128 bf16 tile (two boxes)
constexpr uint32_t kOffQ = 0;
constexpr uint32_t kOffK = kOffQ + kTile;        // 2 stages
constexpr uint32_t kOffV = kOffK + 2 * kTile;    // 2 stages
constexpr uint32_t kOffP = kOffV + 2 * kTile;
constexpr uint32_t kOffBar = kOffP + kTile;      // 196608
constexpr uint32_t kOffRed = kOffBar + 256;      // row-max exchange [2][2][128] + l [2][128]
constexpr uint32_t kOffTab = kOffRed + 3072;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleThreshold = 8.0f;        // log2 units

struct Bars {
    uint64_t q_full;
    uint64_t k_full[2], k_empty[2];
    uint64_t v_full[2], v_empty[2];
    uint64_t s_full[2];
    uint64_t p_full;
    uint64_t pv_done;
    uint64_t drain;
    uint32_t tmem_base;
    int abort_flag;
};
static_assert(sizeof(Bars) <= 256, "barrier block");

struct FwdParams {
    CUtensorMap tm_q;
    CUtensorMap tm_k;
    CUtensorMap tm_v;
    AttnArgs a;
    int tab_cap;  // floats of relative-position window that fit in shared memory
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
    asm volatile("bar.sync 1, 256;" ::: "memory");
}

// BIAS: 0 none, 1 relative-position (window in shared memory when it fits,
// else through L1), 2 dense jagged.  SOFTMAX: softmax (true) or GDPA.
// QP: MXFP8 attention -- P is quantised to E4M3 with one E8M0 scale per 32
// keys (counted from the sequence's first key) before P.V; the row sum l
// uses the unquantised weights.
//
// Pipeline (tensor core): QK_0, QK_1, then for each j: [P_j ready] PV_j,
// QK_{j+2}.  S is double-buffered in TMEM (S_0 at column 0, S_1 at 128), so
// the score MMA of tile j+1 runs while the softmax warps work on tile j.
// O lives at column 256.  P goes through shared memory (one buffer): the
// softmax of tile j writes it only after P.V of tile j-1 has completed.
// Each softmax thread owns one query row and one 64-column half of it; the
// two halves exchange their partial row maxima through shared memory.
template <int BIAS, bool SOFTMAX, bool QP>
__global__ void __launch_bounds__(kThreads, 1) tc_fwd_kernel(const __grid_constant__ FwdParams P) {
    const AttnArgs& a = P.a;
    if ((int)blockIdx.x >= *a.item_count || a.hdr->err != 0) return;
    extern __shared__ uint8_t smem_dyn[];
    uint8_t* smem = smem_dyn + ((1024u - (smem_u32(smem_dyn) & 1023u)) & 1023u);
    Bars* bars = reinterpret_cast<Bars*>(smem + kOffBar);
    float* red = reinterpret_cast<float*>(smem + kOffRed);   // [2 parity][2 half][128 rows]
    float* lred = red + 512;                                   // [2 half][128 rows]
    float* tab = reinterpret_cast<float*>(smem + kOffTab);

    const int4 it = a.items[blockIdx.x];
    const int b = it.x, h = it.y, row0 = it.z * BM;
    const int q0 = a.q_off[b], nq = a.q_off[b + 1] - q0;
    const int k0 = a.kv_off[b], nkv = a.kv_off[b + 1] - k0;
    const int rows_hi = min(row0 + BM, nq);
    int kv_end = a.causal ? min(nkv, rows_hi + (nkv - nq)) : nkv;
    kv_end = max(kv_end, 0);
    const int n_tiles = (kv_end + BN - 1) / BN;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    constexpr bool softmax = SOFTMAX;

    // relative-position window: i - j in [lo, lo + tab_len)
    const int tab_lo = row0 - kv_end + 1;
    const int tab_len = kv_end + BM - 1;
    const bool tab_in_smem = BIAS == 1 && tab_len <= P.tab_cap;

    if (threadIdx.x == 0) {
        mbar_init(&bars->q_full, 1);
        for (int s = 0; s < 2; ++s) {
            mbar_init(&bars->k_full[s], 1);
            mbar_init(&bars->k_empty[s], 1);
            mbar_init(&bars->v_full[s], 1);
            mbar_init(&bars->v_empty[s], 1);
            mbar_init(&bars->s_full[s], 1);
        }
        mbar_init(&bars->p_full, 8);
        mbar_init(&bars->pv_done, 1);
        mbar_init(&bars->drain, 1);
        bars->abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(&bars->tmem_base, 512);
        tmem_relinquish();
    }
    if (tab_in_smem) {
        const int C = (a.relpos_len - 1) >> 1;
        const float* src = reinterpret_cast<const float*>(a.bias) + (int64_t)h * a.relpos_len;
        for (int t = threadIdx.x; t < tab_len; t += kThreads) {
            int r = tab_lo + t;
            r = r < -C ? -C : (r > C ? C : r);
            tab[t] = __ldg(src + r + C) * kLog2e;
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bars->tmem_base;
    volatile int* abort_flag = &bars->abort_flag;
    const uint32_t sbase = smem_u32(smem);

    if (warp == 0) {
        // ------------------------------------------------------------ TMA
        if (lane == 0 && n_tiles > 0) {
            tma_prefetch_desc(&P.tm_q);
            tma_prefetch_desc(&P.tm_k);
            tma_prefetch_desc(&P.tm_v);
            mbar_arrive_expect_tx(&bars->q_full, kTile);
            tma_load_3d(smem + kOffQ, &P.tm_q, &bars->q_full, 0, h, q0 + row0);
            tma_load_3d(smem + kOffQ + kBox, &P.tm_q, &bars->q_full, 64, h, q0 + row0);
            int issued = 0;
            for (int j = 0; j < n_tiles; ++j) {
                const int s = j & 1;
                const uint32_t par = ((j >> 1) - 1) & 1;
                const int z = k0 + j * BN;
                if (j >= 2 && !mbar_wait(&bars->k_empty[s], par, abort_flag, a.hdr)) break;
                mbar_arrive_expect_tx(&bars->k_full[s], kTile);
                tma_load_3d(smem + kOffK + s * kTile, &P.tm_k, &bars->k_full[s], 0, h, z);
                tma_load_3d(smem + kOffK + s * kTile + kBox, &P.tm_k, &bars->k_full[s], 64, h, z);
                if (j >= 2 && !mbar_wait(&bars->v_empty[s], par, abort_flag, a.hdr)) { issued = -(j + 1); break; }
                mbar_arrive_expect_tx(&bars->v_full[s], kTile);
                tma_load_3d(smem + kOffV + s * kTile, &P.tm_v, &bars->v_full[s], 0, h, z);
                tma_load_3d(smem + kOffV + s * kTile + kBox, &P.tm_v, &bars->v_full[s], 64, h, z);
                issued = j + 1;
                if (j + 2 < n_tiles) {  // warm L2 for the tiles loaded after the next release
                    const int zn = z + 2 * BN;
                    tma_prefetch_l2_3d(&P.tm_k, 0, h, zn);
                    tma_prefetch_l2_3d(&P.tm_k, 64, h, zn);
                    tma_prefetch_l2_3d(&P.tm_v, 0, h, zn);
                    tma_prefetch_l2_3d(&P.tm_v, 64, h, zn);
                }
            }
            // never leave the CTA with copies in flight: wait for every issued load
            mbar_wait_drain(&bars->q_full, 0, a.hdr);
            const int nk = issued >= 0 ? issued : -issued;       // K loads issued
            const int nv = issued >= 0 ? issued : -issued - 1;   // V loads issued
            for (int j = (nk > 2 ? nk - 2 : 0); j < nk; ++j) mbar_wait_drain(&bars->k_full[j & 1], (j >> 1) & 1, a.hdr);
            for (int j = (nv > 2 ? nv - 2 : 0); j < nv; ++j) mbar_wait_drain(&bars->v_full[j & 1], (j >> 1) & 1, a.hdr);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA
        if (lane == 0 && n_tiles > 0) {
            constexpr uint32_t idesc_qk = idesc_bf16(BM, BN, 0, 0);
            constexpr uint32_t idesc_pv = idesc_bf16(BM, HD, 0, 1);
            const uint32_t tO = tmem + 256;
            const uint32_t qb = sbase + kOffQ, pb = sbase + kOffP;
            bool ok = mbar_wait(&bars->q_full, 0, abort_flag, a.hdr);
            for (int j = 0; ok && j < 2 && j < n_tiles; ++j) {
                if (!mbar_wait(&bars->k_full[j], 0, abort_flag, a.hdr)) { ok = false; break; }
                tc_fence_after();
                const uint32_t kb = sbase + kOffK + j * kTile;
#pragma unroll
                for (int k = 0; k < HD / 16; ++k)
                    mma_bf16_ss(tmem + j * 128, kmajor_desc(qb, k), kmajor_desc(kb, k), idesc_qk, k > 0 ? 1u : 0u);
                mma_commit(&bars->s_full[j]);
                mma_commit(&bars->k_empty[j]);
            }
            for (int j = 0; ok && j < n_tiles; ++j) {
                const int s = j & 1;
                if (!mbar_wait(&bars->p_full, j & 1, abort_flag, a.hdr)) { ok = false; break; }
                if (!mbar_wait(&bars->v_full[s], (j >> 1) & 1, abort_flag, a.hdr)) { ok = false; break; }
                tc_fence_after();
                const uint32_t vb = sbase + kOffV + s * kTile;
#pragma unroll
                for (int k = 0; k < BN / 16; ++k)
                    mma_bf16_ss(tO, kmajor_desc(pb, k), mnmajor_desc(vb, k), idesc_pv,
                                (j > 0 || k > 0) ? 1u : 0u);
                mma_commit(&bars->v_empty[s]);
                mma_commit(&bars->pv_done);
                if (j + 2 < n_tiles) {
                    if (!mbar_wait(&bars->k_full[s], ((j + 2) >> 1) & 1, abort_flag, a.hdr)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t kb = sbase + kOffK + s * kTile;
#pragma unroll
                    for (int k = 0; k < HD / 16; ++k)
                        mma_bf16_ss(tmem + s * 128, kmajor_desc(qb, k), kmajor_desc(kb, k), idesc_qk,
                                    k > 0 ? 1u : 0u);
                    mma_commit(&bars->s_full[s]);
                    mma_commit(&bars->k_empty[s]);
                }
            }
            // all issued MMAs retire before TMEM is released
            mma_commit(&bars->drain);
            mbar_wait_drain(&bars->drain, 0, a.hdr);
        }
    } else {
        // ------------------------------------------------ softmax warps
        const int wq = warp & 3;                 // TMEM lane quarter
        const int grp = (warp - 2) >> 2;         // column half of S / O
        const int r = wq * 32 + lane;            // row within the tile
        const int i = row0 + r;                  // query index within the sequence
        const int c0 = grp * 64;                 // first column of this thread's half
        const uint32_t lane_addr = (uint32_t)(wq * 32) << 16;
        const uint32_t tO = tmem + lane_addr + 256 + c0;
        const float sc = a.scale * kLog2e;
        const int shift = nkv - nq;              // causal: key j visible iff j <= i + shift
        const float inv_n = nkv > 0 ? 1.0f / (float)nkv : 0.f;
        const int C = (a.relpos_len - 1) >> 1;
        const float* tab_g = reinterpret_cast<const float*>(a.bias) + (int64_t)h * a.relpos_len;
        const __nv_bfloat16* dense = reinterpret_cast<const __nv_bfloat16*>(a.bias);
        const int64_t dense_row = (BIAS == 2 && i < nq)
                                      ? a.dense_off[b] + ((int64_t)h * nq + i) * nkv : 0;
        const int jmax_vis = a.causal ? min(nkv - 1, i + shift) : nkv - 1;  // last visible key
        uint8_t* prow = smem + kOffP + grp * kBox + r * 128;
        float m_used = -CUDART_INF_F, l = 0.f;   // l: this half's partial sum
        bool ok = true;
        // Every softmax warp runs the same sequence of named barriers: a failed
        // (timed-out) wait only sets the CTA's abort flag, and the loop is left
        // right after a barrier, where all warps read the same flag.
        for (int j = 0; j < n_tiles; ++j) {
            const int s = j & 1;
            mbar_wait(&bars->s_full[s], (j >> 1) & 1, abort_flag, a.hdr);
            tc_fence_after();
            const int jc = j * BN + c0;          // key index of this half's column 0
            float x[64];
            {
                uint32_t u[2][32];
                tmem_ld32(tmem + lane_addr + s * 128 + c0, u[0]);
                tmem_ld32(tmem + lane_addr + s * 128 + c0 + 32, u[1]);
                tmem_wait_ld();
#pragma unroll
                for (int t = 0; t < 32; ++t) {
                    x[t] = __uint_as_float(u[0][t]);
                    x[32 + t] = __uint_as_float(u[1][t]);
                }
            }
            const int nvis = i < nq ? max(0, min(64, jmax_vis - jc + 1)) : 0;  // visible: [0, nvis)
            if (BIAS == 1 && tab_in_smem) {
                const float* tb = tab + (i - jc - tab_lo);  // tb[-c] = bias(i, jc + c)
#pragma unroll
                for (int c = 0; c < 64; ++c) x[c] = fmaf(x[c], sc, tb[-c]);
            } else if (BIAS == 1) {
#pragma unroll
                for (int c = 0; c < 64; ++c) {
                    int rr = i - (jc + c);
                    rr = rr < -C ? -C : (rr > C ? C : rr);
                    x[c] = fmaf(x[c], sc, __ldg(tab_g + rr + C) * kLog2e);
                }
            } else if (BIAS == 2) {
#pragma unroll
                for (int c = 0; c < 64; ++c)
                    x[c] = fmaf(x[c], sc, c < nvis ? __bfloat162float(dense[dense_row + jc + c]) * kLog2e : 0.f);
            } else {
#pragma unroll
                for (int c = 0; c < 64; ++c) x[c] *= sc;
            }
            if (__any_sync(0xffffffffu, nvis < 64)) {
#pragma unroll
                for (int c = 0; c < 64; ++c) x[c] = c < nvis ? x[c] : -CUDART_INF_F;
            }
            float alpha = 1.f;
            bool rescale = false;
            if (softmax) {
                float pm8[8];
#pragma unroll
                for (int t = 0; t < 8; ++t) pm8[t] = x[t];
#pragma unroll
                for (int c = 8; c < 64; ++c) pm8[c & 7] = fmaxf(pm8[c & 7], x[c]);
                const float pm = fmaxf(fmaxf(fmaxf(pm8[0], pm8[1]), fmaxf(pm8[2], pm8[3])),
                                       fmaxf(fmaxf(pm8[4], pm8[5]), fmaxf(pm8[6], pm8[7])));
                red[(s * 2 + grp) * 128 + r] = pm;
                named_sync_softmax();
                if (*abort_flag) { ok = false; break; }
                const float tmax = fmaxf(pm, red[(s * 2 + (grp ^ 1)) * 128 + r]);
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
            // P.V of the previous tile must be done before O or the P buffer change
            if (j > 0) {
                mbar_wait(&bars->pv_done, (j - 1) & 1, abort_flag, a.hdr);
                tc_fence_after();
            }
            if (softmax && __any_sync(0xffffffffu, rescale)) {
#pragma unroll
                for (int c4 = 0; c4 < 2; ++c4) {
                    uint32_t u[32];
                    tmem_ld32(tO + c4 * 32, u);
                    tmem_wait_ld();
#pragma unroll
                    for (int t = 0; t < 32; ++t) u[t] = __float_as_uint(__uint_as_float(u[t]) * alpha);
                    tmem_st32(tO + c4 * 32, u);
                }
                tmem_wait_st();
                l *= alpha;
            }
            if (softmax) {
                // ex2(-inf) = 0 masks the invisible columns; a row with no visible
                // key yet uses reference 0 so that -inf - ref stays -inf
                const float ref = m_used == -CUDART_INF_F ? 0.f : m_used;
                float ps8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int c = 0; c < 64; ++c) {
                    x[c] = ex2(x[c] - ref);
                    ps8[c & 7] += x[c];
                }
                l += ((ps8[0] + ps8[1]) + (ps8[2] + ps8[3])) + ((ps8[4] + ps8[5]) + (ps8[6] + ps8[7]));
                if (QP) {
                    mx::fake_quant32(x);
                    mx::fake_quant32(x + 32);
                }
            } else {
#pragma unroll
                for (int c = 0; c < 64; ++c) {
                    const float s_nat = x[c] * (1.0f / kLog2e);
                    x[c] = c < nvis ? act_f(a.act, s_nat) * inv_n : 0.f;
                }
            }
            // P half-row -> shared memory, K-major, 128-byte swizzle (chunk ^ row%8)
#pragma unroll
            for (int ch = 0; ch < 8; ++ch) {
                uint4 w;
                w.x = pack_bf16(x[ch * 8 + 0], x[ch * 8 + 1]);
                w.y = pack_bf16(x[ch * 8 + 2], x[ch * 8 + 3]);
                w.z = pack_bf16(x[ch * 8 + 4], x[ch * 8 + 5]);
                w.w = pack_bf16(x[ch * 8 + 6], x[ch * 8 + 7]);
                *reinterpret_cast<uint4*>(prow + ((ch ^ (r & 7)) << 4)) = w;
            }
            // value rows past the sequence end (neighbour data) must not reach P.V
            const int nvalid = nkv - j * BN;
            if (nvalid < BN) {  // same for the whole CTA
                mbar_wait(&bars->v_full[s], (j >> 1) & 1, abort_flag, a.hdr);
                if (r >= nvalid) {
                    uint8_t* vrow = smem + kOffV + s * kTile + grp * kBox + r * 128;
                    const uint4 z = make_uint4(0, 0, 0, 0);
#pragma unroll
                    for (int ch = 0; ch < 8; ++ch) *reinterpret_cast<uint4*>(vrow + ch * 16) = z;
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->p_full);
            if (!softmax && *abort_flag) { ok = false; break; }
        }
        // ------------------------------------------------------ epilogue
        if (ok && n_tiles > 0) mbar_wait(&bars->pv_done, (n_tiles - 1) & 1, abort_flag, a.hdr);
        lred[grp * 128 + r] = l;
        named_sync_softmax();
        ok = ok && !*abort_flag;
        const float l_row = l + lred[(grp ^ 1) * 128 + r];
        if (ok) {
            tc_fence_after();
            const float inv = softmax ? (l_row > 0.f ? 1.f / l_row : 0.f) : 1.f;
            __nv_bfloat16* orow = reinterpret_cast<__nv_bfloat16*>(a.out) + ((int64_t)(q0 + i) * a.H + h) * HD + c0;
#pragma unroll
            for (int c4 = 0; c4 < 2; ++c4) {
                uint32_t u[32];
                if (n_tiles > 0) {
                    tmem_ld32(tO + c4 * 32, u);
                    tmem_wait_ld();
                } else {
#pragma unroll
                    for (int t = 0; t < 32; ++t) u[t] = 0u;
                }
                if (i < nq) {
#pragma unroll
                    for (int t = 0; t < 32; t += 8) {
                        uint4 w;
                        w.x = pack_bf16(__uint_as_float(u[t + 0]) * inv, __uint_as_float(u[t + 1]) * inv);
                        w.y = pack_bf16(__uint_as_float(u[t + 2]) * inv, __uint_as_float(u[t + 3]) * inv);
                        w.z = pack_bf16(__uint_as_float(u[t + 4]) * inv, __uint_as_float(u[t + 5]) * inv);
                        w.w = pack_bf16(__uint_as_float(u[t + 6]) * inv, __uint_as_float(u[t + 7]) * inv);
                        *reinterpret_cast<uint4*>(orow + c4 * 32 + t) = w;
                    }
                }
            }
            if (softmax && grp == 0 && a.lse && i < nq)
                a.lse[(int64_t)(q0 + i) * a.H + h] =
                    l_row > 0.f ? m_used * (1.0f / kLog2e) + logf(l_row) : -CUDART_INF_F;
        }
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
    const int base = 1024 + (int)kOffTab;
    int tab_need = (p.bias_kind == JFA_BIAS_RELPOS) ? (p.max_kv_len + BM - 1) : 0;
    int smem = base + 4 * tab_need;
    if (smem > kSmemLimit) {  // window too long: read the table through L1 instead
        tab_need = 0;
        smem = base;
    }
    P.tab_cap = tab_need;
    int64_t grid = pairs_bound(p.batch, p.max_q_len, p.total_q, BM) * p.heads;
    if (grid <= 0) return cudaSuccess;
    if (grid > 0x7fffffff) return cudaErrorInvalidValue;
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
    kern<<<(unsigned)grid, kThreads, smem, st>>>(P);
    prof_end(st, quant_p ? K_TC_FWD_MXFP8 : K_TC_FWD);
    return cudaGetLastError();
}

}  // namespace jfa
