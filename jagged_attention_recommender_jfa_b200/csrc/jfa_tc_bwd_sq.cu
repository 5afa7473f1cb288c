// Tensor-core jagged attention backward for short query sequences (every
// n_q <= 64; bf16, head_dim 128): query-stationary.
//
// Target-aware cross attention and pooled attention have a few query tokens
// against a long key/value history ("GEM Training: How Meta Doubled the
// Efficiency of Its LLM-Scale Ads Foundation Model", "Challenge 1: Achieving
// High Per-GPU Utilization": asymmetric shapes make intra-kernel pipelining
// less effective).  With one key tile per CTA (the general backward) each CTA
// would see a single short query tile: its fixed costs dominate and dQ is
// added up across CTAs in fp32.  Here one CTA takes a whole (sequence, head):
// its <= 64 query rows, their dO, LSE and D stay in shared memory, the
// key/value tiles stream through a two-stage ring, dK and dV of each key tile
// are complete after that one step (no other query tile contributes) and go
// straight to memory, and dQ^T accumulates in TMEM over the key tiles and is
// written once.  No atomics, no accumulator, no finalize pass.
//
// Per key tile j (128 keys):
//   S^T  = K_j Q^T,  dP^T = V_j dO^T                   (M 128 keys, N 64 queries)
//   P^T  = exp2(S^T - LSE) / GDPA act, dS^T            (16 score warps; P^T and
//                                                       dS^T to shared memory)
//   dK_j = dS^T Q,   dV_j = P^T dO                     (M 128 keys, N 128 d, K 64)
//   dQ^T += K_j^T dS^T                                 (M 128 d, N 64 queries, K 128)
// S^T / dP^T of tile j+1 are issued as soon as the score warps have read
// those of tile j, so they run during tile j's score phase.  K and V tiles
// stream through two-stage rings (a K stage is free once dQ^T of its tile has
// run, a V stage once dP^T has).  dK and dV of a tile leave through a 32 KB
// staging tile in turn: the four score warps of a lane quarter write their
// (key row, 32 d) pieces of its 32 rows, meet on the quarter's mbarrier, and
// each warp then stores eight whole 256-byte rows (one row per half warp and
// instruction) instead of 16-byte pieces of 32 rows 1 KB apart, which the L2
// takes as half-sector writes.
// TMEM: S^T [0,64), dP^T [64,128), dK [128,256), dV [256,384), dQ^T [384,448),
// P^T (bf16 pairs, the A operand of dV) [448,480).
// Warps: 0 TMA, 1 MMA, 2..17 score: warp w reads TMEM lane quarter w % 4, and
// the four consecutive warps 2 + 4g .. 5 + 4g take queries 16 g .. 16 g + 15;
// 18, 19 stage a dense bias (one query row per lane: the 16-byte blocks that
// cover the row's keys of the tile, one bulk copy) into shared memory once
// the score warps have read the previous tile's.  Twenty warps still leave
// 96 registers per thread (five warps per SM sub-partition).
#include <math_constants.h>

#include "jfa_sm100.cuh"

namespace jfa {

using namespace sm100;

bool make_tmap_rows_heads_d(CUtensorMap* map, const void* base, int64_t rows, int heads);
bool make_tmap_rows_heads_d_box(CUtensorMap* map, const void* base, int64_t rows, int heads, int box_rows);

JFA_TRACE_DEFINE(bwdsq)

namespace {

constexpr int BQ = 64, BN = 128, HD = 128;
constexpr int kThreads = 64 + 16 * 32 + 64;
constexpr uint32_t kKBox = 128 * 128;            // [128 rows][64 bf16]
constexpr uint32_t kKTile = 2 * kKBox;           // 128 x 128 bf16
constexpr uint32_t kQBox = 64 * 128;             // [64 rows][64 bf16]
constexpr uint32_t kQTile = 2 * kQBox;           // 64 x 128 bf16
constexpr uint32_t kOffQ = 0;
constexpr uint32_t kOffDO = kOffQ + kQTile;
constexpr int kKStages = 2, kVStages = 2;
constexpr uint32_t kOffK = kOffDO + kQTile;                // K ring
constexpr uint32_t kOffV = kOffK + kKStages * kKTile;      // V ring
constexpr uint32_t kOffDST = kOffV + kVStages * kKTile;    // dS^T [128 keys][64 queries] bf16 (128-byte rows)
constexpr uint32_t kOffOut = kOffDST + 128 * 128;          // dK or dV staging [128 keys][256 bytes]
constexpr uint32_t kOffRow = kOffOut + 128 * 256; // LSE (log2) [64], D [64]
// dense bias rows of a key tile: 64 query rows x 272 bytes (the 16-byte
// blocks that cover 128 bf16 at any 2-byte alignment)
constexpr uint32_t kDRow = 272;
constexpr uint32_t kOffDense = kOffRow + 512;
constexpr uint32_t kOffBar = kOffDense + BQ * kDRow;
constexpr uint32_t kSmemBytes = kOffBar + 256 + 1024;
constexpr float kLog2e = 1.4426950408889634f;

struct Bars {
    uint64_t q_full;
    uint64_t k_full[kKStages], k_empty[kKStages];
    uint64_t v_full[kVStages], v_empty[kVStages];
    uint64_t s_full;
    uint64_t sp_free;    // 16 score warps read S^T / dP^T
    uint64_t ds_full;    // 16 score warps wrote P^T / dS^T
    uint64_t dkv_full;   // dK, dV, dQ^T of the key tile done
    uint64_t dkv_free;   // 16 score warps read dK / dV
    uint64_t rows_full;  // LSE / D staged (2 warps)
    uint64_t dense_full, dense_empty;   // dense bias rows staged (2 warps) / read (16)
    uint64_t out_full[4], out_read[4];  // per lane quarter: its staging rows written / read back (4 warps)
    uint64_t drain;
    uint32_t tmem_base;
    int abort_flag;
};
static_assert(sizeof(Bars) <= 256, "barrier block");

struct SqParams {
    CUtensorMap tm_q;    // box 64 rows
    CUtensorMap tm_do;   // box 64 rows
    CUtensorMap tm_k;    // box 128 rows
    CUtensorMap tm_v;
    AttnArgs a;
};

constexpr uint32_t kDescHi = sw128_desc_hi(1024u);
// K-major operand made of 64-column boxes `box` bytes apart: K step k = 16
// elements (32 bytes within a 128-byte row, then the next box)
__device__ __forceinline__ uint64_t kdesc(uint32_t lo, int k, uint32_t box) {
    return sw128_desc(lo + (uint32_t)(k >> 2) * (box >> 4) + (uint32_t)(k & 3) * 2u, kDescHi);
}
// MN-major operand (rows = K, 128-byte rows of the MN dimension): K step of
// 16 rows = 2048 bytes; the MN halves `box` bytes apart (LBO)
__device__ __forceinline__ uint64_t mdesc(uint32_t lo, int k) {
    return sw128_desc(lo + (uint32_t)k * 128u, kDescHi);
}

// 16 fp32 (bits) -> bf16 at columns 16 g .. +15 of row r of a 128-byte-row
// swizzled tile
__device__ __forceinline__ void store16_bf16(uint8_t* tile, int r, int g, const uint32_t (&v)[16]) {
    uint8_t* row = tile + r * 128;
#pragma unroll
    for (int u = 0; u < 2; ++u) {
        const int ch = 2 * g + u;
        uint4 w;
        w.x = pack_bf16(__uint_as_float(v[8 * u + 0]), __uint_as_float(v[8 * u + 1]));
        w.y = pack_bf16(__uint_as_float(v[8 * u + 2]), __uint_as_float(v[8 * u + 3]));
        w.z = pack_bf16(__uint_as_float(v[8 * u + 4]), __uint_as_float(v[8 * u + 5]));
        w.w = pack_bf16(__uint_as_float(v[8 * u + 6]), __uint_as_float(v[8 * u + 7]));
        *reinterpret_cast<uint4*>(row + ((ch ^ (r & 7)) << 4)) = w;
    }
}

// zero row r (128 bytes per box) of a tile made of `boxes` boxes `box` bytes apart
__device__ __forceinline__ void zero_row(uint8_t* tile, int r, int boxes, uint32_t box) {
    const uint4 z = make_uint4(0, 0, 0, 0);
    for (int b = 0; b < boxes; ++b)
#pragma unroll
        for (int ch = 0; ch < 8; ++ch) *reinterpret_cast<uint4*>(tile + b * box + r * 128 + ch * 16) = z;
}

template <int BIAS, bool SOFTMAX, bool DBIAS>
__global__ void __launch_bounds__(kThreads, 1) tc_bwd_sq_kernel(const __grid_constant__ SqParams P) {
    const AttnArgs& a = P.a;
    if ((int)blockIdx.x >= *a.item_count || a.hdr->err != 0) return;
    extern __shared__ uint8_t smem_dyn[];
    uint8_t* smem = smem_dyn + ((1024u - (smem_u32(smem_dyn) & 1023u)) & 1023u);
    Bars* bars = reinterpret_cast<Bars*>(smem + kOffBar);
    float* lse2_s = reinterpret_cast<float*>(smem + kOffRow);
    float* dd_s = lse2_s + BQ;

    const int4 it = a.items[blockIdx.x];
    const int b = it.x, h = it.y;
    const int q0 = a.q_off[b], nq = a.q_off[b + 1] - q0;
    const int k0 = a.kv_off[b], nkv = a.kv_off[b + 1] - k0;
    const int shift = nkv - nq;   // causal: key j visible from query i iff j <= i + shift
    const int kv_end = a.causal ? max(0, min(nkv, nq + shift)) : nkv;
    const int nt = (nq > 0) ? (kv_end + BN - 1) / BN : 0;   // key tiles
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        mbar_init(&bars->q_full, 1);
        for (int s = 0; s < kKStages; ++s) {
            mbar_init(&bars->k_full[s], 1);
            mbar_init(&bars->k_empty[s], 1);
        }
        for (int s = 0; s < kVStages; ++s) {
            mbar_init(&bars->v_full[s], 1);
            mbar_init(&bars->v_empty[s], 1);
        }
        mbar_init(&bars->s_full, 1);
        mbar_init(&bars->sp_free, 16);
        mbar_init(&bars->ds_full, 16);
        mbar_init(&bars->dkv_full, 1);
        mbar_init(&bars->dkv_free, 16);
        mbar_init(&bars->rows_full, 2);
        mbar_init(&bars->dense_full, 2);
        for (int q = 0; q < 4; ++q) {
            mbar_init(&bars->out_full[q], 4);
            mbar_init(&bars->out_read[q], 4);
        }
        mbar_init(&bars->dense_empty, 16);
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
        if (lane == 0 && nt > 0) {
            tma_prefetch_desc(&P.tm_q);
            tma_prefetch_desc(&P.tm_do);
            tma_prefetch_desc(&P.tm_k);
            tma_prefetch_desc(&P.tm_v);
            mbar_arrive_expect_tx(&bars->q_full, 2 * kQTile);
            tma_load_3d(smem + kOffQ, &P.tm_q, &bars->q_full, 0, h, q0);
            tma_load_3d(smem + kOffQ + kQBox, &P.tm_q, &bars->q_full, 64, h, q0);
            tma_load_3d(smem + kOffDO, &P.tm_do, &bars->q_full, 0, h, q0);
            tma_load_3d(smem + kOffDO + kQBox, &P.tm_do, &bars->q_full, 64, h, q0);
            // V(j) once dP^T(j - 2) has run, K(j) once dQ^T(j - 3) has run (the
            // order in which those complete)
            int v_issued = 0, k_issued = 0;
            for (int j = 0; j < nt; ++j) {
                const int z = k0 + j * BN;
                const int sv = j % kVStages, sk = j % kKStages;
                if (j >= kVStages &&
                    !mbar_wait(&bars->v_empty[sv], ((j / kVStages) - 1) & 1, abort_flag, a.hdr))
                    break;
                mbar_arrive_expect_tx(&bars->v_full[sv], kKTile);
                tma_load_3d(smem + kOffV + sv * kKTile, &P.tm_v, &bars->v_full[sv], 0, h, z);
                tma_load_3d(smem + kOffV + sv * kKTile + kKBox, &P.tm_v, &bars->v_full[sv], 64, h, z);
                v_issued = j + 1;
                if (j >= kKStages &&
                    !mbar_wait(&bars->k_empty[sk], ((j / kKStages) - 1) & 1, abort_flag, a.hdr))
                    break;
                mbar_arrive_expect_tx(&bars->k_full[sk], kKTile);
                tma_load_3d(smem + kOffK + sk * kKTile, &P.tm_k, &bars->k_full[sk], 0, h, z);
                tma_load_3d(smem + kOffK + sk * kKTile + kKBox, &P.tm_k, &bars->k_full[sk], 64, h, z);
                k_issued = j + 1;
                if (j + 3 < nt) {   // warm L2 for the tiles loaded three steps on
                    tma_prefetch_l2_3d(&P.tm_k, 0, h, z + 3 * BN);
                    tma_prefetch_l2_3d(&P.tm_k, 64, h, z + 3 * BN);
                    tma_prefetch_l2_3d(&P.tm_v, 0, h, z + 3 * BN);
                    tma_prefetch_l2_3d(&P.tm_v, 64, h, z + 3 * BN);
                }
            }
            mbar_wait_drain(&bars->q_full, 0, a.hdr);
            for (int j = v_issued > kVStages ? v_issued - kVStages : 0; j < v_issued; ++j)
                mbar_wait_drain(&bars->v_full[j % kVStages], (j / kVStages) & 1, a.hdr);
            for (int j = k_issued > kKStages ? k_issued - kKStages : 0; j < k_issued; ++j)
                mbar_wait_drain(&bars->k_full[j % kKStages], (j / kKStages) & 1, a.hdr);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA
        if (lane == 0 && nt > 0) {
            constexpr uint32_t id_s = idesc_bf16(128, BQ, 0, 0);     // K-major x K-major
            constexpr uint32_t id_kv = idesc_bf16(128, HD, 0, 1);    // B MN-major
            constexpr uint32_t id_q = idesc_bf16(128, BQ, 1, 1);     // A and B MN-major
            const uint32_t tS = tmem, tdP = tmem + 64, tdK = tmem + 128, tdV = tmem + 256, tdQ = tmem + 384;
            const uint32_t qK = sw128_desc_lo(sbase + kOffQ, 16u), doK = sw128_desc_lo(sbase + kOffDO, 16u);
            const uint32_t qM = sw128_desc_lo(sbase + kOffQ, kQBox), doM = sw128_desc_lo(sbase + kOffDO, kQBox);
            const uint32_t dsK = sw128_desc_lo(sbase + kOffDST, 16u);
            const uint32_t tP = tmem + 448;   // P^T: queries 16k .. 16k + 15 at columns 8k .. 8k + 7
            const uint32_t dsM = sw128_desc_lo(sbase + kOffDST, 16u);
            bool ok = mbar_wait(&bars->q_full, 0, abort_flag, a.hdr);
            auto issue_sp = [&](int j) -> bool {   // S^T, dP^T of key tile j
                const int sk = j % kKStages, sv = j % kVStages;
                if (!mbar_wait(&bars->k_full[sk], (j / kKStages) & 1, abort_flag, a.hdr)) return false;
                if (!mbar_wait(&bars->v_full[sv], (j / kVStages) & 1, abort_flag, a.hdr)) return false;
                if (j > 0 && !mbar_wait(&bars->sp_free, (j - 1) & 1, abort_flag, a.hdr)) return false;
                JFA_TRACE_EV(bwdsq, 1, j, 0);
                tc_fence_after();
                const uint32_t kK = sw128_desc_lo(sbase + kOffK + sk * kKTile, 16u);
                const uint32_t vK = sw128_desc_lo(sbase + kOffV + sv * kKTile, 16u);
#pragma unroll
                for (int k = 0; k < HD / 16; ++k)
                    mma_bf16_ss(tS, kdesc(kK, k, kKBox), kdesc(qK, k, kQBox), id_s, k > 0 ? 1u : 0u);
#pragma unroll
                for (int k = 0; k < HD / 16; ++k)
                    mma_bf16_ss(tdP, kdesc(vK, k, kKBox), kdesc(doK, k, kQBox), id_s, k > 0 ? 1u : 0u);
                mma_commit(&bars->s_full);
                mma_commit(&bars->v_empty[sv]);   // V(j) is read by dP^T(j) only
                return true;
            };
            if (ok) ok = issue_sp(0);
            for (int j = 0; ok && j < nt; ++j) {
                const int s = j % kKStages;
                if (j + 1 < nt && !issue_sp(j + 1)) { ok = false; break; }
                JFA_TRACE_EV(bwdsq, 1, j, 1);
                if (!mbar_wait(&bars->ds_full, j & 1, abort_flag, a.hdr)) { ok = false; break; }
                JFA_TRACE_EV(bwdsq, 1, j, 2);
                if (j > 0 && !mbar_wait(&bars->dkv_free, (j - 1) & 1, abort_flag, a.hdr)) { ok = false; break; }
                JFA_TRACE_EV(bwdsq, 1, j, 3);
                tc_fence_after();
                // dK = dS^T Q, dV = P^T dO: K = the 64 queries (4 steps)
#pragma unroll
                for (int k = 0; k < BQ / 16; ++k)
                    mma_bf16_ss(tdK, kdesc(dsK, k, 0), mdesc(qM, k), id_kv, k > 0 ? 1u : 0u);
#pragma unroll
                for (int k = 0; k < BQ / 16; ++k)
                    mma_bf16_ts(tdV, tP + k * 8, mdesc(doM, k), id_kv, k > 0 ? 1u : 0u);
                // dQ^T += K^T dS^T: A = K MN-major (d halves a box apart), K = 128 keys
                const uint32_t kM = sw128_desc_lo(sbase + kOffK + s * kKTile, kKBox);
#pragma unroll
                for (int k = 0; k < BN / 16; ++k)
                    mma_bf16_ss(tdQ, mdesc(kM, k), mdesc(dsM, k), id_q, (j > 0 || k > 0) ? 1u : 0u);
                mma_commit(&bars->dkv_full);
                mma_commit(&bars->k_empty[s]);
                JFA_TRACE_EV(bwdsq, 1, j, 4);
            }
            mma_commit(&bars->drain);
            mbar_wait_drain(&bars->drain, 0, a.hdr);
        }
    } else if (warp < 18) {
        // ------------------------------------------------ score warps
        auto wwait = [&](uint64_t* bar, uint32_t parity) -> bool {
            return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag, a.hdr));
        };
        const int sw = warp - 2;
        const int wq = warp & 3;               // TMEM lane quarter (a warp reaches lanes 32 (warp % 4) ..)
        const int grp = sw >> 2;               // queries 16 grp .. +15 (warps 2..5, 6..9, ...)
        const int r = wq * 32 + lane;          // key row (S^T, dK, dV) / d row (dQ^T)
        const int qc0 = grp * 16;
        const uint32_t lane_addr = (uint32_t)(wq * 32) << 16;
        const uint32_t tS = tmem + lane_addr + qc0, tdP = tmem + lane_addr + 64 + qc0;
        const uint32_t tdK = tmem + lane_addr + 128 + grp * 32, tdV = tmem + lane_addr + 256 + grp * 32;
        const uint32_t tdQ = tmem + lane_addr + 384 + qc0;
        const float sc = a.scale * kLog2e;
        const float inv_n = nkv > 0 ? 1.0f / (float)nkv : 0.f;
        const int C = (a.relpos_len - 1) >> 1;
        const float* tab = (BIAS == 1) ? reinterpret_cast<const float*>(a.bias) + (int64_t)h * a.relpos_len : nullptr;
        const __nv_bfloat16* dense = reinterpret_cast<const __nv_bfloat16*>(a.bias);
        const int64_t dense_base = (BIAS == 2) ? a.dense_off[b] + (int64_t)h * nq * nkv : 0;
        // staged bias: query row q's keys of a tile start at element
        // (row start index) mod 8 of its row buffer
        const uintptr_t dense_e0 = reinterpret_cast<uintptr_t>(dense + dense_base) >> 1;
        bool ok = nt > 0;
        // LSE (log2 units) and D of the <= 64 queries: two warps stage them
        if (ok && sw < 2) {
            const int qi = sw * 32 + lane;
            float l2 = CUDART_INF_F, dv = 0.f;
            if (qi < nq && SOFTMAX) {
                l2 = a.lse[(int64_t)(q0 + qi) * a.H + h] * kLog2e;
                dv = a.dterm[(int64_t)(q0 + qi) * a.H + h];
            }
            lse2_s[qi] = l2;
            dd_s[qi] = dv;
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->rows_full);
        }
        if (ok) ok = wwait(&bars->rows_full, 0);
        // query rows past the sequence end (neighbour data) must not reach dK /
        // dV: zero them in Q and dO once they have landed
        if (ok) ok = wwait(&bars->q_full, 0);
        if (ok && grp == 0 && r < BQ && r >= nq) {
            zero_row(smem + kOffQ, r, 2, kQBox);
            zero_row(smem + kOffDO, r, 2, kQBox);
        }
        for (int j = 0; ok && j < nt; ++j) {
            const int s = j % kKStages;
            const int jk = j * BN + r;          // key index within the sequence
            const bool jvalid = jk < nkv;
            const bool tr = warp == 2 && lane == 0;
            if (tr) JFA_TRACE_EV(bwdsq, 2, j, 0);
            if (!wwait(&bars->s_full, j & 1)) { ok = false; break; }
            if (tr) JFA_TRACE_EV(bwdsq, 2, j, 1);
            if (BIAS == 2 && !wwait(&bars->dense_full, j & 1)) { ok = false; break; }
            if (tr) JFA_TRACE_EV(bwdsq, 2, j, 2);
            tc_fence_after();
            uint32_t u[16], g[16];
            tmem_ld16(tS, u);
            tmem_ld16(tdP, g);
            tmem_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->sp_free);   // S^T / dP^T of tile j+1 may start
            // key rows past the sequence end (neighbour data) must not reach
            // dQ^T = K^T dS^T; S^T of this tile has completed
            if (grp == 0 && !jvalid) zero_row(smem + kOffK + s * kKTile, r, 2, kKBox);
            const int imin_vis = a.causal ? jk - shift : 0;   // queries i >= imin_vis see key jk
            const bool all_vis = jvalid && qc0 + 15 < nq && qc0 >= imin_vis;
            const bool none_vis = !jvalid || qc0 >= nq || qc0 + 15 < imin_vis;
            if (none_vis) {
#pragma unroll
                for (int v = 0; v < 16; ++v) u[v] = 0u, g[v] = 0u;
            } else {
                float x[16];
                if (BIAS == 1) {
#pragma unroll
                    for (int v = 0; v < 16; ++v)
                        x[v] = fmaf(__uint_as_float(u[v]), sc,
                                    __ldg(tab + min(max(qc0 + v - jk, -C), C) + C) * kLog2e);
                } else if (BIAS == 2) {
                    __nv_bfloat16 bh[16];
#pragma unroll
                    for (int v = 0; v < 16; ++v) {
                        const int qq = min(qc0 + v, nq - 1);
                        const int e = (int)((dense_e0 + (uintptr_t)qq * (uintptr_t)nkv) & 7u) + r;
                        bh[v] = reinterpret_cast<const __nv_bfloat16*>(smem + kOffDense + qq * kDRow)[e];
                    }
#pragma unroll
                    for (int v = 0; v < 16; ++v)
                        x[v] = fmaf(__uint_as_float(u[v]), sc, __bfloat162float(bh[v]) * kLog2e);
                } else {
#pragma unroll
                    for (int v = 0; v < 16; ++v) x[v] = __uint_as_float(u[v]) * sc;
                }
                if (SOFTMAX) {
#pragma unroll
                    for (int v = 0; v < 16; ++v) {
                        const float p = ex2(x[v] - lse2_s[qc0 + v]);
                        u[v] = __float_as_uint(p);
                        g[v] = __float_as_uint(p * (__uint_as_float(g[v]) - dd_s[qc0 + v]));
                    }
                } else {
#pragma unroll
                    for (int v = 0; v < 16; ++v) {
                        const float sn = x[v] * (1.0f / kLog2e);
                        const float sg = sigmoid_fast(act_arg(a.act, sn));
                        u[v] = __float_as_uint(sn * sg * inv_n);
                        g[v] = __float_as_uint(__uint_as_float(g[v]) * act_grad_from(a.act, sn, sg) * inv_n);
                    }
                }
                if (!all_vis) {
#pragma unroll
                    for (int v = 0; v < 16; ++v) {
                        const int qi = qc0 + v;
                        const bool vis = jvalid && qi < nq && qi >= imin_vis;
                        u[v] = vis ? u[v] : 0u;
                        g[v] = vis ? g[v] : 0u;
                    }
                }
                if (DBIAS && BIAS == 2 && jvalid) {
                    __nv_bfloat16* dcol = reinterpret_cast<__nv_bfloat16*>(a.dbias) + dense_base + jk;
#pragma unroll
                    for (int v = 0; v < 16; ++v)
                        if (qc0 + v < nq) dcol[(int64_t)(qc0 + v) * nkv] = __float2bfloat16_rn(__uint_as_float(g[v]));
                }
                if (DBIAS && BIAS == 1) {
                    float* dtab = reinterpret_cast<float*>(a.dbias) + (int64_t)h * a.relpos_len;
#pragma unroll
                    for (int v = 0; v < 16; ++v)
                        if (g[v] != 0u) atomicAdd(dtab + min(max(qc0 + v - jk, -C), C) + C, __uint_as_float(g[v]));
                }
            }
            if (BIAS == 2) {   // this tile's staged bias rows are read
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars->dense_empty);
            }
            // P^T to TMEM and dS^T to shared memory; the MMAs of the previous tile
            // that read them have completed (this warp saw their commit below)
            {   // P^T (bf16 pairs): queries qc0 .. qc0 + 15 at columns 448 + 8 grp ..
                uint32_t pw[8];
#pragma unroll
                for (int t = 0; t < 8; ++t) pw[t] = pack_bf16(__uint_as_float(u[2 * t]), __uint_as_float(u[2 * t + 1]));
                tmem_st8(tmem + lane_addr + 448 + grp * 8, pw);
            }
            store16_bf16(smem + kOffDST, r, grp, g);
            fence_proxy_async_smem();
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->ds_full);
            if (tr) JFA_TRACE_EV(bwdsq, 2, j, 3);
            // dK and dV of this key tile are complete: write them out
            if (!wwait(&bars->dkv_full, j & 1)) { ok = false; break; }
            if (tr) JFA_TRACE_EV(bwdsq, 2, j, 4);
            tc_fence_after();
            uint32_t uk[32], uv[32];
            tmem_ld32(tdK, uk);
            tmem_ld32(tdV, uv);
            tmem_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->dkv_free);
            if (tr) JFA_TRACE_EV(bwdsq, 2, j, 5);
            // dK (scaled) then dV through the staging tile, one 8 KB part per lane
            // quarter: the four warps of a quarter hold its 32 key rows (32 d each)
            // and meet on their own barrier.  Local row lr, 16-byte chunk c of its
            // 256 bytes at chunk c ^ (lr % 16) (a warp's rows then fall on
            // distinct banks in each quarter warp); warp grp stores rows
            // 8 grp .. 8 grp + 7 of the part.
            uint8_t* stg = smem + kOffOut + wq * (32 * 256);
            const int lr = lane;
#pragma unroll
            for (int tsr = 0; tsr < 2; ++tsr) {
                const int use = 2 * j + tsr;
                if (use > 0 && !wwait(&bars->out_read[wq], (use - 1) & 1)) { ok = false; break; }
                const uint32_t (&vals)[32] = tsr ? uv : uk;
                const float mul = tsr ? 1.0f : a.scale;
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    uint4 w4;
                    w4.x = pack_bf16(__uint_as_float(vals[8 * q + 0]) * mul, __uint_as_float(vals[8 * q + 1]) * mul);
                    w4.y = pack_bf16(__uint_as_float(vals[8 * q + 2]) * mul, __uint_as_float(vals[8 * q + 3]) * mul);
                    w4.z = pack_bf16(__uint_as_float(vals[8 * q + 4]) * mul, __uint_as_float(vals[8 * q + 5]) * mul);
                    w4.w = pack_bf16(__uint_as_float(vals[8 * q + 6]) * mul, __uint_as_float(vals[8 * q + 7]) * mul);
                    const int c = 4 * grp + q;
                    *reinterpret_cast<uint4*>(stg + lr * 256 + ((c ^ (lr & 15)) << 4)) = w4;
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars->out_full[wq]);
                if (!wwait(&bars->out_full[wq], use & 1)) { ok = false; break; }
                __nv_bfloat16* base = reinterpret_cast<__nv_bfloat16*>(tsr ? a.dv : a.dk);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int row = 8 * grp + 2 * i + (lane >> 4), c = lane & 15;   // local row
                    const uint4 w4 = *reinterpret_cast<const uint4*>(stg + row * 256 + ((c ^ (row & 15)) << 4));
                    const int key = j * BN + wq * 32 + row;
                    if (key < nkv)
                        *reinterpret_cast<uint4*>(base + ((int64_t)(k0 + key) * a.H + h) * HD + c * 8) = w4;
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars->out_read[wq]);
            }
            if (!ok) break;
            if (tr) JFA_TRACE_EV(bwdsq, 2, j, 6);
        }
        // dQ = scale * (dQ^T)^T: d row r, queries qc0 .. +15; every dQ^T MMA
        // retired with the last dkv_full
        if (ok && !*abort_flag) {
            tc_fence_after();
            uint32_t uq[16];
            tmem_ld16(tdQ, uq);
            tmem_wait_ld();
            __nv_bfloat16* dq = reinterpret_cast<__nv_bfloat16*>(a.dq) + ((int64_t)q0 * a.H + h) * HD + r;
#pragma unroll
            for (int v = 0; v < 16; ++v)
                if (qc0 + v < nq) dq[(int64_t)(qc0 + v) * a.H * HD] = __float2bfloat16_rn(__uint_as_float(uq[v]) * a.scale);
        }
        // a sequence without keys (or whose rows see none): zero dQ
        if (nq > 0 && nt == 0 && grp == 0) {
            __nv_bfloat16* dq = reinterpret_cast<__nv_bfloat16*>(a.dq) + ((int64_t)q0 * a.H + h) * HD + r;
            for (int qi = 0; qi < nq; ++qi) dq[(int64_t)qi * a.H * HD] = __float2bfloat16_rn(0.f);
        }
    } else if (BIAS == 2 && nt > 0) {
        // ------------------------------------------------ dense bias stagers
        const int row = (warp - 18) * 32 + lane;   // query row of this lane
        const bool has_row = row < nq;
        const __nv_bfloat16* dense = reinterpret_cast<const __nv_bfloat16*>(a.bias);
        const int64_t row_off = has_row ? a.dense_off[b] + ((int64_t)h * nq + row) * nkv : 0;
        uint8_t* dst = smem + kOffDense + row * kDRow;
        int staged = 0;
        for (int j = 0; j < nt; ++j) {
            // the buffer is free once the score warps have read tile j - 1
            if (j > 0 && !__all_sync(0xffffffffu, mbar_wait(&bars->dense_empty, (j - 1) & 1, abort_flag, a.hdr)))
                break;
            const int jc = j * BN;
            const int nk = min(BN, nkv - jc);   // keys of this tile (>= 1)
            // the 16-byte blocks covering the row's nk bias values: every block
            // holds a value of the bias tensor, so the copy stays in its allocation
            uintptr_t src = 0;
            uint32_t bytes = 0;
            if (has_row) {
                const uintptr_t first = reinterpret_cast<uintptr_t>(dense + row_off + jc);
                src = first & ~static_cast<uintptr_t>(15);
                bytes = (uint32_t)(((first + 2u * (uint32_t)nk + 15u) & ~static_cast<uintptr_t>(15)) - src);
            }
            const uint32_t total = __reduce_add_sync(0xffffffffu, bytes);
            if (lane == 0) mbar_arrive_expect_tx(&bars->dense_full, total);
            __syncwarp();
            if (bytes) bulk_load(dst, reinterpret_cast<const void*>(src), bytes, &bars->dense_full);
            if (has_row && j + 1 < nt) {   // warm L2 for the next tile's rows
                prefetch_l2(dense + row_off + jc + BN);
                prefetch_l2(dense + row_off + min(jc + 2 * BN, nkv) - 1);
            }
            staged = j + 1;
        }
        // never leave the CTA with copies in flight
        if (staged > 0 && lane == 0) mbar_wait_drain(&bars->dense_full, (staged - 1) & 1, a.hdr);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// dK = dV = 0 for the key rows of sequences without queries (they have no
// work item); one warp per (row, head), 128 elements each.
__global__ void __launch_bounds__(256) sq_zero_kv(const int32_t* __restrict__ q_off,
                                                  const int32_t* __restrict__ kv_off, int B, int H,
                                                  const WsHeader* hdr, __nv_bfloat16* __restrict__ dk,
                                                  __nv_bfloat16* __restrict__ dv) {
    if (hdr->err != 0) return;
    const int lane = threadIdx.x & 31, wpb = blockDim.x >> 5;
    for (int b = blockIdx.x; b < B; b += gridDim.x) {
        if (q_off[b + 1] != q_off[b]) continue;
        const int64_t r0 = (int64_t)kv_off[b] * H, r1 = (int64_t)kv_off[b + 1] * H;
        for (int64_t row = r0 + (threadIdx.x >> 5); row < r1; row += wpb) {
            reinterpret_cast<uint2*>(dk + row * HD)[lane] = make_uint2(0u, 0u);
            reinterpret_cast<uint2*>(dv + row * HD)[lane] = make_uint2(0u, 0u);
        }
    }
}

}  // namespace

constexpr int kSmemLimitSq = 232448;

// The query-stationary backward: items are (sequence, head) pairs (the
// forward's schedule at 256-row query blocks; every n_q <= 64).  D comes from
// the caller's pre-pass; dK / dV rows of keys that no query sees are zeroed
// by that pre-pass too.
cudaError_t tc_backward_sq_launch(const jfa_problem& p, const AttnArgs& a, cudaStream_t st) {
    SqParams P{};
    if (!make_tmap_rows_heads_d_box(&P.tm_q, a.q, p.total_q, p.heads, BQ) ||
        !make_tmap_rows_heads_d_box(&P.tm_do, a.dout, p.total_q, p.heads, BQ) ||
        !make_tmap_rows_heads_d(&P.tm_k, a.k, p.total_kv, p.heads) ||
        !make_tmap_rows_heads_d(&P.tm_v, a.v, p.total_kv, p.heads))
        return cudaErrorInvalidValue;
    P.a = a;
    const int bias = p.bias_kind == JFA_BIAS_RELPOS ? 1 : (p.bias_kind == JFA_BIAS_DENSE_JAGGED ? 2 : 0);
    const bool sm = a.act == JFA_ACT_SOFTMAX, db = a.dbias != nullptr;
    void (*kern)(SqParams) = nullptr;
    if (bias == 0) kern = sm ? tc_bwd_sq_kernel<0, true, false> : tc_bwd_sq_kernel<0, false, false>;
    else if (bias == 1)
        kern = db ? (sm ? tc_bwd_sq_kernel<1, true, true> : tc_bwd_sq_kernel<1, false, true>)
                  : (sm ? tc_bwd_sq_kernel<1, true, false> : tc_bwd_sq_kernel<1, false, false>);
    else
        kern = db ? (sm ? tc_bwd_sq_kernel<2, true, true> : tc_bwd_sq_kernel<2, false, true>)
                  : (sm ? tc_bwd_sq_kernel<2, true, false> : tc_bwd_sq_kernel<2, false, false>);
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemLimitSq);
    if (e != cudaSuccess) return e;
    static_assert(kSmemBytes <= (uint32_t)kSmemLimitSq, "shared memory");
    if (p.batch > 0) {
        const int zb = p.batch < 148 * 4 ? p.batch : 148 * 4;
        sq_zero_kv<<<zb, 256, 0, st>>>(a.q_off, a.kv_off, p.batch, p.heads, a.hdr,
                                       reinterpret_cast<__nv_bfloat16*>(a.dk),
                                       reinterpret_cast<__nv_bfloat16*>(a.dv));
    }
    const int64_t grid = (int64_t)p.batch * p.heads;
    if (grid <= 0) return cudaGetLastError();
    if (grid > 0x7fffffff) return cudaErrorInvalidValue;
    prof_begin(st);
    kern<<<(unsigned)grid, kThreads, kSmemBytes, st>>>(P);
    prof_end(st, K_TC_BWD_SQ);
    return cudaGetLastError();
}

}  // namespace jfa
