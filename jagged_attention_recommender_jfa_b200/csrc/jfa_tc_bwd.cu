// Tensor-core (tcgen05) jagged attention backward for bf16, head_dim 128.
//
// Removing padding exposes backward accumulation as a bottleneck ("Meta GEM
// Training Efficiency: Why LLM-Scale Recommenders Need a Different Stack",
// section "Bottleneck move 1").  Three kernels:
//
//   tc_bwd_pre       D[t,h] = sum_d dO*O (softmax) with a warp-shuffle row
//                    reduction; zeroes the fp32 dQ accumulator rows.
//   tc_bwd_kernel    persistent, one CTA per SM, taking (sequence, head,
//                    128-key tile) work items of the key-tile schedule from a
//                    counter.  K and V of the tile stay in shared memory; the
//                    query tiles that can see the keys stream through (Q and
//                    dO in a three-buffer ring):
//                      S^T  = K Q^T,  dP^T = V dO^T           (TMEM, fp32)
//                      P^T  = exp2(S^T - LSE), dS^T = P^T (dP^T - D)
//                             (or GDPA: act(S)/n_kv, dP act'(S)/n_kv)
//                             P^T (bf16) back to TMEM over S^T, dS^T (bf16)
//                             to shared memory
//                      dK  += dS^T Q                         (TMEM)
//                      dV  += P^T dO    (A operand from TMEM)
//                      dQ^T = K^T dS^T over the dP^T columns, read out by
//                             the score warps and added to the fp32
//                             accumulator with coalesced reductions (a warp
//                             covers 32 consecutive d of one query row)
//                    dK and dV run over the tile's two query halves, the
//                    first while the score warps form the second; once the
//                    whole dS^T is formed, dQ^T of tile t goes ahead of the
//                    second halves, then S^T, dP^T of tile t+1 follow:
//                    dQ^T(t) is read out while those run, and Q / dO
//                    come from a three-buffer ring that fetches Q(t+1) two
//                    tiles ahead and dO(t+1) once dK(t) has retired (both
//                    warmed in L2 a tile earlier).
//   tc_bwd_dq_finalize  dQ = bf16(scale * accumulator).
//
// Warp roles: warp 0 TMA, warp 1 MMA, warps 2..17 score warps in four groups
// of four; a thread of group g owns one key row and its 16-query chunks g
// and g + 4 (for the dQ^T read-out: one d row and queries 32g .. 32g + 31).
// The backward needs no row reduction (LSE and D are given), so the chunks
// never talk.
// TMEM columns: dV [0,128), dK [128,256), S^T / P^T [256,384),
// dP^T / dQ^T [384,512).
#include <math_constants.h>

#include "jfa_sm100.cuh"

namespace jfa {

using namespace sm100;

bool make_tmap_rows_heads_d(CUtensorMap* map, const void* base, int64_t rows, int heads);

JFA_TRACE_DEFINE(bwd)

namespace {

constexpr int BM = 128, BN = 128, HD = 128;
constexpr int NG = 4;                 // column groups: a score thread owns one 32-column chunk
constexpr int kThreads = 64 + NG * 128;
constexpr uint32_t kBox = 128 * 128;
constexpr uint32_t kTile = 2 * kBox;
constexpr uint32_t kOffK = 0;
constexpr uint32_t kOffV = kOffK + kTile;
// Q and dO of the query tiles share a ring of three tile buffers, filled in
// the order Q(0), dO(0), Q(1), dO(1), ...: load n (Q(n/2) for even n, dO(n/2)
// for odd n) goes to buffer n % 3, once load n - 3 has been consumed -- so
// Q(t) is fetched as soon as dV(t-2) has retired and dO(t) once dK(t-1) has.
constexpr uint32_t kOffQD = kOffV + kTile;        // three buffers
constexpr uint32_t kOffDST = kOffQD + 3 * kTile;
constexpr uint32_t kOffBar = kOffDST + kTile;     // 196608
constexpr uint32_t kOffRow = kOffBar + 512;       // lse2[2][128], D[2][128] (double-buffered)
// Relative-position bias window of a query tile, 2 stages: 272 entries of the
// prepared table (entry t = table entries t .. t+3, log2(e)-scaled) from the
// smallest index the tile's (query, key) pairs need; a thread reads its run
// of 16 entries as four float4s, consecutive key rows consecutive entries.
constexpr int kWin = 272;
constexpr uint32_t kWinBytes = kWin * 16;          // 4352
constexpr uint32_t kOffWin = kOffRow + 2048;
// Relative-position bias gradient of a query tile, 2 buffers: the 255
// diagonals i - j of a 128 x 128 tile, entry e = (i - qb0) - (j - j0) + 127,
// summed in shared memory and added to the table once per tile.
constexpr int kDbWin = 256;
constexpr uint32_t kOffDb = kOffWin + 2 * kWinBytes;
constexpr uint32_t kOffEnd = kOffDb + 2 * kDbWin * 4;
constexpr float kLog2e = 1.4426950408889634f;

struct Bars {
    uint64_t k_full, v_full;   // the item's K / V tile loaded
    uint64_t k_free, v_free;   // the item's last MMA reading K (dQ^T) / V (dP^T) retired
    uint64_t buf_full[3], buf_empty[3];   // the Q / dO ring
    uint64_t s_full;
    uint64_t ds_half;       // 16 score warps: queries 0..63 of the tile done
    uint64_t ds_full;       // 16 score warps
    uint64_t dq_full;
    uint64_t dq_empty;      // 16 score warps
    uint64_t rows_full[2];  // LSE / D of a query tile staged (4 warps of group 0)
    uint64_t rows_free[2];  // ... and read by every score warp (16)
    uint64_t bias_full[2];  // bias window of a query tile loaded
    uint64_t db_done[2];    // 16 score warps: their bias-gradient sums of a tile are in
    uint64_t db_free[2];    // the tile's flusher warp added the buffer to the table and cleared it
    uint64_t fin;           // the item's MMAs have retired
    uint64_t dkv_free;      // 16 score warps: the item's dK / dV read out of TMEM
    uint64_t item_full[2];  // the TMA warp published the next work item
    uint64_t item_empty[2]; // ... and the MMA thread and 16 score warps read it
    uint64_t drain;
    uint32_t tmem_base;
    int abort_flag;
    int item_ring[2];
};
static_assert(sizeof(Bars) <= 512, "barrier block");

struct BwdParams {
    CUtensorMap tm_q;
    CUtensorMap tm_k;
    CUtensorMap tm_v;
    CUtensorMap tm_do;
    AttnArgs a;
};

// First entry of the bias window of the query tile starting at query qb0
// (keys j0 ..): the smallest table index a pair of the tile can need, clamped
// so that the window lies inside the prepared table.
__device__ __forceinline__ int bias_window_start(int qb0, int j0, int C, int stride) {
    return min(max(qb0 - j0 - (BN - 1) + C, 0), stride - kWin);
}

// Shared-memory operand descriptors of a 128 x 128 bf16 tile (two 64-column
// 128B-swizzled boxes) at K step k (16 elements), from the tile's precomputed
// lower word: K-major (rows = M or N, 64 K per box row) steps 32 B within a
// row and kBox to the next box; MN-major (rows = K) steps 16 rows = 2048 B,
// its two 64-element halves kBox apart (LBO).
constexpr uint32_t kDescHi = sw128_desc_hi(1024u);
__device__ __forceinline__ uint32_t kmajor_lo(uint32_t tile_base) { return sw128_desc_lo(tile_base, 16u); }
__device__ __forceinline__ uint32_t mnmajor_lo(uint32_t tile_base) { return sw128_desc_lo(tile_base, kBox); }
__device__ __forceinline__ uint64_t kmajor_desc(uint32_t lo, int k) {
    return sw128_desc(lo + (uint32_t)(k >> 2) * (kBox >> 4) + (uint32_t)(k & 3) * 2u, kDescHi);
}
__device__ __forceinline__ uint64_t mnmajor_desc(uint32_t lo, int k) {
    return sw128_desc(lo + (uint32_t)k * 128u, kDescHi);
}

// Stores 16 fp32 values (bit patterns) as bf16: columns 16*c16 .. +15 of row r
// of a K-major 128B-swizzled tile.
__device__ __forceinline__ void store_half_chunk_bits(uint8_t* tile, int r, int c16, const uint32_t (&v)[16]) {
    uint8_t* row = tile + (c16 >> 2) * kBox + r * 128;
#pragma unroll
    for (int u = 0; u < 2; ++u) {
        const int ch = (c16 & 3) * 2 + u;
        uint4 w;
        w.x = pack_bf16(__uint_as_float(v[8 * u + 0]), __uint_as_float(v[8 * u + 1]));
        w.y = pack_bf16(__uint_as_float(v[8 * u + 2]), __uint_as_float(v[8 * u + 3]));
        w.z = pack_bf16(__uint_as_float(v[8 * u + 4]), __uint_as_float(v[8 * u + 5]));
        w.w = pack_bf16(__uint_as_float(v[8 * u + 6]), __uint_as_float(v[8 * u + 7]));
        *reinterpret_cast<uint4*>(row + ((ch ^ (r & 7)) << 4)) = w;
    }
}

__device__ __forceinline__ void zero_row(uint8_t* tile, int r) {
    const uint4 z = make_uint4(0, 0, 0, 0);
#pragma unroll
    for (int ch = 0; ch < 8; ++ch) {
        *reinterpret_cast<uint4*>(tile + r * 128 + ch * 16) = z;
        *reinterpret_cast<uint4*>(tile + kBox + r * 128 + ch * 16) = z;
    }
}

// One work item of the key-tile schedule: (sequence, head, 128-key tile) and
// the query tiles that see its keys, from the first key's first query to the
// last key's last (all of them without a causal rule or window).
struct BItem {
    int b, h, j0, q0, nq, k0, nkv, shift, i_start, nt;
};

template <bool WINDOW>
__device__ __forceinline__ BItem load_bitem(const AttnArgs& a, int idx) {
    const int4 it = a.items[idx];
    BItem w;
    w.b = it.x;
    w.h = it.y;
    w.j0 = it.z * BN;
    w.q0 = a.q_off[w.b];
    w.nq = a.q_off[w.b + 1] - w.q0;
    w.k0 = a.kv_off[w.b];
    w.nkv = a.kv_off[w.b + 1] - w.k0;
    w.shift = w.nkv - w.nq;   // causal: key j visible from query i iff j <= i + shift
    w.i_start = WINDOW ? vis_query_lo(a.causal, a.window, w.j0, w.nq, w.nkv)
                       : (a.causal ? max(0, w.j0 - w.shift) : 0);
    const int i_end = WINDOW ? vis_query_hi(a.window, min(w.j0 + BN, w.nkv) - 1, w.nq, w.nkv) + 1 : w.nq;
    w.nt = i_end > w.i_start ? (i_end - w.i_start + BM - 1) / BM : 0;
    return w;
}

// BIAS: 0 none, 1 relative-position, 2 dense jagged.  SOFTMAX: softmax (true)
// or GDPA.  DBIAS: also the bias gradient -- ds of every pair written to the
// dense bias gradient, or summed along the diagonals of each tile in shared
// memory and added to the relative-position table gradient by one warp
// (score warp t % 16 for tile t, at the start of tile t + 1).  WINDOW: a
// sliding window (the query range of a key tile ends before the sequence).
//
// Persistent: one CTA per SM takes work items from the key-tile schedule --
// its block index first, then the next unclaimed one from a counter in the
// workspace header (claimed by the TMA warp when it starts the item and
// passed to the other roles through a two-entry ring in shared memory), so
// that the items of one (sequence, head) still run at about the same time.
// The barrier phases count tiles and items of the CTA, not of the item; an
// item's K and V are loaded once its predecessor's MMAs have retired, and
// its first dK / dV MMA waits until the score warps have read the
// predecessor's dK / dV out of TMEM, so that the next item's first loads and
// S^T, dP^T overlap the previous item's read-out and stores.
template <int BIAS, bool SOFTMAX, bool DBIAS, bool WINDOW>
__global__ void __launch_bounds__(kThreads, 1) tc_bwd_kernel(const __grid_constant__ BwdParams P) {
    const AttnArgs& a = P.a;
    const int n_items = *a.item_count;
    if ((int)blockIdx.x >= n_items || a.hdr->err != 0) return;
    extern __shared__ uint8_t smem_dyn[];
    uint8_t* smem = smem_dyn + ((1024u - (smem_u32(smem_dyn) & 1023u)) & 1023u);
    Bars* bars = reinterpret_cast<Bars*>(smem + kOffBar);
    float* lse2_s = reinterpret_cast<float*>(smem + kOffRow);  // [2][128]
    float* dd_s = lse2_s + 256;                                 // [2][128]
    const int G = gridDim.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    constexpr bool softmax = SOFTMAX;

    if (threadIdx.x == 0) {
        mbar_init(&bars->k_full, 1);
        mbar_init(&bars->v_full, 1);
        mbar_init(&bars->k_free, 1);
        mbar_init(&bars->v_free, 1);
        for (int s3 = 0; s3 < 3; ++s3) {
            mbar_init(&bars->buf_full[s3], 1);
            mbar_init(&bars->buf_empty[s3], 1);
        }
        for (int s2 = 0; s2 < 2; ++s2) {
            mbar_init(&bars->rows_full[s2], 4);
            mbar_init(&bars->rows_free[s2], NG * 4);
            mbar_init(&bars->bias_full[s2], 1);
            mbar_init(&bars->item_full[s2], 1);
            mbar_init(&bars->item_empty[s2], 1 + NG * 4);
        }
        mbar_init(&bars->s_full, 1);
        mbar_init(&bars->ds_half, NG * 4);
        mbar_init(&bars->ds_full, NG * 4);
        mbar_init(&bars->dq_full, 1);
        mbar_init(&bars->dq_empty, NG * 4);
        mbar_init(&bars->fin, 1);
        mbar_init(&bars->dkv_free, NG * 4);
        mbar_init(&bars->drain, 1);
        for (int s2 = 0; s2 < 2; ++s2) {
            mbar_init(&bars->db_done[s2], NG * 4);
            mbar_init(&bars->db_free[s2], 1);
        }
        bars->abort_flag = 0;
        fence_barrier_init();
    }
    constexpr bool kDbRel = DBIAS && BIAS == 1, kDbDense = DBIAS && BIAS == 2;
    float* db_win = reinterpret_cast<float*>(smem + kOffDb);   // [2][kDbWin]
    if (kDbRel)
        for (int e = threadIdx.x; e < 2 * kDbWin; e += blockDim.x) db_win[e] = 0.f;
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
    volatile int* item_ring = bars->item_ring;

    if (warp == 0) {
        // ------------------------------------------------------------ TMA
        // Q(t+1) is loaded once dK += dS^T Q(t) has retired; dO(t+2) into
        // the buffer of dO(t) once dV += P^T dO(t) has
        if (lane == 0) {
            tma_prefetch_desc(&P.tm_q);
            tma_prefetch_desc(&P.tm_k);
            tma_prefetch_desc(&P.tm_v);
            tma_prefetch_desc(&P.tm_do);
            int issued = 0, kf = 0, gtile = 0;   // ring loads, items with tiles, tiles of the CTA
            bool ok = true;
            for (int k = 0; ok; ++k) {
                int idx = k == 0 ? (int)blockIdx.x : G + atomicAdd(&a.hdr->kv_queue, 1);
                if (idx >= n_items) idx = -1;
                const int slot = k & 1;
                if (k >= 2 && !mbar_wait(&bars->item_empty[slot], ((k >> 1) - 1) & 1, abort_flag, a.hdr)) break;
                item_ring[slot] = idx;
                mbar_arrive(&bars->item_full[slot]);   // release: the entry is visible to the waiters
                if (idx < 0) break;
                const BItem w = load_bitem<WINDOW>(a, idx);
                if (w.nt == 0) continue;
                if (kf > 0) {
                    // warm L2 with the item's K, V and first Q, dO while the
                    // previous item finishes
                    const int zk = w.k0 + w.j0, zq = w.q0 + w.i_start;
                    tma_prefetch_l2_3d(&P.tm_k, 0, w.h, zk);
                    tma_prefetch_l2_3d(&P.tm_k, 64, w.h, zk);
                    tma_prefetch_l2_3d(&P.tm_v, 0, w.h, zk);
                    tma_prefetch_l2_3d(&P.tm_v, 64, w.h, zk);
                    tma_prefetch_l2_3d(&P.tm_q, 0, w.h, zq);
                    tma_prefetch_l2_3d(&P.tm_q, 64, w.h, zq);
                    tma_prefetch_l2_3d(&P.tm_do, 0, w.h, zq);
                    tma_prefetch_l2_3d(&P.tm_do, 64, w.h, zq);
                }
                // V replaces the previous item's once its last dP^T has retired,
                // K once its last dQ^T has (both ahead of the item's last dK, dV)
                if (kf > 0 && !mbar_wait(&bars->v_free, (kf - 1) & 1, abort_flag, a.hdr)) break;
                mbar_arrive_expect_tx(&bars->v_full, kTile);
                tma_load_3d(smem + kOffV, &P.tm_v, &bars->v_full, 0, w.h, w.k0 + w.j0);
                tma_load_3d(smem + kOffV + kBox, &P.tm_v, &bars->v_full, 64, w.h, w.k0 + w.j0);
                if (kf > 0 && !mbar_wait(&bars->k_free, (kf - 1) & 1, abort_flag, a.hdr)) break;
                mbar_arrive_expect_tx(&bars->k_full, kTile);
                tma_load_3d(smem + kOffK, &P.tm_k, &bars->k_full, 0, w.h, w.k0 + w.j0);
                tma_load_3d(smem + kOffK + kBox, &P.tm_k, &bars->k_full, 64, w.h, w.k0 + w.j0);
                ++kf;
                // load n of the item is ring load N = issued: Q(n/2) (with a
                // relative-position bias also the tile's bias window) or dO(n/2);
                // the window's stage (gt & 1) was last read for tile gt-2, whose
                // score phase ended before dV(gt-2), which frees the buffer that
                // Q(gt) goes to
                for (int n = 0; n < 2 * w.nt; ++n) {
                    const int N = issued, bf = N % 3, use = N / 3, t = n >> 1, gt = gtile + t;
                    if (use > 0 && !mbar_wait(&bars->buf_empty[bf], (use - 1) & 1, abort_flag, a.hdr)) {
                        ok = false;
                        break;
                    }
                    JFA_TRACE_EV(bwd, 0, gt, n & 1);
                    const int z = w.q0 + w.i_start + t * BM;
                    uint8_t* dst = smem + kOffQD + bf * kTile;
                    const CUtensorMap* map = (n & 1) ? &P.tm_do : &P.tm_q;
                    mbar_arrive_expect_tx(&bars->buf_full[bf], kTile);
                    tma_load_3d(dst, map, &bars->buf_full[bf], 0, w.h, z);
                    tma_load_3d(dst + kBox, map, &bars->buf_full[bf], 64, w.h, z);
                    if ((n & 1) == 0 && t + 1 < w.nt) {  // warm L2 for the next tile's Q and dO
                        tma_prefetch_l2_3d(&P.tm_q, 0, w.h, z + BM);
                        tma_prefetch_l2_3d(&P.tm_q, 64, w.h, z + BM);
                        tma_prefetch_l2_3d(&P.tm_do, 0, w.h, z + BM);
                        tma_prefetch_l2_3d(&P.tm_do, 64, w.h, z + BM);
                    }
                    if (BIAS == 1 && (n & 1) == 0) {
                        const int C = (a.relpos_len - 1) >> 1;
                        const int w0 = bias_window_start(w.i_start + t * BM, w.j0, C, a.bias4_stride);
                        const float* src = a.bias4 + 4 * ((int64_t)w.h * a.bias4_stride + w0);
                        mbar_arrive_expect_tx(&bars->bias_full[gt & 1], kWinBytes);
                        bulk_load(smem + kOffWin + (gt & 1) * kWinBytes, src, kWinBytes, &bars->bias_full[gt & 1]);
                    }
                    issued = N + 1;
                }
                gtile += w.nt;
            }
            // never leave the CTA with copies in flight
            if (kf > 0) {
                mbar_wait_drain(&bars->v_full, (kf - 1) & 1, a.hdr);
                mbar_wait_drain(&bars->k_full, (kf - 1) & 1, a.hdr);
            }
            for (int n = issued > 3 ? issued - 3 : 0; n < issued; ++n)
                mbar_wait_drain(&bars->buf_full[n % 3], (n / 3) & 1, a.hdr);
            if (BIAS == 1) {
                const int nq_loads = (issued + 1) / 2;   // Q loads, one bias window each
                for (int gt = nq_loads > 2 ? nq_loads - 2 : 0; gt < nq_loads; ++gt)
                    mbar_wait_drain(&bars->bias_full[gt & 1], (gt >> 1) & 1, a.hdr);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA
        if (lane == 0) {
            constexpr uint32_t idesc_nt = idesc_bf16(128, 128, 0, 0);  // K-major x K-major
            constexpr uint32_t idesc_nn = idesc_bf16(128, 128, 0, 1);  // B MN-major
            constexpr uint32_t idesc_tn = idesc_bf16(128, 128, 1, 1);  // A and B MN-major
            const uint32_t tdV = tmem, tdK = tmem + 128, tS = tmem + 256, tdP = tmem + 384;
            // descriptor lower words of every operand tile, computed once
            const uint32_t kK = kmajor_lo(sbase + kOffK), kM = mnmajor_lo(sbase + kOffK);
            const uint32_t vK = kmajor_lo(sbase + kOffV);
            // the ring's buffers, K-major (S^T, dP^T) and MN-major (dK, dV) views
            auto ringK = [&](int bf) { return kmajor_lo(sbase + kOffQD + (uint32_t)bf * kTile); };
            auto ringM = [&](int bf) { return mnmajor_lo(sbase + kOffQD + (uint32_t)bf * kTile); };
            const uint32_t dsK = kmajor_lo(sbase + kOffDST), dsM = mnmajor_lo(sbase + kOffDST);
            // gt: tile of the CTA (its Q is ring load 2 gt, its dO load 2 gt + 1)
            auto issue_s = [&](int gt) {  // S^T = K Q^T
                const uint32_t q = ringK((2 * gt) % 3);
#pragma unroll
                for (int k = 0; k < HD / 16; ++k)
                    mma_bf16_ss(tS, kmajor_desc(kK, k), kmajor_desc(q, k), idesc_nt, k > 0 ? 1u : 0u);
            };
            auto issue_dp = [&](int gt) {  // dP^T = V dO^T
                const uint32_t d = ringK((2 * gt + 1) % 3);
#pragma unroll
                for (int k = 0; k < HD / 16; ++k)
                    mma_bf16_ss(tdP, kmajor_desc(vK, k), kmajor_desc(d, k), idesc_nt, k > 0 ? 1u : 0u);
            };
            auto wait_load = [&](int n) { return mbar_wait(&bars->buf_full[n % 3], (n / 3) & 1, abort_flag, a.hdr); };
            // dK += dS^T Q and dV += P^T dO run over the tile's query halves:
            // the first four K steps (queries 0..63) as soon as the score
            // warps have formed that half, the rest after the whole tile; the
            // item's first tile (t = 0) starts the accumulators
            auto issue_dk = [&](int gt, int t, int k_lo) {  // A = dS^T K-major in smem, B = Q MN-major
                const uint32_t qM = ringM((2 * gt) % 3);
#pragma unroll
                for (int k = k_lo; k < k_lo + 4; ++k)
                    mma_bf16_ss(tdK, kmajor_desc(dsK, k), mnmajor_desc(qM, k), idesc_nn,
                                (t > 0 || k > 0) ? 1u : 0u);
            };
            auto issue_dv = [&](int gt, int t, int k_lo) {  // A = P^T from TMEM: queries 16k.. at column 16k
                const uint32_t d = ringM((2 * gt + 1) % 3);
#pragma unroll
                for (int k = k_lo; k < k_lo + 4; ++k)
                    mma_bf16_ts(tdV, tS + 16 * k, mnmajor_desc(d, k), idesc_nn, (t > 0 || k > 0) ? 1u : 0u);
            };
            bool ok = true;
            int kf = 0, gtile = 0;
            for (int k = 0; ok; ++k) {
                const int slot = k & 1;
                if (!mbar_wait(&bars->item_full[slot], (k >> 1) & 1, abort_flag, a.hdr)) { ok = false; break; }
                const int idx = item_ring[slot];
                mbar_arrive(&bars->item_empty[slot]);
                if (idx < 0) break;
                const BItem w = load_bitem<WINDOW>(a, idx);
                if (w.nt == 0) continue;
                // dP^T of the first tile overwrites the previous item's last dQ^T
                ok = mbar_wait(&bars->k_full, kf & 1, abort_flag, a.hdr) && wait_load(2 * gtile);
                if (!ok) break;
                tc_fence_after();
                issue_s(gtile);
                ok = mbar_wait(&bars->v_full, kf & 1, abort_flag, a.hdr) && wait_load(2 * gtile + 1) &&
                     (gtile == 0 || mbar_wait(&bars->dq_empty, (gtile - 1) & 1, abort_flag, a.hdr));
                if (!ok) break;
                tc_fence_after();
                issue_dp(gtile);
                if (w.nt == 1) mma_commit(&bars->v_free);
                mma_commit(&bars->s_full);
                for (int t = 0; ok && t < w.nt; ++t) {
                    const int gt = gtile + t;
                    if (!mbar_wait(&bars->ds_half, gt & 1, abort_flag, a.hdr)) { ok = false; break; }
                    // the item's first dK / dV overwrite the previous item's,
                    // which the score warps must have read out
                    if (t == 0 && kf > 0 && !mbar_wait(&bars->dkv_free, (kf - 1) & 1, abort_flag, a.hdr)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    issue_dk(gt, t, 0);
                    issue_dv(gt, t, 0);
                    if (!mbar_wait(&bars->ds_full, gt & 1, abort_flag, a.hdr)) { ok = false; break; }
                    JFA_TRACE_EV(bwd, 1, gt, 0);
                    tc_fence_after();
                    // dQ^T = K^T dS^T over the dP^T columns (A = K, B = dS^T, both
                    // MN-major), ahead of the second halves of dK and dV, so that its
                    // read-out and reductions start while those run
#pragma unroll
                    for (int k = 0; k < BN / 16; ++k)
                        mma_bf16_ss(tdP, mnmajor_desc(kM, k), mnmajor_desc(dsM, k), idesc_tn, k > 0 ? 1u : 0u);
                    mma_commit(&bars->dq_full);
                    if (t + 1 == w.nt) mma_commit(&bars->k_free);   // the item's last use of K
                    issue_dk(gt, t, 4);
                    mma_commit(&bars->buf_empty[(2 * gt) % 3]);
                    issue_dv(gt, t, 4);
                    mma_commit(&bars->buf_empty[(2 * gt + 1) % 3]);
                    JFA_TRACE_EV(bwd, 1, gt, 1);
                    if (t + 1 < w.nt) {
                        // S^T(t+1) overwrites P^T(t): issued after dV, which reads it
                        if (!wait_load(2 * gt + 2)) { ok = false; break; }
                        JFA_TRACE_EV(bwd, 1, gt, 2);
                        tc_fence_after();
                        issue_s(gt + 1);
                        if (!wait_load(2 * gt + 3) || !mbar_wait(&bars->dq_empty, gt & 1, abort_flag, a.hdr)) {
                            ok = false;
                            break;
                        }
                        JFA_TRACE_EV(bwd, 1, gt, 3);
                        tc_fence_after();
                        issue_dp(gt + 1);
                        if (t + 2 == w.nt) mma_commit(&bars->v_free);   // the item's last use of V
                        mma_commit(&bars->s_full);
                    }
                }
                if (!ok) break;
                mma_commit(&bars->fin);
                gtile += w.nt;
                ++kf;
            }
            mma_commit(&bars->drain);
            mbar_wait_drain(&bars->drain, 0, a.hdr);
        }
    } else {
        // ------------------------------------------------ score warps
        // waits taken by a whole warp: the result is made warp-uniform, so that a
        // timed-out wait ends the warp's loop on every lane together
        auto wwait = [&](uint64_t* bar, uint32_t parity) -> bool {
            return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag, a.hdr));
        };
        const int wq = warp & 3;                 // TMEM lane quarter
        const int grp = (warp - 2) >> 2;         // 32-column chunk of the row
        const int r = wq * 32 + lane;            // key row (S^T, dV, dK) / d row (dQ^T)
        const uint32_t lane_addr = (uint32_t)(wq * 32) << 16;
        const uint32_t cofs = (uint32_t)grp * 32;
        const uint32_t tdV = tmem + lane_addr + cofs, tdK = tmem + lane_addr + 128 + cofs;
        const uint32_t tS = tmem + lane_addr + 256, tdP = tmem + lane_addr + 384 + cofs;
        const float sc = a.scale * kLog2e;
        const int C = (a.relpos_len - 1) >> 1;
        const __nv_bfloat16* dense = reinterpret_cast<const __nv_bfloat16*>(a.bias);
        const int sw = warp - 2;
        bool ok = true;
        int kf = 0, gtile = 0;
        for (int kk = 0; ok; ++kk) {
            const int slot = kk & 1;
            if (!wwait(&bars->item_full[slot], (kk >> 1) & 1)) { ok = false; break; }
            const int idx = item_ring[slot];
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->item_empty[slot]);
            if (idx < 0) break;
            const BItem w = load_bitem<WINDOW>(a, idx);
            const int h = w.h, j0 = w.j0, q0 = w.q0, nq = w.nq, nkv = w.nkv;
            const int i_start = w.i_start, nt = w.nt;
            const int j = j0 + r;                    // key index within the sequence
            const bool jvalid = j < nkv;
            const int k0 = w.k0;
            // this thread's 32 columns of its dK and dV rows
            auto kv32 = [&]() {
                return ((reinterpret_cast<uintptr_t>(a.dk) | reinterpret_cast<uintptr_t>(a.dv)) & 31) == 0;
            };
            auto grad_rows = [&](__nv_bfloat16*& dkrow, __nv_bfloat16*& dvrow) {
                const int64_t o = ((int64_t)(k0 + j) * a.H + h) * HD + cofs;
                dkrow = reinterpret_cast<__nv_bfloat16*>(a.dk) + o;
                dvrow = reinterpret_cast<__nv_bfloat16*>(a.dv) + o;
            };
            if (nt == 0) {
                // no query sees these keys: zero gradients, no tensor-core work
                if (jvalid && !*abort_flag) {
                    __nv_bfloat16 *dkrow, *dvrow;
                    grad_rows(dkrow, dvrow);
                    uint32_t z[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e) z[e] = 0u;
#pragma unroll
                    for (int e = 0; e < 32; e += 16) {
                        store_bf16x16(dkrow + e, z, 1.0f, kv32());
                        store_bf16x16(dvrow + e, z, 1.0f, kv32());
                    }
                }
                continue;
            }
            const float inv_n = nkv > 0 ? 1.0f / (float)nkv : 0.f;
            const int64_t dense_base = (BIAS == 2) ? a.dense_off[w.b] + (int64_t)h * nq * nkv : 0;
            // LSE (log2 units) and D of a query tile: group 0 stages them into one
            // of two buffers a tile ahead (rows_full), every warp releases the
            // buffer after reading it (rows_free); buffers by the CTA's tile gt
            auto fetch_rowstats = [&](int t, float& l2, float& dv) {
                const int qi = i_start + t * BM + r;
                l2 = CUDART_INF_F;
                dv = 0.f;
                if (qi < nq && softmax) {
                    l2 = a.lse[(int64_t)(q0 + qi) * a.H + h] * kLog2e;
                    dv = a.dterm[(int64_t)(q0 + qi) * a.H + h];
                }
            };
            auto stage_rowstats = [&](int gt, float l2, float dv) -> bool {
                // the buffer's readers (tile gt - 2) have all released it
                if (gt >= 2 && !wwait(&bars->rows_free[gt & 1], ((gt - 2) >> 1) & 1)) return false;
                lse2_s[(gt & 1) * 128 + r] = l2;
                dd_s[(gt & 1) * 128 + r] = dv;
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars->rows_full[gt & 1]);
                return true;
            };
            // the first query tile's dense bias block (read once from HBM) into L1
            // and L2 while the K / V / Q / dO loads are in flight: query row r,
            // keys j0 .. j0 + 127 span at most three lines
            if (BIAS == 2 && grp < 3 && i_start + r < nq)
                prefetch_l1(dense + dense_base + (int64_t)(i_start + r) * nkv + min(j0 + 63 * grp + grp / 2, nkv - 1));
            if (grp == 0) {
                float l2, dv;
                fetch_rowstats(0, l2, dv);
                if (!stage_rowstats(gtile, l2, dv)) { ok = false; break; }
            }
            // relative-position bias gradient: the flusher of tile gt (score warp
            // gt % 16) adds the tile's diagonal sums to the table and clears them
            float* dtab = kDbRel ? reinterpret_cast<float*>(a.dbias) + (int64_t)h * a.relpos_len : nullptr;
            auto flush_db = [&](int tt, int gt) -> bool {
                if (!wwait(&bars->db_done[gt & 1], (gt >> 1) & 1)) return false;
                float* dw = db_win + (gt & 1) * kDbWin;
                const int d0 = (i_start + tt * BM) - j0 - (BN - 1);   // diagonal i - j of entry 0
                for (int e = lane; e < 2 * BN - 1; e += 32) {
                    const float val = dw[e];
                    if (val != 0.f) atomicAdd(dtab + (min(max(d0 + e, -C), C) + C), val);
                    dw[e] = 0.f;
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars->db_free[gt & 1]);
                return true;
            };
            const int tslot = (warp == 2 && lane == 0) ? 2 : ((warp == kThreads / 32 - 1 && lane == 0) ? 3 : -1);
#define SC_EV(ev)                                      \
    do {                                               \
        if (tslot >= 0) JFA_TRACE_EV(bwd, tslot, gt, ev); \
    } while (0)
            // A failed (timed-out) wait sets the CTA's abort flag; every later wait
            // then returns at once, and the warps leave the loop independently
            // (the loop has no CTA-wide barrier).
            for (int t = 0; t < nt; ++t) {
                const int gt = gtile + t;
                SC_EV(0);
                const int qb0 = i_start + t * BM;    // query index of the tile's row 0
                const int buf = gt & 1;
                float nl2 = CUDART_INF_F, ndv = 0.f;
                if (grp == 0 && t + 1 < nt) fetch_rowstats(t + 1, nl2, ndv);
                // the next query tile's dense bias block (read once from HBM) into
                // L2: query row r, keys j0 .. j0 + 127 span at most three lines
                if (BIAS == 2 && grp < 3 && t + 1 < nt && qb0 + BM + r < nq)
                    prefetch_l2(dense + dense_base + (int64_t)(qb0 + BM + r) * nkv + min(j0 + 63 * grp + grp / 2, nkv - 1));
                if (!wwait(&bars->s_full, gt & 1)) { ok = false; break; }
                SC_EV(1);
                tc_fence_after();
                // key rows past the sequence end (neighbour data) must not reach
                // dQ^T = K^T dS^T; S^T = K Q^T of the item's first tile has completed
                if (t == 0 && grp == 0 && !jvalid) zero_row(smem + kOffK, r);
                if (!wwait(&bars->rows_full[buf], (gt >> 1) & 1)) { ok = false; break; }
                if (BIAS == 1 && !wwait(&bars->bias_full[buf], (gt >> 1) & 1)) { ok = false; break; }
                if (kDbRel) {
                    // the previous tile's sums are complete once S^T of this tile exists
                    if (t >= 1 && sw == (gt - 1) % (NG * 4) && !flush_db(t - 1, gt - 1)) { ok = false; break; }
                    // this tile's buffer was flushed after tile gt - 2
                    if (gt >= 2 && !wwait(&bars->db_free[buf], ((gt >> 1) - 1) & 1)) { ok = false; break; }
                }
                SC_EV(2);
                // bias(qc0 + v, j) = table[qc0 - j + C + v]: window entries
                // qc0 - j + C - w0 + 4q hold table[... + 4q + 0..3]
                const int wbase = BIAS == 1 ? (qb0 - j + C) - bias_window_start(qb0, j0, C, a.bias4_stride) : 0;
                const float4* win = reinterpret_cast<const float4*>(smem + kOffWin + buf * kWinBytes);
                // queries imin_vis .. imax_vis see key j
                const int imin_vis = WINDOW ? vis_query_lo(a.causal, a.window, j, nq, nkv)
                                            : (a.causal ? j - (nkv - nq) : 0);
                const int imax_vis = WINDOW ? vis_query_hi(a.window, j, nq, nkv) : nq - 1;
                // one 16-column part: scores u (TMEM bits) -> P in place, dP g -> dS in place
                auto process = [&](uint32_t (&u)[16], uint32_t (&g)[16], int c16) {
                    const int qc0 = qb0 + c16 * 16;      // query index of the part's column 0
                    const bool all_vis = jvalid && (qc0 + 15 <= imax_vis) && (qc0 >= imin_vis);
                    const bool none_vis = !jvalid || qc0 > imax_vis || (qc0 + 15 < imin_vis);
                    if (none_vis) {
    #pragma unroll
                        for (int v = 0; v < 16; ++v) u[v] = 0u, g[v] = 0u;
                        return;
                    }
                    float x[16];
                    const float2 sc2 = make_float2(sc, sc);
                    if (BIAS == 1) {
                        float bb[16];
                        const int s0 = qc0 - j + C;                       // table index of bias(qc0, j)
                        const int wr = wbase + c16 * 16;                  // its window entry
                        if (s0 >= 0 && s0 + 15 <= 2 * C && wr >= 0 && wr + 12 < kWin) {
    #pragma unroll
                            for (int q = 0; q < 4; ++q) {
                                const float4 t4 = win[wr + 4 * q];
                                bb[4 * q] = t4.x, bb[4 * q + 1] = t4.y, bb[4 * q + 2] = t4.z, bb[4 * q + 3] = t4.w;
                            }
                        } else {
    #pragma unroll
                            // log2(e)-scaled table of head h: entry t at tab4[4 t]
                            const float* tab4 = a.bias4 + (int64_t)h * 4 * a.bias4_stride;
                            for (int v = 0; v < 16; ++v) bb[v] = __ldg(tab4 + 4 * min(max(s0 + v, 0), 2 * C));
                        }
    #pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            const float2 r2 = fma2(make_float2(__uint_as_float(u[2 * e]), __uint_as_float(u[2 * e + 1])),
                                                   sc2, make_float2(bb[2 * e], bb[2 * e + 1]));
                            x[2 * e] = r2.x, x[2 * e + 1] = r2.y;
                        }
                    } else if (BIAS == 2) {
                        // bias(qc0 + v, j): sixteen unconditional loads (rows and key
                        // clamped into the sequence, invalid entries masked below), so
                        // that they are all in flight together
                        const __nv_bfloat16* col = dense + dense_base + min(j, nkv - 1);
                        __nv_bfloat16 bh[16];
    #pragma unroll
                        for (int v = 0; v < 16; ++v) bh[v] = col[(int64_t)min(qc0 + v, nq - 1) * nkv];
    #pragma unroll
                        for (int v = 0; v < 16; ++v)
                            x[v] = fmaf(__uint_as_float(u[v]), sc, __bfloat162float(bh[v]) * kLog2e);
                    } else {
    #pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            const float2 r2 = mul2(make_float2(__uint_as_float(u[2 * e]), __uint_as_float(u[2 * e + 1])), sc2);
                            x[2 * e] = r2.x, x[2 * e + 1] = r2.y;
                        }
                    }
                    if (SOFTMAX) {
                        // P = 2^(x - lse), dS = P (dP - D); lse and D of the 16 query
                        // columns are broadcast reads of the staged row statistics
                        const float4* l4 = reinterpret_cast<const float4*>(lse2_s + buf * 128 + c16 * 16);
                        const float4* d4 = reinterpret_cast<const float4*>(dd_s + buf * 128 + c16 * 16);
    #pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            const float4 L = l4[q], D = d4[q];
                            const float2 y0 = sub2(make_float2(x[4 * q], x[4 * q + 1]), make_float2(L.x, L.y));
                            const float2 y1 = sub2(make_float2(x[4 * q + 2], x[4 * q + 3]), make_float2(L.z, L.w));
                            const float2 p0 = make_float2(ex2(y0.x), ex2(y0.y));
                            const float2 p1 = make_float2(ex2(y1.x), ex2(y1.y));
                            const float2 t0 = sub2(make_float2(__uint_as_float(g[4 * q]), __uint_as_float(g[4 * q + 1])),
                                                   make_float2(D.x, D.y));
                            const float2 t1 = sub2(make_float2(__uint_as_float(g[4 * q + 2]), __uint_as_float(g[4 * q + 3])),
                                                   make_float2(D.z, D.w));
                            const float2 d0 = mul2(p0, t0), d1 = mul2(p1, t1);
                            u[4 * q] = __float_as_uint(p0.x), u[4 * q + 1] = __float_as_uint(p0.y);
                            u[4 * q + 2] = __float_as_uint(p1.x), u[4 * q + 3] = __float_as_uint(p1.y);
                            g[4 * q] = __float_as_uint(d0.x), g[4 * q + 1] = __float_as_uint(d0.y);
                            g[4 * q + 2] = __float_as_uint(d1.x), g[4 * q + 3] = __float_as_uint(d1.y);
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
                            const bool vis = jvalid && qi <= imax_vis && qi >= imin_vis;
                            u[v] = vis ? u[v] : 0u;
                            g[v] = vis ? g[v] : 0u;
                        }
                    }
                    // bias gradient: d beta(i, j) = ds_ij (g, masked pairs 0)
                    if (kDbDense && jvalid) {
                        __nv_bfloat16* col = reinterpret_cast<__nv_bfloat16*>(a.dbias) + dense_base + j;
    #pragma unroll
                        for (int v = 0; v < 16; ++v)
                            if (qc0 + v < nq) col[(int64_t)(qc0 + v) * nkv] = __float2bfloat16_rn(__uint_as_float(g[v]));
                    }
                    if (kDbRel) {
                        // diagonal entry (qc0 + v - qb0) - r + 127; for a fixed v the
                        // lanes (consecutive r) hit consecutive entries
                        float* dw = db_win + buf * kDbWin + (c16 * 16 - r + (BN - 1));
    #pragma unroll
                        for (int v = 0; v < 16; ++v) atomicAdd(dw + v, __uint_as_float(g[v]));
                    }
                };
                // Two 16-column halves: half hh of group grp is query chunk
                // c16 = 4 hh + grp (columns 16 c16 ..), so that every group's first
                // half together covers queries 0..63 and dK / dV can start on them.
                // P^T (bf16 pairs) goes back to TMEM over the first 8 of the
                // chunk's own S^T columns (no other warp reads them), dS^T to
                // shared memory for dK and dQ^T.  Query rows past the sequence end
                // (neighbour data) must not reach dV / dK: S^T and dP^T of the
                // tile have completed, so Q and dO may be edited.
                if (qb0 + r >= nq) {
                    if (grp == 0) zero_row(smem + kOffQD + ((2 * gt) % 3) * kTile, r);
                    else if (grp == 1) zero_row(smem + kOffQD + ((2 * gt + 1) % 3) * kTile, r);
                }
    #pragma unroll 1
                for (int hh = 0; hh < 2; ++hh) {
                    uint32_t u[16], g[16];
                    const int c16 = hh * 4 + grp;
                    tmem_ld16(tS + c16 * 16, u);
                    tmem_ld16(tdP - cofs + c16 * 16, g);
                    tmem_wait_ld();
                    process(u, g, c16);
                    store_half_chunk_bits(smem + kOffDST, r, c16, g);
                    uint32_t pk[8];
    #pragma unroll
                    for (int e = 0; e < 8; ++e) pk[e] = pack_bf16(__uint_as_float(u[2 * e]), __uint_as_float(u[2 * e + 1]));
                    tmem_st8(tS + c16 * 16, pk);
                    if (hh == 0) {
                        tmem_wait_st();
                        fence_proxy_async_smem();
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&bars->ds_half);
                    }
                }
                tmem_wait_st();
                SC_EV(3);
                fence_proxy_async_smem();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(&bars->rows_free[buf]);
                    mbar_arrive(&bars->ds_full);
                    if (kDbRel) mbar_arrive(&bars->db_done[buf]);
                }
                // LSE / D of tile t+1 into the other buffer, whose readers (tile
                // gt-1) have all released it
                if (grp == 0 && t + 1 < nt && !stage_rowstats(gt + 1, nl2, ndv)) {
                    ok = false;
                    break;
                }
                // dQ^T of this query tile: TMEM lane r = d, column c = query qb0 + 32 grp + c
                if (!wwait(&bars->dq_full, gt & 1)) { ok = false; break; }
                SC_EV(4);
                tc_fence_after();
                uint32_t dqv[32];
                tmem_ld32(tdP, dqv);
                tmem_wait_ld();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars->dq_empty);  // columns free for dP^T of t+1
                SC_EV(5);
                {
                    const int qc = qb0 + grp * 32;
                    float* dst = a.dq_acc + ((int64_t)(q0 + qc) * a.H + h) * HD + r;
                    const int64_t stride = (int64_t)a.H * HD;
                    const int nvalid = min(32, nq - qc);   // warp-uniform
    #pragma unroll
                    for (int c = 0; c < 32; ++c)
                        if (c < nvalid) atomicAdd(dst + c * stride, __uint_as_float(dqv[c]));
                }
                SC_EV(6);
            }
#undef SC_EV
            if (!ok) break;
            if (kDbRel && sw == (gtile + nt - 1) % (NG * 4) && !flush_db(nt - 1, gtile + nt - 1)) { ok = false; break; }
            // -------------------------------------------------- item epilogue
            if (!wwait(&bars->fin, kf & 1)) { ok = false; break; }
            tc_fence_after();
            uint32_t uk[32], uv[32];
            tmem_ld32(tdK, uk);
            tmem_ld32(tdV, uv);
            tmem_wait_ld();
            // dK / dV columns free for the next item's first MMAs
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->dkv_free);
            if (jvalid && !*abort_flag) {
                __nv_bfloat16 *dkrow, *dvrow;
                grad_rows(dkrow, dvrow);
#pragma unroll
                for (int e = 0; e < 32; e += 16) {
                    store_bf16x16(dkrow + e, uk + e, a.scale, kv32());
                    store_bf16x16(dvrow + e, uv + e, 1.0f, kv32());
                }
            }
            gtile += nt;
            ++kf;
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// D = rowsum(dO * O) (softmax only) and zeroed dQ accumulator; one warp per
// (token, head) row of 128 elements.
__global__ void __launch_bounds__(256) tc_bwd_pre(const __nv_bfloat16* __restrict__ out,
                                                  const __nv_bfloat16* __restrict__ dout,
                                                  float* __restrict__ dterm, float* __restrict__ dq_acc,
                                                  int64_t rows, int softmax) {
    const int64_t row = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= rows) return;
    reinterpret_cast<float4*>(dq_acc + row * HD)[lane] = make_float4(0.f, 0.f, 0.f, 0.f);
    if (!softmax) return;
    const uint2 uo = reinterpret_cast<const uint2*>(out + row * HD)[lane];
    const uint2 ug = reinterpret_cast<const uint2*>(dout + row * HD)[lane];
    const float2 o0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&uo.x));
    const float2 o1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&uo.y));
    const float2 g0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&ug.x));
    const float2 g1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&ug.y));
    float acc = o0.x * g0.x + o0.y * g0.y + o1.x * g1.x + o1.y * g1.y;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (lane == 0) dterm[row] = acc;
}

// dQ = bf16(scale * accumulator); 8 elements per thread.
__global__ void __launch_bounds__(256) tc_bwd_dq_finalize(const float* __restrict__ dq_acc,
                                                          __nv_bfloat16* __restrict__ dq,
                                                          int64_t n8, float scale) {
    const int64_t t = (int64_t)blockIdx.x * 256 + threadIdx.x;
    if (t >= n8) return;
    const float4 x = reinterpret_cast<const float4*>(dq_acc)[2 * t];
    const float4 y = reinterpret_cast<const float4*>(dq_acc)[2 * t + 1];
    uint4 w;
    w.x = pack_bf16(x.x * scale, x.y * scale);
    w.y = pack_bf16(x.z * scale, x.w * scale);
    w.z = pack_bf16(y.x * scale, y.y * scale);
    w.w = pack_bf16(y.z * scale, y.w * scale);
    reinterpret_cast<uint4*>(dq)[t] = w;
}

}  // namespace



// D = rowsum(dO * O) and the zeroed dQ accumulator
cudaError_t tc_bwd_pre_launch(const jfa_problem& p, const AttnArgs& a, cudaStream_t st) {
    const int64_t rows = p.total_q * p.heads;
    if (rows > 0) {
        prof_begin(st);
        tc_bwd_pre<<<(unsigned)((rows + 7) / 8), 256, 0, st>>>(
            reinterpret_cast<const __nv_bfloat16*>(a.out), reinterpret_cast<const __nv_bfloat16*>(a.dout),
            a.dterm, a.dq_acc, rows, a.act == JFA_ACT_SOFTMAX ? 1 : 0);
        prof_end(st, K_TC_BWD_PRE);
    }
    return cudaGetLastError();
}

cudaError_t tc_backward_launch(const jfa_problem& p, const AttnArgs& a, const AttnArgs& kv,
                               cudaStream_t st) {
    const int64_t rows = p.total_q * p.heads;
    {
        cudaError_t e0 = tc_bwd_pre_launch(p, a, st);
        if (e0 != cudaSuccess) return e0;
    }
    BwdParams P{};
    if (!make_tmap_rows_heads_d(&P.tm_q, a.q, p.total_q, p.heads) ||
        !make_tmap_rows_heads_d(&P.tm_k, a.k, p.total_kv, p.heads) ||
        !make_tmap_rows_heads_d(&P.tm_v, a.v, p.total_kv, p.heads) ||
        !make_tmap_rows_heads_d(&P.tm_do, a.dout, p.total_q, p.heads))
        return cudaErrorInvalidValue;
    P.a = kv;
    const int smem = 1024 + (int)kOffEnd;
    const int bias = p.bias_kind == JFA_BIAS_RELPOS ? 1 : (p.bias_kind == JFA_BIAS_DENSE_JAGGED ? 2 : 0);
    const bool sm = a.act == JFA_ACT_SOFTMAX;
    const bool db = a.dbias != nullptr;
    void (*kern)(BwdParams) = nullptr;
    if (a.window > 0) {
        if (bias == 0) kern = sm ? tc_bwd_kernel<0, true, false, true> : tc_bwd_kernel<0, false, false, true>;
        else if (bias == 1)
            kern = db ? (sm ? tc_bwd_kernel<1, true, true, true> : tc_bwd_kernel<1, false, true, true>)
                      : (sm ? tc_bwd_kernel<1, true, false, true> : tc_bwd_kernel<1, false, false, true>);
        else
            kern = db ? (sm ? tc_bwd_kernel<2, true, true, true> : tc_bwd_kernel<2, false, true, true>)
                      : (sm ? tc_bwd_kernel<2, true, false, true> : tc_bwd_kernel<2, false, false, true>);
    } else {
        if (bias == 0) kern = sm ? tc_bwd_kernel<0, true, false, false> : tc_bwd_kernel<0, false, false, false>;
        else if (bias == 1)
            kern = db ? (sm ? tc_bwd_kernel<1, true, true, false> : tc_bwd_kernel<1, false, true, false>)
                      : (sm ? tc_bwd_kernel<1, true, false, false> : tc_bwd_kernel<1, false, false, false>);
        else
            kern = db ? (sm ? tc_bwd_kernel<2, true, true, false> : tc_bwd_kernel<2, false, true, false>)
                      : (sm ? tc_bwd_kernel<2, true, false, false> : tc_bwd_kernel<2, false, false, false>);
    }
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    // persistent: one CTA per SM (at most one per work item)
    int64_t grid = pairs_bound(p.batch, p.max_kv_len, p.total_kv, BN) * p.heads;
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (grid > sms) grid = sms;
    if (grid > 0) {
        prof_begin(st);
        kern<<<(unsigned)grid, kThreads, smem, st>>>(P);
        prof_end(st, K_TC_BWD);
    }
    const int64_t n8 = rows * HD / 8;
    if (n8 > 0) {
        prof_begin(st);
        tc_bwd_dq_finalize<<<(unsigned)((n8 + 255) / 256), 256, 0, st>>>(
            a.dq_acc, reinterpret_cast<__nv_bfloat16*>(a.dq), n8, a.scale);
        prof_end(st, K_TC_DQ_FINALIZE);
    }
    return cudaGetLastError();
}

}  // namespace jfa
