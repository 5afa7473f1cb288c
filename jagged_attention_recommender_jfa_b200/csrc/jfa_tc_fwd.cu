// Tensor-core (tcgen05) jagged attention forward for bf16, head_dim 128.
//
// Attention runs directly on the packed jagged buffers ("Meta GEM Training
// Efficiency: Why LLM-Scale Recommenders Need a Different Stack", section
// "Bottleneck move 1"): a work item is (sequence, head, 256-row query block),
// taken from the longest-first schedule.  The block is two 128-row query
// tiles held in slots A and B (the CTA's odd items swap which slot holds the
// upper rows) that share one stream of 128-row key/value tiles (a
// two-stage ring fetched by TMA); rows of a key tile past the sequence end
// belong to the neighbouring sequence and are masked out of the scores (and
// zeroed in the value tile) before they can contribute.
//
// Warp roles (576 threads, persistent: one CTA per SM walks its share of the
// work list):
//   warps 0..7  softmax / activation and epilogue of tile A, warps 8..15 of
//               tile B; warp w owns TMEM lanes 32*(w%4) .. +31 and one half
//               (64 columns) of each of those rows: the two warps that share
//               rows sit on the same SM sub-partition and exchange their
//               partial row maxima through shared memory and a two-arrival
//               mbarrier
//   warp 16     TMEM allocator and MMA issuer (one thread)
//   warp 17     TMA producer (one thread)
//
// Per key tile j, tile T in {A, B}:
//   S_T = Q_T K_j^T                  (tcgen05, 128x128x128, fp32 in TMEM)
//   softmax warps of T: scale + bias + mask and the row maximum (the biased
//   scores go back to TMEM over S), then the online softmax in the log2
//   domain (or GDPA act(s)/n_kv); P (bf16) written back to TMEM, each half of
//   the row over the first half of its own S columns (keys 0..63 to columns
//   0..31, keys 64..127 to columns 64..95)
//   O_T += P_T V_j                   (tcgen05, A = P from TMEM, B = V MN-major)
// The tensor core alternates between the tiles: while the softmax warps of
// one tile work, it runs P.V and the next Q K^T of the other; a slot whose
// rows end one key tile before the other's starts its next item during that
// last key tile.  The rescale of
// O by exp2(m_old - m_new) is lazy: it happens only when a row's running
// maximum grows by more than 8 (a factor 256), otherwise the old maximum stays
// the reference; the final O / l is exact either way.
//
// TMEM: S_A [0,128), S_B [128,256), O_A [256,384), O_B [384,512).  The
// warps of a tile never wait on each other except for the pairwise maximum
// exchange.
#include <math_constants.h>

#include "jfa_sm100.cuh"

namespace jfa {

using namespace sm100;

JFA_TRACE_DEFINE(fwd)

namespace {

constexpr int BM = 128, BN = 128, HD = 128;
constexpr int kBlockRows = 2 * BM;          // query rows per work item (tiles A and B)
constexpr int kMmaWarp = 16, kTmaWarp = 17;
constexpr int kThreads = 32 * 18;
constexpr int CW = 64;                      // columns of a key tile per softmax thread
constexpr uint32_t kBox = 128 * 128;        // bytes of one [128 rows][64 bf16] box
constexpr uint32_t kTile = 2 * kBox;        // one 128 x 128 bf16 tile (two boxes)
constexpr uint32_t kOffQ = 0;                    // Q_A, Q_B
constexpr uint32_t kOffK = kOffQ + 2 * kTile;    // 2 stages
constexpr uint32_t kOffV = kOffK + 2 * kTile;    // 2 stages
// Relative-position bias window of a key tile, 2 stages: 384 entries of the
// prepared table (entry t = table entries t .. t+3, log2(e)-scaled) starting
// at w0, so that a thread's run of 128 entries is read as 16-byte float4s;
// consecutive rows read consecutive entries, which keeps a quarter-warp's
// reads on distinct banks.
constexpr int kWin = 384;                          // float4 entries
constexpr uint32_t kWinBytes = kWin * 16;          // 6144
constexpr uint32_t kOffBias = kOffV + 2 * kTile;   // 196608
constexpr uint32_t kOffRed = kOffBias + 2 * kWinBytes;   // [2 parity][2 tiles][2 halves][128] row maxima
constexpr uint32_t kOffLred = kOffRed + 2 * 2 * 2 * 128 * 4;     // same shape, row sums at the epilogue
constexpr uint32_t kOffBar = kOffLred + 2 * 2 * 2 * 128 * 4;
constexpr uint32_t kSmemBytes = kOffBar + 512 + 1024;  // + alignment slack
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleThreshold = 8.0f;        // log2 units

struct Bars {
    uint64_t q_full[2], q_free[2];   // per tile slot
    uint64_t k_full[2], k_empty[2];
    uint64_t v_full[2], v_empty[2];
    uint64_t s_full[2];    // per tile
    uint64_t p_full[2];    // per tile: its 8 softmax warps
    uint64_t pv_done[2];   // per tile
    uint64_t o_free[2];    // per tile: its 8 softmax warps, after the epilogue read O
    uint64_t bias_full[2]; // per stage: bias window loaded
    uint64_t pair[8];      // [tile][lane quarter]: the two half-row warps exchanged
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

// Shared-memory operand descriptors at K step k (16 elements), from the
// tile's precomputed lower word.  K-major (Q, K): box k/4, +32 B per step.
// MN-major (V: keys x d, d contiguous): 16 keys = 2048 B per step, 8-key
// groups 1024 B apart (SBO), the two 64-column halves kBox apart (LBO).
constexpr uint32_t kDescHi = sw128_desc_hi(1024u);
__device__ __forceinline__ uint32_t kmajor_lo(uint32_t tile_base) { return sw128_desc_lo(tile_base, 16u); }
__device__ __forceinline__ uint32_t mnmajor_lo(uint32_t tile_base) { return sw128_desc_lo(tile_base, kBox); }
__device__ __forceinline__ uint64_t kmajor_desc(uint32_t lo, int k) {
    return sw128_desc(lo + (uint32_t)(k >> 2) * (kBox >> 4) + (uint32_t)(k & 3) * 2u, kDescHi);
}
__device__ __forceinline__ uint64_t mnmajor_desc(uint32_t lo, int k) {
    return sw128_desc(lo + (uint32_t)k * 128u, kDescHi);
}

// The work item a CTA takes at its r-th turn: items are listed longest
// first and dealt out in snake order (0..G-1, G-1..0, ...), which evens out
// the per-CTA totals of a decreasing cost list.
__device__ __forceinline__ int item_of_turn(int r, int c, int G) {
    return r * G + ((r & 1) ? (G - 1 - c) : c);
}

// 16 consecutive bf16 starting at p (2-byte aligned) as floats, read as the
// three 16-byte blocks that cover them (the last only when needed).  Reading
// whole aligned blocks never leaves the allocation that holds the 32 bytes.
// Word s + k of the blocks, shifted right by 16 p bits across its neighbour,
// is the pair (2k, 2k+1), with s, p the word and half offset of p.
__device__ __forceinline__ void dense_bias16(const __nv_bfloat16* p, float (&bb)[16]) {
    const uintptr_t addr = reinterpret_cast<uintptr_t>(p);
    const uint4* blk = reinterpret_cast<const uint4*>(addr & ~static_cast<uintptr_t>(15));
    const int e0 = (int)(addr & 15) >> 1;      // element offset in the first block, 0..7
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

struct Item {
    int b, h, row0, q0, nq, k0, nkv;
    int sw;       // tile slot t holds the rows row0 + (t ^ sw) * 128 .. +127
    int jb;       // first key tile of the block (0 unless a sliding window starts later)
    int n_t[2];   // key tiles of slots A and B from jb (0: the slot has no rows or sees no key)
    int n;        // key tiles of the block
};

// The CTA's odd items swap the slots' rows: under the causal rule the lower
// 128 rows take one key tile more than the upper ones, and alternating which
// slot has the extra key tile lets each slot start its next item a key tile
// early every other item (see the MMA thread).
template <bool WINDOW>
__device__ __forceinline__ Item load_item(const AttnArgs& a, int idx, int sw) {
    const int4 it = a.items[idx];
    Item w;
    w.b = it.x;
    w.h = it.y;
    w.row0 = it.z * kBlockRows;
    w.q0 = a.q_off[w.b];
    w.nq = a.q_off[w.b + 1] - w.q0;
    w.k0 = a.kv_off[w.b];
    w.nkv = a.kv_off[w.b + 1] - w.k0;
    // both tiles stream the key tiles from the one tile A's first row needs
    // (tile B's rows see the same or later keys; a key tile of the band that
    // B does not see is masked for it)
    w.sw = sw;
    w.jb = WINDOW ? vis_key_lo(a.window, w.row0, w.nq, w.nkv) / BN : 0;
#pragma unroll
    for (int t = 0; t < 2; ++t) {
        const int lo = w.row0 + (t ^ sw) * BM, hi = min(lo + BM, w.nq);
        if (hi <= lo) {
            w.n_t[t] = 0;
            continue;
        }
        if (WINDOW) {
            const int kv_end = vis_key_hi(a.causal, a.window, hi - 1, w.nq, w.nkv) + 1;
            w.n_t[t] = max((kv_end + BN - 1) / BN - w.jb, 0);
        } else {
            const int kv_end = max(a.causal ? min(w.nkv, hi + (w.nkv - w.nq)) : w.nkv, 0);
            w.n_t[t] = (kv_end + BN - 1) / BN;
        }
    }
    w.n = max(w.n_t[0], w.n_t[1]);
    return w;
}

// First table entry of the bias window of key tile jc for the block at row0:
// the smallest index any (row, key) pair of the block can need, clamped so
// that the window lies inside the prepared table.
__device__ __forceinline__ int bias_window_start(int row0, int jc, int C, int stride) {
    return min(max(row0 - jc - (BN - 1) + C, 0), stride - kWin);
}

// BIAS: 0 none, 1 relative-position (log2(e)-scaled table staged per key tile),
// 2 dense jagged.  SOFTMAX: softmax (true) or GDPA.  WINDOW: a sliding window
// (a lower key bound per row and a first key tile per item).
//
// Tensor-core order per item (n key tiles; tile T has n_T <= n of them):
//   QK_A(0), QK_B(0), then for each j: [P_A(j)] PV_A(j), QK_A(j+1),
//   [P_B(j)] PV_B(j), QK_B(j+1).
// Barrier phases follow per-CTA counters: g (key tiles so far, for the K/V
// ring), gt[T] (steps of tile T so far), mt[T] (items with steps for T so
// far), nk (items so far, for Q).
template <int BIAS, bool SOFTMAX, bool WINDOW>
__global__ void __launch_bounds__(kThreads, 1) tc_fwd_kernel(const __grid_constant__ FwdParams P) {
    const AttnArgs& a = P.a;
    const int n_items = *a.item_count;
    if (a.hdr->err != 0 || (int)blockIdx.x >= n_items) return;
    const bool out32 = (reinterpret_cast<uintptr_t>(a.out) & 31) == 0;
    extern __shared__ uint8_t smem_dyn[];
    uint8_t* smem = smem_dyn + ((1024u - (smem_u32(smem_dyn) & 1023u)) & 1023u);
    Bars* bars = reinterpret_cast<Bars*>(smem + kOffBar);
    const int G = gridDim.x, cta = blockIdx.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    constexpr bool softmax = SOFTMAX;

    if (threadIdx.x == 0) {
        mbar_init(&bars->q_full[0], 1);
        mbar_init(&bars->q_free[0], 1);
        mbar_init(&bars->q_full[1], 1);
        mbar_init(&bars->q_free[1], 1);
        for (int s = 0; s < 2; ++s) {
            mbar_init(&bars->k_full[s], 1);
            mbar_init(&bars->k_empty[s], 1);
            mbar_init(&bars->v_full[s], 1);
            mbar_init(&bars->v_empty[s], 1);
            mbar_init(&bars->s_full[s], 1);
            mbar_init(&bars->p_full[s], 8);
            mbar_init(&bars->pv_done[s], 1);
            mbar_init(&bars->o_free[s], 8);
            mbar_init(&bars->bias_full[s], 1);
        }
        for (int q = 0; q < 8; ++q) mbar_init(&bars->pair[q], 2);
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
        if (lane == 0) {
            tma_prefetch_desc(&P.tm_q);
            tma_prefetch_desc(&P.tm_k);
            tma_prefetch_desc(&P.tm_v);
            int g = 0;                // key tiles issued
            int nq[2] = {0, 0};       // Q tiles issued per slot (items where the slot sees keys)
            bool ok = true;
            // Q of a slot replaces the slot's previous one once that item's last
            // Q K^T of the slot has retired.  The slot that ended the previous
            // item a key tile early (its first score MMA of this item goes out
            // then) gets its Q before the item's first key tile, the other one
            // after it.
            auto load_q = [&](const Item& w, int t) -> bool {
                if (w.n_t[t] == 0) return true;
                if (nq[t] > 0 && !mbar_wait(&bars->q_free[t], (nq[t] - 1) & 1, abort_flag, a.hdr)) return false;
                const int z = w.q0 + w.row0 + (t ^ w.sw) * BM;
                mbar_arrive_expect_tx(&bars->q_full[t], kTile);
                tma_load_3d(smem + kOffQ + t * kTile, &P.tm_q, &bars->q_full[t], 0, w.h, z);
                tma_load_3d(smem + kOffQ + t * kTile + kBox, &P.tm_q, &bars->q_full[t], 64, w.h, z);
                ++nq[t];
                return true;
            };
            int early = 0;
            for (int r = 0; ok; ++r) {
                const int idx = item_of_turn(r, cta, G);
                if (idx >= n_items) break;
                const Item w = load_item<WINDOW>(a, idx, r & 1);
                if (w.n == 0) continue;
                if (!load_q(w, early)) { ok = false; break; }
                for (int j = 0; j < w.n; ++j, ++g) {
                    if (j == 1 && !load_q(w, early ^ 1)) { ok = false; break; }
                    const int s = g & 1;
                    const uint32_t par = ((g >> 1) - 1) & 1;
                    const int z = w.k0 + (w.jb + j) * BN;
                    if (g >= 2 && !mbar_wait(&bars->k_empty[s], par, abort_flag, a.hdr)) { ok = false; break; }
                    JFA_TRACE_EV(fwd, 0, g, 0);
                    // test hook: CTA 0 leaves out its first key tile (load and
                    // expected bytes), so that the waits on it run out
                    const bool skip = a.test_skip_load && cta == 0 && g == 0;
                    if (!skip) {
                        mbar_arrive_expect_tx(&bars->k_full[s], kTile);
                        tma_load_3d(smem + kOffK + s * kTile, &P.tm_k, &bars->k_full[s], 0, w.h, z);
                        tma_load_3d(smem + kOffK + s * kTile + kBox, &P.tm_k, &bars->k_full[s], 64, w.h, z);
                    }
                    if (g >= 2 && !mbar_wait(&bars->v_empty[s], par, abort_flag, a.hdr)) { ok = false; break; }
                    JFA_TRACE_EV(fwd, 0, g, 1);
                    mbar_arrive_expect_tx(&bars->v_full[s], kTile);
                    tma_load_3d(smem + kOffV + s * kTile, &P.tm_v, &bars->v_full[s], 0, w.h, z);
                    tma_load_3d(smem + kOffV + s * kTile + kBox, &P.tm_v, &bars->v_full[s], 64, w.h, z);
                    if (BIAS == 1) {
                        // the stage's previous window was read by the softmax warps of
                        // both tiles before its P.V, hence before v_empty above
                        const int C = (a.relpos_len - 1) >> 1;
                        const int w0 = bias_window_start(w.row0, (w.jb + j) * BN, C, a.bias4_stride);
                        const float* src = a.bias4 + 4 * ((int64_t)w.h * a.bias4_stride + w0);
                        mbar_arrive_expect_tx(&bars->bias_full[s], kWinBytes);
                        bulk_load(smem + kOffBias + s * kWinBytes, src, kWinBytes, &bars->bias_full[s]);
                    }
                    if (j + 2 < w.n) {  // warm L2 for the tiles loaded after the next release
                        tma_prefetch_l2_3d(&P.tm_k, 0, w.h, z + 2 * BN);
                        tma_prefetch_l2_3d(&P.tm_k, 64, w.h, z + 2 * BN);
                        tma_prefetch_l2_3d(&P.tm_v, 0, w.h, z + 2 * BN);
                        tma_prefetch_l2_3d(&P.tm_v, 64, w.h, z + 2 * BN);
                    }
                }
                if (ok && w.n == 1 && !load_q(w, early ^ 1)) { ok = false; break; }
                early = (w.n_t[1] == w.n - 1 && w.n_t[0] == w.n) ? 1 : 0;
            }
            // never leave the CTA with copies in flight: wait for the last loads
            for (int t = 0; t < 2; ++t)
                if (nq[t] > 0) mbar_wait_drain(&bars->q_full[t], (nq[t] - 1) & 1, a.hdr);
            for (int t = (g > 2 ? g - 2 : 0); t < g; ++t) {
                mbar_wait_drain(&bars->k_full[t & 1], (t >> 1) & 1, a.hdr);
                mbar_wait_drain(&bars->v_full[t & 1], (t >> 1) & 1, a.hdr);
                if (BIAS == 1) mbar_wait_drain(&bars->bias_full[t & 1], (t >> 1) & 1, a.hdr);
            }
        }
    } else if (warp == kMmaWarp) {
        // ------------------------------------------------------------ MMA
        if (lane == 0) {
            constexpr uint32_t idesc_qk = idesc_bf16(BM, BN, 0, 0);
            constexpr uint32_t idesc_pv = idesc_bf16(BM, HD, 0, 1);
            int g = 0;
            int gt[2] = {0, 0}, mt[2] = {0, 0}, nq[2] = {0, 0};   // steps, items, Q tiles per slot
            bool ok = true;
            // descriptor lower words of every operand tile, computed once
            const uint32_t qK0 = kmajor_lo(sbase + kOffQ), qK1 = kmajor_lo(sbase + kOffQ + kTile);
            const uint32_t kK0 = kmajor_lo(sbase + kOffK), kK1 = kmajor_lo(sbase + kOffK + kTile);
            const uint32_t vM0 = mnmajor_lo(sbase + kOffV), vM1 = mnmajor_lo(sbase + kOffV + kTile);
            // user of key/value step j of an item: slot A while j < n_A, slot B while j < n_B
            auto first_user = [](const Item& w, int j) { return j < w.n_t[0] ? 0 : 1; };
            auto last_user = [](const Item& w, int j) { return j < w.n_t[1] ? 1 : 0; };
            // S_T = Q_T K_j^T into S_T for step j of item w (first key tile g0).
            // The first score MMA on a key tile waits for its load and the last
            // releases the stage (wait_k / release_k); Q_T is released by the
            // slot's last score MMA of the item (its first waits for Q_T).
            auto issue_qk = [&](const Item& w, int g0, int t, int j, bool wait_k, bool release_k) -> bool {
                const int gg = g0 + j, s = gg & 1;
                if (j == 0) {
                    if (!mbar_wait(&bars->q_full[t], nq[t] & 1, abort_flag, a.hdr)) return false;
                    ++nq[t];
                }
                if (wait_k) {
                    if (!mbar_wait(&bars->k_full[s], (gg >> 1) & 1, abort_flag, a.hdr)) return false;
                    JFA_TRACE_EV(fwd, 1, gg, 0);
                }
                tc_fence_after();
                const uint32_t qd = t ? qK1 : qK0, kd = s ? kK1 : kK0;
#pragma unroll
                for (int k = 0; k < HD / 16; ++k)
                    mma_bf16_ss(tmem + t * 128, kmajor_desc(qd, k), kmajor_desc(kd, k), idesc_qk, k > 0 ? 1u : 0u);
                mma_commit(&bars->s_full[t]);
                if (release_k) mma_commit(&bars->k_empty[s]);
                if (j == w.n_t[t] - 1) mma_commit(&bars->q_free[t]);
                return true;
            };
            // in item order the first user issues first and the last releases
            auto issue_qk_ordered = [&](const Item& w, int g0, int t, int j) -> bool {
                return issue_qk(w, g0, t, j, t == first_user(w, j), t == last_user(w, j));
            };
            int early = -1;   // slot whose first score MMA of this item went out during the previous one
            for (int r = 0; ok; ++r) {
                const int idx = item_of_turn(r, cta, G);
                if (idx >= n_items) break;
                const Item w = load_item<WINDOW>(a, idx, r & 1);
                if (w.n == 0) continue;
                const int g0 = g;
                // after an early slot's score MMA on the item's first key tile the
                // other slot's comes second: it releases the stage
                for (int t = 0; t < 2 && ok; ++t)
                    if (w.n_t[t] > 0 && t != early)
                        ok = early >= 0 ? issue_qk(w, g0, t, 0, true, true) : issue_qk_ordered(w, g0, t, 0);
                early = -1;
                for (int j = 0; ok && j < w.n; ++j, ++g) {
                    const int s = g & 1;
                    for (int t = 0; t < 2 && ok; ++t) {
                        if (j >= w.n_t[t]) continue;
                        if (!mbar_wait(&bars->p_full[t], gt[t] & 1, abort_flag, a.hdr)) { ok = false; break; }
                        JFA_TRACE_EV(fwd, 1, g, 1 + 2 * t);
                        // the epilogue of this slot's previous item must be done with O_T
                        if (j == 0 && mt[t] > 0 &&
                            !mbar_wait(&bars->o_free[t], (mt[t] - 1) & 1, abort_flag, a.hdr)) { ok = false; break; }
                        if (t == first_user(w, j) &&
                            !mbar_wait(&bars->v_full[s], (g >> 1) & 1, abort_flag, a.hdr)) { ok = false; break; }
                        tc_fence_after();
                        const uint32_t vd = s ? vM1 : vM0;
                        const uint32_t tP = tmem + t * 128;   // P (bf16 pairs) over S_T: keys 16k.. at 8k + (k >= 4 ? 32 : 0)
                        const uint32_t tO = tmem + 256 + t * 128;
#pragma unroll
                        for (int k = 0; k < BN / 16; ++k)
                            mma_bf16_ts(tO, tP + k * 8 + (k >= 4 ? 32 : 0), mnmajor_desc(vd, k), idesc_pv,
                                        (j > 0 || k > 0) ? 1u : 0u);
                        mma_commit(&bars->pv_done[t]);
                        if (t == last_user(w, j)) mma_commit(&bars->v_empty[s]);
                        JFA_TRACE_EV(fwd, 1, g, 2 + 2 * t);
                        ++gt[t];
                        if (j == 0) ++mt[t];
                        // S_T(j+1) overwrites P_T(j): issued after the P.V that reads it
                        if (j + 1 < w.n_t[t]) ok = issue_qk_ordered(w, g0, t, j + 1);
                    }
                    // A slot with one key tile fewer than the other ends the item a
                    // step early: its first score MMA of the next item goes out now,
                    // while the other slot works on the item's last key tile.  Its
                    // Q and key tile need only releases issued above (the slot's Q by
                    // its last score MMA a step earlier, the key stage by both
                    // slots' score MMAs a step earlier and their P.V just now).
                    for (int es = 0; es < 2 && ok; ++es) {
                        if (j != w.n_t[es] - 1 || j + 2 != w.n || w.n_t[es ^ 1] != w.n) continue;
                        for (int r2 = r + 1;; ++r2) {
                            const int idx2 = item_of_turn(r2, cta, G);
                            if (idx2 >= n_items) break;
                            const Item w2 = load_item<WINDOW>(a, idx2, r2 & 1);
                            if (w2.n == 0) continue;
                            if (w2.n_t[es] > 0) {
                                // issued before the other slot's: it waits for the
                                // load, and releases the stage only as sole user
                                ok = issue_qk(w2, g0 + w.n, es, 0, true, w2.n_t[es ^ 1] == 0);
                                early = es;
                            }
                            break;
                        }
                    }
                }
            }
            // all issued MMAs retire before TMEM is released
            mma_commit(&bars->drain);
            mbar_wait_drain(&bars->drain, 0, a.hdr);
        }
    } else {
        // ------------------------------------------------ softmax warps
        // waits taken by a whole warp: the result is made warp-uniform, so that a
        // timed-out wait ends the warp's loop on every lane together
        auto wwait = [&](uint64_t* bar, uint32_t parity) -> bool {
            return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag, a.hdr));
        };
        const int tt = warp >> 3;                // query tile: 0 = A, 1 = B
        const int hf = (warp >> 2) & 1;          // half of the row: columns 64 hf .. +63
        const int wq = warp & 3;                 // TMEM lane quarter
        const int r_ = wq * 32 + lane;           // row within the tile
        const int cb = hf * CW;                  // first column of this thread
        const uint32_t lane_addr = (uint32_t)(wq * 32) << 16;
        const uint32_t tS = tmem + lane_addr + tt * 128;
        const uint32_t tO = tmem + lane_addr + 256 + tt * 128 + cb;
        float* red = reinterpret_cast<float*>(smem + kOffRed);
        float* lred = reinterpret_cast<float*>(smem + kOffLred);
        // exchange with the warp that holds the other half of these rows: both
        // write, arrive, and wait (bounded) for the other's arrival
        uint64_t* pair_bar = &bars->pair[tt * 4 + wq];
        int n_pair = 0;
        auto pair_sync = [&]() -> bool {
            __syncwarp();
            if (lane == 0) mbar_arrive(pair_bar);
            return wwait(pair_bar, (n_pair++) & 1);
        };
        const float sc = a.scale * kLog2e;
        const float2 sc2 = make_float2(sc, sc);
        const int C = (a.relpos_len - 1) >> 1;
        int gt = 0, gkv = 0, mt = 0;   // steps of this tile, key tiles of the CTA, items of this tile
        bool ok = true;
        const int tslot = (warp == 0 && lane == 0) ? 2 : ((warp == 8 && lane == 0) ? 3 : -1);
#define SM_EV(ev)                                      \
    do {                                               \
        if (tslot >= 0) JFA_TRACE_EV(fwd, tslot, gt, ev); \
    } while (0)
        // Every wait is a bounded mbarrier wait (the pair exchange too), so a
        // failed (timed-out) wait simply ends this warp's loop.
        for (int rr = 0; ok; ++rr) {
            const int idx = item_of_turn(rr, cta, G);
            if (idx >= n_items) break;
            const Item w = load_item<WINDOW>(a, idx, rr & 1);
            const int n = w.n_t[tt];
            const int gkv_item = gkv;
            gkv += w.n;
            const int i = w.row0 + (tt ^ w.sw) * BM + r_;   // query index within the sequence
            if (n == 0) {
                // rows that see no key (no keys at all, or causal with n_q > n_kv):
                // zero output, LSE = -inf; the tensor core never touches this tile
                if (i < w.nq) {
                    __nv_bfloat16* orow = reinterpret_cast<__nv_bfloat16*>(a.out) + ((int64_t)(w.q0 + i) * a.H + w.h) * HD + cb;
#pragma unroll
                    for (int t = 0; t < CW; t += 8) *reinterpret_cast<uint4*>(orow + t) = make_uint4(0, 0, 0, 0);
                    if (softmax && a.lse && hf == 0) a.lse[(int64_t)(w.q0 + i) * a.H + w.h] = -CUDART_INF_F;
                }
                continue;
            }
            const float inv_n = w.nkv > 0 ? 1.0f / (float)w.nkv : 0.f;
            const float half_c = inv_n * (0.5f / kLog2e);   // GDPA: act(s) / n_kv = x half_c (1 + tanh)
            const int jmax_vis = WINDOW ? vis_key_hi(a.causal, a.window, i, w.nq, w.nkv)
                                        : (a.causal ? min(w.nkv - 1, i + (w.nkv - w.nq)) : w.nkv - 1);
            const int jmin_vis = WINDOW ? vis_key_lo(a.window, i, w.nq, w.nkv) : 0;
            const float* tab4 = (BIAS == 1) ? a.bias4 + (int64_t)w.h * 4 * a.bias4_stride : nullptr;
            const __nv_bfloat16* dense = reinterpret_cast<const __nv_bfloat16*>(a.bias);
            const int64_t dense_row = (BIAS == 2 && i < w.nq)
                                          ? a.dense_off[w.b] + ((int64_t)w.h * w.nq + i) * w.nkv : 0;
            float m_used = -CUDART_INF_F, l = 0.f;
            // a dense bias row segment (this thread's 64 keys of a key tile, read
            // once from HBM) is brought into L2 a key tile ahead
            auto prefetch_bias_seg = [&](int jt) {
                if (BIAS == 2 && i < w.nq && jt < n) {
                    const int kj = (w.jb + jt) * BN + cb;
                    const int k_lo = min(kj, w.nkv - 1), k_hi = min(kj + CW - 1, w.nkv - 1);
                    prefetch_l2(dense + dense_row + k_lo);
                    prefetch_l2(dense + dense_row + k_hi);
                }
            };
            prefetch_bias_seg(0);
            for (int j = 0; j < n; ++j, ++gt) {
                SM_EV(0);
                if (!wwait(&bars->s_full[tt], gt & 1)) { ok = false; break; }
                SM_EV(1);
                tc_fence_after();
                const int jc = (w.jb + j) * BN;      // key index of column 0
                const int gk = gkv_item + j, sk = gk & 1;   // key / value / bias stage
                if (BIAS == 1 && !wwait(&bars->bias_full[sk], (gk >> 1) & 1)) { ok = false; break; }
                const int nvis = i < w.nq ? max(0, min(BN, jmax_vis - jc + 1)) : 0;   // visible: [nlo, nvis)
                const int nlo = WINDOW ? jmin_vis - jc : 0;
                const bool masked_half = __any_sync(0xffffffffu, nvis < cb + CW || (WINDOW && nlo > cb));
                // bias(i, jc + c) = table[lo + 127 - c], lo = i - jc - 127 + C: the run
                // table[lo .. lo+127] as the window entries lo - w0 + 4q, or clamped
                // reads of the table when the run leaves the table or the window
                const int lo = i - jc - (BN - 1) + C;
                const int wrel = BIAS == 1 ? lo - bias_window_start(w.row0, jc, C, a.bias4_stride) : 0;
                const bool win_ok = BIAS == 1 && lo >= 0 && lo + (BN - 1) <= 2 * C && wrel >= 0 && wrel + BN - 4 < kWin;
                const float4* win = reinterpret_cast<const float4*>(smem + kOffBias + sk * kWinBytes) + wrel;
                // ---- pass 1: x = scale * s + bias (log2 units), masked to -inf, back
                //      to TMEM over s; the maximum of this half of the row
                float pm = -CUDART_INF_F;
                // chunk c + 1 is loaded while chunk c is worked on (a wait covers
                // every earlier load, so the next chunk's load goes out after it)
                uint32_t ub[2][16];
                tmem_ld16(tS + cb, ub[0]);
#pragma unroll
                for (int c = 0; c < CW / 16; ++c) {
                    const int cc = cb + c * 16;      // first column of the chunk
                    tmem_wait_ld();
                    if (c + 1 < CW / 16) tmem_ld16(tS + cc + 16, ub[(c + 1) & 1]);
                    float* x = reinterpret_cast<float*>(ub[c & 1]);
                    uint32_t* u = ub[c & 1];
                    if (BIAS == 1) {
                        float bb[16];   // bb[v] = bias(i, jc + cc + v) = table[lo + 127 - cc - v]
                        if (win_ok) {
                            // window entries lo - w0 + 124 - cc - 4q hold table[lo + 124 - cc - 4q + 0..3]
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
                            // the row's 16 bf16 (32 bytes, any 2-byte alignment) from
                            // the three 16-byte blocks that hold them: three loads
                            // instead of sixteen (a warp's lanes are on 32 rows)
                            float bb[16];
                            dense_bias16(dense + dense_row + jc + cc, bb);
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
                                            cc + v < nvis ? __bfloat162float(dense[dense_row + jc + cc + v]) * kLog2e : 0.f);
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
                        for (int v = 0; v < 16; ++v) x[v] = (cc + v < nvis && (!WINDOW || cc + v >= nlo)) ? x[v] : -CUDART_INF_F;
                    }
                    if (softmax) {
                        const float m0 = max3(x[0], x[1], x[2]), m1 = max3(x[3], x[4], x[5]);
                        const float m2 = max3(x[6], x[7], x[8]), m3 = max3(x[9], x[10], x[11]);
                        const float m4 = max3(x[12], x[13], x[14]);
                        pm = max3(pm, max3(m0, m1, m2), max3(m3, m4, x[15]));
                    }
                    tmem_st16(tS + cc, *reinterpret_cast<uint32_t(*)[16]>(u));
                }
                SM_EV(2);
                prefetch_bias_seg(j + 1);
                float ref = 0.f;
                if (softmax) {
                    // row maximum of both halves (exchange buffer by step parity)
                    float* rp = red + ((gt & 1) * 4 + tt * 2) * 128;
                    rp[hf * 128 + r_] = pm;
                    if (!pair_sync()) { ok = false; break; }
                    pm = fmaxf(pm, rp[(hf ^ 1) * 128 + r_]);
                    // lazy rescale: keep the reference unless the row maximum grew by
                    // more than 8 (a factor 2^8); the reference is then the maximum
                    // itself, so the largest weight is 1.  Both halves of a row take
                    // the same decision.
                    float alpha = 1.f;
                    bool rescale = false;
                    const bool need = pm > m_used + kRescaleThreshold;
                    const float m_new = need ? pm : m_used;
                    if (need && m_used != -CUDART_INF_F) {
                        alpha = ex2(m_used - m_new);
                        rescale = true;
                    } else if (need) {
                        l = 0.f;  // first visible key of this row
                    }
                    m_used = m_new;
                    // a rescale of O needs every earlier P.V of this tile retired
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
                    // ex2(-inf) = 0 masks the invisible columns; a row with no visible
                    // key yet uses reference 0 so that -inf - ref stays -inf
                    ref = m_used == -CUDART_INF_F ? 0.f : m_used;
                }
                tmem_wait_st();
                SM_EV(3);
                // ---- pass 2: P (bf16 pairs) -> TMEM over the first half of this
                //      thread's own S columns: keys cb + 16c .. +15 to columns
                //      cb + 8c .. +7, which hold x of chunks already read
                {
                    const float2 ref2 = make_float2(ref, ref);
                    float2 ps = make_float2(0.f, 0.f), ps2 = make_float2(0.f, 0.f);
                    uint32_t ub[2][16];
                    tmem_ld16(tS + cb, ub[0]);
#pragma unroll
                    for (int c = 0; c < CW / 16; ++c) {
                        const int cc = cb + c * 16;
                        tmem_wait_ld();
                        if (c + 1 < CW / 16) tmem_ld16(tS + cc + 16, ub[(c + 1) & 1]);
                        float* x = reinterpret_cast<float*>(ub[c & 1]);
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
                                x[v] = (cc + v < nvis && (!WINDOW || cc + v >= nlo)) ? gdpa_weight_log2<JFA_ACT_SILU>(x[v], half_c) : 0.f;
                        } else {
#pragma unroll
                            for (int v = 0; v < 16; ++v)
                                x[v] = (cc + v < nvis && (!WINDOW || cc + v >= nlo)) ? gdpa_weight_log2<JFA_ACT_GELU_TANH>(x[v], half_c) : 0.f;
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
                // value rows past the sequence end (neighbour data) must not reach P.V;
                // the first tile that uses this key tile clears them before its P is
                // released (both tiles read the same V stage)
                const int nvalid = w.nkv - jc;
                const int clearer = (j < w.n_t[0]) ? 0 : 1;
                if (nvalid < BN && tt == clearer) {  // same for the whole tile
                    if (!wwait(&bars->v_full[sk], (gk >> 1) & 1)) { ok = false; break; }
                    if (r_ >= nvalid) {
                        uint8_t* vrow = smem + kOffV + sk * kTile + hf * kBox + r_ * 128;
                        const uint4 z = make_uint4(0, 0, 0, 0);
#pragma unroll
                        for (int ch = 0; ch < 8; ++ch) *reinterpret_cast<uint4*>(vrow + ch * 16) = z;
                    }
                }
                SM_EV(4);
                fence_proxy_async_smem();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars->p_full[tt]);
            }
            if (!ok) break;
            // ---------------------------------------------------- epilogue
            if (!wwait(&bars->pv_done[tt], (gt - 1) & 1)) { ok = false; break; }
            SM_EV(5);
            tc_fence_after();
            float l_row = l;
            if (softmax) {
                float* lp = lred + ((mt & 1) * 4 + tt * 2) * 128;
                lp[hf * 128 + r_] = l;
                if (!pair_sync()) { ok = false; break; }
                l_row += lp[(hf ^ 1) * 128 + r_];
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
            // O_T free for this tile's next item
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->o_free[tt]);
            if (softmax && hf == 0 && i < w.nq && a.lse)
                a.lse[(int64_t)(w.q0 + i) * a.H + w.h] =
                    l_row > 0.f ? m_used * (1.0f / kLog2e) + logf(l_row) : -CUDART_INF_F;
            SM_EV(6);
        }
#undef SM_EV
    }
    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
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
// 64 d x 1 head x box_rows rows with the 128-byte swizzle.
bool make_tmap_rows_heads_d_box(CUtensorMap* map, const void* base, int64_t rows, int heads,
                                int box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {(cuuint64_t)HD, (cuuint64_t)heads, (cuuint64_t)(rows > 0 ? rows : 1)};
    cuuint64_t strides[2] = {(cuuint64_t)HD * 2, (cuuint64_t)heads * HD * 2};
    cuuint32_t box[3] = {64, 1, (cuuint32_t)box_rows};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides,
                    box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

bool make_tmap_rows_heads_d(CUtensorMap* map, const void* base, int64_t rows, int heads) {
    return make_tmap_rows_heads_d_box(map, base, rows, heads, 128);
}

constexpr int kSmemLimit = 232448;  // 227 KB opt-in per CTA

cudaError_t tc_forward_launch(const jfa_problem& p, const AttnArgs& a, cudaStream_t st) {
    FwdParams P{};
    if (!make_tmap_rows_heads_d(&P.tm_q, a.q, p.total_q, p.heads) ||
        !make_tmap_rows_heads_d(&P.tm_k, a.k, p.total_kv, p.heads) ||
        !make_tmap_rows_heads_d(&P.tm_v, a.v, p.total_kv, p.heads))
        return cudaErrorInvalidValue;
    P.a = a;
    const int smem = (int)kSmemBytes;
    const int64_t items_bound = pairs_bound(p.batch, p.max_q_len, p.total_q, kBlockRows) * p.heads;
    if (items_bound <= 0) return cudaSuccess;
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int grid = (int)(items_bound < sms ? items_bound : sms);
    const int bias = p.bias_kind == JFA_BIAS_RELPOS ? 1 : (p.bias_kind == JFA_BIAS_DENSE_JAGGED ? 2 : 0);
    const bool sm = a.act == JFA_ACT_SOFTMAX;
    const bool win = a.window > 0;
    void (*kern)(FwdParams) = nullptr;
    if (bias == 0) {
        kern = win ? (sm ? tc_fwd_kernel<0, true, true> : tc_fwd_kernel<0, false, true>)
                   : (sm ? tc_fwd_kernel<0, true, false> : tc_fwd_kernel<0, false, false>);
    } else if (bias == 1) {
        kern = win ? (sm ? tc_fwd_kernel<1, true, true> : tc_fwd_kernel<1, false, true>)
                   : (sm ? tc_fwd_kernel<1, true, false> : tc_fwd_kernel<1, false, false>);
    } else {
        kern = win ? (sm ? tc_fwd_kernel<2, true, true> : tc_fwd_kernel<2, false, true>)
                   : (sm ? tc_fwd_kernel<2, true, false> : tc_fwd_kernel<2, false, false>);
    }
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemLimit);
    if (e != cudaSuccess) return e;
    prof_begin(st);
    kern<<<grid, kThreads, smem, st>>>(P);
    prof_end(st, K_TC_FWD);
    return cudaGetLastError();
}

}  // namespace jfa
