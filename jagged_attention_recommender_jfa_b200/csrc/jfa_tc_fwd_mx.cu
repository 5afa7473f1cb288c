// Tensor-core MXFP8 jagged attention forward (head_dim 128): block-scaled
// tcgen05 MMAs on E4M3 operands with E8M0 scales per 32 elements.
//
// MXFP8 attention ("GEM Training: How Meta Doubled the Efficiency of Its
// LLM-Scale Ads Foundation Model", opening summary) with the formats of the
// OCP MX v1.0 specification: Q and K carry one scale per 32 elements of d,
// V one per 32 keys of a sequence (the P.V contraction axis), and P is
// quantised per 32 keys in the softmax pass.  Both products run as
// tcgen05.mma.kind::mxf8f6f4.block_scale with fp32 accumulation in TMEM:
//   S_T = Q_T K_j^T   A = Q (E4M3, K-major), B = K (E4M3, K-major),
//                     scale A = Q's per row and 32-wide d block, scale B = K's
//   O_T += P_T V_j    A = P (E4M3, K-major, written to shared memory by the
//                     softmax warps), B = V (E4M3, MN-major), scale A = P's
//                     per row and 32-key block, scale B = V's per d column and
//                     32-key block
// Each MMA instruction covers K = 32, and its scale factors sit in TMEM: for
// an operand of 128 rows, row m's scale is byte k of lane (m % 32) of column
// (m / 32) in every 32-lane quarter (4 columns, replicated), byte k serving the
// k-th 32-wide K step (selected by the scale-factor id).  They are staged in
// shared memory as 32 lanes x 16 bytes and copied to TMEM with
// tcgen05.cp.32x128b.warpx4, which replicates them to the four quarters.
//
// Work item and pipeline as in the bf16 kernel: (sequence, head, 256-row
// query block) from the longest-first schedule, two 128-row query tiles A and
// B sharing one stream of key/value tiles, alternated on the tensor core.  The
// key tiles are 96 rows (three MX blocks of 32), so S_A and S_B use 96 of
// their 128 TMEM columns and the scale factors take the other 32 of each
// (O_A and O_B keep 128 each).
//
// Softmax warps (16: tile x half row x lane quarter) own 48 columns of a row;
// the middle MX block of a key tile (keys 32..63) straddles the two halves,
// whose partial maxima travel with the row maxima through the pair exchange.
// P's block maxima come from the scores (P = 2^(x - ref) is monotone in x),
// so no second exchange is needed.  The reference is an integer (the ceiling
// of the running maximum, rescaled lazily by powers of two), so the codes do
// not depend on it; l sums the unquantised weights.
#include <math_constants.h>

#include "jfa_mx.cuh"
#include "jfa_sm100.cuh"

namespace jfa {

using namespace sm100;

namespace {

constexpr int BM = 128, BN = 96, HD = 128;
constexpr int kBlockRows = 2 * BM;
constexpr int kMmaWarp = 16, kTmaWarp = 17;
constexpr int kThreads = 32 * 18;
constexpr int CW = BN / 2;                      // 48 columns of a key tile per softmax thread
constexpr int NS = 2;                           // key / value stages
constexpr uint32_t kQTile = 128 * 128;          // 128 rows x 128 E4M3 (one 128-byte swizzle box)
constexpr uint32_t kKVTile = BN * 128;          // 96 rows x 128 bytes
constexpr uint32_t kPTile = 128 * 128;          // P: 128 rows x 128 bytes (96 keys used)
constexpr uint32_t kOffQ = 0;                   // Q_A, Q_B
constexpr uint32_t kOffK = kOffQ + 2 * kQTile;  // NS stages
constexpr uint32_t kOffV = kOffK + NS * kKVTile;
constexpr uint32_t kOffP = kOffV + NS * kKVTile;   // P_A, P_B
constexpr int kWin = 384;                          // relative-position window, float4 entries
constexpr uint32_t kWinBytes = kWin * 16;
constexpr uint32_t kOffBias = kOffP + 2 * kPTile;
constexpr uint32_t kRedBytes = 2 * 2 * 2 * 128 * 4;   // [parity][tile][half][row]
constexpr uint32_t kOffRed = kOffBias + NS * kWinBytes;  // row maxima
constexpr uint32_t kOffBred = kOffRed + kRedBytes;        // partial maxima of the middle MX block
constexpr uint32_t kOffLred = kOffBred + kRedBytes;       // row sums at the epilogue
// scale factors staged for tcgen05.cp: 32 lanes x 16 bytes each
constexpr uint32_t kSfChunk = 512;
constexpr uint32_t kOffSfQ = kOffLred + kRedBytes;        // [item parity][tile]
constexpr uint32_t kOffSfK = kOffSfQ + 4 * kSfChunk;      // [stage]
constexpr uint32_t kOffSfV = kOffSfK + NS * kSfChunk;     // [stage]
constexpr uint32_t kOffSfP = kOffSfV + NS * kSfChunk;     // [tile]
constexpr uint32_t kOffBar = kOffSfP + 2 * kSfChunk;
constexpr uint32_t kSmemBytes = kOffBar + 512 + 1024;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleThreshold = 8.0f;

// TMEM columns: S_T at 128 T (96 used), O_T at 256 + 128 T; the scale
// factors fill the 32 columns left after each S (4 columns per group)
constexpr uint32_t kColS = 0;        // S_A [0, 96), S_B [128, 224)
constexpr uint32_t kColO = 256;      // O_A [256, 384), O_B [384, 512)
constexpr uint32_t kColSfQ = 96;     // [item parity][tile] x 4
constexpr uint32_t kColSfP = 112;    // [tile][step parity] x 4
constexpr uint32_t kColSfK = 224;    // [4 slots] x 4
constexpr uint32_t kColSfV = 240;    // [4 slots] x 4

struct Bars {
    uint64_t q_full, q_free;
    uint64_t k_full[NS], k_empty[NS];
    uint64_t v_full[NS], v_empty[NS];
    uint64_t s_full[2];
    uint64_t p_full[2];
    uint64_t pv_done[2];
    uint64_t o_free[2];
    uint64_t bias_full[NS];
    uint64_t pair[8];
    uint64_t drain;
    uint32_t tmem_base;
    int abort_flag;
};
static_assert(sizeof(Bars) <= 512, "barrier block");

struct MxParams {
    CUtensorMap tm_q;   // E4M3 [total_q][H][128]
    CUtensorMap tm_k;
    CUtensorMap tm_v;
    AttnArgs a;
    const uint8_t* qs;      // [total_q][H][4]   E8M0, blocks along d
    const uint8_t* ks;      // [total_kv][H][4]
    const uint8_t* vs;      // [n_blocks][H][128] E8M0, blocks of 32 keys per sequence
    const int32_t* vbase;   // [B] first V block of each sequence
    int64_t total_q, total_kv, n_vblocks;
};

// 128-byte swizzled K-major operand (rows of 128 bytes): K step k = 32 bytes.
constexpr uint32_t kDescHi = sw128_desc_hi(1024u);
__device__ __forceinline__ uint64_t kmajor_desc(uint32_t lo, int k) {
    return sw128_desc(lo + (uint32_t)k * 2u, kDescHi);
}
// MN-major (V: keys x d, d contiguous, 128 bytes per key row): K step of 32
// keys = 4096 bytes, 8-key groups 1024 bytes apart.
__device__ __forceinline__ uint64_t mnmajor_desc(uint32_t lo, int k) {
    return sw128_desc(lo + (uint32_t)k * 256u, kDescHi);
}
// Unswizzled K-major descriptor of a 32-row x 16-byte scale-factor chunk
// (core matrices of 8 rows x 16 bytes, 128 bytes apart) for tcgen05.cp.
__device__ __forceinline__ uint64_t sf_chunk_desc(uint32_t addr) {
    const uint32_t lo = ((addr & 0x3FFFF) >> 4) | ((16u >> 4) << 16);
    const uint32_t hi = (128u >> 4) | (1u << 14);   // SBO 128, sm_100 version bit, no swizzle
    return sw128_desc(lo, hi);
}

// Instruction descriptor, kind::mxf8f6f4 block-scaled: E4M3 A and B, E8M0
// scales, fp32 accumulator implied; the scale-factor ids select the byte of
// the scale columns (the K step).
__host__ __device__ constexpr uint32_t idesc_mx(int M, int N, int b_mn) {
    return (0u << 7) | (0u << 10)            // A, B: E4M3
           | ((uint32_t)b_mn << 16)          // B major
           | ((uint32_t)(N >> 3) << 17)
           | (1u << 23)                      // scales E8M0
           | ((uint32_t)(M >> 4) << 24);
}
__device__ __forceinline__ uint32_t idesc_sf(uint32_t base, int k) {
    return base | ((uint32_t)k << 29) | ((uint32_t)k << 4);
}

__device__ __forceinline__ void mma_mx_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                          uint32_t idesc, uint32_t sfa, uint32_t sfb,
                                          uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %6, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%4], [%5], p;\n\t}" ::"r"(
            d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(sfa), "r"(sfb), "r"(accumulate)
        : "memory");
}

// shared memory (32 lanes x 128 bits) -> TMEM columns taddr .. +3, replicated
// to all four lane quarters
__device__ __forceinline__ void tmem_cp_sf(uint32_t taddr, uint64_t sdesc) {
    asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}

__device__ __forceinline__ int item_of_turn(int r, int c, int G) {
    return r * G + ((r & 1) ? (G - 1 - c) : c);
}

struct Item {
    int b, h, row0, q0, nq, k0, nkv;
    int jb;       // first key tile of the block (0 unless a sliding window starts later)
    int n_t[2];   // key tiles of tile A and tile B from jb
    int n;
};

template <bool WINDOW>
__device__ __forceinline__ Item load_item(const AttnArgs& a, int idx) {
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
    // (96-key tiles keep the MX blocks of V aligned to the sequence start)
    w.jb = WINDOW ? vis_key_lo(a.window, w.row0, w.nq, w.nkv) / BN : 0;
#pragma unroll
    for (int t = 0; t < 2; ++t) {
        const int lo = w.row0 + t * BM, hi = min(lo + BM, w.nq);
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

__device__ __forceinline__ int bias_window_start(int row0, int jc, int C, int stride) {
    return min(max(row0 - jc - (BN - 1) + C, 0), stride - kWin);
}

// 16 consecutive bf16 of a dense bias row from the three aligned 16-byte
// blocks that hold them (any 2-byte alignment).
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

// The 16 staged scale bytes of lane l: rows l, l + 32, l + 64, l + 96 of an
// operand tile, four K blocks each (row-major [row][H][4] source, one 32-bit
// load per row).  Rows at or past `rows` (the sequence end) read the tile's
// first row, clamped into the tensor.
__device__ __forceinline__ uint4 sf_rows4(const uint8_t* base, int64_t row0, int rows, int64_t total,
                                         int H, int h, int lane) {
    uint32_t v[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        const int r = lane + 32 * c;
        int64_t row = row0 + (r < rows ? r : 0);
        row = row < total ? row : total - 1;
        v[c] = *reinterpret_cast<const uint32_t*>(base + (row * H + h) * 4);
    }
    return make_uint4(v[0], v[1], v[2], v[3]);
}

// The staged V scale bytes of lane l: d columns l, l + 32, l + 64, l + 96 (one
// 32-bit word each), byte kb = the key tile's kb-th block of 32 keys; blocks
// past the sequence's last take scale 2^0 (their values are zero).
__device__ __forceinline__ uint4 sf_v(const uint8_t* vs, int64_t blk0, int nblk, int H, int h,
                                      int lane) {
    uint32_t v[4] = {0u, 0u, 0u, 0u};
#pragma unroll
    for (int kb = 0; kb < 3; ++kb) {
        const bool ok = kb < nblk;
        const uint8_t* src = vs + ((blk0 + (ok ? kb : 0)) * H + h) * 128;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const uint32_t byte = ok ? (uint32_t)src[lane + 32 * c] : 127u;
            v[c] |= byte << (8 * kb);
        }
    }
    return make_uint4(v[0], v[1], v[2], v[3]);
}

template <int BIAS, bool WINDOW>
__global__ void __launch_bounds__(kThreads, 1) tc_fwd_mx_kernel(const __grid_constant__ MxParams P) {
    const AttnArgs& a = P.a;
    const int n_items = *a.item_count;
    if (a.hdr->err != 0 || (int)blockIdx.x >= n_items) return;
    extern __shared__ uint8_t smem_dyn[];
    uint8_t* smem = smem_dyn + ((1024u - (smem_u32(smem_dyn) & 1023u)) & 1023u);
    Bars* bars = reinterpret_cast<Bars*>(smem + kOffBar);
    const int G = gridDim.x, cta = blockIdx.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        mbar_init(&bars->q_full, 2);   // TMA bytes + the staged Q scales
        mbar_init(&bars->q_free, 1);
        for (int s = 0; s < NS; ++s) {
            mbar_init(&bars->k_full[s], 2);
            mbar_init(&bars->k_empty[s], 1);
            mbar_init(&bars->v_full[s], 2);
            mbar_init(&bars->v_empty[s], 1);
            mbar_init(&bars->bias_full[s], 1);
        }
        for (int t = 0; t < 2; ++t) {
            mbar_init(&bars->s_full[t], 1);
            mbar_init(&bars->p_full[t], 8);
            mbar_init(&bars->pv_done[t], 1);
            mbar_init(&bars->o_free[t], 8);
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
        // ---------------------------------------------------- TMA + scales
        // lane 0 issues the tile copies; every lane stages scale bytes
        auto wwait = [&](uint64_t* bar, uint32_t parity) -> bool {
            return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag, a.hdr));
        };
        if (lane == 0) {
            tma_prefetch_desc(&P.tm_q);
            tma_prefetch_desc(&P.tm_k);
            tma_prefetch_desc(&P.tm_v);
        }
        int g = 0, nk = 0;
        bool ok = true;
        for (int r = 0; ok; ++r) {
            const int idx = item_of_turn(r, cta, G);
            if (idx >= n_items) break;
            const Item w = load_item<WINDOW>(a, idx);
            if (w.n == 0) continue;
            if (nk > 0 && !wwait(&bars->q_free, (nk - 1) & 1)) { ok = false; break; }
            if (lane == 0) {
                mbar_arrive_expect_tx(&bars->q_full, 2 * kQTile);
                for (int t = 0; t < 2; ++t)
                    tma_load_3d(smem + kOffQ + t * kQTile, &P.tm_q, &bars->q_full, 0, w.h,
                                w.q0 + w.row0 + t * BM);
            }
            for (int t = 0; t < 2; ++t) {
                const int lo = w.row0 + t * BM;
                const uint4 sf = sf_rows4(P.qs, w.q0 + lo, max(0, min(BM, w.nq - lo)), P.total_q, a.H, w.h, lane);
                *reinterpret_cast<uint4*>(smem + kOffSfQ + ((nk & 1) * 2 + t) * kSfChunk + lane * 16) = sf;
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->q_full);
            ++nk;
            const int nblk = (w.nkv + 31) >> 5;
            for (int j = 0; j < w.n; ++j, ++g) {
                const int s = g % NS;
                const uint32_t par = ((g / NS) - 1) & 1;
                const int jt = w.jb + j;   // key tile of the sequence
                const int z = w.k0 + jt * BN;
                if (g >= NS && !wwait(&bars->k_empty[s], par)) { ok = false; break; }
                if (lane == 0) {
                    mbar_arrive_expect_tx(&bars->k_full[s], kKVTile);
                    tma_load_3d(smem + kOffK + s * kKVTile, &P.tm_k, &bars->k_full[s], 0, w.h, z);
                }
                {
                    const uint4 sf = sf_rows4(P.ks, z, max(0, min(BN, w.nkv - jt * BN)), P.total_kv, a.H, w.h, lane);
                    *reinterpret_cast<uint4*>(smem + kOffSfK + s * kSfChunk + lane * 16) = sf;
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&bars->k_full[s]);
                }
                if (g >= NS && !wwait(&bars->v_empty[s], par)) { ok = false; break; }
                if (lane == 0) {
                    mbar_arrive_expect_tx(&bars->v_full[s], kKVTile);
                    tma_load_3d(smem + kOffV + s * kKVTile, &P.tm_v, &bars->v_full[s], 0, w.h, z);
                    if (BIAS == 1) {
                        const int C = (a.relpos_len - 1) >> 1;
                        const int w0 = bias_window_start(w.row0, jt * BN, C, a.bias4_stride);
                        const float* src = a.bias4 + 4 * ((int64_t)w.h * a.bias4_stride + w0);
                        mbar_arrive_expect_tx(&bars->bias_full[s], kWinBytes);
                        bulk_load(smem + kOffBias + s * kWinBytes, src, kWinBytes, &bars->bias_full[s]);
                    }
                    if (j + 2 < w.n) {
                        tma_prefetch_l2_3d(&P.tm_k, 0, w.h, z + 2 * BN);
                        tma_prefetch_l2_3d(&P.tm_v, 0, w.h, z + 2 * BN);
                    }
                }
                {
                    const uint4 sf = sf_v(P.vs, (int64_t)P.vbase[w.b] + 3 * jt, nblk - 3 * jt, a.H, w.h, lane);
                    *reinterpret_cast<uint4*>(smem + kOffSfV + s * kSfChunk + lane * 16) = sf;
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&bars->v_full[s]);
                }
            }
        }
        // never leave the CTA with copies in flight
        if (lane == 0) {
            if (nk > 0) mbar_wait_drain(&bars->q_full, (nk - 1) & 1, a.hdr);
            for (int t = (g > NS ? g - NS : 0); t < g; ++t) {
                mbar_wait_drain(&bars->k_full[t % NS], (t / NS) & 1, a.hdr);
                mbar_wait_drain(&bars->v_full[t % NS], (t / NS) & 1, a.hdr);
                if (BIAS == 1) mbar_wait_drain(&bars->bias_full[t % NS], (t / NS) & 1, a.hdr);
            }
        }
    } else if (warp == kMmaWarp) {
        // ------------------------------------------------------------ MMA
        if (lane == 0) {
            constexpr uint32_t id_qk = idesc_mx(BM, BN, 0);
            constexpr uint32_t id_pv = idesc_mx(BM, HD, 1);
            int g = 0, nk = 0;
            int gt[2] = {0, 0}, mt[2] = {0, 0};
            bool ok = true;
            const uint32_t qlo[2] = {sw128_desc_lo(sbase + kOffQ, 16u), sw128_desc_lo(sbase + kOffQ + kQTile, 16u)};
            const uint32_t plo[2] = {sw128_desc_lo(sbase + kOffP, 16u), sw128_desc_lo(sbase + kOffP + kPTile, 16u)};
            for (int r = 0; ok; ++r) {
                const int idx = item_of_turn(r, cta, G);
                if (idx >= n_items) break;
                const Item w = load_item<WINDOW>(a, idx);
                if (w.n == 0) continue;
                if (!mbar_wait(&bars->q_full, nk & 1, abort_flag, a.hdr)) { ok = false; break; }
                tc_fence_after();
                const int qp = nk & 1;
                for (int t = 0; t < 2; ++t)
                    tmem_cp_sf(tmem + kColSfQ + (qp * 2 + t) * 4,
                               sf_chunk_desc(sbase + kOffSfQ + (qp * 2 + t) * kSfChunk));
                ++nk;
                auto first_user = [&](int j) { return j < w.n_t[0] ? 0 : 1; };
                auto last_user = [&](int j) { return j < w.n_t[1] ? 1 : 0; };
                const int g0 = g;
                auto issue_qk = [&](int t, int j) -> bool {
                    const int gg = g0 + j, s = gg % NS, slot = gg & 3;
                    if (t == first_user(j)) {
                        if (!mbar_wait(&bars->k_full[s], (gg / NS) & 1, abort_flag, a.hdr)) return false;
                        tc_fence_after();
                        tmem_cp_sf(tmem + kColSfK + slot * 4, sf_chunk_desc(sbase + kOffSfK + s * kSfChunk));
                    }
                    const uint32_t klo = sw128_desc_lo(sbase + kOffK + s * kKVTile, 16u);
                    const uint32_t sfa = tmem + kColSfQ + (qp * 2 + t) * 4, sfb = tmem + kColSfK + slot * 4;
#pragma unroll
                    for (int k = 0; k < HD / 32; ++k)
                        mma_mx_ss(tmem + kColS + t * 128, kmajor_desc(qlo[t], k), kmajor_desc(klo, k),
                                  idesc_sf(id_qk, k), sfa | ((uint32_t)k << 30), sfb | ((uint32_t)k << 30),
                                  k > 0 ? 1u : 0u);
                    mma_commit(&bars->s_full[t]);
                    if (t == last_user(j)) mma_commit(&bars->k_empty[s]);
                    if (j == w.n - 1 && t == last_user(j)) mma_commit(&bars->q_free);
                    return true;
                };
                for (int t = 0; t < 2 && ok; ++t)
                    if (w.n_t[t] > 0) ok = issue_qk(t, 0);
                for (int j = 0; ok && j < w.n; ++j, ++g) {
                    const int s = g % NS, slot = g & 3;
                    for (int t = 0; t < 2 && ok; ++t) {
                        if (j >= w.n_t[t]) continue;
                        if (!mbar_wait(&bars->p_full[t], gt[t] & 1, abort_flag, a.hdr)) { ok = false; break; }
                        if (j == 0 && mt[t] > 0 &&
                            !mbar_wait(&bars->o_free[t], (mt[t] - 1) & 1, abort_flag, a.hdr)) { ok = false; break; }
                        if (t == first_user(j)) {
                            if (!mbar_wait(&bars->v_full[s], (g / NS) & 1, abort_flag, a.hdr)) { ok = false; break; }
                            tc_fence_after();
                            tmem_cp_sf(tmem + kColSfV + slot * 4, sf_chunk_desc(sbase + kOffSfV + s * kSfChunk));
                        }
                        tc_fence_after();
                        const uint32_t sfp = tmem + kColSfP + (t * 2 + (gt[t] & 1)) * 4;
                        tmem_cp_sf(sfp, sf_chunk_desc(sbase + kOffSfP + t * kSfChunk));
                        const uint32_t vlo = sw128_desc_lo(sbase + kOffV + s * kKVTile, 16u);
                        const uint32_t sfv = tmem + kColSfV + slot * 4;
#pragma unroll
                        for (int k = 0; k < BN / 32; ++k)
                            mma_mx_ss(tmem + kColO + t * HD, kmajor_desc(plo[t], k), mnmajor_desc(vlo, k),
                                      idesc_sf(id_pv, k), sfp | ((uint32_t)k << 30), sfv | ((uint32_t)k << 30),
                                      (j > 0 || k > 0) ? 1u : 0u);
                        mma_commit(&bars->pv_done[t]);
                        if (t == last_user(j)) mma_commit(&bars->v_empty[s]);
                        ++gt[t];
                        if (j == 0) ++mt[t];
                        if (j + 1 < w.n_t[t]) ok = issue_qk(t, j + 1);
                    }
                }
            }
            mma_commit(&bars->drain);
            mbar_wait_drain(&bars->drain, 0, a.hdr);
        }
    } else {
        // ------------------------------------------------ softmax warps
        auto wwait = [&](uint64_t* bar, uint32_t parity) -> bool {
            return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag, a.hdr));
        };
        const int tt = warp >> 3;                // query tile: 0 = A, 1 = B
        const int hf = (warp >> 2) & 1;          // half of the row: keys 48 hf .. +47
        const int wq = warp & 3;                 // TMEM lane quarter
        const int r_ = wq * 32 + lane;           // row within the tile
        const int cb = hf * CW;
        const uint32_t lane_addr = (uint32_t)(wq * 32) << 16;
        const uint32_t tS = tmem + lane_addr + kColS + tt * 128;
        const uint32_t tO = tmem + lane_addr + kColO + tt * HD + hf * 64;
        float* red = reinterpret_cast<float*>(smem + kOffRed);
        float* bred = reinterpret_cast<float*>(smem + kOffBred);
        float* lred = reinterpret_cast<float*>(smem + kOffLred);
        uint8_t* prow = smem + kOffP + tt * kPTile + r_ * 128;
        uint8_t* sfp = smem + kOffSfP + tt * kSfChunk + lane * 16 + wq * 4;
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
        int gt = 0, gkv = 0, mt = 0;
        bool ok = true;
        for (int rr = 0; ok; ++rr) {
            const int idx = item_of_turn(rr, cta, G);
            if (idx >= n_items) break;
            const Item w = load_item<WINDOW>(a, idx);
            const int n = w.n_t[tt];
            const int gkv_item = gkv;
            gkv += w.n;
            const int i = w.row0 + tt * BM + r_;
            if (n == 0) {
                if (i < w.nq) {
                    __nv_bfloat16* orow = reinterpret_cast<__nv_bfloat16*>(a.out) + ((int64_t)(w.q0 + i) * a.H + w.h) * HD + hf * 64;
#pragma unroll
                    for (int t = 0; t < 64; t += 8) *reinterpret_cast<uint4*>(orow + t) = make_uint4(0, 0, 0, 0);
                    if (a.lse && hf == 0) a.lse[(int64_t)(w.q0 + i) * a.H + w.h] = -CUDART_INF_F;
                }
                continue;
            }
            const int jmax_vis = WINDOW ? vis_key_hi(a.causal, a.window, i, w.nq, w.nkv)
                                        : (a.causal ? min(w.nkv - 1, i + (w.nkv - w.nq)) : w.nkv - 1);
            const int jmin_vis = WINDOW ? vis_key_lo(a.window, i, w.nq, w.nkv) : 0;
            const float* tab4 = (BIAS == 1) ? a.bias4 + (int64_t)w.h * 4 * a.bias4_stride : nullptr;
            const __nv_bfloat16* dense = reinterpret_cast<const __nv_bfloat16*>(a.bias);
            const int64_t dense_row = (BIAS == 2 && i < w.nq)
                                          ? a.dense_off[w.b] + ((int64_t)w.h * w.nq + i) * w.nkv : 0;
            float m_used = -CUDART_INF_F, l = 0.f;
            for (int j = 0; j < n; ++j, ++gt) {
                if (!wwait(&bars->s_full[tt], gt & 1)) { ok = false; break; }
                tc_fence_after();
                const int jc = (w.jb + j) * BN;
                const int gk = gkv_item + j, sk = gk % NS;
                if (BIAS == 1 && !wwait(&bars->bias_full[sk], (gk / NS) & 1)) { ok = false; break; }
                const int nvis = i < w.nq ? max(0, min(BN, jmax_vis - jc + 1)) : 0;   // visible: [nlo, nvis)
                const int nlo = WINDOW ? jmin_vis - jc : 0;
                const bool masked_half = __any_sync(0xffffffffu, nvis < cb + CW || (WINDOW && nlo > cb));
                const int lo = i - jc - (BN - 1) + C;
                const int wrel = BIAS == 1 ? lo - bias_window_start(w.row0, jc, C, a.bias4_stride) : 0;
                const bool win_ok = BIAS == 1 && lo >= 0 && lo + (BN - 1) <= 2 * C && wrel >= 0 && wrel + BN - 4 < kWin;
                const float4* win = reinterpret_cast<const float4*>(smem + kOffBias + sk * kWinBytes) + wrel;
                // ---- pass 1: x = scale * s + bias (log2 units), masked, back to
                //      TMEM; the row maximum and the maxima of the MX blocks
                float cmax[CW / 16];
                uint32_t ub[2][16];
                tmem_ld16(tS + cb, ub[0]);
#pragma unroll
                for (int c = 0; c < CW / 16; ++c) {
                    const int cc = cb + c * 16;
                    tmem_wait_ld();
                    if (c + 1 < CW / 16) tmem_ld16(tS + cc + 16, ub[(c + 1) & 1]);
                    float* x = reinterpret_cast<float*>(ub[c & 1]);
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
                                x[v] = fmaf(x[v], sc, cc + v < nvis ? __bfloat162float(dense[dense_row + jc + cc + v]) * kLog2e : 0.f);
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
                    const float m0 = max3(x[0], x[1], x[2]), m1 = max3(x[3], x[4], x[5]);
                    const float m2 = max3(x[6], x[7], x[8]), m3 = max3(x[9], x[10], x[11]);
                    const float m4 = max3(x[12], x[13], x[14]);
                    cmax[c] = max3(max3(m0, m1, m2), max3(m3, m4, x[15]), -CUDART_INF_F);
                    tmem_st16(tS + cc, *reinterpret_cast<uint32_t(*)[16]>(x));
                }
                // MX blocks of this half: hf 0 holds block 0 (chunks 0, 1) and
                // the low half of block 1 (chunk 2); hf 1 the high half of
                // block 1 (chunk 0) and block 2 (chunks 1, 2)
                const float own_blk = hf == 0 ? fmaxf(cmax[0], cmax[1]) : fmaxf(cmax[1], cmax[2]);
                const float mid_part = hf == 0 ? cmax[2] : cmax[0];
                float pm = fmaxf(own_blk, mid_part);
                float* rp = red + ((gt & 1) * 4 + tt * 2) * 128;
                float* bp = bred + ((gt & 1) * 4 + tt * 2) * 128;
                rp[hf * 128 + r_] = pm;
                bp[hf * 128 + r_] = mid_part;
                if (!pair_sync()) { ok = false; break; }
                pm = fmaxf(pm, rp[(hf ^ 1) * 128 + r_]);
                const float mid_blk = fmaxf(mid_part, bp[(hf ^ 1) * 128 + r_]);
                // lazy rescale with an integer reference (powers of two)
                float alpha = 1.f;
                bool rescale = false;
                const bool need = pm > m_used + kRescaleThreshold;
                const float m_new = need ? ceilf(pm) : m_used;
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
                        for (int c = 0; c < 2; ++c) {
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
                const float ref = m_used == -CUDART_INF_F ? 0.f : m_used;
                tmem_wait_st();
                // shared exponents of P's blocks from the block maxima:
                // amax = 2^(max x - ref), the largest weight of the block
                const int X_own = mx::shared_exponent(own_blk == -CUDART_INF_F ? 0.f : ex2(own_blk - ref));
                const int X_mid = mx::shared_exponent(mid_blk == -CUDART_INF_F ? 0.f : ex2(mid_blk - ref));
                // ---- pass 2: P = 2^(x - ref), l += P, E4M3 codes to shared memory
                {
                    const float2 ref2 = make_float2(ref, ref);
                    float2 ps = make_float2(0.f, 0.f);
                    uint32_t ub2[2][16];
                    tmem_ld16(tS + cb, ub2[0]);
#pragma unroll
                    for (int c = 0; c < CW / 16; ++c) {
                        const int cc = cb + c * 16;
                        tmem_wait_ld();
                        if (c + 1 < CW / 16) tmem_ld16(tS + cc + 16, ub2[(c + 1) & 1]);
                        float* x = reinterpret_cast<float*>(ub2[c & 1]);
#pragma unroll
                        for (int v = 0; v < 16; v += 2) {
                            const float2 y = sub2(make_float2(x[v], x[v + 1]), ref2);
                            x[v] = ex2(y.x);
                            x[v + 1] = ex2(y.y);
                            ps = add2(ps, make_float2(x[v], x[v + 1]));
                        }
                        const bool mid = (hf == 0) ? (c == 2) : (c == 0);
                        const float s2 = mx::pow2_neg(mid ? X_mid : X_own);
                        uint32_t wv[4];
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            const uint32_t lo16 = mx::pack_e4m3x2(x[4 * q] * s2, x[4 * q + 1] * s2);
                            const uint32_t hi16 = mx::pack_e4m3x2(x[4 * q + 2] * s2, x[4 * q + 3] * s2);
                            wv[q] = lo16 | (hi16 << 16);
                        }
                        const int ch = cc >> 4;   // 16-byte chunk of the 128-byte row
                        *reinterpret_cast<uint4*>(prow + ((ch ^ (r_ & 7)) << 4)) = make_uint4(wv[0], wv[1], wv[2], wv[3]);
                    }
                    l += ps.x + ps.y;
                    // P's scales: row r_ (lane, quarter) bytes 0..2 = the three blocks
                    if (hf == 0) {
                        sfp[0] = (uint8_t)(X_own + 127);
                        sfp[1] = (uint8_t)(X_mid + 127);
                    } else {
                        sfp[2] = (uint8_t)(X_own + 127);
                    }
                }
                // value rows past the sequence end must not reach P.V
                const int nvalid = w.nkv - jc;
                const int clearer = (j < w.n_t[0]) ? 0 : 1;
                if (nvalid < BN && tt == clearer) {
                    if (!wwait(&bars->v_full[sk], (gk / NS) & 1)) { ok = false; break; }
                    if (r_ >= nvalid && r_ < BN) {
                        uint8_t* vrow = smem + kOffV + sk * kKVTile + r_ * 128 + hf * 64;
                        const uint4 z = make_uint4(0, 0, 0, 0);
#pragma unroll
                        for (int q = 0; q < 4; ++q) *reinterpret_cast<uint4*>(vrow + q * 16) = z;
                    }
                }
                fence_proxy_async_smem();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars->p_full[tt]);
            }
            if (!ok) break;
            // ---------------------------------------------------- epilogue
            if (!wwait(&bars->pv_done[tt], (gt - 1) & 1)) { ok = false; break; }
            tc_fence_after();
            float* lp = lred + ((mt & 1) * 4 + tt * 2) * 128;
            lp[hf * 128 + r_] = l;
            if (!pair_sync()) { ok = false; break; }
            const float l_row = l + lp[(hf ^ 1) * 128 + r_];
            ++mt;
            const float inv = l_row > 0.f ? 1.f / l_row : 0.f;
            __nv_bfloat16* orow = reinterpret_cast<__nv_bfloat16*>(a.out) + ((int64_t)(w.q0 + i) * a.H + w.h) * HD + hf * 64;
#pragma unroll 1
            for (int c = 0; c < 2; ++c) {
                uint32_t u[32];
                tmem_ld32(tO + c * 32, u);
                tmem_wait_ld();
                if (i < w.nq) {
#pragma unroll
                    for (int t = 0; t < 32; t += 8) {
                        uint4 wv;
                        wv.x = pack_bf16(__uint_as_float(u[t + 0]) * inv, __uint_as_float(u[t + 1]) * inv);
                        wv.y = pack_bf16(__uint_as_float(u[t + 2]) * inv, __uint_as_float(u[t + 3]) * inv);
                        wv.z = pack_bf16(__uint_as_float(u[t + 4]) * inv, __uint_as_float(u[t + 5]) * inv);
                        wv.w = pack_bf16(__uint_as_float(u[t + 6]) * inv, __uint_as_float(u[t + 7]) * inv);
                        *reinterpret_cast<uint4*>(orow + c * 32 + t) = wv;
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->o_free[tt]);
            if (hf == 0 && i < w.nq && a.lse)
                a.lse[(int64_t)(w.q0 + i) * a.H + w.h] =
                    l_row > 0.f ? m_used * (1.0f / kLog2e) + logf(l_row) : -CUDART_INF_F;
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

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

// E4M3 [rows][heads][128] as a 3-D tensor (d, head, row); boxes of 128 bytes
// x 1 head x box_rows rows with the 128-byte swizzle.
bool make_tmap_e4m3(CUtensorMap* map, const void* base, int64_t rows, int heads, int box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {(cuuint64_t)HD, (cuuint64_t)heads, (cuuint64_t)(rows > 0 ? rows : 1)};
    cuuint64_t strides[2] = {(cuuint64_t)HD, (cuuint64_t)heads * HD};
    cuuint32_t box[3] = {128, 1, (cuuint32_t)box_rows};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box,
                    estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// First V scale block of each sequence: exclusive scan of ceil(n / 32).
__global__ void __launch_bounds__(1024) mx_block_base(const int32_t* __restrict__ off, int B,
                                                      int32_t* __restrict__ base) {
    __shared__ int32_t warp_sum[32];
    const int t = threadIdx.x, lane = t & 31, w = t >> 5;
    int carry = 0;
    for (int b0 = 0; b0 < B; b0 += 1024) {
        const int b = b0 + t;
        const int n = b < B ? max(0, off[b + 1] - off[b]) : 0;
        const int cnt = (n + 31) >> 5;
        int x = cnt;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += y;
        }
        if (lane == 31) warp_sum[w] = x;
        __syncthreads();
        if (w == 0) {
            int s = warp_sum[lane];
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, s, o);
                if (lane >= o) s += y;
            }
            warp_sum[lane] = s;
        }
        __syncthreads();
        if (b < B) base[b] = carry + (w > 0 ? warp_sum[w - 1] : 0) + (x - cnt);
        carry += warp_sum[31];
        __syncthreads();
    }
}

}  // namespace

constexpr int kSmemLimitMx = 232448;

// MXFP8 forward on quantised operands: q8/k8/v8 E4M3 codes, qs/ks scales
// along d ([rows][H][4]), vs along 32-key blocks ([n_vblocks][H][128]);
// vbase: device int32 [B] workspace for the first V block of each sequence.
cudaError_t tc_forward_mx_launch(const jfa_problem& p, const AttnArgs& a, const void* q8,
                                 const uint8_t* qs, const void* k8, const uint8_t* ks,
                                 const void* v8, const uint8_t* vs, int64_t n_vblocks,
                                 int32_t* vbase, cudaStream_t st) {
    MxParams P{};
    if (!make_tmap_e4m3(&P.tm_q, q8, p.total_q, p.heads, BM) ||
        !make_tmap_e4m3(&P.tm_k, k8, p.total_kv, p.heads, BN) ||
        !make_tmap_e4m3(&P.tm_v, v8, p.total_kv, p.heads, BN))
        return cudaErrorInvalidValue;
    P.a = a;
    P.qs = qs;
    P.ks = ks;
    P.vs = vs;
    P.vbase = vbase;
    P.total_q = p.total_q;
    P.total_kv = p.total_kv;
    P.n_vblocks = n_vblocks;
    mx_block_base<<<1, 1024, 0, st>>>(a.kv_off, p.batch, vbase);
    const int64_t items_bound = pairs_bound(p.batch, p.max_q_len, p.total_q, kBlockRows) * p.heads;
    if (items_bound <= 0) return cudaGetLastError();
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int grid = (int)(items_bound < sms ? items_bound : sms);
    const int bias = p.bias_kind == JFA_BIAS_RELPOS ? 1 : (p.bias_kind == JFA_BIAS_DENSE_JAGGED ? 2 : 0);
    void (*kern)(MxParams) =
        a.window > 0 ? (bias == 0 ? tc_fwd_mx_kernel<0, true> : (bias == 1 ? tc_fwd_mx_kernel<1, true> : tc_fwd_mx_kernel<2, true>))
                     : (bias == 0 ? tc_fwd_mx_kernel<0, false> : (bias == 1 ? tc_fwd_mx_kernel<1, false> : tc_fwd_mx_kernel<2, false>));
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemLimitMx);
    if (e != cudaSuccess) return e;
    static_assert(kSmemBytes <= (uint32_t)kSmemLimitMx, "shared memory");
    prof_begin(st);
    kern<<<grid, kThreads, kSmemBytes, st>>>(P);
    prof_end(st, K_TC_FWD_MXFP8);
    return cudaGetLastError();
}

}  // namespace jfa
