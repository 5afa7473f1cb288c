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

#include "jfa_sm100.cuh"

namespace jfa {

using namespace sm100;

namespace {

constexpr int BM = 128, BN = 128, HD = 128;
constexpr int NS = 2;                       // key/value stages
constexpr int kThreads = 192;
constexpr uint32_t kBox = 128 * 128;        // bytes of one [128 rows][64 bf16] box
constexpr uint32_t kTile = 2 * kBox;        // one 128 x 128 bf16 tile (two boxes)
constexpr uint32_t kOffQ = 0;
constexpr uint32_t kOffK = kOffQ + kTile;
constexpr uint32_t kOffV = kOffK + NS * kTile;
constexpr uint32_t kOffP = kOffV + NS * kTile;
constexpr uint32_t kOffBar = kOffP + kTile;  // 196608
constexpr uint32_t kOffTab = kOffBar + 256;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleThreshold = 8.0f;    // log2 units

struct Bars {
    uint64_t q_full;
    uint64_t kv_full[NS];
    uint64_t kv_empty[NS];
    uint64_t s_full;
    uint64_t p_full;
    uint64_t o_full;
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

// BIAS: 0 none, 1 relative-position (window in shared memory when it fits,
// else through L1), 2 dense jagged.  SOFTMAX: softmax (true) or GDPA.
template <int BIAS, bool SOFTMAX>
__global__ void __launch_bounds__(kThreads, 1) tc_fwd_kernel(const __grid_constant__ FwdParams P) {
    const AttnArgs& a = P.a;
    if ((int)blockIdx.x >= *a.item_count || a.hdr->err != 0) return;
    extern __shared__ uint8_t smem_dyn[];
    // 1024-byte alignment for the swizzle atoms
    uint8_t* smem = smem_dyn + ((1024u - (smem_u32(smem_dyn) & 1023u)) & 1023u);
    Bars* bars = reinterpret_cast<Bars*>(smem + kOffBar);
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
        for (int s = 0; s < NS; ++s) {
            mbar_init(&bars->kv_full[s], 1);
            mbar_init(&bars->kv_empty[s], 1);
        }
        mbar_init(&bars->s_full, 1);
        mbar_init(&bars->p_full, 4);
        mbar_init(&bars->o_full, 1);
        mbar_init(&bars->drain, 1);
        bars->abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(&bars->tmem_base, 256);
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
                const int s = j % NS;
                if (j >= NS && !mbar_wait(&bars->kv_empty[s], ((j / NS) - 1) & 1, abort_flag, a.hdr))
                    break;
                uint8_t* kd = smem + kOffK + s * kTile;
                uint8_t* vd = smem + kOffV + s * kTile;
                mbar_arrive_expect_tx(&bars->kv_full[s], 2 * kTile);
                const int z = k0 + j * BN;
                tma_load_3d(kd, &P.tm_k, &bars->kv_full[s], 0, h, z);
                tma_load_3d(kd + kBox, &P.tm_k, &bars->kv_full[s], 64, h, z);
                tma_load_3d(vd, &P.tm_v, &bars->kv_full[s], 0, h, z);
                tma_load_3d(vd + kBox, &P.tm_v, &bars->kv_full[s], 64, h, z);
                issued = j + 1;
            }
            // never leave the CTA with copies in flight: wait for every issued stage
            mbar_wait_drain(&bars->q_full, 0, a.hdr);
            for (int j = (issued > NS ? issued - NS : 0); j < issued; ++j)
                mbar_wait_drain(&bars->kv_full[j % NS], (j / NS) & 1, a.hdr);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA
        if (lane == 0 && n_tiles > 0) {
            constexpr uint32_t idesc_qk = idesc_bf16(BM, BN, 0, 0);
            constexpr uint32_t idesc_pv = idesc_bf16(BM, HD, 0, 1);
            const uint32_t tS = tmem, tO = tmem + 128;
            const uint32_t qb = sbase + kOffQ, pb = sbase + kOffP;
            bool ok = mbar_wait(&bars->q_full, 0, abort_flag, a.hdr);
            for (int j = 0; ok && j < n_tiles; ++j) {
                const int s = j % NS;
                if (!mbar_wait(&bars->kv_full[s], (j / NS) & 1, abort_flag, a.hdr)) { ok = false; break; }
                tc_fence_after();
                if (j > 0) {
                    if (!mbar_wait(&bars->p_full, (j - 1) & 1, abort_flag, a.hdr)) { ok = false; break; }
                    tc_fence_after();
                    const int sp = (j - 1) % NS;
                    const uint32_t vb = sbase + kOffV + sp * kTile;
#pragma unroll
                    for (int k = 0; k < BN / 16; ++k)
                        mma_bf16_ss(tO, kmajor_desc(pb, k), mnmajor_desc(vb, k), idesc_pv,
                                    (j - 1 > 0 || k > 0) ? 1u : 0u);
                    mma_commit(&bars->kv_empty[sp]);
                }
                const uint32_t kb = sbase + kOffK + s * kTile;
#pragma unroll
                for (int k = 0; k < HD / 16; ++k)
                    mma_bf16_ss(tS, kmajor_desc(qb, k), kmajor_desc(kb, k), idesc_qk, k > 0 ? 1u : 0u);
                mma_commit(&bars->s_full);
            }
            if (ok && mbar_wait(&bars->p_full, (n_tiles - 1) & 1, abort_flag, a.hdr)) {
                tc_fence_after();
                const int sp = (n_tiles - 1) % NS;
                const uint32_t vb = sbase + kOffV + sp * kTile;
#pragma unroll
                for (int k = 0; k < BN / 16; ++k)
                    mma_bf16_ss(tO, kmajor_desc(pb, k), mnmajor_desc(vb, k), idesc_pv,
                                (n_tiles - 1 > 0 || k > 0) ? 1u : 0u);
                mma_commit(&bars->kv_empty[sp]);
                mma_commit(&bars->o_full);
            }
            // all issued MMAs retire before TMEM is released
            mma_commit(&bars->drain);
            mbar_wait_drain(&bars->drain, 0, a.hdr);
        }
    } else {
        // ------------------------------------------------ softmax warps
        const int wq = warp & 3;                 // TMEM lane quarter
        const int r = wq * 32 + lane;            // row within the tile
        const int i = row0 + r;                  // query index within the sequence
        const uint32_t lane_addr = (uint32_t)(wq * 32) << 16;
        const uint32_t tS = tmem + lane_addr, tO = tmem + lane_addr + 128;
        const float sc = a.scale * kLog2e;
        const int shift = nkv - nq;              // causal: key j visible iff j <= i + shift
        const float inv_n = nkv > 0 ? 1.0f / (float)nkv : 0.f;
        const int C = (a.relpos_len - 1) >> 1;
        const float* tab_g = reinterpret_cast<const float*>(a.bias) + (int64_t)h * a.relpos_len;
        const __nv_bfloat16* dense = reinterpret_cast<const __nv_bfloat16*>(a.bias);
        const int64_t dense_row = (BIAS == 2 && i < nq)
                                      ? a.dense_off[b] + ((int64_t)h * nq + i) * nkv : 0;
        uint8_t* prow = smem + kOffP + r * 128;
        float m_used = -CUDART_INF_F, l = 0.f;
        bool ok = true;
        for (int j = 0; j < n_tiles; ++j) {
            ok = __all_sync(0xffffffffu, mbar_wait(&bars->s_full, j & 1, abort_flag, a.hdr));
            if (!ok) break;
            tc_fence_after();
            const int j0 = j * BN;
            float x[BN];
#pragma unroll
            for (int c4 = 0; c4 < BN / 32; ++c4) {
                uint32_t u[32];
                tmem_ld32(tS + c4 * 32, u);
                tmem_wait_ld();
#pragma unroll
                for (int t = 0; t < 32; ++t) x[c4 * 32 + t] = __uint_as_float(u[t]);
            }
            // scale, bias, mask (log2 domain for softmax, natural for GDPA)
            const int jmax_vis = a.causal ? min(nkv - 1, i + shift) : nkv - 1;  // last visible key
            const int nvis = i < nq ? min(BN, jmax_vis - j0 + 1) : 0;  // visible columns: [0, nvis)
            // bias (log2 units), added in place
            if (BIAS == 1 && tab_in_smem) {
                const float* tb = tab + (i - j0 - tab_lo);  // tb[-c] = bias(i, j0 + c)
#pragma unroll
                for (int c = 0; c < BN; ++c) x[c] = fmaf(x[c], sc, tb[-c]);
            } else if (BIAS == 1) {
#pragma unroll
                for (int c = 0; c < BN; ++c) {
                    int rr = i - (j0 + c);
                    rr = rr < -C ? -C : (rr > C ? C : rr);
                    x[c] = fmaf(x[c], sc, __ldg(tab_g + rr + C) * kLog2e);
                }
            } else if (BIAS == 2) {
#pragma unroll
                for (int c = 0; c < BN; ++c)
                    x[c] = fmaf(x[c], sc, c < nvis ? __bfloat162float(dense[dense_row + j0 + c]) * kLog2e : 0.f);
            } else {
#pragma unroll
                for (int c = 0; c < BN; ++c) x[c] *= sc;
            }
            if (__any_sync(0xffffffffu, nvis < BN)) {
#pragma unroll
                for (int c = 0; c < BN; ++c) x[c] = c < nvis ? x[c] : -CUDART_INF_F;
            }
            float tmax = -CUDART_INF_F;
#pragma unroll
            for (int c = 0; c < BN; ++c) tmax = fmaxf(tmax, x[c]);
            if (softmax) {
                // lazy rescale: keep the reference maximum unless it grew by > 2^8
                const bool need = tmax > m_used + kRescaleThreshold;
                const float m_new = need ? tmax : m_used;
                if (__any_sync(0xffffffffu, need && j > 0 && m_used != -CUDART_INF_F)) {
                    const float alpha = (need && m_used != -CUDART_INF_F) ? ex2(m_used - m_new) : 1.f;
#pragma unroll
                    for (int c4 = 0; c4 < HD / 32; ++c4) {
                        uint32_t u[32];
                        tmem_ld32(tO + c4 * 32, u);
                        tmem_wait_ld();
#pragma unroll
                        for (int t = 0; t < 32; ++t) u[t] = __float_as_uint(__uint_as_float(u[t]) * alpha);
                        tmem_st32(tO + c4 * 32, u);
                    }
                    tmem_wait_st();
                    l *= alpha;
                } else if (need) {
                    // first tile with a visible key: nothing accumulated yet
                    l = 0.f;
                }
                m_used = m_new;
                // ex2(-inf) = 0 masks the invisible columns; a row with no visible
                // key yet uses reference 0 so that -inf - ref stays -inf
                const float ref = m_used == -CUDART_INF_F ? 0.f : m_used;
                float psum0 = 0.f, psum1 = 0.f;
#pragma unroll
                for (int c = 0; c < BN; c += 2) {
                    x[c] = ex2(x[c] - ref);
                    x[c + 1] = ex2(x[c + 1] - ref);
                    psum0 += x[c];
                    psum1 += x[c + 1];
                }
                l += psum0 + psum1;
            } else {
#pragma unroll
                for (int c = 0; c < BN; ++c) {
                    const float s_nat = x[c] * (1.0f / kLog2e);
                    x[c] = c < nvis ? act_f(a.act, s_nat) * inv_n : 0.f;
                }
            }
            // P row -> shared memory, K-major, 128-byte swizzle (chunk ^ row%8)
#pragma unroll
            for (int half = 0; half < 2; ++half) {
#pragma unroll
                for (int ch = 0; ch < 8; ++ch) {
                    const int c = half * 64 + ch * 8;
                    uint4 w;
                    w.x = pack_bf16(x[c + 0], x[c + 1]);
                    w.y = pack_bf16(x[c + 2], x[c + 3]);
                    w.z = pack_bf16(x[c + 4], x[c + 5]);
                    w.w = pack_bf16(x[c + 6], x[c + 7]);
                    *reinterpret_cast<uint4*>(prow + half * kBox + ((ch ^ (r & 7)) << 4)) = w;
                }
            }
            // value rows past the sequence end (neighbour data) must not reach P.V
            const int nvalid = nkv - j0;
            if (nvalid < BN && r >= nvalid) {
                uint8_t* vrow = smem + kOffV + (j % NS) * kTile + r * 128;
                const uint4 z = make_uint4(0, 0, 0, 0);
#pragma unroll
                for (int ch = 0; ch < 8; ++ch) {
                    *reinterpret_cast<uint4*>(vrow + ch * 16) = z;
                    *reinterpret_cast<uint4*>(vrow + kBox + ch * 16) = z;
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->p_full);
        }
        // ------------------------------------------------------ epilogue
        if (ok && n_tiles > 0) ok = __all_sync(0xffffffffu, mbar_wait(&bars->o_full, 0, abort_flag, a.hdr));
        if (ok) {
            tc_fence_after();
            const float inv = softmax ? (l > 0.f ? 1.f / l : 0.f) : 1.f;
            __nv_bfloat16* orow = reinterpret_cast<__nv_bfloat16*>(a.out) + ((int64_t)(q0 + i) * a.H + h) * HD;
#pragma unroll
            for (int c4 = 0; c4 < HD / 32; ++c4) {
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
            if (softmax && a.lse && i < nq)
                a.lse[(int64_t)(q0 + i) * a.H + h] =
                    l > 0.f ? m_used * (1.0f / kLog2e) + logf(l) : -CUDART_INF_F;
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 256);
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

cudaError_t tc_forward_launch(const jfa_problem& p, const AttnArgs& a, cudaStream_t st) {
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
    if (bias == 0) kern = sm ? tc_fwd_kernel<0, true> : tc_fwd_kernel<0, false>;
    else if (bias == 1) kern = sm ? tc_fwd_kernel<1, true> : tc_fwd_kernel<1, false>;
    else kern = sm ? tc_fwd_kernel<2, true> : tc_fwd_kernel<2, false>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemLimit);
    if (e != cudaSuccess) return e;
    prof_begin(st);
    kern<<<(unsigned)grid, kThreads, smem, st>>>(P);
    prof_end(st, K_TC_FWD);
    return cudaGetLastError();
}

}  // namespace jfa
