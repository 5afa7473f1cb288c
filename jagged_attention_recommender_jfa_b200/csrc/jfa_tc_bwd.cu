// Tensor-core (tcgen05) jagged attention backward for bf16, head_dim 128.
//
// Removing padding exposes backward accumulation as a bottleneck ("Meta GEM
// Training Efficiency: Why LLM-Scale Recommenders Need a Different Stack",
// section "Bottleneck move 1").  Three kernels:
//
//   tc_bwd_pre       D[t,h] = sum_d dO*O (softmax) with a warp-shuffle row
//                    reduction; zeroes the fp32 dQ accumulator rows.
//   tc_bwd_kernel    one CTA per (sequence, head, 128-key tile) work item of
//                    the longest-first key-tile schedule.  K and V of the tile
//                    stay in shared memory; the query tiles that can see the
//                    keys stream through:
//                      S^T  = K Q^T,  dP^T = V dO^T           (TMEM, fp32)
//                      P^T  = exp2(S^T - LSE), dS^T = P^T (dP^T - D)
//                             (or GDPA: act(S)/n_kv, dP act'(S)/n_kv)
//                      dV  += P^T dO,  dK += dS^T Q             (TMEM)
//                      dQ_t = dS K  -> added to the fp32 accumulator with
//                             vector reductions (red.global.add.v4.f32)
//   tc_bwd_dq_finalize  dQ = bf16(scale * accumulator).
//
// Warp roles as in the forward: warp 0 TMA, warp 1 MMA, warps 2..5 one
// key row (or, for dQ, one query row) per thread.
// TMEM columns: dV [0,128), dK [128,256), S^T and dQ_t [256,384), dP^T [384,512).
#include <math_constants.h>

#include "jfa_sm100.cuh"

namespace jfa {

using namespace sm100;

bool make_tmap_rows_heads_d(CUtensorMap* map, const void* base, int64_t rows, int heads);

namespace {

constexpr int BM = 128, BN = 128, HD = 128;
constexpr int kThreads = 192;
constexpr uint32_t kBox = 128 * 128;
constexpr uint32_t kTile = 2 * kBox;
constexpr uint32_t kOffK = 0;
constexpr uint32_t kOffV = kOffK + kTile;
constexpr uint32_t kOffQ = kOffV + kTile;
constexpr uint32_t kOffDO = kOffQ + kTile;
constexpr uint32_t kOffPT = kOffDO + kTile;
constexpr uint32_t kOffDST = kOffPT + kTile;
constexpr uint32_t kOffBar = kOffDST + kTile;  // 196608
constexpr uint32_t kOffRow = kOffBar + 256;     // lse2[128], D[128]
constexpr uint32_t kOffTab = kOffRow + 1024;
constexpr float kLog2e = 1.4426950408889634f;

struct Bars {
    uint64_t kv_full;
    uint64_t q_full;
    uint64_t q_empty;
    uint64_t s_full;
    uint64_t ds_full;
    uint64_t dq_full;
    uint64_t dq_empty;
    uint64_t fin;
    uint64_t drain;
    uint32_t tmem_base;
    int abort_flag;
};

struct BwdParams {
    CUtensorMap tm_q;
    CUtensorMap tm_k;
    CUtensorMap tm_v;
    CUtensorMap tm_do;
    AttnArgs a;
    int tab_cap;
};

__device__ __forceinline__ uint64_t kmajor_desc(uint32_t tile_base, int k) {
    return smem_desc_sw128(tile_base + (uint32_t)(k >> 2) * kBox + (uint32_t)(k & 3) * 32u, 16u,
                           1024u);
}

__device__ __forceinline__ uint64_t mnmajor_desc(uint32_t tile_base, int k) {
    return smem_desc_sw128(tile_base + (uint32_t)k * 2048u, kBox, 1024u);
}

__device__ __forceinline__ void red_add_v4(float* addr, float a, float b, float c, float d) {
    asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(addr), "f"(a), "f"(b), "f"(c),
                 "f"(d)
                 : "memory");
}

__device__ __forceinline__ void named_sync_softmax() {
    asm volatile("bar.sync 1, 128;" ::: "memory");
}

// Stores the 32 values of chunk c4 (columns 32*c4 .. +31) of row r into a
// K-major 128B-swizzled bf16 tile.
__device__ __forceinline__ void store_chunk_bf16(uint8_t* tile, int r, int c4, const float (&v)[32]) {
    uint8_t* row = tile + (c4 >> 1) * kBox + r * 128;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        const int ch = (c4 & 1) * 4 + u;
        uint4 w;
        w.x = pack_bf16(v[8 * u + 0], v[8 * u + 1]);
        w.y = pack_bf16(v[8 * u + 2], v[8 * u + 3]);
        w.z = pack_bf16(v[8 * u + 4], v[8 * u + 5]);
        w.w = pack_bf16(v[8 * u + 6], v[8 * u + 7]);
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

__global__ void __launch_bounds__(kThreads, 1) tc_bwd_kernel(const __grid_constant__ BwdParams P) {
    const AttnArgs& a = P.a;
    if ((int)blockIdx.x >= *a.item_count || a.hdr->err != 0) return;
    extern __shared__ uint8_t smem_dyn[];
    uint8_t* smem = smem_dyn + ((1024u - (smem_u32(smem_dyn) & 1023u)) & 1023u);
    Bars* bars = reinterpret_cast<Bars*>(smem + kOffBar);
    float* lse2_s = reinterpret_cast<float*>(smem + kOffRow);
    float* dd_s = lse2_s + 128;
    float* tab = reinterpret_cast<float*>(smem + kOffTab);

    const int4 it = a.items[blockIdx.x];
    const int b = it.x, h = it.y, j0 = it.z * BN;
    const int q0 = a.q_off[b], nq = a.q_off[b + 1] - q0;
    const int k0 = a.kv_off[b], nkv = a.kv_off[b + 1] - k0;
    const int shift = nkv - nq;  // causal: key j visible from query i iff j <= i + shift
    const int i_start = a.causal ? max(0, j0 - shift) : 0;
    const int nt = nq > i_start ? (nq - i_start + BM - 1) / BM : 0;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const bool softmax = a.act == JFA_ACT_SOFTMAX;
    const int tab_lo = i_start - j0 - (BN - 1);
    const int tab_len = nq - i_start + BN - 1;
    const bool tab_in_smem = a.bias_kind == JFA_BIAS_RELPOS && nt > 0 && tab_len <= P.tab_cap;

    if (threadIdx.x == 0) {
        mbar_init(&bars->kv_full, 1);
        mbar_init(&bars->q_full, 1);
        mbar_init(&bars->q_empty, 1);
        mbar_init(&bars->s_full, 1);
        mbar_init(&bars->ds_full, 4);
        mbar_init(&bars->dq_full, 1);
        mbar_init(&bars->dq_empty, 4);
        mbar_init(&bars->fin, 1);
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
        if (lane == 0 && nt > 0) {
            tma_prefetch_desc(&P.tm_q);
            tma_prefetch_desc(&P.tm_k);
            tma_prefetch_desc(&P.tm_v);
            tma_prefetch_desc(&P.tm_do);
            mbar_arrive_expect_tx(&bars->kv_full, 2 * kTile);
            tma_load_3d(smem + kOffK, &P.tm_k, &bars->kv_full, 0, h, k0 + j0);
            tma_load_3d(smem + kOffK + kBox, &P.tm_k, &bars->kv_full, 64, h, k0 + j0);
            tma_load_3d(smem + kOffV, &P.tm_v, &bars->kv_full, 0, h, k0 + j0);
            tma_load_3d(smem + kOffV + kBox, &P.tm_v, &bars->kv_full, 64, h, k0 + j0);
            int issued = 0;
            for (int t = 0; t < nt; ++t) {
                if (t > 0 && !mbar_wait(&bars->q_empty, (t - 1) & 1, abort_flag, a.hdr)) break;
                const int z = q0 + i_start + t * BM;
                mbar_arrive_expect_tx(&bars->q_full, 2 * kTile);
                tma_load_3d(smem + kOffQ, &P.tm_q, &bars->q_full, 0, h, z);
                tma_load_3d(smem + kOffQ + kBox, &P.tm_q, &bars->q_full, 64, h, z);
                tma_load_3d(smem + kOffDO, &P.tm_do, &bars->q_full, 0, h, z);
                tma_load_3d(smem + kOffDO + kBox, &P.tm_do, &bars->q_full, 64, h, z);
                issued = t + 1;
            }
            mbar_wait_drain(&bars->kv_full, 0, a.hdr);
            if (issued > 0) mbar_wait_drain(&bars->q_full, (issued - 1) & 1, a.hdr);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA
        if (lane == 0 && nt > 0) {
            constexpr uint32_t idesc_nt = idesc_bf16(128, 128, 0, 0);  // K-major x K-major
            constexpr uint32_t idesc_nn = idesc_bf16(128, 128, 0, 1);  // B MN-major
            constexpr uint32_t idesc_tn = idesc_bf16(128, 128, 1, 1);  // A and B MN-major
            const uint32_t tdV = tmem, tdK = tmem + 128, tS = tmem + 256, tdP = tmem + 384;
            const uint32_t kb = sbase + kOffK, vb = sbase + kOffV, qb = sbase + kOffQ,
                           dob = sbase + kOffDO, ptb = sbase + kOffPT, dsb = sbase + kOffDST;
            bool ok = mbar_wait(&bars->kv_full, 0, abort_flag, a.hdr);
            for (int t = 0; ok && t < nt; ++t) {
                if (!mbar_wait(&bars->q_full, t & 1, abort_flag, a.hdr)) { ok = false; break; }
                if (t > 0 && !mbar_wait(&bars->dq_empty, (t - 1) & 1, abort_flag, a.hdr)) { ok = false; break; }
                tc_fence_after();
#pragma unroll
                for (int k = 0; k < HD / 16; ++k)
                    mma_bf16_ss(tS, kmajor_desc(kb, k), kmajor_desc(qb, k), idesc_nt, k > 0 ? 1u : 0u);
#pragma unroll
                for (int k = 0; k < HD / 16; ++k)
                    mma_bf16_ss(tdP, kmajor_desc(vb, k), kmajor_desc(dob, k), idesc_nt, k > 0 ? 1u : 0u);
                mma_commit(&bars->s_full);
                if (!mbar_wait(&bars->ds_full, t & 1, abort_flag, a.hdr)) { ok = false; break; }
                tc_fence_after();
#pragma unroll
                for (int k = 0; k < BM / 16; ++k)
                    mma_bf16_ss(tdV, kmajor_desc(ptb, k), mnmajor_desc(dob, k), idesc_nn,
                                (t > 0 || k > 0) ? 1u : 0u);
#pragma unroll
                for (int k = 0; k < BM / 16; ++k)
                    mma_bf16_ss(tdK, kmajor_desc(dsb, k), mnmajor_desc(qb, k), idesc_nn,
                                (t > 0 || k > 0) ? 1u : 0u);
#pragma unroll
                for (int k = 0; k < BN / 16; ++k)
                    mma_bf16_ss(tS, mnmajor_desc(dsb, k), mnmajor_desc(kb, k), idesc_tn, k > 0 ? 1u : 0u);
                mma_commit(&bars->q_empty);
                mma_commit(&bars->dq_full);
            }
            if (ok) mma_commit(&bars->fin);
            mma_commit(&bars->drain);
            mbar_wait_drain(&bars->drain, 0, a.hdr);
        }
    } else {
        // ------------------------------------------------ score warps
        const int wq = warp & 3;
        const int r = wq * 32 + lane;            // key row (S^T, dV, dK) / query row (dQ)
        const int j = j0 + r;                    // key index within the sequence
        const bool jvalid = j < nkv;
        const uint32_t lane_addr = (uint32_t)(wq * 32) << 16;
        const uint32_t tdV = tmem + lane_addr, tdK = tmem + lane_addr + 128;
        const uint32_t tS = tmem + lane_addr + 256, tdP = tmem + lane_addr + 384;
        const float sc = a.scale * kLog2e;
        const float inv_n = nkv > 0 ? 1.0f / (float)nkv : 0.f;
        const int C = (a.relpos_len - 1) >> 1;
        const float* tab_g = reinterpret_cast<const float*>(a.bias) + (int64_t)h * a.relpos_len;
        const __nv_bfloat16* dense = reinterpret_cast<const __nv_bfloat16*>(a.bias);
        const int64_t dense_base = (a.bias_kind == JFA_BIAS_DENSE_JAGGED) ? a.dense_off[b] + (int64_t)h * nq * nkv : 0;
        bool ok = true;
        for (int t = 0; ok && t < nt; ++t) {
            const int qb0 = i_start + t * BM;    // query index of the tile's row 0
            {
                const int qi = qb0 + r;
                float l2 = CUDART_INF_F, dv = 0.f;
                if (qi < nq && softmax) {
                    const float lse = a.lse[(int64_t)(q0 + qi) * a.H + h];
                    l2 = lse * kLog2e;
                    dv = a.dterm[(int64_t)(q0 + qi) * a.H + h];
                }
                lse2_s[r] = l2;
                dd_s[r] = dv;
            }
            named_sync_softmax();
            ok = __all_sync(0xffffffffu, mbar_wait(&bars->s_full, t & 1, abort_flag, a.hdr));
            if (!ok) break;
            tc_fence_after();
            // key rows past the sequence end (neighbour data) must not reach dS K;
            // S^T = K Q^T of the first tile has completed, so K may be edited now
            if (t == 0 && !jvalid) zero_row(smem + kOffK, r);
            const int imin_vis = a.causal ? j - shift : 0;  // queries i >= imin_vis see key j
#pragma unroll 1
            for (int c4 = 0; c4 < BM / 32; ++c4) {
                uint32_t us[32], up[32];
                tmem_ld32(tS + c4 * 32, us);
                tmem_ld32(tdP + c4 * 32, up);
                tmem_wait_ld();
                float pv[32], dsv[32];
#pragma unroll
                for (int u = 0; u < 32; ++u) {
                    const int il = c4 * 32 + u;
                    const int qi = qb0 + il;
                    const bool vis = jvalid && qi < nq && qi >= imin_vis;
                    float p = 0.f, ds = 0.f;
                    if (vis) {
                        float bias = 0.f;
                        if (a.bias_kind == JFA_BIAS_RELPOS) {
                            if (tab_in_smem) {
                                bias = tab[(qi - j) - tab_lo];
                            } else {
                                int rr = qi - j;
                                rr = rr < -C ? -C : (rr > C ? C : rr);
                                bias = __ldg(tab_g + rr + C) * kLog2e;
                            }
                        } else if (a.bias_kind == JFA_BIAS_DENSE_JAGGED) {
                            bias = __bfloat162float(dense[dense_base + (int64_t)qi * nkv + j]) * kLog2e;
                        }
                        const float s2 = fmaf(__uint_as_float(us[u]), sc, bias);
                        const float dp = __uint_as_float(up[u]);
                        if (softmax) {
                            p = ex2(s2 - lse2_s[il]);
                            ds = p * (dp - dd_s[il]);
                        } else {
                            const float sn = s2 * (1.0f / kLog2e);
                            p = act_f(a.act, sn) * inv_n;
                            ds = dp * act_grad_f(a.act, sn) * inv_n;
                        }
                    }
                    pv[u] = p;
                    dsv[u] = ds;
                }
                store_chunk_bf16(smem + kOffPT, r, c4, pv);
                store_chunk_bf16(smem + kOffDST, r, c4, dsv);
            }
            // query rows past the sequence end must not reach dV / dK
            if (qb0 + r >= nq) {
                zero_row(smem + kOffQ, r);
                zero_row(smem + kOffDO, r);
            }
            fence_proxy_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->ds_full);
            // dQ of this query tile: row r of TMEM = query qb0 + r
            ok = __all_sync(0xffffffffu, mbar_wait(&bars->dq_full, t & 1, abort_flag, a.hdr));
            if (!ok) break;
            tc_fence_after();
            const int qi = qb0 + r;
            float* acc = a.dq_acc + ((int64_t)(q0 + qi) * a.H + h) * HD;
#pragma unroll 1
            for (int c4 = 0; c4 < HD / 32; ++c4) {
                uint32_t u[32];
                tmem_ld32(tS + c4 * 32, u);
                tmem_wait_ld();
                if (qi < nq) {
#pragma unroll
                    for (int v = 0; v < 32; v += 4)
                        red_add_v4(acc + c4 * 32 + v, __uint_as_float(u[v]), __uint_as_float(u[v + 1]),
                                   __uint_as_float(u[v + 2]), __uint_as_float(u[v + 3]));
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->dq_empty);
        }
        // ------------------------------------------------------ epilogue
        if (ok && nt > 0) ok = __all_sync(0xffffffffu, mbar_wait(&bars->fin, 0, abort_flag, a.hdr));
        if (ok) {
            tc_fence_after();
            __nv_bfloat16* dkrow = reinterpret_cast<__nv_bfloat16*>(a.dk) + ((int64_t)(k0 + j) * a.H + h) * HD;
            __nv_bfloat16* dvrow = reinterpret_cast<__nv_bfloat16*>(a.dv) + ((int64_t)(k0 + j) * a.H + h) * HD;
#pragma unroll 1
            for (int c4 = 0; c4 < HD / 32; ++c4) {
                uint32_t uk[32], uv[32];
                if (nt > 0) {
                    tmem_ld32(tdK + c4 * 32, uk);
                    tmem_ld32(tdV + c4 * 32, uv);
                    tmem_wait_ld();
                } else {
#pragma unroll
                    for (int t = 0; t < 32; ++t) uk[t] = 0u, uv[t] = 0u;
                }
                if (jvalid) {
#pragma unroll
                    for (int t = 0; t < 32; t += 8) {
                        uint4 wk, wv;
                        wk.x = pack_bf16(__uint_as_float(uk[t + 0]) * a.scale, __uint_as_float(uk[t + 1]) * a.scale);
                        wk.y = pack_bf16(__uint_as_float(uk[t + 2]) * a.scale, __uint_as_float(uk[t + 3]) * a.scale);
                        wk.z = pack_bf16(__uint_as_float(uk[t + 4]) * a.scale, __uint_as_float(uk[t + 5]) * a.scale);
                        wk.w = pack_bf16(__uint_as_float(uk[t + 6]) * a.scale, __uint_as_float(uk[t + 7]) * a.scale);
                        wv.x = pack_bf16(__uint_as_float(uv[t + 0]), __uint_as_float(uv[t + 1]));
                        wv.y = pack_bf16(__uint_as_float(uv[t + 2]), __uint_as_float(uv[t + 3]));
                        wv.z = pack_bf16(__uint_as_float(uv[t + 4]), __uint_as_float(uv[t + 5]));
                        wv.w = pack_bf16(__uint_as_float(uv[t + 6]), __uint_as_float(uv[t + 7]));
                        *reinterpret_cast<uint4*>(dkrow + c4 * 32 + t) = wk;
                        *reinterpret_cast<uint4*>(dvrow + c4 * 32 + t) = wv;
                    }
                }
            }
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

constexpr int kSmemLimitBwd = 232448;

cudaError_t tc_backward_launch(const jfa_problem& p, const AttnArgs& a, const AttnArgs& kv,
                               cudaStream_t st) {
    const int64_t rows = p.total_q * p.heads;
    if (rows > 0) {
        prof_begin(st);
        tc_bwd_pre<<<(unsigned)((rows + 7) / 8), 256, 0, st>>>(
            reinterpret_cast<const __nv_bfloat16*>(a.out), reinterpret_cast<const __nv_bfloat16*>(a.dout),
            a.dterm, a.dq_acc, rows, a.act == JFA_ACT_SOFTMAX ? 1 : 0);
        prof_end(st, K_TC_BWD_PRE);
    }
    BwdParams P{};
    if (!make_tmap_rows_heads_d(&P.tm_q, a.q, p.total_q, p.heads) ||
        !make_tmap_rows_heads_d(&P.tm_k, a.k, p.total_kv, p.heads) ||
        !make_tmap_rows_heads_d(&P.tm_v, a.v, p.total_kv, p.heads) ||
        !make_tmap_rows_heads_d(&P.tm_do, a.dout, p.total_q, p.heads))
        return cudaErrorInvalidValue;
    P.a = kv;
    const int base = 1024 + (int)kOffTab;
    int tab_need = (p.bias_kind == JFA_BIAS_RELPOS) ? (p.max_q_len + BN - 1) : 0;
    int smem = base + 4 * tab_need;
    if (smem > kSmemLimitBwd) {
        tab_need = 0;
        smem = base;
    }
    P.tab_cap = tab_need;
    cudaError_t e = cudaFuncSetAttribute(tc_bwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemLimitBwd);
    if (e != cudaSuccess) return e;
    int64_t grid = pairs_bound(p.batch, p.max_kv_len, p.total_kv, BN) * p.heads;
    if (grid > 0x7fffffff) return cudaErrorInvalidValue;
    if (grid > 0) {
        prof_begin(st);
        tc_bwd_kernel<<<(unsigned)grid, kThreads, smem, st>>>(P);
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
