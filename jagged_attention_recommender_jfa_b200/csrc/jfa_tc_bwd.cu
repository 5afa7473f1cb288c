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
//                      dQ_t = dS K  -> staged in shared memory (fp32,
//                             128B-swizzled 32-column chunks) and added to
//                             the fp32 accumulator by TMA reduce-add
//   tc_bwd_dq_finalize  dQ = bf16(scale * accumulator).
//
// Warp roles: warp 0 TMA, warp 1 MMA, warps 2..17 score warps in four groups
// of four; a thread owns one key row (or, for dQ, one query row) and one
// 32-column chunk of it.  The backward needs no row reduction (LSE and D are
// given), so the chunks never talk.
// TMEM columns: dV [0,128), dK [128,256), S^T and dQ_t [256,384), dP^T [384,512).
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
constexpr uint32_t kOffQ = kOffV + kTile;
constexpr uint32_t kOffDO = kOffQ + kTile;
constexpr uint32_t kOffPT = kOffDO + kTile;
constexpr uint32_t kOffDST = kOffPT + kTile;
constexpr uint32_t kOffBar = kOffDST + kTile;  // 196608
constexpr uint32_t kOffRow = kOffBar + 256;     // lse2[2][128], D[2][128] (double-buffered)
constexpr uint32_t kOffEnd = kOffRow + 2048;
constexpr float kLog2e = 1.4426950408889634f;

struct Bars {
    uint64_t kv_full;
    uint64_t q_full;
    uint64_t q_empty;
    uint64_t do_full;
    uint64_t do_empty;
    uint64_t s_full;
    uint64_t ds_full;
    uint64_t dq_full;
    uint64_t dq_empty;
    uint64_t stage_free;
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
    CUtensorMap tm_dq;  // fp32 accumulator, boxes of 32 columns x 128 rows, 128B swizzle
    AttnArgs a;
    int tab_cap;  // bias table entries that fit in shared memory
};

__device__ __forceinline__ uint64_t kmajor_desc(uint32_t tile_base, int k) {
    return smem_desc_sw128(tile_base + (uint32_t)(k >> 2) * kBox + (uint32_t)(k & 3) * 32u, 16u,
                           1024u);
}

__device__ __forceinline__ uint64_t mnmajor_desc(uint32_t tile_base, int k) {
    return smem_desc_sw128(tile_base + (uint32_t)k * 2048u, kBox, 1024u);
}

__device__ __forceinline__ void named_sync_score() {
    asm volatile("bar.sync 1, %0;" ::"n"(NG * 128) : "memory");
}

// TMA reduce-add of a shared-memory tile into global memory (no multicast).
__device__ __forceinline__ void tma_reduce_add_3d(const CUtensorMap* map, const void* src, int x,
                                                  int y, int z) {
    asm volatile(
        "cp.reduce.async.bulk.tensor.3d.global.shared::cta.add.tile.bulk_group"
        " [%0, {%2, %3, %4}], [%1];" ::"l"(reinterpret_cast<uint64_t>(map)),
        "r"(smem_u32(src)), "r"(x), "r"(y), "r"(z)
        : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read_all() {
    asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// Stores 16 fp32 values (bit patterns) as bf16: columns 16*c16 .. +15 of row r
// of a K-major 128B-swizzled tile.
__device__ __forceinline__ void store_half_chunk_bits(uint8_t* tile, int r, int c16, const uint32_t (&v)[16]) {
    uint8_t* row = tile + (c16 >> 2) * kBox + r * 128;
#pragma unroll
    for (int u = 0; u < 2; ++u) {
        const int ch = (c16 & 3) * 2 + u;
        uint4 w;
        w.x = pack_bf16_p(__uint_as_float(v[8 * u + 0]), __uint_as_float(v[8 * u + 1]));
        w.y = pack_bf16_p(__uint_as_float(v[8 * u + 2]), __uint_as_float(v[8 * u + 3]));
        w.z = pack_bf16_p(__uint_as_float(v[8 * u + 4]), __uint_as_float(v[8 * u + 5]));
        w.w = pack_bf16_p(__uint_as_float(v[8 * u + 6]), __uint_as_float(v[8 * u + 7]));
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

// BIAS: 0 none, 1 relative-position, 2 dense jagged.  SOFTMAX: softmax (true)
// or GDPA.
template <int BIAS, bool SOFTMAX>
__global__ void __launch_bounds__(kThreads, 1) tc_bwd_kernel(const __grid_constant__ BwdParams P) {
    const AttnArgs& a = P.a;
    if ((int)blockIdx.x >= *a.item_count || a.hdr->err != 0) return;
    extern __shared__ uint8_t smem_dyn[];
    uint8_t* smem = smem_dyn + ((1024u - (smem_u32(smem_dyn) & 1023u)) & 1023u);
    Bars* bars = reinterpret_cast<Bars*>(smem + kOffBar);
    float* lse2_s = reinterpret_cast<float*>(smem + kOffRow);  // [2][128]
    float* dd_s = lse2_s + 256;                                 // [2][128]

    const int4 it = a.items[blockIdx.x];
    const int b = it.x, h = it.y, j0 = it.z * BN;
    const int q0 = a.q_off[b], nq = a.q_off[b + 1] - q0;
    const int k0 = a.kv_off[b], nkv = a.kv_off[b + 1] - k0;
    const int shift = nkv - nq;  // causal: key j visible from query i iff j <= i + shift
    const int i_start = a.causal ? max(0, j0 - shift) : 0;
    const int nt = nq > i_start ? (nq - i_start + BM - 1) / BM : 0;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    constexpr bool softmax = SOFTMAX;
    // relative-position bias of this CTA's (query, key) range, log2(e)-scaled:
    // tab[t] = bias(i, j) for i - j = tab_lo + t, kept in shared memory when
    // it fits
    const int tab_lo = i_start - j0 - (BN - 1);
    const int tab_len = nq - i_start + BN - 1;
    const bool tab_in_smem = BIAS == 1 && nt > 0 && tab_len <= P.tab_cap;
    float* tab = reinterpret_cast<float*>(smem + kOffEnd);

    if (threadIdx.x == 0) {
        mbar_init(&bars->kv_full, 1);
        mbar_init(&bars->q_full, 1);
        mbar_init(&bars->q_empty, 1);
        mbar_init(&bars->do_full, 1);
        mbar_init(&bars->do_empty, 1);
        mbar_init(&bars->s_full, 1);
        mbar_init(&bars->ds_full, NG * 4);
        mbar_init(&bars->dq_full, 1);
        mbar_init(&bars->dq_empty, NG * 4);
        mbar_init(&bars->stage_free, 1);
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
        const float* src = a.bias4 + (int64_t)h * 4 * a.bias4_stride;   // copy 0
        for (int t = threadIdx.x; t < tab_len; t += kThreads)
            tab[t] = __ldg(src + min(max(tab_lo + t, -C), C) + C);
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
            tma_prefetch_desc(&P.tm_dq);
            mbar_arrive_expect_tx(&bars->kv_full, 2 * kTile);
            tma_load_3d(smem + kOffK, &P.tm_k, &bars->kv_full, 0, h, k0 + j0);
            tma_load_3d(smem + kOffK + kBox, &P.tm_k, &bars->kv_full, 64, h, k0 + j0);
            tma_load_3d(smem + kOffV, &P.tm_v, &bars->kv_full, 0, h, k0 + j0);
            tma_load_3d(smem + kOffV + kBox, &P.tm_v, &bars->kv_full, 64, h, k0 + j0);
            // Q of tile t+1 is loaded as soon as dK += dS^T Q of tile t has retired,
            // dO as soon as dV += P^T dO has (the MMAs of a tile run dK, dV, dQ)
            int issued_q = 0, issued_do = 0;
            for (int t = 0; t < nt; ++t) {
                const int z = q0 + i_start + t * BM;
                if (t > 0 && !mbar_wait(&bars->q_empty, (t - 1) & 1, abort_flag, a.hdr)) break;
                JFA_TRACE_EV(bwd, 0, t, 0);
                mbar_arrive_expect_tx(&bars->q_full, kTile);
                tma_load_3d(smem + kOffQ, &P.tm_q, &bars->q_full, 0, h, z);
                tma_load_3d(smem + kOffQ + kBox, &P.tm_q, &bars->q_full, 64, h, z);
                issued_q = t + 1;
                if (t > 0 && !mbar_wait(&bars->do_empty, (t - 1) & 1, abort_flag, a.hdr)) break;
                JFA_TRACE_EV(bwd, 0, t, 1);
                mbar_arrive_expect_tx(&bars->do_full, kTile);
                tma_load_3d(smem + kOffDO, &P.tm_do, &bars->do_full, 0, h, z);
                tma_load_3d(smem + kOffDO + kBox, &P.tm_do, &bars->do_full, 64, h, z);
                issued_do = t + 1;
                if (t + 1 < nt) {  // warm L2 for the next query tile (single-buffered)
                    tma_prefetch_l2_3d(&P.tm_q, 0, h, z + BM);
                    tma_prefetch_l2_3d(&P.tm_q, 64, h, z + BM);
                    tma_prefetch_l2_3d(&P.tm_do, 0, h, z + BM);
                    tma_prefetch_l2_3d(&P.tm_do, 64, h, z + BM);
                }
            }
            mbar_wait_drain(&bars->kv_full, 0, a.hdr);
            if (issued_q > 0) mbar_wait_drain(&bars->q_full, (issued_q - 1) & 1, a.hdr);
            if (issued_do > 0) mbar_wait_drain(&bars->do_full, (issued_do - 1) & 1, a.hdr);
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
                JFA_TRACE_EV(bwd, 1, t, 0);
                if (t > 0 && !mbar_wait(&bars->dq_empty, (t - 1) & 1, abort_flag, a.hdr)) { ok = false; break; }
                JFA_TRACE_EV(bwd, 1, t, 1);
                tc_fence_after();
#pragma unroll
                for (int k = 0; k < HD / 16; ++k)
                    mma_bf16_ss(tS, kmajor_desc(kb, k), kmajor_desc(qb, k), idesc_nt, k > 0 ? 1u : 0u);
                if (!mbar_wait(&bars->do_full, t & 1, abort_flag, a.hdr)) { ok = false; break; }
                JFA_TRACE_EV(bwd, 1, t, 2);
                tc_fence_after();
#pragma unroll
                for (int k = 0; k < HD / 16; ++k)
                    mma_bf16_ss(tdP, kmajor_desc(vb, k), kmajor_desc(dob, k), idesc_nt, k > 0 ? 1u : 0u);
                mma_commit(&bars->s_full);
                JFA_TRACE_EV(bwd, 1, t, 3);
                if (!mbar_wait(&bars->ds_full, t & 1, abort_flag, a.hdr)) { ok = false; break; }
                JFA_TRACE_EV(bwd, 1, t, 4);
                tc_fence_after();
#pragma unroll
                for (int k = 0; k < BM / 16; ++k)
                    mma_bf16_ss(tdK, kmajor_desc(dsb, k), mnmajor_desc(qb, k), idesc_nn,
                                (t > 0 || k > 0) ? 1u : 0u);
                mma_commit(&bars->q_empty);
#pragma unroll
                for (int k = 0; k < BM / 16; ++k)
                    mma_bf16_ss(tdV, kmajor_desc(ptb, k), mnmajor_desc(dob, k), idesc_nn,
                                (t > 0 || k > 0) ? 1u : 0u);
                mma_commit(&bars->do_empty);
#pragma unroll
                for (int k = 0; k < BN / 16; ++k)
                    mma_bf16_ss(tS, mnmajor_desc(dsb, k), mnmajor_desc(kb, k), idesc_tn, k > 0 ? 1u : 0u);
                mma_commit(&bars->dq_full);
                JFA_TRACE_EV(bwd, 1, t, 5);
            }
            if (ok) mma_commit(&bars->fin);
            mma_commit(&bars->drain);
            mbar_wait_drain(&bars->drain, 0, a.hdr);
        }
    } else {
        // ------------------------------------------------ score warps
        const int wq = warp & 3;                 // TMEM lane quarter
        const int grp = (warp - 2) >> 2;         // 32-column chunk of the row
        const int r = wq * 32 + lane;            // key row (S^T, dV, dK) / query row (dQ)
        const int j = j0 + r;                    // key index within the sequence
        const bool jvalid = j < nkv;
        const uint32_t lane_addr = (uint32_t)(wq * 32) << 16;
        const uint32_t cofs = (uint32_t)grp * 32;
        const uint32_t tdV = tmem + lane_addr + cofs, tdK = tmem + lane_addr + 128 + cofs;
        const uint32_t tS = tmem + lane_addr + 256 + cofs, tdP = tmem + lane_addr + 384 + cofs;
        const float sc = a.scale * kLog2e;
        const float inv_n = nkv > 0 ? 1.0f / (float)nkv : 0.f;
        const int C = (a.relpos_len - 1) >> 1;
        // log2(e)-scaled table (copy 0 of the four shifted copies)
        const float* tab4 = (BIAS == 1) ? a.bias4 + (int64_t)h * 4 * a.bias4_stride : nullptr;
        const __nv_bfloat16* dense = reinterpret_cast<const __nv_bfloat16*>(a.bias);
        const int64_t dense_base = (BIAS == 2) ? a.dense_off[b] + (int64_t)h * nq * nkv : 0;
        const bool leader = (warp == 2 && lane == 0);
        bool ok = true;
        // LSE (log2 units) and D of a query tile, staged by group 0 into one of
        // two buffers; the next tile's values are fetched a tile ahead.
        auto fetch_rowstats = [&](int t, float& l2, float& dv) {
            const int qi = i_start + t * BM + r;
            l2 = CUDART_INF_F;
            dv = 0.f;
            if (qi < nq && softmax) {
                l2 = a.lse[(int64_t)(q0 + qi) * a.H + h] * kLog2e;
                dv = a.dterm[(int64_t)(q0 + qi) * a.H + h];
            }
        };
        if (nt > 0) {
            if (grp == 0) {
                float l2, dv;
                fetch_rowstats(0, l2, dv);
                lse2_s[r] = l2;
                dd_s[r] = dv;
            }
            named_sync_score();
        }
        const int tslot = (warp == 2 && lane == 0) ? 2 : ((warp == kThreads / 32 - 1 && lane == 0) ? 3 : -1);
#define SC_EV(ev)                                     \
    do {                                              \
        if (tslot >= 0) JFA_TRACE_EV(bwd, tslot, t, ev); \
    } while (0)
        for (int t = 0; t < nt; ++t) {
            SC_EV(0);
            const int qb0 = i_start + t * BM;    // query index of the tile's row 0
            const int buf = t & 1;
            float nl2 = CUDART_INF_F, ndv = 0.f;
            if (grp == 0 && t + 1 < nt) fetch_rowstats(t + 1, nl2, ndv);
            // failed waits below only set the CTA's abort flag; the loop is left
            // right after the named barrier, so every score warp runs the same
            // sequence of barriers
            mbar_wait(&bars->s_full, t & 1, abort_flag, a.hdr);
            SC_EV(1);
            tc_fence_after();
            // key rows past the sequence end (neighbour data) must not reach dS K;
            // S^T = K Q^T of the first tile has completed, so K may be edited now
            if (t == 0 && grp == 0 && !jvalid) zero_row(smem + kOffK, r);
            // the previous tile's dQ reduce must have read its staging (which
            // overlays the P^T / dS^T buffers) before they are rewritten
            if (t > 0) {
                if (leader) {
                    bulk_wait_read_all();
                    mbar_arrive(&bars->stage_free);
                }
                mbar_wait(&bars->stage_free, (t - 1) & 1, abort_flag, a.hdr);
            }
            SC_EV(2);
            const int imin_vis = a.causal ? j - shift : 0;  // queries i >= imin_vis see key j
            // one 16-column part: scores u (TMEM bits) -> P in place, dP g -> dS in place
            auto process = [&](uint32_t (&u)[16], uint32_t (&g)[16], int c16) {
                const int qc0 = qb0 + c16 * 16;      // query index of the part's column 0
                const bool all_vis = jvalid && (qc0 + 15 < nq) && (qc0 >= imin_vis);
                const bool none_vis = !jvalid || qc0 >= nq || (qc0 + 15 < imin_vis);
                if (none_vis) {
#pragma unroll
                    for (int v = 0; v < 16; ++v) u[v] = 0u, g[v] = 0u;
                    return;
                }
                float x[16];
                const float2 sc2 = make_float2(sc, sc);
                if (BIAS == 1) {
                    float bb[16];
                    if (tab_in_smem) {
                        const float* tb = tab + (qc0 - j - tab_lo);   // tb[v] = bias(qc0 + v, j)
#pragma unroll
                        for (int v = 0; v < 16; ++v) bb[v] = tb[v];
                    } else {
                        const int s0 = qc0 - j + C;                   // table index of bias(qc0, j)
#pragma unroll
                        for (int v = 0; v < 16; ++v) bb[v] = __ldg(tab4 + min(max(s0 + v, 0), 2 * C));
                    }
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const float2 r2 = fma2(make_float2(__uint_as_float(u[2 * e]), __uint_as_float(u[2 * e + 1])),
                                               sc2, make_float2(bb[2 * e], bb[2 * e + 1]));
                        x[2 * e] = r2.x, x[2 * e + 1] = r2.y;
                    }
                } else if (BIAS == 2) {
#pragma unroll
                    for (int v = 0; v < 16; ++v) {
                        const int qi = qc0 + v;
                        const float bv = (jvalid && qi < nq)
                            ? __bfloat162float(dense[dense_base + (int64_t)qi * nkv + j]) * kLog2e : 0.f;
                        x[v] = fmaf(__uint_as_float(u[v]), sc, bv);
                    }
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
                        u[v] = __float_as_uint(act_f(a.act, sn) * inv_n);
                        g[v] = __float_as_uint(__uint_as_float(g[v]) * act_grad_f(a.act, sn) * inv_n);
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
            };
#pragma unroll 1
            for (int hh = 0; hh < 2; ++hh) {
                uint32_t u[16], g[16];
                tmem_ld16(tS + hh * 16, u);
                tmem_ld16(tdP + hh * 16, g);
                tmem_wait_ld();
                const int c16 = grp * 2 + hh;
                process(u, g, c16);
                store_half_chunk_bits(smem + kOffPT, r, c16, u);
                store_half_chunk_bits(smem + kOffDST, r, c16, g);
            }
            // query rows past the sequence end must not reach dV / dK
            if (qb0 + r >= nq) {
                if (grp == 0) zero_row(smem + kOffQ, r);
                else if (grp == 1) zero_row(smem + kOffDO, r);
            }
            SC_EV(3);
            fence_proxy_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->ds_full);
            // dQ of this query tile: TMEM row r = query qb0 + r; staged as fp32
            // 32-column chunks (128B swizzle) over the P^T / dS^T buffers, which
            // the finished MMAs no longer read
            mbar_wait(&bars->dq_full, t & 1, abort_flag, a.hdr);
            SC_EV(4);
            tc_fence_after();
            const bool qvalid = qb0 + r < nq;
            uint32_t u2[32];
            tmem_ld32(tS, u2);
            tmem_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->dq_empty);  // TMEM columns free for S^T of t+1
            SC_EV(5);
            {
                uint8_t* row = smem + kOffPT + grp * (128 * 128) + r * 128;
#pragma unroll
                for (int v = 0; v < 8; ++v) {
                    uint4 w = qvalid ? make_uint4(u2[4 * v], u2[4 * v + 1], u2[4 * v + 2], u2[4 * v + 3])
                                     : make_uint4(0, 0, 0, 0);
                    *reinterpret_cast<uint4*>(row + ((v ^ (r & 7)) << 4)) = w;
                }
            }
            if (grp == 0 && t + 1 < nt) {
                lse2_s[(buf ^ 1) * 128 + r] = nl2;
                dd_s[(buf ^ 1) * 128 + r] = ndv;
            }
            fence_proxy_async_smem();
            SC_EV(6);
            named_sync_score();
            SC_EV(7);
            if (*abort_flag) { ok = false; break; }
            if (leader) {
                const int z = q0 + qb0;
#pragma unroll
                for (int c4 = 0; c4 < 4; ++c4)
                    tma_reduce_add_3d(&P.tm_dq, smem + kOffPT + c4 * (128 * 128), c4 * 32, h, z);
                bulk_commit();
            }
        }
#undef SC_EV
        if (leader) bulk_wait_all();
        // ------------------------------------------------------ epilogue
        if (ok && nt > 0) ok = __all_sync(0xffffffffu, mbar_wait(&bars->fin, 0, abort_flag, a.hdr));
        if (ok && !*abort_flag) {
            tc_fence_after();
            __nv_bfloat16* dkrow = reinterpret_cast<__nv_bfloat16*>(a.dk) + ((int64_t)(k0 + j) * a.H + h) * HD + cofs;
            __nv_bfloat16* dvrow = reinterpret_cast<__nv_bfloat16*>(a.dv) + ((int64_t)(k0 + j) * a.H + h) * HD + cofs;
            {
                const int cc = 0;
                uint32_t uk[32], uv[32];
                if (nt > 0) {
                    tmem_ld32(tdK, uk);
                    tmem_ld32(tdV, uv);
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
                        *reinterpret_cast<uint4*>(dkrow + cc * 32 + t) = wk;
                        *reinterpret_cast<uint4*>(dvrow + cc * 32 + t) = wv;
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


// fp32 accumulator [rows][heads][128] as a 3-D tensor (d, head, row); boxes of
// 32 d x 1 head x 128 rows (128 bytes inner) with the 128-byte swizzle.
static bool make_tmap_dq_acc(CUtensorMap* map, void* base, int64_t rows, int heads) {
    typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                      const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                      const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                      CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return false;
        fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    cuuint64_t dims[3] = {(cuuint64_t)HD, (cuuint64_t)heads, (cuuint64_t)(rows > 0 ? rows : 1)};
    cuuint64_t strides[2] = {(cuuint64_t)HD * 4, (cuuint64_t)heads * HD * 4};
    cuuint32_t box[3] = {32, 1, 128};
    cuuint32_t estr[3] = {1, 1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, base, dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

constexpr int kSmemLimit = 232448;  // opt-in shared memory per block

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
    if (!make_tmap_dq_acc(&P.tm_dq, a.dq_acc, p.total_q, p.heads)) return cudaErrorInvalidValue;
    P.a = kv;
    const int base = 1024 + (int)kOffEnd;
    int tab_need = (p.bias_kind == JFA_BIAS_RELPOS) ? (p.max_q_len + BN - 1) : 0;
    int smem = base + 4 * tab_need;
    if (smem > kSmemLimit) {
        tab_need = (kSmemLimit - base) / 4;
        smem = kSmemLimit;
    }
    P.tab_cap = tab_need;
    const int bias = p.bias_kind == JFA_BIAS_RELPOS ? 1 : (p.bias_kind == JFA_BIAS_DENSE_JAGGED ? 2 : 0);
    const bool sm = a.act == JFA_ACT_SOFTMAX;
    void (*kern)(BwdParams) = nullptr;
    if (bias == 0) kern = sm ? tc_bwd_kernel<0, true> : tc_bwd_kernel<0, false>;
    else if (bias == 1) kern = sm ? tc_bwd_kernel<1, true> : tc_bwd_kernel<1, false>;
    else kern = sm ? tc_bwd_kernel<2, true> : tc_bwd_kernel<2, false>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    int64_t grid = pairs_bound(p.batch, p.max_kv_len, p.total_kv, BN) * p.heads;
    if (grid > 0x7fffffff) return cudaErrorInvalidValue;
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
