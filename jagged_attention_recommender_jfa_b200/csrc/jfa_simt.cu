// CUDA-core (fp32 arithmetic) jagged attention kernels: forward, backward
// preprocess (D = rowsum(dO * O)), dQ and dK/dV.
//
// These serve every head size (32, 64, 128), the fp32 element type, and any
// problem the tensor-core kernels do not take.  Each CTA takes one work item
// of the longest-first schedule (blockIdx.x -> items[blockIdx.x]) and works
// entirely inside one sequence, so neighbouring sequences in the packed
// buffers are never mixed in ("Meta GEM Training Efficiency: Why LLM-Scale
// Recommenders Need a Different Stack", section "Bottleneck move 1" and FAQ
// "What is a jagged tensor?").  The backward is split into a query-tile pass
// (dQ) and a key-tile pass (dK, dV) that both recompute the scores, so that
// every gradient row has exactly one writer and the result is deterministic.
//
// Thread layout (256 threads): row r = tid / 4 of the tile, quad lane
// c = tid % 4.  Score columns owned by a thread: c + 4 * jj.  Output columns:
// 16 * g + 4 * c .. +3 for g < d / 16 (conflict-free float4 reads of a
// shared-memory row by the four lanes of a row).
#include <math_constants.h>

#include "jfa_common.cuh"

namespace jfa {

namespace {

constexpr int kThreads = 256;

template <int D>
struct SimtCfg {
    static constexpr int LD = D + 4;  // padded row stride (floats) in shared memory
};

template <int D, typename T>
__device__ __forceinline__ void load_rows(float* dst, const T* src, int64_t row_stride_elems,
                                          int first_row, int n_rows_valid, int n_rows_tile) {
    constexpr int LD = SimtCfg<D>::LD;
    constexpr int V4 = D / 4;
    for (int e = threadIdx.x; e < n_rows_tile * V4; e += kThreads) {
        int rr = e / V4, cc = (e % V4) * 4;
        float4 val = make_float4(0.f, 0.f, 0.f, 0.f);
        if (rr < n_rows_valid) val = load4(src + (int64_t)(first_row + rr) * row_stride_elems + cc);
        *reinterpret_cast<float4*>(dst + rr * LD + cc) = val;
    }
}

// ---------------------------------------------------------------------------
// Forward: one CTA per (sequence, head, 64-row query tile).
// ---------------------------------------------------------------------------
template <int D, typename T>
__global__ void __launch_bounds__(kThreads) simt_fwd(AttnArgs a) {
    constexpr int BM = 64, BN = 32, LD = SimtCfg<D>::LD, G = D / 16, LP = BN + 4;
    extern __shared__ __align__(16) float sm[];
    float* Qs = sm;
    float* Ks = Qs + BM * LD;
    float* Vs = Ks + BN * LD;
    float* Ps = Vs + BN * LD;
    if ((int)blockIdx.x >= *a.item_count || a.hdr->err != 0) return;
    const int4 it = a.items[blockIdx.x];
    const int b = it.x, h = it.y, row0 = it.z * BM;
    const int q0 = a.q_off[b], nq = a.q_off[b + 1] - q0;
    const int k0 = a.kv_off[b], nkv = a.kv_off[b + 1] - k0;
    const int H = a.H;
    const int tid = threadIdx.x, r = tid >> 2, c = tid & 3;
    const int i = row0 + r;
    const T* Q = reinterpret_cast<const T*>(a.q) + (int64_t)h * D;
    const T* K = reinterpret_cast<const T*>(a.k) + (int64_t)h * D;
    const T* V = reinterpret_cast<const T*>(a.v) + (int64_t)h * D;
    const int rows_hi = min(row0 + BM, nq);
    load_rows<D, T>(Qs, Q, (int64_t)H * D, q0 + row0, rows_hi - row0, BM);
    // keys seen by rows [row0, rows_hi): the first row's first to the last row's last
    const int kv_begin = vis_key_lo(a.window, row0, nq, nkv);
    const int kv_end = max(vis_key_hi(a.causal, a.window, rows_hi - 1, nq, nkv) + 1, 0);
    const bool softmax = a.act == JFA_ACT_SOFTMAX;
    float m = -CUDART_INF_F, l = 0.f;
    float4 o[G];
#pragma unroll
    for (int g = 0; g < G; ++g) o[g] = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int j0 = kv_begin; j0 < kv_end; j0 += BN) {
        __syncthreads();
        const int nvalid = min(BN, nkv - j0);
        load_rows<D, T>(Ks, K, (int64_t)H * D, k0 + j0, nvalid, BN);
        load_rows<D, T>(Vs, V, (int64_t)H * D, k0 + j0, nvalid, BN);
        __syncthreads();
        float s[BN / 4];
#pragma unroll
        for (int jj = 0; jj < BN / 4; ++jj) s[jj] = 0.f;
#pragma unroll 4
        for (int dd = 0; dd < D; dd += 4) {
            float4 qv = *reinterpret_cast<const float4*>(Qs + r * LD + dd);
#pragma unroll
            for (int jj = 0; jj < BN / 4; ++jj) {
                float4 kv = *reinterpret_cast<const float4*>(Ks + (c + 4 * jj) * LD + dd);
                s[jj] += qv.x * kv.x + qv.y * kv.y + qv.z * kv.z + qv.w * kv.w;
            }
        }
        float tmax = -CUDART_INF_F;
#pragma unroll
        for (int jj = 0; jj < BN / 4; ++jj) {
            const int j = j0 + c + 4 * jj;
            const bool ok = i < nq && j < nkv && key_visible(a.causal, a.window, i, j, nq, nkv);
            float x = ok ? s[jj] * a.scale + bias_at<T>(a, b, h, nq, nkv, i, j) : -CUDART_INF_F;
            s[jj] = x;
            tmax = fmaxf(tmax, x);
        }
        float p[BN / 4];
        if (softmax) {
            tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 1));
            tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 2));
            const float m_new = fmaxf(m, tmax);
            const float alpha = (m_new == -CUDART_INF_F) ? 1.f : expf(m - m_new);
            float psum = 0.f;
#pragma unroll
            for (int jj = 0; jj < BN / 4; ++jj) {
                p[jj] = (s[jj] == -CUDART_INF_F) ? 0.f : expf(s[jj] - m_new);
                psum += p[jj];
            }
            psum += __shfl_xor_sync(0xffffffffu, psum, 1);
            psum += __shfl_xor_sync(0xffffffffu, psum, 2);
            l = l * alpha + psum;
            m = m_new;
#pragma unroll
            for (int g = 0; g < G; ++g) {
                o[g].x *= alpha; o[g].y *= alpha; o[g].z *= alpha; o[g].w *= alpha;
            }
        } else {
            const float inv_n = 1.0f / (float)nkv;
#pragma unroll
            for (int jj = 0; jj < BN / 4; ++jj)
                p[jj] = (s[jj] == -CUDART_INF_F) ? 0.f : act_f(a.act, s[jj]) * inv_n;
        }
#pragma unroll
        for (int jj = 0; jj < BN / 4; ++jj) Ps[r * LP + c + 4 * jj] = p[jj];
        __syncthreads();
        const int jn = min(BN, kv_end - j0);
        for (int jl = 0; jl < jn; ++jl) {
            const float pv = Ps[r * LP + jl];
#pragma unroll
            for (int g = 0; g < G; ++g) {
                float4 vv = *reinterpret_cast<const float4*>(Vs + jl * LD + 16 * g + 4 * c);
                o[g].x += pv * vv.x; o[g].y += pv * vv.y; o[g].z += pv * vv.z; o[g].w += pv * vv.w;
            }
        }
    }
    if (i < nq) {
        float inv = 1.f;
        if (softmax) inv = l > 0.f ? 1.f / l : 0.f;
        T* O = reinterpret_cast<T*>(a.out) + ((int64_t)(q0 + i) * H + h) * D;
#pragma unroll
        for (int g = 0; g < G; ++g)
            store4(O + 16 * g + 4 * c, make_float4(o[g].x * inv, o[g].y * inv, o[g].z * inv, o[g].w * inv));
        if (softmax && c == 0 && a.lse)
            a.lse[(int64_t)(q0 + i) * H + h] = l > 0.f ? m + logf(l) : -CUDART_INF_F;
    }
}

// ---------------------------------------------------------------------------
// Backward preprocess: D[t, h] = sum_d dO[t,h,d] * O[t,h,d]; one warp per row
// with a warp-shuffle reduction.
// ---------------------------------------------------------------------------
template <int D, typename T>
__global__ void __launch_bounds__(kThreads) simt_bwd_pre(const T* __restrict__ out,
                                                          const T* __restrict__ dout,
                                                          float* __restrict__ dterm,
                                                          int64_t rows) {
    const int64_t row = (int64_t)blockIdx.x * (kThreads / 32) + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= rows) return;
    float acc = 0.f;
    for (int e = lane; e < D; e += 32)
        acc += to_f(out[row * D + e]) * to_f(dout[row * D + e]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) dterm[row] = acc;
}

// Recomputes the probability (softmax: exp(s - lse)) or activation weight
// (GDPA: act(s) / n_kv) of one valid score, and its score gradient given
// dp = dO_i . v_j.
__device__ __forceinline__ void weight_and_dscore(int act, float s, float lse_i, float d_i,
                                                  float inv_n, float dp, float& w, float& ds) {
    if (act == JFA_ACT_SOFTMAX) {
        w = (lse_i == -CUDART_INF_F) ? 0.f : expf(s - lse_i);
        ds = w * (dp - d_i);
    } else {
        const float sg = sigmoid_fast(act_arg(act, s));
        w = s * sg * inv_n;
        ds = dp * act_grad_from(act, s, sg) * inv_n;
    }
}

// ---------------------------------------------------------------------------
// dQ: one CTA per (sequence, head, 64-row query tile); loops over key tiles.
// ---------------------------------------------------------------------------
template <int D, typename T>
__global__ void __launch_bounds__(kThreads) simt_bwd_dq(AttnArgs a) {
    constexpr int BM = 64, BN = 32, LD = SimtCfg<D>::LD, G = D / 16, LP = BN + 4;
    extern __shared__ __align__(16) float sm[];
    float* Qs = sm;
    float* dOs = Qs + BM * LD;
    float* Ks = dOs + BM * LD;
    float* Vs = Ks + BN * LD;
    float* dSs = Vs + BN * LD;
    if ((int)blockIdx.x >= *a.item_count || a.hdr->err != 0) return;
    const int4 it = a.items[blockIdx.x];
    const int b = it.x, h = it.y, row0 = it.z * BM;
    const int q0 = a.q_off[b], nq = a.q_off[b + 1] - q0;
    const int k0 = a.kv_off[b], nkv = a.kv_off[b + 1] - k0;
    const int H = a.H;
    const int tid = threadIdx.x, r = tid >> 2, c = tid & 3;
    const int i = row0 + r;
    const T* Q = reinterpret_cast<const T*>(a.q) + (int64_t)h * D;
    const T* dO = reinterpret_cast<const T*>(a.dout) + (int64_t)h * D;
    const T* K = reinterpret_cast<const T*>(a.k) + (int64_t)h * D;
    const T* V = reinterpret_cast<const T*>(a.v) + (int64_t)h * D;
    const int rows_hi = min(row0 + BM, nq);
    load_rows<D, T>(Qs, Q, (int64_t)H * D, q0 + row0, rows_hi - row0, BM);
    load_rows<D, T>(dOs, dO, (int64_t)H * D, q0 + row0, rows_hi - row0, BM);
    const bool softmax = a.act == JFA_ACT_SOFTMAX;
    float lse_i = 0.f, d_i = 0.f;
    if (i < nq && softmax) {
        lse_i = a.lse[(int64_t)(q0 + i) * H + h];
        d_i = a.dterm[(int64_t)(q0 + i) * H + h];
    }
    const float inv_n = nkv > 0 ? 1.0f / (float)nkv : 0.f;
    // keys seen by rows [row0, rows_hi): the first row's first to the last row's last
    const int kv_begin = vis_key_lo(a.window, row0, nq, nkv);
    const int kv_end = max(vis_key_hi(a.causal, a.window, rows_hi - 1, nq, nkv) + 1, 0);
    float4 acc[G];
#pragma unroll
    for (int g = 0; g < G; ++g) acc[g] = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int j0 = kv_begin; j0 < kv_end; j0 += BN) {
        __syncthreads();
        const int nvalid = min(BN, nkv - j0);
        load_rows<D, T>(Ks, K, (int64_t)H * D, k0 + j0, nvalid, BN);
        load_rows<D, T>(Vs, V, (int64_t)H * D, k0 + j0, nvalid, BN);
        __syncthreads();
        float s[BN / 4], dp[BN / 4];
#pragma unroll
        for (int jj = 0; jj < BN / 4; ++jj) s[jj] = 0.f, dp[jj] = 0.f;
#pragma unroll 4
        for (int dd = 0; dd < D; dd += 4) {
            float4 qv = *reinterpret_cast<const float4*>(Qs + r * LD + dd);
            float4 gv = *reinterpret_cast<const float4*>(dOs + r * LD + dd);
#pragma unroll
            for (int jj = 0; jj < BN / 4; ++jj) {
                float4 kv = *reinterpret_cast<const float4*>(Ks + (c + 4 * jj) * LD + dd);
                float4 vv = *reinterpret_cast<const float4*>(Vs + (c + 4 * jj) * LD + dd);
                s[jj] += qv.x * kv.x + qv.y * kv.y + qv.z * kv.z + qv.w * kv.w;
                dp[jj] += gv.x * vv.x + gv.y * vv.y + gv.z * vv.z + gv.w * vv.w;
            }
        }
#pragma unroll
        for (int jj = 0; jj < BN / 4; ++jj) {
            const int j = j0 + c + 4 * jj;
            const bool ok = i < nq && j < nkv && key_visible(a.causal, a.window, i, j, nq, nkv);
            float ds = 0.f;
            if (ok) {
                float x = s[jj] * a.scale + bias_at<T>(a, b, h, nq, nkv, i, j);
                float w;
                weight_and_dscore(a.act, x, lse_i, d_i, inv_n, dp[jj], w, ds);
            }
            dSs[r * LP + c + 4 * jj] = ds;
            // bias gradient: d beta = ds (this pass visits every pair once)
            if (a.dbias) {
                if (a.bias_kind == JFA_BIAS_DENSE_JAGGED) {
                    if (i < nq && j < nkv)
                        reinterpret_cast<T*>(a.dbias)[a.dense_off[b] + ((int64_t)h * nq + i) * nkv + j] = from_f<T>(ds);
                } else if (ok) {
                    const int C = (a.relpos_len - 1) >> 1;
                    const int rr = min(max(i - j, -C), C) + C;
                    atomicAdd(reinterpret_cast<float*>(a.dbias) + (int64_t)h * a.relpos_len + rr, ds);
                }
            }
        }
        __syncthreads();
        const int jn = min(BN, kv_end - j0);
        for (int jl = 0; jl < jn; ++jl) {
            const float dsv = dSs[r * LP + jl];
#pragma unroll
            for (int g = 0; g < G; ++g) {
                float4 kv = *reinterpret_cast<const float4*>(Ks + jl * LD + 16 * g + 4 * c);
                acc[g].x += dsv * kv.x; acc[g].y += dsv * kv.y; acc[g].z += dsv * kv.z; acc[g].w += dsv * kv.w;
            }
        }
    }
    if (i < nq) {
        T* dQ = reinterpret_cast<T*>(a.dq) + ((int64_t)(q0 + i) * H + h) * D;
        const float sc = a.scale;
#pragma unroll
        for (int g = 0; g < G; ++g)
            store4(dQ + 16 * g + 4 * c, make_float4(acc[g].x * sc, acc[g].y * sc, acc[g].z * sc, acc[g].w * sc));
    }
}

// ---------------------------------------------------------------------------
// dK, dV: one CTA per (sequence, head, 64-row key tile); loops over the
// 32-row query tiles that can see the tile.
// ---------------------------------------------------------------------------
template <int D, typename T>
__global__ void __launch_bounds__(kThreads) simt_bwd_dkdv(AttnArgs a) {
    constexpr int BN = 64, BM = 32, LD = SimtCfg<D>::LD, G = D / 16, LP = BM + 4;
    extern __shared__ __align__(16) float sm[];
    float* Ks = sm;
    float* Vs = Ks + BN * LD;
    float* Qs = Vs + BN * LD;
    float* dOs = Qs + BM * LD;
    float* Ps = dOs + BM * LD;
    float* dSs = Ps + BN * LP;
    float* rowstat = dSs + BN * LP;  // [BM] lse, [BM] D
    if ((int)blockIdx.x >= *a.item_count || a.hdr->err != 0) return;
    const int4 it = a.items[blockIdx.x];
    const int b = it.x, h = it.y, col0 = it.z * BN;
    const int q0 = a.q_off[b], nq = a.q_off[b + 1] - q0;
    const int k0 = a.kv_off[b], nkv = a.kv_off[b + 1] - k0;
    const int H = a.H;
    const int tid = threadIdx.x, r = tid >> 2, c = tid & 3;
    const int j = col0 + r;
    const T* Q = reinterpret_cast<const T*>(a.q) + (int64_t)h * D;
    const T* dO = reinterpret_cast<const T*>(a.dout) + (int64_t)h * D;
    const T* K = reinterpret_cast<const T*>(a.k) + (int64_t)h * D;
    const T* V = reinterpret_cast<const T*>(a.v) + (int64_t)h * D;
    const int cols_hi = min(col0 + BN, nkv);
    load_rows<D, T>(Ks, K, (int64_t)H * D, k0 + col0, cols_hi - col0, BN);
    load_rows<D, T>(Vs, V, (int64_t)H * D, k0 + col0, cols_hi - col0, BN);
    const bool softmax = a.act == JFA_ACT_SOFTMAX;
    const float inv_n = nkv > 0 ? 1.0f / (float)nkv : 0.f;
    // queries that see keys [col0, cols_hi): the first key's first to the last key's last
    const int i_start = vis_query_lo(a.causal, a.window, col0, nq, nkv);
    const int i_end = vis_query_hi(a.window, cols_hi - 1, nq, nkv) + 1;
    float4 dk[G], dv[G];
#pragma unroll
    for (int g = 0; g < G; ++g) dk[g] = make_float4(0.f, 0.f, 0.f, 0.f), dv[g] = dk[g];
    for (int i0 = i_start; i0 < i_end; i0 += BM) {
        __syncthreads();
        const int nvalid = min(BM, nq - i0);
        load_rows<D, T>(Qs, Q, (int64_t)H * D, q0 + i0, nvalid, BM);
        load_rows<D, T>(dOs, dO, (int64_t)H * D, q0 + i0, nvalid, BM);
        if (tid < BM) {
            float lv = 0.f, dv_ = 0.f;
            if (tid < nvalid && softmax) {
                lv = a.lse[(int64_t)(q0 + i0 + tid) * H + h];
                dv_ = a.dterm[(int64_t)(q0 + i0 + tid) * H + h];
            }
            rowstat[tid] = lv;
            rowstat[BM + tid] = dv_;
        }
        __syncthreads();
        float s[BM / 4], dp[BM / 4];
#pragma unroll
        for (int ii = 0; ii < BM / 4; ++ii) s[ii] = 0.f, dp[ii] = 0.f;
#pragma unroll 4
        for (int dd = 0; dd < D; dd += 4) {
            float4 kv = *reinterpret_cast<const float4*>(Ks + r * LD + dd);
            float4 vv = *reinterpret_cast<const float4*>(Vs + r * LD + dd);
#pragma unroll
            for (int ii = 0; ii < BM / 4; ++ii) {
                float4 qv = *reinterpret_cast<const float4*>(Qs + (c + 4 * ii) * LD + dd);
                float4 gv = *reinterpret_cast<const float4*>(dOs + (c + 4 * ii) * LD + dd);
                s[ii] += qv.x * kv.x + qv.y * kv.y + qv.z * kv.z + qv.w * kv.w;
                dp[ii] += gv.x * vv.x + gv.y * vv.y + gv.z * vv.z + gv.w * vv.w;
            }
        }
#pragma unroll
        for (int ii = 0; ii < BM / 4; ++ii) {
            const int il = c + 4 * ii, i = i0 + il;
            const bool ok = i < nq && j < nkv && key_visible(a.causal, a.window, i, j, nq, nkv);
            float w = 0.f, ds = 0.f;
            if (ok) {
                float x = s[ii] * a.scale + bias_at<T>(a, b, h, nq, nkv, i, j);
                weight_and_dscore(a.act, x, rowstat[il], rowstat[BM + il], inv_n, dp[ii], w, ds);
            }
            Ps[r * LP + il] = w;
            dSs[r * LP + il] = ds;
        }
        __syncthreads();
        for (int il = 0; il < nvalid; ++il) {
            const float w = Ps[r * LP + il], ds = dSs[r * LP + il];
#pragma unroll
            for (int g = 0; g < G; ++g) {
                float4 gv = *reinterpret_cast<const float4*>(dOs + il * LD + 16 * g + 4 * c);
                float4 qv = *reinterpret_cast<const float4*>(Qs + il * LD + 16 * g + 4 * c);
                dv[g].x += w * gv.x; dv[g].y += w * gv.y; dv[g].z += w * gv.z; dv[g].w += w * gv.w;
                dk[g].x += ds * qv.x; dk[g].y += ds * qv.y; dk[g].z += ds * qv.z; dk[g].w += ds * qv.w;
            }
        }
    }
    if (j < nkv) {
        T* dK = reinterpret_cast<T*>(a.dk) + ((int64_t)(k0 + j) * H + h) * D;
        T* dV = reinterpret_cast<T*>(a.dv) + ((int64_t)(k0 + j) * H + h) * D;
        const float sc = a.scale;
#pragma unroll
        for (int g = 0; g < G; ++g) {
            store4(dK + 16 * g + 4 * c, make_float4(dk[g].x * sc, dk[g].y * sc, dk[g].z * sc, dk[g].w * sc));
            store4(dV + 16 * g + 4 * c, dv[g]);
        }
    }
}

template <int D>
constexpr size_t fwd_smem() { return sizeof(float) * (64 * (D + 4) + 2 * 32 * (D + 4) + 64 * 36); }
template <int D>
constexpr size_t dq_smem() { return sizeof(float) * (2 * 64 * (D + 4) + 2 * 32 * (D + 4) + 64 * 36); }
template <int D>
constexpr size_t dkdv_smem() { return sizeof(float) * (2 * 64 * (D + 4) + 2 * 32 * (D + 4) + 2 * 64 * 36 + 64); }

template <int D, typename T>
cudaError_t launch_fwd_t(const AttnArgs& a, int grid, cudaStream_t st) {
    static bool configured = false;
    if (!configured) {
        cudaError_t e = cudaFuncSetAttribute(simt_fwd<D, T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)fwd_smem<D>());
        if (e != cudaSuccess) return e;
        configured = true;
    }
    prof_begin(st);
    simt_fwd<D, T><<<grid, kThreads, fwd_smem<D>(), st>>>(a);
    prof_end(st, K_SIMT_FWD);
    return cudaGetLastError();
}

template <int D, typename T>
cudaError_t launch_bwd_t(const AttnArgs& a, int grid_q, int grid_kv, int64_t rows, cudaStream_t st) {
    static bool configured = false;
    if (!configured) {
        cudaError_t e = cudaFuncSetAttribute(simt_bwd_dq<D, T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)dq_smem<D>());
        if (e != cudaSuccess) return e;
        e = cudaFuncSetAttribute(simt_bwd_dkdv<D, T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)dkdv_smem<D>());
        if (e != cudaSuccess) return e;
        configured = true;
    }
    if (a.act == JFA_ACT_SOFTMAX && rows > 0) {
        int64_t blocks = (rows + (kThreads / 32) - 1) / (kThreads / 32);
        prof_begin(st);
        simt_bwd_pre<D, T><<<(unsigned)blocks, kThreads, 0, st>>>(
            reinterpret_cast<const T*>(a.out), reinterpret_cast<const T*>(a.dout), a.dterm, rows);
        prof_end(st, K_SIMT_BWD_PRE);
    }
    if (grid_q > 0) {
        prof_begin(st);
        simt_bwd_dq<D, T><<<grid_q, kThreads, dq_smem<D>(), st>>>(a);
        prof_end(st, K_SIMT_BWD_DQ);
    }
    return cudaGetLastError();
}

template <int D, typename T>
cudaError_t launch_dkdv_t(const AttnArgs& a, int grid_kv, cudaStream_t st) {
    if (grid_kv > 0) {
        prof_begin(st);
        simt_bwd_dkdv<D, T><<<grid_kv, kThreads, dkdv_smem<D>(), st>>>(a);
        prof_end(st, K_SIMT_BWD_DKDV);
    }
    return cudaGetLastError();
}

}  // namespace

// Forward with 64-row query tiles; `grid` >= number of schedule items.
cudaError_t simt_forward(const AttnArgs& a, int head_dim, bool bf16, int grid, cudaStream_t st) {
    if (grid <= 0) return cudaSuccess;
    switch (head_dim) {
        case 32: return bf16 ? launch_fwd_t<32, __nv_bfloat16>(a, grid, st) : launch_fwd_t<32, float>(a, grid, st);
        case 64: return bf16 ? launch_fwd_t<64, __nv_bfloat16>(a, grid, st) : launch_fwd_t<64, float>(a, grid, st);
        case 128: return bf16 ? launch_fwd_t<128, __nv_bfloat16>(a, grid, st) : launch_fwd_t<128, float>(a, grid, st);
    }
    return cudaErrorInvalidValue;
}

// Backward: D preprocess + dQ pass (query items in a.items) then the dK/dV
// pass (key items in kv_args.items).
cudaError_t simt_backward(const AttnArgs& a, const AttnArgs& kv_args, int head_dim, bool bf16,
                          int grid_q, int grid_kv, int64_t rows, cudaStream_t st) {
    cudaError_t e = cudaErrorInvalidValue;
    switch (head_dim) {
        case 32:
            e = bf16 ? launch_bwd_t<32, __nv_bfloat16>(a, grid_q, grid_kv, rows, st) : launch_bwd_t<32, float>(a, grid_q, grid_kv, rows, st);
            if (e == cudaSuccess) e = bf16 ? launch_dkdv_t<32, __nv_bfloat16>(kv_args, grid_kv, st) : launch_dkdv_t<32, float>(kv_args, grid_kv, st);
            break;
        case 64:
            e = bf16 ? launch_bwd_t<64, __nv_bfloat16>(a, grid_q, grid_kv, rows, st) : launch_bwd_t<64, float>(a, grid_q, grid_kv, rows, st);
            if (e == cudaSuccess) e = bf16 ? launch_dkdv_t<64, __nv_bfloat16>(kv_args, grid_kv, st) : launch_dkdv_t<64, float>(kv_args, grid_kv, st);
            break;
        case 128:
            e = bf16 ? launch_bwd_t<128, __nv_bfloat16>(a, grid_q, grid_kv, rows, st) : launch_bwd_t<128, float>(a, grid_q, grid_kv, rows, st);
            if (e == cudaSuccess) e = bf16 ? launch_dkdv_t<128, __nv_bfloat16>(kv_args, grid_kv, st) : launch_dkdv_t<128, float>(kv_args, grid_kv, st);
            break;
    }
    return e;
}

}  // namespace jfa
