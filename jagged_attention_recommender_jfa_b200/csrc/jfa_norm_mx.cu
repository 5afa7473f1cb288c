// Normalisation fused with MX quantisation: the producer of MXFP8 attention
// operands writes E4M3 codes and E8M0 scales directly, so no separate cast
// pass reads the bf16 tensor again ("Meta GEM Training Efficiency: Why
// LLM-Scale Recommenders Need a Different Stack", "Bottleneck move 2": scale
// generation, casting and extra HBM traffic can eat the low-precision gain;
// "Meta Enhances GEM Training Efficiency with Advanced LLM-Scale
// Innovations", "Implementing Ultra-Low-Precision Methods").
//
// Per row of D elements (a token's model vector, or one head's d for a
// per-head Q / K norm with rows = tokens x heads):
//   RMSNorm  : y = x * gamma / sqrt(mean(x^2) + eps)
//   LayerNorm: y = (x - mean(x)) * gamma / sqrt(mean((x - mean)^2) + eps) + beta
// in fp32 (IEEE square root and division), then MX quantisation of y along
// the row as jfa_quantize_mxfp8 does along d: per 32 consecutive elements
// X = floor(log2 amax) - 8, codes = E4M3_rne_satfinite(y * 2^-X), scale byte
// X + 127.
//
// Threads: one thread per 32-element block; a row's blocks are one group of
// G = D / 32 lanes when G divides 32 (several rows per warp), else a whole
// warp that loops over the row's blocks.  The row statistics are group-wide
// shuffle reductions; the row is read once from HBM into registers when it
// fits (G <= 32), otherwise re-read from L2 for the second pass.
#include "jfa_common.cuh"
#include "jfa_mx.cuh"

namespace jfa {
namespace {

__device__ __forceinline__ void load32(const __nv_bfloat16* p, float (&f)[32]) {
    const uint4* src = reinterpret_cast<const uint4*>(p);
#pragma unroll
    for (int t = 0; t < 4; ++t) {
        const uint4 raw = src[t];
        const __nv_bfloat162* p2 = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const float2 v = __bfloat1622float2(p2[u]);
            f[8 * t + 2 * u] = v.x;
            f[8 * t + 2 * u + 1] = v.y;
        }
    }
}

__device__ __forceinline__ float group_sum(float v, int width) {
    for (int o = width >> 1; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o, width);
    return v;
}

// y of one 32-element block quantised: codes and the scale byte
__device__ __forceinline__ void quant_block(const float (&y)[32], uint8_t* codes, uint8_t* scale) {
    float amax = 0.f;
#pragma unroll
    for (int t = 0; t < 32; ++t) amax = fmaxf(amax, fabsf(y[t]));
    const int X = mx::shared_exponent(amax);
    const float s = mx::pow2_neg(X);
    uint32_t w[8];
#pragma unroll
    for (int t = 0; t < 8; ++t) {
        const uint32_t lo = mx::pack_e4m3x2(y[4 * t] * s, y[4 * t + 1] * s);
        const uint32_t hi = mx::pack_e4m3x2(y[4 * t + 2] * s, y[4 * t + 3] * s);
        w[t] = lo | (hi << 16);
    }
    uint4* dst = reinterpret_cast<uint4*>(codes);
    dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
    dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
    *scale = (uint8_t)(X + 127);
}

// Rows of G <= 32 blocks: one lane per block, 32 / G rows per warp.
__global__ void __launch_bounds__(256) norm_quant_small(const __nv_bfloat16* __restrict__ x, int64_t rows,
                                                        int D, const float* __restrict__ gamma,
                                                        const float* __restrict__ beta, float eps,
                                                        int layernorm, uint8_t* __restrict__ codes,
                                                        uint8_t* __restrict__ scales) {
    const int G = D >> 5;
    const int64_t gid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t row = gid / G;
    const int blk = (int)(gid % G);
    const bool live = row < rows;
    float f[32];
    const int64_t r = live ? row : rows - 1;   // dead lanes still take part in the shuffles
    load32(x + r * D + blk * 32, f);
    float s = 0.f;
#pragma unroll
    for (int t = 0; t < 32; ++t) s += f[t];
    const float mean = layernorm ? group_sum(s, G) / (float)D : 0.f;
    float q = 0.f;
#pragma unroll
    for (int t = 0; t < 32; ++t) {
        const float c = f[t] - mean;
        q = fmaf(c, c, q);
    }
    const float var = group_sum(q, G) / (float)D;
    const float inv = 1.0f / sqrtf(var + eps);
    if (!live) return;
#pragma unroll
    for (int t = 0; t < 32; ++t) {
        const int c = blk * 32 + t;
        const float g = gamma ? gamma[c] : 1.f;
        const float b = (layernorm && beta) ? beta[c] : 0.f;
        f[t] = (f[t] - mean) * inv * g + b;
    }
    quant_block(f, codes + row * D + blk * 32, scales + row * G + blk);
}

// Rows of G > 32 blocks: one warp per row, lanes loop over the blocks.
__global__ void __launch_bounds__(256) norm_quant_wide(const __nv_bfloat16* __restrict__ x, int64_t rows,
                                                       int D, const float* __restrict__ gamma,
                                                       const float* __restrict__ beta, float eps,
                                                       int layernorm, uint8_t* __restrict__ codes,
                                                       uint8_t* __restrict__ scales) {
    const int G = D >> 5;
    const int lane = threadIdx.x & 31;
    const int64_t row = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    if (row >= rows) return;   // whole warps leave together
    const __nv_bfloat16* xr = x + row * D;
    float s = 0.f;
    for (int blk = lane; blk < G; blk += 32) {
        float f[32];
        load32(xr + blk * 32, f);
#pragma unroll
        for (int t = 0; t < 32; ++t) s += f[t];
    }
    const float mean = layernorm ? group_sum(s, 32) / (float)D : 0.f;
    float q = 0.f;
    for (int blk = lane; blk < G; blk += 32) {
        float f[32];
        load32(xr + blk * 32, f);
#pragma unroll
        for (int t = 0; t < 32; ++t) {
            const float c = f[t] - mean;
            q = fmaf(c, c, q);
        }
    }
    const float var = group_sum(q, 32) / (float)D;
    const float inv = 1.0f / sqrtf(var + eps);
    for (int blk = lane; blk < G; blk += 32) {
        float f[32];
        load32(xr + blk * 32, f);
#pragma unroll
        for (int t = 0; t < 32; ++t) {
            const int c = blk * 32 + t;
            const float g = gamma ? gamma[c] : 1.f;
            const float b = (layernorm && beta) ? beta[c] : 0.f;
            f[t] = (f[t] - mean) * inv * g + b;
        }
        quant_block(f, codes + row * D + blk * 32, scales + row * G + blk);
    }
}

}  // namespace
}  // namespace jfa

extern "C" jfa_status jfa_norm_quantize_mxfp8(const void* x, int64_t rows, int32_t D,
                                              const float* gamma, const float* beta, float eps,
                                              int layernorm, uint8_t* codes, uint8_t* scales,
                                              jfa_stream_t stream) {
    if (rows < 0 || D < 32 || (D % 32) != 0 || D > 16384 || !(eps > 0.f))
        return jfa::set_last_error(JFA_ERR_INVALID_ARGUMENT,
                                   "norm_quantize: rows >= 0, D a multiple of 32 in [32, 16384], eps > 0");
    if (rows == 0) return JFA_OK;
    if (!x || !codes || !scales)
        return jfa::set_last_error(JFA_ERR_INVALID_ARGUMENT, "norm_quantize: NULL tensor");
    if ((reinterpret_cast<uintptr_t>(x) & 15) || (reinterpret_cast<uintptr_t>(codes) & 15))
        return jfa::set_last_error(JFA_ERR_INVALID_ARGUMENT, "norm_quantize: x and codes 16-byte aligned");
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const int G = D / 32;
    const __nv_bfloat16* xb = reinterpret_cast<const __nv_bfloat16*>(x);
    jfa::prof_begin(st);
    if (G <= 32 && (32 % G) == 0) {
        const int64_t threads = rows * G;
        const unsigned grid = (unsigned)((threads + 255) / 256);
        jfa::norm_quant_small<<<grid, 256, 0, st>>>(xb, rows, D, gamma, beta, eps, layernorm ? 1 : 0,
                                                    codes, scales);
    } else {
        const unsigned grid = (unsigned)((rows * 32 + 255) / 256);
        jfa::norm_quant_wide<<<grid, 256, 0, st>>>(xb, rows, D, gamma, beta, eps, layernorm ? 1 : 0,
                                                   codes, scales);
    }
    jfa::prof_end(st, jfa::K_NORM_QUANT);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess)
        return jfa::set_last_error(JFA_ERR_CUDA, "norm_quantize: %s", cudaGetErrorString(e));
    return JFA_OK;
}
