// MX (OCP Microscaling v1.0) quantisation of bf16 tensors to E4M3 elements
// with one E8M0 power-of-two scale per 32 elements, for the MXFP8 attention
// path ("GEM Training: How Meta Doubled the Efficiency of Its LLM-Scale Ads
// Foundation Model", opening summary: mixed ultra-low precision training
// including MXFP8 attention; "Meta GEM Training Efficiency: Why LLM-Scale
// Recommenders Need a Different Stack", "Bottleneck move 2": scale generation
// and casting must not eat the gain, so the pass is a single streaming read).
//
//   X     = floor(log2(amax)) - 8   (8 = largest E4M3 exponent), in [-127, 127]
//   code  = E4M3_rne_satfinite(x * 2^-X)
//   scale = X + 127                  (E8M0 byte)
// x * 2^-X is exact in fp32 (a power-of-two scaling of a bf16 value whose
// result lies below 2^9), so the only rounding is the hardware's
// round-to-nearest-even conversion with saturation (cvt.rn.satfinite).
#include "jfa_common.cuh"
#include "jfa_mx.cuh"

namespace jfa {

namespace {

using mx::shared_exponent;
using mx::pow2_neg;
using mx::pow2;
using mx::pack_e4m3x2;
using mx::decode_e4m3x2;

// Blocks of 32 consecutive elements along d: one thread per block.
__global__ void __launch_bounds__(256) quant_along_d(const __nv_bfloat16* __restrict__ x,
                                                     int64_t n_blocks, uint8_t* __restrict__ codes,
                                                     uint8_t* __restrict__ scales) {
    int64_t blk = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (blk >= n_blocks) return;
    const uint4* src = reinterpret_cast<const uint4*>(x + blk * 32);
    uint4 raw[4];
#pragma unroll
    for (int t = 0; t < 4; ++t) raw[t] = src[t];
    float f[32];
#pragma unroll
    for (int t = 0; t < 4; ++t) {
        const __nv_bfloat162* p2 = reinterpret_cast<const __nv_bfloat162*>(&raw[t]);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            float2 v = __bfloat1622float2(p2[u]);
            f[8 * t + 2 * u] = v.x;
            f[8 * t + 2 * u + 1] = v.y;
        }
    }
    float amax = 0.f;
#pragma unroll
    for (int t = 0; t < 32; ++t) amax = fmaxf(amax, fabsf(f[t]));
    const int X = shared_exponent(amax);
    const float s = pow2_neg(X);
    uint32_t w[8];
#pragma unroll
    for (int t = 0; t < 8; ++t) {
        uint32_t lo = pack_e4m3x2(f[4 * t] * s, f[4 * t + 1] * s);
        uint32_t hi = pack_e4m3x2(f[4 * t + 2] * s, f[4 * t + 3] * s);
        w[t] = lo | (hi << 16);
    }
    uint4* dst = reinterpret_cast<uint4*>(codes + blk * 32);
    dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
    dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
    scales[blk] = (uint8_t)(X + 127);
}

// Blocks of 32 consecutive rows of one sequence: grid (sequence, row block),
// threads over the heads * d columns (coalesced along the row).
__global__ void __launch_bounds__(256) quant_along_rows(const __nv_bfloat16* __restrict__ x,
                                                        const int32_t* __restrict__ off, int B,
                                                        int64_t total_rows, int cols,
                                                        uint8_t* __restrict__ codes,
                                                        uint8_t* __restrict__ scales) {
    const int b = blockIdx.x, blk = blockIdx.y;
    const int r0 = off[b], n = off[b + 1] - r0;
    // rows outside [0, total_rows) are never touched, whatever the offsets say
    if (blk * 32 >= n || r0 < 0 || (int64_t)r0 + n > total_rows) return;
    // first block index of sequence b = sum_{b' < b} ceil(n(b') / 32)
    __shared__ int64_t s_part[256];
    int64_t part = 0;
    for (int bb = threadIdx.x; bb < b; bb += blockDim.x) part += (off[bb + 1] - off[bb] + 31) / 32;
    s_part[threadIdx.x] = part;
    __syncthreads();
    for (int st = 128; st > 0; st >>= 1) {
        if ((int)threadIdx.x < st) s_part[threadIdx.x] += s_part[threadIdx.x + st];
        __syncthreads();
    }
    const int64_t gblk = s_part[0] + blk;
    const int rows = min(32, n - blk * 32);
    const __nv_bfloat16* base = x + (int64_t)(r0 + blk * 32) * cols;
    uint8_t* cbase = codes + (int64_t)(r0 + blk * 32) * cols;
    for (int col = threadIdx.x; col < cols; col += blockDim.x) {
        float f[32];
        float amax = 0.f;
#pragma unroll
        for (int t = 0; t < 32; ++t) {
            f[t] = t < rows ? __bfloat162float(base[(int64_t)t * cols + col]) : 0.f;
            amax = fmaxf(amax, fabsf(f[t]));
        }
        const int X = shared_exponent(amax);
        const float s = pow2_neg(X);
#pragma unroll
        for (int t = 0; t < 32; t += 2) {
            uint16_t two = pack_e4m3x2(f[t] * s, f[t + 1] * s);
            if (t < rows) cbase[(int64_t)t * cols + col] = (uint8_t)(two & 0xFF);
            if (t + 1 < rows) cbase[(int64_t)(t + 1) * cols + col] = (uint8_t)(two >> 8);
        }
        scales[gblk * cols + col] = (uint8_t)(X + 127);
    }
}

// Quantise-dequantise ("fake quantisation") along d: the output holds, in
// bf16, exactly the value E4M3(x * 2^-X) * 2^X that an MXFP8 operand
// represents (3 mantissa bits times a power of two fit bf16 exactly).
__global__ void __launch_bounds__(256) fake_quant_along_d(const __nv_bfloat16* __restrict__ x,
                                                          int64_t n_blocks,
                                                          __nv_bfloat16* __restrict__ y) {
    int64_t blk = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (blk >= n_blocks) return;
    const uint4* src = reinterpret_cast<const uint4*>(x + blk * 32);
    uint4 raw[4];
#pragma unroll
    for (int t = 0; t < 4; ++t) raw[t] = src[t];
    float f[32];
#pragma unroll
    for (int t = 0; t < 4; ++t) {
        const __nv_bfloat162* p2 = reinterpret_cast<const __nv_bfloat162*>(&raw[t]);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            float2 v = __bfloat1622float2(p2[u]);
            f[8 * t + 2 * u] = v.x;
            f[8 * t + 2 * u + 1] = v.y;
        }
    }
    float amax = 0.f;
#pragma unroll
    for (int t = 0; t < 32; ++t) amax = fmaxf(amax, fabsf(f[t]));
    const int X = shared_exponent(amax);
    const float s = pow2_neg(X), back = pow2(X);
    uint4 out[4];
    uint32_t* o32 = reinterpret_cast<uint32_t*>(out);
#pragma unroll
    for (int t = 0; t < 16; ++t) {
        const float2 d2 = decode_e4m3x2(pack_e4m3x2(f[2 * t] * s, f[2 * t + 1] * s));
        __nv_bfloat162 b2 = __floats2bfloat162_rn(d2.x * back, d2.y * back);
        o32[t] = *reinterpret_cast<uint32_t*>(&b2);
    }
    uint4* dst = reinterpret_cast<uint4*>(y + blk * 32);
#pragma unroll
    for (int t = 0; t < 4; ++t) dst[t] = out[t];
}

// Quantise-dequantise along 32-row blocks of each sequence.
__global__ void __launch_bounds__(256) fake_quant_along_rows(const __nv_bfloat16* __restrict__ x,
                                                             const int32_t* __restrict__ off,
                                                             int64_t total_rows, int cols,
                                                             __nv_bfloat16* __restrict__ y) {
    const int b = blockIdx.x, blk = blockIdx.y;
    const int r0 = off[b], n = off[b + 1] - r0;
    if (blk * 32 >= n || r0 < 0 || (int64_t)r0 + n > total_rows) return;
    const int rows = min(32, n - blk * 32);
    const __nv_bfloat16* base = x + (int64_t)(r0 + blk * 32) * cols;
    __nv_bfloat16* obase = y + (int64_t)(r0 + blk * 32) * cols;
    for (int col = threadIdx.x; col < cols; col += blockDim.x) {
        float f[32];
        float amax = 0.f;
#pragma unroll
        for (int t = 0; t < 32; ++t) {
            f[t] = t < rows ? __bfloat162float(base[(int64_t)t * cols + col]) : 0.f;
            amax = fmaxf(amax, fabsf(f[t]));
        }
        const int X = shared_exponent(amax);
        const float s = pow2_neg(X), back = pow2(X);
#pragma unroll
        for (int t = 0; t < 32; t += 2) {
            const float2 d2 = decode_e4m3x2(pack_e4m3x2(f[t] * s, f[t + 1] * s));
            if (t < rows) obase[(int64_t)t * cols + col] = __float2bfloat16_rn(d2.x * back);
            if (t + 1 < rows) obase[(int64_t)(t + 1) * cols + col] = __float2bfloat16_rn(d2.y * back);
        }
    }
}

}  // namespace

// MXFP8 operands for the attention passes: Q and K quantised along d, V along
// 32-row blocks of each sequence, each returned dequantised in bf16.
cudaError_t mx_fake_quant_qkv(const void* q, const void* k, const void* v, const int32_t* kv_off,
                              int64_t total_q, int64_t total_kv, int heads, int d, int batch,
                              int max_kv_len, void* qf, void* kf, void* vf, cudaStream_t st) {
    const int64_t nq_blocks = total_q * heads * (d / 32), nk_blocks = total_kv * heads * (d / 32);
    prof_begin(st);
    if (nq_blocks > 0)
        fake_quant_along_d<<<(unsigned)((nq_blocks + 255) / 256), 256, 0, st>>>(
            reinterpret_cast<const __nv_bfloat16*>(q), nq_blocks, reinterpret_cast<__nv_bfloat16*>(qf));
    if (nk_blocks > 0)
        fake_quant_along_d<<<(unsigned)((nk_blocks + 255) / 256), 256, 0, st>>>(
            reinterpret_cast<const __nv_bfloat16*>(k), nk_blocks, reinterpret_cast<__nv_bfloat16*>(kf));
    prof_end(st, K_QUANT_ALONG_D);
    if (batch > 0 && max_kv_len > 0) {
        dim3 grid(batch, (max_kv_len + 31) / 32);
        prof_begin(st);
        fake_quant_along_rows<<<grid, 256, 0, st>>>(reinterpret_cast<const __nv_bfloat16*>(v), kv_off,
                                                    total_kv, heads * d, reinterpret_cast<__nv_bfloat16*>(vf));
        prof_end(st, K_QUANT_ALONG_ROWS);
    }
    return cudaGetLastError();
}

cudaError_t quantize_mx(const void* x, int64_t rows, int heads, int d, const int32_t* offsets,
                        int batch, int max_rows_per_seq, int along_rows, uint8_t* codes,
                        uint8_t* scales, cudaStream_t st) {
    const __nv_bfloat16* xb = reinterpret_cast<const __nv_bfloat16*>(x);
    if (!along_rows) {
        int64_t n_blocks = rows * heads * (d / 32);
        if (n_blocks == 0) return cudaSuccess;
        int64_t grid = (n_blocks + 255) / 256;
        prof_begin(st);
        quant_along_d<<<(unsigned)grid, 256, 0, st>>>(xb, n_blocks, codes, scales);
        prof_end(st, K_QUANT_ALONG_D);
    } else {
        if (batch == 0 || max_rows_per_seq == 0) return cudaSuccess;
        dim3 grid(batch, (max_rows_per_seq + 31) / 32);
        prof_begin(st);
        quant_along_rows<<<grid, 256, 0, st>>>(xb, offsets, batch, rows, heads * d, codes, scales);
        prof_end(st, K_QUANT_ALONG_ROWS);
    }
    return cudaGetLastError();
}

}  // namespace jfa
