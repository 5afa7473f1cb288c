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

// Blocks of 32 consecutive elements along d: one thread per block (64-byte
// loads).  CODES: E4M3 codes and the E8M0 scale; DEQ: the dequantised value
// E4M3(x * 2^-X) * 2^X in bf16 (exact: 3 mantissa bits times a power of two).
template <bool CODES, bool DEQ>
__global__ void __launch_bounds__(256) mx_along_d(const __nv_bfloat16* __restrict__ x,
                                                  int64_t n_blocks, uint8_t* __restrict__ codes,
                                                  uint8_t* __restrict__ scales,
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
    uint16_t two[16];
#pragma unroll
    for (int t = 0; t < 16; ++t) two[t] = pack_e4m3x2(f[2 * t] * s, f[2 * t + 1] * s);
    if (CODES) {
        uint32_t w[8];
#pragma unroll
        for (int t = 0; t < 8; ++t) w[t] = (uint32_t)two[2 * t] | ((uint32_t)two[2 * t + 1] << 16);
        uint4* dst = reinterpret_cast<uint4*>(codes + blk * 32);
        dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
        dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
        scales[blk] = (uint8_t)(X + 127);
    }
    if (DEQ) {
        uint4 out[4];
        uint32_t* o32 = reinterpret_cast<uint32_t*>(out);
#pragma unroll
        for (int t = 0; t < 16; ++t) {
            const float2 d2 = decode_e4m3x2(two[t]);
            __nv_bfloat162 b2 = __floats2bfloat162_rn(d2.x * back, d2.y * back);
            o32[t] = *reinterpret_cast<uint32_t*>(&b2);
        }
        uint4* dst = reinterpret_cast<uint4*>(y + blk * 32);
#pragma unroll
        for (int t = 0; t < 4; ++t) dst[t] = out[t];
    }
}

// Blocks of 32 consecutive rows of one sequence.  Grid (sequence, slot): a
// CTA takes its sequence's row blocks slot, slot + gridDim.y, ... (at most
// kRowSlots CTAs per sequence, so a short batch of long sequences launches
// no idle CTAs); a thread takes two adjacent columns, so a warp reads 128
// contiguous bytes of each row, and all 32 loads of a block are in flight
// before the first conversion.
constexpr int kRowSlots = 16;

// first block index of sequence b = sum_{b' < b} ceil(n(b') / 32)
__device__ int64_t seq_block_base(const int32_t* __restrict__ off, int b) {
    __shared__ int64_t s_warp[8];
    int64_t part = 0;
    for (int bb = threadIdx.x; bb < b; bb += blockDim.x) part += (off[bb + 1] - off[bb] + 31) / 32;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
    if ((threadIdx.x & 31) == 0) s_warp[threadIdx.x >> 5] = part;
    __syncthreads();
    int64_t total = 0;
#pragma unroll
    for (int w = 0; w < 8; ++w) total += s_warp[w];
    return total;
}

// CODES: E4M3 codes and E8M0 scales; DEQ: the dequantised value
// E4M3(x * 2^-X) * 2^X in bf16 (exact).
template <bool CODES, bool DEQ>
__global__ void __launch_bounds__(256, 4) mx_along_rows(const __nv_bfloat16* __restrict__ x,
                                                     const int32_t* __restrict__ off,
                                                     int64_t total_rows, int cols,
                                                     uint8_t* __restrict__ codes,
                                                     uint8_t* __restrict__ scales,
                                                     __nv_bfloat16* __restrict__ y) {
    const int b = blockIdx.x;
    const int r0 = off[b], n = off[b + 1] - r0;
    // rows outside [0, total_rows) are never touched, whatever the offsets say
    if (n <= 0 || r0 < 0 || (int64_t)r0 + n > total_rows) return;
    const int nblk = (n + 31) / 32;
    if ((int)blockIdx.y >= nblk) return;
    const int64_t blk0 = CODES ? seq_block_base(off, b) : 0;
    const bool scale_pairs = ((reinterpret_cast<uintptr_t>(scales) & 1) == 0);
    for (int blk = blockIdx.y; blk < nblk; blk += gridDim.y) {
        const int rows = min(32, n - blk * 32);
        const int64_t row0 = (int64_t)r0 + (int64_t)blk * 32;
        for (int c = threadIdx.x * 2; c < cols; c += blockDim.x * 2) {
            // one running address per pass (not 32 precomputed ones); rows
            // past a short last block repeat its last row, which leaves the
            // block maximum as zero padding would
            const __nv_bfloat16* src = x + row0 * cols + c;
            uint32_t raw[32];
#pragma unroll
            for (int t = 0; t < 32; ++t) {
                raw[t] = __ldg(reinterpret_cast<const unsigned int*>(src));
                if (t + 1 < rows) src += cols;
            }
            // block maxima of |x| in bf16 (exact: a maximum rounds nothing)
            __nv_bfloat162 m = __float2bfloat162_rn(0.f);
#pragma unroll
            for (int t = 0; t < 32; ++t) m = __hmax2(m, __habs2(*reinterpret_cast<const __nv_bfloat162*>(&raw[t])));
            const float2 am = __bfloat1622float2(m);
            const int X0 = shared_exponent(am.x), X1 = shared_exponent(am.y);
            const float s0 = pow2_neg(X0), s1 = pow2_neg(X1);
            const float b0 = pow2(X0), b1 = pow2(X1);
            uint8_t* cdst = CODES ? codes + row0 * cols + c : nullptr;
            __nv_bfloat16* ydst = DEQ ? y + row0 * cols + c : nullptr;
#pragma unroll
            for (int t = 0; t < 32; ++t) {
                const float2 v = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw[t]));
                const uint16_t two = pack_e4m3x2(v.x * s0, v.y * s1);
                if (t < rows) {
                    if (DEQ) {
                        const float2 d = decode_e4m3x2(two);
                        *reinterpret_cast<__nv_bfloat162*>(ydst) = __floats2bfloat162_rn(d.x * b0, d.y * b1);
                    }
                    if (CODES) *reinterpret_cast<uint16_t*>(cdst) = two;
                }
                if (DEQ) ydst += cols;
                if (CODES) cdst += cols;
            }
            if (CODES) {
                uint8_t* sp = scales + (blk0 + blk) * cols + c;
                if (scale_pairs) {
                    *reinterpret_cast<uint16_t*>(sp) = (uint16_t)((X0 + 127) | ((X1 + 127) << 8));
                } else {
                    sp[0] = (uint8_t)(X0 + 127);
                    sp[1] = (uint8_t)(X1 + 127);
                }
            }
        }
    }
}

}  // namespace

// codes / scales (both or neither) and / or the dequantised bf16 `dequant`.
cudaError_t quantize_mx(const void* x, int64_t rows, int heads, int d, const int32_t* offsets,
                        int batch, int max_rows_per_seq, int along_rows, uint8_t* codes,
                        uint8_t* scales, void* dequant, cudaStream_t st) {
    const __nv_bfloat16* xb = reinterpret_cast<const __nv_bfloat16*>(x);
    __nv_bfloat16* y = reinterpret_cast<__nv_bfloat16*>(dequant);
    const bool cd = codes != nullptr, dq = dequant != nullptr;
    if (!cd && !dq) return cudaSuccess;
    if (!along_rows) {
        int64_t n_blocks = rows * heads * (d / 32);
        if (n_blocks == 0) return cudaSuccess;
        const unsigned grid = (unsigned)((n_blocks + 255) / 256);
        prof_begin(st);
        if (cd && dq) mx_along_d<true, true><<<grid, 256, 0, st>>>(xb, n_blocks, codes, scales, y);
        else if (cd) mx_along_d<true, false><<<grid, 256, 0, st>>>(xb, n_blocks, codes, scales, y);
        else mx_along_d<false, true><<<grid, 256, 0, st>>>(xb, n_blocks, codes, scales, y);
        prof_end(st, K_QUANT_ALONG_D);
    } else {
        if (batch == 0 || max_rows_per_seq == 0) return cudaSuccess;
        const int slots = (max_rows_per_seq + 31) / 32 < kRowSlots ? (max_rows_per_seq + 31) / 32 : kRowSlots;
        dim3 grid(batch, slots);
        const int cols = heads * d;
        prof_begin(st);
        if (cd && dq) mx_along_rows<true, true><<<grid, 256, 0, st>>>(xb, offsets, rows, cols, codes, scales, y);
        else if (cd) mx_along_rows<true, false><<<grid, 256, 0, st>>>(xb, offsets, rows, cols, codes, scales, y);
        else mx_along_rows<false, true><<<grid, 256, 0, st>>>(xb, offsets, rows, cols, codes, scales, y);
        prof_end(st, K_QUANT_ALONG_ROWS);
    }
    return cudaGetLastError();
}


// MXFP8 operands for the attention passes: Q and K quantised along d, V along
// 32-row blocks of each sequence, each returned dequantised in bf16.
cudaError_t mx_fake_quant_qkv(const void* q, const void* k, const void* v, const int32_t* kv_off,
                              int64_t total_q, int64_t total_kv, int heads, int d, int batch,
                              int max_kv_len, void* qf, void* kf, void* vf, cudaStream_t st) {
    cudaError_t e = quantize_mx(q, total_q, heads, d, nullptr, 0, 0, 0, nullptr, nullptr, qf, st);
    if (e == cudaSuccess) e = quantize_mx(k, total_kv, heads, d, nullptr, 0, 0, 0, nullptr, nullptr, kf, st);
    if (e == cudaSuccess)
        e = quantize_mx(v, total_kv, heads, d, kv_off, batch, max_kv_len, 1, nullptr, nullptr, vf, st);
    return e;
}

}  // namespace jfa
