// MX (OCP Microscaling v1.0) element helpers shared by the quantiser and the
// attention kernels: E8M0 shared exponent, power-of-two scales and the
// hardware E4M3 conversions (round-to-nearest-even, saturating).
#pragma once

#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <stdint.h>

namespace jfa {
namespace mx {

// floor(log2(amax)) - 8 clamped to the E8M0 range; amax >= 0 finite.
__device__ __forceinline__ int shared_exponent(float amax) {
    uint32_t bits = __float_as_uint(amax);
    int e = (int)((bits >> 23) & 0xFF);
    if (e == 0) return -127;  // zero or fp32-subnormal amax: floor(log2) < -126
    int X = (e - 127) - 8;
    return X < -127 ? -127 : (X > 127 ? 127 : X);
}

// 2^-X as a float, X in [-127, 119] for finite bf16 inputs.
__device__ __forceinline__ float pow2_neg(int X) {
    int e = 127 - X;
    if (e >= 255) e = 254;
    if (e <= 0) return 0.f;
    return __uint_as_float((uint32_t)e << 23);
}

// 2^X as a float for X in [-127, 127] (2^-127 is an fp32 subnormal).
__device__ __forceinline__ float pow2(int X) {
    if (X >= -126) return __uint_as_float((uint32_t)(X + 127) << 23);
    return __uint_as_float(1u << 22);
}

__device__ __forceinline__ uint16_t pack_e4m3x2(float lo, float hi) {
    __nv_fp8x2_storage_t s = __nv_cvt_float2_to_fp8x2(make_float2(lo, hi), __NV_SATFINITE, __NV_E4M3);
    return (uint16_t)s;
}

// E4M3 code pair -> two floats (exact: every E4M3 value is an fp16 value).
__device__ __forceinline__ float2 decode_e4m3x2(uint16_t two) {
    __half2_raw h = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)two, __NV_E4M3);
    return __half22float2(*reinterpret_cast<__half2*>(&h));
}

// In place: the 32 values become E4M3(v * 2^-X) * 2^X with X from their amax.
__device__ __forceinline__ void fake_quant32(float* v) {
    float amax = 0.f;
#pragma unroll
    for (int t = 0; t < 32; ++t) amax = fmaxf(amax, fabsf(v[t]));
    const int X = shared_exponent(amax);
    const float s = pow2_neg(X), back = pow2(X);
#pragma unroll
    for (int t = 0; t < 32; t += 2) {
        const float2 d = decode_e4m3x2(pack_e4m3x2(v[t] * s, v[t + 1] * s));
        v[t] = d.x * back;
        v[t + 1] = d.y * back;
    }
}

}  // namespace mx
}  // namespace jfa
