// quant_core.cuh -- the per-element arithmetic of the absmax int8 quantiser,
// shared by the standalone quantiser kernels and the stack GEMV that
// quantises its own activations, so that both give identical codes.
//
//   amax = max_k |x|, s = fl32(127/amax), q = clamp(rne(fl32(x*s)), -127, 127),
//   x_scale = fl32(amax/127), x_sum = sum q; amax == 0 gives zeros.
//
// BitNet b1.58 quantises activations to 8 bits per token by their largest
// magnitude (1bit.systems post "the full arc ...", paper list item 1); the
// pages give no formula, so this is the plainest reading (symmetric 127,
// multiply by the fp32 reciprocal scale, round half to even). Each rounding
// is an explicit _rn intrinsic, so results do not depend on contraction or
// fast-math settings.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace tq {

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Largest magnitude of the eight bf16 values in a 16-byte vector.
__device__ __forceinline__ float absmax8(uint4 u)
{
    float a = fmaxf(fabsf(bf16_lo(u.x)), fabsf(bf16_hi(u.x)));
    a = fmaxf(a, fmaxf(fabsf(bf16_lo(u.y)), fabsf(bf16_hi(u.y))));
    a = fmaxf(a, fmaxf(fabsf(bf16_lo(u.z)), fabsf(bf16_hi(u.z))));
    a = fmaxf(a, fmaxf(fabsf(bf16_lo(u.w)), fabsf(bf16_hi(u.w))));
    return a;
}

// s = 127 / amax (0 for an all-zero row) and x_scale = amax / 127.
__device__ __forceinline__ float quant_inv_scale(float amax)
{
    return amax > 0.0f ? __fdiv_rn(127.0f, amax) : 0.0f;
}
__device__ __forceinline__ float quant_scale(float amax)
{
    return amax > 0.0f ? __fdiv_rn(amax, 127.0f) : 0.0f;
}

__device__ __forceinline__ int code_of(float v, float s)
{
    int r = __float2int_rn(__fmul_rn(v, s));  // one fp32 rounding, then ties-to-even
    return min(max(r, -127), 127);
}

// Quantise two bf16 values held in one 32-bit word; returns two int8 codes in
// the low 16 bits and adds them to *sum.
__device__ __forceinline__ uint32_t quant2(uint32_t w, float s, int *sum)
{
    int a = code_of(bf16_lo(w), s);
    int b = code_of(bf16_hi(w), s);
    *sum += a + b;
    return (uint32_t(a) & 0xFFu) | ((uint32_t(b) & 0xFFu) << 8);
}

// Eight codes (8 bytes) of a 16-byte vector of bf16 values.
__device__ __forceinline__ uint2 quant8(uint4 u, float s, int *sum)
{
    uint2 o;
    o.x = quant2(u.x, s, sum) | (quant2(u.y, s, sum) << 16);
    o.y = quant2(u.z, s, sum) | (quant2(u.w, s, sum) << 16);
    return o;
}

}  // namespace tq
