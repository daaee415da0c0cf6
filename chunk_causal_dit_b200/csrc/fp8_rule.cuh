// fp8_rule.cuh -- the E4M3 quantization rule shared by the stand-alone quantizers
// and the append kernel's fused Q quantization, so that both produce the same bits.
//
// For a group of values x: amax = max |x| (exact in fp32); the dequantization
// scale is amax / 448 and the quantization multiplier 448 / amax, both IEEE fp32
// divisions (1 when amax = 0); code = E4M3 rounding, ties to even, with
// saturation, of the IEEE fp32 product x * (448 / amax).
#pragma once
#include <cstdint>

namespace wf {

constexpr float kE4M3Max = 448.0f;

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// two E4M3 codes in the low 16 bits: `lo` in bits 0-7, `hi` in bits 8-15
__device__ __forceinline__ uint32_t e4m3x2(float lo, float hi)
{
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}

__device__ __forceinline__ float fp8_scale(float amax)
{
    return amax > 0.0f ? __fdiv_rn(amax, kE4M3Max) : 1.0f;
}

__device__ __forceinline__ float fp8_inv(float amax)
{
    return amax > 0.0f ? __fdiv_rn(kE4M3Max, amax) : 1.0f;
}

// 4 codes of x0..x3 * inv, packed little-endian
__device__ __forceinline__ uint32_t quant4(float x0, float x1, float x2, float x3, float inv)
{
    return e4m3x2(__fmul_rn(x0, inv), __fmul_rn(x1, inv)) |
           (e4m3x2(__fmul_rn(x2, inv), __fmul_rn(x3, inv)) << 16);
}

// 8 codes of the 8 bf16 values in u (one 16-byte row piece), packed little-endian
__device__ __forceinline__ uint2 quant8(const uint4 &u, float inv)
{
    return make_uint2(quant4(bf16_lo(u.x), bf16_hi(u.x), bf16_lo(u.y), bf16_hi(u.y), inv),
                      quant4(bf16_lo(u.z), bf16_hi(u.z), bf16_lo(u.w), bf16_hi(u.w), inv));
}

// max |x| of the 8 bf16 values in u
__device__ __forceinline__ float absmax8(const uint4 &u)
{
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
    float a = 0.0f;
#pragma unroll
    for (int e = 0; e < 4; ++e) a = fmaxf(a, fmaxf(fabsf(bf16_lo(w[e])), fabsf(bf16_hi(w[e]))));
    return a;
}

}  // namespace wf
