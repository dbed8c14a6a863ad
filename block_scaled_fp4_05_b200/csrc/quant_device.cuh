// Device arithmetic of the block quantizer, shared by the quantizer kernels
// and by the decode GEMM that quantizes its activation in place: the BF16
// magnitude maximum of 8 values, the block scale (E8M0 or E4M3, as in
// fp4_quantize) and the E2M1 conversion of 8 values.  One definition, so
// that both produce the same bytes.
#pragma once

#include <cuda_runtime.h>
#include <cuda_fp16.h>
#include <cstdint>
#include <cfloat>

#include "fp4_internal.h"

namespace fp4 {
namespace qdev {

__device__ __forceinline__ uint4 ld_stream(const uint4* p)
{
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

// Largest BF16 magnitude (sign cleared, as an integer) of 8 packed values.
__device__ __forceinline__ uint32_t absmax8(uint4 v)
{
    const uint32_t m = 0x7FFF7FFFu;
    uint32_t a = __vmaxu2(v.x & m, v.y & m);
    uint32_t b = __vmaxu2(v.z & m, v.w & m);
    a = __vmaxu2(a, b);
    return max(a & 0xFFFFu, a >> 16);
}

// Unsigned E4M3 round-to-nearest-even, saturating at 448.
__device__ __forceinline__ uint32_t cvt_e4m3(float t)
{
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.0f), "f"(t));
    return r & 0xFFu;
}

__device__ __forceinline__ float e4m3_value(uint32_t byte)
{
    uint32_t h2;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"((uint16_t)byte));
    return __half2float(__ushort_as_half((unsigned short)(h2 & 0xFFFFu)));
}

// Block scale from the block's BF16 magnitude bits.  Writes the multiplier
// applied to the elements and returns the stored scale byte.
template <int FMT>
__device__ __forceinline__ uint32_t block_scale(uint32_t amax_bits, float gs, float denom,
                                                float* inv)
{
    const float amax = __uint_as_float(amax_bits << 16);
    if (FMT == kMx) {
        // e = ceil(log2(max(amax, 1e-8) / 6)).  For amax = f * 2^E, f in
        // [1, 2): e = E - 2 when f <= 1.5, else E - 1 (f > 1.5 <=> the 7-bit
        // BF16 mantissa exceeds 64).
        int e;
        if (amax < 1e-8f) {
            e = -29;
        } else {
            const int Eb = (int)((amax_bits >> 7) & 0xFF);
            e = Eb - 129 + ((amax_bits & 0x7F) > 64 ? 1 : 0);
        }
        *inv = __uint_as_float((uint32_t)(127 - e) << 23);  // 2^-e, exact
        return (uint32_t)(e + 127);
    } else if (FMT == kP1) {
        // e = ceil(log2(max(amax / (6 * S_global), 1e-8))) with the ratio
        // formed in FP32; for a = f * 2^E (a is normal), e = E when f == 1,
        // else E + 1; capped at 127.  S_block = 2^e, eff = S_block * S_global.
        const float a = fmaxf(__fdiv_rn(amax, denom), 1e-8f);
        const uint32_t ab = __float_as_uint(a);
        const int e = min((int)(ab >> 23) - 127 + ((ab & 0x7FFFFFu) ? 1 : 0), 127);
        const float eff = __fmul_rn(__uint_as_float((uint32_t)(e + 127) << 23), gs);
        *inv = (eff == 0.0f) ? 0.0f : fminf(__frcp_rn(eff), FLT_MAX);
        return (uint32_t)(e + 127);
    } else {
        const float t = __fdiv_rn(amax, denom);
        const uint32_t sb = cvt_e4m3(t);
        const float eff = __fmul_rn(e4m3_value(sb), gs);
        *inv = (eff == 0.0f) ? 0.0f : fminf(__frcp_rn(eff), FLT_MAX);
        return sb;
    }
}

// Eight BF16 values times `inv` (FP32 products), rounded to E2M1 with
// round-to-nearest-even and saturation: 8 nibbles, element 0 in the lowest.
// cvt...e2m1x2 puts its first source in the high nibble, its second in the
// low nibble.
__device__ __forceinline__ uint32_t quantize8(uint4 v, float inv)
{
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    float f[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        f[2 * i] = __fmul_rn(__uint_as_float(w[i] << 16), inv);
        f[2 * i + 1] = __fmul_rn(__uint_as_float(w[i] & 0xFFFF0000u), inv);
    }
    uint32_t out;
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
        "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
        : "=r"(out)
        : "f"(f[0]), "f"(f[1]), "f"(f[2]), "f"(f[3]), "f"(f[4]), "f"(f[5]), "f"(f[6]), "f"(f[7]));
    return out;
}

}  // namespace qdev
}  // namespace fp4
