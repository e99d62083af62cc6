// Device helpers shared by the kernels that produce MXFP4 operands
// (quantize_act, pack_weights and the fused FFN epilogue of dual_gemm):
// BF16 rounding, the OCP MX shared exponent, E2M1 conversion, and the FP32
// tanh-form GELU used between the two FFN projections.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <cstdint>

namespace osm {
namespace mx {

__device__ __forceinline__ float bf16_bits_to_f32(uint32_t h) { return __uint_as_float(h << 16); }

// FP32 -> BF16 bits, round to nearest even (cvt.rn.bf16.f32).
__device__ __forceinline__ uint32_t f32_to_bf16_bits(float f) {
    return static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(f)));
}

// Two FP32 values -> BF16 pair (RNE each, one cvt.rn.bf16x2.f32): lo in
// bits 0-15, hi in bits 16-31.
__device__ __forceinline__ uint32_t bf16x2_bits(float lo, float hi) {
    uint32_t d;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(hi), "f"(lo));
    return d;
}

// Two FP32 values -> binary16 pair (RNE each, one cvt.rn.f16x2.f32): lo in
// bits 0-15, hi in bits 16-31.
__device__ __forceinline__ uint32_t f16x2_bits(float lo, float hi) {
    uint32_t d;
    asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(hi), "f"(lo));
    return d;
}

// Two FP32 values -> two E4M3 codes (RNE, saturating at +-448): lo in bits
// 0-7, hi in bits 8-15.
__device__ __forceinline__ uint32_t e4m3x2_bits(float lo, float hi) {
    uint16_t d;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(d) : "f"(hi), "f"(lo));
    return d;
}

// Two E4M3 codes (lo in bits 0-7) -> their values (exact: E4M3 is a subset
// of binary16).
__device__ __forceinline__ float2 e4m3x2_to_f32(uint32_t codes) {
    uint32_t h;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h) : "h"(static_cast<uint16_t>(codes)));
    return __half22float2(*reinterpret_cast<const __half2*>(&h));
}

// NVFP4 block scales of two blocks from their maxima (BF16 bit patterns,
// sign clear): S = E4M3_RNE_satfinite(fp32(amax * k)) with k = fp32(1/6) *
// 2^-g, and each block's element multiplier R = fp32(1 / (S * 2^g)), 0 when
// S is 0. Returns the two codes (lo in bits 0-7).
__device__ __forceinline__ uint32_t nv_block_scales(uint32_t amax_lo, uint32_t amax_hi, float k, float p2g,
                                                    float* r_lo, float* r_hi) {
    const uint32_t s2 = e4m3x2_bits(__fmul_rn(bf16_bits_to_f32(amax_lo), k), __fmul_rn(bf16_bits_to_f32(amax_hi), k));
    const float2 d = e4m3x2_to_f32(s2);
    *r_lo = (s2 & 0xFFu) ? __frcp_rn(__fmul_rn(d.x, p2g)) : 0.0f;
    *r_hi = (s2 & 0xFF00u) ? __frcp_rn(__fmul_rn(d.y, p2g)) : 0.0f;
    return s2;
}

// Eight BF16 values (4 packed words) times a power of two, each rounded
// back to BF16 (exact unless the product leaves the normal range).
__device__ __forceinline__ uint4 scale_bf16x8(uint4 v, float f) {
    const float2 f2 = make_float2(f, f);
    auto one = [&](uint32_t w) {
        const float2 x = __fmul2_rn(make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u)), f2);
        return bf16x2_bits(x.x, x.y);
    };
    return make_uint4(one(v.x), one(v.y), one(v.z), one(v.w));
}

// max(|a|, |b|) of each BF16 half of two packed words; the sign bits of the
// result are the XOR of the inputs' signs (mask them off before use).
__device__ __forceinline__ uint32_t bf16x2_absmax(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

// For a BF16 block maximum (bit pattern, sign clear): the MX exponent
// X = floor(log2 amax) - 2 clamped to [-127, 127] (amax 0 -> -127) is
// max(e - 129, -127) with e the biased exponent field -- a subnormal or zero
// amax is below 2^-126, so its X clamps to -127, and e <= 254 keeps X <= 125.
// Returns X; *inv receives 2^-X (exact, normal).
__device__ __forceinline__ int bf16_block_exponent(uint32_t amax_bits, float* inv) {
    const int e = static_cast<int>(amax_bits >> 7);
    const int X = max(e - 129, -127);
    *inv = __uint_as_float(static_cast<uint32_t>(127 - X) << 23);
    return X;
}

// MX shared exponent X = floor(log2 amax) - 2, clamped to [-127, 127],
// amax == 0 -> -127. amax is a finite, non-negative float; floor(log2) is
// read from the exponent field (subnormals from the leading mantissa bit).
__device__ __forceinline__ int exponent(float amax) {
    const uint32_t u = __float_as_uint(amax);
    if (u == 0u) return -127;
    const int e = static_cast<int>((u >> 23) & 0xFFu);
    const int fl = e ? e - 127 : (31 - __clz(u & 0x7FFFFFu)) - 149;
    int X = fl - 2;
    X = X < -127 ? -127 : X;
    X = X > 127 ? 127 : X;
    return X;
}

// 2^-X as an exact float for X in [-127, 127].
__device__ __forceinline__ float exp2_neg(int X) {
    return X <= 126 ? __uint_as_float(static_cast<uint32_t>(127 - X) << 23)
                    : __uint_as_float(0x00400000u >> (X - 127));
}

// Two FP32 values -> E2M1x2 (round to nearest even, saturating at +-6),
// element `lo` in the low nibble; the sign of a code is the sign of its
// input, also for inputs that round to zero.
__device__ __forceinline__ uint32_t e2m1x2(float lo, float hi) {
    uint16_t out;
    asm("{\n\t.reg .b8 b;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b, %2, %1;\n\t"
        "cvt.u16.u8 %0, b;\n\t}"
        : "=h"(out)
        : "f"(lo), "f"(hi));
    return out;
}

// Eight BF16 values (4 packed words, element 0 in the low half of word 0)
// scaled by `inv` (a power of two, so exact) -> eight E2M1 codes, element i
// in nibble i. The scaling is two packed FP32 multiplies per word (each lane
// an IEEE multiply), and the four code bytes are packed in one step.
__device__ __forceinline__ uint32_t encode8_words(uint32_t w0, uint32_t w1, uint32_t w2, uint32_t w3, float inv) {
    const float2 iv = make_float2(inv, inv);
    const float2 v0 = __fmul2_rn(make_float2(__uint_as_float(w0 << 16), __uint_as_float(w0 & 0xFFFF0000u)), iv);
    const float2 v1 = __fmul2_rn(make_float2(__uint_as_float(w1 << 16), __uint_as_float(w1 & 0xFFFF0000u)), iv);
    const float2 v2 = __fmul2_rn(make_float2(__uint_as_float(w2 << 16), __uint_as_float(w2 & 0xFFFF0000u)), iv);
    const float2 v3 = __fmul2_rn(make_float2(__uint_as_float(w3 << 16), __uint_as_float(w3 & 0xFFFF0000u)), iv);
    uint32_t out;
    asm("{\n\t.reg .b8 c0, c1, c2, c3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 c0, %2, %1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 c1, %4, %3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 c2, %6, %5;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 c3, %8, %7;\n\t"
        "mov.b32 %0, {c0, c1, c2, c3};\n\t}"
        : "=r"(out)
        : "f"(v0.x), "f"(v0.y), "f"(v1.x), "f"(v1.y), "f"(v2.x), "f"(v2.y), "f"(v3.x), "f"(v3.y));
    return out;
}

__device__ __forceinline__ float2 splat2(float a) { return make_float2(a, a); }

// 2^z and 1/d on the special-function unit (ex2.approx.ftz.f32,
// rcp.approx.ftz.f32: hardware instructions of a few ulp; subnormal results
// flush to zero).
__device__ __forceinline__ float ex2_approx(float z) {
    float r;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(z));
    return r;
}
__device__ __forceinline__ float rcp_approx(float d) {
    float r;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(d));
    return r;
}

// GELU in its tanh form, 0.5 x (1 + tanh(u)) with u = sqrt(2/pi)(x +
// 0.044715 x^3), on two values at once. Since 0.5 (1 + tanh(u)) =
// 1 / (1 + exp(-2u)), GELU(x) = x / (1 + 2^z) with z = -2 u log2(e) =
// x (A + B x^2), A = -2 sqrt(2/pi) log2(e), B = 0.044715 A: three packed FP32
// operations give z, the special-function unit gives 2^z and the
// reciprocal, and one more multiply the result. z is capped at 126 so that
// 1 + 2^z stays finite (GELU(x) is then below |x| 2^-126 in magnitude); for
// z below -126, 2^z flushes to 0 and the result is x. Within 5e-7 |GELU(x)|
// + 2e-8 |x| of the exact function (measured against an FP64 evaluation on
// the device).
__device__ __forceinline__ float2 gelu2(float2 x) {
    const float2 x2 = __fmul2_rn(x, x);
    const float2 t = __ffma2_rn(x2, splat2(-0x1.a5a7d0p-4f), splat2(-0x1.26aec2p+1f));
    const float2 z = __fmul2_rn(x, t);
    const float2 e = make_float2(ex2_approx(fminf(z.x, 126.0f)), ex2_approx(fminf(z.y, 126.0f)));
    const float2 d = __fadd2_rn(e, splat2(1.0f));
    return __fmul2_rn(x, make_float2(rcp_approx(d.x), rcp_approx(d.y)));
}

// Byte offset of E8M0 scale (row r, 32-block b) in the tcgen05 block-scale
// layout: 512-byte atoms of 128 rows x 4 blocks.
__device__ __forceinline__ int64_t sf_offset(int64_t r, int64_t b, int64_t katoms) {
    return ((r >> 7) * katoms + (b >> 2)) * 512 + (r & 31) * 16 + ((r & 127) >> 5) * 4 + (b & 3);
}

}  // namespace mx
}  // namespace osm
