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

// The GELU below works on two values at once with the packed FP32
// instructions of sm_100 (fma / mul / add .rn.f32x2): each lane of a packed
// operation is one IEEE operation rounded to nearest even, so every element
// goes through exactly the operations of the scalar definition, in the same
// order, at half the instruction count. Negated operands are written as
// negated constants (x (-c) = (-x) c exactly).
__device__ __forceinline__ float2 splat2(float a) { return make_float2(a, a); }

// exp(a) for a <= 0 in FP32: a clamped to -100, Cody-Waite reduction
// a = n ln2 + r with ln2 split into a 12-bit high part and a low remainder,
// the degree-7 Taylor polynomial of exp(r) in Horner form with fused
// multiply-adds, then p * 2^n rounded once, or 0 for n < -126. n =
// round(a log2 e) comes from one fused multiply-add onto 1.5*2^23 (FP32
// spacing 1 there), so its integer value is read off the low bits of the sum
// and the factor 2^n is built from bits (an exponent field clamped at 0
// gives the factor 0). Every operation is an explicitly rounded intrinsic so
// that no contraction or reassociation changes the result.
__device__ __forceinline__ float2 gelu_exp_neg2(float2 a) {
    const float2 ac = make_float2(fmaxf(a.x, -100.0f), fmaxf(a.y, -100.0f));
    const float2 t = __ffma2_rn(ac, splat2(0x1.715476p+0f), splat2(0x1.8p+23f));
    const float2 n = __fadd2_rn(t, splat2(-0x1.8p+23f));
    float2 r = __ffma2_rn(n, splat2(-0x1.62e4p-1f), ac);
    r = __ffma2_rn(n, splat2(-0x1.7f7d1cp-20f), r);
    float2 q = __ffma2_rn(splat2(0x1.a01a02p-13f), r, splat2(0x1.6c16c2p-10f));
    q = __ffma2_rn(q, r, splat2(0x1.111112p-7f));
    q = __ffma2_rn(q, r, splat2(0x1.555556p-5f));
    q = __ffma2_rn(q, r, splat2(0x1.555556p-3f));
    q = __ffma2_rn(q, r, splat2(0.5f));
    q = __ffma2_rn(q, r, splat2(1.0f));
    q = __ffma2_rn(q, r, splat2(1.0f));
    // t = 1.5*2^23 + n with n in [-145, 0]: its bit pattern is that of 1.5*2^23 plus n
    const int ex = max(static_cast<int>(__float_as_uint(t.x) - 0x4B400000u) + 127, 0);
    const int ey = max(static_cast<int>(__float_as_uint(t.y) - 0x4B400000u) + 127, 0);
    return __fmul2_rn(q, make_float2(__uint_as_float(static_cast<uint32_t>(ex) << 23),
                                     __uint_as_float(static_cast<uint32_t>(ey) << 23)));
}

// 1/d for d in [1, 2], given nd = -d: linear seed 24/17 - (8/17) d, then
// three Newton steps y <- y + y (1 - d y) as two fused multiply-adds each.
__device__ __forceinline__ float2 gelu_recip2_neg(float2 nd) {
    float2 y = __ffma2_rn(splat2(0x1.e1e1e2p-2f), nd, splat2(0x1.69696ap+0f));
#pragma unroll
    for (int i = 0; i < 3; ++i) {
        const float2 e = __ffma2_rn(nd, y, splat2(1.0f));
        y = __ffma2_rn(y, e, y);
    }
    return y;
}

// GELU_tanh(x) = 0.5 x (1 + tanh(u)), u = sqrt(2/pi)(x + 0.044715 x^3), for
// finite x, through 0.5 (1 + tanh(u)) = sigma(2u): with E = exp(-2|u|),
// x sigma(2u) = x/(1+E) for u >= 0 and x E/(1+E) for u < 0; u has the sign
// of x and 0 <= E <= 1, so the numerator is max(x, x E). Operations per
// element in this order: x2 = x x; k = fma(C1, x2, 1); u = (C0 x) k; E; y =
// recip(1 + E) (1 + E formed as -(1 + E) = fma(E, -1, -1), the same rounding
// with the sign flipped); max(x, x E) y. No division, no branch.
__device__ __forceinline__ float2 gelu_tanh2(float2 x) {
    const float2 x2 = __fmul2_rn(x, x);
    const float2 k = __ffma2_rn(splat2(0x1.6e4e26p-5f), x2, splat2(1.0f));    // C1 = 0.044715
    const float2 u = __fmul2_rn(__fmul2_rn(splat2(0x1.988454p-1f), x), k);   // C0 = sqrt(2/pi)
    const float2 E = gelu_exp_neg2(__fmul2_rn(make_float2(fabsf(u.x), fabsf(u.y)), splat2(-2.0f)));
    const float2 y = gelu_recip2_neg(__ffma2_rn(E, splat2(-1.0f), splat2(-1.0f)));
    const float2 xE = __fmul2_rn(x, E);
    return __fmul2_rn(make_float2(fmaxf(x.x, xE.x), fmaxf(x.y, xE.y)), y);
}

// Byte offset of E8M0 scale (row r, 32-block b) in the tcgen05 block-scale
// layout: 512-byte atoms of 128 rows x 4 blocks.
__device__ __forceinline__ int64_t sf_offset(int64_t r, int64_t b, int64_t katoms) {
    return ((r >> 7) * katoms + (b >> 2)) * 512 + (r & 31) * 16 + ((r & 127) >> 5) * 4 + (b & 3);
}

}  // namespace mx
}  // namespace osm
