// sq_div.cuh -- correctly rounded fp32 division and int8 code rounding, fast.
//
// The quantisers divide twice per element (x / s_k for the smoothed value and
// v / scale for the code), and IEEE division is a long instruction sequence
// that would make those kernels compute-bound.  Two cheaper forms with the
// same results are used:
//
// 1. div_rn(x, d, r) with r = RN(1/d): Markstein's division (P. Markstein,
//    "Computation of elementary functions on the IBM RISC System/6000
//    processor", IBM J. Res. Develop. 34(1), 1990):
//        q0 = RN(x * r);   e = x - q0 * d  (exact, one FMA);   q = RN(q0 + e * r)
//    gives the correctly rounded quotient RN(x / d) when no intermediate is
//    subnormal or overflows.  It is used when |x| and |d| lie in [2^-60, 2^61)
//    (or x == 0), where the quotient and the remainder stay normal; any other
//    operand takes the IEEE division.  The divisor's reciprocal is prepared by
//    div_recip(), which returns 0 for a divisor outside that range.
//
// 2. quant_code(v, scale, rs) with rs = RN(1/scale) and |v| <= 127.x * scale:
//    t = RN(v * rs) lies within 2 ulp(t) <= 2^-16 of the exact quotient, so
//    when t is farther than 2^-14 from a half-integer, round-half-even(t)
//    equals round-half-even of the correctly rounded quotient; otherwise the
//    IEEE division decides.  A NaN or infinite t (scale tiny or zero) also
//    takes the IEEE path.
#pragma once

#include <cstdint>

namespace sq {

__device__ __forceinline__ bool div_operand_ok(float v)
{
    const uint32_t e = (__float_as_uint(v) >> 23) & 0xFFu;
    return (e - 67u) <= 120u;  // 2^-60 <= |v| < 2^61
}

// RN(1/d) when d is usable by div_rn's fast path, else 0.
__device__ __forceinline__ float div_recip(float d)
{
    return div_operand_ok(d) ? __frcp_rn(d) : 0.0f;
}

// RN(x / d); r = div_recip(d).
__device__ __forceinline__ float div_rn(float x, float d, float r)
{
    if (r != 0.0f && (x == 0.0f || div_operand_ok(x))) {
        const float q0 = __fmul_rn(x, r);
        if (x == 0.0f)
            return q0;  // keeps the IEEE sign of a zero quotient
        const float e = __fmaf_rn(-q0, d, x);
        return __fmaf_rn(e, r, q0);
    }
    return __fdiv_rn(x, d);
}

// clamp(round_half_even(RN(v / scale)), -127, 127); rs = RN(1/scale).
__device__ __forceinline__ int quant_code(float v, float scale, float rs)
{
    const float t = __fmul_rn(v, rs);
    const float a = fabsf(t);
    const float fr = a - floorf(a);
    int q;
    if (fabsf(fr - 0.5f) > 0x1p-14f)
        q = __float2int_rn(t);
    else
        q = __float2int_rn(__fdiv_rn(v, scale));
    return max(-127, min(127, q));
}

// Branch-free pieces for vectorised loops: the fast result is always computed
// and a flag says when it may differ from the IEEE result; callers OR the flags
// over a chunk and redo that chunk with __fdiv_rn (rare).
__device__ __forceinline__ bool div_fast_unsafe(float x)
{
    // |x| outside [2^-60, 2^61) and not zero
    const uint32_t a = __float_as_uint(x) & 0x7FFFFFFFu;
    return (a - 0x21800000u) >= (0x5E000000u - 0x21800000u) && a != 0u;
}

// RN(x / d) by Markstein's iteration, r = RN(1/d) != 0 (no range checks; a
// zero x gives +0 or -0, either of which has the same magnitude and code).
__device__ __forceinline__ float div_markstein(float x, float d, float r)
{
    const float q0 = __fmul_rn(x, r);
    const float e = __fmaf_rn(-q0, d, x);
    return __fmaf_rn(e, r, q0);
}

// round_half_even(t) as a float and a flag for "within 2^-14 of a tie".
__device__ __forceinline__ float round_code(float v, float rs, bool &near_tie)
{
    const float t = __fmul_rn(v, rs);
    const float r = rintf(t);
    near_tie = !(fabsf(t - r) < 0.5f - 0x1p-14f);  // also true for NaN t
    return fminf(fmaxf(r, -127.0f), 127.0f);
}

// ----------------------------------------------------------------------------
// Cheap exact quantisation of a smoothed row, x^_k = RN(x_k / s_k):
//
// Row maximum E = max_k |x^_k|.  a_k = RN(|x_k| * r_k), r_k = RN(1/s_k), is
// within 2^-22 (relative) of |x^_k| whenever a_k is normal, so the element that
// attains E satisfies a_k >= A * (1 - 2^-20) for every running maximum A of
// the a's seen so far.  Only such candidates (and the a_k < 2^-100 elements,
// whose relative error is not bounded) get an exact IEEE quotient; E is the
// maximum of those exact quotients.
//
// Codes.  With scale = RN(E/127) and rs = RN(1/scale), t = RN(RN(x_k r_k) rs)
// is within 6 * 2^-24 * |t| <= 4.6e-5 of RN(x^_k / scale) for |t| <= 128 and a
// scale in [2^-100, 2^100]; so wherever t is farther than 2^-13 from a
// half-integer, round-half-even(t) is the code.  Adding 1.5 * 2^23 rounds t to
// an integer half-even and leaves the code in the low byte of the sum.  Near
// ties (about 2^-12 of elements) recompute the exact quotient.
// ----------------------------------------------------------------------------
constexpr float kRoundMagic = 12582912.0f;       // 1.5 * 2^23
constexpr float kCandidateScale = 1.0f - 0x1p-20f;
constexpr float kTieLimit = 0.5f - 0x1p-13f;
constexpr float kTinyQuotient = 0x1p-100f;

__device__ __forceinline__ bool scale_in_fast_range(float sc)
{
    return sc >= 0x1p-100f && sc <= 0x1p100f;
}

// the magic-sum bit pattern whose low byte is the code q (q in [-127, 127])
__device__ __forceinline__ uint32_t code_bits(float q)
{
    return __float_as_uint(__fadd_rn(q, kRoundMagic));
}

// exact code of an exact quotient v / scale
__device__ __forceinline__ uint32_t exact_code_bits(float v, float scale)
{
    return code_bits(fminf(fmaxf(rintf(__fdiv_rn(v, scale)), -127.0f), 127.0f));
}

// fast code bits for t (the approximate quotient); sets tie when unsafe
__device__ __forceinline__ uint32_t fast_code_bits(float t, bool &tie)
{
    const float y = __fadd_rn(t, kRoundMagic);
    const float r = __fsub_rn(y, kRoundMagic);
    tie |= !(fabsf(__fsub_rn(t, r)) < kTieLimit);
    return __float_as_uint(y);
}

// low bytes of four code-bit words packed into one 32-bit word
__device__ __forceinline__ uint32_t pack_code_bytes(uint32_t a, uint32_t b, uint32_t c, uint32_t d)
{
    return __byte_perm(__byte_perm(a, b, 0x0040u), __byte_perm(c, d, 0x0040u), 0x5410u);
}

}  // namespace sq
