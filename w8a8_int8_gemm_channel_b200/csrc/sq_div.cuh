// sq_div.cuh -- exact int8 quantisation of smoothed rows without an IEEE
// division per element.
//
// The quantisers compute, exactly as the IEEE definition does,
//   v_k   = RN(x_k / s_k)  (activations)  or  RN(x_k * s_k)  (weights)
//   scale = RN(max_k |v_k| / 127)
//   code  = clamp(round_half_even(RN(v_k / scale)), -127, 127)
// An IEEE division is a long instruction sequence, so the kernels use cheaper
// forms that provably give the same results:
//
// Row maximum E = max_k |x^_k| (activations, x^_k = RN(x_k / s_k)).  With r_k
// within 1 ulp of 1/s_k (hardware reciprocal), a_k = RN(|x_k| * r_k) is within
// 2^-21 (relative) of |x^_k| whenever a_k is normal, so the element that
// attains E satisfies a_k >= A * (1 - 2^-20), A the row's largest a.  Only such
// candidates get an exact IEEE quotient and E is the maximum of those (a row
// whose A is below 2^-100, or whose divisors leave [2^-60, 2^61), is done
// exactly throughout).
//
// Scale.  RN(E / 127) by Markstein's iteration with the constant RN(1/127)
// (P. Markstein, "Computation of elementary functions on the IBM RISC System/
// 6000 processor", IBM J. Res. Develop. 34(1), 1990): q0 = RN(E r),
// e = E - 127 q0 (exact, one FMA), RN(q0 + e r) is the correctly rounded
// quotient for E in [2^-100, 2^100]; other E take the IEEE division.
//
// Codes.  With rs within 1 ulp of 1/scale, the exact product
// t = RN(x_k r_k) * rs is within 7 * 2^-24 * |t| <= 5.4e-5 of RN(v_k / scale)
// for |t| <= 128 and a scale in [2^-100, 2^100]; so wherever t is farther than
// 2^-13 from a half-integer, round-half-even(t) is the code.  One FMA,
// RN(t + 1.5 * 2^23), rounds t to an integer half-even and leaves the code in
// the low byte of the sum.  Near ties (about 2^-12 of elements) recompute the
// exact quotient.
//
// These bounds were checked on the host against IEEE division on hundreds of
// millions of random and near-tie cases, with every reciprocal perturbed by up
// to 1 ulp.
#pragma once

#include <cstdint>

namespace sq {

constexpr float kRoundMagic = 12582912.0f;  // 1.5 * 2^23
constexpr float kCandidateScale = 1.0f - 0x1p-20f;
constexpr float kTieLimit = 0.5f - 0x1p-13f;
constexpr float kTinyQuotient = 0x1p-100f;

// |v| in [2^-60, 2^61)
__device__ __forceinline__ bool div_operand_ok(float v)
{
    const uint32_t e = (__float_as_uint(v) >> 23) & 0xFFu;
    return (e - 67u) <= 120u;
}

// Hardware reciprocal approximation (at most 1 ulp from 1/v for normal v).
__device__ __forceinline__ float rcp_approx(float v)
{
    float r;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(v));
    return r;
}

// 1/s within 1 ulp when s is usable by the fast paths, else 0.
__device__ __forceinline__ float fast_recip(float sv)
{
    return div_operand_ok(sv) ? rcp_approx(sv) : 0.0f;
}

// RN(E / 127) for E >= 0.
__device__ __forceinline__ float scale_from_max(float E)
{
    constexpr float r127 = 1.0f / 127.0f;
    if (E >= 0x1p-100f && E <= 0x1p100f) {
        const float q0 = __fmul_rn(E, r127);
        const float e = __fmaf_rn(-q0, 127.0f, E);
        return __fmaf_rn(e, r127, q0);
    }
    return __fdiv_rn(E, 127.0f);
}

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

// low bytes of four code-bit words packed into one 32-bit word
__device__ __forceinline__ uint32_t pack_code_bytes(uint32_t a, uint32_t b, uint32_t c, uint32_t d)
{
    return __byte_perm(__byte_perm(a, b, 0x0040u), __byte_perm(c, d, 0x0040u), 0x5410u);
}

}  // namespace sq
