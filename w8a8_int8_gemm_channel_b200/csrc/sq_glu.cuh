// sq_glu.cuh -- the gated feed-forward activation of a decoder layer,
// h = SiLU(gate) * up, computed inside the per-token quantiser that feeds the
// down projection, so that h never travels through HBM.
//
// The per-token quantisation of each layer's activations is memory-bound work
// ("Understanding W8A8 INT8 LLM Quantization", section "Inter-Token Latency
// (ITL)"), and fusing the feed-forward network with its neighbours saves
// memory traffic ("How does SmoothQuant int8 LLM calibration work...",
// section "Hardware Acceleration and Inference Optimization Strategies").
//
// Definition: a fixed sequence of IEEE binary32 operations, so that any
// implementation that follows it gets the same bits.
//   E(x)    = e^x:  0 for x < -87, +inf for x > 88, else Cody and Waite's
//             reduction n = nearest integer to x * RN(log2 e) (by adding and
//             removing 1.5 * 2^23 in one FMA), r = x - n RN(ln 2) - n
//             RN(ln 2 - RN(ln 2)) (two FMAs), the Taylor series of e^r to
//             degree 7 by Horner's rule (one FMA a step, coefficients
//             RN(1/k!)), times 2^n (exact: the result is normal);
//   SiLU(z) = RN(z / RN(1 + E(-z)));
//   v       = RN(SiLU(gate) * up);  h = RN_bf16(v) for bf16 rows (the value an
//             unfused feed-forward step would store), v itself for fp32 rows.
//
// Fast path (bf16 rows).  v' = RN(RN(g * y) * u) with y = rcp(RN(1 + ex2(RN(-g
// log2 e)))) from the hardware approximations.  For gate >= -16 the exponent
// argument's rounding costs at most ln 2 * 23.1 * 2^-24 relative, the
// approximate ex2 and rcp a few 2^-24 each, and the fp32 roundings of both
// sides a few more, so bits(v') lies within about 40 patterns of bits(v)
// (the two share their sign; within one sign the bit patterns are ordered
// like the values, subnormals and infinity included).  Measured on B200 over
// every bf16 gate >= -16 against 4096 up values: at most 14.  RN_bf16 rounds at the
// patterns ending in 0x8000, so RN_bf16(v') = RN_bf16(v) unless such a pattern
// lies within kGluWindow = 64 of bits(v'): about 1 element in 500.  Those
// chunks, and chunks with a gate below -16 (where e^-g grows and the
// argument's rounding with it), take the definition.
#pragma once

#include <cstdint>

#include <cuda_bf16.h>

#include "sq_div.cuh"
#include "sq_mem.cuh"
#include "sq_ptx.cuh"

namespace sq {

constexpr float kLog2e = 0x1.715476p+0f;  // RN(log2 e)
constexpr float kLn2Hi = 0x1.62e430p-1f;  // RN(ln 2)
constexpr float kLn2Lo = -0x1.05c610p-29f;  // RN(ln 2 - RN(ln 2))
constexpr uint32_t kGluWindow = 64;  // fp32 bit patterns either side of v'
constexpr float kGluGateMin = -16.0f;

// e^x by the fixed sequence above
__device__ __forceinline__ float glu_exp(float x)
{
    if (x < -87.0f)
        return 0.0f;
    if (x > 88.0f)
        return __uint_as_float(0x7F800000u);
    const float n = __fsub_rn(__fmaf_rn(x, kLog2e, kRoundMagic), kRoundMagic);
    float r = __fmaf_rn(-n, kLn2Hi, x);
    r = __fmaf_rn(-n, kLn2Lo, r);
    float p = 0x1.a01a02p-13f;           // 1/7!
    p = __fmaf_rn(p, r, 0x1.6c16c2p-10f);  // 1/6!
    p = __fmaf_rn(p, r, 0x1.111112p-7f);   // 1/5!
    p = __fmaf_rn(p, r, 0x1.555556p-5f);   // 1/4!
    p = __fmaf_rn(p, r, 0x1.555556p-3f);   // 1/3!
    p = __fmaf_rn(p, r, 0.5f);             // 1/2!
    p = __fmaf_rn(p, r, 1.0f);
    p = __fmaf_rn(p, r, 1.0f);
    // p * 2^n by the exponent field: p and the result are normal
    return __int_as_float(__float_as_int(p) + (static_cast<int>(n) << 23));
}

// v = RN(SiLU(g) * u) by the definition
__device__ __forceinline__ float glu_value(float g, float u)
{
    const float d = __fadd_rn(1.0f, glu_exp(-g));
    return __fmul_rn(__fdiv_rn(g, d), u);
}

__device__ __forceinline__ float ex2_approx(float x)
{
    float r;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
    return r;
}

// elementwise minimum of two bf16 pairs
__device__ __forceinline__ uint32_t bf2_min(uint32_t a, uint32_t b)
{
    uint32_t d;
    asm("min.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

__device__ __forceinline__ uint32_t bf16x2_rn(float lo, float hi)
{
    const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t *>(&h);
}

// h of one 16-byte chunk by the definition, from the raw gate and up chunks
template <typename T>
__device__ __forceinline__ uint4 glu_chunk_exact(const uint4 &g, const uint4 &u)
{
    constexpr int V = Vec<T>::N;
    float gv[V], uv[V];
    widen<T>(g, gv);
    widen<T>(u, uv);
    if constexpr (V == 8) {
        return make_uint4(bf16x2_rn(glu_value(gv[0], uv[0]), glu_value(gv[1], uv[1])),
                          bf16x2_rn(glu_value(gv[2], uv[2]), glu_value(gv[3], uv[3])),
                          bf16x2_rn(glu_value(gv[4], uv[4]), glu_value(gv[5], uv[5])),
                          bf16x2_rn(glu_value(gv[6], uv[6]), glu_value(gv[7], uv[7])));
    } else {
        return make_uint4(__float_as_uint(glu_value(gv[0], uv[0])), __float_as_uint(glu_value(gv[1], uv[1])),
                          __float_as_uint(glu_value(gv[2], uv[2])), __float_as_uint(glu_value(gv[3], uv[3])));
    }
}

// a bf16 rounding midpoint within kGluWindow patterns of b:
// ((b + 0x8000 + W) mod 2^16) <= 2W, tested in the high half-word
__device__ __forceinline__ bool glu_near_midpoint(uint32_t b)
{
    constexpr uint32_t add = (0x8000u + kGluWindow) << 16;
    constexpr uint32_t lim = (2u * kGluWindow) << 16;
    return (b * 65536u + add) <= lim;
}

// v' of the fast path for one element
__device__ __forceinline__ float glu_value_fast(float g, float u)
{
    const float d = __fadd_rn(ex2_approx(__fmul_rn(g, -kLog2e)), 1.0f);
    return __fmul_rn(__fmul_rn(g, rcp_approx(d)), u);
}

// The rare path, out of line, for a bf16 chunk the fast path could not
// decide (its raw gate and up, still in registers): each element keeps its
// fast value unless it is the one (or ones) that needs the definition.
__device__ __noinline__ uint4 glu_chunk_fix(uint4 g, uint4 u)
{
    float gv[8], uv[8], hv[8];
    widen<__nv_bfloat16>(g, gv);
    widen<__nv_bfloat16>(u, uv);
    for (int e = 0; e < 8; ++e) {
        const float v = glu_value_fast(gv[e], uv[e]);
        hv[e] = (glu_near_midpoint(__float_as_uint(v)) || !(gv[e] >= kGluGateMin)) ? glu_value(gv[e], uv[e]) : v;
    }
    return make_uint4(bf16x2_rn(hv[0], hv[1]), bf16x2_rn(hv[2], hv[3]), bf16x2_rn(hv[4], hv[5]),
                      bf16x2_rn(hv[6], hv[7]));
}

// h of one bf16 chunk by the fast path; `redo` is set when the chunk must take
// the definition instead
__device__ __forceinline__ uint4 glu_chunk_fast(const uint4 &g, const uint4 &u, bool &redo)
{
    const uint32_t gw[4] = {g.x, g.y, g.z, g.w};
    const uint32_t uw[4] = {u.x, u.y, u.z, u.w};
    uint32_t hw[4];
    const float2 nl2e = make_float2(-kLog2e, -kLog2e);
    const float2 one2 = make_float2(1.0f, 1.0f);
    bool near = false;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const float2 g2 = make_float2(__uint_as_float(bf16_lo_bits(gw[k])), __uint_as_float(gw[k] & 0xFFFF0000u));
        const float2 u2 = make_float2(__uint_as_float(bf16_lo_bits(uw[k])), __uint_as_float(uw[k] & 0xFFFF0000u));
        const float2 t = f2_mul(g2, nl2e);
        const float2 d = f2_add(make_float2(ex2_approx(t.x), ex2_approx(t.y)), one2);
        const float2 v = f2_mul(f2_mul(g2, make_float2(rcp_approx(d.x), rcp_approx(d.y))), u2);
        const uint32_t bx = __float_as_uint(v.x), by = __float_as_uint(v.y);
        near |= glu_near_midpoint(bx);
        near |= glu_near_midpoint(by);
        hw[k] = bf16x2_rn(v.x, v.y);
    }
    // the smallest gate of the chunk
    const uint32_t m = bf2_min(bf2_min(gw[0], gw[1]), bf2_min(gw[2], gw[3]));
    const float gmin = fminf(__uint_as_float(bf16_lo_bits(m)), __uint_as_float(m & 0xFFFF0000u));
    redo = near || !(gmin >= kGluGateMin);
    return make_uint4(hw[0], hw[1], hw[2], hw[3]);
}

}  // namespace sq
