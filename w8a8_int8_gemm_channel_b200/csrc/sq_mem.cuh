// sq_mem.cuh -- the HBM-bound stages of the SmoothQuant W8A8 linear layer:
//   * column absmax (calibration statistics A_j, weight input-channel B_j),
//   * smoothing factors s_j = A_j^alpha / B_j^(1-alpha),
//   * smoothed per-output-channel weight quantisation,
//   * dynamic per-token activation quantisation.
//
// Sources (page title, section): "Understanding W8A8 INT8 LLM Quantization" --
// "Why Naive Weight Quantization Doesn't Work, and How GPTQ Fixes It" (scale
// max|w|/127, round(w/scale)), "Why Activation Quantization Is Hard, and How
// SmoothQuant Fixes It" (one dynamic scale per token), "Where the outlier
// actually comes from" and "How the smoothing factor is computed" (absmax per
// channel over calibration samples, s_j, X/s and W*s).
//
// Arithmetic: every rounded step is a single IEEE fp32 operation with
// round-to-nearest-even, spelled with the explicit _rn intrinsics so no
// multiply-add is fused; rounding to int8 is round-half-to-even followed by a
// clamp to [-127, 127]; a zero maximum gives scale 0 and zero codes.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

#include "sq_ptx.cuh"

namespace sq {

// 16-byte vector of inputs: 8 bf16 or 4 fp32 values.
template <typename T>
struct Vec;
template <>
struct Vec<__nv_bfloat16> {
    static constexpr int N = 8;
};
template <>
struct Vec<float> {
    static constexpr int N = 4;
};

__device__ __forceinline__ float bf16_bits_to_f32(uint32_t b16)
{
    return __uint_as_float(b16 << 16);
}

// Load one 16-byte vector (read-only path) and widen it to fp32.
template <typename T>
__device__ __forceinline__ void load_vec(const T *p, float (&v)[Vec<T>::N]);

template <>
__device__ __forceinline__ void load_vec<__nv_bfloat16>(const __nv_bfloat16 *p, float (&v)[8])
{
    uint4 u = __ldg(reinterpret_cast<const uint4 *>(p));
    v[0] = bf16_bits_to_f32(u.x & 0xFFFFu);
    v[1] = bf16_bits_to_f32(u.x >> 16);
    v[2] = bf16_bits_to_f32(u.y & 0xFFFFu);
    v[3] = bf16_bits_to_f32(u.y >> 16);
    v[4] = bf16_bits_to_f32(u.z & 0xFFFFu);
    v[5] = bf16_bits_to_f32(u.z >> 16);
    v[6] = bf16_bits_to_f32(u.w & 0xFFFFu);
    v[7] = bf16_bits_to_f32(u.w >> 16);
}

template <>
__device__ __forceinline__ void load_vec<float>(const float *p, float (&v)[4])
{
    float4 u = __ldg(reinterpret_cast<const float4 *>(p));
    v[0] = u.x;
    v[1] = u.y;
    v[2] = u.z;
    v[3] = u.w;
}

// Streaming (evict-first) variant for data read exactly once.
template <typename T>
__device__ __forceinline__ void load_vec_stream(const T *p, float (&v)[Vec<T>::N]);

template <>
__device__ __forceinline__ void load_vec_stream<__nv_bfloat16>(const __nv_bfloat16 *p,
                                                               float (&v)[8])
{
    uint4 u = __ldcs(reinterpret_cast<const uint4 *>(p));
    v[0] = bf16_bits_to_f32(u.x & 0xFFFFu);
    v[1] = bf16_bits_to_f32(u.x >> 16);
    v[2] = bf16_bits_to_f32(u.y & 0xFFFFu);
    v[3] = bf16_bits_to_f32(u.y >> 16);
    v[4] = bf16_bits_to_f32(u.z & 0xFFFFu);
    v[5] = bf16_bits_to_f32(u.z >> 16);
    v[6] = bf16_bits_to_f32(u.w & 0xFFFFu);
    v[7] = bf16_bits_to_f32(u.w >> 16);
}

template <>
__device__ __forceinline__ void load_vec_stream<float>(const float *p, float (&v)[4])
{
    float4 u = __ldcs(reinterpret_cast<const float4 *>(p));
    v[0] = u.x;
    v[1] = u.y;
    v[2] = u.z;
    v[3] = u.w;
}

// clamp(round_half_even(v / scale), -127, 127) as a byte; scale > 0.
__device__ __forceinline__ uint32_t quant_code(float v, float scale)
{
    int q = __float2int_rn(__fdiv_rn(v, scale));
    q = max(-127, min(127, q));
    return static_cast<uint32_t>(q) & 0xFFu;
}

// ----------------------------------------------------------------------------
// Column absmax: out[j] = max(out[j], max_r |x[r, j]|), out as fp32 bit
// patterns (non-negative floats order like their unsigned bit patterns).
// Block: 256 threads = 256 consecutive 16-byte column chunks; blockIdx.y
// selects a band of `rows_per_block` rows.  Coalesced 16-byte loads, one
// atomicMax per channel per CTA.
// ----------------------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(256) col_absmax_kernel(const T *__restrict__ x, int64_t R,
                                                          int64_t K, int64_t ld,
                                                          int64_t rows_per_block,
                                                          unsigned int *__restrict__ out_bits)
{
    constexpr int V = Vec<T>::N;
    const int64_t chunks = K / V;
    const int64_t c = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (c >= chunks)
        return;
    const int64_t r0 = static_cast<int64_t>(blockIdx.y) * rows_per_block;
    const int64_t r1 = min(R, r0 + rows_per_block);
    float m[V];
#pragma unroll
    for (int i = 0; i < V; ++i)
        m[i] = 0.0f;
    const T *p = x + r0 * ld + c * V;
    int64_t r = r0;
    for (; r + 4 <= r1; r += 4, p += 4 * ld) {
        float a[V], b[V], d[V], e[V];
        load_vec_stream<T>(p, a);
        load_vec_stream<T>(p + ld, b);
        load_vec_stream<T>(p + 2 * ld, d);
        load_vec_stream<T>(p + 3 * ld, e);
#pragma unroll
        for (int i = 0; i < V; ++i)
            m[i] = fmaxf(m[i], fmaxf(fmaxf(fabsf(a[i]), fabsf(b[i])), fmaxf(fabsf(d[i]), fabsf(e[i]))));
    }
    for (; r < r1; ++r, p += ld) {
        float a[V];
        load_vec_stream<T>(p, a);
#pragma unroll
        for (int i = 0; i < V; ++i)
            m[i] = fmaxf(m[i], fabsf(a[i]));
    }
#pragma unroll
    for (int i = 0; i < V; ++i)
        atomicMax(out_bits + c * V + i, __float_as_uint(m[i]));
}

// ----------------------------------------------------------------------------
// Smoothing factors, in place: on entry s holds B_j (as written by the
// column-absmax kernel); on exit s_j = A_j^alpha / B_j^(1-alpha) evaluated in
// fp64 and rounded once, or 1 where A_j or B_j is 0.  aw (optional) receives B_j.
// ----------------------------------------------------------------------------
__global__ void smooth_factors_kernel(const float *__restrict__ ax, float *s, float *aw, int64_t K,
                                      float alpha)
{
    const int64_t j = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (j >= K)
        return;
    const float a = ax[j];
    const float b = s[j];
    if (aw != nullptr)
        aw[j] = b;
    float r = 1.0f;
    if (a != 0.0f && b != 0.0f) {
        const double al = static_cast<double>(alpha);
        const double num = pow(static_cast<double>(a), al);
        const double den = pow(static_cast<double>(b), 1.0 - al);
        r = __double2float_rn(__ddiv_rn(num, den));
    }
    s[j] = r;
}

// ----------------------------------------------------------------------------
// Block-wide max of non-negative floats (all threads receive the result).
// ----------------------------------------------------------------------------
__device__ __forceinline__ float block_max(float v, float *red /* >= 32 floats */)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        v = fmaxf(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nwarps = (blockDim.x + 31) >> 5;
    __syncthreads();  // red may still be read by a previous call
    if (lane == 0)
        red[warp] = v;
    __syncthreads();
    float r = lane < nwarps ? red[lane] : 0.0f;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        r = fmaxf(r, __shfl_xor_sync(0xFFFFFFFFu, r, o));
    return r;
}

// Store the codes of one 16-byte input vector: 8 codes (bf16 input) as 8
// bytes or 4 codes (fp32 input) as 4 bytes.
template <int V>
__device__ __forceinline__ void store_codes(int8_t *dst, const uint32_t (&q)[V]);

template <>
__device__ __forceinline__ void store_codes<8>(int8_t *dst, const uint32_t (&q)[8])
{
    uint2 u;
    u.x = q[0] | (q[1] << 8) | (q[2] << 16) | (q[3] << 24);
    u.y = q[4] | (q[5] << 8) | (q[6] << 16) | (q[7] << 24);
    *reinterpret_cast<uint2 *>(dst) = u;
}

template <>
__device__ __forceinline__ void store_codes<4>(int8_t *dst, const uint32_t (&q)[4])
{
    *reinterpret_cast<uint32_t *>(dst) = q[0] | (q[1] << 8) | (q[2] << 16) | (q[3] << 24);
}

// ----------------------------------------------------------------------------
// Row quantiser shared by the weight and the activation paths.  One CTA per
// row; each thread keeps CPT 16-byte chunks of the row in registers so the
// row is read from memory once.
//   MODE_W:  v = w * s   (smoothed weight, "multiply the weight input channel")
//   MODE_X:  v = x / s   (smoothed activation, "divide the activation by s")
//   scale = max|v| / 127;  code = clamp(rint(v / scale)).
// ----------------------------------------------------------------------------
enum RowMode { MODE_W = 0, MODE_X = 1 };

template <typename T, int CPT, int MODE>
__global__ void __launch_bounds__(1024) quant_rows_kernel(const T *__restrict__ in, int64_t K,
                                                           const float *__restrict__ s,
                                                           int8_t *__restrict__ q,
                                                           float *__restrict__ scale_out)
{
    constexpr int V = Vec<T>::N;
    __shared__ float red[32];
    const int64_t row = blockIdx.x;
    const int64_t chunks = K / V;
    const T *src = in + row * K;
    float v[CPT][V];
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < CPT; ++i) {
        const int64_t c = threadIdx.x + static_cast<int64_t>(i) * blockDim.x;
        if (c < chunks) {
            float x[V];
            load_vec_stream<T>(src + c * V, x);
            const float4 *sp = reinterpret_cast<const float4 *>(s + c * V);
#pragma unroll
            for (int h = 0; h < V / 4; ++h) {
                const float4 s4 = __ldg(sp + h);
                const float sv[4] = {s4.x, s4.y, s4.z, s4.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float t = (MODE == MODE_W) ? __fmul_rn(x[h * 4 + e], sv[e])
                                                     : __fdiv_rn(x[h * 4 + e], sv[e]);
                    v[i][h * 4 + e] = t;
                    amax = fmaxf(amax, fabsf(t));
                }
            }
        }
    }
    amax = block_max(amax, red);
    const float scale = __fdiv_rn(amax, 127.0f);
    if (threadIdx.x == 0)
        scale_out[row] = scale;
    int8_t *dst = q + row * K;
#pragma unroll
    for (int i = 0; i < CPT; ++i) {
        const int64_t c = threadIdx.x + static_cast<int64_t>(i) * blockDim.x;
        if (c < chunks) {
            uint32_t code[V];
#pragma unroll
            for (int e = 0; e < V; ++e)
                code[e] = (amax != 0.0f) ? quant_code(v[i][e], scale) : 0u;
            store_codes<V>(dst + c * V, code);
        }
    }
}

}  // namespace sq
