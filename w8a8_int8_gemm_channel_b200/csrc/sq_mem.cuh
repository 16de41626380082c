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

#include "sq_div.cuh"
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

template <typename T>
__device__ __forceinline__ uint4 ld_chunk(const T *p)
{
    return __ldcs(reinterpret_cast<const uint4 *>(p));
}

template <typename T>
__device__ __forceinline__ void widen(const uint4 &u, float (&v)[Vec<T>::N]);

// bf16 bits -> fp32: the low half moved up by a byte permute (no shift), the
// high half masked
__device__ __forceinline__ uint32_t bf16_lo_bits(uint32_t u) { return __byte_perm(u, 0u, 0x1044u); }

template <>
__device__ __forceinline__ void widen<__nv_bfloat16>(const uint4 &u, float (&v)[8])
{
    v[0] = __uint_as_float(bf16_lo_bits(u.x));
    v[1] = __uint_as_float(u.x & 0xFFFF0000u);
    v[2] = __uint_as_float(bf16_lo_bits(u.y));
    v[3] = __uint_as_float(u.y & 0xFFFF0000u);
    v[4] = __uint_as_float(bf16_lo_bits(u.z));
    v[5] = __uint_as_float(u.z & 0xFFFF0000u);
    v[6] = __uint_as_float(bf16_lo_bits(u.w));
    v[7] = __uint_as_float(u.w & 0xFFFF0000u);
}

template <>
__device__ __forceinline__ void widen<float>(const uint4 &u, float (&v)[4])
{
    v[0] = __uint_as_float(u.x);
    v[1] = __uint_as_float(u.y);
    v[2] = __uint_as_float(u.z);
    v[3] = __uint_as_float(u.w);
}

// ----------------------------------------------------------------------------
// Column absmax: out[j] = max(out[j], max_r |x[r, j]|), out as fp32 bit
// patterns (non-negative floats order like their unsigned bit patterns).
// Block: 256 threads = 256 consecutive 16-byte column chunks; blockIdx.y
// selects a band of `rows_per_block` rows.  The CTAs of a cluster (consecutive
// bands, kColClusterRows of them) combine their partial maxima through
// distributed shared memory, and the cluster's first CTA issues one atomicMax
// per channel, so the global atomics are 1/kColClusterRows of one per CTA.
// ----------------------------------------------------------------------------
constexpr int kColThreads = 256;
constexpr int kColClusterRows = 8;

__device__ __forceinline__ void cluster_sync_all()
{
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::
                     : "memory");
}

__device__ __forceinline__ float4 ld_shared_cluster_f4(uint32_t addr)
{
    float4 v;
    asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                 : "r"(addr)
                 : "memory");
    return v;
}

template <typename T>
__global__ void __launch_bounds__(kColThreads) col_absmax_kernel(const T *__restrict__ x, int64_t R,
                                                                  int64_t K, int64_t ld,
                                                                  int64_t rows_per_block,
                                                                  unsigned int *__restrict__ out_bits)
{
    pdl_prologue();
    constexpr int V = Vec<T>::N;
    constexpr int SLOTS = kColThreads / kColClusterRows;  // chunk columns each CTA combines
    __shared__ __align__(16) float part[kColThreads * V];
    const int64_t chunks = K / V;
    const int64_t c = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    float m[V];
#pragma unroll
    for (int i = 0; i < V; ++i)
        m[i] = 0.0f;
    if (c < chunks) {
        const int64_t r0 = min(R, static_cast<int64_t>(blockIdx.y) * rows_per_block);
        const int64_t r1 = min(R, r0 + rows_per_block);
        const T *p = x + r0 * ld + c * V;
        int64_t r = r0;
        for (; r + 16 <= r1; r += 16, p += 16 * ld) {
            uint4 raw[16];  // sixteen rows in flight per thread
#pragma unroll
            for (int u = 0; u < 16; ++u)
                raw[u] = __ldcs(reinterpret_cast<const uint4 *>(p + u * ld));
#pragma unroll
            for (int u = 0; u < 16; ++u) {
                float a[V];
                widen<T>(raw[u], a);
#pragma unroll
                for (int i = 0; i < V; ++i)
                    m[i] = fmaxf(m[i], fabsf(a[i]));
            }
        }
        for (; r + 8 <= r1; r += 8, p += 8 * ld) {
            uint4 raw[8];  // eight rows in flight per thread
#pragma unroll
            for (int u = 0; u < 8; ++u)
                raw[u] = __ldcs(reinterpret_cast<const uint4 *>(p + u * ld));
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                float a[V];
                widen<T>(raw[u], a);
#pragma unroll
                for (int i = 0; i < V; ++i)
                    m[i] = fmaxf(m[i], fabsf(a[i]));
            }
        }
        for (; r < r1; ++r, p += ld) {
            float a[V];
            load_vec_stream<T>(p, a);
#pragma unroll
            for (int i = 0; i < V; ++i)
                m[i] = fmaxf(m[i], fabsf(a[i]));
        }
    }
#pragma unroll
    for (int i = 0; i < V; i += 4)
        *reinterpret_cast<float4 *>(part + threadIdx.x * V + i) = make_float4(m[i], m[i + 1], m[i + 2], m[i + 3]);
    __syncwarp();
    cluster_sync_all();  // every CTA's partial maxima are visible cluster-wide
    // CTA `rank` combines chunk slots [rank*SLOTS, rank*SLOTS + SLOTS) across the cluster
    if (threadIdx.x < SLOTS) {
        const int slot = static_cast<int>(cluster_ctarank()) * SLOTS + threadIdx.x;
        const int64_t cc = static_cast<int64_t>(blockIdx.x) * blockDim.x + slot;
        if (cc < chunks) {
            const uint32_t local = smem_u32(part + slot * V);
            float t[kColClusterRows][V];
#pragma unroll
            for (int rk = 0; rk < kColClusterRows; ++rk) {
                const uint32_t remote = map_shared_rank(local, rk);
#pragma unroll
                for (int i = 0; i < V; i += 4) {
                    const float4 q = ld_shared_cluster_f4(remote + 4u * i);
                    t[rk][i] = q.x;
                    t[rk][i + 1] = q.y;
                    t[rk][i + 2] = q.z;
                    t[rk][i + 3] = q.w;
                }
            }
            float mm[V];
#pragma unroll
            for (int i = 0; i < V; ++i) {
                mm[i] = t[0][i];
#pragma unroll
                for (int rk = 1; rk < kColClusterRows; ++rk)
                    mm[i] = fmaxf(mm[i], t[rk][i]);
                atomicMax(out_bits + cc * V + i, __float_as_uint(mm[i]));
            }
        }
    }
    __syncwarp();
    cluster_sync_all();  // no CTA leaves while its shared memory may still be read
}

// ----------------------------------------------------------------------------
// Self-test of the bounded waits: one thread waits on an mbarrier that nothing
// arrives on, with a short limit; the wait gives up, records its location
// code in the device error word and the kernel returns normally.
// ----------------------------------------------------------------------------
__global__ void wait_selftest_kernel(unsigned long long limit_ns)
{
    pdl_prologue();
    __shared__ __align__(8) unsigned long long bar;
    if (threadIdx.x == 0) {
        const uint32_t b = smem_u32(&bar);
        mbar_init(b, 1);
        fence_barrier_init();
        bounded_wait(b, 0, kErrWaitSelfTest, nullptr, limit_ns);  // phase 0 never completes
    }
    __syncthreads();
}

// ----------------------------------------------------------------------------
// RMSNorm gamma with the smoothing folded in: g_j = gamma_j / s_j (one IEEE
// fp32 division per channel).
// ----------------------------------------------------------------------------
__global__ void fold_gamma_kernel(const float *__restrict__ gamma, const float *__restrict__ s,
                                  float *__restrict__ g, int64_t K)
{
    pdl_prologue();
    const int64_t j = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (j < K)
        g[j] = __fdiv_rn(gamma[j], s[j]);
}

// Zero n floats: the accumulator of a column maximum, as a kernel so that it
// takes part in the launch overlap of the stream (a memset does not).
__global__ void zero_f32_kernel(float *__restrict__ p, int64_t n)
{
    pdl_prologue();
    const int64_t j = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (j < n)
        p[j] = 0.0f;
}

// ----------------------------------------------------------------------------
// Smoothing factors, in place: on entry s holds B_j (as written by the
// column-absmax kernel); on exit s_j = A_j^alpha / B_j^(1-alpha) evaluated in
// fp64 and rounded once, or 1 where A_j or B_j is 0.  aw (optional) receives B_j.
// ----------------------------------------------------------------------------
__global__ void smooth_factors_kernel(const float *__restrict__ ax, float *s, float *aw, int64_t K,
                                      float alpha)
{
    pdl_prologue();
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
// Row quantiser shared by the weight and the activation paths: one warp per
// row, persistent over rows.
//   MODE_W:  v = w * s   (smoothed weight: the weight input channel times s)
//   MODE_X:  v = x / s   (smoothed activation: the activation divided by s)
//   scale = max_k |v| / 127;  code = clamp(round_half_even(v / scale), -127, 127)
// Each lane reads 16-byte chunks c = lane + 32 i of the row, SEG chunks at a
// time (a short, fixed instruction footprint).  The row is read twice: the
// second (code) pass hits L1/L2, so HBM sees it once.  With SMEM_S the factors
// s (and for MODE_X their reciprocals) are staged in shared memory once per CTA.
// ----------------------------------------------------------------------------
enum RowMode { MODE_W = 0, MODE_X = 1 };

__device__ __forceinline__ float warp_max(float v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        v = fmaxf(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
    return v;
}

constexpr int kQuantThreads = 256;

// Chunks of up to 8 values passed by value to the out-of-line slow paths.
struct Chunk8 {
    float v[8];
};

// Exact maximum of |x / s| over the elements of one chunk whose approximate
// magnitude a = RN(|x| * RN(1/s)) reaches `thr` (rare: the row's top element).
__device__ __noinline__ float chunk_max_exact(Chunk8 x, Chunk8 a, const float *__restrict__ s_chunk,
                                              int n, float thr)
{
    float em = 0.0f;
    for (int e = 0; e < n; ++e)
        if (a.v[e] >= thr)
            em = fmaxf(em, fabsf(__fdiv_rn(x.v[e], __ldg(s_chunk + e))));
    return em;
}

// Exact codes of one chunk (rare: near ties, scales outside the fast range).
// MODE_W: v = x * s; MODE_X: v = x / s.
__device__ __noinline__ Chunk8 chunk_codes_exact(Chunk8 x, const float *__restrict__ s_chunk, int n,
                                                 int mode_x, float scale)
{
    Chunk8 y;
    for (int e = 0; e < n; ++e) {
        const float sv = __ldg(s_chunk + e);
        const float v = mode_x ? __fdiv_rn(x.v[e], sv) : __fmul_rn(x.v[e], sv);
        y.v[e] = __uint_as_float(scale != 0.0f ? exact_code_bits(v, scale) : code_bits(0.0f));
    }
    return y;
}

// Exact max of |x / s| over one chunk (rows whose divisors leave the fast range).
__device__ __noinline__ float chunk_absmax_div(Chunk8 x, const float *__restrict__ s_chunk, int n)
{
    float m = 0.0f;
    for (int e = 0; e < n; ++e)
        m = fmaxf(m, fabsf(__fdiv_rn(x.v[e], __ldg(s_chunk + e))));
    return m;
}

// Approximate magnitudes a = RN(|x| * r) of one chunk and their maximum.
template <int V>
__device__ __forceinline__ float chunk_approx(const float (&x)[V], const float (&r)[V], Chunk8 &a)
{
    float hi = 0.0f;
#pragma unroll
    for (int e = 0; e < V; ++e) {
        a.v[e] = fabsf(__fmul_rn(x[e], r[e]));
        hi = fmaxf(hi, a.v[e]);
    }
    return hi;
}

// Exact-maximum contribution of one chunk given the row's candidate threshold.
template <int V>
__device__ __forceinline__ float chunk_candidates(const float (&x)[V], const float (&r)[V],
                                                  const float *__restrict__ s_chunk, float thr)
{
    Chunk8 a, xv;
    const float hi = chunk_approx<V>(x, r, a);
    if (hi < thr)
        return 0.0f;
#pragma unroll
    for (int e = 0; e < V; ++e)
        xv.v[e] = x[e];
    return chunk_max_exact(xv, a, s_chunk, V, thr);
}

}  // namespace sq
