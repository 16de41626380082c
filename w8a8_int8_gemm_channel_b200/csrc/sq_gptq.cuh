// sq_gptq.cuh -- GPTQ weight rounding ("Understanding W8A8 INT8 LLM
// Quantization", section "How GPTQ improves on naive quantization"): quantise
// a channel's weights one at a time and push each rounding error onto the
// channel's not yet quantised weights, weighted by the Hessian of the layer's
// output error over the calibration tokens.
//
// Every step is a fixed sequence of IEEE binary64 operations in a fixed index
// order (explicit __fma_rn / __ddiv_rn / __dsqrt_rn, no contraction), so the
// result does not depend on how the work is spread over threads:
//   H[i][j] = sum_t xh[t][i] xh[t][j], t ascending, one FMA a term, with
//             xh = RN_f32(x / s) widened (the smoothed activation);
//   damping d = RN(RN(sum_i H[i][i] / K) * frac), the sum in index order
//             (d = 1 when the sum is 0), added to the diagonal;
//   U       = the upper Cholesky factor of H^-1, through U = J L^-1 J with J
//             the index reversal and L the lower Cholesky factor of J H J:
//             L left-looking, column by column; L^-1 by forward substitution,
//             row by row; every dot product as 32 interleaved partial sums
//             (partial l over k = kb + l, kb + l + 32, ..., ascending, one FMA
//             a term) combined by the xor butterfly o = 16, 8, 4, 2, 1 -- what
//             one warp computes, lane l holding partial l;
//   rows    w = RN_f32(W * s) widened; sw = RN_f32(max |w| / 127); for k in
//             order: q = clamp(rint(w[k] / sw)), e = RN(fma(-q, sw, w[k]) /
//             U[k][k]), w[j] = fma(-e, U[k][j], w[j]) for j > k.
// The Cholesky and the inverse take one launch per column (per row), since
// each depends on all before it; the parallelism is over the rows (columns)
// of that step, one warp per element.  This is offline work, done once per
// layer.
#pragma once

#include <cstdint>

#include <cuda_bf16.h>

#include "sq_mem.cuh"
#include "sq_ptx.cuh"

namespace sq {

constexpr unsigned int kErrGptqPivot = 0xA00;  // H not positive definite (a pivot <= 0)
constexpr int kGptqTile = 16;                  // Hessian tile edge
constexpr int kGptqThreads = 256;

template <typename T>
__device__ __forceinline__ float load_widen(const T *p);
template <>
__device__ __forceinline__ float load_widen<float>(const float *p)
{
    return *p;
}
template <>
__device__ __forceinline__ float load_widen<__nv_bfloat16>(const __nv_bfloat16 *p)
{
    return __uint_as_float(static_cast<uint32_t>(*reinterpret_cast<const uint16_t *>(p)) << 16);
}

// H = xh^T xh over T tokens: one 64 x 64 tile of H per CTA (only tiles on or
// above the diagonal; each also writes its mirror, which holds the same sums
// since a * b = b * a), a 4 x 4 block of it per thread.  Every output's sum
// runs over the tokens in ascending order, 16 tokens a stage; tokens past T
// and columns past K contribute fma(0, b, acc) = acc.
constexpr int kGptqHT = 64;  // Hessian tile edge
template <typename T>
__global__ void __launch_bounds__(256)
    gptq_hessian_kernel(const T *__restrict__ x, int64_t ntok, int64_t K, const float *__restrict__ s,
                        double *__restrict__ H)
{
    pdl_prologue();
    const int bi = blockIdx.y, bj = blockIdx.x;
    if (bi > bj)
        return;
    __shared__ double xa[kGptqTile][kGptqHT];  // [token][column of the i tile]
    __shared__ double xb[kGptqTile][kGptqHT];  // [token][column of the j tile]
    const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
    const int64_t i0 = static_cast<int64_t>(bi) * kGptqHT, j0 = static_cast<int64_t>(bj) * kGptqHT;
    // loads: thread (lt, lc) fetches token lt, columns lc and lc + 16, 32, 48
    const int lt = threadIdx.x / 16, lc = threadIdx.x % 16;
    float si[4], sj[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        si[q] = i0 + lc + 16 * q < K ? s[i0 + lc + 16 * q] : 1.0f;
        sj[q] = j0 + lc + 16 * q < K ? s[j0 + lc + 16 * q] : 1.0f;
    }
    double acc[4][4];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b)
            acc[a][b] = 0.0;
    for (int64_t t0 = 0; t0 < ntok; t0 += kGptqTile) {
        const int64_t t = t0 + lt;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int64_t ci = i0 + lc + 16 * q, cj = j0 + lc + 16 * q;
            xa[lt][lc + 16 * q] =
                (t < ntok && ci < K) ? static_cast<double>(__fdiv_rn(load_widen<T>(x + t * K + ci), si[q])) : 0.0;
            xb[lt][lc + 16 * q] =
                (t < ntok && cj < K) ? static_cast<double>(__fdiv_rn(load_widen<T>(x + t * K + cj), sj[q])) : 0.0;
        }
        __syncthreads();
#pragma unroll
        for (int u = 0; u < kGptqTile; ++u) {
            double av[4], bv[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                av[q] = xa[u][ty + 16 * q];
                bv[q] = xb[u][tx + 16 * q];
            }
#pragma unroll
            for (int a = 0; a < 4; ++a)
#pragma unroll
                for (int b = 0; b < 4; ++b)
                    acc[a][b] = __fma_rn(av[a], bv[b], acc[a][b]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b) {
            const int64_t i = i0 + ty + 16 * a, j = j0 + tx + 16 * b;
            if (i < K && j < K) {
                H[i * K + j] = acc[a][b];
                H[j * K + i] = acc[a][b];
            }
        }
}

// damping, in place (one CTA): the diagonal staged in shared memory, summed
// in index order by one thread
__global__ void __launch_bounds__(kGptqThreads) gptq_damp_kernel(double *__restrict__ H, int64_t K, float frac)
{
    pdl_prologue();
    extern __shared__ double diag[];
    for (int64_t i = threadIdx.x; i < K; i += blockDim.x)
        diag[i] = H[i * K + i];
    __syncthreads();
    __shared__ double d_sh;
    if (threadIdx.x == 0) {
        double sum = 0.0;
        for (int64_t i = 0; i < K; ++i)
            sum = __dadd_rn(sum, diag[i]);
        d_sh = sum == 0.0 ? 1.0 : __dmul_rn(__ddiv_rn(sum, static_cast<double>(K)), static_cast<double>(frac));
    }
    __syncthreads();
    const double d = d_sh;
    for (int64_t i = threadIdx.x; i < K; i += blockDim.x)
        H[i * K + i] = __dadd_rn(diag[i], d);
}

// The fixed-order dot product: lane l sums k = kb + l, kb + l + 32, ... (< ke)
// in ascending order, then the xor butterfly; every lane returns the result.
__device__ __forceinline__ double warp_dot32(const double *__restrict__ a, const double *__restrict__ b, int64_t kb,
                                             int64_t ke, int lane)
{
    double p = 0.0;
    int64_t k = kb + lane;
    for (; k + 96 < ke; k += 128) {  // four loads in flight, the sum in order
        const double a0 = a[k], a1 = a[k + 32], a2 = a[k + 64], a3 = a[k + 96];
        const double b0 = b[k], b1 = b[k + 32], b2 = b[k + 64], b3 = b[k + 96];
        p = __fma_rn(a0, b0, p);
        p = __fma_rn(a1, b1, p);
        p = __fma_rn(a2, b2, p);
        p = __fma_rn(a3, b3, p);
    }
    for (; k < ke; k += 32)
        p = __fma_rn(a[k], b[k], p);
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1)
        p = __dadd_rn(p, __shfl_xor_sync(0xFFFFFFFFu, p, o));
    return p;
}

constexpr int kGptqWarps = 8;  // warps (elements) per CTA in the factor steps

// Column j of L, the lower Cholesky factor of G = J H J (G[a][b] =
// H[K-1-a][K-1-b]), row-major in Lr.  One warp per row i >= j; every warp
// computes the pivot itself (the same operations, so the same bits).
__device__ __forceinline__ void gptq_chol_col(const double *__restrict__ H, int64_t K, int64_t j,
                                              double *__restrict__ Lr, int64_t blk)
{
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t i = j + blk * kGptqWarps + warp;
    if (i >= K)
        return;
    const double *lj = Lr + j * K;
    const double p = __dsub_rn(H[(K - 1 - j) * K + (K - 1 - j)], warp_dot32(lj, lj, 0, j, lane));
    if (!(p > 0.0)) {
        if (lane == 0) {
            record_error(kErrGptqPivot);
            Lr[i * K + j] = __longlong_as_double(0x7FF8000000000000LL);  // NaN from here on
        }
        return;
    }
    const double ljj = __dsqrt_rn(p);
    if (i == j) {
        if (lane == 0)
            Lr[j * K + j] = ljj;
        return;
    }
    const double q = __dsub_rn(H[(K - 1 - i) * K + (K - 1 - j)], warp_dot32(Lr + i * K, lj, 0, j, lane));
    if (lane == 0)
        Lr[i * K + j] = __ddiv_rn(q, ljj);
}

// Row i of N = L^-1, column-major in Nt (Nt[c][k] = N[k][c]).  One warp per
// column c <= i.
__device__ __forceinline__ void gptq_inv_row(const double *__restrict__ Lr, int64_t K, int64_t i,
                                             double *__restrict__ Nt, int64_t blk)
{
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t c = blk * kGptqWarps + warp;
    if (c > i)
        return;
    const double lii = Lr[i * K + i];
    if (c == i) {
        if (lane == 0)
            Nt[i * K + i] = __ddiv_rn(1.0, lii);
        return;
    }
    const double q = warp_dot32(Lr + i * K, Nt + c * K, c, i, lane);
    if (lane == 0)
        Nt[c * K + i] = -__ddiv_rn(q, lii);
}

// Step t of the factorisation, in one launch: column t of L (CTAs
// [0, chol_blocks)) and row t - 1 of L^-1 (the CTAs after them).  Row t - 1 of
// the inverse reads only rows and columns of L up to t - 1, finished by the
// steps before, so the two halves share nothing within the launch.
__global__ void __launch_bounds__(kGptqWarps * 32)
    gptq_factor_step_kernel(const double *__restrict__ H, int64_t K, int64_t t, int64_t chol_blocks,
                            double *__restrict__ Lr, double *__restrict__ Nt)
{
    pdl_prologue();
    const int64_t b = blockIdx.x;
    if (b < chol_blocks)
        gptq_chol_col(H, K, t, Lr, b);
    else
        gptq_inv_row(Lr, K, t - 1, Nt, b - chol_blocks);
}

// U[a][b] = N[K-1-a][K-1-b] = Nt[K-1-b][K-1-a] for b >= a, 0 below the
// diagonal: a transpose through 32 x 32 tiles in shared memory.
__global__ void __launch_bounds__(32 * 8) gptq_u_from_n_kernel(const double *__restrict__ Nt, int64_t K,
                                                               double *__restrict__ U)
{
    pdl_prologue();
    __shared__ double tile[32][33];
    const int64_t a0 = static_cast<int64_t>(blockIdx.y) * 32, b0 = static_cast<int64_t>(blockIdx.x) * 32;
    const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
    // the source block: rows K-1-b (b in [b0, b0+32)), columns K-1-a
    for (int r = ty; r < 32; r += 8) {
        const int64_t b = b0 + r, a = a0 + 31 - tx;  // ascending source addresses across the warp
        tile[r][31 - tx] = (a < K && b < K) ? Nt[(K - 1 - b) * K + (K - 1 - a)] : 0.0;
    }
    __syncthreads();
    for (int r = ty; r < 32; r += 8) {
        const int64_t a = a0 + r, b = b0 + tx;
        if (a < K && b < K)
            U[a * K + b] = b >= a ? tile[tx][r] : 0.0;
    }
}

// GPTQ rounding of the smoothed rows: one warp per row, the row in shared
// memory as fp64.  Every lane computes the code and the error of weight k
// itself (the same operations, so the same bits); lanes then update the
// weights j > k that they own.  STAGE: the CTA copies row k + 1 of U into
// shared memory (cp.async, double-buffered) while its warps apply row k, so
// each row of U crosses from L2 once per CTA instead of once per warp, ahead
// of its use.
template <typename T, bool STAGE>
__global__ void gptq_rows_kernel(const T *__restrict__ w, int64_t N, int64_t K, const float *__restrict__ s,
                                 const double *__restrict__ U, int8_t *__restrict__ wq, float *__restrict__ sw)
{
    pdl_prologue();
    extern __shared__ __align__(16) double rows_sm[];  // [warps][K] rows, then (STAGE) [2][K] rows of U
    const int warps = blockDim.x >> 5;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t n = static_cast<int64_t>(blockIdx.x) * warps + warp;
    const bool active = n < N;  // idle warps still take part in the copies and barriers
    double *r = rows_sm + static_cast<int64_t>(warp) * K;
    double *ubuf = rows_sm + static_cast<int64_t>(warps) * K;
    // U[k][k..K) -> dst[k..K), 16-byte copies from the even index at or below k
    auto stage = [&](int64_t k, double *dst) {
        for (int64_t q2 = (k >> 1) + threadIdx.x; q2 < (K >> 1); q2 += blockDim.x)
            cp_async_16(smem_u32(dst + 2 * q2), U + k * K + 2 * q2, true);
    };
    float amax = 0.0f;
    if (active) {
        for (int64_t k = lane; k < K; k += 32) {
            const float v = __fmul_rn(load_widen<T>(w + n * K + k), s[k]);
            r[k] = static_cast<double>(v);
            amax = fmaxf(amax, fabsf(v));
        }
    }
    amax = warp_max(amax);
    const float scale = __fdiv_rn(amax, 127.0f);
    if (active && lane == 0)
        sw[n] = scale;
    if constexpr (STAGE) {
        stage(0, ubuf);
        cp_async_wait_all();
        __syncthreads();
    } else {
        __syncwarp();
    }
    const double sd = static_cast<double>(scale);
    int8_t *dst = wq + n * K;
    for (int64_t k = 0; k < K; ++k) {
        const double *uk = STAGE ? ubuf + (k & 1) * K : U + k * K;
        if constexpr (STAGE) {
            if (k + 1 < K)  // the next row of U, into the buffer every warp has finished with
                stage(k + 1, ubuf + ((k + 1) & 1) * K);
        }
        if (active) {
            double q = 0.0;
            if (scale != 0.0f) {
                const double rk = r[k];
                q = fmin(fmax(rint(__ddiv_rn(rk, sd)), -127.0), 127.0);
                const double e = __ddiv_rn(__fma_rn(-q, sd, rk), uk[k]);
                for (int64_t j = k + 1 + lane; j < K; j += 32)
                    r[j] = __fma_rn(-e, uk[j], r[j]);
            }
            if (lane == 0)
                dst[k] = static_cast<int8_t>(q);
        }
        if constexpr (STAGE) {
            cp_async_wait_all();
            __syncthreads();
        } else {
            __syncwarp();
        }
    }
}

}  // namespace sq
