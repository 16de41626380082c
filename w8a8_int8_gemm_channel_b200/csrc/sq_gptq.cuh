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
//             L left-looking, column by column, each dot product in ascending
//             k; L^-1 by forward substitution, row by row, each dot product in
//             ascending k;
//   rows    w = RN_f32(W * s) widened; sw = RN_f32(max |w| / 127); for k in
//             order: q = clamp(rint(w[k] / sw)), e = RN(fma(-q, sw, w[k]) /
//             U[k][k]), w[j] = fma(-e, U[k][j], w[j]) for j > k.
// The Cholesky and the inverse take one launch per column (per row), since
// each depends on all before it; the parallelism is over the rows (columns)
// of that step.  This is offline work, done once per layer.
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

// H = xh^T xh over T tokens, one 16 x 16 tile of H per CTA (only tiles on or
// above the diagonal; each also writes its mirror, which holds the same
// sums since a * b = b * a).  Tokens past T contribute fma(0, 0, acc) = acc.
template <typename T>
__global__ void __launch_bounds__(kGptqTile *kGptqTile)
    gptq_hessian_kernel(const T *__restrict__ x, int64_t ntok, int64_t K, const float *__restrict__ s,
                        double *__restrict__ H)
{
    pdl_prologue();
    const int bi = blockIdx.y, bj = blockIdx.x;
    if (bi > bj)
        return;
    __shared__ double xa[kGptqTile][kGptqTile + 1];  // [token][column of the i tile]
    __shared__ double xb[kGptqTile][kGptqTile + 1];  // [token][column of the j tile]
    const int tx = threadIdx.x % kGptqTile, ty = threadIdx.x / kGptqTile;
    const int64_t i0 = static_cast<int64_t>(bi) * kGptqTile, j0 = static_cast<int64_t>(bj) * kGptqTile;
    const float si = s[i0 + tx], sj = s[j0 + tx];
    double acc = 0.0;
    for (int64_t t0 = 0; t0 < ntok; t0 += kGptqTile) {
        const int64_t t = t0 + ty;
        xa[ty][tx] = t < ntok ? static_cast<double>(__fdiv_rn(load_widen<T>(x + t * K + i0 + tx), si)) : 0.0;
        xb[ty][tx] = t < ntok ? static_cast<double>(__fdiv_rn(load_widen<T>(x + t * K + j0 + tx), sj)) : 0.0;
        __syncthreads();
#pragma unroll
        for (int u = 0; u < kGptqTile; ++u)
            acc = __fma_rn(xa[u][ty], xb[u][tx], acc);
        __syncthreads();
    }
    H[(i0 + ty) * K + j0 + tx] = acc;
    H[(j0 + tx) * K + i0 + ty] = acc;
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

// zero a K x K fp64 matrix (U's lower triangle stays zero)
__global__ void gptq_zero_kernel(double *__restrict__ p, int64_t n)
{
    pdl_prologue();
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x)
        p[i] = 0.0;
}

// Column j of L, the lower Cholesky factor of G = J H J (G[a][b] =
// H[K-1-a][K-1-b]).  L is stored transposed, Lt[k][i] = L[i][k], so that the
// rows i of one step read consecutive addresses.  Every CTA stages row j of L
// and computes the pivot itself (the same operations, so the same bits).
__global__ void __launch_bounds__(kGptqThreads)
    gptq_chol_col_kernel(const double *__restrict__ H, int64_t K, int64_t j, double *__restrict__ Lt)
{
    pdl_prologue();
    extern __shared__ double lj[];  // L[j][0..j-1]
    __shared__ double piv;
    for (int64_t k = threadIdx.x; k < j; k += blockDim.x)
        lj[k] = Lt[k * K + j];
    __syncthreads();
    if (threadIdx.x == 0) {
        double p = H[(K - 1 - j) * K + (K - 1 - j)];
        for (int64_t k = 0; k < j; ++k)
            p = __fma_rn(-lj[k], lj[k], p);
        if (!(p > 0.0)) {
            record_error(kErrGptqPivot);
            piv = __longlong_as_double(0x7FF8000000000000LL);  // NaN from here on
        } else {
            piv = __dsqrt_rn(p);
        }
    }
    __syncthreads();
    const double ljj = piv;
    const int64_t i = j + static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (i >= K)
        return;
    if (i == j) {
        Lt[j * K + j] = ljj;
        return;
    }
    double q = H[(K - 1 - i) * K + (K - 1 - j)];
    for (int64_t k = 0; k < j; ++k)
        q = __fma_rn(-Lt[k * K + i], lj[k], q);
    Lt[j * K + i] = __ddiv_rn(q, ljj);
}

// Row i of N = L^-1, written straight into U at the reversed positions:
// N[i][c] -> U[K-1-i][K-1-c].  Thread c sums L[i][k] N[k][c] over k = c..i-1
// in ascending k; all threads walk k together (a thread joins at k = c), so
// that each step reads one row of N at consecutive addresses.
__global__ void __launch_bounds__(kGptqThreads)
    gptq_inv_row_kernel(const double *__restrict__ Lt, int64_t K, int64_t i, double *__restrict__ U)
{
    pdl_prologue();
    const int64_t c = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    const double lii = Lt[i * K + i];
    if (c > i)
        return;
    if (c == i) {
        U[(K - 1 - i) * K + (K - 1 - i)] = __ddiv_rn(1.0, lii);
        return;
    }
    // the CTA's first column: its threads join from there
    const int64_t k0 = static_cast<int64_t>(blockIdx.x) * blockDim.x;
    double q = 0.0;
    for (int64_t k = k0; k < i; ++k) {
        const double lik = Lt[k * K + i];
        const double nkc = U[(K - 1 - k) * K + (K - 1 - c)];
        if (k >= c)
            q = __fma_rn(lik, nkc, q);
    }
    U[(K - 1 - i) * K + (K - 1 - c)] = -__ddiv_rn(q, lii);
}

// GPTQ rounding of the smoothed rows: one warp per row, the row in shared
// memory as fp64.  Every lane computes the code and the error of weight k
// itself (the same operations, so the same bits); lanes then update the
// weights j > k that they own.
template <typename T>
__global__ void gptq_rows_kernel(const T *__restrict__ w, int64_t N, int64_t K, const float *__restrict__ s,
                                 const double *__restrict__ U, int8_t *__restrict__ wq, float *__restrict__ sw)
{
    pdl_prologue();
    extern __shared__ double rows_sm[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t n = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + warp;
    if (n >= N)
        return;
    double *r = rows_sm + static_cast<int64_t>(warp) * K;
    float amax = 0.0f;
    for (int64_t k = lane; k < K; k += 32) {
        const float v = __fmul_rn(load_widen<T>(w + n * K + k), s[k]);
        r[k] = static_cast<double>(v);
        amax = fmaxf(amax, fabsf(v));
    }
    amax = warp_max(amax);
    const float scale = __fdiv_rn(amax, 127.0f);
    if (lane == 0)
        sw[n] = scale;
    __syncwarp();
    const double sd = static_cast<double>(scale);
    int8_t *dst = wq + n * K;
    for (int64_t k = 0; k < K; ++k) {
        double q = 0.0;
        if (scale != 0.0f) {
            const double rk = r[k];
            q = fmin(fmax(rint(__ddiv_rn(rk, sd)), -127.0), 127.0);
            const double e = __ddiv_rn(__fma_rn(-q, sd, rk), U[k * K + k]);
            const double *uk = U + k * K;
            for (int64_t j = k + 1 + lane; j < K; j += 32)
                r[j] = __fma_rn(-e, uk[j], r[j]);
        }
        if (lane == 0)
            dst[k] = static_cast<int8_t>(q);
        __syncwarp();
    }
}

}  // namespace sq
