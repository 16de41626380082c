// sq_rowquant.cuh -- warp-cooperative quantisation of one row slice, shared
// by the standalone quantisers and the GEMM kernel's fused prologue.
//
//   MODE_X (activations):  v_k = RN(x_k / s_k)       (smoothed activation)
//   MODE_W (weights):      v_k = RN(x_k * s_k)       (smoothed weight)
//   scale = RN(max_k |v_k| / 127);  code_k = clamp(round_half_even(RN(v_k / scale)), -127, 127)
//
// Lane L of the warp handles the 16-byte chunks c = L + 32 i of the slice.  A
// slice of at most 32*SEG chunks is loaded once and kept in registers for all
// passes; longer slices are streamed in segments and re-read (from L1/L2).
// The arithmetic is the one described in sq_div.cuh: the exact maximum comes
// from an approximate maximum plus exact quotients for its candidates, the
// codes from the rounding fast path with an exact fallback near ties.
#pragma once

#include <cstdint>

#include "sq_div.cuh"
#include "sq_glu.cuh"
#include "sq_mem.cuh"

namespace sq {

template <typename T, int SEG>
__device__ __forceinline__ void warp_load_slice(const T *__restrict__ src, int nch, int base, int lane,
                                                uint4 (&raw)[SEG])
{
    constexpr int V = Vec<T>::N;
#pragma unroll
    for (int i = 0; i < SEG; ++i) {
        const int c = base + lane + 32 * i;
        raw[i] = c < nch ? __ldg(reinterpret_cast<const uint4 *>(src + static_cast<int64_t>(c) * V))
                         : make_uint4(0u, 0u, 0u, 0u);
    }
}

// Exact max_k |v_k| over the slice (the same value in every lane).
//   factor(c, f): MODE_X -> f = RN(1/s) of chunk c (0 never occurs unless
//                 bad_divisor); MODE_W -> f = s of chunk c.
//   sptr(c):      pointer to the s values of chunk c (for the exact paths).
// `raw` is scratch for SEG chunks per lane.
template <typename T, int MODE, int SEG, typename FactorFn, typename SPtrFn>
__device__ __forceinline__ float warp_slice_absmax(const T *__restrict__ src, int nch, int lane,
                                                   bool bad_divisor, FactorFn factor, SPtrFn sptr,
                                                   uint4 (&raw)[SEG])
{
    constexpr int V = Vec<T>::N;
    const bool single = nch <= 32 * SEG;
    constexpr int HI = 16;  // chunks per lane covered by the kept maxima (slices up to 32*HI chunks)
    if (MODE == MODE_X && nch <= 32 * HI && !bad_divisor) {
        // the slice is read once; approximate maxima of chunk pairs stay in
        // registers and the exact pass only revisits the pairs near the row maximum
        float hi[HI / 2];
        float amax = 0.0f;
#pragma unroll
        for (int g = 0; g < HI / SEG; ++g) {
            warp_load_slice<T, SEG>(src, nch, g * 32 * SEG, lane, raw);
#pragma unroll
            for (int i = 0; i < SEG; ++i) {
                const int j = g * SEG + i;
                const int c = min(g * 32 * SEG + lane + 32 * i, nch - 1);
                float x[V], f[V];
                Chunk8 a;
                widen<T>(raw[i], x);
                factor(c, f);
                const float h = chunk_approx<V>(x, f, a);
                hi[j / 2] = (j & 1) ? fmaxf(hi[j / 2], h) : h;
                amax = fmaxf(amax, h);
            }
        }
        const float A = warp_max(amax);
        const float thr = __fmul_rn(A, kCandidateScale);
        const bool exact_all = A < kTinyQuotient;
        float emax = 0.0f;
#pragma unroll
        for (int j = 0; j < HI; ++j) {
            const int cj = (j / SEG) * 32 * SEG + lane + 32 * (j % SEG);
            if ((exact_all || hi[j / 2] >= thr) && cj < nch) {
                float x[V], f[V];
                // re-read the chunk (L1) so the row need not stay in registers
                widen<T>(__ldg(reinterpret_cast<const uint4 *>(src + static_cast<int64_t>(cj) * V)), x);
                if (!exact_all) {
                    factor(cj, f);
                    emax = fmaxf(emax, chunk_candidates<V>(x, f, sptr(cj), thr));
                } else {
                    Chunk8 xv;
#pragma unroll
                    for (int e = 0; e < V; ++e)
                        xv.v[e] = x[e];
                    emax = fmaxf(emax, chunk_absmax_div(xv, sptr(cj), V));
                }
            }
        }
        return warp_max(emax);
    }
    float thr = 0.0f;
    bool exact_all = bad_divisor;
    if (MODE == MODE_X && !bad_divisor) {
        float amax = 0.0f;
#pragma unroll 1
        for (int base = 0; base < nch; base += 32 * SEG) {
            warp_load_slice<T, SEG>(src, nch, base, lane, raw);
#pragma unroll
            for (int i = 0; i < SEG; ++i) {
                const int c = min(base + lane + 32 * i, nch - 1);
                float x[V], f[V];
                Chunk8 a;
                widen<T>(raw[i], x);
                factor(c, f);
                amax = fmaxf(amax, chunk_approx<V>(x, f, a));
            }
        }
        const float A = warp_max(amax);
        thr = __fmul_rn(A, kCandidateScale);
        exact_all = A < kTinyQuotient;
    }
    float emax = 0.0f;
#pragma unroll 1
    for (int base = 0; base < nch; base += 32 * SEG) {
        if (!(single && MODE == MODE_X && !bad_divisor))
            warp_load_slice<T, SEG>(src, nch, base, lane, raw);
#pragma unroll
        for (int i = 0; i < SEG; ++i) {
            const int c = min(base + lane + 32 * i, nch - 1);
            float x[V], f[V];
            widen<T>(raw[i], x);
            if constexpr (MODE == MODE_W) {
                factor(c, f);
#pragma unroll
                for (int e = 0; e < V; ++e)
                    emax = fmaxf(emax, fabsf(__fmul_rn(x[e], f[e])));
            } else if (!exact_all) {
                factor(c, f);
                emax = fmaxf(emax, chunk_candidates<V>(x, f, sptr(c), thr));
            } else {
                Chunk8 xv;
#pragma unroll
                for (int e = 0; e < V; ++e)
                    xv.v[e] = x[e];
                emax = fmaxf(emax, chunk_absmax_div(xv, sptr(c), V));
            }
        }
    }
    return warp_max(emax);
}

// Codes of the slice for a given scale; store(c, packed) receives the V codes
// of chunk c packed little-endian into a uint2 (bf16 input) or uint32 (fp32).
// The slice is read again (from L1/L2), SEG chunks per lane at a time.
template <typename T, int MODE, int SEG, typename FactorFn, typename SPtrFn, typename StoreFn>
__device__ __forceinline__ void warp_slice_codes(const T *__restrict__ src, int nch, int lane,
                                                 bool bad_divisor, float scale, FactorFn factor,
                                                 SPtrFn sptr, StoreFn store)
{
    uint4 raw[SEG];
    constexpr int V = Vec<T>::N;
    const float rsc = rcp_approx(scale);
    const bool fast = scale_in_fast_range(scale) && !bad_divisor;
#pragma unroll 1
    for (int base = 0; base < nch; base += 32 * SEG) {
        warp_load_slice<T, SEG>(src, nch, base, lane, raw);
#pragma unroll
        for (int i = 0; i < SEG; ++i) {
            const int c = base + lane + 32 * i;
            const int cc = min(c, nch - 1);
            float x[V], f[V];
            uint32_t y[V];
            widen<T>(raw[i], x);
            bool tie = !fast;
            if (fast) {
                factor(cc, f);
                // y = RN(a * rsc + 1.5*2^23) rounds the product a*rsc half-even to an
                // integer in one step (the code is y's low byte); d = a*rsc - that
                // integer decides whether the fast result is safe (|d| < 0.5 - 2^-13)
                float dmax = 0.0f;
#pragma unroll
                for (int e = 0; e < V; ++e) {
                    const float a = __fmul_rn(x[e], f[e]);
                    const float yy = __fmaf_rn(a, rsc, kRoundMagic);
                    const float r = __fsub_rn(yy, kRoundMagic);
                    dmax = fmaxf(dmax, fabsf(__fmaf_rn(a, rsc, -r)));
                    y[e] = __float_as_uint(yy);
                }
                tie = !(dmax < kTieLimit);  // NaN (scale too small) also takes the exact path
            }
            if (tie) {
                Chunk8 xv;
#pragma unroll
                for (int e = 0; e < V; ++e)
                    xv.v[e] = x[e];
                const Chunk8 yy = chunk_codes_exact(xv, sptr(cc), V, MODE == MODE_X, scale);
#pragma unroll
                for (int e = 0; e < V; ++e)
                    y[e] = __float_as_uint(yy.v[e]);
            }
            if (c < nch) {
                if constexpr (V == 8)
                    store(c, make_uint2(pack_code_bytes(y[0], y[1], y[2], y[3]),
                                        pack_code_bytes(y[4], y[5], y[6], y[7])));
                else
                    store(c, make_uint2(pack_code_bytes(y[0], y[1], y[2], y[3]), 0u));
            }
        }
    }
}

// Stage n factors from s into dst (RN(1/s) when RECIP, else s itself; nothing
// stored unless STORE), threads t, t+nt, ... of a group, four float4 loads in
// flight per thread per round.  Returns non-zero when some reciprocal is
// unusable by the fast division (its divisor lies outside [2^-60, 2^61)).
template <bool RECIP, bool STORE>
__device__ __forceinline__ int stage_factors(const float *__restrict__ s, int n, float *dst, int t, int nt)
{
    int bad = 0;
    const int nv = n >> 2;  // n is a multiple of 16
    const float4 *s4 = reinterpret_cast<const float4 *>(s);
    for (int j0 = t; j0 < nv; j0 += 4 * nt) {
        float4 v[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int j = j0 + u * nt;
            v[u] = j < nv ? __ldg(s4 + j) : make_float4(1.f, 1.f, 1.f, 1.f);
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int j = j0 + u * nt;
            if (j < nv) {
                float4 r = v[u];
                if (RECIP) {
                    r = make_float4(fast_recip(v[u].x), fast_recip(v[u].y), fast_recip(v[u].z), fast_recip(v[u].w));
                    bad |= (r.x == 0.0f) | (r.y == 0.0f) | (r.z == 0.0f) | (r.w == 0.0f);
                }
                if (STORE)
                    reinterpret_cast<float4 *>(dst)[j] = r;
            }
        }
    }
    return bad;
}

// ----------------------------------------------------------------------------
// Standalone quantiser, two kernels:
//   row_scale_kernel  one warp per row (persistent): the exact row maximum and
//                     scale = RN(max/127), read-only, no CTA barriers;
//   row_codes_kernel  elementwise given the row scales: each thread owns one
//                     16-byte column chunk (its factors live in registers) and
//                     walks a band of rows with several rows in flight.
// The codes kernel re-reads the rows; for activations (and weights) that fit
// the 126 MB L2 that second read is served from L2.
// ----------------------------------------------------------------------------
template <typename T, int MODE, int SEG, bool SMEM_S>
__global__ void __launch_bounds__(kQuantThreads, 2)
    row_scale_kernel(const T *__restrict__ in, int64_t rows, int64_t K, const float *__restrict__ s,
                     float *__restrict__ scale_out)
{
    pdl_prologue();
    constexpr int V = Vec<T>::N;
    extern __shared__ float4 smem_f4[];
    float *f_sm = reinterpret_cast<float *>(smem_f4);
    int bad_divisor = 0;
    if constexpr (SMEM_S || MODE == MODE_X) {
        bad_divisor = stage_factors<MODE == MODE_X, SMEM_S>(s, static_cast<int>(K), f_sm, threadIdx.x,
                                                            blockDim.x);
        bad_divisor = __syncthreads_or(bad_divisor);
    }
    const int lane = threadIdx.x & 31;
    const int warps = blockDim.x >> 5;
    const int nch = static_cast<int>(K / V);
    auto factor = [&](int c, float (&f)[V]) {
#pragma unroll
        for (int h = 0; h < V / 4; ++h) {
            float4 v4;
            if constexpr (SMEM_S) {
                v4 = reinterpret_cast<const float4 *>(f_sm + static_cast<int64_t>(c) * V)[h];
            } else {
                v4 = __ldg(reinterpret_cast<const float4 *>(s + static_cast<int64_t>(c) * V) + h);
                if constexpr (MODE == MODE_X)
                    v4 = make_float4(fast_recip(v4.x), fast_recip(v4.y), fast_recip(v4.z), fast_recip(v4.w));
            }
            f[4 * h] = v4.x;
            f[4 * h + 1] = v4.y;
            f[4 * h + 2] = v4.z;
            f[4 * h + 3] = v4.w;
        }
    };
    auto sptr = [&](int c) { return s + static_cast<int64_t>(c) * V; };
    for (int64_t row = static_cast<int64_t>(blockIdx.x) * warps + (threadIdx.x >> 5); row < rows;
         row += static_cast<int64_t>(gridDim.x) * warps) {
        uint4 raw[SEG];
        const float E = warp_slice_absmax<T, MODE, SEG>(in + row * K, nch, lane, bad_divisor != 0, factor,
                                                        sptr, raw);
        if (lane == 0)
            scale_out[row] = scale_from_max(E);
    }
}

// Side task of the activation quantisers inside sq_linear: clear n ints (the
// tile counters of the GEMM that follows), spread over the grid.
__device__ __forceinline__ void clear_ints(int *p, int n)
{
    if (p == nullptr)
        return;
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x)
        p[i] = 0;
}

template <typename T, int MODE>
__global__ void __launch_bounds__(256) row_codes_kernel(const T *__restrict__ in, int64_t rows, int64_t K,
                                                        const float *__restrict__ s,
                                                        const float *__restrict__ scale,
                                                        int64_t rows_per_block, int8_t *__restrict__ q,
                                                        int *__restrict__ zero, int nzero)
{
    pdl_prologue();
    clear_ints(zero, nzero);
    constexpr int V = Vec<T>::N;
    constexpr int U = 4;  // rows in flight per thread
    const int64_t nch = K / V;
    const int64_t c = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (c >= nch)
        return;
    // this thread's factors: MODE_X -> 1/s (1 ulp), MODE_W -> s
    float f[V];
    bool bad = false;
#pragma unroll
    for (int h = 0; h < V; h += 4) {
        const float4 v4 = __ldg(reinterpret_cast<const float4 *>(s + c * V + h));
        const float sv[4] = {v4.x, v4.y, v4.z, v4.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            f[h + e] = (MODE == MODE_X) ? fast_recip(sv[e]) : sv[e];
            bad |= (MODE == MODE_X) && f[h + e] == 0.0f;
        }
    }
    const int64_t r0 = static_cast<int64_t>(blockIdx.y) * rows_per_block;
    const int64_t r1 = min(rows, r0 + rows_per_block);
    for (int64_t r = r0; r < r1; r += U) {
        uint4 raw[U];
        float sc[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const bool ok = r + u < r1;
            raw[u] = ok ? __ldg(reinterpret_cast<const uint4 *>(in + (r + u) * K + c * V)) : make_uint4(0u, 0u, 0u, 0u);
            sc[u] = ok ? __ldg(scale + r + u) : 1.0f;
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const bool live = r + u < r1;
            float x[V];
            widen<T>(raw[u], x);
            const float rsc = rcp_approx(sc[u]);
            bool tie = bad || !scale_in_fast_range(sc[u]);
            uint32_t y[V];
            float dmax = 0.0f;
#pragma unroll
            for (int e = 0; e < V; ++e) {
                const float a = __fmul_rn(x[e], f[e]);
                const float yy = __fmaf_rn(a, rsc, kRoundMagic);
                const float rr = __fsub_rn(yy, kRoundMagic);
                dmax = fmaxf(dmax, fabsf(__fmaf_rn(a, rsc, -rr)));
                y[e] = __float_as_uint(yy);
            }
            tie |= !(dmax < kTieLimit);
            if (tie && live) {
                Chunk8 xv;
#pragma unroll
                for (int e = 0; e < V; ++e)
                    xv.v[e] = x[e];
                const Chunk8 yy = chunk_codes_exact(xv, s + c * V, V, MODE == MODE_X, sc[u]);
#pragma unroll
                for (int e = 0; e < V; ++e)
                    y[e] = __float_as_uint(yy.v[e]);
            }
            if (live) {
                int8_t *dst = q + (r + u) * K + c * V;
                if constexpr (V == 8)
                    *reinterpret_cast<uint2 *>(dst) = make_uint2(pack_code_bytes(y[0], y[1], y[2], y[3]),
                                                                 pack_code_bytes(y[4], y[5], y[6], y[7]));
                else
                    *reinterpret_cast<uint32_t *>(dst) = pack_code_bytes(y[0], y[1], y[2], y[3]);
            }
        }
    }
}

// ----------------------------------------------------------------------------
// Single-pass quantiser: each row is read from HBM once and stays in
// registers from the maximum to the codes.  G = 2^log2g warps share one row
// (a CTA of 8 warps holds 8/G rows at a time); lane L of warp g holds the
// 16-byte chunks c = 32 g + L + 32 G i, i < CH, so each step i of the G warps
// covers 32 G consecutive chunks.  Persistent over rows.
//
// Maximum.  bf16 rows: a bound p_k = RN_bf16(|x_k| * RN_bf16(|f_k|)) in
// packed bf16 arithmetic, with f_k = RN(1/s_k) to 1 ulp (activations) or s_k
// (weights), lies within a factor 1 +- 0.0079 of |v_k| (two bf16 roundings of
// relative size 2^-8 each, plus the reciprocal's and v's fp32 roundings).  So
// the element attaining the exact maximum E has p_k >= A (1 - 2^-5), A the
// largest bound, and only the chunks reaching that threshold are recomputed
// exactly (IEEE x/s or x*s).  fp32 rows: fp32 bounds a_k = RN(|x_k| f_k)
// within 2^-21 and the threshold A (1 - 2^-20); weights need none (a_k is
// v_k).  Rows whose bound leaves [2^-100, FLT_MAX], or whose divisors leave
// the fast range, are recomputed exactly throughout.
// Codes.  The rounding fast path of sq_div.cuh, in packed fp32 pairs.
// ----------------------------------------------------------------------------
__device__ __forceinline__ void named_barrier_sync(int id, int threads)
{
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

// Factor tables in shared memory: f[K] fp32 (RN(1/s) when RECIP, else s)
// and, with BF, fb[K] = RN_bf16(|f|) as bf16 pairs.  Returns non-zero when
// some reciprocal is unusable by the fast paths.
template <bool RECIP, bool BF>
__device__ __forceinline__ int stage_factor_tables(const float *__restrict__ s, int n, float *f, uint32_t *fb,
                                                   int t, int nt)
{
    int bad = 0;
    const int nv = n >> 2;  // n is a multiple of 16
    const float4 *s4 = reinterpret_cast<const float4 *>(s);
    for (int j0 = t; j0 < nv; j0 += 4 * nt) {
        float4 v[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int j = j0 + u * nt;
            v[u] = j < nv ? __ldg(s4 + j) : make_float4(1.f, 1.f, 1.f, 1.f);
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int j = j0 + u * nt;
            if (j < nv) {
                float4 r = v[u];
                if (RECIP) {
                    r = make_float4(fast_recip(v[u].x), fast_recip(v[u].y), fast_recip(v[u].z), fast_recip(v[u].w));
                    bad |= (r.x == 0.0f) | (r.y == 0.0f) | (r.z == 0.0f) | (r.w == 0.0f);
                }
                reinterpret_cast<float4 *>(f)[j] = r;
                if (BF) {
                    const __nv_bfloat162 lo = __floats2bfloat162_rn(fabsf(r.x), fabsf(r.y));
                    const __nv_bfloat162 hi = __floats2bfloat162_rn(fabsf(r.z), fabsf(r.w));
                    reinterpret_cast<uint2 *>(fb)[j] =
                        make_uint2(*reinterpret_cast<const uint32_t *>(&lo), *reinterpret_cast<const uint32_t *>(&hi));
                }
            }
        }
    }
    return bad;
}

// Rare paths of the single-pass quantisers, kept out of the unrolled chunk
// loops (which only record a bit per chunk); they compute one 16-byte chunk
// exactly.
//   exact maximum of |v| over the chunk (v = x / s or x * s), given its raw bits
template <typename T, int MODE>
__device__ __noinline__ float chunk_exact_absmax(uint4 raw, const float *__restrict__ sc)
{
    constexpr int V = Vec<T>::N;
    float x[V];
    widen<T>(raw, x);
    float m = 0.0f;
    for (int e = 0; e < V; ++e) {
        const float sv = __ldg(sc + e);
        m = fmaxf(m, fabsf(MODE == MODE_X ? __fdiv_rn(x[e], sv) : __fmul_rn(x[e], sv)));
    }
    return m;
}

__device__ __forceinline__ void store_code_words(int8_t *dst, const uint32_t *y, int n)
{
    if (n == 8)
        *reinterpret_cast<uint2 *>(dst) =
            make_uint2(pack_code_bytes(y[0], y[1], y[2], y[3]), pack_code_bytes(y[4], y[5], y[6], y[7]));
    else
        *reinterpret_cast<uint32_t *>(dst) = pack_code_bytes(y[0], y[1], y[2], y[3]);
}

//   exact codes of the chunk from its raw bits (the caller takes them from the
//   registers or re-reads them from L2), overwriting what the fast path stored
template <typename T, int MODE>
__device__ __noinline__ void chunk_store_exact_codes(uint4 raw, const float *__restrict__ sc, float scale, int8_t *dst)
{
    constexpr int V = Vec<T>::N;
    float x[V];
    widen<T>(raw, x);
    uint32_t y[8];
    for (int e = 0; e < V; ++e) {
        const float sv = __ldg(sc + e);
        const float v = MODE == MODE_X ? __fdiv_rn(x[e], sv) : __fmul_rn(x[e], sv);
        y[e] = scale != 0.0f ? exact_code_bits(v, scale) : code_bits(0.0f);
    }
    store_code_words(dst, y, V);
}

//   exact codes of a chunk of the normalised, smoothed row a = (h * rinv) * g
template <typename T>
__device__ __noinline__ void chunk_store_exact_codes_norm(const T *__restrict__ p, const float *g, float rinv,
                                                          float scale, int8_t *dst)
{
    constexpr int V = Vec<T>::N;
    float x[V];
    widen<T>(__ldg(reinterpret_cast<const uint4 *>(p)), x);
    uint32_t y[8];
    for (int e = 0; e < V; ++e) {
        const float a = __fmul_rn(__fmul_rn(x[e], rinv), g[e]);
        y[e] = scale != 0.0f ? exact_code_bits(a, scale) : code_bits(0.0f);
    }
    store_code_words(dst, y, V);
}

// bytes of shared memory the factor tables of a K-column row take (bf: with
// the bf16 table)
__host__ __device__ constexpr int64_t row_quant_smem(int64_t K, bool bf) { return K * 4 + (bf ? K * 2 : 0); }

// FIT: the G warps of a row cover its chunks exactly (32 CH G = K / V), so
// no chunk needs a bounds check.  BB (bf16 rows only): bound |v| in packed
// bf16 arithmetic (fewer instructions, a wider candidate window and a second
// factor table in shared memory) instead of fp32.  GLU: each input row is
// [gate | up] (2K values) and the row quantised is h = SiLU(gate) * up
// (sq_glu.cuh), written to hout as well when hout is not null.
template <typename T, int MODE, int CH, bool FIT, bool BB, bool GLU = false, bool TAB = true,
          int THREADS = kQuantThreads>
__global__ void __launch_bounds__(THREADS, (THREADS >= 1024 ? 1
                                            : THREADS > kQuantThreads ? 2
                                            : GLU ? (CH <= 8 ? 2 : 1)
                                                  : (CH <= 8 ? 3 : 2)))
    row_quant_kernel(const T *__restrict__ in, int64_t rows, int64_t K, const float *__restrict__ s,
                     int log2g, int8_t *__restrict__ q, float *__restrict__ scale_out, T *__restrict__ hout,
                     int *__restrict__ zero, int nzero)
{
    static_assert(TAB || !BB, "the bf16 bound needs its table");
    constexpr bool tab = TAB;
    // TAB = false (few rows, fp32 bound only): no factor table; each lane reads
    // its chunks' s_k from global memory and takes the hardware reciprocal
    // itself; a chunk with an s_k outside the fast range bounds its elements
    // by +inf, which makes it an exact candidate and sends its codes to the
    // exact path
    pdl_prologue();
    clear_ints(zero, nzero);
    constexpr int V = Vec<T>::N;
    constexpr bool BF = BB && (V == 8);  // the bf16 bound
    constexpr int WARPS = THREADS / 32;
    extern __shared__ float4 smem_f4[];
    float *f_sm = reinterpret_cast<float *>(smem_f4);
    uint32_t *fb_sm = reinterpret_cast<uint32_t *>(f_sm + K);
    __shared__ float red[2][WARPS];
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int G = 1 << log2g;
    const int slot = warp >> log2g;
    const int g = warp & (G - 1);
    const int slots = WARPS >> log2g;
    const int nch = static_cast<int>(K / V);
    const int c0 = 32 * g + lane;
    const int cstep = 32 * G;
    int64_t row = static_cast<int64_t>(blockIdx.x) * slots + slot;
    const int64_t rstride = static_cast<int64_t>(gridDim.x) * slots;

    const int64_t ld = GLU ? 2 * K : K;  // input row stride
    uint4 raw[CH];
    uint4 uraw[GLU ? CH : 1];  // GLU: the up half of the row
    auto load_row = [&](int64_t r) {
        const T *src = in + r * ld;
#pragma unroll
        for (int i = 0; i < CH; ++i) {
            const int c = c0 + cstep * i;
            raw[i] = (FIT || c < nch) ? ld_chunk<T>(src + static_cast<int64_t>(c) * V) : make_uint4(0u, 0u, 0u, 0u);
        }
        if constexpr (GLU) {
#pragma unroll
            for (int i = 0; i < CH; ++i) {
                const int c = c0 + cstep * i;
                uraw[i] = (FIT || c < nch) ? ld_chunk<T>(src + K + static_cast<int64_t>(c) * V)
                                           : make_uint4(0u, 0u, 0u, 0u);
            }
        }
    };
    if (row < rows)
        load_row(row);
    // factor tables staged while the first row's loads are in flight
    const bool bad_divisor =
        tab ? __syncthreads_or(stage_factor_tables<MODE == MODE_X, BF>(s, static_cast<int>(K), f_sm, fb_sm,
                                                                       threadIdx.x, blockDim.x)) != 0
            : false;
    // f_k of chunk c; without the table, whether some s_k of it is outside
    // the range of the fast paths
    auto factor_pairs = [&](int c, float2 (&f2)[V / 2]) -> bool {
        bool bad = false;
#pragma unroll
        for (int h = 0; h < V / 4; ++h) {
            float4 v4;
            if (tab) {
                v4 = reinterpret_cast<const float4 *>(f_sm + static_cast<int64_t>(c) * V)[h];
            } else {
                v4 = __ldg(reinterpret_cast<const float4 *>(s + static_cast<int64_t>(c) * V) + h);
                if (MODE == MODE_X) {
                    bad |= !div_operand_ok(v4.x) || !div_operand_ok(v4.y) || !div_operand_ok(v4.z) ||
                           !div_operand_ok(v4.w);
                    v4 = make_float4(rcp_approx(v4.x), rcp_approx(v4.y), rcp_approx(v4.z), rcp_approx(v4.w));
                }
            }
            f2[2 * h] = make_float2(v4.x, v4.y);
            f2[2 * h + 1] = make_float2(v4.z, v4.w);
        }
        return bad;
    };
    // maximum over the G warps of this row; alternating buffers, so a buffer
    // is rewritten only after every warp of the group has passed the barrier
    // that follows its last read
    int nred = 0;
    auto group_max = [&](float v) -> float {
        v = warp_max(v);
        if (G == 1)
            return v;
        float *r = red[nred & 1];
        ++nred;
        if (lane == 0)
            r[warp] = v;
        named_barrier_sync(1 + slot, 32 * G);
        float m = r[slot << log2g];
        for (int j = 1; j < G; ++j)
            m = fmaxf(m, r[(slot << log2g) + j]);
        return m;
    };

    while (row < rows) {
        if constexpr (GLU) {
            // 0. h = SiLU(gate) * up into raw[]: the fast path for bf16 rows,
            // the definition for fp32 rows and for the elements the fast path
            // cannot decide (their chunks keep the gate in raw[] until a loop
            // outside the unrolled one fixes them from the registers)
            uint32_t redo = 0;
#pragma unroll
            for (int i = 0; i < CH; ++i) {
                const int c = c0 + cstep * i;
                if (FIT || c < nch) {
                    if constexpr (V == 8) {
                        bool r;
                        const uint4 hv = glu_chunk_fast(raw[i], uraw[i], r);
                        raw[i] = r ? raw[i] : hv;
                        redo |= r ? (1u << i) : 0u;
                    } else {
                        raw[i] = glu_chunk_exact<T>(raw[i], uraw[i]);
                    }
                }
            }
            if constexpr (V == 8) {
                while (redo != 0u) {
                    const int i = __ffs(redo) - 1;
                    redo &= redo - 1u;
                    uint4 gq = raw[0], uq = uraw[0];
#pragma unroll
                    for (int j = 1; j < CH; ++j)
                        if (j == i) {
                            gq = raw[j];
                            uq = uraw[j];
                        }
                    const uint4 hv = glu_chunk_fix(gq, uq);
#pragma unroll
                    for (int j = 0; j < CH; ++j)
                        if (j == i)
                            raw[j] = hv;
                }
            }
            if (hout != nullptr) {
#pragma unroll
                for (int i = 0; i < CH; ++i) {
                    const int c = c0 + cstep * i;
                    if (FIT || c < nch)
                        *reinterpret_cast<uint4 *>(hout + row * K + static_cast<int64_t>(c) * V) = raw[i];
                }
            }
        }
        // 1. bounds of |v| per chunk, the row's largest bound A, the exact maximum E
        float hm[CH];
        float am = 0.0f;
#pragma unroll
        for (int i = 0; i < CH; ++i) {
            const int c = c0 + cstep * i;
            hm[i] = 0.0f;
            if (FIT || c < nch) {
                if constexpr (BF) {
                    const uint4 fb = *reinterpret_cast<const uint4 *>(fb_sm + static_cast<int64_t>(c) * 4);
                    uint32_t p = bf2_mul(raw[i].x & 0x7FFF7FFFu, fb.x);
                    p = bf2_max(p, bf2_mul(raw[i].y & 0x7FFF7FFFu, fb.y));
                    p = bf2_max(p, bf2_mul(raw[i].z & 0x7FFF7FFFu, fb.z));
                    p = bf2_max(p, bf2_mul(raw[i].w & 0x7FFF7FFFu, fb.w));
                    hm[i] = bf2_hmax_f32(p);
                } else {
                    float x[V];
                    float2 f2[V / 2];
                    widen<T>(raw[i], x);
                    const bool bad = factor_pairs(c, f2);
                    float h = 0.0f;
#pragma unroll
                    for (int e = 0; e < V; e += 2) {
                        const float2 a = f2_mul(make_float2(x[e], x[e + 1]), f2[e / 2]);
                        h = fmaxf(h, fmaxf(fabsf(a.x), fabsf(a.y)));
                    }
                    hm[i] = bad ? __int_as_float(0x7f800000) : h;
                }
                am = fmaxf(am, hm[i]);
            }
        }
        // Each warp takes its own exact-maximum candidates against its own
        // largest bound A, so one exchange of the warps' exact maxima gives E:
        // the chunk holding the row's exact maximum has a bound within the
        // candidate window of its warp's largest bound, as of the row's.  A
        // chunk whose bound is not finite (without the table, an s_k outside
        // the fast range; or an overflowing product) is a candidate and has
        // its codes taken exactly.
        const float A = warp_max(am);
        float E = A;  // fp32-bounded weights: the bounds are the values themselves
        uint32_t unbounded = 0;
#pragma unroll
        for (int i = 0; i < CH; ++i)
            unbounded |= !(hm[i] <= 0x1.fffffep127f) ? (1u << i) : 0u;
        if (BF || MODE == MODE_X) {
            const bool exact_all = bad_divisor || !(A >= kTinyQuotient) || !(A <= 0x1.fffffep127f);
            const float thr = __fmul_rn(A, BF ? 0.96875f : kCandidateScale);
            uint32_t cand = 0;  // chunks that may hold the exact maximum
#pragma unroll
            for (int i = 0; i < CH; ++i) {
                const int c = c0 + cstep * i;
                cand |= ((FIT || c < nch) && (exact_all || hm[i] >= thr)) ? (1u << i) : 0u;
            }
            float em = 0.0f;
            while (cand != 0u) {  // rare: those chunks exactly, taken from the registers
                const int i = __ffs(cand) - 1;
                cand &= cand - 1u;
                uint4 v = raw[0];
#pragma unroll
                for (int j = 1; j < CH; ++j)
                    if (j == i)
                        v = raw[j];
                const int64_t c = c0 + cstep * i;
                em = fmaxf(em, chunk_exact_absmax<T, MODE>(v, s + c * V));
            }
            E = group_max(em);
        } else {
            E = group_max(A);
        }

        // 2. scale and codes, from the registers
        const float scale = scale_from_max(E);
        if (g == 0 && lane == 0)
            scale_out[row] = scale;
        const float rsc = rcp_approx(scale);
        const bool fast = scale_in_fast_range(scale) && !bad_divisor;
        const float2 rsc2 = make_float2(rsc, rsc);
        const float2 nrsc2 = make_float2(-rsc, -rsc);
        const float2 magic2 = make_float2(kRoundMagic, kRoundMagic);
        const float2 nmagic2 = make_float2(-kRoundMagic, -kRoundMagic);
        int8_t *dst = q + row * K;
        uint32_t ties = 0;  // chunks whose codes need the exact path
#pragma unroll
        for (int i = 0; i < CH; ++i) {
            const int c = c0 + cstep * i;
            if (FIT || c < nch) {
                float x[V];
                uint32_t y[V];
                float2 f2[V / 2];
                widen<T>(raw[i], x);
                factor_pairs(c, f2);
                float dmax = 0.0f;
#pragma unroll
                for (int e = 0; e < V; e += 2) {
                    // yy = RN(a * rsc + 1.5*2^23): a*rsc rounded half-even to an
                    // integer r (the code is yy's low byte); dd = r - a*rsc
                    const float2 a = f2_mul(make_float2(x[e], x[e + 1]), f2[e / 2]);
                    const float2 yy = f2_fma(a, rsc2, magic2);
                    const float2 rr = f2_add(yy, nmagic2);
                    const float2 dd = f2_fma(a, nrsc2, rr);
                    dmax = fmaxf(dmax, fmaxf(fabsf(dd.x), fabsf(dd.y)));
                    y[e] = __float_as_uint(yy.x);
                    y[e + 1] = __float_as_uint(yy.y);
                }
                // NaN (scale too small) and scales outside the fast range also go exact
                ties |= (!fast || !(dmax < kTieLimit)) ? (1u << i) : 0u;
                store_code_words(dst + static_cast<int64_t>(c) * V, y, V);
            }
        }
        ties |= unbounded;
        while (ties != 0u) {  // rare: near ties; every chunk when the scale is outside the fast range
            const int i = __ffs(ties) - 1;
            ties &= ties - 1u;
            const int64_t c = c0 + cstep * i;
            uint4 v;
            if (GLU || !tab) {  // h exists only in the registers; few rows: latency counts, registers do not
                v = raw[0];
#pragma unroll
                for (int j = 1; j < CH; ++j)
                    if (j == i)
                        v = raw[j];
            } else {  // re-read from L2: keeps raw[] dead after the code loop
                v = __ldg(reinterpret_cast<const uint4 *>(in + row * K + c * V));
            }
            chunk_store_exact_codes<T, MODE>(v, s + c * V, scale, dst + c * V);
        }
        row += rstride;
        if (row < rows)
            load_row(row);
    }
}

// ----------------------------------------------------------------------------
// RMSNorm with gamma / s folded in, then per-token int8 quantisation: one
// read of each token's hidden vector h, written as codes and a scale.
//   ms   = sum_k h_k^2 / K + eps   (squares exact in fp64, fp64 sums)
//   rinv = RN_f32(1 / sqrt(ms))    (IEEE fp64 sqrt and division; 0 if ms = 0)
//   a_k  = RN(RN(h_k * rinv) * g_k)
//   scale = RN(max |a| / 127),  code = clamp(rne(RN(a / scale)), -127, 127)
// a is computed exactly, so its maximum needs no candidate pass; the codes use
// the rounding fast path of sq_div.cuh with the exact fallback near ties.
// Same row layout as row_quant_kernel: G = 2^log2g warps per row, the row in
// registers, g staged in shared memory.
// ----------------------------------------------------------------------------
template <typename T, int CH>
__global__ void __launch_bounds__(kQuantThreads, (CH <= 8 ? 3 : 2))
    rmsnorm_quant_kernel(const T *__restrict__ in, int64_t rows, int64_t K, const float *__restrict__ gam,
                         float eps, int log2g, int8_t *__restrict__ q, float *__restrict__ scale_out,
                         float *__restrict__ rinv_out)
{
    pdl_prologue();
    constexpr int V = Vec<T>::N;
    constexpr int WARPS = kQuantThreads / 32;
    extern __shared__ float4 smem_f4[];
    float *g_sm = reinterpret_cast<float *>(smem_f4);
    __shared__ float red[2][WARPS];
    __shared__ double redd[2][WARPS];
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int G = 1 << log2g;
    const int slot = warp >> log2g;
    const int g = warp & (G - 1);
    const int slots = WARPS >> log2g;
    const int nch = static_cast<int>(K / V);
    const int c0 = 32 * g + lane;
    const int cstep = 32 * G;
    int64_t row = static_cast<int64_t>(blockIdx.x) * slots + slot;
    const int64_t rstride = static_cast<int64_t>(gridDim.x) * slots;

    uint4 raw[CH];
    auto load_row = [&](int64_t r) {
        const T *src = in + r * K;
#pragma unroll
        for (int i = 0; i < CH; ++i) {
            const int c = c0 + cstep * i;
            raw[i] = c < nch ? ld_chunk<T>(src + static_cast<int64_t>(c) * V) : make_uint4(0u, 0u, 0u, 0u);
        }
    };
    if (row < rows)
        load_row(row);
    {
        const float4 *g4 = reinterpret_cast<const float4 *>(gam);
        for (int j = threadIdx.x; j < static_cast<int>(K / 4); j += blockDim.x)
            reinterpret_cast<float4 *>(g_sm)[j] = __ldg(g4 + j);
    }
    __syncthreads();
    auto gvals = [&](int c, float (&f)[V]) {
#pragma unroll
        for (int h = 0; h < V / 4; ++h) {
            const float4 v4 = reinterpret_cast<const float4 *>(g_sm + static_cast<int64_t>(c) * V)[h];
            f[4 * h] = v4.x;
            f[4 * h + 1] = v4.y;
            f[4 * h + 2] = v4.z;
            f[4 * h + 3] = v4.w;
        }
    };
    // reductions over the G warps of this row (alternating buffers, as in row_quant_kernel)
    int nred = 0;
    auto group_max = [&](float v) -> float {
        v = warp_max(v);
        if (G == 1)
            return v;
        float *r = red[nred & 1];
        ++nred;
        if (lane == 0)
            r[warp] = v;
        named_barrier_sync(1 + slot, 32 * G);
        float m = r[slot << log2g];
        for (int j = 1; j < G; ++j)
            m = fmaxf(m, r[(slot << log2g) + j]);
        return m;
    };
    int nredd = 0;
    auto group_sum = [&](double v) -> double {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1)
            v = __dadd_rn(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
        if (G == 1)
            return v;
        double *r = redd[nredd & 1];
        ++nredd;
        if (lane == 0)
            r[warp] = v;
        named_barrier_sync(1 + slot, 32 * G);
        double t = r[slot << log2g];
        for (int j = 1; j < G; ++j)
            t = __dadd_rn(t, r[(slot << log2g) + j]);
        return t;
    };

    while (row < rows) {
        // 1. 1/RMS of the token
        double ss = 0.0;
#pragma unroll
        for (int i = 0; i < CH; ++i) {
            if (c0 + cstep * i < nch) {
                float x[V];
                widen<T>(raw[i], x);
#pragma unroll
                for (int e = 0; e < V; ++e) {
                    const double v = static_cast<double>(x[e]);
                    ss = __fma_rn(v, v, ss);  // v*v is exact in fp64
                }
            }
        }
        ss = group_sum(ss);
        const double ms = __dadd_rn(__ddiv_rn(ss, static_cast<double>(K)), static_cast<double>(eps));
        const float rinv = ms > 0.0 ? __double2float_rn(__ddiv_rn(1.0, __dsqrt_rn(ms))) : 0.0f;
        if (g == 0 && lane == 0 && rinv_out != nullptr)
            rinv_out[row] = rinv;

        // 2. the smoothed activations a and their exact maximum
        float am = 0.0f;
#pragma unroll
        for (int i = 0; i < CH; ++i) {
            const int c = c0 + cstep * i;
            if (c < nch) {
                float x[V], f[V];
                widen<T>(raw[i], x);
                gvals(c, f);
#pragma unroll
                for (int e = 0; e < V; ++e)
                    am = fmaxf(am, fabsf(__fmul_rn(__fmul_rn(x[e], rinv), f[e])));
            }
        }
        const float E = group_max(am);

        // 3. scale and codes
        const float scale = scale_from_max(E);
        if (g == 0 && lane == 0)
            scale_out[row] = scale;
        const float rsc = rcp_approx(scale);
        const bool fast = scale_in_fast_range(scale);
        int8_t *dst = q + row * K;
        uint32_t ties = 0;  // chunks whose codes need the exact path
#pragma unroll
        for (int i = 0; i < CH; ++i) {
            const int c = c0 + cstep * i;
            if (c < nch) {
                float x[V], f[V];
                uint32_t y[V];
                widen<T>(raw[i], x);
                gvals(c, f);
                float dmax = 0.0f;
#pragma unroll
                for (int e = 0; e < V; ++e) {
                    const float a = __fmul_rn(__fmul_rn(x[e], rinv), f[e]);
                    const float yy = __fmaf_rn(a, rsc, kRoundMagic);
                    const float rr = __fsub_rn(yy, kRoundMagic);
                    dmax = fmaxf(dmax, fabsf(__fmaf_rn(a, -rsc, rr)));
                    y[e] = __float_as_uint(yy);
                }
                ties |= (!fast || !(dmax < kTieLimit)) ? (1u << i) : 0u;
                store_code_words(dst + static_cast<int64_t>(c) * V, y, V);
            }
        }
        while (ties != 0u) {  // rare: near ties; every chunk when the scale is outside the fast range
            const int i = __ffs(ties) - 1;
            ties &= ties - 1u;
            const int64_t c = c0 + cstep * i;
            chunk_store_exact_codes_norm<T>(in + row * K + c * V, g_sm + c * V, rinv, scale, dst + c * V);
        }
        row += rstride;
        if (row < rows)
            load_row(row);
    }
}

}  // namespace sq
