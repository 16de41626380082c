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
    if (MODE == MODE_X && single && !bad_divisor) {
        // one load; per-chunk approximate maxima stay in registers, so the
        // exact pass only revisits the chunk(s) near the row maximum
        warp_load_slice<T, SEG>(src, nch, 0, lane, raw);
        float hi[SEG];
        float amax = 0.0f;
#pragma unroll
        for (int i = 0; i < SEG; ++i) {
            const int c = min(lane + 32 * i, nch - 1);
            float x[V], f[V];
            Chunk8 a;
            widen<T>(raw[i], x);
            factor(c, f);
            hi[i] = chunk_approx<V>(x, f, a);
            amax = fmaxf(amax, hi[i]);
        }
        const float A = warp_max(amax);
        const float thr = __fmul_rn(A, kCandidateScale);
        const bool exact_all = A < kTinyQuotient;
        float emax = 0.0f;
#pragma unroll
        for (int i = 0; i < SEG; ++i) {
            if (exact_all || hi[i] >= thr) {
                const int c = min(lane + 32 * i, nch - 1);
                float x[V], f[V];
                // re-read the chunk (L1) so the row need not stay in registers
                const uint4 u = (lane + 32 * i < nch)
                                    ? __ldg(reinterpret_cast<const uint4 *>(src + static_cast<int64_t>(c) * V))
                                    : make_uint4(0u, 0u, 0u, 0u);
                widen<T>(u, x);
                if (!exact_all) {
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
    const float rsc = __frcp_rn(scale);
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
                float dmax = 0.0f;
#pragma unroll
                for (int e = 0; e < V; ++e) {
                    const float t = __fmul_rn(__fmul_rn(x[e], f[e]), rsc);
                    const float yy = __fadd_rn(t, kRoundMagic);
                    dmax = fmaxf(dmax, fabsf(__fsub_rn(t, __fsub_rn(yy, kRoundMagic))));
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

// ----------------------------------------------------------------------------
// Standalone quantiser: one warp per row, persistent over rows.  With SMEM_S
// the per-column factors (MODE_X: RN(1/s); MODE_W: s) are staged in shared
// memory once per CTA.
// ----------------------------------------------------------------------------
template <typename T, int MODE, int SEG, bool SMEM_S>
__global__ void __launch_bounds__(kQuantThreads, 2)
    quant_rows_kernel(const T *__restrict__ in, int64_t rows, int64_t K,
                      const float *__restrict__ s, int8_t *__restrict__ q,
                      float *__restrict__ scale_out)
{
    constexpr int V = Vec<T>::N;
    extern __shared__ float4 smem_f4[];
    float *f_sm = reinterpret_cast<float *>(smem_f4);
    int bad_divisor = 0;
    if constexpr (SMEM_S) {
        for (int64_t j = threadIdx.x; j < K; j += blockDim.x) {
            const float sv = __ldg(s + j);
            if constexpr (MODE == MODE_X) {
                const float rv = div_recip(sv);
                bad_divisor |= (rv == 0.0f);
                f_sm[j] = rv;
            } else {
                f_sm[j] = sv;
            }
        }
        bad_divisor = __syncthreads_or(bad_divisor);
    } else if constexpr (MODE == MODE_X) {
        for (int64_t j = threadIdx.x; j < K; j += blockDim.x)
            bad_divisor |= (div_recip(__ldg(s + j)) == 0.0f);
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
                    v4 = make_float4(div_recip(v4.x), div_recip(v4.y), div_recip(v4.z), div_recip(v4.w));
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
        const T *src = in + row * K;
        uint4 raw[SEG];
        const float E = warp_slice_absmax<T, MODE, SEG>(src, nch, lane, bad_divisor != 0, factor, sptr, raw);
        const float scale = __fdiv_rn(E, 127.0f);
        if (lane == 0)
            scale_out[row] = scale;
        int8_t *dst = q + row * K;
        auto store = [&](int c, uint2 u) {
            if constexpr (V == 8)
                *reinterpret_cast<uint2 *>(dst + static_cast<int64_t>(c) * 8) = u;
            else
                *reinterpret_cast<uint32_t *>(dst + static_cast<int64_t>(c) * 4) = u.x;
        };
        warp_slice_codes<T, MODE, 4>(src, nch, lane, bad_divisor != 0, scale, factor, sptr, store);
    }
}

}  // namespace sq
