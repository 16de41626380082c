// sq_quant_cluster.cuh -- per-row int8 quantisation of a few long rows, each
// row spread over the CTAs of one thread-block cluster.
//
//   MODE_X (activations):  v_k = RN(x_k / s_k)
//   MODE_W (weights):      v_k = RN(x_k * s_k)
//   scale = RN(max_k |v_k| / 127);  code_k = clamp(round_half_even(RN(v_k / scale)), -127, 127)
//
// Sources: "Understanding W8A8 INT8 LLM Quantization", "Why Activation
// Quantization Is Hard, and How SmoothQuant Fixes It" (the smoothing division
// and one dynamic scale per token over all its channels); "quant_llm_int8",
// "The architecture: every piece explained" (symmetric int8 with the scale
// max|v| / 127).
//
// The arithmetic is that of the few-row form of row_quant_kernel
// (sq_rowquant.cuh, no factor table): fp32 bounds of |v| from the hardware
// reciprocal, exact quotients for the chunks whose bound comes near the row's
// largest, the codes on the rounding fast path with the exact fallback near
// ties and for rows with a divisor or scale outside the fast range.
//
// Layout.  With a few rows, one CTA a row leaves most SMs idle, and a long
// row's instructions on one SM are most of its latency.  Here the row's K / V
// 16-byte chunks are cut into C contiguous slices (C = the cluster size: 2, 4
// or 8), one per CTA, held in registers (CH chunks a thread).  Each warp
// resolves its exact-maximum candidates against its own largest bound, so the
// row's exact maximum E is combined once: across the warps of a CTA through
// shared memory, then across the cluster -- every CTA stores its maximum into
// each CTA's shared memory (distributed shared memory) and waits at a cluster
// barrier, whose release / acquire orders those stores.  Every CTA of the
// cluster thus derives the same scale; CTA 0 stores it.
// The grid is rows x C CTAs: one cluster a row.
#pragma once

#include <cstdint>

#include "sq_div.cuh"
#include "sq_mem.cuh"
#include "sq_ptx.cuh"
#include "sq_rowquant.cuh"

namespace sq {

constexpr int kQuantClusterThreads = 256;
constexpr int kQuantClusterMax = 8;

template <typename T, int MODE, int CH>
__global__ void __launch_bounds__(kQuantClusterThreads, 2)
    row_quant_cluster_kernel(const T *__restrict__ in, int64_t rows, int64_t K, const float *__restrict__ s,
                             int8_t *__restrict__ q, float *__restrict__ scale_out, int *__restrict__ zero,
                             int nzero)
{
    pdl_prologue();
    clear_ints(zero, nzero);
    constexpr int V = Vec<T>::N;
    constexpr int THREADS = kQuantClusterThreads;
    constexpr int WARPS = THREADS / 32;
    __shared__ float red[WARPS];
    __shared__ float cmax[kQuantClusterMax];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int C = static_cast<int>(cluster_nctarank());
    const int rank = static_cast<int>(cluster_ctarank());
    // the grid is rows x C CTAs, so every cluster has a row
    const int64_t row = blockIdx.x / C;
    const int nch = static_cast<int>(K / V);
    const int span = (nch + C - 1) / C;
    const int cbeg = rank * span;
    const int cend = min(nch, cbeg + span);
    const int c0 = cbeg + static_cast<int>(threadIdx.x);

    uint4 raw[CH];
    const T *src = in + row * K;
#pragma unroll
    for (int i = 0; i < CH; ++i) {
        const int c = c0 + THREADS * i;
        raw[i] = c < cend ? ld_chunk<T>(src + static_cast<int64_t>(c) * V) : make_uint4(0u, 0u, 0u, 0u);
    }
    // f_k of chunk c (MODE_X: the hardware reciprocal of s_k; MODE_W: s_k);
    // returns whether some s_k of it is outside the range of the fast paths
    auto factor_pairs = [&](int c, float2 (&f2)[V / 2]) -> bool {
        bool bad = false;
#pragma unroll
        for (int h = 0; h < V / 4; ++h) {
            float4 v4 = __ldg(reinterpret_cast<const float4 *>(s + static_cast<int64_t>(c) * V) + h);
            if (MODE == MODE_X) {
                bad |= !div_operand_ok(v4.x) || !div_operand_ok(v4.y) || !div_operand_ok(v4.z) ||
                       !div_operand_ok(v4.w);
                v4 = make_float4(rcp_approx(v4.x), rcp_approx(v4.y), rcp_approx(v4.z), rcp_approx(v4.w));
            }
            f2[2 * h] = make_float2(v4.x, v4.y);
            f2[2 * h + 1] = make_float2(v4.z, v4.w);
        }
        return bad;
    };
    // maximum over the row (called once): the CTA's warps, then the
    // cluster's CTAs
    auto row_max = [&](float v) -> float {
        v = warp_max(v);
        if (lane == 0)
            red[warp] = v;
        __syncthreads();
        float m = red[0];
#pragma unroll
        for (int j = 1; j < WARPS; ++j)
            m = fmaxf(m, red[j]);
        if (static_cast<int>(threadIdx.x) < C)
            st_shared_cluster_f32(map_shared_rank(smem_u32(&cmax[rank]), threadIdx.x), m);
        cluster_arrive();
        cluster_wait();
        float r = cmax[0];
        for (int j = 1; j < C; ++j)
            r = fmaxf(r, cmax[j]);
        return r;
    };

    // 1. bounds of |v| per chunk, the row's largest bound A, the exact maximum E
    float hm[CH];
    float am = 0.0f;
#pragma unroll
    for (int i = 0; i < CH; ++i) {
        const int c = c0 + THREADS * i;
        hm[i] = 0.0f;
        if (c < cend) {
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
            am = fmaxf(am, hm[i]);
        }
    }
    // Each warp takes its own exact candidates, against its own largest
    // bound A: the chunk holding the row's exact maximum has a bound within
    // the candidate window of its warp's largest bound, so one exchange of
    // the warps' exact maxima gives E.  A chunk whose bound is not finite (an
    // s_k outside the fast range, or an overflowing product) is a candidate
    // and has its codes taken exactly.
    const float A = warp_max(am);
    float E = A;  // weights: the fp32 products are the values themselves
    uint32_t unbounded = 0;
#pragma unroll
    for (int i = 0; i < CH; ++i)
        unbounded |= !(hm[i] <= 0x1.fffffep127f) ? (1u << i) : 0u;
    if (MODE == MODE_X) {
        const bool exact_all = !(A >= kTinyQuotient) || !(A <= 0x1.fffffep127f);
        const float thr = __fmul_rn(A, kCandidateScale);
        uint32_t cand = 0;  // chunks that may hold the exact maximum
#pragma unroll
        for (int i = 0; i < CH; ++i) {
            const int c = c0 + THREADS * i;
            cand |= (c < cend && (exact_all || hm[i] >= thr)) ? (1u << i) : 0u;
        }
        float em = 0.0f;
        while (cand != 0u) {  // rare: those chunks exactly, from the registers
            const int i = __ffs(cand) - 1;
            cand &= cand - 1u;
            uint4 v = raw[0];
#pragma unroll
            for (int j = 1; j < CH; ++j)
                if (j == i)
                    v = raw[j];
            const int64_t c = c0 + THREADS * i;
            em = fmaxf(em, chunk_exact_absmax<T, MODE>(v, s + c * V));
        }
        E = row_max(em);
    } else {
        E = row_max(A);
    }

    // 2. scale and codes, from the registers
    const float scale = scale_from_max(E);
    if (rank == 0 && threadIdx.x == 0)
        scale_out[row] = scale;
    const float rsc = rcp_approx(scale);
    const bool fast = scale_in_fast_range(scale);
    const float2 rsc2 = make_float2(rsc, rsc);
    const float2 nrsc2 = make_float2(-rsc, -rsc);
    const float2 magic2 = make_float2(kRoundMagic, kRoundMagic);
    const float2 nmagic2 = make_float2(-kRoundMagic, -kRoundMagic);
    int8_t *dst = q + row * K;
    uint32_t ties = 0;  // chunks whose codes need the exact path
#pragma unroll
    for (int i = 0; i < CH; ++i) {
        const int c = c0 + THREADS * i;
        if (c < cend) {
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
        const int64_t c = c0 + THREADS * i;
        uint4 v = raw[0];
#pragma unroll
        for (int j = 1; j < CH; ++j)
            if (j == i)
                v = raw[j];
        chunk_store_exact_codes<T, MODE>(v, s + c * V, scale, dst + c * V);
    }
}

}  // namespace sq
