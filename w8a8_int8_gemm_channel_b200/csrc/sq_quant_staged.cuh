// sq_quant_staged.cuh -- the per-token (and per-output-channel) int8
// quantiser for bf16 rows, with every row brought into shared memory by a
// bulk copy ahead of its use.
//
//   MODE_X (activations):  v_k = RN(x_k / s_k)       (smoothed activation)
//   MODE_W (weights):      v_k = RN(x_k * s_k)       (smoothed weight)
//   scale = RN(max_k |v_k| / 127);  code_k = clamp(round_half_even(RN(v_k / scale)), -127, 127)
//
// Sources: "Understanding W8A8 INT8 LLM Quantization", "Why Activation
// Quantization Is Hard, and How SmoothQuant Fixes It" (one dynamic scale per
// token, max |x| / 127) and "Why Naive Weight Quantization Doesn't Work..."
// (one scale per output channel); the smoothing division and multiplication
// of "Where the outlier actually comes from".
//
// The arithmetic is that of sq_div.cuh and of row_quant_kernel: a packed
// bf16 bound of |v| per chunk, exact quotients for the chunks within 2^-5 of
// the row's largest bound (bf16 bound) or 2^-20 (fp32 bound), the scale by
// Markstein's iteration, and the codes from the rounding fast path with the
// exact IEEE path near ties.  What differs is how the rows move:
//   * a CTA of 8 warps holds 8 / G groups of G warps; each group owns
//     `nslots` row buffers in shared memory, and its leader thread keeps them
//     filled with the group's next rows by 1-D bulk copies (cp.async.bulk,
//     completion on an mbarrier), so nslots rows per group are in flight
//     however long the arithmetic of the current one takes;
//   * lane L of warp g of a group takes the 16-byte chunks c = 32 g + L +
//     32 G i, i < CH, of the row: one shared-memory load each, kept in
//     registers for every pass.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

#include "sq_div.cuh"
#include "sq_mem.cuh"
#include "sq_ptx.cuh"
#include "sq_rowquant.cuh"

namespace sq {

// 1-D bulk copy global -> shared, completion (bytes) on an mbarrier; both
// addresses 16-byte aligned, size a multiple of 16.
__device__ __forceinline__ void bulk_load(uint32_t dst, const void *src, uint32_t bytes, uint32_t bar)
{
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
                 "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
                 : "memory");
}

// shared memory of the staged quantiser: factor tables, then the row slots
// (128-byte aligned), then one mbarrier per slot
__host__ __device__ constexpr int64_t staged_tables_bytes(int64_t K, bool bf) { return K * 4 + (bf ? K * 2 : 0); }

__host__ __device__ constexpr int64_t staged_slots_offset(int64_t K, bool bf)
{
    return (staged_tables_bytes(K, bf) + 127) / 128 * 128;
}

__host__ __device__ constexpr int64_t staged_smem_bytes(int64_t K, bool bf, int groups, int nslots)
{
    return staged_slots_offset(K, bf) + static_cast<int64_t>(groups) * nslots * K * 2 +
           static_cast<int64_t>(groups) * nslots * 8;
}

// Rare paths, element by element.  A chunk is flagged as a whole by the
// cheap passes, but usually only one of its 8 elements needs the exact
// quotient; the chunk is re-read from the row buffer in shared memory.
//   candidates: the exact |v| of the elements whose own bound reaches thr
//   (all of them when exact_all), maximum over those.  The element that
//   attains the row maximum has a bound >= thr, as the chunk test assumes.
template <int MODE, bool BF>
__device__ __noinline__ float staged_candidates(uint32_t saddr, const uint32_t *fb, const float *f,
                                                const float *__restrict__ sc, float thr, bool exact_all)
{
    uint4 r;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "r"(saddr));
    const uint32_t w[4] = {r.x, r.y, r.z, r.w};
    float m = 0.0f;
#pragma unroll
    for (int h = 0; h < 4; ++h) {
        float b[2];
        if constexpr (BF) {
            const uint32_t p = bf2_mul(w[h] & 0x7FFF7FFFu, fb[h]);
            b[0] = __uint_as_float(p << 16);
            b[1] = __uint_as_float(p & 0xFFFF0000u);
        } else {
            b[0] = fabsf(__fmul_rn(__uint_as_float(w[h] << 16), f[2 * h]));
            b[1] = fabsf(__fmul_rn(__uint_as_float(w[h] & 0xFFFF0000u), f[2 * h + 1]));
        }
#pragma unroll
        for (int k = 0; k < 2; ++k) {
            if (exact_all || b[k] >= thr) {
                const float x = __uint_as_float(k == 0 ? (w[h] << 16) : (w[h] & 0xFFFF0000u));
                const float sv = __ldg(sc + 2 * h + k);
                m = fmaxf(m, fabsf(MODE == MODE_X ? __fdiv_rn(x, sv) : __fmul_rn(x, sv)));
            }
        }
    }
    return m;
}

//   ties: the elements whose fast code lies within 2^-13 of a rounding tie
//   (every element when !fast) get the exact code, one byte store each; the
//   fast path has already stored the chunk's other codes.
template <int MODE>
__device__ __noinline__ void staged_ties(uint32_t saddr, const float *f, const float *__restrict__ sc, float scale,
                                         float rsc, bool fast, int8_t *dst)
{
    uint4 r;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "r"(saddr));
    const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        const float x = __uint_as_float((e & 1) ? (w[e >> 1] & 0xFFFF0000u) : (w[e >> 1] << 16));
        const float a = __fmul_rn(x, f[e]);
        const float yy = __fmaf_rn(a, rsc, kRoundMagic);
        const float dd = __fmaf_rn(a, -rsc, __fadd_rn(yy, -kRoundMagic));
        if (!fast || !(fabsf(dd) < kTieLimit)) {
            const float sv = __ldg(sc + e);
            const float v = MODE == MODE_X ? __fdiv_rn(x, sv) : __fmul_rn(x, sv);
            const uint32_t cb = scale != 0.0f ? exact_code_bits(v, scale) : code_bits(0.0f);
            dst[e] = static_cast<int8_t>(cb & 0xFFu);
        }
    }
}

template <int MODE, int CH, bool BF>
__global__ void __launch_bounds__(kQuantThreads, CH >= 14 ? 1 : 2)
    row_quant_staged_kernel(const __nv_bfloat16 *__restrict__ in, int64_t rows, int64_t K,
                            const float *__restrict__ s, int log2g, int nslots, int8_t *__restrict__ q,
                            float *__restrict__ scale_out, int *__restrict__ zero, int nzero)
{
    pdl_prologue();
    clear_ints(zero, nzero);
    constexpr int V = 8;
    constexpr int WARPS = kQuantThreads / 32;
    extern __shared__ __align__(128) uint8_t qs_smem[];
    float *f_sm = reinterpret_cast<float *>(qs_smem);
    uint32_t *fb_sm = reinterpret_cast<uint32_t *>(f_sm + K);
    __shared__ float red[2][WARPS];
    __shared__ int abort_sm;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int G = 1 << log2g;
    const int group = warp >> log2g;
    const int g = warp & (G - 1);
    const int groups = WARPS >> log2g;
    const int c0 = 32 * g + lane;
    const int cstep = 32 * G;
    const uint32_t row_bytes = static_cast<uint32_t>(K * 2);
    const uint32_t slots = smem_u32(qs_smem) + static_cast<uint32_t>(staged_slots_offset(K, BF));
    const uint32_t bars = slots + static_cast<uint32_t>(groups * nslots) * row_bytes;
    auto slot_addr = [&](int j) { return slots + static_cast<uint32_t>(group * nslots + j) * row_bytes; };
    auto slot_bar = [&](int j) { return bars + 8u * static_cast<uint32_t>(group * nslots + j); };
    const bool leader = g == 0 && lane == 0;
    const int64_t row0 = static_cast<int64_t>(blockIdx.x) * groups + group;
    const int64_t rstride = static_cast<int64_t>(gridDim.x) * groups;

    if (threadIdx.x == 0) {
        for (int j = 0; j < groups * nslots; ++j)
            mbar_init(bars + 8u * j, 1);
        abort_sm = 0;
        fence_barrier_init();
    }
    __syncthreads();
    uint32_t pending = 0;  // leader: slots with a copy in flight
    if (leader) {
        for (int j = 0; j < nslots; ++j) {
            const int64_t r = row0 + j * rstride;
            if (r < rows) {
                mbar_arrive_expect_tx(slot_bar(j), row_bytes);
                bulk_load(slot_addr(j), in + r * K, row_bytes, slot_bar(j));
                pending |= 1u << j;
            }
        }
    }
    // factor tables, staged while the first rows are in flight
    const bool bad_divisor = __syncthreads_or(stage_factor_tables<MODE == MODE_X, BF>(
                                 s, static_cast<int>(K), f_sm, fb_sm, threadIdx.x, blockDim.x)) != 0;
    auto factor_pairs = [&](int c, float2 (&f2)[V / 2]) {
#pragma unroll
        for (int h = 0; h < V / 4; ++h) {
            const float4 v4 = reinterpret_cast<const float4 *>(f_sm + static_cast<int64_t>(c) * V)[h];
            f2[2 * h] = make_float2(v4.x, v4.y);
            f2[2 * h + 1] = make_float2(v4.z, v4.w);
        }
    };
    int nred = 0;
    auto group_max = [&](float v) -> float {
        v = warp_max(v);
        if (G == 1)
            return v;
        float *r = red[nred & 1];
        ++nred;
        if (lane == 0)
            r[warp] = v;
        named_barrier_sync(1 + group, 32 * G);
        float m = r[group << log2g];
        for (int j = 1; j < G; ++j)
            m = fmaxf(m, r[(group << log2g) + j]);
        return m;
    };
    auto group_sync = [&]() {
        if (G == 1)
            __syncwarp();
        else
            named_barrier_sync(1 + group, 32 * G);
    };

    int j = 0;
    for (int64_t row = row0; row < rows; row += rstride, ++j) {
        const int slot = j % nslots;
        const uint32_t par = static_cast<uint32_t>(j / nslots) & 1u;
        const bool ok = bounded_wait(slot_bar(slot), par, kErrWaitRow, &abort_sm);
        if (!__all_sync(0xFFFFFFFFu, ok))
            break;
        if (leader)
            pending &= ~(1u << slot);
        const uint32_t sbase = slot_addr(slot);
        uint4 raw[CH];
#pragma unroll
        for (int i = 0; i < CH; ++i) {
            const uint32_t a = sbase + static_cast<uint32_t>(c0 + cstep * i) * 16u;
            asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                         : "=r"(raw[i].x), "=r"(raw[i].y), "=r"(raw[i].z), "=r"(raw[i].w)
                         : "r"(a));
        }
        // 1. bounds of |v| per chunk, the row's largest bound A, the exact maximum E
        float hm[CH];
        float am = 0.0f;
#pragma unroll
        for (int i = 0; i < CH; ++i) {
            if constexpr (BF) {
                const uint4 fb = *reinterpret_cast<const uint4 *>(fb_sm + static_cast<int64_t>(c0 + cstep * i) * 4);
                uint32_t p = bf2_mul(raw[i].x & 0x7FFF7FFFu, fb.x);
                p = bf2_max(p, bf2_mul(raw[i].y & 0x7FFF7FFFu, fb.y));
                p = bf2_max(p, bf2_mul(raw[i].z & 0x7FFF7FFFu, fb.z));
                p = bf2_max(p, bf2_mul(raw[i].w & 0x7FFF7FFFu, fb.w));
                hm[i] = bf2_hmax_f32(p);
            } else {
                float x[V];
                float2 f2[V / 2];
                widen<__nv_bfloat16>(raw[i], x);
                factor_pairs(c0 + cstep * i, f2);
                float h = 0.0f;
#pragma unroll
                for (int e = 0; e < V; e += 2) {
                    const float2 a = f2_mul(make_float2(x[e], x[e + 1]), f2[e / 2]);
                    h = fmaxf(h, fmaxf(fabsf(a.x), fabsf(a.y)));
                }
                hm[i] = h;
            }
            am = fmaxf(am, hm[i]);
        }
        const float A = group_max(am);
        float E = A;  // fp32-bounded weights: the bounds are the values themselves
        if (BF || MODE == MODE_X) {
            const bool exact_all = bad_divisor || !(A >= kTinyQuotient) || !(A <= 0x1.fffffep127f);
            const float thr = __fmul_rn(A, BF ? 0.96875f : kCandidateScale);
            uint32_t cand = 0;
#pragma unroll
            for (int i = 0; i < CH; ++i)
                cand |= (exact_all || hm[i] >= thr) ? (1u << i) : 0u;
            float em = 0.0f;
            while (cand != 0u) {  // rare: the candidate elements exactly
                const int i = __ffs(cand) - 1;
                cand &= cand - 1u;
                const int64_t c = c0 + cstep * i;
                em = fmaxf(em, staged_candidates<MODE, BF>(sbase + static_cast<uint32_t>(c) * 16u, fb_sm + c * 4,
                                                           f_sm + c * V, s + c * V, thr, exact_all));
            }
            E = group_max(em);
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
        uint32_t ties = 0;
#pragma unroll
        for (int i = 0; i < CH; ++i) {
            const int c = c0 + cstep * i;
            float x[V];
            uint32_t y[V];
            float2 f2[V / 2];
            widen<__nv_bfloat16>(raw[i], x);
            factor_pairs(c, f2);
            float dmax = 0.0f;
#pragma unroll
            for (int e = 0; e < V; e += 2) {
                const float2 a = f2_mul(make_float2(x[e], x[e + 1]), f2[e / 2]);
                const float2 yy = f2_fma(a, rsc2, magic2);
                const float2 rr = f2_add(yy, nmagic2);
                const float2 dd = f2_fma(a, nrsc2, rr);
                dmax = fmaxf(dmax, fmaxf(fabsf(dd.x), fabsf(dd.y)));
                y[e] = __float_as_uint(yy.x);
                y[e + 1] = __float_as_uint(yy.y);
            }
            ties |= (!fast || !(dmax < kTieLimit)) ? (1u << i) : 0u;
            store_code_words(dst + static_cast<int64_t>(c) * V, y, V);
        }
        while (ties != 0u) {  // rare: near ties; every element when the scale is outside the fast range
            const int i = __ffs(ties) - 1;
            ties &= ties - 1u;
            const int64_t c = c0 + cstep * i;
            staged_ties<MODE>(sbase + static_cast<uint32_t>(c) * 16u, f_sm + c * V, s + c * V, scale, rsc, fast,
                              dst + c * V);
        }
        // every warp of the group is done with the slot: refill it
        group_sync();
        if (leader) {
            const int64_t r = row + static_cast<int64_t>(nslots) * rstride;
            if (r < rows) {
                mbar_arrive_expect_tx(slot_bar(slot), row_bytes);
                bulk_load(sbase, in + r * K, row_bytes, slot_bar(slot));
                pending |= 1u << slot;
            }
        }
    }
    // after a timeout the copies still in flight land before the CTA leaves
    if (leader && abort_sm) {
        for (int k = 0; k < nslots; ++k)
            if (pending & (1u << k)) {
                // the phase a pending copy completes: parity of that slot's next use
                int jj = j;
                while (jj % nslots != k)
                    ++jj;
                bounded_wait(slot_bar(k), static_cast<uint32_t>(jj / nslots) & 1u, kErrWaitDrain, nullptr,
                             kWaitTimeoutNs / 4);
            }
    }
}

}  // namespace sq
