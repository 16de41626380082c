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
// The arithmetic is that of sq_div.cuh and of row_quant_kernel: an fp32
// bound a_k = RN(x_k * f_k) of |v| per element (f_k the hardware reciprocal
// of s_k for activations, s_k itself for weights), exact quotients for the
// elements within 2^-20 of the largest bound, the scale by Markstein's
// iteration, and the codes from the rounding fast path with the exact IEEE
// path near ties.  What differs is how the rows move and where a_k lives:
//   * s is brought into shared memory whole by one bulk copy (cp.async.bulk),
//     issued before any row, so every exact step reads s_k there;
//   * a CTA of THREADS / 32 warps holds groups of G warps; each group owns
//     `nslots` row buffers in shared memory, filled with the group's next rows
//     by bulk copies (completion on an mbarrier), so nslots rows per group
//     are in flight however long the arithmetic of the current one takes;
//     the last warp of the group to finish with a buffer refills it, so no
//     warp waits for another at the end of a row;
//   * lane L of warp g of a group takes the 16-byte chunks c = 32 g + L +
//     32 G i, i < CH, of the row: one shared-memory load each; the products
//     a_k of the first pass stay in registers for the second, which then
//     only rounds them;
//   * E = max_k |v_k|: each warp takes the exact |v| of its own elements
//     within 2^-20 of its own largest bound (a superset of those within
//     2^-20 of the row's largest, and every element it adds is a real |v_k|,
//     so the maximum is unchanged), then one exchange across the group.
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

// Row buffers a group holds at most.
constexpr int kStagedMaxSlots = 4;

// shared memory of the staged quantiser: s (K fp32), then the row slots
// (128-byte aligned), then one mbarrier per slot and one for s
__host__ __device__ constexpr int64_t staged_slots_offset(int64_t K) { return (K * 4 + 127) / 128 * 128; }

__host__ __device__ constexpr int64_t staged_smem_bytes(int64_t K, int groups, int nslots)
{
    return staged_slots_offset(K) + static_cast<int64_t>(groups) * nslots * K * 2 +
           (static_cast<int64_t>(groups) * nslots + 1) * 8;
}

__device__ __forceinline__ uint4 lds_u4(uint32_t addr)
{
    uint4 r;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "r"(addr));
    return r;
}

// s_k and f_k of a chunk's eight elements, s from shared memory
template <int MODE>
__device__ __forceinline__ void chunk_factors(uint32_t s_addr, float (&sv)[8], float (&f)[8])
{
    const uint4 s0 = lds_u4(s_addr), s1 = lds_u4(s_addr + 16u);
    const uint32_t w[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        sv[e] = __uint_as_float(w[e]);
        f[e] = MODE == MODE_X ? rcp_approx(sv[e]) : sv[e];
    }
}

// Rare paths, element by element.  A chunk is flagged as a whole by the
// register passes, but usually only one of its 8 elements needs the exact
// quotient; the chunk is re-read from its row buffer.
//   candidates: the exact |v| of the elements whose bound reaches thr (all of
//   them when exact_all), maximum over those.
template <int MODE>
__device__ __noinline__ float staged_candidates(uint32_t raw_addr, uint32_t s_addr, float thr, bool exact_all)
{
    const uint4 r = lds_u4(raw_addr);
    float sv[8], f[8], x[8];
    chunk_factors<MODE>(s_addr, sv, f);
    widen<__nv_bfloat16>(r, x);
    float m = 0.0f;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        if (exact_all || fabsf(__fmul_rn(x[e], f[e])) >= thr)
            m = fmaxf(m, fabsf(MODE == MODE_X ? __fdiv_rn(x[e], sv[e]) : __fmul_rn(x[e], sv[e])));
    }
    return m;
}

//   ties: the elements whose fast code lies within 2^-13 of a rounding tie
//   (every element when !fast) get the exact code, one byte store each; the
//   fast path has already stored the chunk's other codes.
template <int MODE>
__device__ __noinline__ void staged_ties(uint32_t raw_addr, uint32_t s_addr, float scale, float rsc, bool fast,
                                         int8_t *dst)
{
    const uint4 r = lds_u4(raw_addr);
    float sv[8], f[8], x[8];
    chunk_factors<MODE>(s_addr, sv, f);
    widen<__nv_bfloat16>(r, x);
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        const float a = __fmul_rn(x[e], f[e]);
        const float yy = __fmaf_rn(a, rsc, kRoundMagic);
        const float dd = __fmaf_rn(a, -rsc, __fadd_rn(yy, -kRoundMagic));
        if (!fast || !(fabsf(dd) < kTieLimit)) {
            const float v = MODE == MODE_X ? __fdiv_rn(x[e], sv[e]) : __fmul_rn(x[e], sv[e]);
            const uint32_t cb = scale != 0.0f ? exact_code_bits(v, scale) : code_bits(0.0f);
            dst[e] = static_cast<int8_t>(cb & 0xFFu);
        }
    }
}

// THREADS = 256 (8 warps), or 512 (16 warps) where an SM holds one CTA.
template <int MODE, int CH, int THREADS = kQuantThreads>
__global__ void __launch_bounds__(THREADS, (CH >= 14 || THREADS > kQuantThreads) ? 1 : 2)
    row_quant_staged_kernel(const __nv_bfloat16 *__restrict__ in, int64_t rows, int64_t K,
                            const float *__restrict__ s, int log2g, int nslots, int8_t *__restrict__ q,
                            float *__restrict__ scale_out, int *__restrict__ zero, int nzero)
{
    pdl_prologue();
    clear_ints(zero, nzero);
    constexpr int V = 8;
    constexpr int WARPS = THREADS / 32;
    extern __shared__ __align__(128) uint8_t qs_smem[];
    __shared__ float red[2][WARPS];
    __shared__ int okv[2][WARPS];
    __shared__ int done_cnt[WARPS][kStagedMaxSlots];  // warps of a group done with a buffer
    __shared__ uint32_t inflight[WARPS];               // buffers of a group with a copy in flight
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
    const uint32_t stab = smem_u32(qs_smem);
    const float *s_sm = reinterpret_cast<const float *>(qs_smem);
    const uint32_t slots = stab + static_cast<uint32_t>(staged_slots_offset(K));
    const uint32_t bars = slots + static_cast<uint32_t>(groups * nslots) * row_bytes;
    const uint32_t tab_bar = bars + 8u * static_cast<uint32_t>(groups * nslots);
    auto slot_addr = [&](int j) { return slots + static_cast<uint32_t>(group * nslots + j) * row_bytes; };
    auto slot_bar = [&](int j) { return bars + 8u * static_cast<uint32_t>(group * nslots + j); };
    const bool leader = g == 0 && lane == 0;
    const int64_t row0 = static_cast<int64_t>(blockIdx.x) * groups + group;
    const int64_t rstride = static_cast<int64_t>(gridDim.x) * groups;

    if (threadIdx.x == 0) {
        for (int j = 0; j <= groups * nslots; ++j)
            mbar_init(bars + 8u * j, 1);
        abort_sm = 0;
        fence_barrier_init();
    }
    for (int i = threadIdx.x; i < WARPS * kStagedMaxSlots; i += THREADS)
        done_cnt[i / kStagedMaxSlots][i % kStagedMaxSlots] = 0;
    if (threadIdx.x < WARPS)
        inflight[threadIdx.x] = 0u;
    __syncthreads();
    // s first, then the group's first rows
    if (threadIdx.x == 0) {
        mbar_arrive_expect_tx(tab_bar, static_cast<uint32_t>(K * 4));
        bulk_load(stab, s, static_cast<uint32_t>(K * 4), tab_bar);
    }
    if (leader) {
        uint32_t bits = 0;
        for (int j = 0; j < nslots; ++j) {
            const int64_t r = row0 + j * rstride;
            if (r < rows) {
                mbar_arrive_expect_tx(slot_bar(j), row_bytes);
                bulk_load(slot_addr(j), in + r * K, row_bytes, slot_bar(j));
                bits |= 1u << j;
            }
        }
        atomicOr(&inflight[group], bits);
    }
    const bool tab_ok = bounded_wait(tab_bar, 0, kErrWaitRow, &abort_sm);
    const bool tab_fail = __syncthreads_or(!tab_ok) != 0;
    // divisors outside the range of the fast paths send every row to the exact path
    int bad = 0;
    if (MODE == MODE_X && !tab_fail)
        for (int k = threadIdx.x; k < K; k += THREADS)
            bad |= !div_operand_ok(s_sm[k]);
    const bool bad_divisor = __syncthreads_or(bad) != 0;

    // maximum over the G warps of this row: one value a warp, read back by
    // the lanes in parallel; alternating buffers, so a buffer is rewritten
    // only after every warp of the group has passed the barrier that follows
    // its last read
    // with it, whether every warp of the group had its row (the group then
    // goes on or leaves together)
    int nred = 0;
    auto group_max = [&](float v, bool ok_w, bool &ok_g) -> float {
        v = warp_max(v);
        if (G == 1) {
            ok_g = ok_w;
            return v;
        }
        float *r = red[nred & 1];
        int *o = okv[nred & 1];
        ++nred;
        if (lane == 0) {
            r[warp] = v;
            o[warp] = ok_w ? 1 : 0;
        }
        named_barrier_sync(1 + group, 32 * G);
        ok_g = __all_sync(0xFFFFFFFFu, lane < G ? o[(group << log2g) + lane] != 0 : true);
        return warp_max(lane < G ? r[(group << log2g) + lane] : 0.0f);
    };

    int j = 0;
    for (int64_t row = row0; row < rows && !tab_fail; row += rstride, ++j) {
        const int slot = j % nslots;
        const uint32_t par = static_cast<uint32_t>(j / nslots) & 1u;
        const bool ok = __all_sync(0xFFFFFFFFu, bounded_wait(slot_bar(slot), par, kErrWaitRow, &abort_sm));
        if (G == 1 && !ok)
            break;  // (a group of several warps leaves together, after its exchange)
        if (leader && ok)
            atomicAnd(&inflight[group], ~(1u << slot));
        const uint32_t sbase = slot_addr(slot);
        // 1. the products a_k (kept for pass 2) and the bounds
        float a[CH][V];
        float hm[CH];
        float am = 0.0f;
#pragma unroll
        for (int i = 0; i < CH; ++i) {
            const uint32_t c = static_cast<uint32_t>(c0 + cstep * i);
            const uint4 r = lds_u4(sbase + c * 16u);
            float sv[V], f[V], x[V];
            chunk_factors<MODE>(stab + c * 32u, sv, f);
            widen<__nv_bfloat16>(r, x);
            const float2 p0 = f2_mul(make_float2(x[0], x[1]), make_float2(f[0], f[1]));
            const float2 p1 = f2_mul(make_float2(x[2], x[3]), make_float2(f[2], f[3]));
            const float2 p2 = f2_mul(make_float2(x[4], x[5]), make_float2(f[4], f[5]));
            const float2 p3 = f2_mul(make_float2(x[6], x[7]), make_float2(f[6], f[7]));
            a[i][0] = p0.x;
            a[i][1] = p0.y;
            a[i][2] = p1.x;
            a[i][3] = p1.y;
            a[i][4] = p2.x;
            a[i][5] = p2.y;
            a[i][6] = p3.x;
            a[i][7] = p3.y;
            const float h01 = fmaxf(fabsf(p0.x), fabsf(p0.y)), h23 = fmaxf(fabsf(p1.x), fabsf(p1.y));
            const float h45 = fmaxf(fabsf(p2.x), fabsf(p2.y)), h67 = fmaxf(fabsf(p3.x), fabsf(p3.y));
            hm[i] = fmaxf(fmaxf(h01, h23), fmaxf(h45, h67));
            am = fmaxf(am, hm[i]);
        }
        // 2. E, exact: this warp's candidates, then one exchange (weights:
        // a_k is v_k itself)
        float ew = warp_max(am);
        if (MODE == MODE_X) {
            const float Aw = ew;
            const bool exact_all = bad_divisor || !(Aw >= kTinyQuotient) || !(Aw <= 0x1.fffffep127f);
            const float thr = __fmul_rn(Aw, kCandidateScale);
            uint32_t cand = 0;
#pragma unroll
            for (int i = 0; i < CH; ++i)
                cand |= (exact_all || hm[i] >= thr) ? (1u << i) : 0u;
            float em = 0.0f;
            while (cand != 0u) {  // rare: the candidate elements exactly
                const int i = __ffs(cand) - 1;
                cand &= cand - 1u;
                const uint32_t c = static_cast<uint32_t>(c0 + cstep * i);
                em = fmaxf(em, staged_candidates<MODE>(sbase + c * 16u, stab + c * 32u, thr, exact_all));
            }
            ew = em;
        }
        bool go = true;
        const float E = group_max(ew, ok, go);
        if (!go)
            break;  // some warp of the group timed out waiting for the row

        // 3. scale and codes, from the products in registers
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
            uint32_t y[V];
            float dmax = 0.0f;
#pragma unroll
            for (int e = 0; e < V; e += 2) {
                const float2 av = make_float2(a[i][e], a[i][e + 1]);
                const float2 yy = f2_fma(av, rsc2, magic2);
                const float2 rr = f2_add(yy, nmagic2);
                const float2 dd = f2_fma(av, nrsc2, rr);
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
            const uint32_t c = static_cast<uint32_t>(c0 + cstep * i);
            staged_ties<MODE>(sbase + c * 16u, stab + c * 32u, scale, rsc, fast, dst + static_cast<int64_t>(c) * V);
        }
        // 4. this warp is done with the buffer; the group's last refills it
        __syncwarp();
        if (lane == 0) {
            __threadfence_block();
            if (atomicAdd(&done_cnt[group][slot], 1) == G - 1) {
                done_cnt[group][slot] = 0;
                const int64_t r = row + static_cast<int64_t>(nslots) * rstride;
                if (r < rows) {
                    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                    mbar_arrive_expect_tx(slot_bar(slot), row_bytes);
                    bulk_load(sbase, in + r * K, row_bytes, slot_bar(slot));
                    atomicOr(&inflight[group], 1u << slot);
                }
            }
        }
    }
    // after a timeout the copies still in flight land before the CTA leaves
    __syncthreads();
    if (threadIdx.x == 0 && !tab_ok)
        bounded_wait(tab_bar, 0, kErrWaitDrain, nullptr, kWaitTimeoutNs / 4);
    if (leader && abort_sm) {
        const uint32_t pend = inflight[group];
        for (int k = 0; k < nslots; ++k)
            if (pend & (1u << k)) {
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
