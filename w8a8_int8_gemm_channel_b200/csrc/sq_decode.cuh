// sq_decode.cuh -- the W8A8 GEMM for few tokens (M <= 128) inside sq_linear:
// a stream over the int8 weight, split evenly over every SM.
//
//   acc[m, n] = sum_k xq[m, k] * wq[n, k]     y[m, n] = ((float)acc * sx[m]) * sw[n]
//
// Sources: "quant_llm_int8", "The architecture: every piece explained" (int32
// accumulation, outer-product dequantisation); "Understanding W8A8 INT8 LLM
// Quantization", "Inter-Token Latency (ITL)" (at decode the layer streams its
// weight and the per-token quantisation is memory-bound work every step pays).
//
// Work.  The weight takes the 128-row MMA side (a tile = 128 output channels)
// and the tokens form the MMA N dimension (BNX padded token rows).  A unit is
// one 128-byte k block of one tile (16 KB of weight); the T * KB units, tile
// by tile, are cut into G equal contiguous ranges, one per CTA and one CTA per
// SM, so every SM streams the same number of weight bytes whatever N and K
// are.  A CTA's range covers whole tiles in its middle and at most a part of
// a tile at either end.
//
// Reduction.  A tile that several CTAs share is summed through the caller's
// workspace: each contributor writes its int32 partial to its own slot, then
// counts itself in the tile's counter (the counters are cleared by the
// quantiser kernel that sq_linear runs just before); the contributor that
// completes the count adds the slots and stores the dequantised tile.
// Integer addition, so the result does not depend on the order.
//
// Overlap with the quantiser.  sq_linear launches this kernel right after its
// own quantiser kernel, with programmatic dependent launch.  That quantiser
// waits for every earlier grid on the stream before it lets this grid start,
// so when this grid runs, every earlier write (to the weight and its scales
// in particular) is complete and visible.  The producer therefore issues the
// weight loads of the first stages (and an L2 prefetch of the CTA's whole
// weight range) before griddepcontrol.wait, and only the activation codes
// and scales -- the quantiser's outputs -- wait for it: the weight stream
// overlaps the quantisation.
//
// Roles (192 threads):
//   warp 0      TMA producer: per unit a 128 x 128-byte weight tile and a
//               BNX x 128-byte tile of the codes, 128-byte swizzle, no multicast
//   warp 1      TMEM allocation; tcgen05.mma.kind::i8, M = 128, N = BNX, K = 32,
//               rotating over NACC accumulators; two accumulator sets, so a
//               range's next tile accumulates while the epilogue drains one
//   warps 2..5  epilogue: tcgen05.ld, then either the dequantised tile
//               (a tile this CTA owns alone) or the partial and the count
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#include "sq_gemm.cuh"
#include "sq_ptx.cuh"

namespace sq {

constexpr int kDecThreads = 192;
constexpr unsigned int kErrWaitDecode = 0xB00;  // decode GEMM epilogue waiting for an accumulator

// First unit of CTA c when U units are cut into G ranges.
__host__ __device__ __forceinline__ int64_t dec_start(int64_t c, int64_t U, int64_t G) { return c * U / G; }

// The CTA whose range holds unit u: the largest c with dec_start(c) <= u.
__host__ __device__ __forceinline__ int64_t dec_owner(int64_t u, int64_t U, int64_t G) { return ((u + 1) * G - 1) / U; }

// Accumulators a tile rotates over, and TMEM columns (two sets).
template <int BNX>
struct DecCfg {
    static constexpr int NACC = BNX >= 128 ? 2 : 4;
    static constexpr int TMEM_COLS = 2 * NACC * BNX;
    static constexpr int W_BYTES = kBM * kBK;   // 16 KB
    static constexpr int X_BYTES = BNX * kBK;
    static constexpr int STAGE_BYTES = W_BYTES + X_BYTES;
    static_assert(BNX == 32 || BNX == 64 || BNX == 128, "token tile");
    static_assert(TMEM_COLS <= 512 && (TMEM_COLS & (TMEM_COLS - 1)) == 0, "TMEM columns");
};

// shared memory: 1024 alignment slack, the ring, barriers (full, empty,
// tfull[2], tempty[2], drain), the TMEM slot, the abort flag and the
// last-contributor flag, then the token scales (at most 128 floats)
constexpr int kDecSxBytes = 128 * 4;
__host__ __device__ constexpr int dec_smem_bytes(int stage_bytes, int stages)
{
    return 1024 + stages * stage_bytes + (2 * stages + 5) * 8 + 16 + kDecSxBytes;
}

// store_col_chunk with the token scales read from shared memory
template <int OUT>
__device__ __forceinline__ void dec_store_chunk(const uint32_t (&r)[32], float swn, const float *sx_s, int m0,
                                                int M, void *__restrict__ y, int64_t n, int N)
{
    const int valid = min(32, M - m0);
#pragma unroll
    for (int j = 0; j < 32; ++j) {
        if (j < valid) {
            const int64_t idx = static_cast<int64_t>(m0 + j) * N + n;
            if constexpr (OUT == OUT_S32) {
                reinterpret_cast<int32_t *>(y)[idx] = static_cast<int32_t>(r[j]);
            } else {
                const float o = __fmul_rn(__fmul_rn(__int2float_rn(static_cast<int>(r[j])), sx_s[m0 + j]), swn);
                if constexpr (OUT == OUT_F32)
                    reinterpret_cast<float *>(y)[idx] = o;
                else
                    reinterpret_cast<__nv_bfloat16 *>(y)[idx] = __float2bfloat16_rn(o);
            }
        }
    }
}

// barrier of the four epilogue warps (named barrier 2)
__device__ __forceinline__ void dec_bar_sync() { asm volatile("bar.sync 2, 128;" ::: "memory"); }

// Slot of the partial that CTA c writes for tile t (0: the range's first
// tile, 1: its last); ws holds G x 2 slots of 128 rows x BNX int32, each
// row's tokens contiguous.
__device__ __forceinline__ int32_t *dec_slot(int32_t *ws, int64_t c, int slot, int BNX)
{
    return ws + (c * 2 + slot) * static_cast<int64_t>(BNX) * kBM;
}

// pre_wait: bit 0 -- issue the first stages' weight loads before
// griddepcontrol.wait; bit 1 -- also prefetch the rest of the range into L2.
template <int BNX, int OUT>
__global__ void __launch_bounds__(kDecThreads, 1)
    gemm_decode_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
                       const float *__restrict__ sx, const float *__restrict__ sw, void *__restrict__ y,
                       int32_t *__restrict__ ws, int *__restrict__ cnt, int M, int N, int K, int64_t U,
                       int G, int stages, int pre_wait)
{
    using Cfg = DecCfg<BNX>;
    constexpr int NACC = Cfg::NACC;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const bool producer = warp == 0 && lane == 0;

    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t *gb = smem_raw + (base - raw);
    const uint32_t sW = base;
    const uint32_t sX = base + stages * Cfg::W_BYTES;
    const uint32_t bars = sX + stages * Cfg::X_BYTES;
    auto full_bar = [&](int i) { return bars + 8u * i; };
    auto empty_bar = [&](int i) { return bars + 8u * (stages + i); };
    auto tfull_bar = [&](int b) { return bars + 8u * (2 * stages + b); };
    auto tempty_bar = [&](int b) { return bars + 8u * (2 * stages + 2 + b); };
    const uint32_t drain_bar = bars + 8u * (2 * stages + 4);
    const uint32_t misc_off = (bars - base) + 8u * (2 * stages + 5);
    volatile uint32_t *tmem_slot = reinterpret_cast<volatile uint32_t *>(gb + misc_off);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(gb + misc_off + 4);
    volatile int *last_flag = reinterpret_cast<volatile int *>(gb + misc_off + 8);
    float *sx_s = reinterpret_cast<float *>(gb + misc_off + 16);

    const int64_t c = blockIdx.x;
    const int KB = (K + kBK - 1) / kBK;
    const int64_t u0 = dec_start(c, U, G), u1 = dec_start(c + 1, U, G);
    const int64_t first_tile = u0 / KB;

    if (threadIdx.x == 32) {
        for (int i = 0; i < stages; ++i) {
            mbar_init(full_bar(i), 1);
            mbar_init(empty_bar(i), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(tfull_bar(b), 1);
            mbar_init(tempty_bar(b), 4);  // the 4 epilogue warps
        }
        mbar_init(drain_bar, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (producer) {
        // the tensor maps are this launch's own parameters: fetched while
        // the grid before still runs
        tma_prefetch_desc(&tmW);
        tma_prefetch_desc(&tmX);
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(const_cast<uint32_t *>(tmem_slot)), Cfg::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem_base = *tmem_slot;
    // Up to here nothing touched global memory but the tensor maps.  Every
    // thread but the producer waits for the grid before (the quantiser) now;
    // the producer first requests weight tiles when that is allowed.
    if (!(producer && (pre_wait & 1)))
        asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

    uint32_t issued_mask = 0, issued_parity = 0;
    bool mma_issued_any = false;

    if (warp == 0) {
        if (lane == 0) {
            const int64_t nu = u1 - u0;
            // units whose weight tile is requested before the wait
            const int pre = (pre_wait & 1) ? static_cast<int>(nu < stages ? nu : stages) : 0;
            for (int i = 0; i < pre; ++i) {
                const int64_t u = u0 + i;
                mbar_arrive_expect_tx(full_bar(i), Cfg::STAGE_BYTES);
                tma_load_2d(sW + i * Cfg::W_BYTES, &tmW, full_bar(i), static_cast<int32_t>(u % KB) * kBK,
                            static_cast<int32_t>(u / KB) * kBM);
                issued_mask |= 1u << i;
            }
            if (pre_wait & 1) {
                // the rest of the range into L2 while the quantiser runs
                if (pre_wait & 2)
                    for (int64_t u = u0 + pre; u < u1; ++u)
                        tma_prefetch_l2_2d(&tmW, static_cast<int32_t>(u % KB) * kBK,
                                           static_cast<int32_t>(u / KB) * kBM);
                asm volatile("griddepcontrol.wait;" ::: "memory");
            }
            for (int i = 0; i < pre; ++i)
                tma_load_2d(sX + i * Cfg::X_BYTES, &tmX, full_bar(i), static_cast<int32_t>((u0 + i) % KB) * kBK, 0);
            int stage = pre % stages;
            uint32_t phase = (pre == stages) ? 1u : 0u;
            for (int64_t u = u0 + pre; u < u1; ++u) {
                if (!bounded_wait(empty_bar(stage), phase ^ 1u, kErrWaitProducer, abort_flag))
                    break;
                mbar_arrive_expect_tx(full_bar(stage), Cfg::STAGE_BYTES);
                const int32_t kx = static_cast<int32_t>(u % KB) * kBK;
                tma_load_2d(sW + stage * Cfg::W_BYTES, &tmW, full_bar(stage), kx, static_cast<int32_t>(u / KB) * kBM);
                tma_load_2d(sX + stage * Cfg::X_BYTES, &tmX, full_bar(stage), kx, 0);
                issued_mask |= 1u << stage;
                issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
                if (++stage == stages) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_i8(kBM, BNX);
            int stage = 0;
            uint32_t phase = 0;
            int acc = 0;
            uint32_t acc_phase = 0;
            bool ok = true;
            for (int64_t u = u0; u < u1 && ok;) {
                const int64_t t = u / KB;
                const int64_t seg_end = min(u1, (t + 1) * KB);
                if (!bounded_wait(tempty_bar(acc), acc_phase ^ 1u, kErrWaitAccEmpty, abort_flag))
                    break;
                tc_fence_after_sync();
                const uint32_t d0 = tmem_base + static_cast<uint32_t>(acc * NACC * BNX);
                int step = 0;
                for (; u < seg_end; ++u) {
                    if (!bounded_wait(full_bar(stage), phase, kErrWaitMma, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after_sync();
                    const uint32_t a0 = sW + stage * Cfg::W_BYTES;
                    const uint32_t b0 = sX + stage * Cfg::X_BYTES;
#pragma unroll
                    for (int k = 0; k < kBK / 32; ++k, ++step)
                        mma_i8(d0 + static_cast<uint32_t>((step % NACC) * BNX), smem_desc_k_sw128(a0 + 32 * k),
                               smem_desc_k_sw128(b0 + 32 * k), idesc, step >= NACC ? 1u : 0u);
                    mma_issued_any = true;
                    mma_commit(empty_bar(stage));
                    if (++stage == stages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok)
                    break;
                mma_commit(tfull_bar(acc));
                acc ^= 1;
                if (acc == 0)
                    acc_phase ^= 1u;
            }
        }
    } else {
        // epilogue warps 2..5: warp w reads TMEM lanes 32 (w % 4) .. +31
        const int quarter = warp & 3;
        const int row = quarter * 32 + lane;  // weight row within the tile
        const int et = threadIdx.x - 64;      // 0..127
        // the token scales into shared memory while the weight streams, so
        // that no store after the last MMA waits for a global load
        if (OUT != OUT_S32 && et < M)
            sx_s[et] = __ldg(sx + et);
        dec_bar_sync();
        int acc = 0;
        uint32_t acc_phase = 0;
        for (int64_t u = u0; u < u1;) {
            const int64_t t = u / KB;
            const int64_t seg_begin = u;
            const int64_t seg_end = min(u1, (t + 1) * KB);
            u = seg_end;
            const bool whole = seg_begin == t * KB && seg_end == (t + 1) * KB;
            const int64_t n = t * kBM + row;
            const float swn = (OUT != OUT_S32 && n < N) ? __ldg(sw + n) : 0.0f;
            const bool ok = bounded_wait(tfull_bar(acc), acc_phase, kErrWaitAccFull, abort_flag);
            if (!__all_sync(0xFFFFFFFFu, ok))
                break;
            tc_fence_after_sync();
            const int slot = t == first_tile ? 0 : 1;
            int32_t *mine = dec_slot(ws, c, slot, BNX);
            const uint32_t lane_addr =
                tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + static_cast<uint32_t>(acc * NACC * BNX);
#pragma unroll 1
            for (int cc = 0; cc < BNX / 32; ++cc) {
                if (cc * 32 >= M)
                    break;
                uint32_t r[32], q[32];
                tmem_ld_32x32b_x32(lane_addr + cc * 32, r);
                tmem_ld_wait();
#pragma unroll 1
                for (int a = 1; a < NACC; ++a) {
                    tmem_ld_32x32b_x32(lane_addr + static_cast<uint32_t>(a * BNX) + cc * 32, q);
                    tmem_ld_wait();
#pragma unroll
                    for (int j = 0; j < 32; ++j)
                        r[j] += q[j];  // exact int32 sums
                }
                if (whole) {
                    if (n < N)
                        dec_store_chunk<OUT>(r, swn, sx_s, cc * 32, M, y, n, N);
                } else {
                    // this row's partial, the valid tokens only, 16 bytes at a time
                    int4 *dst = reinterpret_cast<int4 *>(mine + row * BNX + cc * 32);
                    const int nv = (min(M - cc * 32, 32) + 3) >> 2;
#pragma unroll
                    for (int v = 0; v < 8; ++v)
                        if (v < nv)
                            dst[v] = make_int4(r[4 * v], r[4 * v + 1], r[4 * v + 2], r[4 * v + 3]);
                }
            }
            // the accumulator set is free for the next tile of the range
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(tempty_bar(acc));
            acc ^= 1;
            if (acc == 0)
                acc_phase ^= 1u;
            if (whole)
                continue;
            // count this partial in (one release by one thread after the
            // barrier of the epilogue warps); the contributor that completes
            // the count adds every contributor's slot and stores the tile
            dec_bar_sync();
            const int64_t cf = dec_owner(t * KB, U, G), cl = dec_owner((t + 1) * KB - 1, U, G);
            if (et == 0) {
                // release: this CTA's partial (ordered before it by the
                // barrier) precedes the count; acquire: the other
                // contributors' partials precede the reads that follow
                const int old = atom_add_acq_rel_gpu(cnt + t, 1);
                *last_flag = old == static_cast<int>(cl - cf);
            }
            dec_bar_sync();
            if (*last_flag) {
                // On the range's last segment every stage of the ring has been
                // consumed (the accumulator-full signal follows the last MMA),
                // so with one token chunk (BNX = 32) the contributors' partials
                // can land there: all of them in flight at once, whatever the
                // register budget.  Thread `row` owns the 16-byte words
                // (i, v, row), i the contributor and v the token quad, laid out
                // so a warp's accesses are contiguous.
                const int64_t S = cl - cf + 1;
                const bool ring_free = seg_end == u1;
                const int4 *land = reinterpret_cast<const int4 *>(gb + (sW - base));
#pragma unroll 1
                for (int cc = 0; cc < BNX / 32; ++cc) {
                    if (cc * 32 >= M)
                        break;
                    const int nv = (min(M - cc * 32, 32) + 3) >> 2;
                    uint32_t r[32];
#pragma unroll
                    for (int j = 0; j < 32; ++j)
                        r[j] = 0u;
                    // this row's partial in contributor c2's slot
                    auto part = [&](int64_t c2) {
                        return reinterpret_cast<const int4 *>(
                            dec_slot(ws, c2, dec_start(c2, U, G) / KB == t ? 0 : 1, BNX) + row * BNX + cc * 32);
                    };
                    auto add4 = [&](int v, int4 a) {
                        r[4 * v] += static_cast<uint32_t>(a.x);
                        r[4 * v + 1] += static_cast<uint32_t>(a.y);
                        r[4 * v + 2] += static_cast<uint32_t>(a.z);
                        r[4 * v + 3] += static_cast<uint32_t>(a.w);
                    };
                    if (BNX == 32 && ring_free && S * nv * kBM * 16 <= static_cast<int64_t>(stages) * Cfg::STAGE_BYTES) {
                        for (int64_t i = 0; i < S; ++i) {
                            const int4 *p = part(cf + i);
                            for (int v = 0; v < nv; ++v)
                                cp_async_16(sW + static_cast<uint32_t>(((i * nv + v) * kBM + row) * 16), p + v, true);
                        }
                        cp_async_wait_all();
                        for (int64_t i = 0; i < S; ++i) {
#pragma unroll
                            for (int v = 0; v < 8; ++v)
                                if (v < nv)
                                    add4(v, land[(i * nv + v) * kBM + row]);
                        }
                    } else if (nv <= 2) {
                        // at most 8 tokens: four contributors' loads in flight at a time
                        for (int64_t c2 = cf; c2 <= cl; c2 += 4) {
                            int4 a[4][2];
#pragma unroll
                            for (int i = 0; i < 4; ++i)
#pragma unroll
                                for (int v = 0; v < 2; ++v)
                                    a[i][v] = (c2 + i <= cl && v < nv) ? __ldcg(part(c2 + i) + v) : make_int4(0, 0, 0, 0);
#pragma unroll
                            for (int i = 0; i < 4; ++i)
#pragma unroll
                                for (int v = 0; v < 2; ++v)
                                    add4(v, a[i][v]);
                        }
                    } else {
                        // two contributors' loads in flight at a time
                        for (int64_t c2 = cf; c2 <= cl; c2 += 2) {
                            int4 a[8], b[8];
                            const bool two = c2 + 1 <= cl;
                            const int4 *pa = part(c2);
                            const int4 *pb = two ? part(c2 + 1) : pa;
#pragma unroll
                            for (int v = 0; v < 8; ++v) {
                                a[v] = v < nv ? __ldcg(pa + v) : make_int4(0, 0, 0, 0);
                                b[v] = (two && v < nv) ? __ldcg(pb + v) : make_int4(0, 0, 0, 0);
                            }
#pragma unroll
                            for (int v = 0; v < 8; ++v) {
                                add4(v, a[v]);
                                add4(v, b[v]);
                            }
                        }
                    }
                    if (n < N)
                        dec_store_chunk<OUT>(r, swn, sx_s, cc * 32, M, y, n, N);
                }
            }
            dec_bar_sync();  // last_flag is rewritten by the next partial tile
        }
    }

    // ---- teardown ------------------------------------------------------------
    if (warp == 1 && lane == 0 && *abort_flag && mma_issued_any) {
        mma_commit(drain_bar);
        bounded_wait(drain_bar, 0, kErrWaitDrain, nullptr, kWaitTimeoutNs / 4);
    }
    if (warp == 0 && lane == 0 && *abort_flag) {
        for (int i = 0; i < stages; ++i)
            if (issued_mask & (1u << i))
                bounded_wait(full_bar(i), (issued_parity >> i) & 1u, kErrWaitDrain, nullptr, kWaitTimeoutNs / 4);
    }
    tc_fence_before_sync();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after_sync();
        tmem_dealloc(tmem_base, Cfg::TMEM_COLS);
    }
}

}  // namespace sq
