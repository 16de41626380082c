// sq_slab.cuh -- the W8A8 GEMM for at most 32 tokens: every CTA owns a slab of
// whole output channels over the full K, so no partial sum crosses CTAs.
//
//   acc[m, n] = sum_k xq[m, k] * wq[n, k]     y[m, n] = ((float)acc * sx[m]) * sw[n]
//
// Sources: "quant_llm_int8", "The architecture: every piece explained" (int32
// accumulation, outer-product dequantisation); "Understanding W8A8 INT8 LLM
// Quantization", "Inter-Token Latency (ITL)" (at decode the layer streams its
// weight: the time is the weight's bytes over the memory bandwidth).
//
// Work.  The N output channels are cut into R = N / 16 groups of 16; CTA c of
// G takes groups [c R / G, (c + 1) R / G): a slab of nt = 16 * (floor or ceil
// of R / G) channels, and all of K.  Every SM streams a slab of the weight
// once; the token codes (M x K bytes, a few hundred KB at most) are read by
// every CTA and come from L2.  Nothing is reduced across CTAs, so there is no
// workspace and no second pass: the CTA that accumulates a slab stores it.
//
// The MMA.  tcgen05.mma.kind::i8 with M = 128 (the tokens), N = nt (the slab),
// K = 32.  Only BNX rows of each 128-row token tile are loaded (BNX = 8, 16
// or 32, M <= BNX; TMA fills rows past M with zeros); the other rows of the
// operand read whatever shared memory follows the tile -- inside this CTA's
// allocation by construction -- and only reach accumulator lanes >= BNX,
// which nothing reads.  A slab accumulates over NACC rotating accumulators
// (consecutive MMAs write different TMEM columns), summed exactly by the
// epilogue.
//
// Overlap with the quantiser.  As for the weight-streaming kernel: when the
// grid before is the library's own quantiser (pre_wait = 1), the weight
// loads of the first stages are issued before griddepcontrol.wait, and only
// the token codes wait for it.
//
// Roles (192 threads):
//   warp 0      TMA producer: per 128-byte k block an nt x 128-byte weight
//               tile and a BNX x 128-byte tile of the codes, 128-byte swizzle,
//               no multicast
//   warp 1      TMEM allocation, the MMAs
//   warps 2..5  epilogue: warp w reads TMEM lanes 32 (w % 4) .. +31, i.e.
//               tokens; a warp with no token < M skips
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#include "sq_gemm.cuh"
#include "sq_ptx.cuh"

namespace sq {

constexpr int kSlabThreads = 192;
constexpr int kSlabMaxNt = 256;       // widest slab: one MMA's N
constexpr int kSlabTmemCols = 512;    // NACC x column stride, always the whole TMEM

// accumulators a slab rotates over, and their column stride
__host__ __device__ constexpr int slab_nacc(int nt) { return nt <= 128 ? 4 : 2; }
__host__ __device__ constexpr int slab_col_stride(int nt) { return nt <= 128 ? 128 : 256; }

// Shared-memory layout (offsets from the 1024-aligned base): the code tiles
// of every stage and k block, then the weight tiles, then the barriers (full
// and empty per stage, tfull, drain), the TMEM slot and the abort flag, then
// the slab's weight scales (nt_max floats).  The MMA reads 128 rows of a code
// tile; rows past BNX lie in the memory after it, which the layout keeps
// inside the allocation.
struct SlabLayout {
    uint32_t w_off, bar_off, sw_off, total;
};

__host__ __device__ constexpr SlabLayout slab_layout(int bnx, int nt_max, int stages, int kbs)
{
    const uint32_t xr = static_cast<uint32_t>(stages * kbs * bnx * kBK);
    const uint32_t wr = static_cast<uint32_t>(stages * kbs * nt_max * kBK);
    const uint32_t footprint = xr - static_cast<uint32_t>(bnx * kBK) + static_cast<uint32_t>(kBM * kBK);
    const uint32_t end = (xr + wr > footprint ? xr + wr : footprint);
    const uint32_t bar = (end + 7u) & ~7u;
    const uint32_t swo = (bar + static_cast<uint32_t>(2 * stages + 2) * 8u + 16u + 15u) & ~15u;
    return SlabLayout{xr, bar, swo, swo + static_cast<uint32_t>(nt_max) * 4u};
}

// 1024 bytes of alignment slack on top of the layout
__host__ __device__ constexpr int slab_smem_bytes(int bnx, int nt_max, int stages, int kbs)
{
    return 1024 + static_cast<int>(slab_layout(bnx, nt_max, stages, kbs).total);
}

// Dequantise and store `valid` (<= 32, a multiple of 16) accumulator columns
// of token m: channels n0 .. n0 + valid - 1, contiguous in y's row m.  sw_s
// points at the shared-memory copy of sw[n0 .. n0 + valid - 1].
template <int OUT>
__device__ __forceinline__ void slab_store(const uint32_t (&r)[32], float sxm, const float *sw_s, int n0,
                                           int valid, int N, void *__restrict__ y, int64_t m)
{
    if constexpr (OUT == OUT_S32) {
        uint4 *dst = reinterpret_cast<uint4 *>(reinterpret_cast<int32_t *>(y) + m * N + n0);
#pragma unroll
        for (int v = 0; v < 8; ++v)
            if (v * 4 < valid)
                dst[v] = make_uint4(r[4 * v], r[4 * v + 1], r[4 * v + 2], r[4 * v + 3]);
    } else {
        float o[32];
        const float4 *sw4 = reinterpret_cast<const float4 *>(sw_s);
#pragma unroll
        for (int v = 0; v < 8; ++v) {
            const float4 t = (v * 4 < valid) ? sw4[v] : make_float4(0.f, 0.f, 0.f, 0.f);
            o[4 * v] = __fmul_rn(__fmul_rn(__int2float_rn(static_cast<int>(r[4 * v])), sxm), t.x);
            o[4 * v + 1] = __fmul_rn(__fmul_rn(__int2float_rn(static_cast<int>(r[4 * v + 1])), sxm), t.y);
            o[4 * v + 2] = __fmul_rn(__fmul_rn(__int2float_rn(static_cast<int>(r[4 * v + 2])), sxm), t.z);
            o[4 * v + 3] = __fmul_rn(__fmul_rn(__int2float_rn(static_cast<int>(r[4 * v + 3])), sxm), t.w);
        }
        if constexpr (OUT == OUT_F32) {
            uint4 *dst = reinterpret_cast<uint4 *>(reinterpret_cast<float *>(y) + m * N + n0);
#pragma unroll
            for (int v = 0; v < 8; ++v)
                if (v * 4 < valid)
                    dst[v] = make_uint4(__float_as_uint(o[4 * v]), __float_as_uint(o[4 * v + 1]),
                                        __float_as_uint(o[4 * v + 2]), __float_as_uint(o[4 * v + 3]));
        } else {
            uint32_t p[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                __nv_bfloat162 h = __floats2bfloat162_rn(o[2 * j], o[2 * j + 1]);
                p[j] = *reinterpret_cast<uint32_t *>(&h);
            }
            uint4 *dst = reinterpret_cast<uint4 *>(reinterpret_cast<__nv_bfloat16 *>(y) + m * N + n0);
#pragma unroll
            for (int v = 0; v < 4; ++v)
                if (v * 8 < valid)
                    dst[v] = make_uint4(p[4 * v], p[4 * v + 1], p[4 * v + 2], p[4 * v + 3]);
        }
    }
}

// tmW_lo / tmW_hi: the weight with boxes of nt_lo / nt_hi rows (the two slab
// widths); tmX: the codes, boxes of BNX rows.  kbs k blocks a stage.
template <int BNX, int OUT>
__global__ void __launch_bounds__(kSlabThreads, 1)
    gemm_slab_kernel(const __grid_constant__ CUtensorMap tmW_lo, const __grid_constant__ CUtensorMap tmW_hi,
                     const __grid_constant__ CUtensorMap tmX, const float *__restrict__ sx,
                     const float *__restrict__ sw, void *__restrict__ y, int M, int N, int K, int G, int nt_hi,
                     int stages, int kbs, int pre_wait)
{
    static_assert(BNX == 8 || BNX == 16 || BNX == 32, "token tile");
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const bool producer = warp == 0 && lane == 0;

    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t *gb = smem_raw + (base - raw);
    const SlabLayout L = slab_layout(BNX, nt_hi, stages, kbs);
    const uint32_t sX = base, sW = base + L.w_off;
    const uint32_t bars = base + L.bar_off;
    auto full_bar = [&](int i) { return bars + 8u * i; };
    auto empty_bar = [&](int i) { return bars + 8u * (stages + i); };
    const uint32_t tfull_bar = bars + 8u * (2 * stages);
    const uint32_t drain_bar = bars + 8u * (2 * stages + 1);
    volatile uint32_t *tmem_slot = reinterpret_cast<volatile uint32_t *>(gb + L.bar_off + 8u * (2 * stages + 2));
    volatile int *abort_flag = reinterpret_cast<volatile int *>(gb + L.bar_off + 8u * (2 * stages + 2) + 4u);

    // this CTA's slab: channels n0 .. n0 + nt - 1
    const int R = N / 16;
    const int g0 = static_cast<int>(static_cast<int64_t>(blockIdx.x) * R / G);
    const int g1 = static_cast<int>(static_cast<int64_t>(blockIdx.x + 1) * R / G);
    const int n0 = 16 * g0, nt = 16 * (g1 - g0);
    const CUtensorMap *tmW = nt == nt_hi ? &tmW_hi : &tmW_lo;
    const int nacc = slab_nacc(nt), cstride = slab_col_stride(nt);
    const int KB = (K + kBK - 1) / kBK;
    const int nsteps = (KB + kbs - 1) / kbs;
    const uint32_t x_tile = static_cast<uint32_t>(BNX * kBK), w_tile = static_cast<uint32_t>(nt_hi * kBK);
    auto x_addr = [&](int stage, int kk) { return sX + static_cast<uint32_t>(stage * kbs + kk) * x_tile; };
    auto w_addr = [&](int stage, int kk) { return sW + static_cast<uint32_t>(stage * kbs + kk) * w_tile; };
    auto step_kbs = [&](int s) { return min(kbs, KB - s * kbs); };
    auto kx = [&](int j) { return j * kBK; };

    if (threadIdx.x == 32) {
        for (int i = 0; i < stages; ++i) {
            mbar_init(full_bar(i), 1);
            mbar_init(empty_bar(i), 1);
        }
        mbar_init(tfull_bar, 1);
        mbar_init(drain_bar, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (producer) {
        // the tensor maps are this launch's own parameters: fetched while
        // the grid before still runs
        tma_prefetch_desc(tmW);
        tma_prefetch_desc(&tmX);
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(const_cast<uint32_t *>(tmem_slot)), kSlabTmemCols);
        tmem_relinquish();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem_base = *tmem_slot;
    // Nothing but the tensor maps has touched global memory yet.  Every thread but the producer
    // waits for the grid before now; the producer first requests weight
    // tiles when that is allowed.
    if (!(producer && (pre_wait & 1)))
        asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

    uint32_t issued_mask = 0, issued_parity = 0;
    bool mma_issued_any = false;

    if (warp == 0) {
        if (lane == 0) {
            const int pre = (pre_wait & 1) ? min(nsteps, stages) : 0;
            for (int s = 0; s < pre; ++s) {
                const int n = step_kbs(s);
                mbar_arrive_expect_tx(full_bar(s), static_cast<uint32_t>(n) * (x_tile + static_cast<uint32_t>(nt) * kBK));
                for (int kk = 0; kk < n; ++kk)
                    tma_load_2d(w_addr(s, kk), tmW, full_bar(s), kx(s * kbs + kk), n0);
                issued_mask |= 1u << s;
            }
            if (pre_wait & 1)
                asm volatile("griddepcontrol.wait;" ::: "memory");
            for (int s = 0; s < pre; ++s)
                for (int kk = 0; kk < step_kbs(s); ++kk)
                    tma_load_2d(x_addr(s, kk), &tmX, full_bar(s), kx(s * kbs + kk), 0);
            int stage = pre % stages;
            uint32_t phase = (pre == stages) ? 1u : 0u;
            for (int s = pre; s < nsteps; ++s) {
                if (!bounded_wait(empty_bar(stage), phase ^ 1u, kErrWaitProducer, abort_flag))
                    break;
                const int n = step_kbs(s);
                mbar_arrive_expect_tx(full_bar(stage),
                                      static_cast<uint32_t>(n) * (x_tile + static_cast<uint32_t>(nt) * kBK));
                for (int kk = 0; kk < n; ++kk) {
                    tma_load_2d(w_addr(stage, kk), tmW, full_bar(stage), kx(s * kbs + kk), n0);
                    tma_load_2d(x_addr(stage, kk), &tmX, full_bar(stage), kx(s * kbs + kk), 0);
                }
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
            const uint32_t idesc = idesc_i8(kBM, nt);
            int stage = 0, step = 0;
            uint32_t phase = 0;
            bool ok = true;
            for (int s = 0; s < nsteps; ++s) {
                if (!bounded_wait(full_bar(stage), phase, kErrWaitMma, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after_sync();
                for (int kk = 0; kk < step_kbs(s); ++kk) {
                    const uint32_t a0 = x_addr(stage, kk), b0 = w_addr(stage, kk);
#pragma unroll
                    for (int k = 0; k < kBK / 32; ++k, ++step)
                        mma_i8(tmem_base + static_cast<uint32_t>((step % nacc) * cstride),
                               smem_desc_k_sw128(a0 + 32 * k), smem_desc_k_sw128(b0 + 32 * k), idesc,
                               step >= nacc ? 1u : 0u);
                }
                mma_issued_any = true;
                mma_commit(empty_bar(stage));
                if (++stage == stages) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
            if (ok)
                mma_commit(tfull_bar);
        }
    } else {
        // epilogue warps 2..5: warp w reads TMEM lanes (tokens) 32 (w % 4) .. +31.
        // While the weight streams they bring the slab's weight scales into
        // shared memory and each token's scale into a register, so that the
        // stores after the last MMA wait for no global load.
        const int quarter = warp & 3;
        const int64_t m = quarter * 32 + lane;
        float *sw_s = reinterpret_cast<float *>(gb + L.sw_off);
        if constexpr (OUT != OUT_S32)
            for (int j = threadIdx.x - 64; j < nt; j += 128)
                sw_s[j] = __ldg(sw + n0 + j);
        const float sxm = (OUT != OUT_S32 && m < M) ? __ldg(sx + m) : 0.0f;
        asm volatile("bar.sync 2, 128;" ::: "memory");  // the four epilogue warps
        const bool ok = bounded_wait(tfull_bar, 0, kErrWaitAccFull, abort_flag);
        if (__all_sync(0xFFFFFFFFu, ok) && quarter * 32 < M) {
            tc_fence_after_sync();
            const uint32_t lane_addr = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16);
            // the accumulators written: every one when there are at least nacc MMAs
            const int nused = min(nacc, KB * (kBK / 32));
#pragma unroll 1
            for (int cb = 0; cb * 32 < nt; ++cb) {
                // two accumulators' loads in flight at a time, summed exactly
                uint32_t r[32], q[32];
                tmem_ld_32x32b_x32(lane_addr + static_cast<uint32_t>(cb * 32), r);
                if (nused > 1)
                    tmem_ld_32x32b_x32(lane_addr + static_cast<uint32_t>(cstride + cb * 32), q);
                tmem_ld_wait();
                if (nused > 1) {
#pragma unroll
                    for (int j = 0; j < 32; ++j)
                        r[j] += q[j];
                }
#pragma unroll 1
                for (int a = 2; a < nused; a += 2) {
                    uint32_t q2[32];
                    tmem_ld_32x32b_x32(lane_addr + static_cast<uint32_t>(a * cstride + cb * 32), q);
                    if (a + 1 < nused)
                        tmem_ld_32x32b_x32(lane_addr + static_cast<uint32_t>((a + 1) * cstride + cb * 32), q2);
                    tmem_ld_wait();
#pragma unroll
                    for (int j = 0; j < 32; ++j)
                        r[j] += q[j] + (a + 1 < nused ? q2[j] : 0u);
                }
                if (m < M)
                    slab_store<OUT>(r, sxm, sw_s + cb * 32, n0 + cb * 32, min(32, nt - cb * 32), N, y, m);
            }
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
        tmem_dealloc(tmem_base, kSlabTmemCols);
    }
}

}  // namespace sq
