// sq_gemm.cuh -- the W8A8 GEMM on the sm_100a tensor cores.
//
//   acc[m, n] = sum_k xq[m, k] * wq[n, k]      (int8 x int8 -> int32, exact)
//   y[m, n]   = ((float)acc[m, n] * sx[m]) * sw[n]
//
// Source: "quant_llm_int8", sections "The architecture: every piece explained"
// and "End-to-end flow" (integer matmul accumulating in int32; dequantisation
// by the outer product of the per-row activation scales and the per-column
// weight scales); "Understanding W8A8 INT8 LLM Quantization", "How the Model
// Was Compressed" (W8A8 runs the matmul on the INT8 tensor cores).
//
// Design (one CTA per SM, persistent over output tiles):
//   warp 0      TMA producer: 2-D tiled loads (128-byte swizzle, no multicast)
//               of a 128 x 128-byte A tile and a BN x 128-byte B tile per stage
//               into a STAGES-deep shared-memory ring (full/empty mbarriers).
//   warp 1      allocates tensor memory and issues tcgen05.mma.kind::i8
//               (M=128, N=BN, K=32 per instruction, 4 per stage) into one of
//               two int32 accumulators in TMEM; tcgen05.commit frees each
//               stage and publishes each finished accumulator.
//   warps 2..5  epilogue: tcgen05.ld of the accumulator (one TMEM lane = one
//               accumulator row per thread), the dequantising multiply, and
//               the store; the second accumulator lets the epilogue of tile i
//               overlap the main loop of tile i+1.
// SWAP = false: A = xq (rows m), B = wq (rows n)       -- large M (prefill)
// SWAP = true:  A = wq (rows n), B = xq (rows m)       -- small M: the weight
//               fills the 128-row MMA side and the few tokens form N = BN.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#include "sq_ptx.cuh"

namespace sq {

enum OutKind { OUT_F32 = 0, OUT_BF16 = 1, OUT_S32 = 2 };

constexpr int kGemmThreads = 192;
constexpr int kBM = 128;  // MMA M (rows of A per tile)
constexpr int kBK = 128;  // bytes of K per stage (one 128-byte swizzle row)

__host__ __device__ constexpr int pow2_at_least(int v, int lo)
{
    int p = lo;
    while (p < v)
        p <<= 1;
    return p;
}

template <int BN, int STAGES>
struct GemmCfg {
    static constexpr int A_BYTES = kBM * kBK;
    static constexpr int B_BYTES = BN * kBK;
    static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
    static constexpr int TMEM_COLS = pow2_at_least(2 * BN, 32);
    static constexpr int NUM_BARS = 2 * STAGES + 5;  // full, empty, tfull[2], tempty[2], drain
    static constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + NUM_BARS * 8 + 16;
    static_assert(BN % 32 == 0 && BN >= 32 && BN <= 256, "MMA N (the epilogue reads 32 columns at a time)");
    static_assert(B_BYTES % 1024 == 0, "stage alignment");
    static_assert(TMEM_COLS <= 512, "TMEM");
};

// Dequantise and store 32 accumulator columns of one accumulator row
// (non-swapped: row m, columns n0..n0+31, contiguous in y).
template <int OUT>
__device__ __forceinline__ void store_row_chunk(const uint32_t (&r)[32], float sxm,
                                                const float *__restrict__ sw, int n0, int N,
                                                void *__restrict__ y, int64_t m)
{
    const int valid = min(32, N - n0);  // 32 or 16 (N % 16 == 0)
    if constexpr (OUT == OUT_S32) {
        uint4 *dst = reinterpret_cast<uint4 *>(reinterpret_cast<int32_t *>(y) + m * N + n0);
#pragma unroll
        for (int v = 0; v < 8; ++v)
            if (v * 4 < valid)
                dst[v] = make_uint4(r[4 * v], r[4 * v + 1], r[4 * v + 2], r[4 * v + 3]);
    } else {
        float w[32];
        const float4 *sw4 = reinterpret_cast<const float4 *>(sw + n0);
#pragma unroll
        for (int v = 0; v < 8; ++v) {
            float4 t = (v * 4 < valid) ? __ldg(sw4 + v) : make_float4(0.f, 0.f, 0.f, 0.f);
            w[4 * v] = t.x;
            w[4 * v + 1] = t.y;
            w[4 * v + 2] = t.z;
            w[4 * v + 3] = t.w;
        }
        float o[32];
#pragma unroll
        for (int j = 0; j < 32; ++j)
            o[j] = __fmul_rn(__fmul_rn(__int2float_rn(static_cast<int>(r[j])), sxm), w[j]);
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
            uint4 *dst =
                reinterpret_cast<uint4 *>(reinterpret_cast<__nv_bfloat16 *>(y) + m * N + n0);
#pragma unroll
            for (int v = 0; v < 4; ++v)
                if (v * 8 < valid)
                    dst[v] = make_uint4(p[4 * v], p[4 * v + 1], p[4 * v + 2], p[4 * v + 3]);
        }
    }
}

// Dequantise and store 32 accumulator columns of one accumulator row in the
// swapped orientation: the row is output channel n, the columns are tokens
// m0..m0+31 (strided by N in y; lanes of a warp hold consecutive n, so each
// store instruction of the warp is contiguous).
template <int OUT>
__device__ __forceinline__ void store_col_chunk(const uint32_t (&r)[32], float swn,
                                                const float *__restrict__ sx, int m0, int M,
                                                void *__restrict__ y, int64_t n, int N)
{
    const int valid = min(32, M - m0);
#pragma unroll
    for (int j = 0; j < 32; ++j) {
        if (j < valid) {
            const int64_t idx = static_cast<int64_t>(m0 + j) * N + n;
            if constexpr (OUT == OUT_S32) {
                reinterpret_cast<int32_t *>(y)[idx] = static_cast<int32_t>(r[j]);
            } else {
                const float sxm = __ldg(sx + m0 + j);
                const float o =
                    __fmul_rn(__fmul_rn(__int2float_rn(static_cast<int>(r[j])), sxm), swn);
                if constexpr (OUT == OUT_F32)
                    reinterpret_cast<float *>(y)[idx] = o;
                else
                    reinterpret_cast<__nv_bfloat16 *>(y)[idx] = __float2bfloat16_rn(o);
            }
        }
    }
}

template <int BN, int STAGES, int OUT, bool SWAP>
__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_i8_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const float *__restrict__ sx, const float *__restrict__ sw,
                   void *__restrict__ y, int M, int N, int K)
{
    // the tensor maps are this launch's own parameters: fetched before the
    // wait for the grid before
    if (threadIdx.x == 0) {
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
    }
    pdl_prologue();
    using Cfg = GemmCfg<BN, STAGES>;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t *gbase = smem_raw + (base - raw);
    const uint32_t sA = base;
    const uint32_t sB = base + STAGES * Cfg::A_BYTES;
    const uint32_t sBar = sB + STAGES * Cfg::B_BYTES;
    auto full_bar = [&](int s) { return sBar + 8u * s; };
    auto empty_bar = [&](int s) { return sBar + 8u * (STAGES + s); };
    auto tfull_bar = [&](int b) { return sBar + 8u * (2 * STAGES + b); };
    auto tempty_bar = [&](int b) { return sBar + 8u * (2 * STAGES + 2 + b); };
    const uint32_t drain_bar = sBar + 8u * (2 * STAGES + 4);
    const uint32_t slot_off = (sBar - base) + 8u * Cfg::NUM_BARS;
    volatile uint32_t *tmem_slot = reinterpret_cast<volatile uint32_t *>(gbase + slot_off);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(gbase + slot_off + 4);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(full_bar(s), 1);
            mbar_init(empty_bar(s), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(tfull_bar(b), 1);
            mbar_init(tempty_bar(b), 4);
        }
        mbar_init(drain_bar, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(const_cast<uint32_t *>(tmem_slot)), Cfg::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem_base = *tmem_slot;

    const int rows_a = SWAP ? N : M;
    const int rows_b = SWAP ? M : N;
    const int a_tiles = (rows_a + kBM - 1) / kBM;
    const int b_tiles = (rows_b + BN - 1) / BN;
    const int total = a_tiles * b_tiles;
    const int k_blocks = (K + kBK - 1) / kBK;

    uint32_t issued_mask = 0, issued_parity = 0;  // producer bookkeeping for the abort drain
    bool mma_issued_any = false;

    if (warp == 0) {
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            for (int t = blockIdx.x; t < total; t += gridDim.x) {
                const int a_blk = t % a_tiles, b_blk = t / a_tiles;
                for (int kb = 0; kb < k_blocks; ++kb) {
                    if (!bounded_wait(empty_bar(stage), phase ^ 1u, kErrWaitProducer, abort_flag))
                        goto producer_done;
                    mbar_arrive_expect_tx(full_bar(stage), Cfg::STAGE_BYTES);
                    tma_load_2d(sA + stage * Cfg::A_BYTES, &tmA, full_bar(stage), kb * kBK,
                                a_blk * kBM);
                    tma_load_2d(sB + stage * Cfg::B_BYTES, &tmB, full_bar(stage), kb * kBK,
                                b_blk * BN);
                    issued_mask |= 1u << stage;
                    issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
        producer_done:;
        }
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_i8(kBM, BN);
            int stage = 0;
            uint32_t phase = 0;
            int acc = 0;
            uint32_t acc_phase = 0;
            for (int t = blockIdx.x; t < total; t += gridDim.x) {
                if (!bounded_wait(tempty_bar(acc), acc_phase ^ 1u, kErrWaitAccEmpty, abort_flag))
                    break;
                tc_fence_after_sync();
                const uint32_t d = tmem_base + static_cast<uint32_t>(acc * BN);
                bool ok = true;
                for (int kb = 0; kb < k_blocks; ++kb) {
                    if (!bounded_wait(full_bar(stage), phase, kErrWaitMma, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after_sync();
                    const uint32_t a0 = sA + stage * Cfg::A_BYTES;
                    const uint32_t b0 = sB + stage * Cfg::B_BYTES;
#pragma unroll
                    for (int k = 0; k < kBK / 32; ++k)
                        mma_i8(d, smem_desc_k_sw128(a0 + 32 * k), smem_desc_k_sw128(b0 + 32 * k),
                               idesc, (kb | k) != 0 ? 1u : 0u);
                    mma_issued_any = true;
                    mma_commit(empty_bar(stage));
                    if (++stage == STAGES) {
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
        // epilogue warps 2..5; warp w may read TMEM lanes 32*(w%4) .. +31
        const int quarter = warp & 3;
        const int row = quarter * 32 + lane;
        int acc = 0;
        uint32_t acc_phase = 0;
        for (int t = blockIdx.x; t < total; t += gridDim.x) {
            const int a_blk = t % a_tiles, b_blk = t / a_tiles;
            const bool ok = bounded_wait(tfull_bar(acc), acc_phase, kErrWaitAccFull, abort_flag);
            if (!__all_sync(0xFFFFFFFFu, ok))
                break;
            tc_fence_after_sync();
            const int64_t arow = static_cast<int64_t>(a_blk) * kBM + row;
            const uint32_t tbase =
                tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + static_cast<uint32_t>(acc * BN);
            if constexpr (!SWAP) {
                const float sxm = (arow < M && OUT != OUT_S32) ? __ldg(sx + arow) : 0.0f;
#pragma unroll 1
                for (int c = 0; c < BN / 32; ++c) {
                    const int n0 = b_blk * BN + c * 32;
                    if (n0 >= N)
                        break;
                    uint32_t r[32];
                    tmem_ld_32x32b_x32(tbase + c * 32, r);
                    tmem_ld_wait();
                    if (arow < M)
                        store_row_chunk<OUT>(r, sxm, sw, n0, N, y, arow);
                    __syncwarp();
                }
            } else {
                const float swn = (arow < N && OUT != OUT_S32) ? __ldg(sw + arow) : 0.0f;
#pragma unroll 1
                for (int c = 0; c < BN / 32; ++c) {
                    const int m0 = b_blk * BN + c * 32;
                    if (m0 >= M)
                        break;
                    uint32_t r[32];
                    tmem_ld_32x32b_x32(tbase + c * 32, r);
                    tmem_ld_wait();
                    if (arow < N)
                        store_col_chunk<OUT>(r, swn, sx, m0, M, y, arow, N);
                    __syncwarp();
                }
            }
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(tempty_bar(acc));
            acc ^= 1;
            if (acc == 0)
                acc_phase ^= 1u;
        }
    }

    // ---- teardown ----------------------------------------------------------
    if (warp == 1 && lane == 0 && *abort_flag && mma_issued_any) {
        // let every MMA this CTA issued finish before TMEM is released
        mma_commit(drain_bar);
        bounded_wait(drain_bar, 0, kErrWaitDrain, nullptr, kWaitTimeoutNs / 4);
    }
    if (warp == 0 && lane == 0 && *abort_flag) {
        // wait for TMA copies still in flight into this CTA's shared memory
        for (int s = 0; s < STAGES; ++s)
            if (issued_mask & (1u << s))
                bounded_wait(full_bar(s), (issued_parity >> s) & 1u, kErrWaitDrain, nullptr,
                             kWaitTimeoutNs / 4);
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
