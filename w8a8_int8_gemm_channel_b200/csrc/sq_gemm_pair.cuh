// sq_gemm_pair.cuh -- the prefill W8A8 GEMM on CTA pairs (tcgen05 cta_group::2).
//
//   acc[m, n] = sum_k xq[m, k] * wq[n, k]      (int8 x int8 -> int32, exact)
//   y[m, n]   = ((float)acc[m, n] * sx[m]) * sw[n]
//
// Source: "quant_llm_int8", sections "The architecture: every piece explained"
// and "End-to-end flow" (integer matmul accumulating in int32, dequantisation
// by the outer product of the per-row and per-column scales).
//
// An output tile is 256 rows (tokens) x BN columns (output channels) and is
// computed by the two CTAs of a cluster pair, one per SM:
//   * CTA r of the pair loads A rows [m0 + 128 r, +128) and B rows
//     [n0 + r BN/2, +BN/2) into its own shared memory (plain TMA, no
//     multicast); the completion bytes of both CTAs' loads land on the stage's
//     barrier in the first CTA;
//   * the first CTA issues tcgen05.mma.cta_group::2 (M = 256, N = BN, K = 32),
//     which reads both CTAs' halves and accumulates 128 rows in each CTA's
//     TMEM; its commits free the stage in both CTAs and publish the
//     accumulator to both epilogues;
//   * both CTAs' epilogues read their own 128 accumulator rows and store them;
//     all eight epilogue warps release the accumulator on the first CTA's
//     barrier.
// Per SM and 128-byte k block this moves 16 KB of A and BN/2 x 128 bytes of B
// for 128 x BN outputs: with BN = 256 a third less operand traffic from L2
// per operation than a 128 x 256 tile on one SM.  Two accumulators in TMEM
// let the epilogue of one tile overlap the main loop of the next.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#include "sq_decode.cuh"
#include "sq_gemm.cuh"
#include "sq_ptx.cuh"

namespace sq {

constexpr int kPairThreads = 192;
constexpr int kPairBM = 256;  // rows of an output tile (128 per CTA)

template <int BN, int STAGES>
struct PairCfg {
    static constexpr int A_BYTES = 128 * kBK;       // this CTA's 128 rows of A
    static constexpr int B_BYTES = (BN / 2) * kBK;  // this CTA's BN/2 rows of B
    static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
    static constexpr int TMEM_COLS = pow2_at_least(2 * BN, 32);
    static constexpr int NUM_BARS = 2 * STAGES + 5;  // full, empty, tfull[2], tempty[2], drain
    static constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + NUM_BARS * 8 + 16;
    static_assert(BN % 32 == 0 && BN >= 64 && BN <= 256, "MMA N (multiple of 32 for the epilogue)");
    static_assert(B_BYTES % 1024 == 0, "stage alignment (8-row swizzle atoms)");
    static_assert(TMEM_COLS <= 512, "TMEM");
    static_assert(SMEM_BYTES <= 232448, "shared memory");
};

// The work of one pair: its data-parallel tiles t = pair, pair + pairs, ...
// below sk_first, then its contiguous range of the stream-K units (one unit
// = one 128-byte k block of one tile; the sk_units units of tiles sk_first,
// sk_first + 1, ... are cut into `pairs` equal ranges, as in sq_decode.cuh).
struct PairSeg {
    int tile, kb0, kb1;
    bool whole;
};

struct PairSched {
    int pair, pairs, sk_first, KB;
    int64_t U, u0, u1;  // stream-K units and this pair's range
    int t;
    int64_t u;
    __device__ __forceinline__ PairSched(int pair_, int pairs_, int sk_first_, int KB_, int64_t U_)
        : pair(pair_), pairs(pairs_), sk_first(sk_first_), KB(KB_), U(U_), u0(dec_start(pair_, U_, pairs_)),
          u1(dec_start(pair_ + 1, U_, pairs_)), t(pair_), u(u0)
    {
    }
    __device__ __forceinline__ bool next(PairSeg &s)
    {
        if (t < sk_first) {
            s.tile = t;
            s.kb0 = 0;
            s.kb1 = KB;
            s.whole = true;
            t += pairs;
            return true;
        }
        if (u < u1) {
            const int64_t j = u / KB;
            s.tile = sk_first + static_cast<int>(j);
            s.kb0 = static_cast<int>(u - j * KB);
            s.kb1 = static_cast<int>(min(static_cast<int64_t>(KB), s.kb0 + (u1 - u)));
            s.whole = s.kb0 == 0 && s.kb1 == KB;
            u += s.kb1 - s.kb0;
            return true;
        }
        return false;
    }
    // first stream-K tile of this pair's range (its partial slot 0)
    __device__ __forceinline__ int first_sk_tile() const { return sk_first + static_cast<int>(u0 / KB); }
};

// Output tile t of the pair kernel -> (m block, n block).  Tiles go in
// groups of up to group_m m blocks: within a group the m block varies
// fastest, then the n block, and groups follow in m (group_m >= m_tiles: m
// fastest throughout).  With groups of 8, the 74 pairs that work at the same
// time touch about 8 + 10 tiles' k slices at M = 8192 instead of 32 + 3, so
// more of each slice comes from L2: measured on B200, DRAM reads of 8192 x
// 8192 x 28672 fell from 3.8 to 2.1 GB and its time by 5%, while 8192 x
// 57344 x 8192 (DRAM reads 3.7 -> 2.8 GB) became 1.7% slower; the launcher
// groups long-K shapes only.
__device__ __forceinline__ void pair_tile_mn(int t, int m_tiles, int n_tiles, int group_m, int &m_blk, int &n_blk)
{
    const int per_group = group_m * n_tiles;
    const int g = t / per_group;
    const int r = t - g * per_group;
    const int gm = min(group_m, m_tiles - g * group_m);  // m blocks in this group
    m_blk = g * group_m + r % gm;
    n_blk = r / gm;
}

// Partial-sum slot of CTA `cta` (blockIdx.x) of the pair kernel: ws holds
// 2 slots per CTA of 128 rows x BN int32, column-chunk-major (32 columns of
// 128 rows, the rows contiguous).
__device__ __forceinline__ int32_t *pair_slot(int32_t *ws, int64_t cta, int slot, int BN)
{
    return ws + (cta * 2 + slot) * static_cast<int64_t>(BN) * 128;
}

template <int BN, int STAGES, int OUT>
__global__ void __launch_bounds__(kPairThreads, 1)
    gemm_i8_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                        const float *__restrict__ sx, const float *__restrict__ sw, void *__restrict__ y,
                        int M, int N, int K, int sk_first, int64_t sk_units, int32_t *__restrict__ ws,
                        int *__restrict__ cnt, int group_m)
{
    // the tensor maps are this launch's own parameters: fetched before the
    // wait for the grid before
    if (threadIdx.x == 0) {
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
    }
    pdl_prologue();
    using Cfg = PairCfg<BN, STAGES>;
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
    volatile int *last_flag = reinterpret_cast<volatile int *>(gbase + slot_off + 8);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();  // 0: the pair's first CTA (issues the MMAs)
    const int pair = static_cast<int>(blockIdx.x >> 1);
    const int pairs = static_cast<int>(gridDim.x >> 1);

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(full_bar(s), 1);
            mbar_init(empty_bar(s), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(tfull_bar(b), 1);
            mbar_init(tempty_bar(b), 8);  // 4 epilogue warps in each CTA
        }
        mbar_init(drain_bar, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc_pair(smem_u32(const_cast<uint32_t *>(tmem_slot)), Cfg::TMEM_COLS);
        tmem_relinquish_pair();
    }
    tc_fence_before_sync();
    __syncthreads();
    cluster_arrive();  // both CTAs' barriers and TMEM exist before any cross-CTA use
    cluster_wait();
    tc_fence_after_sync();
    const uint32_t tmem_base = *tmem_slot;

    const int m_tiles = (M + kPairBM - 1) / kPairBM;
    const int n_tiles = (N + BN - 1) / BN;
    const int k_blocks = (K + kBK - 1) / kBK;

    uint32_t issued_mask = 0, issued_parity = 0;  // producer: last phase issued per stage
    bool mma_issued_any = false;

    if (warp == 0) {
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            PairSched sch(pair, pairs, sk_first, k_blocks, sk_units);
            PairSeg sg;
            while (sch.next(sg)) {
                int m_blk, n_blk;
                pair_tile_mn(sg.tile, m_tiles, n_tiles, group_m, m_blk, n_blk);
                const int a_row = m_blk * kPairBM + static_cast<int>(rank) * 128;
                const int b_row = n_blk * BN + static_cast<int>(rank) * (BN / 2);
                for (int kb = sg.kb0; kb < sg.kb1; ++kb) {
                    if (!bounded_wait(empty_bar(stage), phase ^ 1u, kErrWaitProducer, abort_flag))
                        goto producer_done;
                    if (rank == 0)
                        mbar_arrive_expect_tx(full_bar(stage), 2u * Cfg::STAGE_BYTES);
                    const uint32_t fb = map_shared_rank(full_bar(stage), 0);
                    tma_load_2d_pair(sA + stage * Cfg::A_BYTES, &tmA, fb, kb * kBK, a_row);
                    tma_load_2d_pair(sB + stage * Cfg::B_BYTES, &tmB, fb, kb * kBK, b_row);
                    issued_mask |= 1u << stage;
                    issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            // every commit that frees a stage of this CTA has arrived before
            // the CTA may leave (they are multicast from the first CTA)
            for (int s = 0; s < STAGES; ++s)
                if (issued_mask & (1u << s))
                    if (!bounded_wait(empty_bar(s), (issued_parity >> s) & 1u, kErrWaitDrain, abort_flag))
                        break;
        producer_done:;
        }
    } else if (warp == 1) {
        if (lane == 0 && rank == 0) {
            constexpr uint32_t idesc = idesc_i8(kPairBM, BN);
            int stage = 0;
            uint32_t phase = 0;
            int acc = 0;
            uint32_t acc_phase = 0;
            PairSched sch(pair, pairs, sk_first, k_blocks, sk_units);
            PairSeg sg;
            while (sch.next(sg)) {
                if (!bounded_wait_cluster(tempty_bar(acc), acc_phase ^ 1u, kErrWaitAccEmpty, abort_flag))
                    break;
                tc_fence_after_sync();
                const uint32_t d = tmem_base + static_cast<uint32_t>(acc * BN);
                bool ok = true;
                for (int kb = sg.kb0; kb < sg.kb1; ++kb) {
                    if (!bounded_wait(full_bar(stage), phase, kErrWaitMma, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after_sync();
                    const uint32_t a0 = sA + stage * Cfg::A_BYTES;
                    const uint32_t b0 = sB + stage * Cfg::B_BYTES;
#pragma unroll
                    for (int k = 0; k < kBK / 32; ++k)
                        mma_i8_pair(d, smem_desc_k_sw128(a0 + 32 * k), smem_desc_k_sw128(b0 + 32 * k), idesc,
                                    (kb > sg.kb0 || k != 0) ? 1u : 0u);
                    mma_issued_any = true;
                    mma_commit_pair(empty_bar(stage), 0x3);
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok)
                    break;
                mma_commit_pair(tfull_bar(acc), 0x3);
                acc ^= 1;
                if (acc == 0)
                    acc_phase ^= 1u;
            }
        }
    } else {
        // epilogue warps 2..5: warp w reads TMEM lanes 32 (w % 4) .. +31
        const int quarter = warp & 3;
        const int row = quarter * 32 + lane;
        const int et = threadIdx.x - 64;  // 0..127
        const uint32_t tempty_first = map_shared_rank(tempty_bar(0), 0);
        int acc = 0;
        uint32_t acc_phase = 0;
        PairSched sch(pair, pairs, sk_first, k_blocks, sk_units);
        const int first_sk = sch.first_sk_tile();
        PairSeg sg;
        while (sch.next(sg)) {
            int m_blk, n_blk;
            pair_tile_mn(sg.tile, m_tiles, n_tiles, group_m, m_blk, n_blk);
            const bool ok = bounded_wait(tfull_bar(acc), acc_phase, kErrWaitAccFull, abort_flag);
            if (!__all_sync(0xFFFFFFFFu, ok))
                break;
            tc_fence_after_sync();
            const int64_t m = static_cast<int64_t>(m_blk) * kPairBM + rank * 128 + row;
            const uint32_t tbase =
                tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + static_cast<uint32_t>(acc * BN);
            const float sxm = (m < M && OUT != OUT_S32) ? __ldg(sx + m) : 0.0f;
            int32_t *mine = sg.whole ? nullptr : pair_slot(ws, blockIdx.x, sg.tile == first_sk ? 0 : 1, BN);
#pragma unroll 1
            for (int c = 0; c < BN / 32; ++c) {
                const int n0 = n_blk * BN + c * 32;
                if (n0 >= N)
                    break;
                uint32_t r[32];
                tmem_ld_32x32b_x32(tbase + c * 32, r);
                tmem_ld_wait();
                if (sg.whole) {
                    if (m < M)
                        store_row_chunk<OUT>(r, sxm, sw, n0, N, y, m);
                } else {
#pragma unroll
                    for (int j = 0; j < 32; ++j)
                        mine[(c * 32 + j) * 128 + row] = static_cast<int32_t>(r[j]);
                }
                __syncwarp();
            }
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0)
                mbar_arrive_remote_release(tempty_first + 8u * acc);
            acc ^= 1;
            if (acc == 0)
                acc_phase ^= 1u;
            if (sg.whole)
                continue;
            // this CTA's half of a tile shared by several pairs: count the
            // partial in; the pair that completes the count adds every
            // contributor's slot (same half) and stores the tile half
            const int64_t ut = static_cast<int64_t>(sg.tile - sk_first) * k_blocks;
            const int64_t pf = dec_owner(ut, sk_units, pairs), pl = dec_owner(ut + k_blocks - 1, sk_units, pairs);
            __threadfence();
            asm volatile("bar.sync 2, 128;" ::: "memory");
            if (et == 0) {
                const int old = atomicAdd(cnt + 2 * (sg.tile - sk_first) + static_cast<int>(rank), 1);
                *last_flag = old == static_cast<int>(pl - pf);
            }
            asm volatile("bar.sync 2, 128;" ::: "memory");
            if (*last_flag) {
                __threadfence();
#pragma unroll 1
                for (int c = 0; c < BN / 32; ++c) {
                    const int n0 = n_blk * BN + c * 32;
                    if (n0 >= N)
                        break;
                    uint32_t r[32];
#pragma unroll
                    for (int j = 0; j < 32; ++j)
                        r[j] = 0u;
                    for (int64_t p2 = pf; p2 <= pl; ++p2) {
                        const int s2 = (sk_first + static_cast<int>(dec_start(p2, sk_units, pairs) / k_blocks) ==
                                        sg.tile)
                                           ? 0
                                           : 1;
                        const int32_t *src = pair_slot(ws, 2 * p2 + rank, s2, BN) + (c * 32) * 128 + row;
#pragma unroll
                        for (int j = 0; j < 32; ++j)
                            r[j] += static_cast<uint32_t>(__ldcg(src + j * 128));
                    }
                    if (m < M)
                        store_row_chunk<OUT>(r, sxm, sw, n0, N, y, m);
                }
            }
            asm volatile("bar.sync 2, 128;" ::: "memory");  // last_flag is rewritten by the next partial tile
        }
    }

    // ---- teardown ----------------------------------------------------------
    if (warp == 1 && lane == 0 && rank == 0 && *abort_flag && mma_issued_any) {
        // every MMA of the pair finishes before either CTA releases TMEM
        mma_commit_pair_local(drain_bar);
        bounded_wait(drain_bar, 0, kErrWaitDrain, nullptr, kWaitTimeoutNs / 4);
    }
    if (warp == 0 && lane == 0 && rank == 0 && *abort_flag) {
        // copies still in flight complete on the first CTA's full barriers
        for (int s = 0; s < STAGES; ++s)
            if (issued_mask & (1u << s))
                bounded_wait(full_bar(s), (issued_parity >> s) & 1u, kErrWaitDrain, nullptr, kWaitTimeoutNs / 4);
    }
    tc_fence_before_sync();
    __syncthreads();
    cluster_arrive();  // neither CTA leaves while the other may still touch its memory
    cluster_wait();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after_sync();
        tmem_dealloc_pair(tmem_base, Cfg::TMEM_COLS);
    }
}

}  // namespace sq
