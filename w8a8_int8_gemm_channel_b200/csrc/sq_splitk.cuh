// sq_splitk.cuh -- the W8A8 GEMM for few tokens (decode-shaped, M <= 128),
// with the per-token activation quantisation optionally fused in.
//
//   acc[m, n] = sum_k xq[m, k] * wq[n, k]     y[m, n] = ((float)acc * sx[m]) * sw[n]
//
// Sources: "quant_llm_int8", "The architecture: every piece explained" (int32
// accumulation, outer-product dequantisation); "Understanding W8A8 INT8 LLM
// Quantization", "Why Activation Quantization Is Hard, and How SmoothQuant
// Fixes It" (one dynamic scale per token over all channels) and "Inter-Token
// Latency (ITL)" (per-token quantisation is memory-bound work that every
// decode step pays; here it is done inside the GEMM kernel).
//
// With few tokens the layer is a stream over the int8 weight.  The weight
// takes the 128-row MMA side (A = 128 output channels), the tokens form the
// MMA N dimension (B = BNX padded token rows), and K is split across the CTAs
// of a thread-block cluster so that about one CTA per SM streams weight tiles:
//   warp 0      TMA producer: weight tiles (and, unfused, token tiles) into a
//               shared-memory ring, 128-byte swizzle, no multicast
//   warp 1      TMEM allocation and tcgen05.mma.kind::i8, M=128, N=BNX, K=32
//   warps 2..7  FUSED: quantise this CTA's K slice of the tokens straight into
//               the swizzled shared-memory B operand.  Each CTA first reduces
//               |x/s| over its slice, the partial maxima are exchanged across
//               the cluster through distributed shared memory (remote stores
//               plus remote mbarrier arrivals), and every CTA derives the same
//               per-token scales from the combined maxima.
//   warps 4..7  epilogue: tcgen05.ld of the int32 partial accumulator into the
//               CTA's shared memory; after a cluster barrier the cluster's
//               first CTA adds the other CTAs' partials (DSMEM loads; integer
//               addition, so the order does not matter), dequantises and stores.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#include "sq_div.cuh"
#include "sq_gemm.cuh"
#include "sq_mem.cuh"
#include "sq_ptx.cuh"
#include "sq_rowquant.cuh"

namespace sq {

constexpr int kSplitThreads = 256;
constexpr int kSplitWorkers = 192;  // warps 2..7
constexpr int kMaxSplits = 8;
constexpr int kFusedMaxSliceElems = 4096;  // K elements of one CTA's slice (128 KB / 32 tokens)

__device__ __forceinline__ void named_bar_sync(int id, int threads)
{
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

__device__ __forceinline__ int4 ld_shared_cluster_i4(uint32_t addr)
{
    int4 v;
    asm volatile("ld.shared::cluster.v4.s32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(addr)
                 : "memory");
    return v;
}

// Shared-memory layout of one split-K CTA (offsets from a 1024-aligned base).
struct SplitLayout {
    uint32_t a, b, part, pmax, wpmax, sxs, rsl, bars, misc, total;
};

// A stage holds `kbs` consecutive 128-byte k blocks (one barrier handshake per stage).
template <int BNX>
__host__ __device__ inline SplitLayout split_layout(int stages, bool fused, int kb_per_split, int kbs)
{
    SplitLayout L;
    uint32_t o = 0;
    L.a = o;
    o += stages * kbs * kBM * kBK;
    L.b = o;
    o += fused ? static_cast<uint32_t>(BNX) * kBK * kb_per_split
               : static_cast<uint32_t>(stages) * kbs * BNX * kBK;
    L.part = o;
    o += kBM * (BNX + 4) * 4;
    L.pmax = o;
    o += kMaxSplits * BNX * 4;
    L.wpmax = o;
    o += (kSplitWorkers / 32) * (BNX + 1) * 4;
    L.sxs = o;
    o += 2 * BNX * 4;
    o = (o + 15u) & ~15u;
    L.rsl = o;
    o += fused ? kFusedMaxSliceElems * 4 : 0;
    L.bars = o;
    o += (2 * stages + 5) * 8;
    L.misc = o;
    o += 16;
    L.total = o;
    return L;
}

// LSU: the weight and token tiles are copied by warps 4..7 with 16-byte
// cp.async (load/store unit) straight into the swizzled operand layout
// instead of by TMA; the epilogue runs on the same warps afterwards.
constexpr int kLsuLoaders = 128;

template <int BNX, int OUT, bool FUSED, typename TIN, bool LSU = false>
__global__ void __launch_bounds__(kSplitThreads, 1)
    gemm_splitk_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
                       const int8_t *__restrict__ wq, const int8_t *__restrict__ xq,
                       const TIN *__restrict__ x, const float *__restrict__ s,
                       const float *__restrict__ sx, const float *__restrict__ sw,
                       void *__restrict__ y, int M, int N, int K, int splits, int kb_per_split,
                       int stages, int kbs)
{
    // the tensor maps are this launch's own parameters: fetched before the
    // wait for the grid before
    if (threadIdx.x == 0) {
        tma_prefetch_desc(&tmW);
        if (!FUSED)
            tma_prefetch_desc(&tmX);
    }
    pdl_prologue();
    static_assert(BNX % 32 == 0 && BNX <= 128, "token tile");
    static_assert(!FUSED || BNX == 32, "the fused prologue handles up to 32 tokens");
    // NACC independent accumulators: consecutive MMAs rotate over them so no
    // MMA waits on the previous one's accumulation (with N = BNX this small
    // the accumulate dependency, not the tensor pipe, would set the pace);
    // the epilogue adds them (exact int32).
    constexpr int NACC = BNX <= 128 ? 4 : 2;
    constexpr uint32_t TMEM_COLS = BNX * NACC;
    constexpr int PSTRIDE = BNX + 4;  // padded int32 row stride of the partial buffer
    const SplitLayout L = split_layout<BNX>(stages, FUSED, kb_per_split, kbs);

    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t *g = smem_raw + (base - raw);
    const uint32_t sA = base + L.a, sB = base + L.b;
    int32_t *part = reinterpret_cast<int32_t *>(g + L.part);
    float *pmax = reinterpret_cast<float *>(g + L.pmax);
    float *wpmax = reinterpret_cast<float *>(g + L.wpmax);
    float *sxs = reinterpret_cast<float *>(g + L.sxs);
    const uint32_t bars = base + L.bars;
    auto full_bar = [&](int i) { return bars + 8u * i; };
    auto empty_bar = [&](int i) { return bars + 8u * (stages + i); };
    const uint32_t xready_bar = bars + 8u * (2 * stages);
    const uint32_t tfull_bar = xready_bar + 8u;
    const uint32_t pmax_bar = xready_bar + 16u;
    const uint32_t drain_bar = xready_bar + 24u;
    volatile uint32_t *tmem_slot = reinterpret_cast<volatile uint32_t *>(g + L.misc);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(g + L.misc + 4);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const int n_blk = blockIdx.x / splits;
    const int k_blocks = (K + kBK - 1) / kBK;
    const int kb0 = static_cast<int>(rank) * kb_per_split;
    const int kb1 = min(kb0 + kb_per_split, k_blocks);
    const int nkb = max(0, kb1 - kb0);

    if (threadIdx.x == 0) {
        for (int i = 0; i < stages; ++i) {
            mbar_init(full_bar(i), LSU ? kLsuLoaders : 1);
            mbar_init(empty_bar(i), 1);
        }
        mbar_init(xready_bar, kSplitWorkers);
        mbar_init(tfull_bar, 1);
        mbar_init(pmax_bar, static_cast<uint32_t>(splits) * 32u);
        mbar_init(drain_bar, 1);
        *abort_flag = 0;
        *reinterpret_cast<volatile int *>(g + L.misc + 8) = 0;
        fence_barrier_init();
    }
    if (warp == 2 && lane == 0) {
        // request this CTA's whole weight slice into L2 at once: the ring's
        // loads then wait on L2 rather than on HBM latency
        for (int kb = kb0; kb < kb1; ++kb)
            tma_prefetch_l2_2d(&tmW, kb * kBK, n_blk * kBM);
    }
    // the epilogue's scales, fetched while the main loop runs
    float swn_pre = 0.0f;
    if (warp >= 4) {
        const int64_t n = static_cast<int64_t>(n_blk) * kBM + (warp & 3) * 32 + lane;
        if (OUT != OUT_S32 && n < N)
            swn_pre = __ldg(sw + n);
        if (!FUSED && OUT != OUT_S32 && threadIdx.x - 128 < M)
            sxs[threadIdx.x - 128] = __ldg(sx + (threadIdx.x - 128));
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(const_cast<uint32_t *>(tmem_slot)), TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before_sync();
    __syncthreads();
    cluster_arrive();  // phase 1: this CTA's barriers exist (waited for before any remote access)
    bool waited_phase1 = false;
    tc_fence_after_sync();
    const uint32_t tmem_base = *tmem_slot;

    uint32_t issued_mask = 0, issued_parity = 0;
    bool mma_issued_any = false;

    const int nst = (nkb + kbs - 1) / kbs;  // stages this CTA streams
    const uint32_t a_stage = static_cast<uint32_t>(kbs) * kBM * kBK;
    const uint32_t b_stage = static_cast<uint32_t>(kbs) * BNX * kBK;
    if (warp == 0 && !LSU) {
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            for (int g = 0; g < nst; ++g) {
                const int cnt = min(kbs, nkb - g * kbs);
                if (!bounded_wait(empty_bar(stage), phase ^ 1u, kErrWaitProducer, abort_flag))
                    break;
                mbar_arrive_expect_tx(full_bar(stage),
                                      static_cast<uint32_t>(cnt) * (kBM * kBK + (FUSED ? 0 : BNX * kBK)));
                for (int i = 0; i < cnt; ++i) {
                    const int kb = kb0 + g * kbs + i;
                    tma_load_2d(sA + stage * a_stage + i * (kBM * kBK), &tmW, full_bar(stage), kb * kBK,
                                n_blk * kBM);
                    if (!FUSED)
                        tma_load_2d(sB + stage * b_stage + i * (BNX * kBK), &tmX, full_bar(stage), kb * kBK, 0);
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
            constexpr uint32_t idesc = idesc_i8(kBM, BNX);
            bool ok = true;
            if (FUSED)
                ok = bounded_wait(xready_bar, 0, kErrWaitPrologue, abort_flag);
            if (ok) {
                tc_fence_after_sync();
                int stage = 0;
                uint32_t phase = 0;
                for (int g = 0; g < nst; ++g) {
                    if (!bounded_wait(full_bar(stage), phase, kErrWaitMma, abort_flag)) {
                        ok = false;
                        break;
                    }
                    if (LSU)
                        fence_proxy_async_smem();  // the tiles were written through the generic proxy
                    tc_fence_after_sync();
                    const int cnt = min(kbs, nkb - g * kbs);
                    for (int i = 0; i < cnt; ++i) {
                        const int j = g * kbs + i;  // k block within this CTA's slice
                        const uint32_t a0 = sA + stage * a_stage + i * (kBM * kBK);
                        const uint32_t b0 = FUSED ? sB + j * (BNX * kBK) : sB + stage * b_stage + i * (BNX * kBK);
#pragma unroll
                        for (int k = 0; k < kBK / 32; ++k) {
                            const int step = j * (kBK / 32) + k;  // MMA index within the slice
                            mma_i8(tmem_base + static_cast<uint32_t>((step % NACC) * BNX),
                                   smem_desc_k_sw128(a0 + 32 * k), smem_desc_k_sw128(b0 + 32 * k), idesc,
                                   step >= NACC ? 1u : 0u);
                        }
                    }
                    mma_issued_any = true;
                    mma_commit(empty_bar(stage));
                    if (++stage == stages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            if (ok)
                mma_commit(tfull_bar);
        }
    }

    if constexpr (FUSED) {
        // ---- in-kernel per-token quantisation of this CTA's K slice ----------
        // Each worker warp owns whole token rows of the slice (rows ww, ww+6,
        // ...) and runs the standalone quantiser's arithmetic on them; the
        // slice's reciprocals RN(1/s) are staged in shared memory.
        if (warp >= 2) {
            constexpr int V = Vec<TIN>::N;
            const int wi = threadIdx.x - 64;
            const int ww = wi >> 5;  // worker warp 0..5
            const int64_t k0 = static_cast<int64_t>(kb0) * kBK;
            const int64_t k1 = min(static_cast<int64_t>(kb1) * kBK, static_cast<int64_t>(K));
            const int nch = static_cast<int>((k1 - k0) / V);
            float *rsl = reinterpret_cast<float *>(g + L.rsl);
            volatile int *bad_flag = reinterpret_cast<volatile int *>(g + L.misc + 8);
            const int bad = stage_factors<true, true>(s + k0, static_cast<int>(k1 - k0), rsl, wi, kSplitWorkers);
            if (bad)
                *bad_flag = 1;
            named_bar_sync(1, kSplitWorkers);
            const bool bad_divisor = *bad_flag != 0;
            auto factor = [&](int c, float (&f)[V]) {
#pragma unroll
                for (int h = 0; h < V / 4; ++h) {
                    const float4 v4 = reinterpret_cast<const float4 *>(rsl + c * V)[h];
                    f[4 * h] = v4.x;
                    f[4 * h + 1] = v4.y;
                    f[4 * h + 2] = v4.z;
                    f[4 * h + 3] = v4.w;
                }
            };
            auto sptr = [&](int c) { return s + k0 + static_cast<int64_t>(c) * V; };
            // (a) exact partial absmax of x/s per token over the slice
#pragma unroll 1
            for (int m = ww; m < M; m += kSplitWorkers / 32) {
                uint4 raw[8];
                const float E = warp_slice_absmax<TIN, MODE_X, 8>(x + static_cast<int64_t>(m) * K + k0, nch,
                                                                   lane, bad_divisor, factor, sptr, raw);
                if (lane == 0)
                    wpmax[m] = E;
            }
            named_bar_sync(1, kSplitWorkers);
            cluster_wait();  // every CTA of the cluster has initialised its barriers
            waited_phase1 = true;
            // (b) this CTA's partial maxima to every CTA of the cluster
            if (ww == 0) {
                const float p = lane < M ? wpmax[lane] : 0.0f;
                const uint32_t slot = smem_u32(pmax + rank * BNX + lane);
                for (int r = 0; r < splits; ++r)
                    st_shared_cluster_f32(map_shared_rank(slot, r), p);
                for (int r = 0; r < splits; ++r)
                    mbar_arrive_remote_release(map_shared_rank(pmax_bar, r));
            }
            // (c) combined maxima -> per-token scales (identical in every CTA)
            bounded_wait_cluster(pmax_bar, 0, kErrWaitCluster, abort_flag);
            if (wi < BNX) {
                float a = 0.0f;
                for (int r = 0; r < splits; ++r)
                    a = fmaxf(a, pmax[r * BNX + wi]);
                sxs[wi] = scale_from_max(a);
            }
            named_bar_sync(1, kSplitWorkers);
            // (d) codes of the slice into the swizzled K-major B operand
            uint8_t *bres = g + L.b;
#pragma unroll 1
            for (int m = ww; m < M; m += kSplitWorkers / 32) {
                auto store = [&](int c, uint2 u) {
                    const int kk = c * V;    // byte offset inside the slice
                    const int jb = kk >> 7;  // 128-byte k block
                    const int kin = kk & 127;
                    const uint32_t off = static_cast<uint32_t>(jb) * (BNX * kBK) + (m >> 3) * 1024u +
                                         (m & 7) * 128u + ((((kin >> 4) ^ (m & 7)) & 7) << 4) + (kin & 15);
                    if constexpr (V == 8)
                        *reinterpret_cast<uint2 *>(bres + off) = u;
                    else
                        *reinterpret_cast<uint32_t *>(bres + off) = u.x;
                };
                warp_slice_codes<TIN, MODE_X, 4>(x + static_cast<int64_t>(m) * K + k0, nch, lane,
                                                 bad_divisor, sxs[m], factor, sptr, store);
            }
            fence_proxy_async_smem();
            mbar_arrive(xready_bar);
        }
    }

    if constexpr (LSU) {
        // ---- weight and token tiles through the load/store unit ------------
        // thread t copies 16-byte chunk (t & 7) of rows (t >> 3) + 16 i of the
        // 128-byte k block, to the position the 128-byte swizzle gives it
        if (warp >= 4) {
            const int t = static_cast<int>(threadIdx.x) - 128;
            const int j = t & 7;
            const int rbase = t >> 3;
            const int64_t n0 = static_cast<int64_t>(n_blk) * kBM;
            int stage = 0;
            uint32_t phase = 0;
            for (int g = 0; g < nkb; ++g) {
                if (!bounded_wait(empty_bar(stage), phase ^ 1u, kErrWaitProducer, abort_flag))
                    break;
                const int64_t kk = static_cast<int64_t>(kb0 + g) * kBK + j * 16;
                const bool kv = kk < K;
                const uint32_t sa = sA + stage * (kBM * kBK);
#pragma unroll
                for (int i = 0; i < kBM / 16; ++i) {
                    const int r = rbase + 16 * i;
                    const int64_t n = n0 + r;
                    const bool v = kv && n < N;
                    cp_async_16(sa + (r >> 3) * 1024u + (r & 7) * 128u + (((j ^ r) & 7) << 4), wq + (v ? n * K + kk : 0),
                                v);
                }
                const uint32_t sb = sB + stage * (BNX * kBK);
#pragma unroll
                for (int i = 0; i < BNX / 16; ++i) {
                    const int r = rbase + 16 * i;
                    const bool v = kv && r < M;
                    cp_async_16(sb + (r >> 3) * 1024u + (r & 7) * 128u + (((j ^ r) & 7) << 4),
                                xq + (v ? static_cast<int64_t>(r) * K + kk : 0), v);
                }
                cp_async_arrive(full_bar(stage));
                if (++stage == stages) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
            cp_async_wait_all();  // nothing of this thread's is in flight past here
        }
    }

    // ---- epilogue part 1: every CTA parks its int32 partial in shared memory
    if (warp >= 4) {
        const int quarter = warp & 3;
        const int row = quarter * 32 + lane;
        const bool ok = bounded_wait(tfull_bar, 0, kErrWaitAccFull, abort_flag);
        if (__all_sync(0xFFFFFFFFu, ok)) {
            tc_fence_after_sync();
#pragma unroll 1
            for (int c = 0; c < BNX / 32; ++c) {
                uint32_t r[32], t[32];
                const uint32_t lane_addr = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + c * 32;
                tmem_ld_32x32b_x32(lane_addr, r);
                tmem_ld_wait();
#pragma unroll 1
                for (int a = 1; a < NACC; ++a) {
                    tmem_ld_32x32b_x32(lane_addr + static_cast<uint32_t>(a * BNX), t);
                    tmem_ld_wait();
#pragma unroll
                    for (int q = 0; q < 32; ++q)
                        r[q] += t[q];  // exact int32 sums
                }
                int4 *dst = reinterpret_cast<int4 *>(part + row * PSTRIDE + c * 32);
#pragma unroll
                for (int v = 0; v < 8; ++v)
                    dst[v] = make_int4(r[4 * v], r[4 * v + 1], r[4 * v + 2], r[4 * v + 3]);
            }
        }
    }

    // ---- teardown of the async machinery (before the cluster barrier) -------
    if (warp == 1 && lane == 0 && *abort_flag && mma_issued_any) {
        mma_commit(drain_bar);
        bounded_wait(drain_bar, 0, kErrWaitDrain, nullptr, kWaitTimeoutNs / 4);
    }
    if (warp == 0 && lane == 0 && *abort_flag) {
        for (int i = 0; i < stages; ++i)
            if (issued_mask & (1u << i))
                bounded_wait(full_bar(i), (issued_parity >> i) & 1u, kErrWaitDrain, nullptr,
                             kWaitTimeoutNs / 4);
    }
    if (!waited_phase1)
        cluster_wait();
    tc_fence_before_sync();
    __syncthreads();
    cluster_arrive();  // phase 2: every CTA's partial is in its shared memory
    cluster_wait();

    // ---- epilogue part 2: the cluster's first CTA reduces and stores --------
    if (rank == 0 && warp >= 4) {
        const int quarter = warp & 3;
        const int row = quarter * 32 + lane;
        const int64_t n = static_cast<int64_t>(n_blk) * kBM + row;
        const float swn = swn_pre;
        const uint32_t my = smem_u32(part + row * PSTRIDE);
#pragma unroll 1
        for (int c = 0; c < BNX / 32; ++c) {
            if (c * 32 >= M)
                break;
            int acc[32];
#pragma unroll
            for (int v = 0; v < 8; ++v) {
                const int4 t = *reinterpret_cast<const int4 *>(part + row * PSTRIDE + c * 32 + 4 * v);
                acc[4 * v] = t.x;
                acc[4 * v + 1] = t.y;
                acc[4 * v + 2] = t.z;
                acc[4 * v + 3] = t.w;
            }
            for (int r = 1; r < splits; ++r) {
                const uint32_t remote = map_shared_rank(my, r) + static_cast<uint32_t>(c * 32 * 4);
#pragma unroll
                for (int v = 0; v < 8; ++v) {
                    const int4 t = ld_shared_cluster_i4(remote + 16u * v);
                    acc[4 * v] += t.x;
                    acc[4 * v + 1] += t.y;
                    acc[4 * v + 2] += t.z;
                    acc[4 * v + 3] += t.w;
                }
            }
            if (n < N) {
                const int m0 = c * 32;
#pragma unroll
                for (int jj = 0; jj < 32; ++jj) {
                    const int m = m0 + jj;
                    if (m < M) {
                        const int64_t idx = static_cast<int64_t>(m) * N + n;
                        if constexpr (OUT == OUT_S32) {
                            reinterpret_cast<int32_t *>(y)[idx] = acc[jj];
                        } else {
                            const float sxm = sxs[m];
                            const float o = __fmul_rn(__fmul_rn(__int2float_rn(acc[jj]), sxm), swn);
                            if constexpr (OUT == OUT_F32)
                                reinterpret_cast<float *>(y)[idx] = o;
                            else
                                reinterpret_cast<__nv_bfloat16 *>(y)[idx] = __float2bfloat16_rn(o);
                        }
                    }
                }
            }
        }
    }
    cluster_arrive();  // phase 3: peers keep their shared memory until it has been read
    cluster_wait();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after_sync();
        tmem_dealloc(tmem_base, TMEM_COLS);
    }
}

}  // namespace sq
