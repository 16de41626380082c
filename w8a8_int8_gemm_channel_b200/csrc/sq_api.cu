// sq_api.cu -- the C ABI of libsq (declared in include/sq.h): argument
// validation on the host, tensor-map creation and kernel launches.  No entry
// point allocates memory; no C++ exception crosses the interface.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <cstdint>
#include <cstring>
#include <cstdio>
#include <cstdlib>
#include <mutex>
#include <tuple>
#include <type_traits>
#include <vector>
#include <utility>
#include <climits>

#include "sq.h"
#include "sq_gemm.cuh"
#include "sq_gemm_pair.cuh"
#include "sq_mem.cuh"
#include "sq_ptx.cuh"
#include "sq_gptq.cuh"
#include "sq_splitk.cuh"
#include "sq_decode.cuh"
#include "sq_slab.cuh"
#include "sq_quant_staged.cuh"
#include "sq_quant_cluster.cuh"

namespace {

using sq::OUT_BF16;
using sq::OUT_F32;
using sq::OUT_S32;

constexpr int kMaxDevices = 64;
constexpr int kMaxDynSmem = 232448;  // 227 KB of dynamic shared memory per CTA on sm_100
constexpr int kSmSmemBytes = 233472;  // shared memory of one SM (228 KB)

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline bool valid_dtype(sq_dtype dt) { return dt == SQ_F32 || dt == SQ_BF16; }

inline size_t dtype_size(sq_dtype dt) { return dt == SQ_F32 ? 4 : 2; }

inline sq_status launch_status()
{
    cudaError_t e = cudaPeekAtLastError();
    if (e != cudaSuccess) {
        cudaGetLastError();
        return SQ_ERR_CUDA;
    }
    return SQ_OK;
}

struct DeviceInfo {
    int sms = 0;
    bool ok = false;
};

bool device_info(DeviceInfo &info)
{
    static DeviceInfo cache[kMaxDevices];
    static std::mutex mu;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
        return false;
    std::lock_guard<std::mutex> lk(mu);
    if (!cache[dev].ok) {
        int sms = 0;
        if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return false;
        cache[dev].sms = sms;
        cache[dev].ok = true;
    }
    info = cache[dev];
    return true;
}

// Launch plans are printed to stderr when SQ_DEBUG_PLAN is set (diagnostics).
bool debug_plan()
{
    static const bool on = std::getenv("SQ_DEBUG_PLAN") != nullptr;
    return on;
}

// Programmatic dependent launch for every kernel of the library (each one
// begins with griddepcontrol.wait, so it sees all work before it on the
// stream); SQ_PDL=0 turns the attribute off.
bool pdl_enabled()
{
    static const bool on = !(std::getenv("SQ_PDL") && std::atoi(std::getenv("SQ_PDL")) == 0);
    return on;
}

// Launch `kernel` on `st`.  Kernels that use cluster features (distributed
// shared memory, cluster barriers, remote mbarrier arrivals) pass their
// cluster shape cx x cy, which is set even when it is 1 x 1; other kernels
// pass cx = 0.
template <typename... KArgs, typename... Args>
sq_status launch_kernel(void (*kernel)(KArgs...), dim3 grid, dim3 block, int smem, cudaStream_t st, int cx,
                        int cy, Args &&...args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = static_cast<size_t>(smem);
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    unsigned n = 0;
    if (cx > 0) {
        attr[n].id = cudaLaunchAttributeClusterDimension;
        attr[n].val.clusterDim.x = static_cast<unsigned>(cx);
        attr[n].val.clusterDim.y = static_cast<unsigned>(cy);
        attr[n].val.clusterDim.z = 1;
        ++n;
    }
    if (pdl_enabled()) {
        attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[n].val.programmaticStreamSerializationAllowed = 1;
        ++n;
    }
    cfg.attrs = attr;
    cfg.numAttrs = n;
    if (cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...) != cudaSuccess) {
        cudaGetLastError();
        return SQ_ERR_CUDA;
    }
    return launch_status();
}

// ---- tensor maps -----------------------------------------------------------
PFN_cuTensorMapEncodeTiled_v12000 encode_fn()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// int8 matrix [rows, cols] (cols contiguous, row pitch = cols bytes); box of
// 128 bytes x box_rows rows, 128-byte swizzle, zero fill out of bounds.
bool make_tmap_i8(CUtensorMap *map, const void *base, int64_t rows, int64_t cols, int box_rows)
{
    auto fn = encode_fn();
    if (fn == nullptr)
        return false;
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols)};
    cuuint32_t box[2] = {static_cast<cuuint32_t>(sq::kBK), static_cast<cuuint32_t>(box_rows)};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(base), dims, strides,
                    box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// ---- per-kernel one-time attribute setup ----------------------------------
// `done_mask` must be distinct for every kernel instantiation (all GEMM
// instantiations share one function-pointer type), so each caller owns it.
template <typename KernelT>
bool ensure_smem_attr(KernelT kernel, int bytes, std::atomic<uint64_t> &done_mask)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
        return false;
    const uint64_t bit = 1ull << dev;
    if (done_mask.load(std::memory_order_acquire) & bit)
        return true;
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) !=
        cudaSuccess)
        return false;
    done_mask.fetch_or(bit, std::memory_order_release);
    return true;
}

// ---- column absmax ---------------------------------------------------------
template <typename T>
sq_status launch_col_absmax(const T *x, int64_t R, int64_t K, int64_t ld, float *out,
                            cudaStream_t st)
{
    DeviceInfo di;
    if (!device_info(di))
        return SQ_ERR_CUDA;
    constexpr int V = sq::Vec<T>::N;
    constexpr int CL = sq::kColClusterRows;
    const int64_t chunks = K / V;
    const int64_t col_blocks = (chunks + sq::kColThreads - 1) / sq::kColThreads;
    // one wave of about 4 CTAs of 256 threads per SM (measured best from 1 to
    // 12 for calibration batches and weights alike), in clusters of CL row
    // bands; bands are whole multiples of the 16 rows a thread keeps in
    // flight.  SQ_COL_PER_SM overrides the CTAs per SM.
    static const int force_per_sm = std::getenv("SQ_COL_PER_SM") ? std::atoi(std::getenv("SQ_COL_PER_SM")) : 0;
    const int per_sm = force_per_sm > 0 ? force_per_sm : 4;
    const int64_t want = std::max<int64_t>(CL, (int64_t)di.sms * per_sm / col_blocks);
    int64_t rows_per_block = std::max<int64_t>(16, ((R + want - 1) / want + 15) / 16 * 16);
    int64_t row_blocks = (R + rows_per_block - 1) / rows_per_block;
    while (row_blocks > 65528) {
        rows_per_block *= 2;
        row_blocks = (R + rows_per_block - 1) / rows_per_block;
    }
    row_blocks = (row_blocks + CL - 1) / CL * CL;  // whole clusters; surplus bands are empty
    return launch_kernel(sq::col_absmax_kernel<T>, dim3(static_cast<unsigned>(col_blocks), static_cast<unsigned>(row_blocks)),
                         dim3(sq::kColThreads), 0, st, 1, CL, x, R, K, ld, rows_per_block,
                         reinterpret_cast<unsigned int *>(out));
}

// ---- row quantisers ----------------------------------------------------------
constexpr int64_t kSmemFactorBytes = 112 * 1024;  // per-column factors staged in shared memory

// Two launches: row scales (one warp per row), then the codes (elementwise).
template <typename T, int MODE, bool SMEM_S>
sq_status launch_row_scale(const T *in, int64_t rows, int64_t K, const float *s, float *scale,
                           cudaStream_t st, const DeviceInfo &di)
{
    auto kernel = sq::row_scale_kernel<T, MODE, 16, SMEM_S>;
    const int smem = SMEM_S ? static_cast<int>(K * sizeof(float)) : 0;
    static std::atomic<uint64_t> attr_done{0};
    if (SMEM_S && !ensure_smem_attr(kernel, kMaxDynSmem, attr_done))
        return SQ_ERR_CUDA;
    const int per_sm = smem <= 96 * 1024 ? 2 : 1;
    const int warps = sq::kQuantThreads / 32;
    const int64_t blocks = std::min<int64_t>((rows + warps - 1) / warps, (int64_t)per_sm * di.sms);
    return launch_kernel(kernel, dim3(static_cast<unsigned>(blocks)), dim3(sq::kQuantThreads), smem, st, 0, 0, in, rows,
                         K, s, scale);
}

// Single-pass quantiser (row in registers): 2^log2g warps per row, CH chunks
// per lane.
// log2 of the warps per row for an exact fit of `ch` chunks a lane (-1: none)
inline int exact_fit_log2g(int64_t nch, int ch)
{
    for (int log2g = 0; log2g <= 3; ++log2g)
        if (((int64_t)32 * ch << log2g) == nch)
            return log2g;
    return -1;
}

template <typename T, int MODE, int CH, bool FIT, bool BB, bool GLU = false, bool TAB = true,
          int THREADS = sq::kQuantThreads>
sq_status launch_row_quant_cfg(const T *in, int64_t rows, int64_t K, const float *s, int8_t *q,
                               float *scale, int log2g, cudaStream_t st, const DeviceInfo &di, T *hout = nullptr,
                               int *zero = nullptr, int nzero = 0)
{
    auto kernel = sq::row_quant_kernel<T, MODE, CH, FIT, BB, GLU, TAB, THREADS>;
    const int smem = TAB ? static_cast<int>(sq::row_quant_smem(K, BB)) : 0;
    static std::atomic<uint64_t> attr_done{0};
    // the kernel also has a little static shared memory (the group maxima)
    if (!ensure_smem_attr(kernel, kMaxDynSmem - 1024, attr_done))
        return SQ_ERR_CUDA;
    // resident CTAs per SM for this shared-memory size, cached per size
    static std::mutex mu;
    static std::vector<std::pair<int, int>> occ;  // smem -> CTAs per SM (one device type)
    int per_sm = 0;
    {
        std::lock_guard<std::mutex> lk(mu);
        for (auto &e : occ)
            if (e.first == smem)
                per_sm = e.second;
    }
    if (per_sm == 0) {
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, THREADS, smem) !=
                cudaSuccess ||
            per_sm < 1) {
            cudaGetLastError();
            return SQ_ERR_CUDA;
        }
        std::lock_guard<std::mutex> lk(mu);
        occ.emplace_back(smem, per_sm);
    }
    // few rows: spread each row over more warps so that every SM has work
    // (not for FIT, whose G is fixed by the row length)
    while (!FIT && log2g < 3 && rows * (1 << log2g) < (int64_t)di.sms * per_sm * (THREADS / 32))
        ++log2g;
    const int slots = (THREADS / 32) >> log2g;
    const int64_t blocks = std::min<int64_t>((rows + slots - 1) / slots, (int64_t)per_sm * di.sms);
    if (debug_plan())
        std::fprintf(stderr, "sq quant rows=%lld K=%lld: single pass CH=%d G=%d per_sm=%d blocks=%lld\n",
                     (long long)rows, (long long)K, CH, 1 << log2g, per_sm, (long long)blocks);
    return launch_kernel(kernel, dim3(static_cast<unsigned>(blocks)), dim3(THREADS), smem, st, 0, 0, in, rows,
                         K, s, log2g, q, scale, hout, zero, nzero);
}

// The quantiser with the gated feed-forward activation in front (rows of
// [gate | up], 2K values each): single pass only, 8 chunks per lane (two CTAs
// per SM: the up half doubles the registers a row takes) or 16 for rows too
// long for that (one CTA per SM).
template <typename T>
sq_status launch_glu_quant(const T *gu, int64_t rows, int64_t K, const float *s, int8_t *q, float *scale, T *hout,
                           cudaStream_t st)
{
    DeviceInfo di;
    if (!device_info(di))
        return SQ_ERR_CUDA;
    if (rows > 2147483647LL)
        return SQ_ERR_UNSUPPORTED;
    constexpr int V = sq::Vec<T>::N;
    const int64_t nch = K / V;
    const bool bb = V == 8 && sq::row_quant_smem(K, true) <= 64 * 1024;
    if (sq::row_quant_smem(K, bb) > kMaxDynSmem - 1024)
        return SQ_ERR_UNSUPPORTED;
#define SQ_GLU_CFG(CH_, FIT_, BB_) \
    launch_row_quant_cfg<T, sq::MODE_X, CH_, FIT_, BB_, true>(gu, rows, K, s, q, scale, log2g, st, di, hout)
    // an exact fit once the rows give every SM 4 warps or more; fewer rows
    // rather spread over more warps (the SiLU step makes a row's work heavier
    // than in sq_quant_act: measured at M = 128 and 1024, I = 4096)
    const int64_t min_warps = (int64_t)di.sms * 4;
    if constexpr (V == 8) {  // 7 chunks a lane where that fits exactly and 8 does not
        int log2g = exact_fit_log2g(nch, 8) < 0 ? exact_fit_log2g(nch, 7) : -1;
        if (log2g >= 0 && rows * (1 << log2g) >= min_warps)
            return bb ? SQ_GLU_CFG(7, true, true) : SQ_GLU_CFG(7, true, false);
    }
    for (int ch : {8, 16}) {
        int log2g = 0;
        while (log2g < 3 && ((int64_t)32 * ch << log2g) < nch)
            ++log2g;
        if (((int64_t)32 * ch << log2g) < nch)
            continue;
        const bool fit = ((int64_t)32 * ch << log2g) == nch && rows * (1 << log2g) >= min_warps;
        if (ch == 8) {
            if (bb)
                return fit ? SQ_GLU_CFG(8, true, true) : SQ_GLU_CFG(8, false, true);
            return fit ? SQ_GLU_CFG(8, true, false) : SQ_GLU_CFG(8, false, false);
        }
        return fit ? SQ_GLU_CFG(16, true, false) : SQ_GLU_CFG(16, false, false);
#undef SQ_GLU_CFG
    }
    return SQ_ERR_UNSUPPORTED;
}

// The staged quantiser (bf16 rows brought into shared memory by bulk
// copies): rows of exactly 32 * CH * G chunks, CH in {7, 8, 14} and G in
// {1, 2, 4, 8} (16 with 512-thread CTAs).  Returns false (nothing launched)
// for other rows.
template <int MODE, int CH, int THREADS = sq::kQuantThreads>
sq_status launch_staged_cfg(const __nv_bfloat16 *in, int64_t rows, int64_t K, const float *s, int8_t *q,
                            float *scale, int log2g, cudaStream_t st, const DeviceInfo &di, int *zero, int nzero)
{
    auto kernel = sq::row_quant_staged_kernel<MODE, CH, THREADS>;
    static std::atomic<uint64_t> attr_done{0};
    if (!ensure_smem_attr(kernel, kMaxDynSmem - 1024, attr_done))
        return SQ_ERR_CUDA;
    const int groups = (THREADS / 32) >> log2g;
    // two CTAs an SM with two row buffers a group where that fits (256
    // threads), else one CTA with as many buffers (up to 4) as fit
    int nslots = 0, per_sm = 0;
    // (an SM's shared memory, less 1 KB reserved a CTA and 512 bytes of static arrays)
    const int64_t per_cta2 = kSmSmemBytes / 2 - 1024 - 512;
    if (THREADS == sq::kQuantThreads && sq::staged_smem_bytes(K, groups, 2) <= per_cta2) {
        nslots = 2;
        per_sm = 2;
        if (sq::staged_smem_bytes(K, groups, 3) <= per_cta2)
            nslots = 3;
    } else {
        for (int n = sq::kStagedMaxSlots; n >= 2 && nslots == 0; --n)
            if (sq::staged_smem_bytes(K, groups, n) <= kMaxDynSmem - 1024)
                nslots = n;
        per_sm = 1;
    }
    if (nslots == 0)
        return SQ_ERR_UNSUPPORTED;
    const int smem = static_cast<int>(sq::staged_smem_bytes(K, groups, nslots));
    const int64_t blocks = std::min<int64_t>((rows + groups - 1) / groups, (int64_t)per_sm * di.sms);
    if (debug_plan())
        std::fprintf(stderr, "sq staged quant rows=%lld K=%lld: CH=%d G=%d threads=%d slots=%d per_sm=%d blocks=%lld smem=%d\n",
                     (long long)rows, (long long)K, CH, 1 << log2g, THREADS, nslots, per_sm, (long long)blocks, smem);
    return launch_kernel(kernel, dim3(static_cast<unsigned>(blocks)), dim3(THREADS), smem, st, 0, 0, in, rows, K, s,
                         log2g, nslots, q, scale, zero, nzero);
}

template <int MODE>
bool launch_staged(const __nv_bfloat16 *in, int64_t rows, int64_t K, const float *s, int8_t *q, float *scale,
                   cudaStream_t st, const DeviceInfo &di, int *zero, int nzero, sq_status &r)
{
    // for few rows the quantiser is latency-bound and the register-resident
    // kernel (smaller shared memory, so it shares an SM with the few-token
    // GEMM that follows it in sq_linear) is used; SQ_QUANT_STAGED=0 turns the
    // staged kernel off, =2 takes it for any row count (same arithmetic)
    static const int mode = std::getenv("SQ_QUANT_STAGED") ? std::atoi(std::getenv("SQ_QUANT_STAGED")) : 1;
    if (mode == 0 || (mode == 1 && rows < 256))
        return false;
    const int64_t nch = K / 8;
    // rows of 3584 chunks (K = 28672): the factor table and two rows fill an
    // SM's shared memory, so one CTA of 16 warps (7 chunks a lane) rather
    // than 8 warps of 14; SQ_QUANT_STAGED512=0 takes the 8-warp form
    static const bool w512 =
        !(std::getenv("SQ_QUANT_STAGED512") && std::atoi(std::getenv("SQ_QUANT_STAGED512")) == 0);
    if (w512 && nch == 32 * 7 * 16) {
        r = launch_staged_cfg<MODE, 7, 512>(in, rows, K, s, q, scale, 4, st, di, zero, nzero);
        return r != SQ_ERR_UNSUPPORTED;
    }
    for (int ch : {8, 7, 14}) {
        for (int log2g = 0; log2g <= 3; ++log2g) {
            if ((int64_t)32 * ch << log2g != nch)
                continue;
            if (ch == 8)
                r = launch_staged_cfg<MODE, 8>(in, rows, K, s, q, scale, log2g, st, di, zero, nzero);
            else if (ch == 7)
                r = launch_staged_cfg<MODE, 7>(in, rows, K, s, q, scale, log2g, st, di, zero, nzero);
            else
                r = launch_staged_cfg<MODE, 14>(in, rows, K, s, q, scale, log2g, st, di, zero, nzero);
            return r != SQ_ERR_UNSUPPORTED;
        }
    }
    return false;
}

// The cluster form of the few-row quantiser: C CTAs a row (sq_quant_cluster.cuh).
template <typename T, int MODE, int CH>
sq_status launch_quant_cluster_cfg(const T *in, int64_t rows, int64_t K, const float *s, int8_t *q, float *scale,
                                   int C, cudaStream_t st, int *zero, int nzero)
{
    auto kernel = sq::row_quant_cluster_kernel<T, MODE, CH>;
    if (debug_plan())
        std::fprintf(stderr, "sq quant rows=%lld K=%lld: cluster of %d CTAs a row, CH=%d\n", (long long)rows,
                     (long long)K, C, CH);
    return launch_kernel(kernel, dim3(static_cast<unsigned>(rows * C)), dim3(sq::kQuantClusterThreads), 0, st, C, 1,
                         in, rows, K, s, q, scale, zero, nzero);
}

// Few rows of many chunks (more than 512: over 2 chunks a lane on 8 warps): a
// cluster of C CTAs a row, the largest C in {8, 4, 2} that keeps one CTA an SM
// (rows x C <= SMs) and leaves every CTA a slice of at least 128 chunks.
// Measured in the decode chain of sq_linear calls (1 to 32 tokens) at
// K = 14336: 4 to 8 SMs a row took about 2 us less a call than one.  At
// K = 4096 (512 chunks) 2 to 4 SMs a row took 2 us more while the form
// exchanged twice a row; with one exchange, 4 SMs a row came within 0.3 us a
// pass of one (2 SMs: 5 us slower), so such rows keep the one-CTA forms.
// Returns false (nothing launched) when no C qualifies.  SQ_QUANT_CLUSTER=0
// turns the form off, =2 takes it for rows of 512 chunks or fewer too;
// SQ_QUANT_CLUSTER_MIN sets the smallest slice in chunks (tuning).
template <typename T, int MODE>
bool launch_quant_cluster(const T *in, int64_t rows, int64_t K, const float *s, int8_t *q, float *scale,
                          cudaStream_t st, const DeviceInfo &di, int *zero, int nzero, sq_status &r)
{
    static const int mode = std::getenv("SQ_QUANT_CLUSTER") ? std::atoi(std::getenv("SQ_QUANT_CLUSTER")) : 1;
    static const int min_span =
        std::getenv("SQ_QUANT_CLUSTER_MIN") ? std::max(32, std::atoi(std::getenv("SQ_QUANT_CLUSTER_MIN"))) : 128;
    constexpr int V = sq::Vec<T>::N;
    const int64_t nch = K / V;
    // C >= 2 and CH <= 8 cover rows of up to 2 * 8 * 256 chunks
    if (mode == 0 || (mode == 1 && nch <= (int64_t)32 * 8 * 2) || nch > (int64_t)2 * 8 * sq::kQuantClusterThreads)
        return false;
    int C = 0;
    for (int c : {8, 4, 2})
        if (C == 0 && rows * c <= di.sms && (nch + c - 1) / c >= min_span)
            C = c;
    if (C == 0)
        return false;
    const int64_t span = (nch + C - 1) / C;
    int ch = 1;
    while ((int64_t)sq::kQuantClusterThreads * ch < span)
        ch *= 2;
    switch (ch) {
    case 1:
        r = launch_quant_cluster_cfg<T, MODE, 1>(in, rows, K, s, q, scale, C, st, zero, nzero);
        break;
    case 2:
        r = launch_quant_cluster_cfg<T, MODE, 2>(in, rows, K, s, q, scale, C, st, zero, nzero);
        break;
    case 4:
        r = launch_quant_cluster_cfg<T, MODE, 4>(in, rows, K, s, q, scale, C, st, zero, nzero);
        break;
    default:
        r = launch_quant_cluster_cfg<T, MODE, 8>(in, rows, K, s, q, scale, C, st, zero, nzero);
        break;
    }
    return true;
}

// Row counts below which the activation quantiser takes its few-row form.
constexpr int64_t kFewRows = 256;

// `zero` (may be null): nzero ints the quantiser kernel clears on the side.
template <typename T, int MODE>
sq_status launch_quant_rows(const T *in, int64_t rows, int64_t K, const float *s, int8_t *q,
                            float *scale, cudaStream_t st, int *zero = nullptr, int nzero = 0)
{
    DeviceInfo di;
    if (!device_info(di))
        return SQ_ERR_CUDA;
    if (rows > 2147483647LL)
        return SQ_ERR_UNSUPPORTED;
    if constexpr (std::is_same<T, __nv_bfloat16>::value) {
        sq_status r = SQ_OK;
        if (launch_staged<MODE>(in, rows, K, s, q, scale, st, di, zero, nzero, r))
            return r;
    }
    // tuning override (same arithmetic, other kernels): SQ_QUANT_KIND=2 takes
    // the two-kernel path for every K
    static const int force_kind = std::getenv("SQ_QUANT_KIND") ? std::atoi(std::getenv("SQ_QUANT_KIND")) : 0;
    constexpr int V = sq::Vec<T>::N;
    const int64_t nch = K / V;
    // Few rows (decode): the latency of one row is the cost, and a factor
    // table staged in every CTA for one row or two would be most of it.  So
    // one CTA a row, the fewest chunks a lane that cover it, and no table
    // (each lane reads its own s_k): 8 warps while that is at most 2 chunks a
    // lane, else 16 warps (measured at K = 14336 in the decode chain: 3.5
    // chunks a lane on 16 warps took 4 us less a call than 7 on 8 warps; 32
    // warps gained nothing more).  The 16-warp form is held to 64 registers
    // a thread, half an SM's register file.
    // SQ_QUANT_FEW=0 turns the few-row form off; SQ_QUANT_FEW_THREADS=256 or
    // 512 fixes its CTA size (tuning).
    static const bool few_on = !(std::getenv("SQ_QUANT_FEW") && std::atoi(std::getenv("SQ_QUANT_FEW")) == 0);
    static const int few_threads =
        std::getenv("SQ_QUANT_FEW_THREADS") ? std::atoi(std::getenv("SQ_QUANT_FEW_THREADS")) : 0;
    if (few_on && force_kind != 2 && rows < kFewRows) {
        sq_status r = SQ_OK;
        if (launch_quant_cluster<T, MODE>(in, rows, K, s, q, scale, st, di, zero, nzero, r))
            return r;
    }
    if (few_on && force_kind != 2 && rows < kFewRows && nch <= (int64_t)32 * 16 * 8) {
        const bool wide = few_threads == 512 || (few_threads != 256 && nch > (int64_t)32 * 8 * 2);
        const int lg = wide ? 4 : 3;
        int ch = wide ? 1 : 2;
        while (((int64_t)32 * ch << lg) < nch)
            ch *= 2;
        const bool fit = ((int64_t)32 * ch << lg) == nch;
#define SQ_Q_FEW(CH_, TH_) (fit ? launch_row_quant_cfg<T, MODE, CH_, true, false, false, false, TH_>(in, rows, K, s, q, scale, lg, st, di, nullptr, zero, nzero) \
                                : launch_row_quant_cfg<T, MODE, CH_, false, false, false, false, TH_>(in, rows, K, s, q, scale, lg, st, di, nullptr, zero, nzero))
        if (wide) {
            switch (ch) {
            case 1:
                return SQ_Q_FEW(1, 512);
            case 2:
                return SQ_Q_FEW(2, 512);
            case 4:
                return SQ_Q_FEW(4, 512);
            default:
                return SQ_Q_FEW(8, 512);
            }
        }
        switch (ch) {
        case 2:
            return SQ_Q_FEW(2, 256);
        case 4:
            return SQ_Q_FEW(4, 256);
        case 8:
            return SQ_Q_FEW(8, 256);
        default:
            return SQ_Q_FEW(16, 256);
        }
#undef SQ_Q_FEW
    }
    // the bf16 bound while both factor tables stay small (about 3 CTAs per SM)
    const bool bb = V == 8 && sq::row_quant_smem(K, true) <= 64 * 1024;
    if (force_kind != 2 && sq::row_quant_smem(K, bb) <= kMaxDynSmem - 1024) {
        // tuning override: SQ_QUANT_CH=2|4|8 takes that many chunks a lane
        // wherever it fits a row exactly (same arithmetic, another shape)
        static const int force_ch = std::getenv("SQ_QUANT_CH") ? std::atoi(std::getenv("SQ_QUANT_CH")) : 0;
        if (force_ch == 2 || force_ch == 4 || force_ch == 8) {
            int g = -1;
            for (int l = 0; l <= 3 && g < 0; ++l)
                if (((int64_t)32 * force_ch << l) == nch)
                    g = l;
            if (g >= 0) {
#define SQ_Q_CFG(CH_) (bb ? launch_row_quant_cfg<T, MODE, CH_, true, true>(in, rows, K, s, q, scale, g, st, di, nullptr, zero, nzero) \
                          : launch_row_quant_cfg<T, MODE, CH_, true, false>(in, rows, K, s, q, scale, g, st, di, nullptr, zero, nzero))
                if (force_ch == 2)
                    return SQ_Q_CFG(2);
                if (force_ch == 4)
                    return SQ_Q_CFG(4);
                return SQ_Q_CFG(8);
#undef SQ_Q_CFG
            }
        }
        // 8 chunks per lane (three CTAs per SM), 16 for rows too long for that
        for (int ch : {8, 16}) {
            int log2g = 0;
            while (log2g < 3 && ((int64_t)32 * ch << log2g) < nch)
                ++log2g;
            if (((int64_t)32 * ch << log2g) < nch)
                continue;
            // an exact fit drops the bounds checks and idle lanes; it is taken
            // however few the rows (measured: at M = 128 and 1024, K = 4096, as
            // fast as or faster than spreading each row over more warps)
            const bool fit = ((int64_t)32 * ch << log2g) == nch;
            if (bb) {
                if (ch == 8)
                    return fit ? launch_row_quant_cfg<T, MODE, 8, true, true>(in, rows, K, s, q, scale, log2g, st, di, nullptr, zero, nzero)
                               : launch_row_quant_cfg<T, MODE, 8, false, true>(in, rows, K, s, q, scale, log2g, st, di, nullptr, zero, nzero);
                return fit ? launch_row_quant_cfg<T, MODE, 16, true, true>(in, rows, K, s, q, scale, log2g, st, di, nullptr, zero, nzero)
                           : launch_row_quant_cfg<T, MODE, 16, false, true>(in, rows, K, s, q, scale, log2g, st, di, nullptr, zero, nzero);
            }
            if (ch == 8)
                return fit ? launch_row_quant_cfg<T, MODE, 8, true, false>(in, rows, K, s, q, scale, log2g, st, di, nullptr, zero, nzero)
                           : launch_row_quant_cfg<T, MODE, 8, false, false>(in, rows, K, s, q, scale, log2g, st, di, nullptr, zero, nzero);
            return fit ? launch_row_quant_cfg<T, MODE, 16, true, false>(in, rows, K, s, q, scale, log2g, st, di, nullptr, zero, nzero)
                       : launch_row_quant_cfg<T, MODE, 16, false, false>(in, rows, K, s, q, scale, log2g, st, di, nullptr, zero, nzero);
        }
    }
    sq_status r = (K * (int64_t)sizeof(float) <= kSmemFactorBytes)
                      ? launch_row_scale<T, MODE, true>(in, rows, K, s, scale, st, di)
                      : launch_row_scale<T, MODE, false>(in, rows, K, s, scale, st, di);
    if (r != SQ_OK)
        return r;
    const int64_t chunks = K / V;
    const int threads = static_cast<int>(std::min<int64_t>(256, (chunks + 31) / 32 * 32));
    const int64_t col_blocks = (chunks + threads - 1) / threads;
    const int64_t want = std::max<int64_t>(1, (int64_t)di.sms * 8 * 256 / threads / col_blocks);
    int64_t rpb = std::max<int64_t>(4, (rows + want - 1) / want);
    int64_t row_blocks = (rows + rpb - 1) / rpb;
    while (row_blocks > 65535) {
        rpb *= 2;
        row_blocks = (rows + rpb - 1) / rpb;
    }
    dim3 grid(static_cast<unsigned>(col_blocks), static_cast<unsigned>(row_blocks));
    return launch_kernel(sq::row_codes_kernel<T, MODE>, grid, dim3(threads), 0, st, 0, 0, in, rows, K, s,
                         static_cast<const float *>(scale), rpb, q, zero, nzero);
}

int64_t max_quant_k(sq_dtype dt) { return dt == SQ_BF16 ? 65536 : 32768; }

// ---- GEMM ------------------------------------------------------------------
template <int BN, int STAGES, int OUT, bool SWAP>
sq_status launch_gemm_cfg(const int8_t *xq, const float *sx, const int8_t *wq, const float *sw,
                          int64_t M, int64_t N, int64_t K, void *y, cudaStream_t st)
{
    using Cfg = sq::GemmCfg<BN, STAGES>;
    DeviceInfo di;
    if (!device_info(di))
        return SQ_ERR_CUDA;
    CUtensorMap ta, tb;
    const int8_t *a = SWAP ? wq : xq;
    const int8_t *b = SWAP ? xq : wq;
    const int64_t ra = SWAP ? N : M;
    const int64_t rb = SWAP ? M : N;
    if (!make_tmap_i8(&ta, a, ra, K, sq::kBM) || !make_tmap_i8(&tb, b, rb, K, BN))
        return SQ_ERR_CUDA;
    auto kernel = sq::gemm_i8_kernel<BN, STAGES, OUT, SWAP>;
    static std::atomic<uint64_t> attr_done{0};
    if (!ensure_smem_attr(kernel, Cfg::SMEM_BYTES, attr_done))
        return SQ_ERR_CUDA;
    const int64_t tiles = ((ra + sq::kBM - 1) / sq::kBM) * ((rb + BN - 1) / BN);
    const unsigned grid = static_cast<unsigned>(std::min<int64_t>(tiles, di.sms));
    return launch_kernel(kernel, dim3(grid), dim3(sq::kGemmThreads), Cfg::SMEM_BYTES, st, 0, 0, ta, tb, sx, sw, y,
                         static_cast<int>(M), static_cast<int>(N), static_cast<int>(K));
}

// ---- split-K small-M GEMM (optionally with the activation quant fused in) --
constexpr int64_t kFusedSliceBytes = 128 * 1024;  // resident token operand per CTA

struct SplitPlan {
    int splits = 1, kbps = 1, stages = 2, smem = 0, kbs = 1;
    bool ok = false;
};

// Clusters of `csize` CTAs of `threads` threads and `smem` bytes each that the
// device can hold at once (cudaOccupancyMaxActiveClusters), cached per kernel
// and shape.
template <typename KernelT>
int active_clusters(KernelT kernel, int csize, int smem, int threads)
{
    static std::mutex mu;
    struct Entry {
        const void *fn;
        int dev, csize, smem, threads, n;
    };
    static std::vector<Entry> cache;
    int dev = 0;
    cudaGetDevice(&dev);
    const void *fn = reinterpret_cast<const void *>(kernel);
    {
        std::lock_guard<std::mutex> lk(mu);
        for (auto &e : cache)
            if (e.fn == fn && e.dev == dev && e.csize == csize && e.smem == smem && e.threads == threads)
                return e.n;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(csize * 64));
    cfg.blockDim = dim3(static_cast<unsigned>(threads));
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = csize;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, kernel, &cfg) != cudaSuccess) {
        cudaGetLastError();
        n = 0;
    }
    std::lock_guard<std::mutex> lk(mu);
    cache.push_back(Entry{fn, dev, csize, smem, threads, n});
    return n;
}

template <int BNX, bool FUSED, typename KernelT>
SplitPlan plan_splitk(KernelT kernel, int64_t N, int64_t K)
{
    SplitPlan best;
    const int64_t n_tiles = (N + sq::kBM - 1) / sq::kBM;
    const int64_t k_blocks = (K + sq::kBK - 1) / sq::kBK;
    int64_t best_cost = INT64_MAX;
    // tuning overrides (same work, different decomposition): SQ_SPLITK_SPLITS, SQ_SPLITK_STAGES
    static const int force_splits = std::getenv("SQ_SPLITK_SPLITS") ? std::atoi(std::getenv("SQ_SPLITK_SPLITS")) : 0;
    static const int force_stages = std::getenv("SQ_SPLITK_STAGES") ? std::atoi(std::getenv("SQ_SPLITK_STAGES")) : 0;
    static const int force_kbs = std::getenv("SQ_SPLITK_KBS") ? std::atoi(std::getenv("SQ_SPLITK_KBS")) : 0;
    const int kbs = force_kbs > 0 ? force_kbs : 1;
    for (int64_t want = 1; want <= std::min<int64_t>(sq::kMaxSplits, k_blocks); ++want) {
        if (force_splits > 0 && want != force_splits)
            continue;
        const int64_t kbps = (k_blocks + want - 1) / want;
        const int64_t sp = (k_blocks + kbps - 1) / kbps;
        if (sp != want)
            continue;
        if (FUSED && (int64_t)BNX * sq::kBK * kbps > kFusedSliceBytes)
            continue;
        int stages = force_stages > 1 ? force_stages : 8;
        while (stages > 2 &&
               sq::split_layout<BNX>(stages, FUSED, (int)kbps, kbs).total + 1024 > (uint32_t)kMaxDynSmem)
            --stages;
        const int smem = (int)sq::split_layout<BNX>(stages, FUSED, (int)kbps, kbs).total + 1024;
        if (smem > kMaxDynSmem)
            continue;
        const int active = active_clusters(kernel, (int)sp, smem, sq::kSplitThreads);
        if (active <= 0)
            continue;
        const int64_t waves = (n_tiles + active - 1) / active;
        const int64_t cost = waves * (kbps + 4);  // +4: fixed per-CTA cost in k-block units
        if (cost < best_cost) {
            best_cost = cost;
            best.splits = (int)sp;
            best.kbps = (int)kbps;
            best.stages = stages;
            best.smem = smem;
            best.kbs = kbs;
            best.ok = true;
        }
    }
    return best;
}

template <int BNX, int OUT, bool FUSED, typename TIN, bool LSU = false>
sq_status launch_splitk_cfg(const TIN *x, const float *s, const int8_t *xq, const float *sx,
                            const int8_t *wq, const float *sw, int64_t M, int64_t N, int64_t K,
                            void *y, cudaStream_t st)
{
    auto kernel = sq::gemm_splitk_kernel<BNX, OUT, FUSED, TIN, LSU>;
    static std::atomic<uint64_t> attr_done{0};
    if (!ensure_smem_attr(kernel, kMaxDynSmem, attr_done))
        return SQ_ERR_CUDA;
    const SplitPlan p = plan_splitk<BNX, FUSED>(kernel, N, K);
    if (!p.ok || (LSU && p.kbs != 1))
        return SQ_ERR_UNSUPPORTED;
    if (debug_plan())
        std::fprintf(stderr, "[sq] splitk BNX=%d fused=%d M=%lld N=%lld K=%lld: splits=%d kb/split=%d stages=%d kbs=%d smem=%d clusters=%lld active=%d\n",
                     BNX, (int)FUSED, (long long)M, (long long)N, (long long)K, p.splits, p.kbps, p.stages, p.kbs, p.smem,
                     (long long)((N + sq::kBM - 1) / sq::kBM), active_clusters(kernel, p.splits, p.smem, sq::kSplitThreads));
    CUtensorMap tw, tx;
    if (!make_tmap_i8(&tw, wq, N, K, sq::kBM))
        return SQ_ERR_CUDA;
    if (FUSED)
        tx = tw;  // unused by the fused kernel
    else if (!make_tmap_i8(&tx, xq, M, K, BNX))
        return SQ_ERR_CUDA;
    const int64_t n_tiles = (N + sq::kBM - 1) / sq::kBM;
    return launch_kernel(kernel, dim3(static_cast<unsigned>(n_tiles * p.splits)), dim3(sq::kSplitThreads), p.smem, st,
                         p.splits, 1, tw, tx, wq, xq, x, s, sx, sw, y, static_cast<int>(M), static_cast<int>(N),
                         static_cast<int>(K), p.splits, p.kbps, p.stages, p.kbs);
}

size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// ---- the few-token GEMM of sq_linear: a stream over the weight -------------
// sq_linear runs it for M <= kDecodeMaxM; its int32 partials and tile
// counters live in the workspace after the codes and scales.
constexpr int64_t kDecodeMaxM = 128;
constexpr int64_t kDecodeMaxCtas = 160;  // at least the SM count of every sm_100 part

inline int decode_bnx(int64_t M) { return M <= 32 ? 32 : (M <= 64 ? 64 : 128); }

inline int64_t decode_units(int64_t N, int64_t K) { return ((N + sq::kBM - 1) / sq::kBM) * ((K + sq::kBK - 1) / sq::kBK); }


// Workspace of the GEMM when it has one (sq_w8a8_gemm_ws, and sq_linear after
// its codes and scales): tile counters, then partial-sum slots.
//   few tokens (M <= kDecodeMaxM): counters [T], slots [G, 2, BNX, 128];
//   more: counters [4 * kMaxPairs], slots [2 * kMaxPairs, 2, 128, 256].
constexpr int64_t kMaxPairs = 80;  // CTA pairs of the pair kernel a device can hold at once (sm_100: at most 80)

struct GemmWs {
    size_t cnt = 0, slots = 0, total = 0;
    int ncnt = 0;  // counters to clear before each call
};

inline GemmWs gemm_ws_layout(int64_t M, int64_t N, int64_t K, size_t base)
{
    GemmWs w;
    size_t o = base;
    w.cnt = o;
    if (M <= kDecodeMaxM) {
        const int64_t T = (N + sq::kBM - 1) / sq::kBM;
        const int64_t G = std::min<int64_t>(decode_units(N, K), kDecodeMaxCtas);
        w.ncnt = static_cast<int>(T);
        o += align_up(static_cast<size_t>(T) * sizeof(int), 256);
        w.slots = o;
        o += static_cast<size_t>(G) * 2 * decode_bnx(M) * sq::kBM * sizeof(int32_t);
    } else {
        w.ncnt = static_cast<int>(4 * kMaxPairs);
        o += align_up(static_cast<size_t>(w.ncnt) * sizeof(int), 256);
        w.slots = o;
        o += static_cast<size_t>(2 * kMaxPairs) * 2 * 128 * 256 * sizeof(int32_t);
    }
    w.total = o;
    return w;
}

// Workspace of sq_linear: codes [M, K] and scales [M] (the minimum), then the
// GEMM's workspace (used when the caller's workspace holds it too).
struct LinearWs {
    size_t xq = 0, sx = 0, minimum = 0;
    GemmWs g;
};

inline LinearWs linear_ws_layout(int64_t M, int64_t N, int64_t K)
{
    LinearWs w;
    w.xq = 0;
    w.sx = align_up(static_cast<size_t>(M) * static_cast<size_t>(K), 256);
    w.minimum = w.sx + align_up(static_cast<size_t>(M) * sizeof(float), 256);
    w.g = gemm_ws_layout(M, N, K, w.minimum);
    return w;
}

// Shared memory one quantiser CTA of sq_quant_act takes for rows of K values
// (the decode GEMM leaves room for one next to it on an SM).
inline int64_t quant_smem_estimate(int64_t K, sq_dtype dt)
{
    const bool bb = dt == SQ_BF16 && sq::row_quant_smem(K, true) <= 64 * 1024;
    return sq::row_quant_smem(K, bb) + 1024;
}

// CTAs of the weight-streaming GEMM.  The units are cut into G equal
// ranges: with G = S * T (T tiles, S <= KB) every range lies inside one tile,
// so a CTA has one partial tile to sum through the workspace instead of up
// to two; with G = T / D (D dividing T, for T above the SM count) every range
// is D whole tiles and nothing is summed.  A shared tile's epilogue (stores,
// a release, a count, the reduction) costs, in units of streaming, a fixed
// kDecodeEpiUnits plus, per contributor, a part that grows with the tokens
// (its partial's bytes); G is the choice with the fewest units per CTA plus
// that cost.  Fitted to sq_linear calls on B200 (one call, L2 flushed): at
// 1 to 16 tokens three or four CTAs a 4096-long tile were best, at 32 two,
// from 64 one; with K = 14336 four at every token count; at 64 to 128
// tokens and N = 28672, two whole tiles a CTA (42 -> 36 us, 52 -> 40 us).
// Small layers, whose units number at most the SMs, were once cut one unit
// a CTA at no modelled reduction cost; costed like the rest they take fewer,
// longer ranges (64 x 1024 x 2048: 44 -> 19 us; 1 x 1040 x 3088: 21.5 ->
// 17.4 us; 128 x 2048 x 8192: 54 -> 40 us).
constexpr int64_t kDecodeEpiUnits = 4;
inline int64_t decode_epi_units(int64_t M, int64_t S) { return kDecodeEpiUnits + (1 + std::min<int64_t>(M, 64) / 8) * S; }

// Whether the few-token kernels request their first weight tiles before
// griddepcontrol.wait when the grid before is the library's quantiser
// (SQ_DECODE_PREWAIT=1).  Off by default: measured on B200 back to back,
// those loads compete with the quantiser for HBM and delay its completion,
// which every later step waits for (278 against 286 us for the 12-call decode
// workload as one CUDA graph).
inline bool decode_prewait()
{
    static const bool on = std::getenv("SQ_DECODE_PREWAIT") && std::atoi(std::getenv("SQ_DECODE_PREWAIT")) == 1;
    return on;
}

inline int64_t decode_ctas(int64_t M, int64_t N, int64_t K, int64_t sms)
{
    const int64_t T = (N + sq::kBM - 1) / sq::kBM, KB = (K + sq::kBK - 1) / sq::kBK, U = T * KB;
    static const int64_t force = std::getenv("SQ_DECODE_CTAS") ? std::atoll(std::getenv("SQ_DECODE_CTAS")) : 0;
    if (force > 0)
        return std::min(force, std::min(U, sms));
    int64_t best = 0, best_cost = INT64_MAX;
    if (U > sms) {
        // the stream cut over every SM: ranges of `per` units may span two
        // tiles, each tile shared by about KB / per + 1 CTAs; the first
        // partial tile's reduction overlaps the rest of the range, so the
        // second's costs in full and the first's its fixed part
        const int64_t per = (U + sms - 1) / sms;
        const int64_t shared = std::max<int64_t>(2, (KB + per - 1) / per + 1);
        best = sms;
        best_cost = per + decode_epi_units(M, shared) + kDecodeEpiUnits;
    }
    for (int64_t S = 1; S <= KB && S * T <= sms; ++S) {
        const int64_t cost = (KB + S - 1) / S + (S > 1 ? decode_epi_units(M, S) : 0);
        if (cost < best_cost) {
            best_cost = cost;
            best = S * T;
        }
    }
    for (int64_t D = 2; D <= T && T > sms; ++D) {
        if (T % D != 0 || T / D > sms)
            continue;
        const int64_t cost = D * KB;
        if (cost < best_cost) {
            best_cost = cost;
            best = T / D;
        }
    }
    return best > 0 ? best : std::min(U, sms);
}

template <int BNX, int OUT>
sq_status launch_decode_cfg(const int8_t *xq, const float *sx, const int8_t *wq, const float *sw, int64_t M,
                            int64_t N, int64_t K, void *y, int *cnt, int32_t *slots, sq_dtype in_dt,
                            cudaStream_t st)
{
    using Cfg = sq::DecCfg<BNX>;
    DeviceInfo di;
    if (!device_info(di))
        return SQ_ERR_CUDA;
    const int64_t U = decode_units(N, K);
    const int G = static_cast<int>(decode_ctas(M, N, K, std::min<int64_t>(di.sms, kDecodeMaxCtas)));
    // the deepest ring that still leaves room for a quantiser CTA on the SM
    // (the two kernels overlap), within the per-CTA limit
    static const int force_stages = std::getenv("SQ_DECODE_STAGES") ? std::atoi(std::getenv("SQ_DECODE_STAGES")) : 0;
    const int64_t budget =
        std::min<int64_t>(kMaxDynSmem, kSmSmemBytes - 1024 - quant_smem_estimate(K, in_dt) - 1024);
    int stages = force_stages > 1 ? force_stages : 16;
    while (stages > 2 && sq::dec_smem_bytes(Cfg::STAGE_BYTES, stages) > budget)
        --stages;
    const int smem = sq::dec_smem_bytes(Cfg::STAGE_BYTES, stages);
    if (smem > kMaxDynSmem)
        return SQ_ERR_UNSUPPORTED;
    auto kernel = sq::gemm_decode_kernel<BNX, OUT>;
    static std::atomic<uint64_t> attr_done{0};
    if (!ensure_smem_attr(kernel, kMaxDynSmem, attr_done))
        return SQ_ERR_CUDA;
    CUtensorMap tw, tx;
    if (!make_tmap_i8(&tw, wq, N, K, sq::kBM) || !make_tmap_i8(&tx, xq, M, K, BNX))
        return SQ_ERR_CUDA;
    if (debug_plan())
        std::fprintf(stderr, "sq decode M=%lld N=%lld K=%lld: BNX=%d units=%lld ctas=%d stages=%d smem=%d\n",
                     (long long)M, (long long)N, (long long)K, BNX, (long long)U, G, stages, smem);
    // tuning override (same arithmetic): with the early weight loads on,
    // SQ_DECODE_L2PF=1 adds an L2 prefetch of the CTA's whole range (measured
    // on B200: it delays the quantiser's completion, and with it the wait, by
    // more than it saves for a 117 MB weight; neutral for 25 MB)
    static const int l2pf = std::getenv("SQ_DECODE_L2PF") ? std::atoi(std::getenv("SQ_DECODE_L2PF")) : 0;
    const bool prewait = decode_prewait();
    const int flags = (prewait ? 1 : 0) | (prewait && l2pf ? 2 : 0);
    return launch_kernel(kernel, dim3(static_cast<unsigned>(G)), dim3(sq::kDecThreads), smem, st, 0, 0, tw, tx, sx, sw,
                         y, slots, cnt, static_cast<int>(M), static_cast<int>(N), static_cast<int>(K), U, G, stages,
                         flags);
}

template <int OUT>
sq_status launch_decode(const int8_t *xq, const float *sx, const int8_t *wq, const float *sw, int64_t M, int64_t N,
                        int64_t K, void *y, int *cnt, int32_t *slots, sq_dtype in_dt, cudaStream_t st)
{
    switch (decode_bnx(M)) {
    case 32:
        return launch_decode_cfg<32, OUT>(xq, sx, wq, sw, M, N, K, y, cnt, slots, in_dt, st);
    case 64:
        return launch_decode_cfg<64, OUT>(xq, sx, wq, sw, M, N, K, y, cnt, slots, in_dt, st);
    default:
        return launch_decode_cfg<128, OUT>(xq, sx, wq, sw, M, N, K, y, cnt, slots, in_dt, st);
    }
}

// ---- the slab GEMM: at most 32 tokens, whole output channels per CTA -------
// Slabs are 16-channel groups, floor or ceil of R / G of them (R = N / 16);
// G is the fewest CTAs (at most one an SM) that give the narrowest widest
// slab, which is what sets the time.  Used where the narrower slab is at
// least kSlabMinNt channels wide and the wider one fits one MMA (256).  The
// MMA computes 128 token rows of which at most 32 are real, so the tensor
// pipe does 4 to 16 times the useful work, and a narrow slab needs many MMAs
// per weight byte: measured on B200, slabs of 32 or 48 channels are
// MMA-bound (4096 x 14336 at M = 1: 57 us against 26 us for the
// weight-streaming kernel), slabs of 192-208 are not far off the stream
// (28672 x 4096: 30.7 against 31.8-33.9 us, the difference being the
// stream's cross-CTA reduction).  SQ_DECODE_SLAB=0 turns it off.
constexpr int64_t kSlabMinNt = 128;
struct SlabPlan {
    int G = 0, nt_lo = 0, nt_hi = 0;
};

inline SlabPlan plan_slab(int64_t M, int64_t N, int64_t sms)
{
    SlabPlan p;
    static const bool on = !(std::getenv("SQ_DECODE_SLAB") && std::atoi(std::getenv("SQ_DECODE_SLAB")) == 0);
    static const int64_t force = std::getenv("SQ_SLAB_CTAS") ? std::atoll(std::getenv("SQ_SLAB_CTAS")) : 0;
    if (!on || M > 32 || N % 16 != 0)
        return p;
    const int64_t R = N / 16, gmax = std::min<int64_t>(R, sms);
    const int64_t widest = (R + gmax - 1) / gmax;
    if (16 * widest > sq::kSlabMaxNt || 16 * (R / gmax) < kSlabMinNt)
        return p;
    int64_t G = (R + widest - 1) / widest;  // fewest CTAs with that widest slab
    if (force > 0)
        G = std::min<int64_t>(force, gmax);
    p.G = static_cast<int>(G);
    p.nt_lo = static_cast<int>(16 * (R / G));
    p.nt_hi = static_cast<int>(16 * ((R + G - 1) / G));
    return p;
}

inline bool slab_applies(int64_t M, int64_t N)
{
    DeviceInfo di;
    if (!device_info(di))
        return false;
    return plan_slab(M, N, di.sms).G > 0;
}

template <int BNX, int OUT>
sq_status launch_slab_cfg(const int8_t *xq, const float *sx, const int8_t *wq, const float *sw, int64_t M, int64_t N,
                          int64_t K, void *y, sq_dtype in_dt, bool after_quant, cudaStream_t st)
{
    DeviceInfo di;
    if (!device_info(di))
        return SQ_ERR_CUDA;
    const SlabPlan p = plan_slab(M, N, di.sms);
    if (p.G == 0)
        return SQ_ERR_UNSUPPORTED;
    static const int force_kbs = std::getenv("SQ_SLAB_KBS") ? std::atoi(std::getenv("SQ_SLAB_KBS")) : 0;
    const int kbs = force_kbs > 0 ? force_kbs : 2;
    // the deepest ring that fits; after the library's quantiser, one that
    // still leaves room for a quantiser CTA on the SM (the kernels overlap)
    const int64_t budget = after_quant ? std::min<int64_t>(kMaxDynSmem, kSmSmemBytes - 1024 -
                                                                            quant_smem_estimate(K, in_dt) - 1024)
                                       : kMaxDynSmem;
    int stages = 16;
    while (stages > 2 && sq::slab_smem_bytes(BNX, p.nt_hi, stages, kbs) > budget)
        --stages;
    const int smem = sq::slab_smem_bytes(BNX, p.nt_hi, stages, kbs);
    if (smem > kMaxDynSmem)
        return SQ_ERR_UNSUPPORTED;
    auto kernel = sq::gemm_slab_kernel<BNX, OUT>;
    static std::atomic<uint64_t> attr_done{0};
    if (!ensure_smem_attr(kernel, kMaxDynSmem, attr_done))
        return SQ_ERR_CUDA;
    CUtensorMap tlo, thi, tx;
    if (!make_tmap_i8(&tlo, wq, N, K, p.nt_lo) || !make_tmap_i8(&thi, wq, N, K, p.nt_hi) ||
        !make_tmap_i8(&tx, xq, M, K, BNX))
        return SQ_ERR_CUDA;
    if (debug_plan())
        std::fprintf(stderr, "sq slab M=%lld N=%lld K=%lld: BNX=%d ctas=%d nt=%d/%d kbs=%d stages=%d smem=%d pre=%d\n",
                     (long long)M, (long long)N, (long long)K, BNX, p.G, p.nt_lo, p.nt_hi, kbs, stages, smem,
                     (int)after_quant);
    return launch_kernel(kernel, dim3(static_cast<unsigned>(p.G)), dim3(sq::kSlabThreads), smem, st, 0, 0, tlo, thi,
                         tx, sx, sw, y, static_cast<int>(M), static_cast<int>(N), static_cast<int>(K), p.G, p.nt_hi,
                         stages, kbs, (after_quant && decode_prewait()) ? 1 : 0);
}

template <int OUT>
sq_status launch_slab(const int8_t *xq, const float *sx, const int8_t *wq, const float *sw, int64_t M, int64_t N,
                      int64_t K, void *y, sq_dtype in_dt, bool after_quant, cudaStream_t st)
{
    if (M <= 8)
        return launch_slab_cfg<8, OUT>(xq, sx, wq, sw, M, N, K, y, in_dt, after_quant, st);
    if (M <= 16)
        return launch_slab_cfg<16, OUT>(xq, sx, wq, sw, M, N, K, y, in_dt, after_quant, st);
    return launch_slab_cfg<32, OUT>(xq, sx, wq, sw, M, N, K, y, in_dt, after_quant, st);
}

// The stream-K tail of the pair GEMM is off unless SQ_GEMM_SK=1: measured on
// B200 it is slower than whole tiles (1024 x 6144 x 4096: 52 against 35 us;
// 4096 x 6144 x 4096: 93 against 74 us), because the partial sums' reduction
// (a 128 x 256 int32 slot per contributor, read back by the last one) sits at
// the end of the critical path.
bool gemm_sk_enabled()
{
    static const bool on = std::getenv("SQ_GEMM_SK") && std::atoi(std::getenv("SQ_GEMM_SK")) == 1;
    return on;
}

// Prefill GEMM on CTA pairs: 256 x BN output tiles, persistent over tiles.
// With a workspace (slots, cnt not null) and tiles that do not fill whole
// rounds of the co-resident pairs, the last round and the partial one are
// done stream-K: their k blocks are cut into one equal range per pair, and
// tiles shared by several pairs are summed through int32 partials.
// The pair GEMM takes its tiles in groups of kPairGroupM m blocks (m fastest
// within a group, then n; see pair_tile_mn): fewer operand re-reads from DRAM.  In the
// Llama-3-70B step under the 1 kW power cap this mattered for K = 8192 as well
// (2736 -> 2854 TOPS, three interleaved runs each on one B200), though a
// single K = 8192 GEMM timed alone was no faster: the re-reads cost DRAM power.
constexpr int kPairGroupM = 8;

template <int BN, int STAGES, int OUT>
sq_status launch_gemm_pair_cfg(const int8_t *xq, const float *sx, const int8_t *wq, const float *sw,
                               int64_t M, int64_t N, int64_t K, void *y, cudaStream_t st, int32_t *slots = nullptr,
                               int *cnt = nullptr)
{
    using Cfg = sq::PairCfg<BN, STAGES>;
    CUtensorMap ta, tb;
    if (!make_tmap_i8(&ta, xq, M, K, 128) || !make_tmap_i8(&tb, wq, N, K, BN / 2))
        return SQ_ERR_CUDA;
    auto kernel = sq::gemm_i8_pair_kernel<BN, STAGES, OUT>;
    static std::atomic<uint64_t> attr_done{0};
    if (!ensure_smem_attr(kernel, Cfg::SMEM_BYTES, attr_done))
        return SQ_ERR_CUDA;
    const int active = std::min<int>(active_clusters(kernel, 2, Cfg::SMEM_BYTES, sq::kPairThreads),
                                     static_cast<int>(kMaxPairs));
    if (active <= 0)
        return SQ_ERR_CUDA;
    const int64_t tiles = ((M + sq::kPairBM - 1) / sq::kPairBM) * ((N + BN - 1) / BN);
    const int64_t kb = (K + sq::kBK - 1) / sq::kBK;
    int64_t pairs = std::min<int64_t>(tiles, active);
    int64_t sk_first = tiles, sk_units = 0;
    if (slots != nullptr && cnt != nullptr && gemm_sk_enabled() && tiles % active != 0) {
        // the last full round and the partial one; with fewer tiles than
        // pairs, all of them (and no more pairs than units, so that every
        // pair has some)
        const int64_t full = tiles / active;
        sk_first = full >= 1 ? (full - 1) * active : 0;
        sk_units = (tiles - sk_first) * kb;
        pairs = full >= 1 ? active : std::min<int64_t>(active, sk_units);
    }
    if (debug_plan())
        std::fprintf(stderr, "sq gemm pair M=%lld N=%lld K=%lld: BN=%d stages=%d tiles=%lld pairs=%lld sk_first=%lld sk_units=%lld\n",
                     (long long)M, (long long)N, (long long)K, BN, STAGES, (long long)tiles, (long long)pairs,
                     (long long)sk_first, (long long)sk_units);
    // tile order: groups of kPairGroupM m blocks; SQ_PAIR_GROUP_M overrides
    // (a value of at least the m block count gives the m-fastest order)
    static const int force_gm = std::getenv("SQ_PAIR_GROUP_M") ? std::atoi(std::getenv("SQ_PAIR_GROUP_M")) : 0;
    const int group_m = force_gm > 0 ? force_gm : kPairGroupM;
    return launch_kernel(kernel, dim3(static_cast<unsigned>(2 * pairs)), dim3(sq::kPairThreads), Cfg::SMEM_BYTES, st, 2,
                         1, ta, tb, sx, sw, y, static_cast<int>(M), static_cast<int>(N), static_cast<int>(K),
                         static_cast<int>(sk_first), sk_units, slots, cnt, std::max(group_m, 1));
}

// Tile width of the pair GEMM: the fewest rounds of tiles over the
// co-resident pairs, each round costing one tile's time.  Narrower tiles
// re-read more operand bytes per operation from L2, so a tile's time is not
// proportional to its width: measured on B200 (8192 x 28672 x 4096, many
// rounds), 256 / 192 / 128-wide tiles reach 0.94 / 0.81 / 0.62 of the int8
// peak, i.e. relative tile times 271 : 237 : 206.
inline int pick_pair_bn(int64_t M, int64_t N, int pairs)
{
    static const int force = std::getenv("SQ_GEMM_PAIR_BN") ? std::atoi(std::getenv("SQ_GEMM_PAIR_BN")) : -1;
    if (force >= 0)
        return force;
    // 224 and 160 are interpolated between the measured widths
    constexpr int cand[5] = {256, 224, 192, 160, 128};
    constexpr int64_t tile_time[5] = {271, 254, 237, 222, 206};
    int best = 256;
    int64_t best_cost = INT64_MAX;
    for (int i = 0; i < 5; ++i) {
        const int64_t tiles = ((M + sq::kPairBM - 1) / sq::kPairBM) * ((N + cand[i] - 1) / cand[i]);
        const int64_t rounds = (tiles + pairs - 1) / std::max(pairs, 1);
        const int64_t cost = rounds * tile_time[i];
        if (cost < best_cost) {
            best_cost = cost;
            best = cand[i];
        }
    }
    return best;
}

// The weight-streaming kernel runs for few tokens with a workspace unless
// SQ_DECODE_STREAM=0 (the split-K cluster kernel then): measured on B200 back
// to back, the two are within 1% of each other, the stream slightly ahead.
inline bool decode_stream_on()
{
    static const bool on = !(std::getenv("SQ_DECODE_STREAM") && std::atoi(std::getenv("SQ_DECODE_STREAM")) == 0);
    return on;
}


// The GEMM with or without a workspace (cnt, slots; null: none).
//   - Up to 32 tokens on wide layers: the slab kernel (no workspace).
//   - Up to kDecodeMaxM tokens otherwise: the split-K cluster kernel, or with
//     SQ_DECODE_STREAM=1 and a workspace the weight-streaming kernel, whose
//     tile counters the caller's kernel right before has cleared (the
//     quantiser, or the zeroing kernel of sq_w8a8_gemm_ws).
//   - More tokens: the pair kernel (with its stream-K tail under SQ_GEMM_SK=1
//     and a workspace).
// after_quant: the grid right before is the library's own quantiser, so the
// few-token kernels may request their first weight tiles before
// griddepcontrol.wait (that quantiser waited for every earlier grid).
template <int OUT>
sq_status launch_gemm(const int8_t *xq, const float *sx, const int8_t *wq, const float *sw,
                      int64_t M, int64_t N, int64_t K, void *y, cudaStream_t st, int *cnt = nullptr,
                      int32_t *slots = nullptr, sq_dtype in_dt = SQ_BF16, bool after_quant = false)
{
    const float *nf = nullptr;
    const bool ws = cnt != nullptr && slots != nullptr;
    if (slab_applies(M, N))
        return launch_slab<OUT>(xq, sx, wq, sw, M, N, K, y, in_dt, after_quant, st);
    if (ws && M <= kDecodeMaxM && decode_stream_on())
        return launch_decode<OUT>(xq, sx, wq, sw, M, N, K, y, cnt, slots, in_dt, st);
    // weight tiles through the load/store unit (cp.async) or TMA
    static const bool lsu = std::getenv("SQ_SPLITK_LSU") && std::atoi(std::getenv("SQ_SPLITK_LSU")) == 1;
    if (M <= 32)
        return lsu ? launch_splitk_cfg<32, OUT, false, float, true>(nf, nf, xq, sx, wq, sw, M, N, K, y, st)
                   : launch_splitk_cfg<32, OUT, false, float>(nf, nf, xq, sx, wq, sw, M, N, K, y, st);
    if (M <= 64)
        return lsu ? launch_splitk_cfg<64, OUT, false, float, true>(nf, nf, xq, sx, wq, sw, M, N, K, y, st)
                   : launch_splitk_cfg<64, OUT, false, float>(nf, nf, xq, sx, wq, sw, M, N, K, y, st);
    if (M <= 128)
        return lsu ? launch_splitk_cfg<128, OUT, false, float, true>(nf, nf, xq, sx, wq, sw, M, N, K, y, st)
                   : launch_splitk_cfg<128, OUT, false, float>(nf, nf, xq, sx, wq, sw, M, N, K, y, st);
    DeviceInfo di;
    if (!device_info(di))
        return SQ_ERR_CUDA;
    // with the stream-K tail, the widest (most efficient) tile throughout
    const int bn = (ws && gemm_sk_enabled() && !std::getenv("SQ_GEMM_PAIR_BN")) ? 256 : pick_pair_bn(M, N, di.sms / 2);
    switch (bn) {
    case 256:
        return launch_gemm_pair_cfg<256, 6, OUT>(xq, sx, wq, sw, M, N, K, y, st, slots, cnt);
    case 224:
        return launch_gemm_pair_cfg<224, 7, OUT>(xq, sx, wq, sw, M, N, K, y, st, slots, cnt);
    case 192:
        return launch_gemm_pair_cfg<192, 7, OUT>(xq, sx, wq, sw, M, N, K, y, st, slots, cnt);
    case 160:
        return launch_gemm_pair_cfg<160, 8, OUT>(xq, sx, wq, sw, M, N, K, y, st, slots, cnt);
    case 128:
        return launch_gemm_pair_cfg<128, 8, OUT>(xq, sx, wq, sw, M, N, K, y, st, slots, cnt);
    default:  // single-SM 128 x 256 tiles
        return launch_gemm_cfg<256, 4, OUT, false>(xq, sx, wq, sw, M, N, K, y, st);
    }
}

// The fused decode path (activation quant inside the GEMM, no workspace)
// applies to at most 32 tokens when K fits the per-CTA token operand, and
// only when selected.
bool fused_decode_applies(int64_t M, int64_t K)
{
    // off unless SQ_LINEAR_FUSED=1: on B200 the quantiser kernel followed by
    // the split-K GEMM (launch overlapped) is faster than quantising inside
    // the GEMM kernel's prologue
    static const bool on = std::getenv("SQ_LINEAR_FUSED") && std::atoi(std::getenv("SQ_LINEAR_FUSED")) == 1;
    return on && M <= 32 && K <= sq::kMaxSplits * (kFusedSliceBytes / (32 * sq::kBK)) * sq::kBK;
}

template <typename TIN>
sq_status launch_fused_linear(const TIN *x, const float *s, const int8_t *wq, const float *sw,
                              int64_t M, int64_t N, int64_t K, void *y, sq_dtype out_dt,
                              cudaStream_t st)
{
    if (out_dt == SQ_BF16)
        return launch_splitk_cfg<32, OUT_BF16, true, TIN>(x, s, nullptr, nullptr, wq, sw, M, N, K, y, st);
    return launch_splitk_cfg<32, OUT_F32, true, TIN>(x, s, nullptr, nullptr, wq, sw, M, N, K, y, st);
}

constexpr int64_t kMaxDim = 2147483647LL;

sq_status check_gemm_dims(int64_t M, int64_t N, int64_t K)
{
    if (M < 1 || N < 16 || K < 16 || N % 16 != 0 || K % 16 != 0)
        return SQ_ERR_INVALID_ARG;
    if (M > kMaxDim || N > kMaxDim || K > 133144)
        return SQ_ERR_UNSUPPORTED;
    return SQ_OK;
}

// ---- fixed scratch for sq_linear_noalloc -----------------------------------
// The array belongs to this translation unit; in host code its name only
// stands in for the symbol, so the device address is looked up once per
// device with cudaGetSymbolAddress and handed to the kernels as a pointer.
static __device__ __align__(256) uint8_t g_linear_noalloc_scratch[SQ_LINEAR_NOALLOC_SCRATCH_BYTES];

// Device address of the scratch array on the current device (looked up on the
// first call for that device), or nullptr if the lookup fails.
void *noalloc_scratch()
{
    static void *addr[kMaxDevices] = {};
    static std::mutex mu;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
        return nullptr;
    std::lock_guard<std::mutex> lk(mu);
    if (addr[dev] == nullptr) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_linear_noalloc_scratch) != cudaSuccess) {
            cudaGetLastError();
            return nullptr;
        }
        addr[dev] = p;
    }
    return addr[dev];
}

// Fused RMSNorm + quantiser: 2^log2g warps per row, CH chunks per lane.
template <typename T, int CH>
sq_status launch_rmsnorm_quant_cfg(const T *h, int64_t rows, int64_t K, const float *g, float eps, int8_t *q,
                                   float *sx, float *rinv, int log2g, cudaStream_t st, const DeviceInfo &di)
{
    auto kernel = sq::rmsnorm_quant_kernel<T, CH>;
    const int smem = static_cast<int>(K * 4);
    static std::atomic<uint64_t> attr_done{0};
    if (!ensure_smem_attr(kernel, kMaxDynSmem - 1024, attr_done))
        return SQ_ERR_CUDA;
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, sq::kQuantThreads, smem) != cudaSuccess ||
        per_sm < 1) {
        cudaGetLastError();
        return SQ_ERR_CUDA;
    }
    while (log2g < 3 && rows * (1 << log2g) < (int64_t)di.sms * per_sm * (sq::kQuantThreads / 32))
        ++log2g;
    const int slots = (sq::kQuantThreads / 32) >> log2g;
    const int64_t blocks = std::min<int64_t>((rows + slots - 1) / slots, (int64_t)per_sm * di.sms);
    return launch_kernel(kernel, dim3(static_cast<unsigned>(blocks)), dim3(sq::kQuantThreads), smem, st, 0, 0, h, rows,
                         K, g, eps, log2g, q, sx, rinv);
}

template <typename T>
sq_status launch_rmsnorm_quant(const T *h, int64_t rows, int64_t K, const float *g, float eps, int8_t *q, float *sx,
                               float *rinv, cudaStream_t st)
{
    DeviceInfo di;
    if (!device_info(di))
        return SQ_ERR_CUDA;
    constexpr int V = sq::Vec<T>::N;
    const int64_t nch = K / V;
    for (int ch : {8, 16}) {
        int log2g = 0;
        while (log2g < 3 && ((int64_t)32 * ch << log2g) < nch)
            ++log2g;
        if (((int64_t)32 * ch << log2g) < nch)
            continue;
        return ch == 8 ? launch_rmsnorm_quant_cfg<T, 8>(h, rows, K, g, eps, q, sx, rinv, log2g, st, di)
                       : launch_rmsnorm_quant_cfg<T, 16>(h, rows, K, g, eps, q, sx, rinv, log2g, st, di);
    }
    return SQ_ERR_UNSUPPORTED;
}

}  // namespace

// ---------------------------------------------------------------------------
// GPTQ (offline weight rounding)
// ---------------------------------------------------------------------------
constexpr int64_t kGptqMaxK = 16384;  // H is K x K fp64 (2 GiB at the limit)

template <typename T>
sq_status launch_gptq_hessian(const T *x, int64_t ntok, int64_t K, const float *s, double *H, cudaStream_t st)
{
    const unsigned nb = static_cast<unsigned>((K + sq::kGptqHT - 1) / sq::kGptqHT);
    return launch_kernel(sq::gptq_hessian_kernel<T>, dim3(nb, nb), dim3(256), 0, st, 0, 0, x, ntok, K, s, H);
}

template <typename T, bool STAGE>
sq_status launch_gptq_rows_cfg(const T *w, int64_t N, int64_t K, const float *s, const double *U, int8_t *wq,
                               float *sw, cudaStream_t st)
{
    auto kernel = sq::gptq_rows_kernel<T, STAGE>;
    static std::atomic<uint64_t> attr_done{0};
    if (!ensure_smem_attr(kernel, kMaxDynSmem - 1024, attr_done))
        return SQ_ERR_CUDA;
    // one warp per row, the rows (and with STAGE two rows of U) in shared memory as fp64
    const int64_t avail = kMaxDynSmem - 1024 - (STAGE ? 2 * K * 8 : 0);
    const int64_t per_cta = std::max<int64_t>(1, std::min<int64_t>(8, avail / (K * 8)));
    const int smem = static_cast<int>((per_cta + (STAGE ? 2 : 0)) * K * 8);
    const unsigned blocks = static_cast<unsigned>((N + per_cta - 1) / per_cta);
    return launch_kernel(kernel, dim3(blocks), dim3(static_cast<unsigned>(32 * per_cta)), smem, st, 0, 0, w, N, K, s,
                         U, wq, sw);
}

template <typename T>
sq_status launch_gptq_rows(const T *w, int64_t N, int64_t K, const float *s, const double *U, int8_t *wq, float *sw,
                           cudaStream_t st)
{
    // staging U needs room for a row of the weight and two rows of U
    // (SQ_GPTQ_STAGE=0 reads U from L2 instead, as longer rows must)
    static const bool no_stage = std::getenv("SQ_GPTQ_STAGE") && std::atoi(std::getenv("SQ_GPTQ_STAGE")) == 0;
    if (!no_stage && 3 * K * 8 <= kMaxDynSmem - 1024)
        return launch_gptq_rows_cfg<T, true>(w, N, K, s, U, wq, sw, st);
    return launch_gptq_rows_cfg<T, false>(w, N, K, s, U, wq, sw, st);
}

extern "C" {

const char *sq_status_string(sq_status st)
{
    switch (st) {
    case SQ_OK:
        return "SQ_OK";
    case SQ_ERR_INVALID_ARG:
        return "SQ_ERR_INVALID_ARG";
    case SQ_ERR_UNSUPPORTED:
        return "SQ_ERR_UNSUPPORTED";
    case SQ_ERR_CUDA:
        return "SQ_ERR_CUDA";
    case SQ_ERR_TIMEOUT:
        return "SQ_ERR_TIMEOUT";
    }
    return "SQ_ERR_UNKNOWN";
}

int sq_version(void) { return 100; }

sq_status sq_calib_absmax(const void *x, sq_dtype dt, int64_t T, int64_t K, int64_t ldx, float *ax,
                          sq_stream_t stream)
{
    if (x == nullptr || ax == nullptr || !valid_dtype(dt) || T < 1 || K < 16 || K % 16 != 0 ||
        ldx < K || (ldx * static_cast<int64_t>(dtype_size(dt))) % 16 != 0 || !aligned16(x) ||
        !aligned16(ax))
        return SQ_ERR_INVALID_ARG;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (dt == SQ_BF16)
        return launch_col_absmax(static_cast<const __nv_bfloat16 *>(x), T, K, ldx, ax, st);
    return launch_col_absmax(static_cast<const float *>(x), T, K, ldx, ax, st);
}

sq_status sq_smooth_factors(const float *ax, const void *w, sq_dtype dt, int64_t N, int64_t K,
                            float alpha, float *s, float *aw, sq_stream_t stream)
{
    if (ax == nullptr || w == nullptr || s == nullptr || !valid_dtype(dt) || N < 1 || K < 16 ||
        K % 16 != 0 || !aligned16(ax) || !aligned16(w) || !aligned16(s) ||
        (aw != nullptr && !aligned16(aw)) || !(alpha >= 0.0f && alpha <= 1.0f) || s == ax ||
        aw == ax || (aw != nullptr && aw == s))
        return SQ_ERR_INVALID_ARG;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    // B_j accumulates into s (as fp32 bit patterns), then s is overwritten in place.
    const int threads = 256;
    const unsigned blocks = static_cast<unsigned>((K + threads - 1) / threads);
    sq_status r = launch_kernel(sq::zero_f32_kernel, dim3(blocks), dim3(threads), 0, st, 0, 0, s, K);
    if (r != SQ_OK)
        return r;
    r = (dt == SQ_BF16)
                      ? launch_col_absmax(static_cast<const __nv_bfloat16 *>(w), N, K, K, s, st)
                      : launch_col_absmax(static_cast<const float *>(w), N, K, K, s, st);
    if (r != SQ_OK)
        return r;
    return launch_kernel(sq::smooth_factors_kernel, dim3(blocks), dim3(threads), 0, st, 0, 0, ax, s, aw, K, alpha);
}

sq_status sq_smooth_quant_weight(const void *w, sq_dtype dt, int64_t N, int64_t K, const float *s,
                                 int8_t *wq, float *sw, sq_stream_t stream)
{
    if (w == nullptr || s == nullptr || wq == nullptr || sw == nullptr || !valid_dtype(dt) ||
        N < 1 || K < 16 || K % 16 != 0 || !aligned16(w) || !aligned16(s) || !aligned16(wq) ||
        !aligned16(sw))
        return SQ_ERR_INVALID_ARG;
    if (K > max_quant_k(dt) || N > kMaxDim)
        return SQ_ERR_UNSUPPORTED;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (dt == SQ_BF16)
        return launch_quant_rows<__nv_bfloat16, sq::MODE_W>(static_cast<const __nv_bfloat16 *>(w),
                                                             N, K, s, wq, sw, st);
    return launch_quant_rows<float, sq::MODE_W>(static_cast<const float *>(w), N, K, s, wq, sw, st);
}

sq_status sq_quant_act(const void *x, sq_dtype dt, int64_t M, int64_t K, const float *s,
                       int8_t *xq, float *sx, sq_stream_t stream)
{
    if (x == nullptr || s == nullptr || xq == nullptr || sx == nullptr || !valid_dtype(dt) ||
        M < 1 || K < 16 || K % 16 != 0 || !aligned16(x) || !aligned16(s) || !aligned16(xq) ||
        !aligned16(sx))
        return SQ_ERR_INVALID_ARG;
    if (K > max_quant_k(dt) || M > kMaxDim)
        return SQ_ERR_UNSUPPORTED;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (dt == SQ_BF16)
        return launch_quant_rows<__nv_bfloat16, sq::MODE_X>(static_cast<const __nv_bfloat16 *>(x),
                                                             M, K, s, xq, sx, st);
    return launch_quant_rows<float, sq::MODE_X>(static_cast<const float *>(x), M, K, s, xq, sx, st);
}

sq_status sq_fold_gamma(const float *gamma, const float *s, int64_t K, float *g, sq_stream_t stream)
{
    if (gamma == nullptr || s == nullptr || g == nullptr || K < 16 || K % 16 != 0 || !aligned16(gamma) ||
        !aligned16(s) || !aligned16(g))
        return SQ_ERR_INVALID_ARG;
    if (K > kMaxDim)
        return SQ_ERR_UNSUPPORTED;
    const unsigned threads = 256;
    const unsigned blocks = static_cast<unsigned>((K + threads - 1) / threads);
    return launch_kernel(sq::fold_gamma_kernel, dim3(blocks), dim3(threads), 0, reinterpret_cast<cudaStream_t>(stream),
                         0, 0, gamma, s, g, K);
}

sq_status sq_rmsnorm_quant(const void *h, sq_dtype dt, int64_t M, int64_t K, const float *g, float eps,
                           int8_t *xq, float *sx, float *rinv, sq_stream_t stream)
{
    if (h == nullptr || g == nullptr || xq == nullptr || sx == nullptr || !valid_dtype(dt) || M < 1 || K < 16 ||
        K % 16 != 0 || !aligned16(h) || !aligned16(g) || !aligned16(xq) || !aligned16(sx) ||
        (rinv != nullptr && !aligned16(rinv)) || !(eps >= 0.0f) || !(eps <= 3.0e38f))
        return SQ_ERR_INVALID_ARG;
    // one row of 16 chunks per lane over 8 warps; g staged in shared memory
    const int64_t kmax = dt == SQ_BF16 ? 32768 : 16384;
    if (K > kmax || M > kMaxDim)
        return SQ_ERR_UNSUPPORTED;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (dt == SQ_BF16)
        return launch_rmsnorm_quant(static_cast<const __nv_bfloat16 *>(h), M, K, g, eps, xq, sx, rinv, st);
    return launch_rmsnorm_quant(static_cast<const float *>(h), M, K, g, eps, xq, sx, rinv, st);
}

sq_status sq_silu_mul_quant(const void *gu, sq_dtype dt, int64_t M, int64_t I, const float *s, int8_t *xq,
                            float *sx, void *h, sq_stream_t stream)
{
    if (gu == nullptr || s == nullptr || xq == nullptr || sx == nullptr || !valid_dtype(dt) || M < 1 || I < 16 ||
        I % 16 != 0 || !aligned16(gu) || !aligned16(s) || !aligned16(xq) || !aligned16(sx) ||
        (h != nullptr && !aligned16(h)))
        return SQ_ERR_INVALID_ARG;
    const int64_t imax = dt == SQ_BF16 ? 32768 : 16384;
    if (I > imax || M > kMaxDim)
        return SQ_ERR_UNSUPPORTED;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (dt == SQ_BF16)
        return launch_glu_quant(static_cast<const __nv_bfloat16 *>(gu), M, I, s, xq, sx, static_cast<__nv_bfloat16 *>(h),
                                st);
    return launch_glu_quant(static_cast<const float *>(gu), M, I, s, xq, sx, static_cast<float *>(h), st);
}

size_t sq_gptq_workspace_size(int64_t K)
{
    if (K < 16 || K % 16 != 0 || K > kGptqMaxK)
        return 0;
    return 2 * static_cast<size_t>(K) * static_cast<size_t>(K) * sizeof(double);
}

sq_status sq_gptq_hessian(const void *x, sq_dtype dt, int64_t T, int64_t K, const float *s, double *H,
                          sq_stream_t stream)
{
    if (x == nullptr || s == nullptr || H == nullptr || !valid_dtype(dt) || T < 1 || K < 16 || K % 16 != 0 ||
        !aligned16(x) || !aligned16(s) || !aligned16(H))
        return SQ_ERR_INVALID_ARG;
    if (K > kGptqMaxK || T > kMaxDim)
        return SQ_ERR_UNSUPPORTED;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (dt == SQ_BF16)
        return launch_gptq_hessian(static_cast<const __nv_bfloat16 *>(x), T, K, s, H, st);
    return launch_gptq_hessian(static_cast<const float *>(x), T, K, s, H, st);
}

sq_status sq_gptq_factor(double *H, int64_t K, float damp_frac, double *U, void *workspace, size_t ws_bytes,
                         sq_stream_t stream)
{
    if (H == nullptr || U == nullptr || workspace == nullptr || K < 16 || K % 16 != 0 || !aligned16(H) ||
        !aligned16(U) || !aligned16(workspace) || !(damp_frac >= 0.0f) || !(damp_frac <= 1.0e30f) || H == U)
        return SQ_ERR_INVALID_ARG;
    if (K > kGptqMaxK)
        return SQ_ERR_UNSUPPORTED;
    if (ws_bytes < sq_gptq_workspace_size(K))
        return SQ_ERR_INVALID_ARG;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    double *Lr = static_cast<double *>(workspace);  // L, row-major
    double *Nt = Lr + K * K;                         // L^-1, column-major
    static std::atomic<uint64_t> attr_damp{0};
    // the damping kernel also holds a little static shared memory
    if (!ensure_smem_attr(sq::gptq_damp_kernel, kMaxDynSmem - 1024, attr_damp))
        return SQ_ERR_CUDA;
    const int W = sq::kGptqWarps;
    sq_status r = launch_kernel(sq::gptq_damp_kernel, dim3(1), dim3(sq::kGptqThreads), static_cast<int>(K * 8), st, 0,
                                0, H, K, damp_frac);
    // step t: column t of the Cholesky factor of the reversed H (one warp a
    // row) and row t - 1 of its inverse (one warp a column), one launch
    for (int64_t t = 0; t <= K && r == SQ_OK; ++t) {
        const int64_t chol_blocks = t < K ? (K - t + W - 1) / W : 0;
        const int64_t inv_blocks = t >= 1 ? (t + W - 1) / W : 0;
        r = launch_kernel(sq::gptq_factor_step_kernel, dim3(static_cast<unsigned>(chol_blocks + inv_blocks)),
                          dim3(32 * W), 0, st, 0, 0, static_cast<const double *>(H), K, t, chol_blocks, Lr, Nt);
    }
    // U = the inverse, reversed and transposed
    const unsigned tiles = static_cast<unsigned>((K + 31) / 32);
    if (r == SQ_OK)
        r = launch_kernel(sq::gptq_u_from_n_kernel, dim3(tiles, tiles), dim3(256), 0, st, 0, 0,
                          static_cast<const double *>(Nt), K, U);
    return r;
}

sq_status sq_gptq_quant_weight(const void *w, sq_dtype dt, int64_t N, int64_t K, const float *s, const double *U,
                               int8_t *wq, float *sw, sq_stream_t stream)
{
    if (w == nullptr || s == nullptr || U == nullptr || wq == nullptr || sw == nullptr || !valid_dtype(dt) || N < 1 ||
        K < 16 || K % 16 != 0 || !aligned16(w) || !aligned16(s) || !aligned16(U) || !aligned16(wq) ||
        !aligned16(sw))
        return SQ_ERR_INVALID_ARG;
    if (K > kGptqMaxK || N > kMaxDim)
        return SQ_ERR_UNSUPPORTED;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (dt == SQ_BF16)
        return launch_gptq_rows(static_cast<const __nv_bfloat16 *>(w), N, K, s, U, wq, sw, st);
    return launch_gptq_rows(static_cast<const float *>(w), N, K, s, U, wq, sw, st);
}

sq_status sq_w8a8_gemm(const int8_t *xq, const float *sx, const int8_t *wq, const float *sw,
                       int64_t M, int64_t N, int64_t K, void *y, sq_dtype out_dt,
                       sq_stream_t stream)
{
    if (xq == nullptr || sx == nullptr || wq == nullptr || sw == nullptr || y == nullptr ||
        !valid_dtype(out_dt) || !aligned16(xq) || !aligned16(sx) || !aligned16(wq) ||
        !aligned16(sw) || !aligned16(y))
        return SQ_ERR_INVALID_ARG;
    sq_status r = check_gemm_dims(M, N, K);
    if (r != SQ_OK)
        return r;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (out_dt == SQ_BF16)
        return launch_gemm<OUT_BF16>(xq, sx, wq, sw, M, N, K, y, st);
    return launch_gemm<OUT_F32>(xq, sx, wq, sw, M, N, K, y, st);
}

sq_status sq_w8a8_gemm_s32(const int8_t *xq, const int8_t *wq, int64_t M, int64_t N, int64_t K,
                           int32_t *acc, sq_stream_t stream)
{
    if (xq == nullptr || wq == nullptr || acc == nullptr || !aligned16(xq) || !aligned16(wq) ||
        !aligned16(acc))
        return SQ_ERR_INVALID_ARG;
    sq_status r = check_gemm_dims(M, N, K);
    if (r != SQ_OK)
        return r;
    return launch_gemm<OUT_S32>(xq, nullptr, wq, nullptr, M, N, K, acc,
                                reinterpret_cast<cudaStream_t>(stream));
}

size_t sq_linear_workspace_size(int64_t M, int64_t N, int64_t K)
{
    if (M < 1 || N < 1 || K < 1 || fused_decode_applies(M, K))
        return 0;
    return linear_ws_layout(M, N, K).g.total;
}

sq_status sq_linear(const void *x, sq_dtype in_dt, const float *s, const int8_t *wq,
                    const float *sw, int64_t M, int64_t N, int64_t K, void *y, sq_dtype out_dt,
                    void *workspace, size_t ws_bytes, sq_stream_t stream)
{
    if (x == nullptr || s == nullptr || wq == nullptr || sw == nullptr || y == nullptr ||
        !valid_dtype(in_dt) || !valid_dtype(out_dt) || !aligned16(x) || !aligned16(s) ||
        !aligned16(wq) || !aligned16(sw) || !aligned16(y))
        return SQ_ERR_INVALID_ARG;
    sq_status r = check_gemm_dims(M, N, K);
    if (r != SQ_OK)
        return r;
    if (K > max_quant_k(in_dt))
        return SQ_ERR_UNSUPPORTED;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (fused_decode_applies(M, K)) {
        if (in_dt == SQ_BF16)
            return launch_fused_linear(static_cast<const __nv_bfloat16 *>(x), s, wq, sw, M, N, K, y,
                                       out_dt, st);
        return launch_fused_linear(static_cast<const float *>(x), s, wq, sw, M, N, K, y, out_dt, st);
    }
    const LinearWs L = linear_ws_layout(M, N, K);
    if (workspace == nullptr || ws_bytes < L.minimum || !aligned16(workspace))
        return SQ_ERR_INVALID_ARG;
    uint8_t *wsb = static_cast<uint8_t *>(workspace);
    int8_t *xq = reinterpret_cast<int8_t *>(wsb + L.xq);
    float *sx = reinterpret_cast<float *>(wsb + L.sx);
    // the GEMM's own workspace when the caller's holds it: the quantiser
    // clears its tile counters on the side
    const bool gws = ws_bytes >= L.g.total;
    int *cnt = gws ? reinterpret_cast<int *>(wsb + L.g.cnt) : nullptr;
    int32_t *slots = gws ? reinterpret_cast<int32_t *>(wsb + L.g.slots) : nullptr;
    const int ncnt = gws ? L.g.ncnt : 0;
    r = (in_dt == SQ_BF16)
            ? launch_quant_rows<__nv_bfloat16, sq::MODE_X>(static_cast<const __nv_bfloat16 *>(x), M, K, s, xq, sx,
                                                             st, cnt, ncnt)
            : launch_quant_rows<float, sq::MODE_X>(static_cast<const float *>(x), M, K, s, xq, sx, st, cnt, ncnt);
    if (r != SQ_OK)
        return r;
    return out_dt == SQ_BF16 ? launch_gemm<OUT_BF16>(xq, sx, wq, sw, M, N, K, y, st, cnt, slots, in_dt, true)
                             : launch_gemm<OUT_F32>(xq, sx, wq, sw, M, N, K, y, st, cnt, slots, in_dt, true);
}

size_t sq_w8a8_gemm_workspace_size(int64_t M, int64_t N, int64_t K)
{
    if (M < 1 || N < 1 || K < 1)
        return 0;
    return gemm_ws_layout(M, N, K, 0).total;
}

sq_status sq_w8a8_gemm_ws(const int8_t *xq, const float *sx, const int8_t *wq, const float *sw, int64_t M,
                          int64_t N, int64_t K, void *y, sq_dtype out_dt, void *workspace, size_t ws_bytes,
                          sq_stream_t stream)
{
    if (xq == nullptr || sx == nullptr || wq == nullptr || sw == nullptr || y == nullptr || workspace == nullptr ||
        !valid_dtype(out_dt) || !aligned16(xq) || !aligned16(sx) || !aligned16(wq) || !aligned16(sw) ||
        !aligned16(y) || !aligned16(workspace))
        return SQ_ERR_INVALID_ARG;
    sq_status r = check_gemm_dims(M, N, K);
    if (r != SQ_OK)
        return r;
    const GemmWs G = gemm_ws_layout(M, N, K, 0);
    if (ws_bytes < G.total)
        return SQ_ERR_INVALID_ARG;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    uint8_t *wsb = static_cast<uint8_t *>(workspace);
    int *cnt = reinterpret_cast<int *>(wsb + G.cnt);
    int32_t *slots = reinterpret_cast<int32_t *>(wsb + G.slots);
    // the slab and split-K kernels need no counters (and, after a grid of
    // unknown origin, request nothing before griddepcontrol.wait)
    if (slab_applies(M, N) || (M <= kDecodeMaxM && !decode_stream_on()))
        return out_dt == SQ_BF16 ? launch_gemm<OUT_BF16>(xq, sx, wq, sw, M, N, K, y, st)
                                 : launch_gemm<OUT_F32>(xq, sx, wq, sw, M, N, K, y, st);
    // clear the tile counters (a kernel of this library, so the GEMM after it
    // may start on its weight before griddepcontrol.wait)
    r = launch_kernel(sq::zero_f32_kernel, dim3(static_cast<unsigned>((G.ncnt + 255) / 256)), dim3(256), 0, st, 0, 0,
                      reinterpret_cast<float *>(cnt), static_cast<int64_t>(G.ncnt));
    if (r != SQ_OK)
        return r;
    return out_dt == SQ_BF16 ? launch_gemm<OUT_BF16>(xq, sx, wq, sw, M, N, K, y, st, cnt, slots)
                             : launch_gemm<OUT_F32>(xq, sx, wq, sw, M, N, K, y, st, cnt, slots);
}

sq_status sq_linear_noalloc(const void *x, sq_dtype in_dt, const float *s, const int8_t *wq,
                            const float *sw, int64_t M, int64_t N, int64_t K, void *y,
                            sq_dtype out_dt, sq_stream_t stream)
{
    if (x == nullptr || s == nullptr || wq == nullptr || sw == nullptr || y == nullptr ||
        !valid_dtype(in_dt) || !valid_dtype(out_dt) || !aligned16(x) || !aligned16(s) ||
        !aligned16(wq) || !aligned16(sw) || !aligned16(y))
        return SQ_ERR_INVALID_ARG;
    sq_status r = check_gemm_dims(M, N, K);
    if (r != SQ_OK)
        return r;
    // the codes and scales must fit the scratch; the GEMM's own workspace is
    // used when it fits too (else the GEMM runs without one)
    const size_t full = sq_linear_workspace_size(M, N, K);
    const size_t need = full == 0 ? 0 : linear_ws_layout(M, N, K).minimum;
    if (need > SQ_LINEAR_NOALLOC_SCRATCH_BYTES)
        return SQ_ERR_UNSUPPORTED;
    void *ws = nullptr;
    if (need > 0) {
        ws = noalloc_scratch();
        if (ws == nullptr)
            return SQ_ERR_CUDA;
    }
    return sq_linear(x, in_dt, s, wq, sw, M, N, K, y, out_dt, ws, need == 0 ? 0 : SQ_LINEAR_NOALLOC_SCRATCH_BYTES,
                     stream);
}

sq_status sq_selftest_wait_timeout(uint32_t limit_us, sq_stream_t stream)
{
    if (limit_us < 1 || limit_us > 2000000)
        return SQ_ERR_INVALID_ARG;
    return launch_kernel(sq::wait_selftest_kernel, dim3(1), dim3(32), 0, reinterpret_cast<cudaStream_t>(stream), 0, 0,
                         static_cast<unsigned long long>(limit_us) * 1000ull);
}

sq_status sq_device_status(sq_stream_t stream, uint32_t *code)
{
    if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) {
        cudaGetLastError();
        return SQ_ERR_CUDA;
    }
    unsigned int v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, sq::g_sq_device_error, sizeof v) != cudaSuccess ||
        cudaMemcpyToSymbol(sq::g_sq_device_error, &zero, sizeof zero) != cudaSuccess) {
        cudaGetLastError();
        return SQ_ERR_CUDA;
    }
    if (code != nullptr)
        *code = v;
    if (v == 0)
        return SQ_OK;
    return v == sq::kErrGptqPivot ? SQ_ERR_INVALID_ARG : SQ_ERR_TIMEOUT;
}

}  // extern "C"
