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
#include <mutex>

#include "sq.h"
#include "sq_gemm.cuh"
#include "sq_mem.cuh"
#include "sq_ptx.cuh"

namespace {

using sq::OUT_BF16;
using sq::OUT_F32;
using sq::OUT_S32;

constexpr int kMaxDevices = 64;

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
    const int64_t chunks = K / V;
    const int threads = static_cast<int>(std::min<int64_t>(256, ((chunks + 31) / 32) * 32));
    const int64_t col_blocks = (chunks + threads - 1) / threads;
    // about 8 CTAs of 256 threads per SM in total
    const int64_t want = std::max<int64_t>(1, (int64_t)di.sms * 8 * 256 / threads / col_blocks);
    int64_t rows_per_block = std::max<int64_t>(4, (R + want - 1) / want);
    int64_t row_blocks = (R + rows_per_block - 1) / rows_per_block;
    if (row_blocks > 65535) {
        row_blocks = 65535;
        rows_per_block = (R + row_blocks - 1) / row_blocks;
        row_blocks = (R + rows_per_block - 1) / rows_per_block;
    }
    dim3 grid(static_cast<unsigned>(col_blocks), static_cast<unsigned>(row_blocks));
    sq::col_absmax_kernel<T><<<grid, threads, 0, st>>>(
        x, R, K, ld, rows_per_block, reinterpret_cast<unsigned int *>(out));
    return launch_status();
}

// ---- row quantisers ----------------------------------------------------------
template <typename T, int MODE>
sq_status launch_quant_rows(const T *in, int64_t rows, int64_t K, const float *s, int8_t *q,
                            float *scale, cudaStream_t st)
{
    constexpr int V = sq::Vec<T>::N;
    const int64_t chunks = K / V;
    int cpt = 1;
    while (cpt < 8 && (chunks + cpt - 1) / cpt > 1024)
        cpt *= 2;
    if ((chunks + cpt - 1) / cpt > 1024)
        return SQ_ERR_UNSUPPORTED;
    // prefer >= 128 threads per row block when the row is long enough
    while (cpt > 1 && (chunks + cpt - 1) / cpt < 128)
        cpt /= 2;
    const int threads = static_cast<int>(std::max<int64_t>(32, (((chunks + cpt - 1) / cpt + 31) / 32) * 32));
    if (rows > 2147483647LL)
        return SQ_ERR_UNSUPPORTED;
    dim3 grid(static_cast<unsigned>(rows));
    switch (cpt) {
    case 1:
        sq::quant_rows_kernel<T, 1, MODE><<<grid, threads, 0, st>>>(in, K, s, q, scale);
        break;
    case 2:
        sq::quant_rows_kernel<T, 2, MODE><<<grid, threads, 0, st>>>(in, K, s, q, scale);
        break;
    case 4:
        sq::quant_rows_kernel<T, 4, MODE><<<grid, threads, 0, st>>>(in, K, s, q, scale);
        break;
    default:
        sq::quant_rows_kernel<T, 8, MODE><<<grid, threads, 0, st>>>(in, K, s, q, scale);
        break;
    }
    return launch_status();
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
    kernel<<<grid, sq::kGemmThreads, Cfg::SMEM_BYTES, st>>>(ta, tb, sx, sw, y, static_cast<int>(M),
                                                           static_cast<int>(N), static_cast<int>(K));
    return launch_status();
}

template <int OUT>
sq_status launch_gemm(const int8_t *xq, const float *sx, const int8_t *wq, const float *sw,
                      int64_t M, int64_t N, int64_t K, void *y, cudaStream_t st)
{
    if (M <= 32)
        return launch_gemm_cfg<32, 8, OUT, true>(xq, sx, wq, sw, M, N, K, y, st);
    if (M <= 64)
        return launch_gemm_cfg<64, 8, OUT, true>(xq, sx, wq, sw, M, N, K, y, st);
    if (M <= 128)
        return launch_gemm_cfg<128, 6, OUT, true>(xq, sx, wq, sw, M, N, K, y, st);
    return launch_gemm_cfg<256, 4, OUT, false>(xq, sx, wq, sw, M, N, K, y, st);
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

size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

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

}  // namespace

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
    if (cudaMemsetAsync(s, 0, static_cast<size_t>(K) * sizeof(float), st) != cudaSuccess)
        return SQ_ERR_CUDA;
    sq_status r = (dt == SQ_BF16)
                      ? launch_col_absmax(static_cast<const __nv_bfloat16 *>(w), N, K, K, s, st)
                      : launch_col_absmax(static_cast<const float *>(w), N, K, K, s, st);
    if (r != SQ_OK)
        return r;
    const int threads = 256;
    const unsigned blocks = static_cast<unsigned>((K + threads - 1) / threads);
    sq::smooth_factors_kernel<<<blocks, threads, 0, st>>>(ax, s, aw, K, alpha);
    return launch_status();
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
    (void)N;
    if (M < 1 || K < 1)
        return 0;
    return align_up(static_cast<size_t>(M) * static_cast<size_t>(K), 256) +
           align_up(static_cast<size_t>(M) * sizeof(float), 256);
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
    const size_t need = sq_linear_workspace_size(M, N, K);
    if (need > 0 && (workspace == nullptr || ws_bytes < need || !aligned16(workspace)))
        return SQ_ERR_INVALID_ARG;
    int8_t *xq = static_cast<int8_t *>(workspace);
    float *sx = reinterpret_cast<float *>(static_cast<uint8_t *>(workspace) +
                                          align_up(static_cast<size_t>(M) * K, 256));
    r = sq_quant_act(x, in_dt, M, K, s, xq, sx, stream);
    if (r != SQ_OK)
        return r;
    return sq_w8a8_gemm(xq, sx, wq, sw, M, N, K, y, out_dt, stream);
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
    const size_t need = sq_linear_workspace_size(M, N, K);
    if (need > SQ_LINEAR_NOALLOC_SCRATCH_BYTES)
        return SQ_ERR_UNSUPPORTED;
    void *ws = nullptr;
    if (need > 0) {
        ws = noalloc_scratch();
        if (ws == nullptr)
            return SQ_ERR_CUDA;
    }
    return sq_linear(x, in_dt, s, wq, sw, M, N, K, y, out_dt, ws, need, stream);
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
    return v == 0 ? SQ_OK : SQ_ERR_TIMEOUT;
}

}  // extern "C"
