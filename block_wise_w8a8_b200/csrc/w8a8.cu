// w8a8.cu -- the C ABI of libw8a8 (declared in include/w8a8.h): argument checks, the
// guard of the TurboT2VA paper's inference-stack section (guard paragraph: INT8 only for
// CUDA BF16 inputs with flattened M, K, N divisible by 128, else a BF16 linear on the
// retained BF16 weight), TMA descriptor set-up and kernel launches.  Everything is
// enqueued on the caller's stream; nothing is allocated.
#include <cudaTypedefs.h>

#include <algorithm>
#include <mutex>

#include "../../include/w8a8.h"
#include "common.cuh"
#include "gemm.cuh"
#include "norm.cuh"
#include "quant.cuh"

namespace {

using namespace w8a8;

constexpr int kMaxDevices = 64;
// TMA coordinates are signed 32-bit: matrix extents stay below 2^31.
constexpr int64_t kMaxTmaCoord = (int64_t{1} << 31) - 128;
// Per-row operator: K * 127^2 must stay inside INT32 (the accumulator holds all of K).
constexpr int64_t kRowMaxK = 133120;

struct DeviceInfo {
    bool ready = false;
    int sms = 0;
    bool gemm_attr_set[5] = {false, false, false, false, false};
    bool quant_attr_set[3] = {false, false, false};    // by quant::NormKind
    bool rstd_attr_set = false;
    bool norm_attr_set[4] = {false, false, false, false};
    int norm_max_clusters[norm::kMaxCluster + 1] = {};    // by cluster size, 0 = unknown
};
DeviceInfo g_dev[kMaxDevices];
std::mutex g_mu;
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

w8a8_status_t current_device(int &dev)
{
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        cudaGetLastError();
        return W8A8_ERR_CUDA;
    }
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_dev[dev].ready) {
        int sms = 0;
        if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
            cudaGetLastError();
            return W8A8_ERR_CUDA;
        }
        g_dev[dev].sms = sms;
        g_dev[dev].ready = true;
    }
    return W8A8_OK;
}

w8a8_status_t get_encoder()
{
    std::lock_guard<std::mutex> lk(g_mu);
    if (g_encode != nullptr)
        return W8A8_OK;
    void *fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000, cudaEnableDefault,
                                         &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess || fn == nullptr) {
        cudaGetLastError();
        return W8A8_ERR_CUDA;
    }
    g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    return W8A8_OK;
}

// A buffer that kernels on the current device may read/write: device or managed memory
// of this device.
w8a8_status_t check_device_ptr(const void *p)
{
    if (p == nullptr)
        return W8A8_ERR_INVALID_ARG;
    cudaPointerAttributes a;
    if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
        cudaGetLastError();
        return W8A8_ERR_NOT_DEVICE;
    }
    if (a.type != cudaMemoryTypeDevice && a.type != cudaMemoryTypeManaged)
        return W8A8_ERR_NOT_DEVICE;
    int dev = -1;
    cudaGetDevice(&dev);
    if (a.type == cudaMemoryTypeDevice && a.device != dev)
        return W8A8_ERR_NOT_DEVICE;
    return W8A8_OK;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

thread_local cudaError_t t_last_cuda_error = cudaSuccess;

w8a8_status_t cuda_fail(cudaError_t e)
{
    t_last_cuda_error = e;
    cudaGetLastError();
    return W8A8_ERR_CUDA;
}

w8a8_status_t launch_status()
{
    const cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? W8A8_OK : cuda_fail(e);
}

#define W8A8_TRY(expr)                                                                   \
    do {                                                                                 \
        const w8a8_status_t st_ = (expr);                                                \
        if (st_ != W8A8_OK)                                                              \
            return st_;                                                                  \
    } while (0)

// Row-major [rows, cols] matrix of `es`-byte elements; box of box_rows x box_cols
// elements.
w8a8_status_t make_map(CUtensorMap &m, const void *base, CUtensorMapDataType dt, int es,
                       int64_t rows, int64_t cols, uint32_t box_rows, uint32_t box_cols,
                       CUtensorMapSwizzle swizzle)
{
    W8A8_TRY(get_encoder());
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols) * es};
    const cuuint32_t box[2] = {box_cols, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    const CUresult r = g_encode(&m, dt, 2, const_cast<void *>(base), dims, strides, box, estr,
                                CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
                                CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? W8A8_OK : W8A8_ERR_CUDA;
}

// GEMM operand: box of box_rows x 128 bytes, 128-byte swizzle (the UMMA K-major layout).
w8a8_status_t make_operand_map(CUtensorMap &m, const void *base, CUtensorMapDataType dt,
                               int es, int64_t rows, int64_t cols, uint32_t box_rows)
{
    return make_map(m, base, dt, es, rows, cols, box_rows, static_cast<uint32_t>(128 / es),
                    CU_TENSOR_MAP_SWIZZLE_128B);
}

// pdl: launch as a programmatic dependent of the kernel before it on the stream (the
// activation quantizer), so the GEMM's set-up overlaps that kernel's tail.
template <gemm::Mode kMode>
w8a8_status_t launch_gemm(const void *a, const void *b, const gemm::Params &p0,
                          cudaStream_t stream, bool pdl = false)
{
    int dev;
    W8A8_TRY(current_device(dev));
    constexpr bool kInt8 = kMode != gemm::Mode::kBf16;
    CUtensorMap ta, tb;
    const CUtensorMapDataType dt = kInt8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    const int es = kInt8 ? 1 : 2;
    W8A8_TRY(make_operand_map(ta, a, dt, es, p0.M, p0.K, gemm::BM));
    W8A8_TRY(make_operand_map(tb, b, dt, es, p0.N, p0.K, gemm::BN));
    // the block-scaled GEMM stores its output by TMA: 32 x 32 BF16 boxes (64-byte rows)
    // from the epilogue warps' staging buffers, whose layout is the 64-byte swizzle
    CUtensorMap ty = ta;
    if (kMode == gemm::Mode::kI8Scaled)
        W8A8_TRY(make_map(ty, p0.y, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, p0.M, p0.N, 32, 32,
                          CU_TENSOR_MAP_SWIZZLE_64B));
    gemm::Params p = p0;
    p.num_tm = static_cast<int32_t>((p.M + gemm::BM - 1) / gemm::BM);
    p.num_tn = static_cast<int32_t>((p.N + gemm::BN - 1) / gemm::BN);
    p.num_tiles = p.num_tm * p.num_tn;
    const int64_t slice = kInt8 ? 128 : 64;
    p.kslices = static_cast<int32_t>((p.K + slice - 1) / slice);
    auto kern = gemm::gemm_kernel<kMode>;
    {
        std::lock_guard<std::mutex> lk(g_mu);
        if (!g_dev[dev].gemm_attr_set[static_cast<int>(kMode)]) {
            const cudaError_t e = cudaFuncSetAttribute(
                kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(gemm::kSmemBytes));
            if (e != cudaSuccess)
                return cuda_fail(e);
            // The kernel re-splits its registers between warpgroups (setmaxnreg); that
            // split must fit in what the launch provides or the increase would never be
            // granted.  Refuse to launch a build whose register count is too low.
            cudaFuncAttributes fa;
            const cudaError_t e2 = cudaFuncGetAttributes(&fa, kern);
            if (e2 != cudaSuccess)
                return cuda_fail(e2);
            if (fa.numRegs * gemm::NUM_THREADS <
                128 * gemm::kRegsControl + 256 * gemm::kRegsEpilogue)
                return cuda_fail(cudaErrorInvalidConfiguration);
            g_dev[dev].gemm_attr_set[static_cast<int>(kMode)] = true;
        }
    }
    // Work units: whole tiles, except that in the scaled modes a last, partial round of
    // tiles is split into 128-column halves when they all fit in one round (a half takes
    // about half a tile's time: the epilogue, the bottleneck, does half the work).
    const int sms = g_dev[dev].sms;
    p.num_full = p.num_tiles;
    p.num_units = p.num_tiles;
    if (kMode == gemm::Mode::kI8Scaled || kMode == gemm::Mode::kI8Gated) {
        const int tail = p.num_tiles % sms;
        if (tail > 0 && 2 * tail <= sms) {
            p.num_full = p.num_tiles - tail;
            p.num_units = p.num_full + 2 * tail;
        }
    }
    const int grid = std::min(p.num_units, sms);
    if (pdl) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(static_cast<unsigned>(grid));
        cfg.blockDim = dim3(gemm::NUM_THREADS);
        cfg.dynamicSmemBytes = gemm::kSmemBytes;
        cfg.stream = stream;
        cudaLaunchAttribute attr;
        attr.id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr.val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = &attr;
        cfg.numAttrs = 1;
        const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, ta, tb, ty, p);
        return e == cudaSuccess ? launch_status() : cuda_fail(e);
    }
    kern<<<grid, gemm::NUM_THREADS, gemm::kSmemBytes, stream>>>(ta, tb, ty, p);
    return launch_status();
}

// Block quantization of x [rows, cols] (both multiples of 128, buffers already checked):
// one persistent CTA per SM, blocks streamed in by TMA.
template <int kNorm>
w8a8_status_t launch_quantize_t(const uint16_t *x, int64_t rows, int64_t cols, int8_t *q, float *s,
                                const quant::NormArgs &na, bool pdl, cudaStream_t stream)
{
    int dev;
    W8A8_TRY(current_device(dev));
    CUtensorMap tm;
    W8A8_TRY(make_map(tm, x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, rows, cols, 128, 128,
                      CU_TENSOR_MAP_SWIZZLE_NONE));
    auto kern = quant::quantize_blocks_kernel<kNorm>;
    {
        std::lock_guard<std::mutex> lk(g_mu);
        if (!g_dev[dev].quant_attr_set[kNorm]) {
            const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                       static_cast<int>(quant::kQSmemBytes));
            if (e != cudaSuccess)
                return cuda_fail(e);
            g_dev[dev].quant_attr_set[kNorm] = true;
        }
    }
    const int64_t KB = cols / 128;
    const int64_t nblocks = (rows / 128) * KB;
    const int64_t grid = std::min<int64_t>(nblocks, g_dev[dev].sms);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(grid));
    cfg.blockDim = dim3(quant::kQThreads);
    cfg.dynamicSmemBytes = quant::kQSmemBytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr.val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = &attr;
    cfg.numAttrs = pdl ? 1 : 0;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, tm, cols, nblocks, KB, q, s, na);
    return e == cudaSuccess ? launch_status() : cuda_fail(e);
}

w8a8_status_t launch_quantize(const uint16_t *x, int64_t rows, int64_t cols, int8_t *q, float *s,
                              cudaStream_t stream)
{
    return launch_quantize_t<quant::kNone>(x, rows, cols, q, s, quant::NormArgs{}, false, stream);
}

w8a8_status_t quantize_impl(const uint16_t *x, int64_t rows, int64_t cols, int8_t *q, float *s,
                            cudaStream_t stream)
{
    if (rows < 0 || cols < 0)
        return W8A8_ERR_INVALID_ARG;
    if (rows % 128 || cols % 128 || rows > kMaxTmaCoord || cols > kMaxTmaCoord)
        return W8A8_ERR_SHAPE;
    if (rows == 0 || cols == 0)
        return W8A8_OK;
    W8A8_TRY(check_device_ptr(x));
    W8A8_TRY(check_device_ptr(q));
    W8A8_TRY(check_device_ptr(s));
    if (!aligned16(x) || !aligned16(q) || (reinterpret_cast<uintptr_t>(s) & 3u))
        return W8A8_ERR_ALIGNMENT;
    return launch_quantize(x, rows, cols, q, s, stream);
}

size_t round256(size_t v) { return (v + 255) & ~static_cast<size_t>(255); }

bool int8_shape_ok(int64_t M, int64_t K, int64_t N)
{
    return M > 0 && K > 0 && N > 0 && M % 128 == 0 && K % 128 == 0 && N % 128 == 0 &&
           K <= 128 * gemm::KB_MAX;
}

w8a8_status_t check_weight(const w8a8_weight_t *w, int64_t K)
{
    if (w == nullptr || w->w_bf16 == nullptr || w->N < 0 || w->K != K)
        return W8A8_ERR_INVALID_ARG;
    if ((w->wq == nullptr) != (w->ws == nullptr))
        return W8A8_ERR_INVALID_ARG;
    return W8A8_OK;
}

w8a8_status_t gemm_i8_impl(const int8_t *xq, const float *xs, int64_t M, int64_t K,
                           const w8a8_weight_t *w, const uint16_t *bias, uint16_t *y,
                           cudaStream_t stream, const uint16_t *resid = nullptr,
                           const uint16_t *gate = nullptr, int64_t gate_T = 1, bool pdl = false)
{
    gemm::Params p{};
    p.M = M;
    p.N = w->N;
    p.K = K;
    p.xs = xs;
    p.ws = w->ws;
    p.bias = bias;
    p.y = y;
    p.resid = resid;
    p.gate = gate;
    p.gate_T = gate_T;
    if (gate != nullptr)
        return launch_gemm<gemm::Mode::kI8Gated>(xq, w->wq, p, stream, pdl);
    return launch_gemm<gemm::Mode::kI8Scaled>(xq, w->wq, p, stream, pdl);
}

w8a8_status_t bf16_impl(const uint16_t *x, const uint16_t *w, const uint16_t *bias, uint16_t *y,
                        int64_t M, int64_t K, int64_t N, cudaStream_t stream)
{
    if (M == 0 || N == 0)
        return W8A8_OK;
    const bool tc = K > 0 && K % 8 == 0 && aligned16(x) && aligned16(w) && aligned16(y);
    if (tc) {
        gemm::Params p{};
        p.M = M;
        p.N = N;
        p.K = K;
        p.bias = bias;
        p.y = y;
        return launch_gemm<gemm::Mode::kBf16>(x, w, p, stream);
    }
    const dim3 grid(static_cast<unsigned>((N + 63) / 64), static_cast<unsigned>((M + 63) / 64));
    if (grid.y > 65535u)
        return W8A8_ERR_SHAPE;
    gemm::bf16_gemm_simt_kernel<<<grid, 256, 0, stream>>>(x, w, bias, y, M, K, N);
    return launch_status();
}

__global__ void wait_timeout_kernel(uint64_t timeout_ns)
{
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        abort_flag = 0;
        fence_barrier_init();
    }
    __syncthreads();
    if (threadIdx.x == 0)
        mbar_wait(&bar, 0, &abort_flag, timeout_ns);   // nothing ever arrives
}

// ------------------------------------------------------------------ no-allocation variant
// Scratch for w8a8_linear_noalloc: the INT8 codes of the activations (first
// W8A8_NOALLOC_MAX_ELEMS bytes) followed by their FP32 block scales.  It is a module
// global, so every GPU that loads this library holds it until the process exits, and all
// calls of w8a8_linear_noalloc on a device share it.
constexpr size_t kNoAllocCodeBytes = static_cast<size_t>(W8A8_NOALLOC_MAX_ELEMS);
constexpr size_t kNoAllocScaleBytes = (static_cast<size_t>(W8A8_NOALLOC_MAX_ELEMS) / (128 * 128)) * sizeof(float);
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocCodeBytes + kNoAllocScaleBytes];

// Host code cannot use g_noalloc_scratch's name as a device address; its address on each
// device is looked up once, with that device current, and cached here.
void *g_noalloc_ptr[kMaxDevices] = {};

w8a8_status_t noalloc_scratch(int dev, void *&ptr)
{
    std::lock_guard<std::mutex> lk(g_mu);
    if (g_noalloc_ptr[dev] == nullptr) {
        void *p = nullptr;
        const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess || p == nullptr) {
            t_last_cuda_error = e;
            cudaGetLastError();
            return W8A8_ERR_CUDA;
        }
        g_noalloc_ptr[dev] = p;
    }
    ptr = g_noalloc_ptr[dev];
    return W8A8_OK;
}

// rstd of every row of x [M, K] (M a multiple of norm::kSRows, K of 128): one CTA per
// norm::kSRows rows.
w8a8_status_t launch_row_rstd(const uint16_t *x, int64_t M, int64_t K, float eps, float *rstd,
                              cudaStream_t stream)
{
    int dev;
    W8A8_TRY(current_device(dev));
    CUtensorMap tm;
    W8A8_TRY(make_map(tm, x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, M, K, norm::kSRows, 64,
                      CU_TENSOR_MAP_SWIZZLE_128B));
    auto kern = norm::row_rstd_kernel;
    {
        std::lock_guard<std::mutex> lk(g_mu);
        if (!g_dev[dev].rstd_attr_set) {
            const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                       static_cast<int>(norm::kSSmemBytes));
            if (e != cudaSuccess)
                return cuda_fail(e);
            g_dev[dev].rstd_attr_set = true;
        }
    }
    kern<<<static_cast<unsigned>(M / norm::kSRows), norm::kSThreads, norm::kSSmemBytes, stream>>>(
        tm, K, eps, rstd);
    return launch_status();
}

// Fused RMSNorm (+ modulation) + block quantization in one grid: clusters of
// C = min(4, K / 128) CTAs (4 = norm::kMaxCluster), one cluster per 128-row strip at a
// time, as many clusters as fit on the device.
template <bool kMod, bool kExactSq>
w8a8_status_t launch_norm_fused(const uint16_t *x, const norm::Params &p, cudaStream_t stream)
{
    int dev;
    W8A8_TRY(current_device(dev));
    CUtensorMap tm;
    W8A8_TRY(make_map(tm, x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, p.MB * 128, p.K, 128, 64,
                      CU_TENSOR_MAP_SWIZZLE_128B));
    auto kern = norm::rmsnorm_quantize_kernel<kMod, kExactSq>;
    const int C = static_cast<int>(std::min<int64_t>(norm::kMaxCluster, p.K / 128));
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeClusterDimension;
    attr.val.clusterDim.x = static_cast<unsigned>(C);
    attr.val.clusterDim.y = 1;
    attr.val.clusterDim.z = 1;
    cfg.blockDim = dim3(norm::kThreads, 1, 1);
    cfg.dynamicSmemBytes = norm::kSmemBytes;
    cfg.stream = stream;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    int max_clusters;
    {
        std::lock_guard<std::mutex> lk(g_mu);
        const int v = static_cast<int>(kMod) * 2 + static_cast<int>(kExactSq);
        if (!g_dev[dev].norm_attr_set[v]) {
            const cudaError_t e = cudaFuncSetAttribute(
                kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(norm::kSmemBytes));
            if (e != cudaSuccess)
                return cuda_fail(e);
            g_dev[dev].norm_attr_set[v] = true;
        }
        if (g_dev[dev].norm_max_clusters[C] == 0) {
            int n = 0;
            cfg.gridDim = dim3(static_cast<unsigned>(C * g_dev[dev].sms), 1, 1);
            if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess || n <= 0) {
                cudaGetLastError();
                n = g_dev[dev].sms / C;
            }
            g_dev[dev].norm_max_clusters[C] = std::max(1, n);
        }
        max_clusters = g_dev[dev].norm_max_clusters[C];
    }
    const int64_t nclusters = std::max<int64_t>(1, std::min<int64_t>(p.MB, max_clusters));
    cfg.gridDim = dim3(static_cast<unsigned>(nclusters * C), 1, 1);
    const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, tm, p);
    if (e != cudaSuccess)
        return cuda_fail(e);
    return launch_status();
}

// RMSNorm (+ modulation) + block quantization as two grids: the rows' rstd
// (norm::row_rstd_kernel), then the block quantizer normalising each block as it arrives
// (quant::quantize_blocks_kernel<kRms / kRmsMod>), launched as a programmatic dependent
// so that its set-up and first loads overlap the end of the first grid.  Without a
// caller's rstd buffer the M floats come from the stream-ordered allocator.
template <bool kMod>
w8a8_status_t launch_norm_split(const uint16_t *x, const norm::Params &p, cudaStream_t stream)
{
    const int64_t M = p.MB * 128;
    float *rstd = p.rstd_out;
    if (rstd == nullptr) {
        void *tmp = nullptr;
        const cudaError_t e = cudaMallocAsync(&tmp, static_cast<size_t>(M) * sizeof(float), stream);
        if (e != cudaSuccess)
            return cuda_fail(e);
        rstd = static_cast<float *>(tmp);
    }
    w8a8_status_t st = launch_row_rstd(x, M, p.K, p.eps, rstd, stream);
    if (st == W8A8_OK) {
        quant::NormArgs na;
        na.rstd = rstd;
        na.gamma = p.gamma;
        na.scale = p.scale;
        na.shift = p.shift;
        na.T = p.T;
        st = launch_quantize_t<kMod ? quant::kRmsMod : quant::kRms>(x, M, p.K, p.q, p.s, na, true, stream);
    }
    if (p.rstd_out == nullptr) {
        const cudaError_t e = cudaFreeAsync(rstd, stream);
        if (e != cudaSuccess && st == W8A8_OK)
            st = cuda_fail(e);
    }
    return st;
}

// Rows per SM from which the two-grid form runs: its row-statistics grid is then bound by
// HBM rather than by each row's chain of K dependent FP64 operations, and x read twice
// costs less than the one-grid form's slot-bound pipeline (measured at K = 2048..16384).
constexpr int64_t kNormSplitRowsPerSm = 192;

template <bool kMod>
w8a8_status_t launch_norm(const uint16_t *x, const norm::Params &p, cudaStream_t stream)
{
    int dev;
    W8A8_TRY(current_device(dev));
    if (p.MB * 128 >= kNormSplitRowsPerSm * g_dev[dev].sms)
        return launch_norm_split<kMod>(x, p, stream);
    return p.eps == 0.0f ? launch_norm_fused<kMod, true>(x, p, stream)
                         : launch_norm_fused<kMod, false>(x, p, stream);
}

// Checks shared by both RMSNorm entry points; fills p (except the modulation fields).
w8a8_status_t norm_common(const w8a8_bf16_t *x, const w8a8_bf16_t *gamma, float eps, int64_t M,
                          int64_t K, int8_t *xq, float *xs, float *rstd_out, norm::Params &p)
{
    if (M < 0 || K < 0 || !(eps >= 0.0f) || !(eps <= 3.4e38f))
        return W8A8_ERR_INVALID_ARG;
    if (M % 128 || K % 128 || M > kMaxTmaCoord || K > kMaxTmaCoord)
        return W8A8_ERR_SHAPE;
    if (M > 0 && K == 0)
        return W8A8_ERR_SHAPE;
    if (M == 0)
        return W8A8_OK;
    W8A8_TRY(check_device_ptr(x));
    if (gamma != nullptr)
        W8A8_TRY(check_device_ptr(gamma));
    W8A8_TRY(check_device_ptr(xq));
    W8A8_TRY(check_device_ptr(xs));
    if (rstd_out != nullptr)
        W8A8_TRY(check_device_ptr(rstd_out));
    if (!aligned16(x) || !aligned16(gamma) || !aligned16(xq) ||
        (reinterpret_cast<uintptr_t>(xs) & 3u) || (reinterpret_cast<uintptr_t>(rstd_out) & 3u))
        return W8A8_ERR_ALIGNMENT;
    p = norm::Params{};
    p.gamma = gamma;
    p.eps = eps;
    p.MB = M / 128;
    p.K = K;
    p.q = xq;
    p.s = xs;
    p.rstd_out = rstd_out;
    return W8A8_OK;
}

// A host buffer: pinned or pageable host memory, not device or managed memory.
w8a8_status_t check_host_ptr(const void *p)
{
    if (p == nullptr)
        return W8A8_ERR_INVALID_ARG;
    cudaPointerAttributes a;
    if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
        cudaGetLastError();
        return W8A8_ERR_INVALID_ARG;
    }
    return (a.type == cudaMemoryTypeHost || a.type == cudaMemoryTypeUnregistered)
               ? W8A8_OK
               : W8A8_ERR_INVALID_ARG;
}

// Rows per chunk of w8a8_linear_host: the caller's, else 4 MiB of x per chunk rounded
// down to 128 rows (at least 128); never more than M.
int64_t host_chunk(int64_t M, int64_t K, int64_t chunk_rows)
{
    int64_t c = chunk_rows;
    if (c <= 0) {
        const int64_t per = K > 0 ? (int64_t{4} << 20) / (2 * K) : (int64_t{1} << 20);
        c = std::max<int64_t>(128, per / 128 * 128);
    }
    return std::min(c, std::max<int64_t>(M, 1));
}

// The two copy streams and seven events of w8a8_linear_host, one set per device,
// created by the first call on that device.
struct HostPipe {
    bool ready = false;
    cudaStream_t h2d = nullptr, d2h = nullptr;
    cudaEvent_t start = nullptr, h2d_done[2] = {}, comp_done[2] = {}, d2h_done[2] = {};
};
HostPipe g_pipe[kMaxDevices];
std::mutex g_host_mu;      // one w8a8_linear_host enqueue at a time

w8a8_status_t host_pipe(int dev, HostPipe *&hp)
{
    std::lock_guard<std::mutex> lk(g_mu);
    HostPipe &h = g_pipe[dev];
    if (!h.ready) {
        cudaError_t e = cudaStreamCreateWithFlags(&h.h2d, cudaStreamNonBlocking);
        if (e == cudaSuccess)
            e = cudaStreamCreateWithFlags(&h.d2h, cudaStreamNonBlocking);
        cudaEvent_t *evs[7] = {&h.start, &h.h2d_done[0], &h.h2d_done[1], &h.comp_done[0],
                               &h.comp_done[1], &h.d2h_done[0], &h.d2h_done[1]};
        for (int i = 0; i < 7 && e == cudaSuccess; ++i)
            e = cudaEventCreateWithFlags(evs[i], cudaEventDisableTiming);
        if (e != cudaSuccess)
            return cuda_fail(e);
        h.ready = true;
    }
    hp = &h;
    return W8A8_OK;
}

} // namespace

extern "C" {

w8a8_status_t w8a8_quantize_weight(const w8a8_bf16_t *w, int64_t N, int64_t K, int8_t *wq,
                                   float *ws, void *stream)
{
    if (N == 0 || K == 0)
        return (N % 128 || K % 128 || N < 0 || K < 0) ? W8A8_ERR_SHAPE : W8A8_OK;
    return quantize_impl(w, N, K, wq, ws, static_cast<cudaStream_t>(stream));
}

w8a8_status_t w8a8_quantize_act(const w8a8_bf16_t *x, int64_t M, int64_t K, int8_t *xq,
                                float *xs, void *stream)
{
    return quantize_impl(x, M, K, xq, xs, static_cast<cudaStream_t>(stream));
}

w8a8_status_t w8a8_rmsnorm_quantize_act(const w8a8_bf16_t *x, const w8a8_bf16_t *gamma,
                                        float eps, int64_t M, int64_t K, int8_t *xq, float *xs,
                                        float *rstd_out, void *stream)
{
    norm::Params p;
    W8A8_TRY(norm_common(x, gamma, eps, M, K, xq, xs, rstd_out, p));
    if (M == 0)
        return W8A8_OK;
    const cudaStream_t st = static_cast<cudaStream_t>(stream);
    return launch_norm<false>(x, p, st);
}

w8a8_status_t w8a8_rmsnorm_mod_quantize_act(const w8a8_bf16_t *x, const w8a8_bf16_t *gamma,
                                            const w8a8_bf16_t *scale, const w8a8_bf16_t *shift,
                                            int64_t T, float eps, int64_t M, int64_t K,
                                            int8_t *xq, float *xs, float *rstd_out, void *stream)
{
    if (T <= 0)
        return W8A8_ERR_INVALID_ARG;
    norm::Params p;
    W8A8_TRY(norm_common(x, gamma, eps, M, K, xq, xs, rstd_out, p));
    if (T % 128 || M % T)
        return W8A8_ERR_SHAPE;
    if (M == 0)
        return W8A8_OK;
    W8A8_TRY(check_device_ptr(scale));
    W8A8_TRY(check_device_ptr(shift));
    if (!aligned16(scale) || !aligned16(shift))
        return W8A8_ERR_ALIGNMENT;
    p.scale = scale;
    p.shift = shift;
    p.T = T;
    const cudaStream_t st = static_cast<cudaStream_t>(stream);
    return launch_norm<true>(x, p, st);
}

size_t w8a8_linear_workspace_bytes(int64_t M, int64_t K, int64_t N)
{
    if (!int8_shape_ok(M, K, N))
        return 0;
    return round256(static_cast<size_t>(M) * static_cast<size_t>(K)) +
           static_cast<size_t>(M / 128) * static_cast<size_t>(K / 128) * sizeof(float);
}

w8a8_status_t w8a8_linear(const w8a8_bf16_t *x, int64_t M, int64_t K, const w8a8_weight_t *w,
                          const w8a8_bf16_t *bias, w8a8_bf16_t *y, void *workspace,
                          size_t workspace_bytes, int *path_taken, void *stream)
{
    if (path_taken != nullptr)
        *path_taken = W8A8_PATH_NONE;
    if (M < 0 || K < 0)
        return W8A8_ERR_INVALID_ARG;
    W8A8_TRY(check_weight(w, K));
    const int64_t N = w->N;
    if (M == 0 || N == 0)
        return W8A8_OK;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (K > 0)
        W8A8_TRY(check_device_ptr(x));
    W8A8_TRY(check_device_ptr(y));
    if (K > 0)
        W8A8_TRY(check_device_ptr(w->w_bf16));
    if (bias != nullptr)
        W8A8_TRY(check_device_ptr(bias));
    const bool int8 = int8_shape_ok(M, K, N) && w->wq != nullptr && aligned16(x) &&
                      aligned16(y) && aligned16(w->wq) && aligned16(workspace) &&
                      (bias == nullptr || aligned16(bias));
    if (int8) {
        W8A8_TRY(check_device_ptr(w->wq));
        W8A8_TRY(check_device_ptr(w->ws));
        const size_t need = w8a8_linear_workspace_bytes(M, K, N);
        if (workspace == nullptr || workspace_bytes < need)
            return W8A8_ERR_WORKSPACE;
        W8A8_TRY(check_device_ptr(workspace));
        int8_t *xq = static_cast<int8_t *>(workspace);
        float *xs = reinterpret_cast<float *>(static_cast<uint8_t *>(workspace) +
                                              round256(static_cast<size_t>(M) * K));
        W8A8_TRY(quantize_impl(x, M, K, xq, xs, st));
        W8A8_TRY(gemm_i8_impl(xq, xs, M, K, w, bias, y, st, nullptr, nullptr, 1, true));
        if (path_taken != nullptr)
            *path_taken = W8A8_PATH_INT8;
        return W8A8_OK;
    }
    W8A8_TRY(bf16_impl(x, w->w_bf16, bias, y, M, K, N, st));
    if (path_taken != nullptr)
        *path_taken = W8A8_PATH_BF16;
    return W8A8_OK;
}

int64_t w8a8_linear_host_chunk_rows(int64_t M, int64_t K)
{
    return host_chunk(M, K, 0);
}

size_t w8a8_linear_host_workspace_bytes(int64_t M, int64_t K, int64_t N, int64_t chunk_rows)
{
    if (M <= 0 || K < 0 || N <= 0 || chunk_rows < 0)
        return 0;
    const int64_t C = host_chunk(M, K, chunk_rows);
    return 2 * round256(static_cast<size_t>(C) * K * 2) + 2 * round256(static_cast<size_t>(C) * N * 2) +
           w8a8_linear_workspace_bytes(C, K, N);
}

w8a8_status_t w8a8_linear_host(const w8a8_bf16_t *x_host, int64_t M, int64_t K,
                               const w8a8_weight_t *w, const w8a8_bf16_t *bias,
                               w8a8_bf16_t *y_host, void *workspace, size_t workspace_bytes,
                               int64_t chunk_rows, int *path_taken, void *stream)
{
    if (path_taken != nullptr)
        *path_taken = W8A8_PATH_NONE;
    if (M < 0 || K < 0 || chunk_rows < 0 || chunk_rows % 128 != 0)
        return W8A8_ERR_INVALID_ARG;
    W8A8_TRY(check_weight(w, K));
    const int64_t N = w->N;
    if (M == 0 || N == 0)
        return W8A8_OK;
    if (K > 0)
        W8A8_TRY(check_host_ptr(x_host));
    W8A8_TRY(check_host_ptr(y_host));
    if (K > 0)
        W8A8_TRY(check_device_ptr(w->w_bf16));
    if (bias != nullptr)
        W8A8_TRY(check_device_ptr(bias));
    const int64_t C = host_chunk(M, K, chunk_rows);
    if (workspace == nullptr || !aligned16(workspace) ||
        workspace_bytes < w8a8_linear_host_workspace_bytes(M, K, N, chunk_rows))
        return W8A8_ERR_WORKSPACE;
    W8A8_TRY(check_device_ptr(workspace));
    // the guard of w8a8_linear, decided once for the whole input (the staging buffers are
    // 256-byte aligned); every chunk then takes the same path
    const bool int8 = int8_shape_ok(M, K, N) && w->wq != nullptr && aligned16(w->wq) &&
                      (bias == nullptr || aligned16(bias));
    if (int8) {
        W8A8_TRY(check_device_ptr(w->wq));
        W8A8_TRY(check_device_ptr(w->ws));
    }
    int dev;
    W8A8_TRY(current_device(dev));
    HostPipe *hp = nullptr;
    W8A8_TRY(host_pipe(dev, hp));

    uint8_t *base = static_cast<uint8_t *>(workspace);
    const size_t xsz = round256(static_cast<size_t>(C) * K * 2);
    const size_t ysz = round256(static_cast<size_t>(C) * N * 2);
    uint16_t *xbuf[2] = {reinterpret_cast<uint16_t *>(base), reinterpret_cast<uint16_t *>(base + xsz)};
    uint16_t *ybuf[2] = {reinterpret_cast<uint16_t *>(base + 2 * xsz),
                         reinterpret_cast<uint16_t *>(base + 2 * xsz + ysz)};
    int8_t *xq = reinterpret_cast<int8_t *>(base + 2 * xsz + 2 * ysz);
    float *xs = reinterpret_cast<float *>(base + 2 * xsz + 2 * ysz + round256(static_cast<size_t>(C) * K));
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int64_t nch = (M + C - 1) / C;

    std::lock_guard<std::mutex> lk(g_host_mu);
    w8a8_status_t status = W8A8_OK;
    cudaError_t e = cudaEventRecord(hp->start, st);
    if (e == cudaSuccess)
        e = cudaStreamWaitEvent(hp->h2d, hp->start, 0);
    if (e == cudaSuccess)
        e = cudaStreamWaitEvent(hp->d2h, hp->start, 0);
    int64_t done = 0;
    for (int64_t i = 0; i < nch && e == cudaSuccess && status == W8A8_OK; ++i) {
        const int b = static_cast<int>(i & 1);
        const int64_t r0 = i * C, rows = std::min(C, M - r0);
        // x chunk in: its buffer was last read by the linear on chunk i - 2
        if (i >= 2)
            e = cudaStreamWaitEvent(hp->h2d, hp->comp_done[b], 0);
        if (e == cudaSuccess && K > 0)
            e = cudaMemcpyAsync(xbuf[b], x_host + r0 * K, static_cast<size_t>(rows) * K * 2,
                                cudaMemcpyHostToDevice, hp->h2d);
        if (e == cudaSuccess)
            e = cudaEventRecord(hp->h2d_done[b], hp->h2d);
        // the linear: after its x chunk landed and after chunk i - 2 left its y buffer
        if (e == cudaSuccess)
            e = cudaStreamWaitEvent(st, hp->h2d_done[b], 0);
        if (e == cudaSuccess && i >= 2)
            e = cudaStreamWaitEvent(st, hp->d2h_done[b], 0);
        if (e != cudaSuccess)
            break;
        if (int8) {
            status = quantize_impl(xbuf[b], rows, K, xq, xs, st);
            if (status == W8A8_OK)
                status = gemm_i8_impl(xq, xs, rows, K, w, bias, ybuf[b], st, nullptr, nullptr, 1, true);
        } else {
            status = bf16_impl(xbuf[b], w->w_bf16, bias, ybuf[b], rows, K, N, st);
        }
        if (status != W8A8_OK)
            break;
        e = cudaEventRecord(hp->comp_done[b], st);
        // y chunk out
        if (e == cudaSuccess)
            e = cudaStreamWaitEvent(hp->d2h, hp->comp_done[b], 0);
        if (e == cudaSuccess)
            e = cudaMemcpyAsync(y_host + r0 * N, ybuf[b], static_cast<size_t>(rows) * N * 2,
                                cudaMemcpyDeviceToHost, hp->d2h);
        if (e == cudaSuccess)
            e = cudaEventRecord(hp->d2h_done[b], hp->d2h);
        if (e == cudaSuccess)
            done = i + 1;
    }
    // the caller's stream waits for the last copies back (both buffers), and for any copy
    // in that an error left without its linear
    if (e == cudaSuccess)
        e = cudaEventRecord(hp->start, hp->h2d);
    if (e == cudaSuccess)
        e = cudaStreamWaitEvent(st, hp->start, 0);
    for (int64_t i = std::max<int64_t>(0, done - 2); i < done; ++i) {
        const cudaError_t e2 = cudaStreamWaitEvent(st, hp->d2h_done[i & 1], 0);
        if (e == cudaSuccess)
            e = e2;
    }
    if (e != cudaSuccess)
        return cuda_fail(e);
    if (status != W8A8_OK)
        return status;
    if (path_taken != nullptr)
        *path_taken = int8 ? W8A8_PATH_INT8 : W8A8_PATH_BF16;
    return W8A8_OK;
}

w8a8_status_t w8a8_linear_noalloc(const w8a8_bf16_t *x, int64_t M, int64_t K,
                                  const w8a8_weight_t *w, const w8a8_bf16_t *bias,
                                  w8a8_bf16_t *y, int *path_taken, void *stream)
{
    if (path_taken != nullptr)
        *path_taken = W8A8_PATH_NONE;
    if (M < 0 || K < 0)
        return W8A8_ERR_INVALID_ARG;
    W8A8_TRY(check_weight(w, K));
    const int64_t N = w->N;
    if (M == 0 || N == 0)
        return W8A8_OK;
    const bool int8 = int8_shape_ok(M, K, N) && w->wq != nullptr && aligned16(x) &&
                      aligned16(y) && aligned16(w->wq) && (bias == nullptr || aligned16(bias));
    if (!int8) {
        // The BF16 fallback needs no scratch: same launch as w8a8_linear's fallback.
        return w8a8_linear(x, M, K, w, bias, y, nullptr, 0, path_taken, stream);
    }
    if (M * K > static_cast<int64_t>(W8A8_NOALLOC_MAX_ELEMS))
        return W8A8_ERR_WORKSPACE;
    W8A8_TRY(check_device_ptr(x));
    W8A8_TRY(check_device_ptr(y));
    W8A8_TRY(check_device_ptr(w->wq));
    W8A8_TRY(check_device_ptr(w->ws));
    if (bias != nullptr)
        W8A8_TRY(check_device_ptr(bias));
    int dev;
    W8A8_TRY(current_device(dev));
    void *scratch = nullptr;
    W8A8_TRY(noalloc_scratch(dev, scratch));
    // The quantize kernel rewrites every code and scale the GEMM then reads, so nothing in
    // the scratch has to be cleared between calls.
    int8_t *xq = static_cast<int8_t *>(scratch);
    float *xs = reinterpret_cast<float *>(static_cast<uint8_t *>(scratch) + kNoAllocCodeBytes);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    W8A8_TRY(launch_quantize(x, M, K, xq, xs, st));
    W8A8_TRY(gemm_i8_impl(xq, xs, M, K, w, bias, y, st));
    if (path_taken != nullptr)
        *path_taken = W8A8_PATH_INT8;
    return W8A8_OK;
}

w8a8_status_t w8a8_linear_prequant(const int8_t *xq, const float *xs, int64_t M, int64_t K,
                                   const w8a8_weight_t *w, const w8a8_bf16_t *bias,
                                   w8a8_bf16_t *y, void *stream)
{
    if (M < 0 || K < 0)
        return W8A8_ERR_INVALID_ARG;
    W8A8_TRY(check_weight(w, K));
    if (w->wq == nullptr)
        return W8A8_ERR_INVALID_ARG;
    if (M == 0 || w->N == 0)
        return W8A8_OK;
    if (!int8_shape_ok(M, K, w->N))
        return W8A8_ERR_SHAPE;
    W8A8_TRY(check_device_ptr(xq));
    W8A8_TRY(check_device_ptr(xs));
    W8A8_TRY(check_device_ptr(w->wq));
    W8A8_TRY(check_device_ptr(w->ws));
    W8A8_TRY(check_device_ptr(y));
    if (bias != nullptr)
        W8A8_TRY(check_device_ptr(bias));
    if (!aligned16(xq) || !aligned16(w->wq) || !aligned16(y) || (bias && !aligned16(bias)))
        return W8A8_ERR_ALIGNMENT;
    return gemm_i8_impl(xq, xs, M, K, w, bias, y, static_cast<cudaStream_t>(stream));
}

w8a8_status_t w8a8_linear_prequant_gated(const int8_t *xq, const float *xs, int64_t M, int64_t K,
                                         const w8a8_weight_t *w, const w8a8_bf16_t *bias,
                                         const w8a8_bf16_t *resid, const w8a8_bf16_t *gate,
                                         int64_t T, w8a8_bf16_t *y, void *stream)
{
    if (M < 0 || K < 0 || T <= 0)
        return W8A8_ERR_INVALID_ARG;
    W8A8_TRY(check_weight(w, K));
    if (w->wq == nullptr)
        return W8A8_ERR_INVALID_ARG;
    if (M % T)
        return W8A8_ERR_SHAPE;
    if (M == 0 || w->N == 0)
        return W8A8_OK;
    if (!int8_shape_ok(M, K, w->N))
        return W8A8_ERR_SHAPE;
    W8A8_TRY(check_device_ptr(xq));
    W8A8_TRY(check_device_ptr(xs));
    W8A8_TRY(check_device_ptr(w->wq));
    W8A8_TRY(check_device_ptr(w->ws));
    W8A8_TRY(check_device_ptr(y));
    W8A8_TRY(check_device_ptr(resid));
    W8A8_TRY(check_device_ptr(gate));
    if (bias != nullptr)
        W8A8_TRY(check_device_ptr(bias));
    if (!aligned16(xq) || !aligned16(w->wq) || !aligned16(y) || (bias && !aligned16(bias)) ||
        !aligned16(resid) || !aligned16(gate))
        return W8A8_ERR_ALIGNMENT;
    return gemm_i8_impl(xq, xs, M, K, w, bias, y, static_cast<cudaStream_t>(stream), resid, gate, T);
}

w8a8_status_t w8a8_bf16_linear(const w8a8_bf16_t *x, const w8a8_bf16_t *w,
                               const w8a8_bf16_t *bias, w8a8_bf16_t *y, int64_t M, int64_t K,
                               int64_t N, void *stream)
{
    if (M < 0 || K < 0 || N < 0)
        return W8A8_ERR_INVALID_ARG;
    if (M == 0 || N == 0)
        return W8A8_OK;
    if (K > 0) {
        W8A8_TRY(check_device_ptr(x));
        W8A8_TRY(check_device_ptr(w));
    }
    W8A8_TRY(check_device_ptr(y));
    if (bias != nullptr)
        W8A8_TRY(check_device_ptr(bias));
    return bf16_impl(x, w, bias, y, M, K, N, static_cast<cudaStream_t>(stream));
}

w8a8_status_t w8a8_rowwise_quantize(const w8a8_bf16_t *x, int64_t rows, int64_t K, int8_t *q,
                                    float *s, void *stream)
{
    if (rows < 0 || K < 0)
        return W8A8_ERR_INVALID_ARG;
    if (K % 8)
        return W8A8_ERR_SHAPE;
    if (rows == 0 || K == 0)
        return rows == 0 ? W8A8_OK : W8A8_ERR_SHAPE;
    W8A8_TRY(check_device_ptr(x));
    W8A8_TRY(check_device_ptr(q));
    W8A8_TRY(check_device_ptr(s));
    if (!aligned16(x) || !aligned16(q) || (reinterpret_cast<uintptr_t>(s) & 3u))
        return W8A8_ERR_ALIGNMENT;
    int dev;
    W8A8_TRY(current_device(dev));
    const int64_t blocks = (rows + quant::kRowWarps - 1) / quant::kRowWarps;
    const int64_t grid = std::min<int64_t>(blocks, static_cast<int64_t>(g_dev[dev].sms) * 16);
    quant::row_quantize_kernel<<<static_cast<unsigned>(grid), quant::kRowWarps * 32, 0,
                                 static_cast<cudaStream_t>(stream)>>>(x, rows, K, q, s);
    return launch_status();
}

w8a8_status_t w8a8_rowwise_linear(const int8_t *xq, const float *xs, int64_t M, int64_t K,
                                  const int8_t *wq, const float *ws, int64_t N,
                                  const w8a8_bf16_t *bias, w8a8_bf16_t *y, void *stream)
{
    if (M < 0 || K < 0 || N < 0)
        return W8A8_ERR_INVALID_ARG;
    if (M == 0 || N == 0)
        return W8A8_OK;
    if (K == 0 || M % 128 || K % 128 || N % 128 || K > kRowMaxK)
        return W8A8_ERR_SHAPE;
    W8A8_TRY(check_device_ptr(xq));
    W8A8_TRY(check_device_ptr(xs));
    W8A8_TRY(check_device_ptr(wq));
    W8A8_TRY(check_device_ptr(ws));
    W8A8_TRY(check_device_ptr(y));
    if (bias != nullptr)
        W8A8_TRY(check_device_ptr(bias));
    if (!aligned16(xq) || !aligned16(wq) || !aligned16(ws) || !aligned16(y) ||
        (reinterpret_cast<uintptr_t>(xs) & 3u) || (bias != nullptr && !aligned16(bias)))
        return W8A8_ERR_ALIGNMENT;
    gemm::Params p{};
    p.M = M;
    p.N = N;
    p.K = K;
    p.xs = xs;
    p.ws = ws;
    p.bias = bias;
    p.y = y;
    return launch_gemm<gemm::Mode::kI8Row>(xq, wq, p, static_cast<cudaStream_t>(stream));
}

w8a8_status_t w8a8_debug_block_sums(const int8_t *xq, const int8_t *wq, int64_t M, int64_t K,
                                    int64_t N, int64_t m0, int64_t rows, int64_t n0, int64_t cols,
                                    int32_t *out, void *stream)
{
    if (M < 0 || K < 0 || N < 0 || m0 < 0 || rows < 0 || n0 < 0 || cols < 0 || m0 + rows > M ||
        n0 + cols > N)
        return W8A8_ERR_INVALID_ARG;
    if (!int8_shape_ok(M, K, N))
        return W8A8_ERR_SHAPE;
    if (rows == 0 || cols == 0)
        return W8A8_OK;
    W8A8_TRY(check_device_ptr(xq));
    W8A8_TRY(check_device_ptr(wq));
    W8A8_TRY(check_device_ptr(out));
    if (!aligned16(xq) || !aligned16(wq))
        return W8A8_ERR_ALIGNMENT;
    // the main loop runs over the 128-aligned rows and columns that cover the window only
    const int64_t mb0 = m0 / 128, mb1 = (m0 + rows + 127) / 128;
    const int64_t nb0 = n0 / 128, nb1 = (n0 + cols + 127) / 128;
    gemm::Params p{};
    p.M = (mb1 - mb0) * 128;
    p.N = (nb1 - nb0) * 128;
    p.K = K;
    p.dump = out;
    p.dm0 = m0 - mb0 * 128;
    p.drows = rows;
    p.dn0 = n0 - nb0 * 128;
    p.dcols = cols;
    return launch_gemm<gemm::Mode::kI8Dump>(xq + mb0 * 128 * K, wq + nb0 * 128 * K, p,
                                            static_cast<cudaStream_t>(stream));
}

int w8a8_device_error(void)
{
    if (cudaDeviceSynchronize() != cudaSuccess) {
        cudaGetLastError();
        return -1;
    }
    int v = 0;
    const int zero = 0;
    if (cudaMemcpyFromSymbol(&v, g_device_error, sizeof(int)) != cudaSuccess ||
        cudaMemcpyToSymbol(g_device_error, &zero, sizeof(int)) != cudaSuccess) {
        cudaGetLastError();
        return -1;
    }
    return v;
}

w8a8_status_t w8a8_debug_wait_timeout(uint64_t timeout_ns, void *stream)
{
    if (timeout_ns > 5000000000ull)
        return W8A8_ERR_INVALID_ARG;
    wait_timeout_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(timeout_ns);
    return launch_status();
}

const char *w8a8_last_cuda_error(void)
{
    return cudaGetErrorString(t_last_cuda_error);
}

const char *w8a8_status_string(w8a8_status_t status)
{
    switch (status) {
    case W8A8_OK: return "ok";
    case W8A8_ERR_INVALID_ARG: return "invalid argument";
    case W8A8_ERR_SHAPE: return "shape not supported by this entry point";
    case W8A8_ERR_NOT_DEVICE: return "buffer is not device memory of the current device";
    case W8A8_ERR_ALIGNMENT: return "buffer not 16-byte aligned";
    case W8A8_ERR_WORKSPACE: return "workspace missing or too small";
    case W8A8_ERR_CUDA: return "CUDA error";
    }
    return "unknown status";
}

} // extern "C"
