/*
 * w8a8.h -- C ABI of the B200 (sm_100a) guarded block-wise W8A8 linear layer.
 *
 * The operation (TurboDiffusion article, bjdmk.com.cn news 725942, section
 * "训练与推理的极致效率", inference list items 3-4; TurboT2VA paper, "TurboT2VA: Fast
 * Large-Scale Text-to-Video-Audio Generation via Score-Regularized Consistency
 * Distillation", inference-stack section, W8A8 operator and guard paragraphs):
 *
 *   X[M,K] (BF16) and W[N,K] (BF16, nn.Linear layout: row n is output channel n) are cut
 *   into 128x128 blocks.  Each block gets one FP32 scale s = max|block| / 127 (s = 1 for an
 *   all-zero block) and INT8 codes q = clamp(round_half_even(v / s), -127, 127), where
 *   v / s is an IEEE FP32 division.  Weights are quantized once ("static"), activations on
 *   every call.  The output is
 *
 *     Y[m,n] = bf16( sum_kb float(P[m,n,kb]) * (xs[m/128,kb] * ws[n/128,kb]) + bias[n] ),
 *     P[m,n,kb] = sum_{k = 128 kb}^{128 kb + 127} xq[m,k] * wq[n,k]   (exact INT32),
 *
 *   i.e. the INT32 partial product of each 128-wide K block is rescaled by the two FP32
 *   block scales before the blocks are summed in FP32.
 *
 *   Guard (TurboT2VA paper, guard paragraph): the INT8 path runs only for BF16 device
 *   buffers whose flattened M, K and N are all multiples of 128; every other shape runs a
 *   BF16 GEMM on the retained BF16 weight.  There is no CPU path.
 *
 * Conventions for every entry point:
 *   - All matrices are row-major and contiguous.  BF16 values are passed as uint16_t
 *     bit patterns (w8a8_bf16_t).  Sizes are element counts.
 *   - Every buffer is owned by the caller and must be device memory (cudaMalloc /
 *     PyTorch CUDA tensors) on the current device.  The library allocates no device
 *     memory and keeps no state between calls other than a small host-side cache.
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream).  All work is
 *     enqueued on it and the call returns without waiting: outputs are ready once the
 *     stream reaches that point.
 *   - Argument errors are reported synchronously by the return code, before anything is
 *     enqueued.  A failed launch returns W8A8_ERR_CUDA.  Faults inside a kernel surface
 *     through the CUDA runtime as usual.  Every wait inside the kernels gives up after
 *     about two seconds; the kernel then records W8A8_DEVERR_TIMEOUT in a device word
 *     that w8a8_device_error() reads and clears.
 *   - Outputs must not overlap inputs.
 */
#ifndef W8A8_H_
#define W8A8_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define W8A8_API __attribute__((visibility("default")))
#else
#define W8A8_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef uint16_t w8a8_bf16_t;   /* bfloat16 bit pattern */

typedef enum {
    W8A8_OK = 0,
    W8A8_ERR_INVALID_ARG = 1,   /* NULL pointer where one is required, negative size  */
    W8A8_ERR_SHAPE = 2,         /* a 128-multiple was required and not given          */
    W8A8_ERR_NOT_DEVICE = 3,    /* a buffer is host memory or on another device       */
    W8A8_ERR_ALIGNMENT = 4,     /* a buffer is not 16-byte aligned                     */
    W8A8_ERR_WORKSPACE = 5,     /* workspace missing or smaller than required          */
    W8A8_ERR_CUDA = 6           /* a CUDA runtime call or a launch failed              */
} w8a8_status_t;

typedef enum {
    W8A8_PATH_INT8 = 0,         /* quantize activations + INT8 block-scaled GEMM       */
    W8A8_PATH_BF16 = 1,         /* guard rejected the shape: BF16 GEMM                 */
    W8A8_PATH_NONE = 2          /* nothing to compute (M == 0 or N == 0)               */
} w8a8_path_t;

/* Device-side error codes read by w8a8_device_error(). */
#define W8A8_DEVERR_NONE 0
#define W8A8_DEVERR_TIMEOUT 1   /* a bounded wait inside a kernel gave up              */

/* A linear layer's weight as the caller keeps it.
 *   w_bf16: [N, K] BF16, always required (the fallback GEMM uses it; the guard
 *           paragraph's "retained BF16 weight copy").
 *   wq:     [N, K] INT8 codes from w8a8_quantize_weight, or NULL when N or K is not a
 *           multiple of 128 (the layer then always takes the BF16 path).
 *   ws:     [N/128, K/128] FP32 block scales, NULL exactly when wq is NULL. */
typedef struct {
    int64_t N;
    int64_t K;
    const w8a8_bf16_t *w_bf16;
    const int8_t *wq;
    const float *ws;
} w8a8_weight_t;

/* Block-wise 128x128 quantization of a weight, done once when the layer is loaded.
 *   w [N, K] BF16 -> wq [N, K] INT8 and ws [N/128, K/128] FP32 (row-major).
 *   N and K must be positive multiples of 128 (else W8A8_ERR_SHAPE); all three buffers
 *   16-byte aligned.  Same arithmetic as w8a8_quantize_act. */
W8A8_API w8a8_status_t w8a8_quantize_weight(const w8a8_bf16_t *w, int64_t N, int64_t K, int8_t *wq,
                                   float *ws, void *stream);

/* Block-wise 128x128 dynamic quantization of activations (TurboDiffusion article,
 * inference list item 4: activations quantized at the weights' block granularity).
 *   x [M, K] BF16 -> xq [M, K] INT8 and xs [M/128, K/128] FP32.
 *   M and K multiples of 128 (else W8A8_ERR_SHAPE; M == 0 is a no-op); 16-byte aligned.
 *   Reads x once and writes xq, xs once. */
W8A8_API w8a8_status_t w8a8_quantize_act(const w8a8_bf16_t *x, int64_t M, int64_t K, int8_t *xq,
                                float *xs, void *stream);

/* RMSNorm fused ahead of the activation quantizer (TurboDiffusion article, inference
 * list item 5: norm kernels re-implemented in CUDA; TurboT2VA paper, fused-operator
 * paragraph).  For each row m:
 *     rstd[m] = fp32( 1 / sqrt( (sum_k x[m,k]^2) / K + eps ) )   (sum and sqrt in FP64)
 *     y[m,k]  = bf16( (x[m,k] * rstd[m]) * gamma[k] )            (FP32 products)
 *   and y is block-quantized exactly as by w8a8_quantize_act, without being stored.
 *   x [M, K] BF16, gamma [K] BF16 or NULL (then y = bf16(x * rstd)) -> xq [M, K] INT8,
 *   xs [M/128, K/128] FP32, and rstd_out [M] FP32 when not NULL.
 *   M, K multiples of 128 (else W8A8_ERR_SHAPE; M == 0 is a no-op), eps >= 0 and finite
 *   (else W8A8_ERR_INVALID_ARG); x, gamma, xq 16-byte aligned, xs and rstd_out 4-byte
 *   aligned.  Two forms, chosen by shape:
 *   - M below 192 rows per SM: one grid; each row's sum of squares is split across a
 *     cluster of CTAs, so its FP64 summation order differs from the running sum above,
 *     and rstd may differ from it by one FP32 ulp on rows whose FP64 value lies within
 *     about 1e-15 of an FP32 rounding boundary.  Each block of x is loaded twice, the
 *     second time mostly from L2.
 *   - M from 192 rows per SM on: a grid that sums each row's squares in column order (so
 *     rstd equals the running-sum definition bit for bit), then the block quantizer
 *     normalising each block as it arrives; x is read twice from HBM.  Without rstd_out
 *     the M floats between the two grids come from the device's stream-ordered
 *     allocator (cudaMallocAsync / cudaFreeAsync on `stream`).
 *   Either way the codes and scales are those of y computed from the rstd returned. */
W8A8_API w8a8_status_t w8a8_rmsnorm_quantize_act(const w8a8_bf16_t *x, const w8a8_bf16_t *gamma,
                                        float eps, int64_t M, int64_t K, int8_t *xq,
                                        float *xs, float *rstd_out, void *stream);

/* Modulated RMSNorm (adaptive scale-shift of diffusion transformers) fused ahead of the
 * activation quantizer (TurboT2VA paper, fused-operator paragraph: modulated RMS
 * normalization and scale-shift modulation, with modality- and timestep-dependent
 * modulation; the page gives no formula, this is the adaptive-norm form).  Rows come in
 * groups of T consecutive rows (one sample's tokens) sharing one modulation row b = m / T:
 *     n[m,k]  = fl(x[m,k] * rstd[m]), times gamma[k] (FP32 product) when gamma != NULL
 *     y[m,k]  = bf16( fl( fl(n[m,k] * fl(1 + scale[b,k])) + shift[b,k] ) )
 *   with rstd as above, and y block-quantized as by w8a8_quantize_act, not stored.
 *   scale, shift [M/T, K] BF16 device buffers, 16-byte aligned.  T > 0 (else
 *   W8A8_ERR_INVALID_ARG), T a multiple of 128 dividing M (else W8A8_ERR_SHAPE); the
 *   other arguments as for w8a8_rmsnorm_quantize_act. */
W8A8_API w8a8_status_t w8a8_rmsnorm_mod_quantize_act(const w8a8_bf16_t *x, const w8a8_bf16_t *gamma,
                                            const w8a8_bf16_t *scale, const w8a8_bf16_t *shift,
                                            int64_t T, float eps, int64_t M, int64_t K,
                                            int8_t *xq, float *xs, float *rstd_out, void *stream);

/* Bytes of device workspace w8a8_linear needs for an M x K activation on the INT8 path:
 * the INT8 codes (M*K bytes, rounded up to 256) followed by the FP32 scales.  Returns 0
 * when the shape takes the BF16 path. */
W8A8_API size_t w8a8_linear_workspace_bytes(int64_t M, int64_t K, int64_t N);

/* The guarded W8A8 linear: Y[M, N] = X[M, K] W^T + bias, BF16 out.
 *   x:    [M, K] BF16 device buffer (flattened leading dimensions).
 *   w:    host pointer to the weight record (the buffers it names are device memory).
 *   bias: [N] BF16 or NULL.
 *   y:    [M, N] BF16.
 *   workspace: device buffer of at least w8a8_linear_workspace_bytes(M, K, N) bytes,
 *          used for the quantized activations; may be NULL when that size is 0.
 *   path_taken: if not NULL, receives the w8a8_path_t that ran.
 * Guard: INT8 path iff M, K, N > 0 and all multiples of 128, K <= 65536, w->wq and
 * w->ws are present, and x, y, wq, workspace are 16-byte aligned.  Otherwise the BF16
 * GEMM runs on w->w_bf16 (any M, K, N >= 0; K == 0 gives y = bias or 0).
 * On the INT8 path two kernels run on `stream`: the activation quantizer, then the GEMM,
 * launched as a programmatic dependent of it (cudaLaunchAttributeProgrammaticStream-
 * Serialization): the GEMM's set-up overlaps the quantizer's last blocks and it reads
 * nothing before the quantizer has completed.  Stream order is unchanged for the
 * caller. */
W8A8_API w8a8_status_t w8a8_linear(const w8a8_bf16_t *x, int64_t M, int64_t K, const w8a8_weight_t *w,
                          const w8a8_bf16_t *bias, w8a8_bf16_t *y, void *workspace,
                          size_t workspace_bytes, int *path_taken, void *stream);

/* Rows per chunk that w8a8_linear_host uses when chunk_rows is 0: 4 MiB of x per chunk
 * (K BF16 values per row), rounded down to a multiple of 128 rows, at least 128. */
W8A8_API int64_t w8a8_linear_host_chunk_rows(int64_t M, int64_t K);

/* Bytes of device workspace w8a8_linear_host needs: two x chunks and two y chunks
 * (C = the chunk rows in use: chunk_rows, or the default above, capped at M), each
 * rounded up to 256 bytes, followed by w8a8_linear_workspace_bytes(C, K, N). */
W8A8_API size_t w8a8_linear_host_workspace_bytes(int64_t M, int64_t K, int64_t N,
                                                 int64_t chunk_rows);

/* w8a8_linear on activations and outputs in HOST memory.  The operation and the guard
 * are those of w8a8_linear (TurboT2VA paper, W8A8 operator and guard paragraphs); the
 * streaming of host buffers through the GPU is this library's own.
 *   x_host: [M, K] BF16 host buffer; y_host: [M, N] BF16 host buffer.  Pinned
 *           (page-locked) memory lets the copies overlap; pageable memory works, slower.
 *           Device or managed pointers here give W8A8_ERR_INVALID_ARG.
 *   w, bias: as for w8a8_linear (device buffers).
 *   workspace: device buffer of at least w8a8_linear_host_workspace_bytes(M, K, N,
 *           chunk_rows) bytes, 16-byte aligned; else W8A8_ERR_WORKSPACE.
 *   chunk_rows: rows per chunk, 0 for w8a8_linear_host_chunk_rows(M, K); a positive value
 *           must be a multiple of 128 (else W8A8_ERR_INVALID_ARG).
 * The guard is decided once for the whole [M, K] input exactly as w8a8_linear decides it
 * (host pointers aside), and every chunk then takes that path, so y_host receives the
 * same bits as w8a8_linear on device copies of x.  The rows go through the GPU in chunks:
 * the copy of chunk i + 1 to the device, the linear on chunk i and the copy of chunk
 * i - 1 back to y_host overlap on three streams.  The linear runs on `stream`; the copies
 * run on two streams of the library's own, which the first call on each device creates
 * (with seven events), so make that first call outside stream capture.  Everything is
 * ordered after the work already enqueued on `stream`, and `stream` waits for the last
 * copy back: when `stream` reaches the end of the call's work, y_host is complete.  Calls
 * are enqueued one at a time (a lock per library); calls that share a workspace must be
 * ordered on the same stream or synchronized. */
W8A8_API w8a8_status_t w8a8_linear_host(const w8a8_bf16_t *x_host, int64_t M, int64_t K,
                                        const w8a8_weight_t *w, const w8a8_bf16_t *bias,
                                        w8a8_bf16_t *y_host, void *workspace,
                                        size_t workspace_bytes, int64_t chunk_rows,
                                        int *path_taken, void *stream);

/* Largest M * K that w8a8_linear_noalloc accepts on the INT8 path (16 Mi elements,
 * e.g. M = K = 4096). */
#define W8A8_NOALLOC_MAX_ELEMS (16777216LL)

/* w8a8_linear for callers that cannot allocate device memory.  The paper has no
 * counterpart to this entry point; it exists for users of this library.
 *
 * Some callers may not call cudaMalloc at all: code embedded in a host program that owns
 * every byte of device memory through its own pool and forbids side allocations, or a
 * latency-critical loop that cannot risk an allocation synchronizing the device or
 * failing under memory pressure.  Such callers cannot provide w8a8_linear's workspace.
 * This entry point computes exactly what w8a8_linear computes, with the same kernels and
 * the same guard, but keeps the quantized activations in a fixed scratch array that is
 * part of the library itself (16 MiB + 4 KiB of device memory, reserved on every GPU
 * that loads the library and held until the process exits).  It calls no allocation
 * routine.  The caller still passes x, the weight record, bias and y.
 *
 *   - INT8-path shapes with M * K > W8A8_NOALLOC_MAX_ELEMS are rejected with
 *     W8A8_ERR_WORKSPACE before anything is enqueued.  Shapes that the guard sends to the
 *     BF16 GEMM need no scratch and are not limited.
 *   - The first call on each device looks up the scratch array's device address (with
 *     that device current) and caches it; make that first call before any stream
 *     capture begins.
 *   - All calls on a device share the one scratch array, and it keeps whatever the last
 *     call wrote.  Nothing in it needs clearing (each call rewrites all it reads), but
 *     calls whose work overlaps on the GPU (different streams, or different host threads,
 *     without ordering between them) race on it and may produce wrong results: order such
 *     calls, e.g. by issuing them on one stream. */
W8A8_API w8a8_status_t w8a8_linear_noalloc(const w8a8_bf16_t *x, int64_t M, int64_t K,
                                           const w8a8_weight_t *w, const w8a8_bf16_t *bias,
                                           w8a8_bf16_t *y, int *path_taken, void *stream);

/* The INT8 GEMM with per-K-block rescale on activations that are already quantized
 * (e.g. by w8a8_rmsnorm_quantize_act).  xq [M, K] INT8, xs [M/128, K/128] FP32, the
 * weight's wq/ws, bias [N] or NULL, y [M, N] BF16.  M, K, N multiples of 128
 * (else W8A8_ERR_SHAPE); K <= 65536. */
W8A8_API w8a8_status_t w8a8_linear_prequant(const int8_t *xq, const float *xs, int64_t M, int64_t K,
                                   const w8a8_weight_t *w, const w8a8_bf16_t *bias,
                                   w8a8_bf16_t *y, void *stream);

/* w8a8_linear_prequant with the gated residual update fused into its epilogue
 * (TurboT2VA paper, fused-operator paragraph: gated residual updates; the page gives no
 * formula, this is the adaptive-norm block's form):
 *     y[m,n] = bf16( fl( resid[m,n] + fl( gate[m/T, n] * v[m,n] ) ) )
 * where v[m,n] is the FP32 value w8a8_linear_prequant would round to BF16 (bias
 * included).  resid [M, N] BF16 may be y itself (an in-place update h += gate * linear);
 * gate [M/T, N] BF16 must not overlap y.  T > 0 (else W8A8_ERR_INVALID_ARG) and dividing
 * M (else W8A8_ERR_SHAPE); resid and gate 16-byte aligned device buffers; the rest as for
 * w8a8_linear_prequant.  There is no BF16-path counterpart: shapes outside the INT8
 * guard are rejected with W8A8_ERR_SHAPE and the caller applies the update itself. */
W8A8_API w8a8_status_t w8a8_linear_prequant_gated(const int8_t *xq, const float *xs, int64_t M,
                                                  int64_t K, const w8a8_weight_t *w,
                                                  const w8a8_bf16_t *bias,
                                                  const w8a8_bf16_t *resid,
                                                  const w8a8_bf16_t *gate, int64_t T,
                                                  w8a8_bf16_t *y, void *stream);

/* The BF16 GEMM that the guard falls back to, callable directly:
 *   y[M, N] = bf16( sum_k x[m,k] w[n,k] (FP32 accumulation) + bias[n] ).
 *   Any M, K, N >= 0.  Uses tcgen05 tensor cores when K is a multiple of 8 and the
 *   buffers are 16-byte aligned, else a CUDA-core kernel. */
W8A8_API w8a8_status_t w8a8_bf16_linear(const w8a8_bf16_t *x, const w8a8_bf16_t *w,
                               const w8a8_bf16_t *bias, w8a8_bf16_t *y, int64_t M, int64_t K,
                               int64_t N, void *stream);

/* ---- The per-row / per-output-channel post-scale operator ---------------------------
 * TurboT2VA paper, inference-stack section, W8A8 operator paragraph: activations get one
 * scale per row (dynamic) and weights one per output channel (static),
 *   s = max(||row||_inf, eps) / 127,  eps = 1e-4 (as the FP32 value nearest it),
 * codes q = clamp(round_half_even(fl32(v / s)), -127, 127) as in the block-wise path,
 * INT8 products accumulated in INT32 over the whole of K, and both scales and the bias
 * applied once: y[m,n] = bf16( fl(fl(float(acc[m,n]) * fl(xs[m] * ws[n])) + bias[n]) ),
 * float(acc) being the INT32 sum rounded to FP32.  (The page's formula itself was lost in
 * extraction; these are the readings the oracle and the kernels share.) */

/* Per-row quantization of x [rows, K] BF16 (activations, or a weight [N, K] for its
 * per-output-channel codes): q [rows, K] INT8 and s [rows] FP32, caller-owned device
 * buffers; x and q 16-byte aligned, s 4-byte aligned.  K a multiple of 8 and > 0 (else
 * W8A8_ERR_SHAPE).  Asynchronous on `stream`. */
W8A8_API w8a8_status_t w8a8_rowwise_quantize(const w8a8_bf16_t *x, int64_t rows, int64_t K,
                                             int8_t *q, float *s, void *stream);

/* y [M, N] BF16 from xq [M, K] / xs [M] (per-row) and wq [N, K] / ws [N] (per output
 * channel), bias [N] BF16 or NULL.  M, K, N multiples of 128 and K <= 133120 (so every
 * INT32 sum fits), else W8A8_ERR_SHAPE; xq, wq, ws, y, bias 16-byte aligned, xs 4-byte
 * aligned, else W8A8_ERR_ALIGNMENT.  The INT8 tcgen05 main loop of w8a8_linear with one
 * accumulator per 128 x 256 tile over all of K.  Asynchronous on `stream`. */
W8A8_API w8a8_status_t w8a8_rowwise_linear(const int8_t *xq, const float *xs, int64_t M, int64_t K,
                                           const int8_t *wq, const float *ws, int64_t N,
                                           const w8a8_bf16_t *bias, w8a8_bf16_t *y,
                                           void *stream);

/* Test hook: the INT32 partial products P[m, n, kb] = sum over the 128 k of K block kb of
 * xq[m, k] wq[n, k] (TurboT2VA paper, W8A8 operator paragraph: INT32 accumulation; the
 * block-wise strategy's per-K-block sums), written by the same tensor-core main loop as
 * w8a8_linear, for xq [M, K] and wq [N, K] (M, K, N multiples of 128, else
 * W8A8_ERR_SHAPE) on the window of rows m0 .. m0 + rows - 1 and columns n0 .. n0 + cols -
 * 1 (any offsets and sizes inside [M, N], else W8A8_ERR_INVALID_ARG).  out: [rows, cols,
 * K/128] INT32 device buffer, caller-owned.  The main loop covers only the 128-aligned
 * rows and columns around the window, so full-size operands can be spot-checked.
 * Asynchronous on `stream`. */
W8A8_API w8a8_status_t w8a8_debug_block_sums(const int8_t *xq, const int8_t *wq, int64_t M, int64_t K,
                                    int64_t N, int64_t m0, int64_t rows, int64_t n0, int64_t cols,
                                    int32_t *out, void *stream);

/* Synchronizes the current device and returns (and clears) the device error word:
 * W8A8_DEVERR_NONE or W8A8_DEVERR_TIMEOUT. */
W8A8_API int w8a8_device_error(void);

/* Test hook for the bounded waits: launches one CTA that waits on a barrier nothing
 * arrives on, giving up after timeout_ns nanoseconds; the device error word then reads
 * W8A8_DEVERR_TIMEOUT.  Touches no caller memory. */
W8A8_API w8a8_status_t w8a8_debug_wait_timeout(uint64_t timeout_ns, void *stream);

/* The CUDA runtime's description of the last CUDA error that made a call of this thread
 * return W8A8_ERR_CUDA ("no error" if none).  Static storage; do not free. */
W8A8_API const char *w8a8_last_cuda_error(void);

/* A short static description of a status code. */
W8A8_API const char *w8a8_status_string(w8a8_status_t status);

#ifdef __cplusplus
}
#endif

#endif /* W8A8_H_ */
