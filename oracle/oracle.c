/*
 * oracle.c -- plain, slow CPU reference for the guarded block-wise W8A8 linear layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check in __graft_entry__.py and
 * the CPU-baseline leg of bench.py load this library.  The CUDA library never calls it,
 * and the two share no source, header, table or helper.
 *
 * What it computes, and where the pages define it:
 *   - Block-wise 128x128 quantization of weights ("static", once) and of activations
 *     (every call), one FP32 scale per block, INT8 codes: TurboDiffusion article
 *     (bjdmk.com.cn news 725942), section "训练与推理的极致效率", inference list,
 *     items 3 and 4; also its "稀疏、蒸馏与全链路量化" section (W8A8, 128x128 blocks).
 *   - Symmetric scale = max|.| / 127: TurboT2VA paper ("TurboT2VA: Fast Large-Scale
 *     Text-to-Video-Audio Generation via Score-Regularized Consistency Distillation"),
 *     inference-stack section, W8A8 operator paragraph (the 127 divisor of its scales).
 *     Where the block is all zeros the scale is 1 (that paragraph's epsilon clamp belongs
 *     to its per-row variant; the block-wise contract takes scale 1 instead).
 *   - INT32 accumulation of INT8 products per 128-wide K block, FP32 block scales
 *     applied to each partial product, then summed ("a blockwise quantization strategy
 *     repeatedly applies scales along the reduction dimension"), bias in the epilogue:
 *     same TurboT2VA paragraph.
 *   - RMSNorm ahead of quantization: TurboDiffusion article, inference list, item 5
 *     (norm kernels re-implemented in Triton or CUDA); TurboT2VA paper, fused-operator
 *     paragraph.
 *   - BF16 fallback linear with the retained BF16 weight: TurboT2VA paper,
 *     inference-stack section, guard paragraph.
 *   - The per-row / per-output-channel post-scale operator (the paper's own W8A8
 *     kernel): TurboT2VA paper, W8A8 operator paragraph (see the per-row section).
 *   - Modulated RMSNorm (adaptive scale-shift) and the gated residual update: TurboT2VA
 *     paper, fused-operator paragraph (see the modulated-RMSNorm section).
 *
 * Readings where the pages are silent (each listed in the design notes):
 *   rounding of x/s to an integer is round-half-to-even; x/s is one IEEE FP32 division
 *   by the stored FP32 scale; codes are clamped to [-127, 127]; the two block scales are
 *   multiplied first (FP32), each block's INT32 sum is converted to FP32 and multiplied
 *   by that product, and the K blocks are summed in ascending order in FP32 with no
 *   fused multiply-add; the bias (BF16 widened to FP32) is added once at the end.
 *   RMSNorm: sum of squares in FP64, rstd = 1/sqrt(mean + eps) in FP64 rounded to FP32,
 *   normalised value = bf16((x * rstd) * gamma) with FP32 products.  Modulated RMSNorm:
 *   bf16(fl(fl(n * fl(1 + scale)) + shift)) with one modulation row per T-row sample;
 *   gated residual: bf16(fl(r + fl(gate * v))) on the unrounded FP32 linear output v.
 *
 * Build: gcc -O2 -std=c11 -ffp-contract=off -fno-fast-math -fopenmp -fPIC -shared.
 * OpenMP splits only independent outputs, so the thread count never changes a bit.
 * All BF16 values cross this interface as uint16_t bit patterns.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define BLOCK 128

/* ---------------------------------------------------------------- BF16 <-> FP32 ---- */

static float bf16_to_f32(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* Round-to-nearest-even FP32 -> BF16 (finite values). */
static uint16_t f32_to_bf16(float f)
{
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    u += 0x7FFFu + ((u >> 16) & 1u);
    return (uint16_t)(u >> 16);
}

/* ---------------------------------------------------------------- quantization ---- */

/* Scale of one block from its largest magnitude. */
static float block_scale(float absmax)
{
    if (absmax == 0.0f)
        return 1.0f;
    return absmax / 127.0f;
}

/* One code: IEEE FP32 quotient, rounded half-to-even (rintf in the default rounding
 * mode), clamped to the symmetric INT8 range. */
static int8_t quantize_one(float x, float s)
{
    float q = rintf(x / s);
    if (q > 127.0f)
        q = 127.0f;
    if (q < -127.0f)
        q = -127.0f;
    return (int8_t)q;
}

/* x: [rows, cols] BF16, rows and cols multiples of 128.
 * q: [rows, cols] INT8 codes; s: [rows/128, cols/128] FP32 scales, row-major. */
int oracle_block_quantize(const uint16_t *x, int64_t rows, int64_t cols, int8_t *q, float *s)
{
    if (rows < 0 || cols < 0 || rows % BLOCK || cols % BLOCK)
        return -1;
    const int64_t rb_n = rows / BLOCK, cb_n = cols / BLOCK;
#pragma omp parallel for collapse(2) schedule(static)
    for (int64_t rb = 0; rb < rb_n; ++rb) {
        for (int64_t cb = 0; cb < cb_n; ++cb) {
            float absmax = 0.0f;
            for (int64_t i = rb * BLOCK; i < (rb + 1) * BLOCK; ++i)
                for (int64_t j = cb * BLOCK; j < (cb + 1) * BLOCK; ++j) {
                    float a = fabsf(bf16_to_f32(x[i * cols + j]));
                    if (a > absmax)
                        absmax = a;
                }
            const float sc = block_scale(absmax);
            s[rb * cb_n + cb] = sc;
            for (int64_t i = rb * BLOCK; i < (rb + 1) * BLOCK; ++i)
                for (int64_t j = cb * BLOCK; j < (cb + 1) * BLOCK; ++j)
                    q[i * cols + j] = quantize_one(bf16_to_f32(x[i * cols + j]), sc);
        }
    }
    return 0;
}

/* ---------------------------------------------------------------- block sums ------- */

/* INT8 x INT8 products summed over K block kb, in 64-bit integers. */
static int64_t block_sum(const int8_t *xrow, const int8_t *wrow, int64_t kb)
{
    int64_t acc = 0;
    for (int64_t k = kb * BLOCK; k < (kb + 1) * BLOCK; ++k)
        acc += (int64_t)xrow[k] * (int64_t)wrow[k];
    return acc;
}

/* out[(i * cols + j) * KB + kb] = sum over K block kb of xq[m0+i, k] * wq[n0+j, k].
 * Every such sum fits INT32 (|sum| <= 128 * 127 * 127). */
int oracle_block_sums(const int8_t *xq, const int8_t *wq, int64_t M, int64_t K, int64_t N,
                      int64_t m0, int64_t rows, int64_t n0, int64_t cols, int32_t *out)
{
    if (K % BLOCK || m0 < 0 || n0 < 0 || rows < 0 || cols < 0 || m0 + rows > M ||
        n0 + cols > N)
        return -1;
    const int64_t kbn = K / BLOCK;
#pragma omp parallel for collapse(2) schedule(static)
    for (int64_t i = 0; i < rows; ++i)
        for (int64_t j = 0; j < cols; ++j)
            for (int64_t kb = 0; kb < kbn; ++kb)
                out[(i * cols + j) * kbn + kb] =
                    (int32_t)block_sum(xq + (m0 + i) * K, wq + (n0 + j) * K, kb);
    return 0;
}

/* ---------------------------------------------------------------- W8A8 linear ------ */

/* One output element: sum over K blocks of FP32(block sum) * (xs * ws), then + bias. */
static float w8a8_output(const int8_t *xq, const float *xs, const int8_t *wq, const float *ws,
                         const uint16_t *bias, int64_t K, int64_t m, int64_t n)
{
    const int64_t kbn = K / BLOCK;
    const int64_t mb = m / BLOCK, nb = n / BLOCK;
    float acc = 0.0f;
    for (int64_t kb = 0; kb < kbn; ++kb) {
        const int64_t p = block_sum(xq + m * K, wq + n * K, kb);
        const float scale = xs[mb * kbn + kb] * ws[nb * kbn + kb];
        const float term = (float)p * scale;
        acc = acc + term;
    }
    const float b = bias ? bf16_to_f32(bias[n]) : 0.0f;
    return acc + b;
}

/* Rows [m0, m0 + rows) of the FP32 output: out[(m - m0) * N + n]. */
int oracle_w8a8_linear(const int8_t *xq, const float *xs, const int8_t *wq, const float *ws,
                       const uint16_t *bias, int64_t M, int64_t K, int64_t N, int64_t m0,
                       int64_t rows, float *out)
{
    if (M % BLOCK || K % BLOCK || N % BLOCK || m0 < 0 || rows < 0 || m0 + rows > M)
        return -1;
#pragma omp parallel for collapse(2) schedule(static)
    for (int64_t i = 0; i < rows; ++i)
        for (int64_t n = 0; n < N; ++n)
            out[i * N + n] = w8a8_output(xq, xs, wq, ws, bias, K, m0 + i, n);
    return 0;
}

/* The FP32 output at count sampled coordinates (ms[t], ns[t]). */
int oracle_w8a8_linear_at(const int8_t *xq, const float *xs, const int8_t *wq, const float *ws,
                          const uint16_t *bias, int64_t M, int64_t K, int64_t N,
                          const int64_t *ms, const int64_t *ns, int64_t count, float *out)
{
    if (M % BLOCK || K % BLOCK || N % BLOCK)
        return -1;
    for (int64_t t = 0; t < count; ++t)
        if (ms[t] < 0 || ms[t] >= M || ns[t] < 0 || ns[t] >= N)
            return -1;
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < count; ++t)
        out[t] = w8a8_output(xq, xs, wq, ws, bias, K, ms[t], ns[t]);
    return 0;
}

/* ---------------------------------------------------------------- per-row W8A8 ----- */
/* The post-scale W8A8 operator of the TurboT2VA paper (inference-stack section, W8A8
 * operator paragraph): dynamic per-row activation scales and static per-output-channel
 * weight scales s = max(||row||_inf, eps) / 127 with eps = 1e-4, INT8 codes per row,
 * INT8 products accumulated in INT32 over the whole of K, then both scales and the bias
 * applied once.  The page's formula itself did not survive extraction; the readings are:
 * eps is the FP32 value nearest 1e-4, the codes follow the block path's rule (IEEE FP32
 * quotient by the stored scale, half-to-even, clamp to [-127, 127]), and the output is
 * fl(fl(float(acc) * fl(sx * sw)) + b), float(acc) being the INT32 sum rounded to FP32. */
#define ROW_EPS 1e-4f

/* x: [rows, cols] BF16 -> q: [rows, cols] INT8 codes, s: [rows] FP32 scales. */
int oracle_row_quantize(const uint16_t *x, int64_t rows, int64_t cols, int8_t *q, float *s)
{
    if (rows < 0 || cols < 0)
        return -1;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        float absmax = 0.0f;
        for (int64_t j = 0; j < cols; ++j) {
            const float a = fabsf(bf16_to_f32(x[r * cols + j]));
            if (a > absmax)
                absmax = a;
        }
        const float sc = (absmax > ROW_EPS ? absmax : ROW_EPS) / 127.0f;
        s[r] = sc;
        for (int64_t j = 0; j < cols; ++j)
            q[r * cols + j] = quantize_one(bf16_to_f32(x[r * cols + j]), sc);
    }
    return 0;
}

/* One output element of the per-row operator. */
static float row_output(const int8_t *xq, const float *xs, const int8_t *wq, const float *ws,
                        const uint16_t *bias, int64_t K, int64_t m, int64_t n)
{
    int64_t acc = 0;
    for (int64_t k = 0; k < K; ++k)
        acc += (int64_t)xq[m * K + k] * (int64_t)wq[n * K + k];
    const float scale = xs[m] * ws[n];
    const float v = (float)(int32_t)acc * scale;
    const float b = bias ? bf16_to_f32(bias[n]) : 0.0f;
    return v + b;
}

/* Rows [m0, m0 + rows) of the FP32 output: out[(m - m0) * N + n].  K < 2^31 / 127^2 keeps
 * every sum inside INT32. */
int oracle_row_linear(const int8_t *xq, const float *xs, const int8_t *wq, const float *ws,
                      const uint16_t *bias, int64_t M, int64_t K, int64_t N, int64_t m0,
                      int64_t rows, float *out)
{
    if (M < 0 || K < 0 || N < 0 || K > 133000 || m0 < 0 || rows < 0 || m0 + rows > M)
        return -1;
#pragma omp parallel for collapse(2) schedule(static)
    for (int64_t i = 0; i < rows; ++i)
        for (int64_t n = 0; n < N; ++n)
            out[i * N + n] = row_output(xq, xs, wq, ws, bias, K, m0 + i, n);
    return 0;
}

/* The FP32 output at count sampled coordinates (ms[t], ns[t]). */
int oracle_row_linear_at(const int8_t *xq, const float *xs, const int8_t *wq, const float *ws,
                         const uint16_t *bias, int64_t M, int64_t K, int64_t N, const int64_t *ms,
                         const int64_t *ns, int64_t count, float *out)
{
    if (M < 0 || K < 0 || N < 0 || K > 133000)
        return -1;
    for (int64_t t = 0; t < count; ++t)
        if (ms[t] < 0 || ms[t] >= M || ns[t] < 0 || ns[t] >= N)
            return -1;
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < count; ++t)
        out[t] = row_output(xq, xs, wq, ws, bias, K, ms[t], ns[t]);
    return 0;
}

/* ---------------------------------------------------------------- RMSNorm ---------- */

static float row_rstd(const uint16_t *xrow, int64_t K, float eps)
{
    double ss = 0.0;
    for (int64_t k = 0; k < K; ++k) {
        const double v = (double)bf16_to_f32(xrow[k]);
        ss += v * v;
    }
    const double mean = ss / (double)K;
    return (float)(1.0 / sqrt(mean + (double)eps));
}

static void row_apply(const uint16_t *xrow, const uint16_t *gamma, float rstd, int64_t K,
                      uint16_t *yrow)
{
    for (int64_t k = 0; k < K; ++k) {
        const float t = bf16_to_f32(xrow[k]) * rstd;
        yrow[k] = f32_to_bf16(t * bf16_to_f32(gamma[k]));
    }
}

/* Rows [m0, m0 + rows): y[(m - m0) * K + k] = bf16((x * rstd_m) * gamma_k); rstd[m - m0]. */
int oracle_rmsnorm(const uint16_t *x, const uint16_t *gamma, float eps, int64_t M, int64_t K,
                   int64_t m0, int64_t rows, uint16_t *y, float *rstd)
{
    if (K <= 0 || m0 < 0 || rows < 0 || m0 + rows > M)
        return -1;
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < rows; ++i) {
        const float r = row_rstd(x + (m0 + i) * K, K, eps);
        rstd[i] = r;
        row_apply(x + (m0 + i) * K, gamma, r, K, y + i * K);
    }
    return 0;
}

/* Same normalisation with a given per-row rstd (rows [m0, m0 + rows), rstd[i]). */
int oracle_rmsnorm_apply(const uint16_t *x, const uint16_t *gamma, const float *rstd,
                         int64_t M, int64_t K, int64_t m0, int64_t rows, uint16_t *y)
{
    if (K <= 0 || m0 < 0 || rows < 0 || m0 + rows > M)
        return -1;
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < rows; ++i)
        row_apply(x + (m0 + i) * K, gamma, rstd[i], K, y + i * K);
    return 0;
}

/* ------------------------------------------- modulated RMSNorm, gated residual ----- */
/* TurboT2VA paper, fused-operator paragraph: normalization combined with modality- and
 * timestep-dependent modulation (modulated RMS normalization, adaptive scale-shift
 * modulation), and gated residual updates.  The page names these operations without
 * formulas; the readings are the adaptive-norm form of diffusion transformers, each
 * group of T consecutive rows (one sample's tokens) sharing one modulation row:
 *   modulated RMSNorm: n = fl(x * rstd), times gamma[k] when gamma is given (FP32
 *     product), then y = bf16( fl( fl(n * fl(1 + scale[b, k])) + shift[b, k] ) ) with
 *     b = m / T; rstd as for the plain RMSNorm; no intermediate BF16 rounding.
 *   gated residual: out = bf16( fl( r[m, n] + fl(gate[b, n] * v[m, n]) ) ), v the FP32
 *     linear output (bias included) that the plain linear would round to BF16, b = m / T.
 */
static void row_apply_mod(const uint16_t *xrow, const uint16_t *gamma, const uint16_t *scale,
                          const uint16_t *shift, float rstd, int64_t K, uint16_t *yrow)
{
    for (int64_t k = 0; k < K; ++k) {
        float n = bf16_to_f32(xrow[k]) * rstd;
        if (gamma)
            n = n * bf16_to_f32(gamma[k]);
        const float a = 1.0f + bf16_to_f32(scale[k]);
        const float u = n * a;
        yrow[k] = f32_to_bf16(u + bf16_to_f32(shift[k]));
    }
}

/* Rows [m0, m0 + rows) of the modulated RMSNorm: x [M, K], gamma [K] or NULL, scale and
 * shift [M / T, K]; y [rows, K] BF16 bits, rstd [rows]. */
int oracle_mod_rmsnorm(const uint16_t *x, const uint16_t *gamma, const uint16_t *scale,
                       const uint16_t *shift, int64_t T, float eps, int64_t M, int64_t K,
                       int64_t m0, int64_t rows, uint16_t *y, float *rstd)
{
    if (K <= 0 || T <= 0 || M % T != 0 || m0 < 0 || rows < 0 || m0 + rows > M)
        return -1;
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < rows; ++i) {
        const int64_t m = m0 + i;
        const int64_t b = m / T;
        const float r = row_rstd(x + m * K, K, eps);
        rstd[i] = r;
        row_apply_mod(x + m * K, gamma, scale + b * K, shift + b * K, r, K, y + i * K);
    }
    return 0;
}

/* Same modulated normalisation with a given per-row rstd (rows [m0, m0 + rows), rstd[i]). */
int oracle_mod_rmsnorm_apply(const uint16_t *x, const uint16_t *gamma, const uint16_t *scale,
                             const uint16_t *shift, int64_t T, const float *rstd, int64_t M,
                             int64_t K, int64_t m0, int64_t rows, uint16_t *y)
{
    if (K <= 0 || T <= 0 || M % T != 0 || m0 < 0 || rows < 0 || m0 + rows > M)
        return -1;
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < rows; ++i) {
        const int64_t m = m0 + i;
        const int64_t b = m / T;
        row_apply_mod(x + m * K, gamma, scale + b * K, shift + b * K, rstd[i], K, y + i * K);
    }
    return 0;
}

/* The gated residual at S points (ms[t], ns[t]) of an [M, N] output: v[t] the FP32 linear
 * output there, r[t] the residual's BF16 bits there, gate [M / T, N]; out[t] BF16 bits. */
int oracle_gated_residual(const float *v, const uint16_t *r, const uint16_t *gate, int64_t T,
                          int64_t M, int64_t N, const int64_t *ms, const int64_t *ns, int64_t S,
                          uint16_t *out)
{
    if (T <= 0 || M % T != 0 || N <= 0 || S < 0)
        return -1;
    for (int64_t t = 0; t < S; ++t)
        if (ms[t] < 0 || ms[t] >= M || ns[t] < 0 || ns[t] >= N)
            return -1;
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < S; ++t) {
        const int64_t b = ms[t] / T;
        const float gv = bf16_to_f32(gate[b * N + ns[t]]) * v[t];
        out[t] = f32_to_bf16(bf16_to_f32(r[t]) + gv);
    }
    return 0;
}

/* ---------------------------------------------------------------- BF16 linear ------ */

static float bf16_output(const uint16_t *x, const uint16_t *w, const uint16_t *bias,
                         int64_t K, int64_t m, int64_t n)
{
    double acc = 0.0;
    for (int64_t k = 0; k < K; ++k)
        acc += (double)bf16_to_f32(x[m * K + k]) * (double)bf16_to_f32(w[n * K + k]);
    const float b = bias ? bf16_to_f32(bias[n]) : 0.0f;
    return (float)acc + b;
}

/* y = x * w^T (+ bias) for any M, K, N; rows [m0, m0 + rows); FP32 out[(m - m0) * N + n]. */
int oracle_bf16_linear(const uint16_t *x, const uint16_t *w, const uint16_t *bias, int64_t M,
                       int64_t K, int64_t N, int64_t m0, int64_t rows, float *out)
{
    if (M < 0 || K < 0 || N < 0 || m0 < 0 || rows < 0 || m0 + rows > M)
        return -1;
#pragma omp parallel for collapse(2) schedule(static)
    for (int64_t i = 0; i < rows; ++i)
        for (int64_t n = 0; n < N; ++n)
            out[i * N + n] = bf16_output(x, w, bias, K, m0 + i, n);
    return 0;
}

int oracle_bf16_linear_at(const uint16_t *x, const uint16_t *w, const uint16_t *bias,
                          int64_t M, int64_t K, int64_t N, const int64_t *ms,
                          const int64_t *ns, int64_t count, float *out)
{
    for (int64_t t = 0; t < count; ++t)
        if (ms[t] < 0 || ms[t] >= M || ns[t] < 0 || ns[t] >= N)
            return -1;
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < count; ++t)
        out[t] = bf16_output(x, w, bias, K, ms[t], ns[t]);
    return 0;
}

/* ---------------------------------------------------------------- helpers ---------- */

/* FP32 -> BF16 (RNE), elementwise, for comparing FP32 outputs after BF16 rounding. */
void oracle_f32_to_bf16(const float *in, int64_t n, uint16_t *out)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = f32_to_bf16(in[i]);
}

/* Threads OpenMP will use (1 when built without OpenMP). */
int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
