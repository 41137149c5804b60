// quant.cuh -- block-wise 128x128 INT8 quantization of BF16 matrices (activations every
// call, weights once), and RMSNorm fused ahead of it.
//
// Per block (TurboDiffusion article, inference list items 3-4; divisor 127 from the
// TurboT2VA paper's W8A8 operator paragraph):
//   s = max|v| / 127 (IEEE FP32 division; s = 1 for an all-zero block)
//   q = clamp(round_half_even(fl32(v / s)), -127, 127)
//
// Codes are computed as y = v * fl32(1/s), rounded to an integer by adding 1.5 * 2^23
// (round-to-nearest-even on the FP32 adder).  |y - fl32(v / s)| <= 1.9e-5 because
// |v / s| <= 127 * (1 + 2^-23) and both the reciprocal and the product are correctly
// rounded, so whenever y is farther than 2^-14 from every half-integer the two round to
// the same integer.  The few entries closer than that are recomputed with the IEEE
// division itself, so the codes equal those of the definition bit for bit.  The clamp
// cannot fire on the fast path (|y| <= 127 * (1 + 2^-22) rounds to at most 127); the
// exact path keeps it.
#pragma once

#include "common.cuh"

namespace w8a8 {
namespace quant {

constexpr float kRoundMagic = 12582912.0f;            // 1.5 * 2^23
constexpr float kTieBand = 0.5f - 1.0f / 16384.0f;     // entries with |y - rne(y)| >= this
constexpr int kThreads = 256;                          // one 128x128 block per CTA pass

// Exact code of one value: IEEE quotient by the stored scale, rint (half to even), clamp.
__device__ __forceinline__ uint32_t code_exact(float v, float sc)
{
    float q = rintf(__fdiv_rn(v, sc));
    q = fminf(fmaxf(q, -127.0f), 127.0f);
    return static_cast<uint32_t>(static_cast<int>(q)) & 0xFFu;
}

// Codes of 8 BF16 values (4 packed words, element 2i in the low half of w[i]) as 8 bytes.
// `exact` forces the division path for all 8 (used when 1/s overflows, i.e. for blocks
// whose scale is below 2^-128).
__device__ __forceinline__ uint2 quantize8(const uint32_t (&w)[4], float sc, float rc, bool exact)
{
    uint32_t t[8];
    float dmax = 0.0f;
    const float2 r2 = make_float2(rc, rc);
    const float2 mg = make_float2(kRoundMagic, kRoundMagic);
    const float2 nmg = make_float2(-kRoundMagic, -kRoundMagic);
    const float2 neg1 = make_float2(-1.0f, -1.0f);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 v = make_float2(bf16_lo(w[i]), bf16_hi(w[i]));
        const float2 y = __fmul2_rn(v, r2);          // ~ v / s
        const float2 tt = __fadd2_rn(y, mg);         // 1.5*2^23 + rne(y): low byte = code
        const float2 n = __fadd2_rn(tt, nmg);        // rne(y), exact
        const float2 d = __ffma2_rn(n, neg1, y);     // y - rne(y), exact, in [-0.5, 0.5]
        dmax = fmaxf(dmax, fmaxf(fabsf(d.x), fabsf(d.y)));
        t[2 * i] = __float_as_uint(tt.x);
        t[2 * i + 1] = __float_as_uint(tt.y);
    }
    if (exact || dmax >= kTieBand) {
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const float v = (j & 1) ? bf16_hi(w[j >> 1]) : bf16_lo(w[j >> 1]);
            t[j] = code_exact(v, sc);
        }
    }
    uint2 out;
    out.x = __byte_perm(__byte_perm(t[0], t[1], 0x0040), __byte_perm(t[2], t[3], 0x0040), 0x5410);
    out.y = __byte_perm(__byte_perm(t[4], t[5], 0x0040), __byte_perm(t[6], t[7], 0x0040), 0x5410);
    return out;
}

// Largest |BF16| among 8 values, as a BF16 magnitude pattern in the low 16 bits
// (for finite values the magnitude order equals the unsigned order of the patterns).
__device__ __forceinline__ uint32_t absmax8_bits(const uint32_t (&w)[4], uint32_t m)
{
#pragma unroll
    for (int i = 0; i < 4; ++i)
        m = __vmaxu2(m, w[i] & 0x7FFF7FFFu);
    return m;
}

// CTA-wide max of per-thread packed magnitudes; returns the block scale (and writes it).
// `red` holds 8 words of shared memory; ends with a barrier so that `red` can be reused
// only after the next call's first barrier.
__device__ __forceinline__ float block_scale_from(uint32_t m2, uint32_t *red)
{
    uint32_t m = max(m2 & 0xFFFFu, m2 >> 16);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
    if ((threadIdx.x & 31) == 0)
        red[threadIdx.x >> 5] = m;
    __syncthreads();
    uint32_t a = red[0];
#pragma unroll
    for (int i = 1; i < kThreads / 32; ++i)
        a = max(a, red[i]);
    const float amax = __uint_as_float(a << 16);
    return (amax == 0.0f) ? 1.0f : __fdiv_rn(amax, 127.0f);
}

// x [rows, K] BF16 -> q [rows, K] INT8, s [rows/128, K/128] FP32.  Grid-stride over the
// (rows/128) * (K/128) blocks.  Thread t covers rows (t / 16) + 16 i, i = 0..7, and the
// 8 columns 8 (t % 16) .. + 7 of the block: a warp's 16-byte loads cover two full
// 256-byte rows, its 8-byte stores two full 128-byte rows.
__global__ void __launch_bounds__(kThreads) quantize_blocks_kernel(
    const uint16_t *__restrict__ x, int64_t K, int64_t nblocks, int64_t KB,
    int8_t *__restrict__ q, float *__restrict__ s)
{
    __shared__ uint32_t red[kThreads / 32];
    const int rg = threadIdx.x >> 4;
    const int cc = threadIdx.x & 15;
    for (int64_t blk = blockIdx.x; blk < nblocks; blk += gridDim.x) {
        const int64_t mb = blk / KB, kb = blk - mb * KB;
        const int64_t off = (mb * 128 + rg) * K + kb * 128 + cc * 8;
        uint32_t w[8][4];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const uint4 v = ld_nc_v4(x + off + static_cast<int64_t>(i) * 16 * K);
            w[i][0] = v.x; w[i][1] = v.y; w[i][2] = v.z; w[i][3] = v.w;
        }
        uint32_t m = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i)
            m = absmax8_bits(w[i], m);
        const float sc = block_scale_from(m, red);
        const float rc = __frcp_rn(sc);
        const bool exact = !(rc <= 3.0e38f);
        if (threadIdx.x == 0)
            s[blk] = sc;
#pragma unroll
        for (int i = 0; i < 8; ++i)
            *reinterpret_cast<uint2 *>(q + off + static_cast<int64_t>(i) * 16 * K) =
                quantize8(w[i], sc, rc, exact);
        __syncthreads();
    }
}

// ------------------------------------------------------------------ fused RMSNorm ------

constexpr int kNormCluster = 8;    // CTAs sharing one 128-row strip

__device__ __forceinline__ uint32_t cluster_ctarank()
{
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

__device__ __forceinline__ void cluster_sync_all()
{
    asm volatile("barrier.cluster.arrive.release.aligned;\n\t"
                 "barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

__device__ __forceinline__ double ld_dsmem_f64(const double *p, uint32_t rank)
{
    uint32_t remote;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(smem_u32(p)), "r"(rank));
    double v;
    asm volatile("ld.shared::cluster.f64 %0, [%1];" : "=d"(v) : "r"(remote) : "memory");
    return v;
}

// RMSNorm + block quantization.  A cluster of 8 CTAs owns one 128-row strip at a time;
// CTA r handles the 128-column blocks r, r + 8, r + 16, ...  Pass 1 sums x^2 per row in
// FP64 over its blocks; the 8 partial sums of each row are exchanged through distributed
// shared memory and added in rank order, so every CTA derives the same rstd.  Pass 2
// re-reads its blocks (the strip was read moments before, so these reads are served by
// L2), forms bf16((x * rstd) * gamma) and quantizes each block as quantize_blocks_kernel.
__global__ void __cluster_dims__(kNormCluster, 1, 1) __launch_bounds__(kThreads)
    rmsnorm_quantize_kernel(const uint16_t *__restrict__ x, const uint16_t *__restrict__ gamma,
                            float eps, int64_t MB, int64_t K, int8_t *__restrict__ q,
                            float *__restrict__ s, float *__restrict__ rstd_out)
{
    __shared__ double part[2][128];
    __shared__ uint32_t red[kThreads / 32];
    const uint32_t rank = cluster_ctarank();
    const int64_t cluster = blockIdx.x / kNormCluster;
    const int64_t nclusters = gridDim.x / kNormCluster;
    const int64_t KB = K / 128;
    const int rg = threadIdx.x >> 4;
    const int cc = threadIdx.x & 15;
    int par = 0;
    for (int64_t mb = cluster; mb < MB; mb += nclusters, par ^= 1) {
        // pass 1: per-row partial sums of squares over this CTA's column blocks
        double acc[8];
#pragma unroll
        for (int i = 0; i < 8; ++i)
            acc[i] = 0.0;
        for (int64_t kb = rank; kb < KB; kb += kNormCluster) {
            const int64_t off = (mb * 128 + rg) * K + kb * 128 + cc * 8;
            uint4 v[8];
#pragma unroll
            for (int i = 0; i < 8; ++i)
                v[i] = ld_nc_v4(x + off + static_cast<int64_t>(i) * 16 * K);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const uint32_t ww[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const double a = bf16_lo(ww[j]), b = bf16_hi(ww[j]);
                    acc[i] = fma(a, a, acc[i]);
                    acc[i] = fma(b, b, acc[i]);
                }
            }
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) {
#pragma unroll
            for (int o = 8; o > 0; o >>= 1)
                acc[i] += __shfl_xor_sync(0xFFFFFFFFu, acc[i], o);
        }
        if (cc == 0) {
#pragma unroll
            for (int i = 0; i < 8; ++i)
                part[par][rg + 16 * i] = acc[i];
        }
        cluster_sync_all();
        float rstd[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            double tot = 0.0;
            for (uint32_t r = 0; r < kNormCluster; ++r)
                tot += ld_dsmem_f64(&part[par][rg + 16 * i], r);
            rstd[i] = static_cast<float>(1.0 / sqrt(tot / static_cast<double>(K) +
                                                    static_cast<double>(eps)));
            if (rstd_out != nullptr && rank == 0 && cc == 0)
                rstd_out[mb * 128 + rg + 16 * i] = rstd[i];
        }
        // pass 2: normalise, round to BF16, quantize each block
        for (int64_t kb = rank; kb < KB; kb += kNormCluster) {
            const int64_t off = (mb * 128 + rg) * K + kb * 128 + cc * 8;
            const uint4 gv = *reinterpret_cast<const uint4 *>(gamma + kb * 128 + cc * 8);
            const uint32_t gw[4] = {gv.x, gv.y, gv.z, gv.w};
            uint32_t w[8][4];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const uint4 v = ld_nc_v4(x + off + static_cast<int64_t>(i) * 16 * K);
                const uint32_t ww[4] = {v.x, v.y, v.z, v.w};
                const float2 r2 = make_float2(rstd[i], rstd[i]);
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const float2 xv = make_float2(bf16_lo(ww[j]), bf16_hi(ww[j]));
                    const float2 gg = make_float2(bf16_lo(gw[j]), bf16_hi(gw[j]));
                    const float2 yv = __fmul2_rn(__fmul2_rn(xv, r2), gg);
                    w[i][j] = pack_bf16x2(yv.x, yv.y);
                }
            }
            uint32_t m = 0;
#pragma unroll
            for (int i = 0; i < 8; ++i)
                m = absmax8_bits(w[i], m);
            const float sc = block_scale_from(m, red);
            const float rc = __frcp_rn(sc);
            const bool exact = !(rc <= 3.0e38f);
            if (threadIdx.x == 0)
                s[mb * KB + kb] = sc;
#pragma unroll
            for (int i = 0; i < 8; ++i)
                *reinterpret_cast<uint2 *>(q + off + static_cast<int64_t>(i) * 16 * K) =
                    quantize8(w[i], sc, rc, exact);
            __syncthreads();
        }
    }
    cluster_sync_all();   // no CTA leaves while a peer may still read its partial sums
}

} // namespace quant
} // namespace w8a8
