// quant.cuh -- block-wise 128x128 INT8 quantization of BF16 matrices (activations every
// call, weights once), and the per-row quantizer of the per-row / per-output-channel
// operator.  (RMSNorm fused ahead of the block quantizer lives in norm.cuh.)
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
//
// codes8 (used after RMSNorm, norm.cuh) trades that band for fewer instructions:
// z = fl(v * fl(1/s) + 49152.5) lies in [2^15, 2^16), where the FP32 grid is 2^-8, so byte 1
// of z's bit pattern is the low byte of floor(z - 49152), the code in two's complement, and
// byte 0 is the fraction of z on that grid.  |z - 49152.5 - fl32(v / s)| < 2^-9 + 2^-16, so
// unless the fraction byte is 0 (z within 2^-9 of an integer) floor(z - 49152) equals
// rne(fl32(v / s)).  A chunk holding such a value (about 3% of 8-value chunks) is re-coded
// with codes8_exact.  In the standalone quantizers that re-coding costs more than codes8
// saves (measured), so they keep quantize8_fast.
#pragma once

#include "common.cuh"

namespace w8a8 {
namespace quant {

constexpr float kRoundMagic = 12582912.0f;            // 1.5 * 2^23
constexpr float kTieBand = 0.5f - 1.0f / 16384.0f;     // entries with |y - rne(y)| >= this
constexpr float kCodeMagic = 49152.5f;                 // 1.5 * 2^15 + 1/2 (codes8)

// Exact code of one value: IEEE quotient by the stored scale, rint (half to even), clamp.
__device__ __forceinline__ uint32_t code_exact(float v, float sc)
{
    float q = rintf(__fdiv_rn(v, sc));
    q = fminf(fmaxf(q, -127.0f), 127.0f);
    return static_cast<uint32_t>(static_cast<int>(q)) & 0xFFu;
}

// Fast codes of 8 BF16 values (as quantize8, without the exact fallback).  Bit i of the
// returned `band` is set when value i's y lies within 2^-14 of a half-integer: its code
// must then be taken from the IEEE division (code_exact) instead.
__device__ __forceinline__ uint2 quantize8_fast(const uint32_t (&w)[4], float rc, uint32_t &band)
{
    uint32_t t[8];
    uint32_t b = 0;
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
        b |= (fabsf(d.x) >= kTieBand ? 1u : 0u) << (2 * i);
        b |= (fabsf(d.y) >= kTieBand ? 1u : 0u) << (2 * i + 1);
        t[2 * i] = __float_as_uint(tt.x);
        t[2 * i + 1] = __float_as_uint(tt.y);
    }
    band = b;
    uint2 out;
    out.x = __byte_perm(__byte_perm(t[0], t[1], 0x0040), __byte_perm(t[2], t[3], 0x0040), 0x5410);
    out.y = __byte_perm(__byte_perm(t[4], t[5], 0x0040), __byte_perm(t[6], t[7], 0x0040), 0x5410);
    return out;
}

// Codes of 8 BF16 values (4 packed words, element 2i in the low half of w[i]) as 8
// bytes, through z = fl(v * rc + 49152.5) (see above).  `tie` is set when some value's
// fraction byte is 0: the chunk must then be re-coded with codes8_exact.
__device__ __forceinline__ uint2 codes8(const uint32_t (&w)[4], float2 rc2, bool &tie)
{
    const float2 mg = make_float2(kCodeMagic, kCodeMagic);
    uint32_t pr[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 z = __ffma2_rn(make_float2(bf16_lo(w[i]), bf16_hi(w[i])), rc2, mg);
        pr[i] = __byte_perm(__float_as_uint(z.x), __float_as_uint(z.y), 0x5410);  // frac code frac code
    }
    const uint32_t fr = __vminu2(__vminu2(pr[0] & 0x00FF00FFu, pr[1] & 0x00FF00FFu),
                                 __vminu2(pr[2] & 0x00FF00FFu, pr[3] & 0x00FF00FFu));
    tie = (fr & 0xFFFFu) == 0 || (fr >> 16) == 0;
    return make_uint2(__byte_perm(pr[0], pr[1], 0x7531), __byte_perm(pr[2], pr[3], 0x7531));
}

// Exact codes of 8 BF16 values, for a chunk that codes8 flagged: quantize8_fast's
// arithmetic (a band about 30 times narrower than codes8's), and the IEEE division for
// the values inside it.
__device__ __forceinline__ uint2 codes8_exact(const uint32_t (&w)[4], float rc, float sc)
{
    const float2 r2 = make_float2(rc, rc);
    const float2 mg = make_float2(kRoundMagic, kRoundMagic);
    const float2 nmg = make_float2(-kRoundMagic, -kRoundMagic);
    const float2 neg1 = make_float2(-1.0f, -1.0f);
    uint32_t t[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 v = make_float2(bf16_lo(w[i]), bf16_hi(w[i]));
        const float2 y = __fmul2_rn(v, r2);          // ~ v / s
        const float2 tt = __fadd2_rn(y, mg);         // 1.5 * 2^23 + rne(y): low byte = code
        const float2 n = __fadd2_rn(tt, nmg);        // rne(y), exact
        const float2 d = __ffma2_rn(n, neg1, y);     // y - rne(y), exact
        t[2 * i] = fabsf(d.x) >= kTieBand ? code_exact(v.x, sc) : __float_as_uint(tt.x);
        t[2 * i + 1] = fabsf(d.y) >= kTieBand ? code_exact(v.y, sc) : __float_as_uint(tt.y);
    }
    return make_uint2(__byte_perm(__byte_perm(t[0], t[1], 0x0040), __byte_perm(t[2], t[3], 0x0040), 0x5410),
                      __byte_perm(__byte_perm(t[4], t[5], 0x0040), __byte_perm(t[6], t[7], 0x0040), 0x5410));
}

// Codes of 8 values whose 1/s overflowed (s below about 2^-128): the IEEE division for all.
__device__ __forceinline__ uint2 codes8_division(const uint32_t (&w)[4], float sc)
{
    uint32_t t[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        t[2 * i] = code_exact(bf16_lo(w[i]), sc);
        t[2 * i + 1] = code_exact(bf16_hi(w[i]), sc);
    }
    return make_uint2(__byte_perm(__byte_perm(t[0], t[1], 0x0040), __byte_perm(t[2], t[3], 0x0040), 0x5410),
                      __byte_perm(__byte_perm(t[4], t[5], 0x0040), __byte_perm(t[6], t[7], 0x0040), 0x5410));
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

// ------------------------------------------------------------------ block quantizer ----
// x [rows, K] BF16 -> q [rows, K] INT8, s [rows/128, K/128] FP32.
//
// Persistent: one CTA per SM takes the 128x128 blocks blockIdx.x + i gridDim.x,
// i = 0, 1, ..., in row-major block order.  Warp 16 (one thread) streams them into a ring
// of kQStages 32 KB shared-memory slots with 2-D TMA loads (no swizzle, no multicast),
// which keeps up to kQStages blocks per SM in flight.  The 16 consumer warps form
// kQGroups independent groups of 4; group g quantizes the CTA's blocks i = g, g + 4, ...,
// so the latency chain of one block (absmax reduction, IEEE scale division, reciprocal)
// overlaps the arithmetic of the other groups' blocks.  Within a group, thread t
// (0..127) holds the 16-byte chunks t + 128 j, j = 0..15 (rows t / 16 + 8 j, columns
// 8 (t % 16) .. + 7).  It reads them once to reduce the block's absmax (packed 16-bit
// magnitudes, warp shuffles, then the 4 warp maxima through shared memory) and once more
// to form the codes, which it writes with 8-byte stores (a warp covers two full 128-byte
// rows of codes).  Every
// wait is a bounded mbarrier wait; no named barrier is used.
constexpr int kQStages = 6;
constexpr int kQGroups = 4;                          // independent consumer groups
constexpr int kQGroupWarps = 4;                      // warps per group
constexpr int kQWarps = kQGroups * kQGroupWarps;    // consumer warps
constexpr int kQChunks = 2048 / (kQGroupWarps * 32); // 16-byte chunks per thread per block
constexpr int kQThreads = (kQWarps + 1) * 32;       // + the TMA producer warp
constexpr uint32_t kQBlockBytes = 128 * 128 * 2;

struct alignas(1024) QSmem {
    uint16_t tile[kQStages][128 * 128];
    uint64_t full[kQStages];
    uint64_t empty[kQStages];
    uint64_t red_full[kQGroups][2];
    alignas(16) uint32_t red[kQGroups][2][kQGroupWarps];
    int abort;
};
constexpr size_t kQSmemBytes = sizeof(QSmem) + 1024;
static_assert(kQGroupWarps == 4, "the group's partial maxima are read as one 16-byte vector");
static_assert(kQStages >= kQGroups, "every group needs a slot of its own");
static_assert((2 * kQStages) % kQGroups == 0,
              "item it - 2 S of the ring must belong to the same group as item it");


// What is quantized: x itself, or x normalised on the way in (RMSNorm with the rstd a
// previous grid computed, optionally followed by the scale-shift modulation; the
// arithmetic of each is spelt out in norm.cuh).
enum NormKind : int { kNone = 0, kRms = 1, kRmsMod = 2 };

struct NormArgs {
    const float *rstd;        // [rows], written by the grid this one depends on
    const uint16_t *gamma;    // [K] BF16, or null (no affine factor)
    const uint16_t *scale;    // [rows / T, K] BF16 (kRmsMod)
    const uint16_t *shift;    // [rows / T, K] BF16 (kRmsMod)
    int64_t T;                // rows sharing one modulation row; a multiple of 128
};

// Eight BF16 values (one 16-byte load) as FP32 numbers.
__device__ __forceinline__ void unpack8_f32(uint4 v, float (&f)[8])
{
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        f[2 * i] = bf16_lo(w[i]);
        f[2 * i + 1] = bf16_hi(w[i]);
    }
}

template <int kNorm>
__global__ void __launch_bounds__(kQThreads, 1)
    quantize_blocks_kernel(const __grid_constant__ CUtensorMap tmX, int64_t K, int64_t nblocks,
                           int64_t KB, int8_t *__restrict__ q, float *__restrict__ s,
                           const NormArgs na)
{
    extern __shared__ uint8_t smem_raw[];
    QSmem &sm = *reinterpret_cast<QSmem *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~static_cast<uintptr_t>(1023));
    const int warp = threadIdx.x >> 5;
    const uint32_t lane = threadIdx.x & 31;
    volatile int *abort = &sm.abort;
    if (threadIdx.x == 0) {
        for (int i = 0; i < kQStages; ++i) {
            mbar_init(&sm.full[i], 1);
            mbar_init(&sm.empty[i], kQGroupWarps);
        }
        for (int g = 0; g < kQGroups; ++g) {
            mbar_init(&sm.red_full[g][0], kQGroupWarps);
            mbar_init(&sm.red_full[g][1], kQGroupWarps);
        }
        sm.abort = 0;
        fence_barrier_init();
    }
    __syncthreads();
    // A GEMM launched after this kernel as a programmatic dependent may start now: its CTAs
    // take SMs as this kernel's CTAs leave them, set up, and wait (griddepcontrol.wait)
    // for this grid's codes and scales before reading them.
    asm volatile("griddepcontrol.launch_dependents;");

    if (warp == kQWarps) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            prefetch_tensormap(&tmX);
            uint32_t it = 0;
            bool ok = true;
            for (int64_t blk = blockIdx.x; blk < nblocks; blk += gridDim.x, ++it) {
                const uint32_t st = it % kQStages, ph = (it / kQStages) & 1;
                if (!mbar_wait(&sm.empty[st], ph ^ 1, abort)) {
                    ok = false;
                    break;
                }
                const int64_t mb = blk / KB, kb = blk - mb * KB;
                mbar_arrive_expect_tx(&sm.full[st], kQBlockBytes);
                tma_load_2d(sm.tile[st], &tmX, &sm.full[st], static_cast<int32_t>(kb * 128),
                            static_cast<int32_t>(mb * 128));
            }
            if (!ok) {
                // the copies already in flight land before shared memory is released
                volatile int no_abort = 0;
                const uint32_t first = it > kQStages ? it - kQStages : 0;
                for (uint32_t j = first; j < it; ++j)
                    mbar_wait(&sm.full[j % kQStages], (j / kQStages) & 1, &no_abort, 100000000ull);
            }
        }
        return;
    }

    // ---------------------------------------------------------------- consumers
    const int g = warp / kQGroupWarps;
    const int gw = warp % kQGroupWarps;
    const int gt = threadIdx.x % (kQGroupWarps * 32);
    const int row0 = gt >> 4;
    const int col = (gt & 15) * 8;
    constexpr int kRowStep = kQGroupWarps * 32 / 16;     // rows between a thread's chunks
    // rstd comes from the grid this one was launched after: wait for its completion
    if (kNorm != kNone)
        asm volatile("griddepcontrol.wait;" ::: "memory");
    uint32_t gi = 0;                                     // this group's block count
    for (int64_t blk = blockIdx.x + static_cast<int64_t>(g) * gridDim.x; blk < nblocks;
         blk += static_cast<int64_t>(kQGroups) * gridDim.x, ++gi) {
        const uint32_t it = gi * kQGroups + g;           // position in the ring's sequence
        const uint32_t st = it % kQStages, ph = (it / kQStages) & 1;
        // the per-row and per-column factors of the normalisation, loaded before the block
        float rs[kNorm != kNone ? kQChunks : 1], gm[8], am[8], sh[8];
        if (kNorm != kNone) {
            const int64_t mb = blk / KB, kb = blk - mb * KB;
#pragma unroll
            for (int j = 0; j < kQChunks; ++j)
                rs[j] = __ldg(na.rstd + mb * 128 + row0 + kRowStep * j);
            if (na.gamma != nullptr) {
                unpack8_f32(__ldg(reinterpret_cast<const uint4 *>(na.gamma + kb * 128 + col)), gm);
            } else {
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    gm[e] = 1.0f;
            }
            if (kNorm == kRmsMod) {
                const int64_t bm = (mb * 128) / na.T;
                unpack8_f32(__ldg(reinterpret_cast<const uint4 *>(na.scale + bm * K + kb * 128 + col)), am);
                unpack8_f32(__ldg(reinterpret_cast<const uint4 *>(na.shift + bm * K + kb * 128 + col)), sh);
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    am[e] = __fadd_rn(1.0f, am[e]);
            }
        }
        // Slot st carries items it - S, it, it + S, ... of different groups.  A parity
        // wait cannot tell phase p from p + 2, so first make sure item it - S has been
        // consumed (the slot's full barrier is then in item it's phase or just past it).
        // That wait is itself unambiguous: item it - 2S belongs to this group and is done.
        if (it >= static_cast<uint32_t>(kQStages) && !mbar_wait(&sm.empty[st], ph ^ 1, abort))
            break;
        if (!mbar_wait(&sm.full[st], ph, abort))
            break;
        uint16_t *tile = sm.tile[st];
        // pass 1 over the tile: absmax (the tile is read again for the codes, which keeps
        // the registers free while the group waits for the block's scale).  When
        // normalising, the BF16 values y are written back in place first.
        uint32_t m2 = 0;
#pragma unroll
        for (int j = 0; j < kQChunks; ++j) {
            uint16_t *chunk = tile + (row0 + kRowStep * j) * 128 + col;
            const uint4 v = ld_shared_v4(chunk);
            uint32_t w[4] = {v.x, v.y, v.z, v.w};
            if (kNorm != kNone) {
                const float2 r2 = make_float2(rs[j], rs[j]);
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    float2 n = __fmul2_rn(make_float2(bf16_lo(w[k]), bf16_hi(w[k])), r2);
                    n = __fmul2_rn(n, make_float2(gm[2 * k], gm[2 * k + 1]));
                    if (kNorm == kRmsMod) {
                        // the shift is added with the scalar __fadd_rn, which is never
                        // contracted with the product into a fused multiply-add; the
                        // definition rounds the product and the sum separately
                        n = __fmul2_rn(n, make_float2(am[2 * k], am[2 * k + 1]));
                        n.x = __fadd_rn(n.x, sh[2 * k]);
                        n.y = __fadd_rn(n.y, sh[2 * k + 1]);
                    }
                    w[k] = pack_bf16x2(n.x, n.y);
                }
                st_shared_v4(chunk, make_uint4(w[0], w[1], w[2], w[3]));
            }
            m2 = absmax8_bits(w, m2);
        }
        uint32_t m = max(m2 & 0xFFFFu, m2 >> 16);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1)
            m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
        const uint32_t rb = gi & 1;
        if (lane == 0) {
            sm.red[g][rb][gw] = m;
            mbar_arrive(&sm.red_full[g][rb]);
        }
        if (!mbar_wait(&sm.red_full[g][rb], (gi >> 1) & 1, abort))
            break;
        const uint4 r4 = ld_shared_v4(&sm.red[g][rb][0]);
        const uint32_t a = max(max(r4.x, r4.y), max(r4.z, r4.w));
        const float amax = __uint_as_float(a << 16);
        const float sc = (amax == 0.0f) ? 1.0f : __fdiv_rn(amax, 127.0f);
        const float rc = __frcp_rn(sc);
        if (gt == 0)
            s[blk] = sc;
        const int64_t mb = blk / KB, kb = blk - mb * KB;
        int8_t *qb = q + (mb * 128 + row0) * K + kb * 128 + col;
        uint32_t band[kQChunks / 4];
#pragma unroll
        for (int j = 0; j < kQChunks; ++j) {
            const uint4 v = ld_shared_v4(tile + (row0 + kRowStep * j) * 128 + col);
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
            uint32_t bj;
            *reinterpret_cast<uint2 *>(qb + static_cast<int64_t>(j) * kRowStep * K) =
                quantize8_fast(w, rc, bj);
            if ((j & 3) == 0)
                band[j >> 2] = bj;
            else
                band[j >> 2] |= bj << (8 * (j & 3));
        }
        // Values near a half-integer (about 0.3% of N(0,1) BF16 data), and every value of
        // a block whose 1/s overflows (s below about 2^-128), get their code from the
        // division.  They are re-read from the tile and patched one byte at a time after
        // the 8-byte stores above (same thread, same address: the later store wins).
        const bool all_exact = !(rc <= 3.0e38f);
#pragma unroll
        for (int k = 0; k < kQChunks / 4; ++k) {
            uint32_t b = all_exact ? 0xFFFFFFFFu : band[k];
            while (b != 0) {
                const int e = __ffs(b) - 1;
                b &= b - 1;
                const int j = 4 * k + (e >> 3);
                const int r = row0 + kRowStep * j, c = col + (e & 7);
                const float v = __uint_as_float(static_cast<uint32_t>(tile[r * 128 + c]) << 16);
                qb[static_cast<int64_t>(j) * kRowStep * K + (e & 7)] =
                    static_cast<int8_t>(code_exact(v, sc));
            }
        }
        // the normalised values this thread wrote into the slot are ordered before the
        // next TMA fill of it (a write of the async proxy)
        if (kNorm != kNone)
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        // every lane is done with the slot (its loads were consumed above)
        __syncwarp();
        if (lane == 0)
            mbar_arrive(&sm.empty[st]);
    }
}

// ------------------------------------------------------------------ per-row quantizer --
// x [rows, K] BF16 -> q [rows, K] INT8, s [rows] FP32 with s = max(||row||_inf, 1e-4) / 127
// (TurboT2VA paper, W8A8 operator paragraph: dynamic per-row activation scales, static
// per-output-channel weight scales; eps = the FP32 value nearest 1e-4).  One warp per row:
// pass 1 reads the row with 16-byte loads for its absmax (warp shuffles), pass 2 reads it
// again (now from L1 / L2) for the codes, written with 8-byte stores.  Values within 2^-14
// of a half-integer are re-coded with the IEEE division, as in quantize_blocks_kernel.
constexpr float kRowEps = 1e-4f;
constexpr int kRowWarps = 8;

__global__ void __launch_bounds__(kRowWarps * 32)
    row_quantize_kernel(const uint16_t *__restrict__ x, int64_t rows, int64_t K,
                        int8_t *__restrict__ q, float *__restrict__ s)
{
    const int lane = threadIdx.x & 31;
    const int64_t nchunks = K / 8;
    for (int64_t r = static_cast<int64_t>(blockIdx.x) * kRowWarps + (threadIdx.x >> 5); r < rows;
         r += static_cast<int64_t>(gridDim.x) * kRowWarps) {
        const uint16_t *xr = x + r * K;
        uint32_t m2 = 0;
#pragma unroll 4
        for (int64_t c = lane; c < nchunks; c += 32) {
            const uint4 v = __ldg(reinterpret_cast<const uint4 *>(xr + c * 8));
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
            m2 = absmax8_bits(w, m2);
        }
        uint32_t m = max(m2 & 0xFFFFu, m2 >> 16);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1)
            m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
        const float amax = __uint_as_float(m << 16);
        const float sc = __fdiv_rn(fmaxf(amax, kRowEps), 127.0f);
        const float rc = __frcp_rn(sc);     // sc >= 1e-4 / 127: no overflow
        if (lane == 0)
            s[r] = sc;
        int8_t *qr = q + r * K;
#pragma unroll 4
        for (int64_t c = lane; c < nchunks; c += 32) {
            const uint4 v = __ldg(reinterpret_cast<const uint4 *>(xr + c * 8));
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
            uint32_t band;
            *reinterpret_cast<uint2 *>(qr + c * 8) = quantize8_fast(w, rc, band);
            while (band != 0) {
                const int e = __ffs(band) - 1;
                band &= band - 1;
                const float v1 = __uint_as_float(static_cast<uint32_t>(xr[c * 8 + e]) << 16);
                qr[c * 8 + e] = static_cast<int8_t>(code_exact(v1, sc));
            }
        }
    }
}

} // namespace quant
} // namespace w8a8
