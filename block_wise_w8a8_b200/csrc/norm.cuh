// norm.cuh -- RMSNorm, optionally followed by the adaptive scale-shift modulation of
// diffusion transformers, fused ahead of the block-wise 128x128 activation quantizer.
//
// Operation (TurboDiffusion article, inference list item 5: norm kernels written for the
// GPU; TurboT2VA paper, fused-operator paragraph: modulated RMS normalization and scale-
// shift modulation, fused, ahead of the W8A8 linears).  For row m of x [M, K]:
//   rstd[m] = fp32( 1 / sqrt( (sum_k x[m,k]^2) / K + eps ) )      sum and sqrt in FP64
//   n       = fl(x[m,k] * rstd[m]), times gamma[k] when gamma is given (FP32 products)
//   y       = bf16(n)                                              plain RMSNorm
//   y       = bf16( fl( fl(n * fl(1 + scale[b,k])) + shift[b,k] ) ), b = m / T   modulated
// and y is block-quantized exactly as quant.cuh does (scale max|y| / 127, codes
// rne(fl32(y / s)) clamped to +-127), without being written out.
//
// Work split.  A cluster of C <= 8 CTAs owns one 128-row strip at a time; CTA r handles
// the strip's 128-column blocks kb = r, r + C, ...  (nb of them).  Each CTA streams its
// blocks into a ring of six 32 KB shared-memory slots with 2-D TMA loads (two 64-column
// boxes per block, 128-byte swizzle, no multicast).  When nb <= 6 the blocks stay in
// their slots from the first pass to the second ("resident"), so x is read from HBM once;
// otherwise every block is loaded twice (the second load normally hits L2).
//
//   pass 1   each thread owns one row of a block and sums its squares in FP64.  The FP64
//            operand is built from the BF16 bits with two integer operations, as |x| *
//            2^-128 (exponent field 0x300 | e, so that every square stays a normal FP64
//            number); the exact sum is the accumulated one times 2^256.  Zero and
//            subnormal inputs come out as tiny non-zero values this way (at most 2^-252
//            per element after rescaling), far below one FP64 ulp of eps for any eps > 0;
//            a separate instantiation converts exactly and runs when eps == 0.
//   exchange the four consumer groups' row partials are added in a fixed order, and the
//            CTA's partial of each row is pushed into every CTA of the cluster with
//            st.async (completion counted in bytes on the receiver's mbarrier), so every
//            CTA adds the same C partials in rank order and derives the same rstd.
//   pass 2   per block, thread t of a group holds rows t/16 + 8 j (j = 0..15), columns
//            8 (t % 16) .. +7.  2a normalises (and modulates), rounds to BF16, writes the
//            values back into the slot and reduces the block's absmax; 2b forms the codes
//            and stores them with 8-byte stores (a warp covers two full 128-byte rows).
//
// Codes.  z = fl(y * fl(1/s) + 49152.5) lies in [2^15, 2^16), where the FP32 grid is
// 2^-8, so byte 1 of z's bit pattern is the low byte of floor(z - 49152) = the code
// (two's complement) and byte 0 is the fraction of z on that grid.  |z - 49152.5 -
// fl32(y / s)| < 2^-9 + 2^-16, so unless the fraction byte is 0 (z within 2^-9 of an
// integer, i.e. y / s near a half-integer) floor(z - 49152) = rne(fl32(y / s)).  Entries
// with fraction byte 0 (about 0.4%), and all entries of a block whose 1/s overflows, are
// recomputed with the IEEE division, so the codes equal those of the definition bit for
// bit.  The clamp cannot fire on the fast path (|y / s| <= 127 (1 + 2^-22)).
//
// Every wait is a bounded mbarrier wait.  The kernel's only unbounded waits are the two
// cluster barriers at its start and end, which every thread reaches after finitely many
// bounded steps.
#pragma once

#include "common.cuh"
#include "quant.cuh"

namespace w8a8 {
namespace norm {

constexpr int kStages = 6;
constexpr int kGroups = 4;
constexpr int kGroupWarps = 4;
constexpr int kWarps = kGroups * kGroupWarps;   // consumer warps
constexpr int kThreads = (kWarps + 1) * 32;     // + the TMA producer warp
constexpr int kMaxCluster = 8;
constexpr uint32_t kBlockBytes = 128 * 128 * 2;
constexpr float kCodeMagic = 49152.5f;          // 1.5 * 2^15 + 1/2
constexpr double kTwo256 = 1.157920892373162e77; // 2^256, exact

struct alignas(1024) Smem {
    uint16_t tile[kStages][128 * 128];         // two [128][64] boxes, 128-byte swizzle
    double part[2][kMaxCluster][128];          // [strip parity][source rank][row]
    double gpart[2][kGroups][128];             // [strip parity][group][row]
    float rstd[kGroups][128];                  // each group's copy of the strip's rstd
    uint64_t full[kStages];
    uint64_t empty[kStages];
    uint64_t red_full[kGroups][2];
    uint64_t pdone[2];                         // all consumer warps wrote gpart
    uint64_t xready[2];                        // all C partials of every row arrived
    uint64_t rready[kGroups];                  // the group's rstd copy is written
    alignas(16) uint32_t red[kGroups][2][kGroupWarps];
    int abort;
};
constexpr size_t kSmemBytes = sizeof(Smem) + 1024;
static_assert(kSmemBytes <= 232448, "exceeds the 227 KB of shared memory a CTA may use");
static_assert(kStages >= kGroups && (2 * kStages) % kGroups == 0,
              "ring item it - 2 S must belong to the same group as item it");

// Element offset of the 16-byte chunk `c` (0..15, eight BF16 values) of `row` in a slot:
// box c / 8, chunk c % 8 of the row's 128 bytes, XOR-swizzled with row % 8.
__device__ __forceinline__ uint32_t chunk_off(int row, int c)
{
    return static_cast<uint32_t>((c >> 3) * (128 * 64) + row * 64 + (((c & 7) ^ (row & 7)) << 3));
}

__device__ __forceinline__ uint32_t cluster_rank()
{
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

__device__ __forceinline__ uint32_t cluster_size()
{
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(r));
    return r;
}

__device__ __forceinline__ void cluster_barrier()
{
    asm volatile("barrier.cluster.arrive.release.aligned;\n\t"
                 "barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

__device__ __forceinline__ uint32_t map_to_rank(const void *p, uint32_t rank)
{
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_u32(p)), "r"(rank));
    return r;
}

// 8-byte store into another CTA's shared memory, its completion counted in bytes on that
// CTA's mbarrier (both addresses already mapped with mapa).
__device__ __forceinline__ void st_async_b64(uint32_t remote, uint64_t v, uint32_t remote_bar)
{
    asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.b64 [%0], %1, [%2];" ::"r"(remote),
                 "l"(v), "r"(remote_bar)
                 : "memory");
}

// |x| * 2^-128 as an FP64 high word, for the BF16 value in the low / high half of w
// (exponent field 0x300 | e, the 7 mantissa bits on top of the FP64 mantissa).
__device__ __forceinline__ double scaled_lo(uint32_t w)
{
    return __hiloint2double(static_cast<int>(((w << 13) & 0x0FFFE000u) | 0x30000000u), 0);
}
__device__ __forceinline__ double scaled_hi(uint32_t w)
{
    return __hiloint2double(static_cast<int>(((w >> 3) & 0x0FFFE000u) | 0x30000000u), 0);
}

struct Params {
    const uint16_t *gamma;    // [K] BF16, or null (no affine factor)
    const uint16_t *scale;    // [M / T, K] BF16 (modulated kernel only)
    const uint16_t *shift;    // [M / T, K] BF16 (modulated kernel only)
    int64_t T;                // rows sharing one modulation row; a multiple of 128
    float eps;
    int64_t MB, K;            // M / 128 strips, K columns
    int8_t *q;                // [M, K]
    float *s;                 // [M / 128, K / 128]
    float *rstd_out;          // [M] or null
};

// Eight BF16 values (four packed words) as FP32 factors.
__device__ __forceinline__ void unpack8(uint4 v, float (&f)[8])
{
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        f[2 * i] = bf16_lo(w[i]);
        f[2 * i + 1] = bf16_hi(w[i]);
    }
}

template <bool kMod, bool kExactSq>
__global__ void __launch_bounds__(kThreads, 1)
    rmsnorm_quantize_kernel(const __grid_constant__ CUtensorMap tmX, const Params p)
{
    extern __shared__ uint8_t smem_raw[];
    Smem &sm = *reinterpret_cast<Smem *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                         ~static_cast<uintptr_t>(1023));
    const int warp = threadIdx.x >> 5;
    const uint32_t lane = threadIdx.x & 31;
    const uint32_t rank = cluster_rank();
    const uint32_t C = cluster_size();
    const int64_t cluster = blockIdx.x / C;
    const int64_t nclusters = gridDim.x / C;
    const int64_t K = p.K;
    const int64_t KB = K / 128;
    const int nb = KB > static_cast<int64_t>(rank) ? static_cast<int>((KB - 1 - rank) / C + 1) : 0;
    const bool resident = nb <= kStages;
    const int per_strip = resident ? nb : 2 * nb;
    volatile int *abort = &sm.abort;
    if (threadIdx.x == 0) {
        for (int i = 0; i < kStages; ++i) {
            mbar_init(&sm.full[i], 1);
            mbar_init(&sm.empty[i], kGroupWarps);
        }
        for (int g = 0; g < kGroups; ++g) {
            mbar_init(&sm.red_full[g][0], kGroupWarps);
            mbar_init(&sm.red_full[g][1], kGroupWarps);
            mbar_init(&sm.rready[g], kGroupWarps);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&sm.pdone[i], kWarps);
            mbar_init(&sm.xready[i], 1);
        }
        sm.abort = 0;
        fence_barrier_init();
    }
    __syncthreads();
    cluster_barrier();      // every CTA's barriers are initialised before anything is sent

    if (warp == kWarps) {
        // ------------------------------------------------------------ TMA producer
        // Items in load order: per strip, the CTA's nb blocks (resident), or its nb blocks
        // for pass 1 followed by the same nb blocks again for pass 2.
        if (lane == 0 && nb > 0) {
            prefetch_tensormap(&tmX);
            uint32_t it = 0;
            bool ok = true;
            for (int64_t mb = cluster; ok && mb < p.MB; mb += nclusters) {
                for (int i = 0; i < per_strip; ++i, ++it) {
                    const uint32_t st = it % kStages, ph = (it / kStages) & 1;
                    if (!mbar_wait(&sm.empty[st], ph ^ 1, abort)) {
                        ok = false;
                        break;
                    }
                    const int64_t kb = rank + static_cast<int64_t>(i < nb ? i : i - nb) * C;
                    mbar_arrive_expect_tx(&sm.full[st], kBlockBytes);
                    tma_load_2d(sm.tile[st], &tmX, &sm.full[st], static_cast<int32_t>(kb * 128),
                                static_cast<int32_t>(mb * 128));
                    tma_load_2d(sm.tile[st] + 128 * 64, &tmX, &sm.full[st],
                                static_cast<int32_t>(kb * 128 + 64), static_cast<int32_t>(mb * 128));
                }
            }
            if (!ok) {
                // the copies already in flight land before shared memory is released
                volatile int no_abort = 0;
                const uint32_t first = it > kStages ? it - kStages : 0;
                for (uint32_t j = first; j < it; ++j)
                    mbar_wait(&sm.full[j % kStages], (j / kStages) & 1, &no_abort, 100000000ull);
            }
        }
        __syncwarp();
        cluster_barrier();
        return;
    }

    // ---------------------------------------------------------------- consumers
    // Group g takes the strip's ring items it with it % 4 == g, in both passes.
    const int g = warp / kGroupWarps;
    const int gw = warp % kGroupWarps;
    const int gt = threadIdx.x % (kGroupWarps * 32);
    const int row0 = gt >> 4;              // pass 2: rows row0 + 8 j
    const int cc = gt & 15;                // pass 2: columns 8 cc .. 8 cc + 7
    const uint32_t o2 = static_cast<uint32_t>((cc >> 3) * (128 * 64) + row0 * 64 + (((cc & 7) ^ row0) << 3));
    uint32_t base = 0;                     // ring items before this strip
    uint32_t gi = 0;                       // this group's pass-2 blocks so far
    bool dead = false;
    int64_t sidx = 0;
    for (int64_t mb = cluster; mb < p.MB; mb += nclusters, ++sidx, base += per_strip) {
        const uint32_t sp = static_cast<uint32_t>(sidx & 1);
        if (threadIdx.x == 0)
            mbar_arrive_expect_tx(&sm.xready[sp], C * 128 * 8);

        // pass 1: sum of squares of row gt over the group's blocks, four FP64 chains
        double a0 = 0.0, a1 = 0.0, a2 = 0.0, a3 = 0.0;
        const int i0 = (g - static_cast<int>(base & 3) + 4) & 3;
        for (int i = i0; i < nb; i += kGroups) {
            const uint32_t it = base + i;
            const uint32_t st = it % kStages, ph = (it / kStages) & 1;
            // Slot st held item it - S before (another group's, possibly still in use):
            // wait for its release first, so that the parity wait on full cannot match an
            // older phase.  Item it - 2 S is known to be released (see the static_assert).
            bool ok = it < static_cast<uint32_t>(kStages) || mbar_wait(&sm.empty[st], ph ^ 1, abort);
            ok = ok && mbar_wait(&sm.full[st], ph, abort);
            if (__any_sync(0xFFFFFFFFu, !ok)) {
                dead = true;
                break;
            }
            const uint16_t *tile = sm.tile[st];
#pragma unroll
            for (int c = 0; c < 16; ++c) {
                const uint4 v = ld_shared_v4(tile + chunk_off(gt, c));
                double d[8];
                if (kExactSq) {
                    d[0] = bf16_lo(v.x); d[1] = bf16_hi(v.x); d[2] = bf16_lo(v.y); d[3] = bf16_hi(v.y);
                    d[4] = bf16_lo(v.z); d[5] = bf16_hi(v.z); d[6] = bf16_lo(v.w); d[7] = bf16_hi(v.w);
                } else {
                    d[0] = scaled_lo(v.x); d[1] = scaled_hi(v.x); d[2] = scaled_lo(v.y); d[3] = scaled_hi(v.y);
                    d[4] = scaled_lo(v.z); d[5] = scaled_hi(v.z); d[6] = scaled_lo(v.w); d[7] = scaled_hi(v.w);
                }
                a0 = fma(d[0], d[0], a0);
                a1 = fma(d[1], d[1], a1);
                a2 = fma(d[2], d[2], a2);
                a3 = fma(d[3], d[3], a3);
                a0 = fma(d[4], d[4], a0);
                a1 = fma(d[5], d[5], a1);
                a2 = fma(d[6], d[6], a2);
                a3 = fma(d[7], d[7], a3);
            }
            if (!resident) {
                // the sums depend on every value read: the slot is free again
                __syncwarp();
                if (lane == 0)
                    mbar_arrive(&sm.empty[st]);
            }
        }
        if (dead)
            break;

        // exchange: the CTA's partial of row gt (groups in order) to every CTA of the
        // cluster; group g sends to ranks g, g + 4
        sm.gpart[sp][g][gt] = (a0 + a1) + (a2 + a3);
        __syncwarp();
        if (lane == 0)
            mbar_arrive(&sm.pdone[sp]);
        bool ok = mbar_wait(&sm.pdone[sp], static_cast<uint32_t>(sidx >> 1) & 1, abort);
        if (__any_sync(0xFFFFFFFFu, !ok)) {
            dead = true;
            break;
        }
        const double cp = ((sm.gpart[sp][0][gt] + sm.gpart[sp][1][gt]) + sm.gpart[sp][2][gt]) +
                          sm.gpart[sp][3][gt];
        for (uint32_t c = static_cast<uint32_t>(g); c < C; c += kGroups)
            st_async_b64(map_to_rank(&sm.part[sp][rank][gt], c),
                         static_cast<uint64_t>(__double_as_longlong(cp)), map_to_rank(&sm.xready[sp], c));
        ok = mbar_wait(&sm.xready[sp], static_cast<uint32_t>(sidx >> 1) & 1, abort);
        if (__any_sync(0xFFFFFFFFu, !ok)) {
            dead = true;
            break;
        }
        double tot = sm.part[sp][0][gt];
        for (uint32_t c = 1; c < C; ++c)
            tot += sm.part[sp][c][gt];
        const double ss = kExactSq ? tot : tot * kTwo256;
        const float r = static_cast<float>(1.0 / sqrt(ss / static_cast<double>(K) + static_cast<double>(p.eps)));
        sm.rstd[g][gt] = r;
        if (p.rstd_out != nullptr && rank == 0 && g == 0)
            p.rstd_out[mb * 128 + gt] = r;
        __syncwarp();
        if (lane == 0)
            mbar_arrive(&sm.rready[g]);
        ok = mbar_wait(&sm.rready[g], static_cast<uint32_t>(sidx & 1), abort);
        if (__any_sync(0xFFFFFFFFu, !ok)) {
            dead = true;
            break;
        }
        float rs[16];
#pragma unroll
        for (int j = 0; j < 16; ++j)
            rs[j] = sm.rstd[g][row0 + 8 * j];
        const int64_t bm = kMod ? (mb * 128) / p.T : 0;     // the strip's modulation row

        // pass 2: normalise (modulate), round to BF16, quantize each of the group's blocks
        const int first = resident ? i0 : nb + ((g - static_cast<int>((base + nb) & 3) + 4) & 3);
        const int last = resident ? nb : 2 * nb;
        for (int i = first; i < last; i += kGroups, ++gi) {
            const int j = resident ? i : i - nb;
            const uint32_t it = base + i;
            const uint32_t st = it % kStages, ph = (it / kStages) & 1;
            if (!resident) {
                bool ok2 = it < static_cast<uint32_t>(kStages) || mbar_wait(&sm.empty[st], ph ^ 1, abort);
                ok2 = ok2 && mbar_wait(&sm.full[st], ph, abort);
                if (__any_sync(0xFFFFFFFFu, !ok2)) {
                    dead = true;
                    break;
                }
            }
            const int64_t kb = rank + static_cast<int64_t>(j) * C;
            const int64_t col = kb * 128 + cc * 8;
            float gm[8], am[8], sh[8];
            if (p.gamma != nullptr) {
                unpack8(__ldg(reinterpret_cast<const uint4 *>(p.gamma + col)), gm);
            } else {
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    gm[e] = 1.0f;
            }
            if (kMod) {
                unpack8(__ldg(reinterpret_cast<const uint4 *>(p.scale + bm * K + col)), am);
                unpack8(__ldg(reinterpret_cast<const uint4 *>(p.shift + bm * K + col)), sh);
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    am[e] = __fadd_rn(1.0f, am[e]);
            }
            uint16_t *tile = sm.tile[st] + o2;

            // 2a: y = bf16(...) written back in place; the block's absmax
            uint32_t m2 = 0;
#pragma unroll
            for (int jj = 0; jj < 16; ++jj) {
                const uint4 v = ld_shared_v4(tile + jj * 512);
                const uint32_t w[4] = {v.x, v.y, v.z, v.w};
                uint32_t o[4];
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    float n0 = __fmul_rn(__fmul_rn(bf16_lo(w[k]), rs[jj]), gm[2 * k]);
                    float n1 = __fmul_rn(__fmul_rn(bf16_hi(w[k]), rs[jj]), gm[2 * k + 1]);
                    if (kMod) {
                        n0 = __fadd_rn(__fmul_rn(n0, am[2 * k]), sh[2 * k]);
                        n1 = __fadd_rn(__fmul_rn(n1, am[2 * k + 1]), sh[2 * k + 1]);
                    }
                    o[k] = pack_bf16x2(n0, n1);
                }
                st_shared_v4(tile + jj * 512, make_uint4(o[0], o[1], o[2], o[3]));
                m2 = quant::absmax8_bits(o, m2);
            }
            uint32_t m = max(m2 & 0xFFFFu, m2 >> 16);
#pragma unroll
            for (int off = 16; off > 0; off >>= 1)
                m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, off));
            const uint32_t rb = gi & 1;
            if (lane == 0) {
                sm.red[g][rb][gw] = m;
                mbar_arrive(&sm.red_full[g][rb]);
            }
            const bool ok3 = mbar_wait(&sm.red_full[g][rb], (gi >> 1) & 1, abort);
            if (__any_sync(0xFFFFFFFFu, !ok3)) {
                dead = true;
                break;
            }
            const uint4 r4 = ld_shared_v4(&sm.red[g][rb][0]);
            const uint32_t a = max(max(r4.x, r4.y), max(r4.z, r4.w));
            const float amax = __uint_as_float(a << 16);
            const float sc = (amax == 0.0f) ? 1.0f : __fdiv_rn(amax, 127.0f);
            const float rc = __frcp_rn(sc);
            if (gt == 0)
                p.s[mb * KB + kb] = sc;

            // 2b: codes from z = y * (1/s) + 49152.5 (byte 1), fraction byte 0 flags a tie
            int8_t *qb = p.q + (mb * 128 + row0) * K + col;
            uint32_t flagged = 0;
#pragma unroll
            for (int jj = 0; jj < 16; ++jj) {
                const uint4 v = ld_shared_v4(tile + jj * 512);
                const uint32_t w[4] = {v.x, v.y, v.z, v.w};
                uint32_t pr[4];
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const uint32_t t0 = __float_as_uint(__fmaf_rn(bf16_lo(w[k]), rc, kCodeMagic));
                    const uint32_t t1 = __float_as_uint(__fmaf_rn(bf16_hi(w[k]), rc, kCodeMagic));
                    pr[k] = __byte_perm(t0, t1, 0x5410);      // frac0 code0 frac1 code1
                }
                *reinterpret_cast<uint2 *>(qb + static_cast<int64_t>(jj) * 8 * K) =
                    make_uint2(__byte_perm(pr[0], pr[1], 0x7531), __byte_perm(pr[2], pr[3], 0x7531));
                const uint32_t fr = __vminu2(__vminu2(pr[0] & 0x00FF00FFu, pr[1] & 0x00FF00FFu),
                                             __vminu2(pr[2] & 0x00FF00FFu, pr[3] & 0x00FF00FFu));
                flagged |= ((fr & 0xFFFFu) == 0 || (fr >> 16) == 0) ? (1u << jj) : 0u;
            }
            // Entries whose fraction byte is 0, and every entry of a block whose 1/s
            // overflows (s below about 2^-128), take their code from the IEEE division;
            // the byte stores land after the 8-byte stores above (same thread, same address).
            const bool all_exact = !(rc <= 3.0e38f);
            if (all_exact)
                flagged = 0xFFFFu;
            while (flagged != 0) {
                const int jj = __ffs(flagged) - 1;
                flagged &= flagged - 1;
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const float y = __uint_as_float(static_cast<uint32_t>(tile[jj * 512 + e]) << 16);
                    const uint32_t t = __float_as_uint(__fmaf_rn(y, rc, kCodeMagic));
                    if (all_exact || (t & 0xFFu) == 0)
                        qb[static_cast<int64_t>(jj) * 8 * K + e] = static_cast<int8_t>(quant::code_exact(y, sc));
                }
            }
            // every lane is done with the slot
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&sm.empty[st]);
        }
        if (dead)
            break;
    }
    __syncwarp();
    cluster_barrier();      // no CTA leaves while a peer may still send to it
}

} // namespace norm
} // namespace w8a8
