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
// Two forms.  rmsnorm_quantize_kernel below does all of it in one grid, each row's sum of
// squares split across a cluster; row_rstd_kernel (end of this file) computes rstd alone,
// one sequential FP64 chain per row, for quant::quantize_blocks_kernel<kRms / kRmsMod>
// to normalise on load.  The library takes the second form from 192 rows per SM on, where
// the row chains keep HBM busy (at M = 32768, K = 4096: 122 against 146 us).
//
// Work split of the one-grid form.  A cluster of C = min(kMaxCluster, K / 128) CTAs
// (kMaxCluster = 4) owns one 128-row strip at a time; CTA r handles the strip's 128-column
// blocks kb = r, r + C, ... (nb of them).  Each CTA streams its blocks into a ring of six
// 32 KB shared-memory slots with 2-D TMA loads (two 64-column boxes per block, 128-byte
// swizzle, no multicast), each block twice: once for the sums of squares and once for the
// codes.  The second load comes about one strip later and is meant to be served by L2 (a
// cluster has about two 1 MB strips in flight); at 32768 x 4096 about two thirds of those
// loads miss it.
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
// Pipelining.  Pass 1 runs one strip ahead of pass 2: the ring carries pass 1 of strip 0,
// then, for each strip s, pass 1 of strip s + 1 followed by pass 2 of strip s.  The
// exchange of strip s + 1 is sent while pass 2 of strip s runs and is awaited only after
// pass 1 of strip s + 2, so its latency is hidden.  The exchange buffers (the CTA's group
// partials, the C received partials, each group's rstd copy) are double-buffered by strip
// parity; a CTA sends the partials of strip s + 1 only after all of its warps have read
// those of strip s, which is what makes two buffers enough.
//
// Codes as in quant.cuh (quant::codes8): one FFMA onto the 2^-8 grid above 49152.5, the
// code in byte 1, and the 0.4% of values whose fraction byte flags a possible tie
// recomputed with the IEEE division, so the codes equal the definition's bit for bit.
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
#ifndef W8A8_NORM_CLUSTER
#define W8A8_NORM_CLUSTER 4
#endif
// CTAs per cluster (per strip).  Four: 37 clusters of one CTA per SM cover all 148 SMs of
// a B200 (clusters of eight fit only 15 times), and each CTA gets K / 512 blocks a strip.
constexpr int kMaxCluster = W8A8_NORM_CLUSTER;
constexpr uint32_t kBlockBytes = 128 * 128 * 2;
constexpr double kTwo256 = 1.157920892373162e77; // 2^256, exact

struct alignas(1024) Smem {
    uint16_t tile[kStages][128 * 128];         // two [128][64] boxes, 128-byte swizzle
    double part[2][kMaxCluster][128];          // [strip parity][source rank][row]
    double gpart[2][kGroups][128];             // [strip parity][group][row]
    float rstd[2][128];                        // [strip parity][row]
    uint64_t full[kStages];
    uint64_t empty[kStages];
    uint64_t red_full[kGroups][2];
    uint64_t pdone[2];                         // all consumer warps wrote gpart
    uint64_t xready[2];                        // all C partials of every row arrived
    uint64_t rready;                           // the strip's rstd is written (all warps)
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
    // strips this cluster handles: mb = cluster + s * nclusters, s = 0 .. ns - 1
    const int64_t ns = cluster < p.MB ? (p.MB - 1 - cluster) / nclusters + 1 : 0;
    volatile int *abort = &sm.abort;
    if (threadIdx.x == 0) {
        for (int i = 0; i < kStages; ++i) {
            mbar_init(&sm.full[i], 1);
            mbar_init(&sm.empty[i], kGroupWarps);
        }
        for (int g = 0; g < kGroups; ++g) {
            mbar_init(&sm.red_full[g][0], kGroupWarps);
            mbar_init(&sm.red_full[g][1], kGroupWarps);
        }
        mbar_init(&sm.rready, kWarps);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&sm.pdone[i], kWarps);
            mbar_init(&sm.xready[i], 1);
        }
        sm.abort = 0;
        fence_barrier_init();
        // expect the partials of the first two strips (the sends may arrive first)
        for (int64_t s = 0; s < 2 && s < ns; ++s)
            mbar_arrive_expect_tx(&sm.xready[s], C * 128 * 8);
    }
    __syncthreads();
    cluster_barrier();      // every CTA's barriers are initialised before anything is sent

    if (warp == kWarps) {
        // ------------------------------------------------------------ TMA producer
        // Items in load order: pass 1 of strip 0, then for each strip s pass 1 of strip
        // s + 1 (if any) and pass 2 of strip s; each pass is the CTA's nb blocks in order.
        if (lane == 0 && nb > 0) {
            prefetch_tensormap(&tmX);
            uint32_t it = 0;
            bool ok = true;
            for (int64_t q = 0; ok && q <= 2 * ns; ++q) {
                // q = 0: pass 1 of strip 0; odd q = 2 k - 1: pass 1 of strip k (there is
                // none for k = ns); even q = 2 k: pass 2 of strip k - 1
                const int64_t s = q == 0 ? 0 : ((q & 1) ? (q + 1) / 2 : q / 2 - 1);
                if (s >= ns)
                    continue;
                const int64_t mb = cluster + s * nclusters;
                for (int j = 0; j < nb; ++j, ++it) {
                    const uint32_t st = it % kStages, ph = (it / kStages) & 1;
                    if (!mbar_wait(&sm.empty[st], ph ^ 1, abort)) {
                        ok = false;
                        break;
                    }
                    const int64_t kb = rank + static_cast<int64_t>(j) * C;
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
    // Group g takes the ring items it with it % 4 == g, in both passes.
    const int g = warp / kGroupWarps;
    const int gw = warp % kGroupWarps;
    const int gt = threadIdx.x % (kGroupWarps * 32);
    const int row0 = gt >> 4;              // pass 2: rows row0 + 8 j
    const int cc = gt & 15;                // pass 2: columns 8 cc .. 8 cc + 7
    const uint32_t o2 = static_cast<uint32_t>((cc >> 3) * (128 * 64) + row0 * 64 + (((cc & 7) ^ row0) << 3));
    uint32_t it_next = 0;                  // ring position of the next pass
    uint32_t gi = 0;                       // this group's pass-2 blocks so far
    bool dead = false;

    // Waits for ring item it (after its slot's previous item, it - 6, has been released:
    // a parity wait on full could otherwise match that older phase; item it - 12 belongs
    // to this group and is released already, see the static_assert).
    auto wait_item = [&](uint32_t it) -> bool {
        const uint32_t st = it % kStages, ph = (it / kStages) & 1;
        bool ok = it < static_cast<uint32_t>(kStages) || mbar_wait(&sm.empty[st], ph ^ 1, abort);
        ok = ok && mbar_wait(&sm.full[st], ph, abort);
        return !__any_sync(0xFFFFFFFFu, !ok);
    };

    // Pass 1 of a strip: row gt's sum of squares over the group's blocks; writes the
    // group's partial into gpart[sp].  Four FP64 chains, added in a fixed order.
    auto pass1 = [&](uint32_t sp) -> bool {
        const uint32_t base = it_next;
        it_next += nb;
        double a0 = 0.0, a1 = 0.0, a2 = 0.0, a3 = 0.0;
        for (int i = (g - static_cast<int>(base & 3) + 4) & 3; i < nb; i += kGroups) {
            const uint32_t it = base + i;
            if (!wait_item(it))
                return false;
            const uint16_t *tile = sm.tile[it % kStages];
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
            // the sums depend on every value read: the slot is free again
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&sm.empty[it % kStages]);
        }
        sm.gpart[sp][g][gt] = (a0 + a1) + (a2 + a3);
        return true;
    };

    // The CTA's partial of row gt for the strip of parity sp, sent to every CTA of the
    // cluster; group g serves ranks g, g + 4.
    auto send = [&](uint32_t sp) {
        const double cp = ((sm.gpart[sp][0][gt] + sm.gpart[sp][1][gt]) + sm.gpart[sp][2][gt]) +
                          sm.gpart[sp][3][gt];
        for (uint32_t c = static_cast<uint32_t>(g); c < C; c += kGroups)
            st_async_b64(map_to_rank(&sm.part[sp][rank][gt], c),
                         static_cast<uint64_t>(__double_as_longlong(cp)), map_to_rank(&sm.xready[sp], c));
    };

    // pass 1 of strip 0 and its exchange
    if (ns > 0) {
        bool ok = pass1(0);
        __syncwarp();
        if (ok && lane == 0)
            mbar_arrive(&sm.pdone[0]);
        ok = ok && mbar_wait(&sm.pdone[0], 0, abort);
        if (__any_sync(0xFFFFFFFFu, !ok))
            dead = true;
        else
            send(0);
    }
    for (int64_t s = 0; s < ns && !dead; ++s) {
        const int64_t mb = cluster + s * nclusters;
        const uint32_t sp = static_cast<uint32_t>(s & 1);
        const bool more = s + 1 < ns;
        // pass 1 of the next strip
        if (more && !pass1(sp ^ 1)) {
            dead = true;
            break;
        }
        // this strip's rstd, once per row: warp 0 of group g takes rows 32 g .. 32 g + 31,
        // adding the row's C partials in rank order
        if (gw == 0) {
            const bool okx = mbar_wait(&sm.xready[sp], static_cast<uint32_t>(s >> 1) & 1, abort);
            if (__any_sync(0xFFFFFFFFu, !okx)) {
                dead = true;
                break;
            }
            const int r = 32 * g + static_cast<int>(lane);
            double tot = sm.part[sp][0][r];
            for (uint32_t c = 1; c < C; ++c)
                tot += sm.part[sp][c][r];
            const double ss = kExactSq ? tot : tot * kTwo256;
            const float rv = static_cast<float>(1.0 / sqrt(ss / static_cast<double>(K) + static_cast<double>(p.eps)));
            sm.rstd[sp][r] = rv;
            if (p.rstd_out != nullptr && rank == 0)
                p.rstd_out[mb * 128 + r] = rv;
            if (threadIdx.x == 0 && s + 2 < ns)
                mbar_arrive_expect_tx(&sm.xready[sp], C * 128 * 8);
        }
        // pdone of the next strip: its group partials are written and this strip's
        // received partials have been read (so the next sends may overwrite them)
        __syncwarp();
        if (lane == 0) {
            if (more)
                mbar_arrive(&sm.pdone[sp ^ 1]);
            mbar_arrive(&sm.rready);
        }
        bool ok = mbar_wait(&sm.rready, sp, abort);
        if (__any_sync(0xFFFFFFFFu, !ok)) {
            dead = true;
            break;
        }
        float rs[16];
#pragma unroll
        for (int j = 0; j < 16; ++j)
            rs[j] = sm.rstd[sp][row0 + 8 * j];
        if (more) {
            ok = mbar_wait(&sm.pdone[sp ^ 1], static_cast<uint32_t>((s + 1) >> 1) & 1, abort);
            if (__any_sync(0xFFFFFFFFu, !ok)) {
                dead = true;
                break;
            }
            send(sp ^ 1);
        }

        // pass 2: normalise (modulate), round to BF16, quantize each of the group's blocks
        const int64_t bm = kMod ? (mb * 128) / p.T : 0;     // the strip's modulation row
        const uint32_t base = it_next;
        it_next += nb;
        for (int i = (g - static_cast<int>(base & 3) + 4) & 3; i < nb; i += kGroups, ++gi) {
            const uint32_t it = base + i;
            const int64_t kb = rank + static_cast<int64_t>(i) * C;
            const int64_t col = kb * 128 + cc * 8;
            // the per-column factors are loaded before the wait for the block
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
            if (!wait_item(it)) {
                dead = true;
                break;
            }
            uint16_t *tile = sm.tile[it % kStages] + o2;

            // 2a: y = bf16(...) written back in place; the block's absmax
            uint32_t m2 = 0;
#pragma unroll
            for (int jj = 0; jj < 16; ++jj) {
                const uint4 v = ld_shared_v4(tile + jj * 512);
                const uint32_t w[4] = {v.x, v.y, v.z, v.w};
                uint32_t o[4];
                const float2 r2 = make_float2(rs[jj], rs[jj]);
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    float2 n = __fmul2_rn(make_float2(bf16_lo(w[k]), bf16_hi(w[k])), r2);
                    n = __fmul2_rn(n, make_float2(gm[2 * k], gm[2 * k + 1]));
                    if (kMod) {
                        // the shift is added with the scalar __fadd_rn, which is never
                        // contracted with the product into a fused multiply-add (the
                        // packed add gives no such guarantee); the definition rounds twice
                        n = __fmul2_rn(n, make_float2(am[2 * k], am[2 * k + 1]));
                        n.x = __fadd_rn(n.x, sh[2 * k]);
                        n.y = __fadd_rn(n.y, sh[2 * k + 1]);
                    }
                    o[k] = pack_bf16x2(n.x, n.y);
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

            // 2b: the codes (quant::codes8: z = y * (1/s) + 49152.5), ties re-done exactly
            int8_t *qb = p.q + (mb * 128 + row0) * K + col;
            const float2 rc2 = make_float2(rc, rc);
            uint32_t flagged = 0;
#pragma unroll
            for (int jj = 0; jj < 16; ++jj) {
                const uint4 v = ld_shared_v4(tile + jj * 512);
                const uint32_t w[4] = {v.x, v.y, v.z, v.w};
                bool tie;
                // streaming store: the codes are not read again by this kernel
                __stcs(reinterpret_cast<uint2 *>(qb + static_cast<int64_t>(jj) * 8 * K), quant::codes8(w, rc2, tie));
                flagged |= tie ? (1u << jj) : 0u;
            }
            // Chunks with a value near a half-integer are re-coded exactly, every chunk of a
            // block whose 1/s overflows (s below about 2^-128) by division; the later
            // 8-byte store to the same address, by the same thread, wins.
            const bool all_exact = !(rc <= 3.0e38f);
            if (all_exact)
                flagged = 0xFFFFu;
            while (flagged != 0) {
                const int jj = __ffs(flagged) - 1;
                flagged &= flagged - 1;
                const uint4 v = ld_shared_v4(tile + jj * 512);
                const uint32_t w[4] = {v.x, v.y, v.z, v.w};
                __stcs(reinterpret_cast<uint2 *>(qb + static_cast<int64_t>(jj) * 8 * K),
                       all_exact ? quant::codes8_division(w, sc) : quant::codes8_exact(w, rc, sc));
            }
            // every lane is done with the slot
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&sm.empty[it % kStages]);
        }
    }
    __syncwarp();
    cluster_barrier();      // no CTA leaves while a peer may still send to it
}

// ------------------------------------------------------------------ row statistics ----
// rstd of every row, with the sum of squares taken in FP64 in column order k = 0, 1, ...,
// K - 1: one sequential chain per row, so every partial sum is rounded exactly as the
// definition's running sum is, and rstd equals it bit for bit.  Each value is converted
// exactly (BF16 -> FP32 by a shift, FP32 -> FP64 by the conversion instruction, which keeps
// zeros, subnormals, infinities and NaNs) and its square is exact in FP64, so the fused
// multiply-add rounds once, as the definition's separate square and add do.
//
// One thread per row.  A CTA of kSWarps consumer warps owns kSRows consecutive rows and
// streams them in [kSRows x 64] boxes (2-D TMA, 128-byte swizzle, no multicast) through a
// ring of kSStages slots, filled by one producer thread.  Thread r reads its row's eight
// 16-byte chunks of a box in column order (chunk c sits at position c ^ (r % 8) of the
// row's 128 bytes, so a warp's reads take the minimum four shared-memory wavefronts).
//
// The chain of K dependent FP64 operations per row sets a floor of roughly K times the
// FP64 latency, whatever M is; with enough rows per SM (M of about 200 rows per SM and
// up) the grid is bound by HBM instead.
constexpr int kSWarps = 2;
constexpr int kSRows = 32 * kSWarps;               // rows per CTA
constexpr int kSStages = 6;
constexpr int kSThreads = (kSWarps + 1) * 32;     // + the TMA producer warp
constexpr uint32_t kSBoxBytes = kSRows * 128;      // [kSRows][64] BF16

struct alignas(1024) SSmem {
    uint16_t box[kSStages][kSRows * 64];
    uint64_t full[kSStages];
    uint64_t empty[kSStages];
    int abort;
};
constexpr size_t kSSmemBytes = sizeof(SSmem) + 1024;
static_assert(kSBoxBytes % 1024 == 0, "128-byte-swizzled boxes start on 1024-byte boundaries");

// acc + the squares of eight BF16 values (four packed words, element 2i in the low half of
// w[i]), added one at a time in element order.
__device__ __forceinline__ double sumsq8(const uint4 v, double acc)
{
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const double lo = static_cast<double>(bf16_lo(w[i]));
        const double hi = static_cast<double>(bf16_hi(w[i]));
        acc = fma(lo, lo, acc);
        acc = fma(hi, hi, acc);
    }
    return acc;
}

__global__ void __launch_bounds__(kSThreads)
    row_rstd_kernel(const __grid_constant__ CUtensorMap tmX, int64_t K, float eps,
                    float *__restrict__ rstd)
{
    extern __shared__ uint8_t smem_raw[];
    SSmem &sm = *reinterpret_cast<SSmem *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~static_cast<uintptr_t>(1023));
    const int warp = threadIdx.x >> 5;
    const uint32_t lane = threadIdx.x & 31;
    volatile int *abort = &sm.abort;
    if (threadIdx.x == 0) {
        for (int i = 0; i < kSStages; ++i) {
            mbar_init(&sm.full[i], 1);
            mbar_init(&sm.empty[i], kSWarps);
        }
        sm.abort = 0;
        fence_barrier_init();
    }
    __syncthreads();
    // the quantizer that reads rstd may launch now; it waits for this grid to complete
    asm volatile("griddepcontrol.launch_dependents;");
    const int nbox = static_cast<int>(K / 64);
    const int32_t row0 = static_cast<int32_t>(blockIdx.x) * kSRows;

    if (warp == kSWarps) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            prefetch_tensormap(&tmX);
            uint32_t st = 0, ph = 0;
            int b = 0;
            for (; b < nbox; ++b) {
                if (!mbar_wait(&sm.empty[st], ph ^ 1, abort))
                    break;
                mbar_arrive_expect_tx(&sm.full[st], kSBoxBytes);
                tma_load_2d(sm.box[st], &tmX, &sm.full[st], b * 64, row0);
                if (++st == kSStages) {
                    st = 0;
                    ph ^= 1;
                }
            }
            if (b < nbox) {
                // the copies already in flight land before shared memory is released
                volatile int no_abort = 0;
                for (int j = b > kSStages ? b - kSStages : 0; j < b; ++j)
                    mbar_wait(&sm.full[j % kSStages], (j / kSStages) & 1, &no_abort, 100000000ull);
            }
        }
        return;
    }

    // ---------------------------------------------------------------- consumers
    const int r = threadIdx.x;                         // row within the CTA
    const uint32_t sw = static_cast<uint32_t>(r & 7);
    double acc = 0.0;
    uint32_t st = 0, ph = 0;
    bool ok = true;
    for (int b = 0; b < nbox; ++b) {
        ok = mbar_wait(&sm.full[st], ph, abort);
        if (__any_sync(0xFFFFFFFFu, !ok)) {
            ok = false;
            break;
        }
        const uint16_t *row = sm.box[st] + r * 64;
#pragma unroll
        for (uint32_t c = 0; c < 8; ++c)
            acc = sumsq8(ld_shared_v4(row + ((c ^ sw) << 3)), acc);
        // the sums depend on every value read: the slot is free again
        __syncwarp();
        if (lane == 0)
            mbar_arrive(&sm.empty[st]);
        if (++st == kSStages) {
            st = 0;
            ph ^= 1;
        }
    }
    if (ok)
        rstd[row0 + r] = static_cast<float>(1.0 / sqrt(acc / static_cast<double>(K) + static_cast<double>(eps)));
}

} // namespace norm
} // namespace w8a8
