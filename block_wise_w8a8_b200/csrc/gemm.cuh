// gemm.cuh -- persistent warp-specialised tcgen05 GEMM for sm_100a.
//
// Modes
//   kI8Scaled : the block-scaled W8A8 GEMM (TurboT2VA paper, inference-stack section,
//               W8A8 operator paragraph: the blockwise strategy applies the scales along
//               the reduction dimension; TurboDiffusion article, inference list item 4:
//               INT8 tensor cores).  For every 128-wide K block kb the INT32 partial
//               product P[m,n,kb] of the INT8 codes is formed by tcgen05.mma kind::i8 in
//               tensor memory, then the epilogue warps add float(P) * (xs * ws) into FP32
//               running sums held in registers.  After the last block: + bias, BF16 store.
//   kI8Gated  : kI8Scaled with the gated residual update of the TurboT2VA paper's fused-
//               operator paragraph in the epilogue: y = bf16(r + gate[m / T] * v).
//   kI8Dump   : same main loop; the epilogue writes P[m,n,kb] of a window itself (test hook).
//   kBf16     : BF16 x BF16 -> FP32 GEMM (kind::f16) for the guard's fallback (TurboT2VA
//               paper, guard paragraph), FP32 accumulation over all of K in tensor memory.
//   kI8Row    : the per-row / per-output-channel post-scale W8A8 operator (TurboT2VA
//               paper, W8A8 operator paragraph): INT8 x INT8 accumulated in INT32 over all
//               of K in tensor memory, both scales and the bias applied once per tile.
//
// Tile 128 x 256 (BM x BN), one 128-byte K slice per pipeline stage (128 INT8 or 64 BF16
// elements = exactly one K block of the INT8 path), 4 stages of 48 KB in shared memory,
// filled by TMA with 128-byte swizzle.  Twelve warps in three warpgroups.  Warpgroup 0:
// warp 0 is the TMA producer, warp 1 allocates TMEM and issues the MMAs (one thread),
// warps 2-3 only wait for the end.  Warpgroups 1-2 (warps 4-11) are the epilogue; warp w
// reads TMEM lanes 32 (w % 4) .. + 31 (the rows it may access) and columns
// 128 ((w - 4) / 4) .. + 127.  The kernel is launched with 168 registers per thread (the
// most 12 warps allow: each SM sub-partition holds 16K registers and 3 of the warps);
// warpgroup 0 then gives registers back (setmaxnreg.dec to 80) and the epilogue
// warpgroups take them (setmaxnreg.inc to 208), enough for 128 FP32 running sums per
// thread.  128 * 80 + 256 * 208 = 63488 <= 384 * 168, the launch's total.
// Two 256-column accumulators in TMEM (all 512 columns) let the MMA of one K block (INT8)
// or tile (BF16) overlap the epilogue of the previous one.
//
// INT32 -> FP32 without conversion instructions: each INT8 accumulator is pre-filled with
// the bit pattern of 1.5 * 2^23 (0x4B400000) and the MMAs accumulate onto it.  Because
// |P| <= 128 * 127^2 < 2^22, the 32-bit word afterwards is the FP32 number 12582912 + P
// exactly; one FP32 subtraction recovers float(P) exactly.  The epilogue then re-fills
// the accumulator with the pattern for the next K block.
#pragma once

#include "common.cuh"

namespace w8a8 {
namespace gemm {

enum class Mode : int { kI8Scaled = 0, kI8Dump = 1, kBf16 = 2, kI8Row = 3, kI8Gated = 4 };

constexpr int BM = 128;
constexpr int BN = 256;
constexpr int KSLICE_BYTES = 128;
constexpr int STAGES = 4;
constexpr int A_BYTES = BM * KSLICE_BYTES;
constexpr int B_BYTES = BN * KSLICE_BYTES;
constexpr int NUM_EPI_WARPS = 8;
constexpr int EPI_WARP0 = 4;                 // first epilogue warp (warpgroup 1)
constexpr int NUM_THREADS = 128 + NUM_EPI_WARPS * 32;
constexpr int kLaunchRegs = 168;
constexpr int kRegsControl = 80;             // warpgroup 0 after setmaxnreg.dec
constexpr int kRegsEpilogue = 208;           // warpgroups 1-2 after setmaxnreg.inc
static_assert(128 * kRegsControl + 256 * kRegsEpilogue <= NUM_THREADS * kLaunchRegs,
              "register split exceeds the launch's registers");
constexpr uint32_t TMEM_COLS = 512;
constexpr int KB_MAX = 512;                  // K <= 65536 on the INT8 path
constexpr uint32_t kAccInit = 0x4B400000u;   // FP32 1.5 * 2^23
constexpr float kAccInitF = 12582912.0f;
constexpr int TILE_GROUP = 16;               // M tiles per rasterisation group

struct alignas(1024) Smem {
    uint8_t a[STAGES][A_BYTES];
    uint8_t b[STAGES][B_BYTES];
    float sx[2][KB_MAX];           // [tile parity][kb]: xs[tm, kb]
    float sw[2][2][KB_MAX];        // [tile parity][N half][kb]: ws[2 tn + half, kb]
    // [tile % 3][column]: bias[256 tn + c] (BF16).  Three copies: the copy for tile i + 1
    // is fetched at the start of tile i, while a slower warp may still be storing tile
    // i - 1 (sx and sw, read only inside the K loop, need two).
    alignas(16) uint16_t sbias[3][BN];
    uint64_t full[STAGES];
    uint64_t empty[STAGES];
    uint64_t tfull[2];
    uint64_t tempty[2];
    uint64_t mma_done;
    uint64_t sready[2];            // scale table sprod[b] written (all epilogue threads)
    alignas(1024) uint8_t stage[8][32 * 64]; // per epilogue warp: 32 rows x 64 bytes
    uint32_t tmem_base;
    int abort;
};
constexpr size_t kSmemBytes = sizeof(Smem) + 1024;
static_assert(kSmemBytes <= 232448, "exceeds the 227 KB of shared memory a CTA may use");

// Byte offset of 16-byte piece c (0..3) of row r (0..31) in an epilogue warp's staging
// buffer: rows of 64 bytes, pieces XOR-swizzled with (r / 2) % 4, so that a warp writing
// one piece of each of its 32 rows, or reading 4 pieces of 8 rows, hits 32 distinct banks
// in every quarter-warp phase.  This is the TMA's 64-byte swizzle (16-byte chunk index
// XOR address bits 7-8) for a buffer aligned to 512 bytes, so a TMA store with
// CU_TENSOR_MAP_SWIZZLE_64B reads the buffer back as plain rows.
__device__ __forceinline__ uint32_t stage_off(int r, int c)
{
    return static_cast<uint32_t>(r * 64 + ((c ^ ((r >> 1) & 3)) << 4));
}

struct Params {
    int64_t M, N, K;
    int32_t num_tm, num_tn, num_tiles, kslices;
    // Work units: units 0 .. num_full - 1 are whole tiles (in tile order); the remaining
    // tiles are each split into two 128-column halves, units num_full + 2 i + h.  The
    // host splits only the scaled modes' last, partial round of tiles.
    int32_t num_full, num_units;
    const float *xs;          // [M/128, K/128] (INT8 modes)
    const float *ws;          // [N/128, K/128] (INT8 modes)
    const uint16_t *bias;     // [N] BF16 or null
    uint16_t *y;              // [M, N] BF16
    // Gated residual (kI8Gated): y = bf16(fl(resid + fl(gate[m / gate_T] * v))) with v the
    // FP32 output of kI8Scaled; resid may be y itself.
    const uint16_t *resid;    // [M, N] BF16
    const uint16_t *gate;     // [M / gate_T, N] BF16
    int64_t gate_T;
    // dump mode: P[m, n, kb] of the window rows dm0 .. dm0 + drows - 1, columns
    // dn0 .. dn0 + dcols - 1 (relative to this launch's operands) into dump, laid out
    // [drows, dcols, K/128]
    int32_t *dump;
    int64_t dm0, drows, dn0, dcols;
};

__device__ __forceinline__ void tile_coords(int t, int num_tm, int num_tn, int &tm, int &tn)
{
    const int per_group = TILE_GROUP * num_tn;
    const int group = t / per_group;
    const int first = group * TILE_GROUP;
    const int gsz = min(num_tm - first, TILE_GROUP);
    const int local = t - group * per_group;
    tm = first + local % gsz;
    tn = local / gsz;
}

// The tile of work unit u and which 128-column half of it (-1: the whole tile).
__device__ __forceinline__ void unit_coords(int u, const Params &p, int &tm, int &tn, int &hs)
{
    if (u < p.num_full) {
        tile_coords(u, p.num_tm, p.num_tn, tm, tn);
        hs = -1;
    } else {
        const int v = u - p.num_full;
        tile_coords(p.num_full + (v >> 1), p.num_tm, p.num_tn, tm, tn);
        hs = v & 1;
    }
}

// The GEMM's bounded mbarrier wait.  Its try_wait carries a suspend-time hint, so a
// waiting thread sleeps in hardware until the phase completes instead of re-polling:
// the TMA producer and the MMA thread share SM sub-partitions with epilogue warps, and
// their polling took issue slots from them.  Otherwise as mbar_wait: false after a
// timeout (recorded, *abort raised) or once another thread has raised *abort.
__device__ __forceinline__ bool try_wait_sleep(uint32_t bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.b32 %0, 1, 0, p;\n\t}\n"
        : "=r"(ok)
        : "r"(bar), "r"(parity), "n"(1000000)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ bool gemm_wait(uint64_t *bar, uint32_t parity, volatile int *abort)
{
    const uint32_t b = smem_u32(bar);
    if (try_wait_sleep(b, parity))
        return true;
    const uint64_t t0 = global_timer_ns();
    while (true) {
        if (try_wait_sleep(b, parity))
            return true;
        if (*abort)
            return false;
        if (global_timer_ns() - t0 > kWaitTimeoutNs) {
            *abort = 1;
            record_device_error(1);
            return false;
        }
    }
}

// TMA store of one 2-D box from shared memory (bulk-group completion, no multicast), and
// the waits on this thread's outstanding bulk groups.
__device__ __forceinline__ void tma_store_2d(const CUtensorMap *map, const void *src, int32_t c0,
                                             int32_t c1)
{
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                     reinterpret_cast<uint64_t>(map)),
                 "r"(smem_u32(src)), "r"(c0), "r"(c1)
                 : "memory");
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
// the bulk stores issued by this thread have finished reading shared memory
__device__ __forceinline__ void tma_store_wait_read() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
// ... and have completed
__device__ __forceinline__ void tma_store_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
// generic-proxy writes to shared memory become visible to the TMA (async proxy)
__device__ __forceinline__ void fence_proxy_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

__device__ __forceinline__ void prefetch_l2(const void *p)
{
    asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}

// Eight BF16 bias values from the tile's copy in shared memory, as FP32.
__device__ __forceinline__ void load_bias8_smem(const uint16_t *b, float (&bb)[8])
{
    const uint4 bv = ld_shared_v4(b);
    bb[0] = bf16_lo(bv.x); bb[1] = bf16_hi(bv.x);
    bb[2] = bf16_lo(bv.y); bb[3] = bf16_hi(bv.y);
    bb[4] = bf16_lo(bv.z); bb[5] = bf16_hi(bv.z);
    bb[6] = bf16_lo(bv.w); bb[7] = bf16_hi(bv.w);
}

// The block scales a tile needs, copied global -> shared with cp.async by the epilogue
// threads one tile ahead (no registers are held while the copies are in flight):
// sx[kb] = xs[tm, kb] and sw[h][kb] = ws[2 tn + h, kb] (0 past the last weight block).
__device__ __forceinline__ void cp_async_4(void *dst, const void *src)
{
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(dst)), "l"(src)
                 : "memory");
}
__device__ __forceinline__ void cp_async_16(void *dst, const void *src)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src)
                 : "memory");
}
__device__ __forceinline__ void cp_async_wait_all()
{
    asm volatile("cp.async.wait_all;" ::: "memory");
}

// The tile's bias columns go to sbias the same way (16 bytes a thread, zeros past N or
// without a bias), so that the tile's final phase reads them from shared memory.
__device__ __forceinline__ void scales_fetch(float *sx, float (*sw)[KB_MAX], uint16_t *sbias,
                                             const Params &p, int tm, int tn, int etid, int nthreads)
{
    const int KB = static_cast<int>(p.K / 128);
    const int NB = static_cast<int>(p.N / 128);
    if (etid < BN / 8) {
        const int64_t n = static_cast<int64_t>(tn) * BN + etid * 8;
        if (p.bias != nullptr && n < p.N)
            cp_async_16(sbias + etid * 8, p.bias + n);
        else
            *reinterpret_cast<uint4 *>(sbias + etid * 8) = make_uint4(0, 0, 0, 0);
    }
    for (int i = etid; i < 3 * KB; i += nthreads) {
        const int which = i / KB, kb = i - which * KB;
        if (which == 0) {
            cp_async_4(sx + kb, p.xs + static_cast<int64_t>(tm) * KB + kb);
        } else {
            const int nb = tn * 2 + which - 1;
            if (nb < NB)
                cp_async_4(&sw[which - 1][kb], p.ws + static_cast<int64_t>(nb) * KB + kb);
            else
                sw[which - 1][kb] = 0.0f;
        }
    }
}

template <Mode kMode>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                const __grid_constant__ CUtensorMap tmY, const Params p)
{
    constexpr bool kInt8 = (kMode != Mode::kBf16);                    // INT8 operands
    constexpr bool kPerKb = (kMode == Mode::kI8Scaled || kMode == Mode::kI8Dump ||
                             kMode == Mode::kI8Gated);                // per-K-block sums
    constexpr bool kScaled = (kMode == Mode::kI8Scaled || kMode == Mode::kI8Gated);
    constexpr int kSliceElems = kInt8 ? 128 : 64;
    extern __shared__ uint8_t smem_raw[];
    Smem &sm = *reinterpret_cast<Smem *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                         ~static_cast<uintptr_t>(1023));
    const int warp = threadIdx.x >> 5;
    const uint32_t lane = threadIdx.x & 31;
    volatile int *abort = &sm.abort;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&sm.full[s], 1);
            mbar_init(&sm.empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&sm.tfull[b], 1);
            mbar_init(&sm.tempty[b], NUM_EPI_WARPS);
        }
        mbar_init(&sm.mma_done, 1);
        mbar_init(&sm.sready[0], NUM_EPI_WARPS * 32);
        mbar_init(&sm.sready[1], NUM_EPI_WARPS * 32);
        sm.abort = 0;
        fence_barrier_init();
        prefetch_tensormap(&tmA);
        prefetch_tensormap(&tmB);
        if (kMode == Mode::kI8Scaled)
            prefetch_tensormap(&tmY);
    }
    if (warp == 1) {
        tmem_alloc(&sm.tmem_base, TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;
    // When launched as a programmatic dependent of the activation quantizer, the set-up
    // above overlaps the quantizer's last blocks; nothing below reads an operand or a
    // scale before that grid has completed and its writes are visible.  A no-op otherwise.
    asm volatile("griddepcontrol.wait;" ::: "memory");
    if (warp < EPI_WARP0) {
    regs_dec<kRegsControl>();
    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            uint32_t it = 0;
            bool ok = true;
            for (int t = blockIdx.x; ok && t < p.num_units; t += gridDim.x) {
                int tm, tn, hs;
                unit_coords(t, p, tm, tn, hs);
                for (int ks = 0; ks < p.kslices; ++ks, ++it) {
                    const uint32_t s = it % STAGES, ph = (it / STAGES) & 1;
                    if (!gemm_wait(&sm.empty[s], ph ^ 1, abort)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&sm.full[s], A_BYTES + B_BYTES);
                    tma_load_2d(sm.a[s], &tmA, &sm.full[s], ks * kSliceElems, tm * BM);
                    tma_load_2d(sm.b[s], &tmB, &sm.full[s], ks * kSliceElems, tn * BN);
                }
            }
            if (!ok) {
                // let the copies already in flight land before shared memory is released
                volatile int no_abort = 0;
                const uint32_t first = it > STAGES ? it - STAGES : 0;
                for (uint32_t j = first; j < it; ++j)
                    mbar_wait(&sm.full[j % STAGES], (j / STAGES) & 1, &no_abort, 100000000ull);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t idesc_full = kInt8 ? idesc_i8_s32(BM, BN) : idesc_bf16_f32(BM, BN);
            const uint32_t idesc_half = idesc_i8_s32(BM, BN / 2);
            uint32_t it = 0, acc_i = 0;
            bool ok = true;
            for (int t = blockIdx.x; ok && t < p.num_units; t += gridDim.x) {
                int tm, tn, hs;
                unit_coords(t, p, tm, tn, hs);
                // a half unit multiplies by rows 128 hs .. 128 hs + 127 of the B tile (16 KB
                // further in shared memory) into the first 128 accumulator columns
                const uint32_t idesc = hs < 0 ? idesc_full : idesc_half;
                const uint64_t b_off = hs < 0 ? 0 : static_cast<uint64_t>(hs) * ((BN / 2) * 128 / 16);
                uint32_t buf = acc_i & 1;
                if (!kPerKb) {
                    if (!gemm_wait(&sm.tempty[buf], (acc_i >> 1) & 1, abort)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                }
                for (int ks = 0; ks < p.kslices; ++ks, ++it) {
                    const uint32_t s = it % STAGES, ph = (it / STAGES) & 1;
                    // the stage first: it is normally loaded long before the accumulator
                    // comes back, so the MMAs go out as soon as the epilogue releases it
                    if (!gemm_wait(&sm.full[s], ph, abort)) {
                        ok = false;
                        break;
                    }
                    if (kPerKb) {
                        buf = acc_i & 1;
                        if (!gemm_wait(&sm.tempty[buf], (acc_i >> 1) & 1, abort)) {
                            ok = false;
                            break;
                        }
                    }
                    tc_fence_after();
                    const uint32_t d = tmem + buf * BN;
                    const uint64_t ad = umma_desc_sw128(smem_u32(sm.a[s]));
                    const uint64_t bd = umma_desc_sw128(smem_u32(sm.b[s])) + b_off;
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        // each MMA consumes 32 bytes of K: advance start address by 32 B
                        if (kPerKb)
                            umma_i8(d, ad + 2 * k, bd + 2 * k, idesc, 1u);
                        else if (kInt8)
                            umma_i8(d, ad + 2 * k, bd + 2 * k, idesc, (ks | k) != 0);
                        else
                            umma_bf16(d, ad + 2 * k, bd + 2 * k, idesc, (ks | k) != 0);
                    }
                    umma_commit(&sm.empty[s]);
                    if (kPerKb) {
                        umma_commit(&sm.tfull[buf]);
                        ++acc_i;
                    }
                }
                if (!kPerKb && ok) {
                    umma_commit(&sm.tfull[buf]);
                    ++acc_i;
                }
            }
            // all MMAs issued by this thread complete before TMEM is released
            umma_commit(&sm.mma_done);
            volatile int no_abort = 0;
            mbar_wait(&sm.mma_done, 0, &no_abort, 100000000ull);
        }
    }
    } else {
        regs_inc<kRegsEpilogue>();
        // ------------------------------------------------------------ epilogue
        const int ew = warp - EPI_WARP0;
        const int quarter = warp & 3;
        const int half = ew >> 2;
        const int etid = ew * 32 + static_cast<int>(lane);
        const int row = quarter * 32 + static_cast<int>(lane);
        const uint32_t lane_base = tmem + (static_cast<uint32_t>(quarter * 32) << 16) + half * 128;

        // The accumulator re-fill pattern lives in 16 registers for the whole kernel
        // (tcgen05.st takes its sources from consecutive registers).
        uint32_t fill[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
            fill[i] = kAccInit;
        if (kPerKb) {
#pragma unroll
            for (int b = 0; b < 2; ++b)
#pragma unroll
                for (int c = 0; c < 8; ++c)
                    tmem_st16(lane_base + b * BN + c * 16, fill);
            tmem_wait_st();
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
            mbar_arrive(&sm.tempty[0]);
            mbar_arrive(&sm.tempty[1]);
        }

        uint32_t acc_i = 0;
        if (kScaled) {
            const int KB = static_cast<int>(p.K / 128);
            constexpr int kEpiThreads = NUM_EPI_WARPS * 32;
            if (static_cast<int>(blockIdx.x) < p.num_units) {
                int tm, tn, hs;
                unit_coords(blockIdx.x, p, tm, tn, hs);
                scales_fetch(sm.sx[0], sm.sw[0], sm.sbias[0], p, tm, tn, etid, kEpiThreads);
                cp_async_wait_all();
            }
            mbar_arrive(&sm.sready[0]);
            // No named barriers here: every wait of the epilogue is a bounded mbarrier
            // wait, so an abort can never leave part of the warps parked in bar.sync.
            int tile_iter = 0;
            for (int t = blockIdx.x; t < p.num_units; t += gridDim.x, ++tile_iter) {
                int tm, tn, hs;
                unit_coords(t, p, tm, tn, hs);
                // A half unit's sums sit in the first 128 accumulator columns: warpgroup 1
                // takes them (for output half hs); warpgroup 2 only keeps step with the
                // accumulator barriers.
                const bool active = hs < 0 || half == 0;
                const int hcol = hs < 0 ? half : hs;
                const int sb = tile_iter & 1;
                // the scales of this tile were copied by all epilogue threads during the
                // previous tile
                if (!gemm_wait(&sm.sready[sb], (tile_iter >> 1) & 1, abort))
                    break;
                const int tnext = t + gridDim.x;
                if (tnext < p.num_units) {
                    int tm2, tn2, hs2;
                    unit_coords(tnext, p, tm2, tn2, hs2);
                    scales_fetch(sm.sx[sb ^ 1], sm.sw[sb ^ 1], sm.sbias[(tile_iter + 1) % 3], p, tm2, tn2, etid, kEpiThreads);
                }
                if (kMode == Mode::kI8Gated && active) {
                    const int64_t pm = static_cast<int64_t>(tm) * BM + row;
                    const int64_t pn = static_cast<int64_t>(tn) * BN + hcol * 128;
                    if (pn < p.N) {
                        prefetch_l2(p.resid + pm * p.N + pn);
                        prefetch_l2(p.resid + pm * p.N + pn + 64);
                    }
                }
                float2 acc[64];
#pragma unroll
                for (int j = 0; j < 64; ++j)
                    acc[j] = make_float2(0.0f, 0.0f);
                bool ok = true;
                if (active) {
                    const uint32_t lb = hs < 0 ? lane_base : lane_base - half * 128;
                    for (int kb = 0; kb < KB; ++kb) {
                        const uint32_t buf = acc_i & 1;
                        if (!gemm_wait(&sm.tfull[buf], (acc_i >> 1) & 1, abort)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        const float sc = sm.sx[sb][kb] * sm.sw[sb][hcol][kb];   // FP32 scale product
                        const float2 sc2 = make_float2(sc, sc);
                        const float2 nmg = make_float2(-kAccInitF, -kAccInitF);
                        const uint32_t tb = lb + buf * BN;
#pragma unroll
                        for (int c = 0; c < 8; ++c) {
                            uint32_t r[16];
                            tmem_ld16(tb + c * 16, r);
                            tmem_wait_ld(r);
#pragma unroll
                            for (int j = 0; j < 8; ++j) {
                                float2 v = make_float2(__uint_as_float(r[2 * j]), __uint_as_float(r[2 * j + 1]));
                                v = __fadd2_rn(v, nmg);                     // float(P), exact
                                acc[c * 8 + j] = __ffma2_rn(v, sc2, acc[c * 8 + j]);
                            }
                            tmem_st16(tb + c * 16, fill);
                        }
                        tmem_wait_st();
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0)
                            mbar_arrive(&sm.tempty[buf]);
                        ++acc_i;
                    }
                } else {
                    // warpgroup 2 during a half unit: keep step with the accumulator barriers
                    for (int kb = 0; kb < KB; ++kb) {
                        const uint32_t buf = acc_i & 1;
                        if (!gemm_wait(&sm.tfull[buf], (acc_i >> 1) & 1, abort)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0)
                            mbar_arrive(&sm.tempty[buf]);
                        ++acc_i;
                    }
                }
                if (!ok)
                    break;
                cp_async_wait_all();
                mbar_arrive(&sm.sready[sb ^ 1]);
                // bias (+ gated residual) + BF16 store.  This thread owns row m, columns
                // n0 .. n0 + 127; its warp owns rows m_w .. m_w + 31 of those columns.  The
                // warp writes them in four rounds of 32 columns through its staging buffer:
                // each thread puts its row's 64 bytes there, then the warp stores 64-byte
                // row segments, 8 rows per instruction (8 cache lines instead of 32).  The
                // gated mode reads the residual the same way in reverse.
                const int64_t m = static_cast<int64_t>(tm) * BM + row;
                const int64_t n0 = static_cast<int64_t>(tn) * BN + hcol * 128;
                const int64_t m_w = m - static_cast<int64_t>(lane);
                if (kMode == Mode::kI8Scaled && active && n0 < p.N) {
                    // Each round: the warp writes its 32 x 32 BF16 block into its staging
                    // buffer and lane 0 hands it to the TMA, which stores it while the warp
                    // goes on; the buffer is rewritten only after the TMA has read it.
                    uint8_t *stg = sm.stage[ew];
#pragma unroll
                    for (int rd = 0; rd < 4; ++rd) {
                        if (lane == 0)
                            tma_store_wait_read();
                        __syncwarp();
#pragma unroll
                        for (int c = 0; c < 4; ++c) {
                            const int c8 = rd * 4 + c;
                            float bb[8];
                            load_bias8_smem(sm.sbias[tile_iter % 3] + hcol * 128 + c8 * 8, bb);
                            uint32_t o[4];
#pragma unroll
                            for (int i = 0; i < 4; ++i)
                                o[i] = pack_bf16x2(acc[c8 * 4 + i].x + bb[2 * i], acc[c8 * 4 + i].y + bb[2 * i + 1]);
                            st_shared_v4(stg + stage_off(static_cast<int>(lane), c), make_uint4(o[0], o[1], o[2], o[3]));
                        }
                        fence_proxy_async_smem();
                        __syncwarp();
                        if (lane == 0)
                            tma_store_2d(&tmY, stg, static_cast<int32_t>(n0 + rd * 32), static_cast<int32_t>(m_w));
                    }
                } else if (active && n0 < p.N) {
                    uint8_t *stg = sm.stage[ew];
                    const int pr = static_cast<int>(lane >> 2), pc = static_cast<int>(lane & 3);
                    const uint16_t *gp = kMode == Mode::kI8Gated ? p.gate + (m / p.gate_T) * p.N + n0 : nullptr;
#pragma unroll
                    for (int rd = 0; rd < 4; ++rd) {
                        const int64_t ncol = n0 + rd * 32;
                        if (kMode == Mode::kI8Gated) {
                            // the residual's 32 x 32 block, 64-byte row segments
                            uint4 rv[4];
#pragma unroll
                            for (int j = 0; j < 4; ++j)
                                rv[j] = *reinterpret_cast<const uint4 *>(p.resid + (m_w + 8 * j + pr) * p.N + ncol + pc * 8);
#pragma unroll
                            for (int j = 0; j < 4; ++j)
                                st_shared_v4(stg + stage_off(8 * j + pr, pc), rv[j]);
                            __syncwarp();
                        }
#pragma unroll
                        for (int c = 0; c < 4; ++c) {
                            const int c8 = rd * 4 + c;
                            float bb[8];
                            load_bias8_smem(sm.sbias[tile_iter % 3] + hcol * 128 + c8 * 8, bb);
                            uint32_t o[4];
                            if (kMode == Mode::kI8Gated) {
                                // gated residual update (TurboT2VA paper, fused-operator
                                // paragraph): one rounding for the product, one for the sum
                                const uint4 gv = __ldg(reinterpret_cast<const uint4 *>(gp + c8 * 8));
                                const uint4 rv = ld_shared_v4(stg + stage_off(static_cast<int>(lane), c));
                                const uint32_t gw[4] = {gv.x, gv.y, gv.z, gv.w};
                                const uint32_t rw[4] = {rv.x, rv.y, rv.z, rv.w};
#pragma unroll
                                for (int i = 0; i < 4; ++i) {
                                    const float v0 = acc[c8 * 4 + i].x + bb[2 * i];
                                    const float v1 = acc[c8 * 4 + i].y + bb[2 * i + 1];
                                    o[i] = pack_bf16x2(__fadd_rn(bf16_lo(rw[i]), __fmul_rn(bf16_lo(gw[i]), v0)),
                                                       __fadd_rn(bf16_hi(rw[i]), __fmul_rn(bf16_hi(gw[i]), v1)));
                                }
                            } else {
#pragma unroll
                                for (int i = 0; i < 4; ++i)
                                    o[i] = pack_bf16x2(acc[c8 * 4 + i].x + bb[2 * i], acc[c8 * 4 + i].y + bb[2 * i + 1]);
                            }
                            st_shared_v4(stg + stage_off(static_cast<int>(lane), c), make_uint4(o[0], o[1], o[2], o[3]));
                        }
                        __syncwarp();
#pragma unroll
                        for (int j = 0; j < 4; ++j)
                            *reinterpret_cast<uint4 *>(p.y + (m_w + 8 * j + pr) * p.N + ncol + pc * 8) =
                                ld_shared_v4(stg + stage_off(8 * j + pr, pc));
                        __syncwarp();
                    }
                }
            }
            // the output stores still in flight complete before the CTA exits
            if (kMode == Mode::kI8Scaled && lane == 0)
                tma_store_wait_all();
        } else if (kMode == Mode::kI8Dump) {
            const int KB = static_cast<int>(p.K / 128);
            for (int t = blockIdx.x; t < p.num_tiles; t += gridDim.x) {
                int tm, tn;
                tile_coords(t, p.num_tm, p.num_tn, tm, tn);
                const int64_t m = static_cast<int64_t>(tm) * BM + row;
                const int64_t n0 = static_cast<int64_t>(tn) * BN + half * 128;
                bool ok = true;
                for (int kb = 0; kb < KB; ++kb) {
                    const uint32_t buf = acc_i & 1;
                    if (!gemm_wait(&sm.tfull[buf], (acc_i >> 1) & 1, abort)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t tb = lane_base + buf * BN;
#pragma unroll 1
                    for (int c = 0; c < 4; ++c) {
                        uint32_t r[32];
                        tmem_ld32(tb + c * 32, r);
                        tmem_wait_ld(r);
                        const int64_t wm = m - p.dm0;
                        if (n0 < p.N && wm >= 0 && wm < p.drows) {
#pragma unroll
                            for (int j = 0; j < 32; ++j) {
                                const float v = __uint_as_float(r[j]) - kAccInitF;
                                const int64_t wn = n0 + c * 32 + j - p.dn0;
                                if (wn >= 0 && wn < p.dcols)
                                    p.dump[(wm * p.dcols + wn) * KB + kb] = static_cast<int32_t>(v);
                            }
                        }
                        tmem_st16(tb + c * 32, fill);
                        tmem_st16(tb + c * 32 + 16, fill);
                    }
                    tmem_wait_st();
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0)
                        mbar_arrive(&sm.tempty[buf]);
                    ++acc_i;
                }
                if (!ok)
                    break;
            }
        } else if (kMode == Mode::kI8Row) {
            // Per-row / per-output-channel scales (TurboT2VA paper, W8A8 operator
            // paragraph): one INT32 accumulator per tile over all of K, read once;
            // y = bf16(fl(fl(float(acc) * fl(xs[m] * ws[n])) + b)), no fused multiply-add.
            for (int t = blockIdx.x; t < p.num_tiles; t += gridDim.x) {
                int tm, tn;
                tile_coords(t, p.num_tm, p.num_tn, tm, tn);
                const uint32_t buf = acc_i & 1;
                if (!gemm_wait(&sm.tfull[buf], (acc_i >> 1) & 1, abort))
                    break;
                tc_fence_after();
                const int64_t m = static_cast<int64_t>(tm) * BM + row;
                const int64_t n0 = static_cast<int64_t>(tn) * BN + half * 128;
                const uint32_t tb = lane_base + buf * BN;
                const float sx = p.xs[m];
#pragma unroll 1
                for (int c = 0; c < 4; ++c) {
                    uint32_t r[32];
                    tmem_ld32(tb + c * 32, r);
                    tmem_wait_ld(r);
                    const int64_t nc = n0 + c * 32;
                    if (nc < p.N) {
                        uint16_t *dst = p.y + m * p.N + nc;
#pragma unroll
                        for (int g = 0; g < 4; ++g) {
                            const float4 w0 = __ldg(reinterpret_cast<const float4 *>(p.ws + nc + g * 8));
                            const float4 w1 = __ldg(reinterpret_cast<const float4 *>(p.ws + nc + g * 8 + 4));
                            const float wsv[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
                            float bb[8];
                            if (p.bias != nullptr) {
                                const uint4 bv = __ldg(reinterpret_cast<const uint4 *>(p.bias + nc + g * 8));
                                bb[0] = bf16_lo(bv.x); bb[1] = bf16_hi(bv.x);
                                bb[2] = bf16_lo(bv.y); bb[3] = bf16_hi(bv.y);
                                bb[4] = bf16_lo(bv.z); bb[5] = bf16_hi(bv.z);
                                bb[6] = bf16_lo(bv.w); bb[7] = bf16_hi(bv.w);
                            } else {
#pragma unroll
                                for (int i = 0; i < 8; ++i)
                                    bb[i] = 0.0f;
                            }
                            float v[8];
#pragma unroll
                            for (int i = 0; i < 8; ++i) {
                                const float a = __int2float_rn(static_cast<int>(r[g * 8 + i]));
                                v[i] = __fadd_rn(__fmul_rn(a, __fmul_rn(sx, wsv[i])), bb[i]);
                            }
                            uint4 o;
                            o.x = pack_bf16x2(v[0], v[1]);
                            o.y = pack_bf16x2(v[2], v[3]);
                            o.z = pack_bf16x2(v[4], v[5]);
                            o.w = pack_bf16x2(v[6], v[7]);
                            *reinterpret_cast<uint4 *>(dst + g * 8) = o;
                        }
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0)
                    mbar_arrive(&sm.tempty[buf]);
                ++acc_i;
            }
        } else {
            // BF16: one accumulator per tile, read once at the end of the tile.
            const bool vec_ok = (p.N % 8) == 0;
            for (int t = blockIdx.x; t < p.num_tiles; t += gridDim.x) {
                int tm, tn;
                tile_coords(t, p.num_tm, p.num_tn, tm, tn);
                const uint32_t buf = acc_i & 1;
                if (!gemm_wait(&sm.tfull[buf], (acc_i >> 1) & 1, abort))
                    break;
                tc_fence_after();
                const int64_t m = static_cast<int64_t>(tm) * BM + row;
                const int64_t n0 = static_cast<int64_t>(tn) * BN + half * 128;
                const uint32_t tb = lane_base + buf * BN;
#pragma unroll 1
                for (int c = 0; c < 4; ++c) {
                    uint32_t r[32];
                    tmem_ld32(tb + c * 32, r);
                    tmem_wait_ld(r);
                    const int64_t nc = n0 + c * 32;
                    if (m < p.M && nc < p.N) {
                        uint16_t *dst = p.y + m * p.N + nc;
                        if (vec_ok && nc + 32 <= p.N) {
#pragma unroll
                            for (int g = 0; g < 4; ++g) {
                                float v[8];
#pragma unroll
                                for (int i = 0; i < 8; ++i) {
                                    v[i] = __uint_as_float(r[g * 8 + i]);
                                    if (p.bias != nullptr)
                                        v[i] += __uint_as_float(static_cast<uint32_t>(p.bias[nc + g * 8 + i]) << 16);
                                }
                                uint4 o;
                                o.x = pack_bf16x2(v[0], v[1]);
                                o.y = pack_bf16x2(v[2], v[3]);
                                o.z = pack_bf16x2(v[4], v[5]);
                                o.w = pack_bf16x2(v[6], v[7]);
                                *reinterpret_cast<uint4 *>(dst + g * 8) = o;
                            }
                        } else {
                            for (int i = 0; i < 32 && nc + i < p.N; ++i) {
                                float v = __uint_as_float(r[i]);
                                if (p.bias != nullptr)
                                    v += __uint_as_float(static_cast<uint32_t>(p.bias[nc + i]) << 16);
                                dst[i] = static_cast<uint16_t>(pack_bf16x2(v, 0.0f) & 0xFFFFu);
                            }
                        }
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0)
                    mbar_arrive(&sm.tempty[buf]);
                ++acc_i;
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
}

// ------------------------------------------------------------------ CUDA-core fallback
// y = x w^T + bias for any shape, alignment or K (including K = 0): 64 x 64 output tile
// per 256-thread CTA, 4 x 4 outputs per thread, FP32 accumulation, K staged through
// shared memory 16 at a time.  Used only when the tensor-core kernel cannot take the
// buffers (K not a multiple of 8, or unaligned pointers).
__global__ void __launch_bounds__(256) bf16_gemm_simt_kernel(
    const uint16_t *__restrict__ x, const uint16_t *__restrict__ w,
    const uint16_t *__restrict__ bias, uint16_t *__restrict__ y, int64_t M, int64_t K, int64_t N)
{
    __shared__ float xs[16][64 + 1];
    __shared__ float wsh[16][64 + 1];
    const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
    const int64_t m0 = static_cast<int64_t>(blockIdx.y) * 64;
    const int64_t n0 = static_cast<int64_t>(blockIdx.x) * 64;
    float acc[4][4] = {};
    for (int64_t k0 = 0; k0 < K; k0 += 16) {
        for (int i = threadIdx.x; i < 16 * 64; i += 256) {
            const int kk = i & 15, rr = i >> 4;
            const int64_t gm = m0 + rr, gn = n0 + rr, gk = k0 + kk;
            xs[kk][rr] = (gm < M && gk < K) ? __uint_as_float(static_cast<uint32_t>(x[gm * K + gk]) << 16) : 0.0f;
            wsh[kk][rr] = (gn < N && gk < K) ? __uint_as_float(static_cast<uint32_t>(w[gn * K + gk]) << 16) : 0.0f;
        }
        __syncthreads();
#pragma unroll
        for (int kk = 0; kk < 16; ++kk) {
            float a[4], b[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                a[i] = xs[kk][ty * 4 + i];
                b[i] = wsh[kk][tx * 4 + i];
            }
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int64_t gm = m0 + ty * 4 + i;
        if (gm >= M)
            continue;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int64_t gn = n0 + tx * 4 + j;
            if (gn >= N)
                continue;
            float v = acc[i][j];
            if (bias != nullptr)
                v += __uint_as_float(static_cast<uint32_t>(bias[gn]) << 16);
            y[gm * N + gn] = static_cast<uint16_t>(pack_bf16x2(v, 0.0f) & 0xFFFFu);
        }
    }
}

} // namespace gemm
} // namespace w8a8
