// conv2d_tcs.cuh -- op A on tcgen05 tensor cores with the nine 3x3 taps read as
// shifted shared-memory operands: no im2col, four images side by side.
//
// What it computes (POPCORNBENCH trace "Kimi-K2.6__l2_p65": the conv formula
// and shapes of its opening analysis, the bias-folding step, the pool
// semantics): every conv output y[n, co, r, c] = b[co] + sum over (ci, ky, kx)
// of w[co, ci, ky, kx] * x[n, ci, r+ky, c+kx], averaged over P x P windows
// (stride P, floor), passed through the sigmoid and summed per image.  Every
// conv output of every kept window is computed -- the same multiply-adds as
// the FP32-FMA kernel -- only on the tensor cores.
//
// Formulation.  A unit of work is (image group g of four images, column tile
// of NCOL conv columns, pooled row ph).  For each of its P conv rows r and each
// tap (ky, kx) one MMA adds
//     D[m, j] += sum_ci A_t[m, ci] * X[ci, j],   j = 4 * c + i,
// with m = 128 weight rows (output channels 0-63 with the TF32 hi part of w,
// then the same 64 with the lo part; the A operand, resident in tensor memory
// for the whole kernel), c = conv column of the tile, i = image
// of the group and X[ci, j] = x[4g + i, ci, r + ky, c0 + c + kx].  The input
// row r + ky is staged in shared memory as the MMA's K-major B operand without
// swizzle: position j = 4c + i owns one 16-byte row holding 4 channels, the
// rows of consecutive positions are 16 bytes apart (8-row groups 128 bytes
// apart), and the next 4 channels sit in a second plane (the leading-byte
// offset).  A tap's column shift kx moves the operand's start address by kx *
// 64 bytes (four positions) and its row shift ky selects another staged row:
// all nine taps read the same staged rows in place.  The P conv rows of a pooled row accumulate into the
// same TMEM accumulator, so the vertical half of the P x P pooling costs
// nothing; the epilogue adds the P columns of each window.
//
// fp32 accuracy (the trace's precision discussion rejects plain TF32 against
// atol = rtol = 1e-4): x = x_hi + x_lo and w = w_hi + w_lo with the hi parts
// truncated to TF32 (exactly representable, so the tensor core reads them
// unchanged) and the lo parts the exact remainders.  Each tap issues two
// MMAs, [w_hi; w_lo] * x_hi and [w_hi; w_lo] * x_lo, which form w_hi x_hi +
// w_lo x_hi + w_hi x_lo + w_lo x_lo: the error-corrected TF32 product
// (Ootomo & Yokota, 2022) plus its smallest term.  Rows m and m + 64 of D are
// added in the epilogue.
//
// B200 design (one CTA per SM, persistent over a contiguous range of units in
// (g, column tile, ph) order, 11 warps):
//   * warps 0-1 (loaders): one input row of the group (4 images x 8*CCH
//     channels x NCOL + 4 columns) per staging buffer: one 4-D TMA box (no
//     multicast; rows, columns, channels and images outside x read 0), or
//     16-byte cp.async copies when rows are not 16-byte aligned.  Consecutive
//     units of a CTA share the two rows between pooled rows, which are loaded
//     once.
//   * warps 3-6 (producers, one row each in turn): transpose a staged row into
//     [channel quad][column][image][4 channels] and split it into TF32 hi/lo
//     rows of a ring of NSLOT row slots.  Staging buffer and slot of row s are s % 4 and
//     s % NSLOT, so each belongs to one producer warp.
//   * warp 2: allocates TMEM (two accumulators of 4 * NCOL columns and the
//     weights, 72 * CCH columns); one thread issues 2 * 9 * CCH MMAs per conv
//     row (M = 128, N = 4 * NCOL = 192 or 128, K = 8, A from tensor memory, B
//     from shared memory: measured 18 % faster per MMA than both operands from
//     shared memory), releases each row slot after the last conv row that
//     reads it, and commits a unit's accumulator.
//   * warps 7-10 (epilogue, one per TMEM lane quarter): tcgen05.ld 32 columns
//     at a time, add the P columns of each window, exchange the hi and lo
//     halves through shared memory (each pair of warps finishes half of every
//     chunk's pooled values), add the bias, apply the sigmoid and accumulate
//     per image; one atomic add per CTA and image.
//   * Every wait is bounded; a wait that runs out sets the CTA abort flag and
//     the device error word, every role leaves its loop, TMA copies and MMAs
//     still in flight are waited for (bounded) and TMEM is freed.
#pragma once

#include "conv1d_tc.cuh"
#include "conv2d_direct.cuh"

namespace fcv {
namespace c2s {

using tc::globaltimer;
using tc::kWaitLimitNs;
using tc::mbar_arrive;
using tc::mbar_arrive_expect_tx;
using tc::mbar_init;
using tc::mbar_try_wait;
using tc::smem_u32;
using tc::tc_commit;
using tc::tc_fence_after;
using tc::tc_fence_before;
using tc::wait_bounded;

constexpr int IMG = 4;          // images per group: the 4 N-elements of a 16-byte core-matrix row
constexpr int CO_BLK = 64;      // output channels per launch (M = 128 = hi | lo)
constexpr int CIN_MAX = 16;     // input channels covered (two 8-channel K chunks)
constexpr int NSTG = 4;         // staging buffers (buffer b belongs to producer warp b)
constexpr int LOAD_WARP0 = 0;   // warps 0-1
constexpr int MMA_WARP = 2;
constexpr int PROD_WARP0 = 3;   // warps 3-6
constexpr int NPRODW = 4;
constexpr int EPI_WARP0 = 7;    // warps 7-10
constexpr int NTHREADS = 11 * 32;
constexpr int SMEM_LIMIT = 227 * 1024;

// Compile-time geometry of one instance.
template <int P, int CCH>
struct Geo {
    static constexpr int NCOL = CCH == 1 ? 48 : 32;       // conv columns per tile
    static constexpr int NMMA = IMG * NCOL;               // MMA N = accumulator columns
    static constexpr int WPT = NCOL / P;                  // pooled windows per tile
    static constexpr int XC = NCOL + 2;                   // staged columns per row (all read by some tap)
    static constexpr uint32_t PLANE = XC * IMG * 16u;     // one quad of channels: 16 bytes per (column, image)
    static constexpr uint32_t HALF = 2u * CCH * PLANE;    // one hi or lo row copy (2 quads per K chunk)
    static constexpr uint32_t SLOT = 2u * HALF;
    static constexpr int NSLOT = 8;                       // ring of staged rows (slot s belongs to warp s % 4)
    // Staging: [channel][image][column] with pitch SP = NCOL + 8 floats (8 or
    // 24 mod 32, so lanes (image 0-3, column 0-7) read distinct banks); a TMA
    // box is SP columns wide, the cp.async path fills NJ aligned 16-byte copies.
    static constexpr int SP = NCOL + 8;
    static constexpr int NJ = SP / 4;
    static constexpr uint32_t STG = IMG * 8u * CCH * SP * 4u;
    static constexpr int V = 32 / P;                      // pooled values per 32-column chunk (8/P windows x 4 images)
    static constexpr int XP = V == 4 ? 4 : V + 4;         // exchange row pitch (floats), conflict-free
    static constexpr int NCHK = NMMA / 32;                // 32-column chunks per accumulator
    static constexpr uint32_t WCOL0 = 2u * NMMA;          // TMEM: weights (A) after the two accumulators
    static constexpr uint32_t TMEM_COLS = 512;
    static_assert(2 * NMMA + 72 * CCH <= 512, "two accumulators and the weights fit tensor memory");
    static_assert(NCOL % P == 0 && 8 % P == 0, "pool must divide a chunk of 8 columns");
    static_assert((SP % 32 == 8 || SP % 32 == 24) && SP >= XC + 3 + 3,
                  "staging pitch: bank spread, and room for the cp.async shift");
    static_assert(NSTG % NPRODW == 0 && NSLOT % NPRODW == 0,
                  "every staging buffer and row slot is used by one producer warp only");
};

// Shared-memory layout (bytes from a 1024-aligned base).
struct Layout {
    uint32_t slots, stg, xbuf, red, bar, misc, total;
};

template <int P, int CCH>
__host__ __device__ constexpr Layout make_layout()
{
    using G = Geo<P, CCH>;
    Layout L{};
    L.slots = 0;
    L.stg = L.slots + G::NSLOT * G::SLOT;
    L.xbuf = L.stg + NSTG * G::STG;
    L.red = L.xbuf + 2u * CO_BLK * G::XP * 4u;
    L.bar = (L.red + 16u * 4u + 7u) & ~7u;
    // stg_full[NSTG] stg_empty[NSTG] slot_full[NSLOT] slot_empty[NSLOT] acc_full[2] acc_empty[2] drain gate
    L.misc = L.bar + (uint32_t)(2 * NSTG + 2 * G::NSLOT + 6) * 8u;
    L.total = L.misc + 16u;
    return L;
}

// Dynamic shared memory requested: the layout plus alignment slack, and at
// least 120 KB so that two CTAs never share an SM (each allocates all 512 TMEM
// columns; a second one on the same SM would wait in tcgen05.alloc).
template <int P, int CCH>
constexpr uint32_t smem_bytes()
{
    return make_layout<P, CCH>().total + 1024u > 120u * 1024u ? make_layout<P, CCH>().total + 1024u : 120u * 1024u;
}

struct Params {
    const float* x;
    const float* w;     // weights of this launch's first output channel
    const float* b;     // bias of this launch's first output channel
    float* out;         // sum mode: out[N]; tap mode: pooled[N, Cout_total, PH, PW]
    int N, Cin, H, W;
    int Cout;           // output channels of this launch (<= 64)
    int co0, Cout_total;
    int PH, PW;
    int CT;             // column tiles per pooled row
    int PHB;            // pooled rows per block of the unit walk
    long long U;        // units = groups * CT * PH
    long long x_elems;  // N * Cin * H * W
    int use_tma;
    unsigned long long wait_ns;  // limit of the main-loop waits
    // Failure-path test (0 in normal calls): role stall_role (1 loader, 2
    // producers, 3 MMA issuer, 4 epilogue) waits, before its unit stall_at, on
    // a barrier nothing completes; the wait runs out after wait_ns and the CTA
    // takes its abort path.
    int stall_role, stall_at;
};

// Units are walked image group by image group; within a group, in blocks of
// PHB pooled rows: every column tile of a block, each down its PHB pooled rows,
// then the next block.  Consecutive units of one column tile share two input
// rows (loaded once), and the column tiles of a block follow each other
// closely, so the columns their boxes share and the rows between blocks are
// still in L2 when the next box needs them.
struct Unit {
    int g, ct, ph;
    int b0, bh;  // first pooled row and height of the block
};

__device__ __forceinline__ Unit decode(const Params& p, long long u)
{
    Unit t;
    const long long per_g = (long long)p.CT * p.PH;
    t.g = (int)(u / per_g);
    const int r = (int)(u - (long long)t.g * per_g);
    const int full = p.PHB * p.CT;  // units of a full block
    const int blk = r / full;
    t.b0 = blk * p.PHB;
    t.bh = min(p.PHB, p.PH - t.b0);
    const int rb = r - blk * full;
    t.ct = rb / t.bh;
    t.ph = t.b0 + (rb - t.ct * t.bh);
    return t;
}

// The unit after t: every role walks its units this way instead of dividing.
__device__ __forceinline__ void next_unit(const Params& p, Unit& t)
{
    if (++t.ph < t.b0 + t.bh) return;
    t.ph = t.b0;
    if (++t.ct < p.CT) return;
    t.ct = 0;
    t.b0 += t.bh;
    if (t.b0 == p.PH) {
        t.b0 = 0;
        ++t.g;
    }
    t.bh = min(p.PHB, p.PH - t.b0);
    t.ph = t.b0;
}

// Shared-memory matrix descriptor, no swizzle (canonical interleaved layout):
// LBO and SBO in bytes, version 1.
__device__ __forceinline__ uint64_t desc_none(uint32_t saddr, uint32_t lbo, uint32_t sbo)
{
    return (uint64_t)((saddr & 0x3FFFFu) >> 4) | ((uint64_t)(lbo >> 4) << 16) | ((uint64_t)(sbo >> 4) << 32) |
           ((uint64_t)1 << 46);
}

// 32 consecutive 32-bit TMEM columns of the warp's 32 lanes.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32])
{
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];\n"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
}

// 4-D tiled TMA load (no multicast) completing on `bar`.
__device__ __forceinline__ void tma_load_4d(uint32_t dst, const CUtensorMap* map, int c0, int c1, int c2, int c3,
                                            uint32_t bar)
{
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4, %5}], "
        "[%6];\n" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(bar)
        : "memory");
}

// Arrive on `bar` once every cp.async this thread issued so far has landed
// (the arrival was counted in the barrier's expected count).
__device__ __forceinline__ void cp_async_arrive_noinc(uint32_t bar)
{
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];\n" ::"r"(bar) : "memory");
}

// Truncation of an fp32 value to TF32 (the top 19 bits); v - trunc(v) is exact.
__device__ __forceinline__ float tf32_trunc(float v) { return __uint_as_float(__float_as_uint(v) & 0xFFFFE000u); }

// First row (0 or 2) of unit u that its CTA has to load: a unit that directly
// follows the previous pooled row of the same column tile reuses that unit's
// last two input rows.
__device__ __forceinline__ int first_row(long long u, long long u0, const Unit& t)
{
    return (u > u0 && t.ph > t.b0) ? 2 : 0;
}

// Weights of this launch as the A operand in tensor memory: block (tap t,
// chunk c) is 8 consecutive columns from WCOL0 + 8 * (t * CCH + c); lane m holds
// row m, rows 0-63 the TF32 hi part of output channels 0-63 and rows 64-127
// their lo part; column k of a block is input channel 8c + k.  Written by the
// four epilogue warps (warp quarter q owns lanes 32q .. 32q + 31).
template <int CCH>
__device__ __forceinline__ void weights_to_tmem(const Params& p, uint32_t tmem, uint32_t wcol0, int q, int lane)
{
    const int m = 32 * q + lane;
    const int co = m & 63;
    const bool hi_part = m < 64;
    const uint32_t taddr = tmem + ((uint32_t)(32 * q) << 16) + wcol0;
#pragma unroll 1
    for (int blk = 0; blk < 9 * CCH; ++blk) {
        const int t = blk / CCH, c = blk - t * CCH;
        uint32_t r[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            const int ci = 8 * c + k;
            const float v = (co < p.Cout && ci < p.Cin) ? __ldg(p.w + ((size_t)co * p.Cin + ci) * 9 + t) : 0.f;
            const float hi = tf32_trunc(v);
            r[k] = __float_as_uint(hi_part ? hi : v - hi);
        }
        asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};\n" ::"r"(
                         taddr + (uint32_t)(8 * blk)),
                     "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]));
    }
    asm volatile("tcgen05.wait::st.sync.aligned;\n" ::: "memory");
}

// D[tmem] (+)= A[tmem] * B[smem], kind::tf32.
__device__ __forceinline__ void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                       uint32_t accumulate)
{
    asm volatile(
        "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
        " tcgen05.mma.cta_group::1.kind::tf32 [%0], [%1], %2, %3, p;\n}\n" ::"r"(d_tmem),
        "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

template <int P, int CCH, int MODE>
__global__ void __launch_bounds__(NTHREADS, 1)
    conv2d_tcs_kernel(const Params p, const __grid_constant__ CUtensorMap x_map)
{
    using G = Geo<P, CCH>;
    constexpr Layout L = make_layout<P, CCH>();
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    const uint32_t sbase = smem_u32(smem);
    const uint32_t bar_stg_full = sbase + L.bar;                       // + 8 * stage
    const uint32_t bar_stg_empty = bar_stg_full + 8 * NSTG;            // + 8 * stage, 1 producer arrival
    const uint32_t bar_slot_full = bar_stg_empty + 8 * NSTG;           // + 8 * slot, 1 producer arrival
    const uint32_t bar_slot_empty = bar_slot_full + 8 * G::NSLOT;      // + 8 * slot, tcgen05.commit
    const uint32_t bar_acc_full = bar_slot_empty + 8 * G::NSLOT;       // + 8 * buf, tcgen05.commit
    const uint32_t bar_acc_empty = bar_acc_full + 16;                  // + 8 * buf, 4 epilogue arrivals
    const uint32_t bar_drain = bar_acc_empty + 16;
    const uint32_t bar_gate = bar_drain + 8;                           // never completed (failure-path test)
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + L.misc);
    volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(smem + L.misc + 4);
    volatile uint32_t* epi_ok = reinterpret_cast<volatile uint32_t*>(smem + L.misc + 8);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long u0 = (long long)blockIdx.x * p.U / gridDim.x;
    const long long u1 = (long long)(blockIdx.x + 1) * p.U / gridDim.x;
    // Failure-path test: false once role `role` is to stall before unit u (its
    // bounded wait on the gate runs out, which sets the abort flag).
    auto not_stalled = [&](int role, long long u) -> bool {
        if (p.stall_role != role || u - u0 != p.stall_at) return true;
        return wait_bounded(bar_gate, 0, abort_flag, p.wait_ns);
    };

    if (threadIdx.x == 0) {
        for (int i = 0; i < NSTG; ++i) {
            mbar_init(bar_stg_full + 8 * i, p.use_tma ? 1u : 32u);  // TMA: expect_tx; cp.async: 32 lanes
            mbar_init(bar_stg_empty + 8 * i, 1);
        }
        for (int i = 0; i < G::NSLOT; ++i) {
            mbar_init(bar_slot_full + 8 * i, 1);
            mbar_init(bar_slot_empty + 8 * i, 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(bar_acc_full + 8 * i, 1);
            mbar_init(bar_acc_empty + 8 * i, 4);
        }
        mbar_init(bar_drain, 1);
        mbar_init(bar_gate, 1);
        *abort_flag = 0u;
        *epi_ok = 1u;
        asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
    }
    if (warp == MMA_WARP) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(smem_u32(tmem_holder)),
                     "r"(G::TMEM_COLS)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;
    if (warp >= EPI_WARP0) weights_to_tmem<CCH>(p, tmem, G::WCOL0, warp & 3, lane);
    tc_fence_before();
    __syncthreads();  // weights in tensor memory before the first MMA
    tc_fence_after();

    if (warp < MMA_WARP) {
        // ------------------------------------------------------------- loaders
        if (p.use_tma) {
            if (warp == LOAD_WARP0 && lane == 0) {
                long long s = 0;
                long long last[NSTG];
                for (int i = 0; i < NSTG; ++i) last[i] = -1;
                bool ok = true;
                Unit ut = decode(p, u0);
                for (long long u = u0; ok && u < u1; ++u, next_unit(p, ut)) {
                    const Unit t = ut;
                    if (!not_stalled(1, u)) break;
                    for (int j = first_row(u, u0, t); j < P + 2; ++j, ++s) {
                        const int st = (int)(s % NSTG);
                        if (!wait_bounded(bar_stg_empty + 8 * st, (uint32_t)((s / NSTG) & 1) ^ 1u, abort_flag,
                                          p.wait_ns)) {
                            ok = false;
                            break;
                        }
                        mbar_arrive_expect_tx(bar_stg_full + 8 * st, G::STG);
                        // map dims (column, image, channel, row): the box lands as [channel][image][column]
                        tma_load_4d(sbase + L.stg + (uint32_t)st * G::STG, &x_map, t.ct * G::NCOL, IMG * t.g, 0,
                                    t.ph * P + j, bar_stg_full + 8 * st);
                        last[st] = s;
                    }
                }
                {
                    // Wait (bounded) for every box still in flight before the CTA
                    // may leave -- also when another role gave up and the boxes
                    // were never consumed.  Normally they have all landed.
                    for (int i = 0; i < NSTG; ++i) {
                        if (last[i] < 0) continue;
                        const uint32_t par = (uint32_t)((last[i] / NSTG) & 1);
                        const unsigned long long t0 = globaltimer();
                        while (!mbar_try_wait(bar_stg_full + 8 * i, par)) {
                            if (globaltimer() - t0 > kWaitLimitNs) break;
                        }
                    }
                }
            }
        } else {
            // 16-byte cp.async copies of the aligned span around each staged
            // (image, channel) row; warp w loads rows s with s % 2 == w.  Rows of
            // images or channels outside x are not read (the producers write
            // zeros for them); bytes past the end of x are zero-filled.
            long long s = 0;
            bool ok = true;
            Unit ut = decode(p, u0);
            for (long long u = u0; ok && u < u1; ++u, next_unit(p, ut)) {
                const Unit t = ut;
                int go = 1;
                if (lane == 0) go = not_stalled(1, u);
                if (!__shfl_sync(0xffffffffu, go, 0)) break;
                for (int j = first_row(u, u0, t); j < P + 2; ++j, ++s) {
                    if ((int)(s & 1) != warp) continue;
                    const int st = (int)(s % NSTG);
                    int good = 1;
                    if (lane == 0)
                        good = wait_bounded(bar_stg_empty + 8 * st, (uint32_t)((s / NSTG) & 1) ^ 1u, abort_flag,
                                            p.wait_ns);
                    good = __shfl_sync(0xffffffffu, good, 0);
                    if (!good) {
                        ok = false;
                        break;
                    }
                    float* dst = reinterpret_cast<float*>(smem + L.stg + (uint32_t)st * G::STG);
                    const int r = t.ph * P + j, c0 = t.ct * G::NCOL;
                    for (int it = lane; it < IMG * 8 * CCH * G::NJ; it += 32) {
                        const int pr = it / G::NJ, q = it - pr * G::NJ;  // (image, channel) pair, copy index
                        const int img = pr / (8 * CCH), c = pr - img * (8 * CCH);
                        const int n = IMG * t.g + img;
                        if (n >= p.N || c >= p.Cin) continue;
                        const long long e0 = (((long long)n * p.Cin + c) * p.H + r) * p.W + c0;
                        const long long e = (e0 & ~3LL) + 4LL * q;
                        const long long left = p.x_elems - e;
                        const int bytes = left >= 4 ? 16 : (left > 0 ? (int)left * 4 : 0);
                        cp_async16(dst + (c * IMG + img) * G::SP + 4 * q, bytes > 0 ? p.x + e : p.x, bytes);
                    }
                    cp_async_arrive_noinc(bar_stg_full + 8 * st);
                }
            }
            cp_async_wait<0>();  // no copy may land after the CTA has left
        }
    } else if (warp == MMA_WARP) {
        // --------------------------------------------------------- MMA issuer
        if (lane == 0) {
            // D fp32, A (tensor memory) and B tf32, B K-major, N = 4 * NCOL, M = 128.
            constexpr uint32_t idesc = (1u << 4) | (2u << 7) | (2u << 10) | ((uint32_t)(G::NMMA >> 3) << 17) |
                                       ((uint32_t)(128 >> 4) << 24);
            const uint32_t a_tmem0 = tmem + G::WCOL0;  // weights: 8 columns per (tap, chunk)
            // B: position rows 16 bytes apart (8-row groups 128 bytes apart), the
            // second channel quad one plane further (leading-byte offset).
            const uint64_t bconst = desc_none(0u, G::PLANE, 128u);
            // Rows are first needed in sequence order, and a row seen full stays
            // until this thread releases it: `confirmed` is the last row seen full,
            // so each conv row waits for one new row at most.  (Checking ahead
            // without blocking -- test_wait on the next row and the next unit's
            // accumulator while MMAs are queued -- measured no faster for the rows
            // and 13-17 % slower for the accumulator.)
            long long s = 0, confirmed = -1;
            bool ok = true;
            Unit ut = decode(p, u0);
            for (long long u = u0; ok && u < u1; ++u, next_unit(p, ut)) {
                const Unit t = ut;
                if (!not_stalled(3, u)) break;
                const int fj = first_row(u, u0, t);
                const long long base = s - fj;
                s += P + 2 - fj;
                const long long i = u - u0;
                const int abuf = (int)(i & 1);
                const bool cont_next = u + 1 < u1 && t.ph + 1 < t.b0 + t.bh;  // the next unit continues this column tile
                if (!wait_bounded(bar_acc_empty + 8 * abuf, (uint32_t)((i >> 1) & 1) ^ 1u, abort_flag, p.wait_ns)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d = tmem + (uint32_t)(abuf * G::NMMA);
                uint32_t acc = 0u;
                for (int dy = 0; ok && dy < P; ++dy) {
                    // rows base+dy .. base+dy+2, in order
                    while (confirmed < base + dy + 2) {
                        const long long q = confirmed + 1;
                        if (!wait_bounded(bar_slot_full + 8 * (int)(q % G::NSLOT), (uint32_t)((q / G::NSLOT) & 1),
                                          abort_flag, p.wait_ns)) {
                            ok = false;
                            break;
                        }
                        confirmed = q;
                        tc_fence_after();
                    }
                    if (!ok) break;
#pragma unroll
                    for (int ky = 0; ky < 3; ++ky) {
                        const uint32_t sh = sbase + L.slots + (uint32_t)((base + dy + ky) % G::NSLOT) * G::SLOT;
#pragma unroll
                        for (int kx = 0; kx < 3; ++kx) {
#pragma unroll
                            for (int c = 0; c < CCH; ++c) {
                                const uint32_t off = (uint32_t)kx * (IMG * 16u) + (uint32_t)(2 * c) * G::PLANE;
                                const uint32_t a = a_tmem0 + 8u * (uint32_t)((3 * ky + kx) * CCH + c);
                                mma_ts(d, a, bconst | (uint64_t)(((sh + off) & 0x3FFFFu) >> 4), idesc, acc);
                                mma_ts(d, a, bconst | (uint64_t)(((sh + G::HALF + off) & 0x3FFFFu) >> 4), idesc, 1u);
                                acc = 1u;
                            }
                        }
                    }
                    tc_commit(bar_slot_empty + 8 * (int)((base + dy) % G::NSLOT));  // row base+dy read for the last time
                }
                if (!ok) break;
                if (!cont_next) {
                    // No continuation: the unit's last two rows are not read again.
                    tc_commit(bar_slot_empty + 8 * (int)((base + P) % G::NSLOT));
                    tc_commit(bar_slot_empty + 8 * (int)((base + P + 1) % G::NSLOT));
                }
                tc_commit(bar_acc_full + 8 * abuf);
            }
            tc_commit(bar_drain);
            const unsigned long long t0 = globaltimer();
            while (!mbar_try_wait(bar_drain, 0)) {
                if (globaltimer() - t0 > kWaitLimitNs) {
                    *abort_flag = 1u;
                    record_device_error(kErrTimeout);
                    break;
                }
            }
        }
        __syncwarp();
    } else if (warp < EPI_WARP0) {
        // ----------------------------------------------------------- producers
        // Row s goes to producer warp s % 4: staging buffer s % NSTG into row
        // slot s % NSLOT as [channel quad][column][image][4 channels], hi and lo
        // copies.  NSTG and NSLOT are multiples of 4, so each buffer and slot is
        // only ever used by one warp, in order: a parity wait is then never more
        // than one phase behind and cannot pass on a stale phase.  Lane
        // (image lane % 4, column lane / 4) makes both the staging reads (pitch
        // 8 or 24 mod 32 floats) and the 16-byte slot stores conflict-free: the
        // 8 lanes a store serves at a time write 128 contiguous bytes.
        const int pw = warp - PROD_WARP0;
        const int img = lane & 3, col_lo = lane >> 2;
        long long s = 0;
        bool ok = true;
        Unit ut = decode(p, u0);
        for (long long u = u0; ok && u < u1; ++u, next_unit(p, ut)) {
            const Unit t = ut;
            int go = 1;
            if (lane == 0 && pw == 0) go = not_stalled(2, u);
            if (!__shfl_sync(0xffffffffu, go, 0)) break;
            for (int j = first_row(u, u0, t); j < P + 2; ++j, ++s) {
                if ((int)(s % NPRODW) != pw) continue;
                const int st = (int)(s % NSTG), sl = (int)(s % G::NSLOT);
                int good = 1;
                if (lane == 0) {
                    good = wait_bounded(bar_slot_empty + 8 * sl, (uint32_t)((s / G::NSLOT) & 1) ^ 1u, abort_flag,
                                        p.wait_ns) &&
                           wait_bounded(bar_stg_full + 8 * st, (uint32_t)((s / NSTG) & 1), abort_flag, p.wait_ns);
                }
                good = __shfl_sync(0xffffffffu, good, 0);
                if (!good) {
                    ok = false;
                    break;
                }
                // every lane acquires the staged data (returns at once)
                for (int spin = 0; !mbar_try_wait(bar_stg_full + 8 * st, (uint32_t)((s / NSTG) & 1)) && spin < (1 << 20);
                     ++spin) {
                }
                const float* sg = reinterpret_cast<const float*>(smem + L.stg + (uint32_t)st * G::STG);
                uint8_t* slot = smem + L.slots + (uint32_t)sl * G::SLOT;
                const int r = t.ph * P + j, c0 = t.ct * G::NCOL;
#pragma unroll 2
                for (int it = 0; it < 2 * CCH * ((G::XC + 7) / 8); ++it) {
                    const int qd = it % (2 * CCH), col = 8 * (it / (2 * CCH)) + col_lo;
                    if (col >= G::XC) continue;
                    float v[4];
                    if (p.use_tma) {
#pragma unroll
                        for (int e = 0; e < 4; ++e) v[e] = sg[((4 * qd + e) * IMG + img) * G::SP + col];
                    } else {
                        const int n = IMG * t.g + img;
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const int c = 4 * qd + e;
                            float x = 0.f;
                            if (n < p.N && c < p.Cin && c0 + col < p.W) {
                                const long long e0 = (((long long)n * p.Cin + c) * p.H + r) * p.W + c0;
                                x = sg[(c * IMG + img) * G::SP + (int)(e0 & 3) + col];
                            }
                            v[e] = x;
                        }
                    }
                    float4 h, l;
                    h.x = tf32_trunc(v[0]); l.x = v[0] - h.x;
                    h.y = tf32_trunc(v[1]); l.y = v[1] - h.y;
                    h.z = tf32_trunc(v[2]); l.z = v[2] - h.z;
                    h.w = tf32_trunc(v[3]); l.w = v[3] - h.w;
                    const uint32_t off = (uint32_t)qd * G::PLANE + ((uint32_t)col * IMG + img) * 16u;
                    *reinterpret_cast<float4*>(slot + off) = h;
                    *reinterpret_cast<float4*>(slot + G::HALF + off) = l;
                }
                asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");  // slot visible to the tensor core
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(bar_slot_full + 8 * sl);
                    mbar_arrive(bar_stg_empty + 8 * st);
                }
            }
        }
    } else {
        // ------------------------------------------------------------ epilogue
        const int q = warp & 3;                  // TMEM lane quarter
        const int ew = warp - EPI_WARP0;         // 0..3
        const int co = 32 * (q & 1) + lane;      // output channel of lanes m and m + 64
        const bool hi_half = q < 2;
        const bool co_ok = co < p.Cout;
        const float bias = co_ok ? __ldg(p.b + co) : 0.f;
        const float inv_area = 1.f / (float)(P * P);
        float* xbuf = reinterpret_cast<float*>(smem + L.xbuf);
        float* red = reinterpret_cast<float*>(smem + L.red);
        float acc[IMG] = {0.f, 0.f, 0.f, 0.f};
        int cur_g = -1;
        // One atomic add per image for this CTA's sums of group cur_g.
        auto flush = [&]() {
#pragma unroll
            for (int img = 0; img < IMG; ++img) {
                float v = acc[img];
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
                if (lane == 0) red[ew * IMG + img] = v;
                acc[img] = 0.f;
            }
            asm volatile("bar.sync 1, 128;\n" ::: "memory");
            if (ew == 0 && lane < IMG && cur_g >= 0) {
                const int n = IMG * cur_g + lane;
                const float v = (red[lane] + red[IMG + lane]) + (red[2 * IMG + lane] + red[3 * IMG + lane]);
                if (n < p.N) atomicAdd(p.out + n, v);
            }
            asm volatile("bar.sync 1, 128;\n" ::: "memory");
        };
        bool ok = true;
        Unit ut = decode(p, u0);
        for (long long u = u0; u < u1; ++u, next_unit(p, ut)) {
            const Unit t = ut;
            const long long i = u - u0;
            const int abuf = (int)(i & 1);
            // One thread waits (bounded); the barrier makes the abort decision the
            // same for all four warps, which meet at named barriers below.
            if (ew == 0 && lane == 0) {
                *epi_ok = (not_stalled(4, u) &&
                           wait_bounded(bar_acc_full + 8 * abuf, (uint32_t)((i >> 1) & 1), abort_flag, p.wait_ns))
                              ? 1u : 0u;
            }
            asm volatile("bar.sync 1, 128;\n" ::: "memory");
            if (!*epi_ok) {
                ok = false;
                break;
            }
            tc_fence_after();  // TMEM loads after the MMAs the waiting thread saw complete
            if (MODE != kTap && t.g != cur_g) {
                if (cur_g >= 0) flush();
                cur_g = t.g;
            }
            const uint32_t taddr = tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(abuf * G::NMMA);
#pragma unroll 1
            for (int k = 0; k < G::NCHK; ++k) {
                uint32_t v[32];
                tmem_ld32(taddr + (uint32_t)(32 * k), v);
                tc::tmem_wait_ld();
                if (k == G::NCHK - 1) {
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(bar_acc_empty + 8 * abuf);  // accumulator free for the MMA
                }
                // Columns 4 * c + i of the chunk: conv column c (0..7), image i.
                float pv[G::V];
#pragma unroll
                for (int w = 0; w < 8 / P; ++w) {
#pragma unroll
                    for (int img = 0; img < IMG; ++img) {
                        float s = 0.f;
#pragma unroll
                        for (int dc = 0; dc < P; ++dc) s += __uint_as_float(v[4 * (P * w + dc) + img]);
                        pv[w * IMG + img] = s;
                    }
                }
                // Each warp pair finishes half of the chunk's pooled values: the hi
                // warps values [0, V/2), the lo warps [V/2, V).  Each writes its
                // partial sums of the other half to shared memory, then adds the
                // partner's partial sums of its own half.
                constexpr int HV = G::V / 2;
                const int mine = hi_half ? 0 : HV, theirs = hi_half ? HV : 0;
                float* xb = xbuf + ((k & 1) * CO_BLK + co) * G::XP;
                if constexpr (HV % 4 == 0) {
#pragma unroll
                    for (int e = 0; e < HV; e += 4)
                        *reinterpret_cast<float4*>(xb + theirs + e) =
                            make_float4(pv[theirs + e], pv[theirs + e + 1], pv[theirs + e + 2], pv[theirs + e + 3]);
                } else {
#pragma unroll
                    for (int e = 0; e < HV; e += 2)
                        *reinterpret_cast<float2*>(xb + theirs + e) = make_float2(pv[theirs + e], pv[theirs + e + 1]);
                }
                asm volatile("bar.sync 1, 128;\n" ::: "memory");
                // the partner's sums of this half, read as 16- or 8-byte vectors
                // (lanes XP floats apart: conflict-free, like the stores)
                float part[HV];
                if constexpr (HV % 4 == 0) {
#pragma unroll
                    for (int e = 0; e < HV; e += 4) {
                        const float4 o = *reinterpret_cast<const float4*>(xb + mine + e);
                        part[e] = o.x; part[e + 1] = o.y; part[e + 2] = o.z; part[e + 3] = o.w;
                    }
                } else {
#pragma unroll
                    for (int e = 0; e < HV; e += 2) {
                        const float2 o = *reinterpret_cast<const float2*>(xb + mine + e);
                        part[e] = o.x; part[e + 1] = o.y;
                    }
                }
#pragma unroll
                for (int e = 0; e < HV; ++e) {
                    const int v = mine + e;           // value index = window * 4 + image
                    const int w = v / IMG, img = v % IMG;
                    const int pwx = t.ct * G::WPT + k * (8 / P) + w;
                    const int n = IMG * t.g + img;
                    if (!co_ok || pwx >= p.PW || n >= p.N) continue;
                    const float pooled = (pv[v] + part[e]) * inv_area + bias;
                    if (MODE == kTap) {
                        p.out[(((size_t)n * p.Cout_total + p.co0 + co) * p.PH + t.ph) * p.PW + pwx] = pooled;
                    } else {
                        acc[img] += __fdividef(1.f, 1.f + __expf(-pooled));  // sigmoid; 0 once exp overflows
                    }
                }
            }
        }
        if (MODE != kTap && ok && cur_g >= 0) flush();
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == MMA_WARP) {
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tmem), "r"(G::TMEM_COLS)
                     : "memory");
    }
}

}  // namespace c2s

// Shapes the shifted-operand tensor-core conv2d covers: Cin <= 16, pool 1, 2,
// 4 or 8 and a 16-byte aligned x (TMA boxes, or 16-byte cp.async copies of
// whole aligned spans when W % 4 != 0); any Cout (launches of up to 64 output
// channels), any H, W and N.
inline bool conv2d_tcs_supported(int Cin, int P, const void* x)
{
    return Cin >= 1 && Cin <= c2s::CIN_MAX && (P == 1 || P == 2 || P == 4 || P == 8) &&
           (reinterpret_cast<uintptr_t>(x) & 15) == 0;
}

template <int P, int CCH, int MODE>
inline int launch_conv2d_tcs_inst(const c2s::Params& prm, int grid, const CUtensorMap& map, cudaStream_t stream)
{
    constexpr uint32_t smem = c2s::smem_bytes<P, CCH>();
    static_assert(smem <= (uint32_t)c2s::SMEM_LIMIT, "shared memory budget");
    auto kern = c2s::conv2d_tcs_kernel<P, CCH, MODE>;
    return launch_cached(kern, (int)smem, [&] { kern<<<grid, c2s::NTHREADS, smem, stream>>>(prm, map); });
}

template <int P, int MODE>
inline int launch_conv2d_tcs_p(const c2s::Params& prm, int CCH, int grid, const CUtensorMap& map,
                               cudaStream_t stream)
{
    return CCH == 1 ? launch_conv2d_tcs_inst<P, 1, MODE>(prm, grid, map, stream)
                    : launch_conv2d_tcs_inst<P, 2, MODE>(prm, grid, map, stream);
}

#ifndef FCV_TCS_BLOCK_ROWS
#define FCV_TCS_BLOCK_ROWS 8
#endif
// Pooled rows per block of the shifted-operand kernel's unit walk.
constexpr int kConv2dTcsBlockRows = FCV_TCS_BLOCK_ROWS;

// MODE: kSumAtomic (out[N], zeroed by the caller) or kTap (pooled values).
// One launch per block of 64 output channels; wait_ns bounds the main-loop
// waits of every launch.
template <int MODE>
inline int launch_conv2d_tcs(const float* x, const float* w, const float* b, int N, int Cin, int H, int W, int Cout,
                             int P, int PH, int PW, float* out, cudaStream_t stream,
                             unsigned long long wait_ns = tc::kWaitLimitNs, int stall_role = 0, int stall_at = 0)
{
    if (!conv2d_tcs_supported(Cin, P, x)) return FCV_ERR_UNSUPPORTED;
    const int CCH = Cin <= 8 ? 1 : 2;
    const int ncol = CCH == 1 ? c2s::Geo<1, 1>::NCOL : c2s::Geo<1, 2>::NCOL;
    c2s::Params prm;
    prm.x = x; prm.out = out;
    prm.N = N; prm.Cin = Cin; prm.H = H; prm.W = W;
    prm.Cout_total = Cout;
    prm.PH = PH; prm.PW = PW;
    const int wpt = ncol / P;
    prm.CT = (PW + wpt - 1) / wpt;
    const long long groups = (N + c2s::IMG - 1) / c2s::IMG;
    prm.U = groups * prm.CT * PH;
    prm.x_elems = (long long)N * Cin * H * W;
    prm.PHB = kConv2dTcsBlockRows;
    prm.wait_ns = wait_ns;
    prm.stall_role = stall_role;
    prm.stall_at = stall_at;
    // x [N][Cin][H][W] as a 4-D tensor with dimensions ordered (column, image,
    // channel, row), so that one box -- one input row of a group: NCOL + 8
    // columns x 4 images x 8 * CCH channels -- lands as [channel][image][column].
    // Needs 16-byte row strides (W % 4 == 0) and an aligned x; otherwise
    // cp.async stages it.
    CUtensorMap map;
    memset(&map, 0, sizeof(map));
    prm.use_tma = 0;
    if ((W & 3) == 0) {
        auto encode = tensor_map_encoder();
        if (!encode) return FCV_ERR_CUDA;
        const cuuint64_t gdim[4] = {(cuuint64_t)W, (cuuint64_t)N, (cuuint64_t)Cin, (cuuint64_t)H};
        const cuuint64_t gstride[3] = {(cuuint64_t)Cin * H * W * 4, (cuuint64_t)H * W * 4, (cuuint64_t)W * 4};
        const cuuint32_t box[4] = {(cuuint32_t)(ncol + 8), (cuuint32_t)c2s::IMG, (cuuint32_t)(8 * CCH), 1};
        const cuuint32_t estride[4] = {1, 1, 1, 1};
        if (encode(&map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, const_cast<float*>(x), gdim, gstride, box, estride,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return FCV_ERR_CUDA;
        prm.use_tma = 1;
    }
    int sms = 0;
    if (device_sm_count(&sms) != FCV_OK) return FCV_ERR_CUDA;
    const int grid = (int)(prm.U < sms ? prm.U : sms);
    for (int co0 = 0; co0 < Cout; co0 += c2s::CO_BLK) {
        prm.co0 = co0;
        prm.Cout = Cout - co0 < c2s::CO_BLK ? Cout - co0 : c2s::CO_BLK;
        prm.w = w + (size_t)co0 * Cin * 9;
        prm.b = b + co0;
        int st = FCV_OK;
        switch (P) {
        case 1: st = launch_conv2d_tcs_p<1, MODE>(prm, CCH, grid, map, stream); break;
        case 2: st = launch_conv2d_tcs_p<2, MODE>(prm, CCH, grid, map, stream); break;
        case 4: st = launch_conv2d_tcs_p<4, MODE>(prm, CCH, grid, map, stream); break;
        default: st = launch_conv2d_tcs_p<8, MODE>(prm, CCH, grid, map, stream); break;
        }
        if (st != FCV_OK) return st;
    }
    return FCV_OK;
}

}  // namespace fcv
