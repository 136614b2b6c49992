// conv1d_tc.cuh -- op B with the pointwise contraction on tcgen05 tensor cores
// through an fp32-accurate 3xTF32 split.
//
// What it computes (POPCORNBENCH trace "Kimi-K2.6__l2_p7", tile-GEMM
// formulation): for every output tile, the depthwise result d[t, c] of a chunk
// of channels is formed on chip and fed straight into the pointwise
// contraction out[t, o] += sum_c d[t, c] * pw[o, c] -- a dense GEMM per batch
// item with M = time, N = output channels, K = input channels.  The trace
// planned mma.sync with TF32 operands and judged plain TF32 (10-bit mantissa)
// too coarse for atol = rtol = 1e-4 (its precision discussion); here each fp32
// operand v is split as hi = round_tf32(v), lo = v - hi, and
//     d * pw ~= d_hi*pw_hi + d_hi*pw_lo + d_lo*pw_hi,
// dropping only d_lo*pw_lo (relative size ~2^-22), accumulated in fp32 in
// tensor memory (the error-corrected TF32 scheme of Ootomo & Yokota, 2022).
// hi is rounded to nearest (ties away from zero) with two integer operations.
//
// B200 design (one CTA per SM, persistent over tiles of 128 times x 256
// output channels, K stepped in chunks of 32 channels = one 128-byte row):
//   * warp 13 (TMA): as soon as a stage is free, one thread loads the raw
//     pw chunk (256 output channels x 32 channels) with a 2-D TMA copy
//     straight into the stage's B_hi buffer; the copy lands in the K-major,
//     128B-swizzled layout the MMA reads.
//   * warps 0-7 (producers): split that pw chunk in place into TF32 hi/lo
//     (B_hi, B_lo); stage the input halo x[n, c0:c0+32, t0-p : ...] in shared
//     memory, compute the depthwise tile with FP32 FMA (4 times x 4 channels
//     per thread from a 16-sample register window; the depthwise weights of
//     all channels stay resident) and write its hi/lo split as the A operand.
//     The halo loads of the next chunk are in flight while the current chunk
//     is computed.
//   * warp 8: allocates 512 TMEM columns (two 128 x 256 fp32 accumulators);
//     one thread issues 12 tcgen05.mma (kind::tf32, M=128, N=256, K=8) per
//     chunk and commits them to the stage's "empty" barrier and, after the
//     last chunk of a tile, to the accumulator's "full" barrier.
//   * warps 9-12 (epilogue): drain one accumulator with tcgen05.ld while the
//     MMAs fill the other, add the bias, transpose 4x4 blocks inside lane
//     quads and store 16 bytes of consecutive times per lane (one warp store
//     covers 128 contiguous bytes in each of 4 output rows).
//   * Every wait is bounded: a wait that runs out sets a CTA abort flag and
//     the device error word, every role then leaves its loop, outstanding
//     MMAs are drained (bounded) and TMEM is freed before the CTA exits.
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>

#include "common.cuh"

namespace fcv {
namespace tc {

constexpr int TM = 128;        // times per tile (UMMA M)
constexpr int TN = 256;        // output channels per tile (UMMA N)
constexpr int KC = 32;         // channels per chunk: one 128-byte fp32 row
constexpr int STAGES = 2;
constexpr int NPROD = 256;     // producer threads, warps 0..7
constexpr int MMA_WARP = 8;
constexpr int TMA_WARP = 13;
constexpr int NTHREADS = 14 * 32;
constexpr int KMAXW = 13;      // largest depthwise kernel (stride 1) of the register window
constexpr int XW_MAX = TM - 1 + KMAXW;  // 140 halo samples per channel at most
constexpr int XU = (XW_MAX + 31) / 32;  // halo samples per lane per channel
constexpr int XWP = 144;       // halo row pitch in floats (multiple of 8)
constexpr int XPP = 2 * XWP;   // pitch of an interleaved channel-pair row
constexpr int XS_FLOATS = KC * XWP + 28;  // 16 pair rows + skew of 4 floats per group of 4 channels
constexpr int DW_MAX = 4000;   // resident depthwise weights: K * round_up(C, 4) at most
constexpr uint32_t TMEM_COLS = 2 * TN;

constexpr uint32_t A_BYTES = TM * KC * 4;    // 16 KB
constexpr uint32_t B_BYTES = TN * KC * 4;    // 32 KB
constexpr uint32_t STAGE_BYTES = 2 * A_BYTES + 2 * B_BYTES;  // A_hi | A_lo | B_hi | B_lo
constexpr uint32_t OFF_XS = STAGES * STAGE_BYTES;
constexpr uint32_t OFF_DWS = OFF_XS + XS_FLOATS * 4;
constexpr uint32_t OFF_BAR = (OFF_DWS + DW_MAX * 4 + 7) & ~7u;
constexpr uint32_t NBAR = 11;  // full[2] empty[2] afull[2] aempty[2] drain tma[2]
constexpr uint32_t OFF_MISC = OFF_BAR + NBAR * 8;
constexpr uint32_t SMEM_USED = OFF_MISC + 16;
constexpr uint32_t SMEM_BYTES = SMEM_USED + 1024;  // slack to align the base to 1024 B

static_assert(XU * 32 >= XW_MAX, "halo prefetch too small");
static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");
static_assert(XWP >= XW_MAX && XWP % 8 == 0, "halo pitch");

// Upper bound on any single wait.  Waits normally last microseconds.
constexpr unsigned long long kWaitLimitNs = 500ull * 1000ull * 1000ull;

// Instruction descriptor: D fp32, A/B tf32, both K-major, N = TN, M = TM.
constexpr uint32_t kIdesc = (1u << 4) | (2u << 7) | (2u << 10) | ((uint32_t)(TN >> 3) << 17) |
                            ((uint32_t)(TM >> 4) << 24);

__device__ __forceinline__ uint32_t smem_u32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(bar) : "memory");
}

__device__ __forceinline__ unsigned long long globaltimer()
{
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;\n" : "=l"(t));
    return t;
}

// Wait for the phase of `bar` with parity `parity`.  Returns false (without
// completing the wait) once the CTA abort flag is set, or after kWaitLimitNs,
// in which case it sets the abort flag and the device error word itself.
__device__ __forceinline__ bool wait_bounded(uint32_t bar, uint32_t parity, volatile uint32_t* abort_flag,
                                             unsigned long long limit_ns = kWaitLimitNs)
{
    if (mbar_try_wait(bar, parity)) return true;
    const unsigned long long t0 = globaltimer();
    for (uint32_t i = 1;; ++i) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((i & 255u) == 0) {
            if (*abort_flag) return false;
            if (globaltimer() - t0 > limit_ns) {
                *abort_flag = 1u;
                record_device_error(kErrTimeout);
                return false;
            }
        }
    }
}

// Self-test of the failure path: one thread waits, with the given limit, on an
// mbarrier that nothing will ever complete.  The wait must give up, set the
// device error word and return; the kernel then exits normally.
__global__ void selftest_wait_timeout_kernel(unsigned long long limit_ns)
{
    __shared__ __align__(8) unsigned long long bar;
    __shared__ uint32_t abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(smem_u32(&bar), 1);
        abort_flag = 0u;
        asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
    }
    __syncthreads();
    if (threadIdx.x == 0) (void)wait_bounded(smem_u32(&bar), 0, &abort_flag, limit_ns);
    __syncthreads();
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory"); }

__device__ __forceinline__ void tc_commit(uint32_t bar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n" ::"r"(bar)
                 : "memory");
}

__device__ __forceinline__ void tc_mma_tf32(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t accumulate)
{
    asm volatile(
        "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
        " tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n}\n" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(kIdesc), "r"(accumulate)
        : "memory");
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16])
{
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
        "%14, %15}, [%16];\n"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
}

__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;\n" ::: "memory"); }

// tcgen05.wait::ld that also names the 16 registers of the load it completes,
// so no use of them can be scheduled above the wait.
__device__ __forceinline__ void tmem_wait_ld16(uint32_t (&r)[16])
{
    asm volatile("tcgen05.wait::ld.sync.aligned;\n"
                 : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
                   "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]),
                   "+r"(r[15])
                 :
                 : "memory");
}

// Shared-memory descriptor of a K-major operand in the canonical 128-byte
// swizzle layout: rows of 128 B, 8-row groups 1024 B apart.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr)
{
    return (uint64_t)((saddr & 0x3FFFFu) >> 4) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
           ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

// Byte offset of the 16-byte chunk `ch` (0..7) of row `row` in a 128B-swizzled tile.
__device__ __forceinline__ uint32_t sw128_off(int row, int ch)
{
    return (uint32_t)((row >> 3) * 1024 + (row & 7) * 128 + ((ch ^ (row & 7)) << 4));
}

// Round an fp32 value to the nearest TF32 value (10 explicit mantissa bits),
// ties away from zero: add half of the 13 dropped bits to the magnitude bits
// and clear them.  A mantissa carry propagates into the exponent as it should.
// Exact for every finite input whose rounded magnitude stays finite.
__device__ __forceinline__ float tf32_round(float v)
{
    return __uint_as_float((__float_as_uint(v) + 0x1000u) & 0xFFFFE000u);
}

// v = hi + lo with hi the TF32 rounding of v; lo = v - hi is exact in fp32 and
// |lo| <= 2^-11 |v|, so dropping lo's bits below TF32 precision costs at most
// 2^-21 |v|.
__device__ __forceinline__ void split4(const float4 v, float4& hi, float4& lo)
{
    hi.x = tf32_round(v.x); lo.x = v.x - hi.x;
    hi.y = tf32_round(v.y); lo.y = v.y - hi.y;
    hi.z = tf32_round(v.z); lo.z = v.z - hi.z;
    hi.w = tf32_round(v.w); lo.w = v.w - hi.w;
}

__device__ __forceinline__ void sts128(uint32_t addr, float4 v)
{
    asm volatile("st.shared.v4.f32 [%0], {%1, %2, %3, %4};\n" ::"r"(addr), "f"(v.x), "f"(v.y), "f"(v.z), "f"(v.w)
                 : "memory");
}

__device__ __forceinline__ float4 lds128(uint32_t addr)
{
    float4 v;
    asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];\n" : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(addr)
                 : "memory");
    return v;
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(bar), "r"(bytes) : "memory");
}

// 2-D tiled TMA load (no multicast) completing on `bar`.
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int x0, int x1, uint32_t bar)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];\n" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x0), "r"(x1), "r"(bar)
        : "memory");
}

struct Params {
    const float* x;
    const float* dw;
    const float* pw;
    const float* bias;
    float* out;
    int C, T, O, K, pad, To;
    int tiles_t, tiles_o, total_tiles;
    int out_vec;  // output rows 16-byte aligned (To % 4 == 0, aligned base)
    // Failure-path test (all 0 in normal calls): role stall_role (1 TMA warp,
    // 2 producers, 3 MMA issuer, 4 epilogue) of every CTA waits, before its
    // stall_at-th tile, on a barrier nothing completes, with limit stall_ns.
    int stall_role = 0, stall_at = 0;
    unsigned long long stall_ns = 0;
};

// The failure-path test hook: true unless role `role` is to stall before its
// `local`-th tile and its wait on `gate` (a barrier nothing completes) ran out,
// which also sets the abort flag and the device error word.  gate == 0: the
// kernel has no gate.
__device__ __forceinline__ bool stall_ok(const Params& p, int role, int local, uint32_t gate,
                                         volatile uint32_t* abort_flag)
{
    if (gate == 0 || p.stall_role != role || local != p.stall_at) return true;
    return wait_bounded(gate, 0, abort_flag, p.stall_ns);
}

struct TileCoord {
    int n, t0, o0;
};

// Tiles are numbered with time fastest, then output-channel tile, then batch:
// CTAs running at the same moment write neighbouring 512-byte segments of the
// same output rows, and both output-channel tiles of a batch item read its
// input while it is still in L2.
// TN_T: output channels per tile.
template <int TN_T = TN>
__device__ __forceinline__ TileCoord decode_tile(const Params& p, int tile)
{
    TileCoord tc;
    tc.t0 = (tile % p.tiles_t) * TM;
    const int rest = tile / p.tiles_t;
    tc.o0 = (rest % p.tiles_o) * TN_T;
    tc.n = rest / p.tiles_o;
    return tc;
}

// 4x4 transpose across the 4 lanes of a quad: lane j holds row j (x0..x3) on
// entry and column j on exit.  Two butterfly stages of xor-shuffles.
__device__ __forceinline__ void quad_transpose(float& x0, float& x1, float& x2, float& x3, int j)
{
    const bool b1 = (j & 2) != 0, b0 = (j & 1) != 0;
    float s0 = b1 ? x0 : x2, s1 = b1 ? x1 : x3;
    float r0 = __shfl_xor_sync(0xffffffffu, s0, 2), r1 = __shfl_xor_sync(0xffffffffu, s1, 2);
    if (b1) { x0 = r0; x1 = r1; } else { x2 = r0; x3 = r1; }
    s0 = b0 ? x0 : x1;
    s1 = b0 ? x2 : x3;
    r0 = __shfl_xor_sync(0xffffffffu, s0, 1);
    r1 = __shfl_xor_sync(0xffffffffu, s1, 1);
    if (b0) { x0 = r0; x2 = r1; } else { x1 = r0; x3 = r1; }
}

// Single-thread MMA issuer: for every tile, wait until its accumulator buffer
// is drained; for every chunk, wait until the producers filled the stage, issue
// the 12 MMAs of the 3xTF32 split (K = 8 each) and commit them to the stage's
// "empty" barrier; after the last chunk commit to the accumulator's "full"
// barrier.  Finally drain every MMA issued (bounded) so TMEM can be freed.
__device__ __forceinline__ void mma_issuer(const Params& p, uint32_t tmem, uint32_t sbase, uint32_t bar_full,
                                           uint32_t bar_empty, uint32_t bar_afull, uint32_t bar_aempty,
                                           uint32_t bar_drain, volatile uint32_t* abort_flag, int nk,
                                           uint32_t gate = 0)
{
    int seq = 0, local = 0;
    bool ok = true;
    for (int tile = blockIdx.x; ok && tile < p.total_tiles; tile += gridDim.x, ++local) {
        const int buf = local & 1;
        if (!stall_ok(p, 3, local, gate, abort_flag)) break;
        if (!wait_bounded(bar_aempty + 8 * buf, ((local >> 1) & 1) ^ 1, abort_flag)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem + (uint32_t)(buf * TN);
        for (int k = 0; k < nk; ++k, ++seq) {
            const int stage = seq & 1;
            if (!wait_bounded(bar_full + 8 * stage, (seq >> 1) & 1, abort_flag)) {
                ok = false;
                break;
            }
            tc_fence_after();
            const uint32_t a_hi = sbase + stage * STAGE_BYTES;
            const uint32_t a_lo = a_hi + A_BYTES;
            const uint32_t b_hi = a_lo + A_BYTES;
            const uint32_t b_lo = b_hi + B_BYTES;
#pragma unroll
            for (int kk = 0; kk < KC / 8; ++kk) {
                const uint32_t koff = 32u * kk;
                const uint64_t dah = sw128_desc(a_hi + koff), dal = sw128_desc(a_lo + koff);
                const uint64_t dbh = sw128_desc(b_hi + koff), dbl = sw128_desc(b_lo + koff);
                tc_mma_tf32(d_tmem, dah, dbh, (k > 0 || kk > 0) ? 1u : 0u);
                tc_mma_tf32(d_tmem, dah, dbl, 1u);
                tc_mma_tf32(d_tmem, dal, dbh, 1u);
            }
            tc_commit(bar_empty + 8 * stage);  // stage free once these MMAs have read it
        }
        if (ok) tc_commit(bar_afull + 8 * buf);  // accumulator complete
    }
    // Drain: every MMA this thread issued has completed before TMEM is freed.
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

// One epilogue warp: drains its 32 TMEM lanes of each finished accumulator
// (TN_E columns, buffer b at column b * TN_E), adds the bias and stores the
// tile's outputs, then frees the buffer.
template <int TN_E = TN>
__device__ __forceinline__ void epilogue_warp(const Params& p, uint32_t tmem, uint32_t bar_afull,
                                              uint32_t bar_aempty, volatile uint32_t* abort_flag, int warp,
                                              int lane, uint32_t gate = 0)
{
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    int local = 0;
    for (int tile = blockIdx.x; tile < p.total_tiles; tile += gridDim.x, ++local) {
        const int buf = local & 1;
        int ok = 1;
        if (lane == 0)
            ok = (stall_ok(p, 4, local, gate, abort_flag) &&
                  wait_bounded(bar_afull + 8 * buf, (local >> 1) & 1, abort_flag)) ? 1 : 0;
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
        tc_fence_after();
        const TileCoord tcd = decode_tile<TN_E>(p, tile);
        const int tw = tcd.t0 + 32 * q;  // first time of this warp's 32 TMEM lanes
        const uint32_t taddr = tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(buf * TN_E);
        // Fast path: all 32 times in range and 16-byte aligned rows.  After a
        // 4x4 transpose inside each lane quad, lane 4k+j holds times
        // tw+4k .. tw+4k+3 of output channels 4j .. 4j+3 (of the 16 loaded), so
        // each 16-byte store instruction covers 128 contiguous bytes of 4 rows.
        const bool vec = tw + 32 <= p.To && p.out_vec;
        const int kq = lane >> 2, jq = lane & 3;
        auto bias_of = [&](int o) { return (p.bias && o < p.O) ? __ldg(p.bias + o) : 0.f; };
        // Blocks of 16 columns, two at a time: their eight 4x4 transposes are
        // independent, so their shuffles overlap.  The bias is added after the
        // transpose, where a lane's four values belong to one output channel.
        auto store_pair = [&](int cb, const uint32_t (&ra)[16], const uint32_t (&rb)[16]) {
            if (vec) {
                float x[2][4][4];
                float bv[2][4];
#pragma unroll
                for (int h = 0; h < 2; ++h)
#pragma unroll
                    for (int m = 0; m < 4; ++m) {
                        const uint32_t(&r)[16] = h ? rb : ra;
                        x[h][m][0] = __uint_as_float(r[m]);
                        x[h][m][1] = __uint_as_float(r[4 + m]);
                        x[h][m][2] = __uint_as_float(r[8 + m]);
                        x[h][m][3] = __uint_as_float(r[12 + m]);
                        bv[h][m] = bias_of(tcd.o0 + (cb + h) * 16 + 4 * jq + m);
                    }
#pragma unroll
                for (int h = 0; h < 2; ++h)
#pragma unroll
                    for (int m = 0; m < 4; ++m) quad_transpose(x[h][m][0], x[h][m][1], x[h][m][2], x[h][m][3], jq);
#pragma unroll
                for (int h = 0; h < 2; ++h)
#pragma unroll
                    for (int m = 0; m < 4; ++m) {
                        // rows = the 4 lanes' times, one output channel per lane
                        const int o = tcd.o0 + (cb + h) * 16 + 4 * jq + m;
                        if (o < p.O) {
                            float* dst = p.out + ((size_t)tcd.n * p.O + o) * p.To + tw + 4 * kq;
                            const float b = bv[h][m];
                            __stcs(reinterpret_cast<float4*>(dst),
                                   make_float4(x[h][m][0] + b, x[h][m][1] + b, x[h][m][2] + b, x[h][m][3] + b));
                        }
                    }
            } else {
                const int t = tw + lane;
                float* out_nt = p.out + (size_t)tcd.n * p.O * p.To + t;
#pragma unroll
                for (int h = 0; h < 2; ++h)
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        const int o = tcd.o0 + (cb + h) * 16 + j;
                        if (t < p.To && o < p.O) out_nt[(size_t)o * p.To] = __uint_as_float((h ? rb : ra)[j]) + bias_of(o);
                    }
            }
        };
        constexpr int NB = TN_E / 16;
        static_assert(NB % 2 == 0, "blocks come in pairs");
#pragma unroll 1
        for (int cb = 0; cb < NB; cb += 2) {
            uint32_t ra[16], rb[16];
            tmem_ld16(taddr + (uint32_t)(cb * 16), ra);
            tmem_ld16(taddr + (uint32_t)((cb + 1) * 16), rb);
            tmem_wait_ld16(ra);
            tmem_wait_ld16(rb);
            store_pair(cb, ra, rb);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar_aempty + 8 * buf);
    }
}

// KT: the depthwise kernel size when known at compile time, 0 for any K <= KMAXW.
template <int KT>
__global__ void __launch_bounds__(NTHREADS, 1)
dwsep_conv1d_tc_kernel(const Params p, const __grid_constant__ CUtensorMap pw_map)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    const uint32_t sbase = smem_u32(smem);
    float* xs = reinterpret_cast<float*>(smem + OFF_XS);
    float* dws = reinterpret_cast<float*>(smem + OFF_DWS);
    const uint32_t bar_full = sbase + OFF_BAR;       // + 8 * stage
    const uint32_t bar_empty = bar_full + 16;        // + 8 * stage
    const uint32_t bar_afull = bar_full + 32;        // + 8 * buf
    const uint32_t bar_aempty = bar_full + 48;       // + 8 * buf
    const uint32_t bar_drain = bar_full + 64;
    const uint32_t bar_tma = bar_full + 72;          // + 8 * stage
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + OFF_MISC);
    volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(smem + OFF_MISC + 4);
    volatile uint32_t* prod_abort = reinterpret_cast<volatile uint32_t*>(smem + OFF_MISC + 8);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int i = 0; i < 2; ++i) {
            mbar_init(bar_full + 8 * i, 8);    // one arrival per producer warp
            mbar_init(bar_empty + 8 * i, 1);   // tcgen05.commit
            mbar_init(bar_afull + 8 * i, 1);   // tcgen05.commit
            mbar_init(bar_aempty + 8 * i, 4);  // one arrival per epilogue warp
        }
        mbar_init(bar_drain, 1);
        mbar_init(bar_tma, 1);       // expect_tx arrival + TMA bytes
        mbar_init(bar_tma + 8, 1);
        *abort_flag = 0u;
        *prod_abort = 0u;
        asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
    }
    if (warp == MMA_WARP) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(smem_u32(tmem_holder)),
                     "r"(TMEM_COLS)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;

    const int nk = (p.C + KC - 1) / KC;

    // Depthwise weights of every channel stay resident, transposed to [K][CP]
    // (CP = C rounded up to 4, zero-padded) so one 16-byte load serves the 4
    // channels a thread computes.
    const int CP = (p.C + 3) & ~3;
    for (int e = threadIdx.x; e < p.K * CP; e += NTHREADS) {
        const int k = e / CP, c = e - (e / CP) * CP;
        dws[e] = c < p.C ? __ldg(p.dw + (size_t)c * p.K + k) : 0.f;
    }
    __syncthreads();

    if (warp < 8) {
        // ------------------------------------------------------------ producers
        const int ptid = threadIdx.x;
        const int cg = lane & 7;               // depthwise: channel group of 4
        const int tq = (lane >> 3) + 4 * warp; // depthwise: times 4*tq .. 4*tq+3
        const int K = KT > 0 ? KT : p.K;
        float xr[4][XU];   // halo of channels 4*warp .. 4*warp+3, samples lane + 32*u
        TileCoord ft = {0, 0, 0};
        auto fetch = [&](int kc) {
            const int c0 = kc * KC;
            const int tb = ft.t0 - p.pad;
            const bool interior = tb >= 0 && tb + 32 * XU <= p.T && c0 + KC <= p.C;
            const float* xw = p.x + ((size_t)ft.n * p.C + c0 + 4 * warp) * p.T + tb + lane;
            if (interior) {
#pragma unroll
                for (int i = 0; i < 4; ++i)
#pragma unroll
                    for (int u = 0; u < XU; ++u) xr[i][u] = __ldg(xw + (size_t)i * p.T + 32 * u);
            } else {
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const bool cok = c0 + 4 * warp + i < p.C;
#pragma unroll
                    for (int u = 0; u < XU; ++u) {
                        const int ti = tb + lane + 32 * u;
                        xr[i][u] = (cok && ti >= 0 && ti < p.T) ? __ldg(xw + (size_t)i * p.T + 32 * u) : 0.f;
                    }
                }
            }
        };

        int seq = 0;
        int tile = blockIdx.x, kc = 0;
        if (tile < p.total_tiles) {
            ft = decode_tile(p, tile);
            fetch(kc);
        }
        while (tile < p.total_tiles) {
            const int stage = seq & 1;
            const uint32_t parity = (seq >> 1) & 1;
            // The TMA of this stage's pw chunk has landed (so the stage is free as well).
            if (ptid == 0 && !wait_bounded(bar_tma + 8 * stage, parity, abort_flag)) *prod_abort = 1u;
            asm volatile("bar.sync 1, 256;\n" ::: "memory");
            if (*prod_abort) break;
            // Thread 0 saw this phase complete, so this returns at once; it gives
            // every producer its own acquire of the TMA bytes.
            for (int spin = 0; !mbar_try_wait(bar_tma + 8 * stage, parity) && spin < (1 << 20); ++spin) {
            }

            const uint32_t a_hi = sbase + stage * STAGE_BYTES;
            const uint32_t a_lo = a_hi + A_BYTES;
            const uint32_t b_hi = a_lo + A_BYTES;
            const uint32_t b_lo = b_hi + B_BYTES;
            const int c0 = kc * KC;

            // Halo of this chunk into shared memory, channel pairs interleaved:
            // xs[(c/2)*XPP + skew + 2*j + (c&1)], skewed by 4 floats per group of 4
            // channels, so the packed depthwise reads both channels of a pair at once.
#pragma unroll
            for (int i = 0; i < 4; i += 2) {
                const int cl = 4 * warp + i;
                float* dst = xs + (cl >> 1) * XPP + 4 * ((cl >> 2) & 7);
#pragma unroll
                for (int u = 0; u < XU; ++u) {
                    const int j = lane + 32 * u;
                    if (j < XWP) *reinterpret_cast<float2*>(dst + 2 * j) = make_float2(xr[i][u], xr[i + 1][u]);
                }
            }
            // pw chunk (raw fp32, as the TMA left it in B_hi), split in place into TF32 hi/lo.
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int row = warp * 32 + i * 4 + (lane >> 3);
                const uint32_t off = sw128_off(row, lane & 7);
                float4 hi, lo;
                split4(lds128(b_hi + off), hi, lo);
                sts128(b_hi + off, hi);
                sts128(b_lo + off, lo);
            }
            asm volatile("bar.sync 1, 256;\n" ::: "memory");  // halo visible to every producer

            // Issue the global loads of the next chunk now; they land while this one is computed.
            if (++kc == nk) {
                kc = 0;
                tile += gridDim.x;
                if (tile < p.total_tiles) ft = decode_tile(p, tile);
            }
            if (tile < p.total_tiles) fetch(kc);

            // Depthwise tile: 4 times x 4 channels per thread, then the TF32 split as the A operand.
            // Depthwise tile: 4 times x 4 channels per thread as two channel pairs,
            // each tap one packed fma.rn.f32x2 per time (both channels of a pair).
            float2 d2[2][4];
#pragma unroll
            for (int h = 0; h < 2; ++h)
#pragma unroll
                for (int r = 0; r < 4; ++r) d2[h][r] = make_float2(0.f, 0.f);
            if (c0 + 4 * cg < p.C) {  // channels past C stay zero (their weights are zero-padded too)
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int pr = 2 * cg + h;  // pair row: channels 4*cg + 2*h, +1
                    const float* xrow = xs + pr * XPP + 4 * cg + 8 * tq;
                    float2 win[16];
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        const float4 v = *reinterpret_cast<const float4*>(xrow + 4 * q);
                        win[2 * q] = make_float2(v.x, v.y);
                        win[2 * q + 1] = make_float2(v.z, v.w);
                    }
                    const float* wcol = dws + c0 + 4 * cg + 2 * h;
                    auto tap = [&](int k) {
                        const float2 wk = *reinterpret_cast<const float2*>(wcol + k * CP);
#pragma unroll
                        for (int r = 0; r < 4; ++r) d2[h][r] = __ffma2_rn(win[k + r], wk, d2[h][r]);
                    };
                    if constexpr (KT > 0) {
#pragma unroll
                        for (int k = 0; k < KT; ++k) tap(k);
                    } else {
#pragma unroll
                        for (int k = 0; k < KMAXW; ++k)
                            if (k < K) tap(k);
                    }
                }
            }
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                const int t = 4 * tq + r;
                float4 hi, lo;
                split4(make_float4(d2[0][r].x, d2[0][r].y, d2[1][r].x, d2[1][r].y), hi, lo);
                const uint32_t off = sw128_off(t, cg);
                sts128(a_hi + off, hi);
                sts128(a_lo + off, lo);
            }
            // Make the generic-proxy writes visible to the tensor core, then signal the stage full.
            asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
            __syncwarp();
            if (lane == 0) mbar_arrive(bar_full + 8 * stage);
            ++seq;
        }
    } else if (warp == MMA_WARP) {
        // ---------------------------------------------------------- MMA issuer
        if (lane == 0)
            mma_issuer(p, tmem, sbase, bar_full, bar_empty, bar_afull, bar_aempty, bar_drain, abort_flag, nk);
        __syncwarp();
    } else if (warp == TMA_WARP) {
        // -------------------------------------------------------- TMA issuer
        if (lane == 0) {
            int seq = 0;
            bool pending[2] = {false, false};
            bool ok = true;
            for (int tile = blockIdx.x; ok && tile < p.total_tiles; tile += gridDim.x) {
                const TileCoord tcd = decode_tile(p, tile);
                for (int k = 0; k < nk; ++k, ++seq) {
                    const int stage = seq & 1;
                    if (!wait_bounded(bar_empty + 8 * stage, ((seq >> 1) & 1) ^ 1, abort_flag)) {
                        ok = false;
                        break;
                    }
                    pending[stage] = false;  // the producers consumed its previous load before the MMA ran
                    mbar_arrive_expect_tx(bar_tma + 8 * stage, B_BYTES);
                    tma_load_2d(sbase + stage * STAGE_BYTES + 2 * A_BYTES, &pw_map, k * KC, tcd.o0,
                                bar_tma + 8 * stage);
                    pending[stage] = true;
                }
            }
            // Wait (bounded) for copies still in flight before the CTA can exit,
            // also when another role gave up and they were never consumed
            // (normally they have all landed and this returns at once).
            {
                for (int st = 0; st < 2; ++st) {
                    if (!pending[st]) continue;
                    const int last = seq - 1 - ((seq - 1 - st) & 1);  // latest sequence number on this stage
                    const unsigned long long t0 = globaltimer();
                    while (last >= 0 && !mbar_try_wait(bar_tma + 8 * st, (last >> 1) & 1)) {
                        if (globaltimer() - t0 > kWaitLimitNs) break;
                    }
                }
            }
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ epilogue
        epilogue_warp(p, tmem, bar_afull, bar_aempty, abort_flag, warp, lane);
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == MMA_WARP) {
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tmem), "r"(TMEM_COLS)
                     : "memory");
    }
}

}  // namespace tc

// Shapes the tensor-core path covers: stride 1 and a depthwise kernel that
// fits the 16-sample register window.  Others take the FP32-FMA path.
inline bool conv1d_tc_supported(int C, int O, int K, int stride, const void* pw = nullptr)
{
    // C % 4 == 0 and a 16-byte aligned pw: the TMA copy of pw needs 16-byte row strides.
    return stride == 1 && K >= 1 && K <= tc::KMAXW && C >= 1 && O >= 1 && (C & 3) == 0 &&
           (reinterpret_cast<uintptr_t>(pw) & 15) == 0 && (long long)C * K <= tc::DW_MAX;
}

// cuTensorMapEncodeTiled, resolved once through the runtime (no libcuda link).
inline PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            f = nullptr;
        return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
    }();
    return fn;
}

inline int launch_dwsep_conv1d_tc(const float* x, const float* dw, const float* pw, const float* bias, int N,
                                  int C, int T, int O, int K, int stride, int pad, int To, float* out,
                                  cudaStream_t stream)
{
    (void)stride;
    tc::Params prm;
    prm.x = x; prm.dw = dw; prm.pw = pw; prm.bias = bias; prm.out = out;
    prm.C = C; prm.T = T; prm.O = O; prm.K = K; prm.pad = pad; prm.To = To;
    prm.tiles_t = (To + tc::TM - 1) / tc::TM;
    prm.tiles_o = (O + tc::TN - 1) / tc::TN;
    const long long total = (long long)N * prm.tiles_t * prm.tiles_o;
    if (total > 0x7fffffffLL) return FCV_ERR_UNSUPPORTED;
    prm.total_tiles = (int)total;
    prm.out_vec = ((To & 3) == 0 && (reinterpret_cast<uintptr_t>(out) & 15) == 0) ? 1 : 0;

    // pw [O][C] as a 2-D tensor: inner dim C (contiguous), outer dim O; one box
    // is 32 channels x 256 output channels, 128B-swizzled; out-of-range rows
    // and columns read as zero.
    auto encode = tensor_map_encoder();
    if (!encode) return FCV_ERR_CUDA;
    CUtensorMap map;
    const cuuint64_t gdim[2] = {(cuuint64_t)C, (cuuint64_t)O};
    const cuuint64_t gstride[1] = {(cuuint64_t)C * sizeof(float)};
    const cuuint32_t box[2] = {(cuuint32_t)tc::KC, (cuuint32_t)tc::TN};
    const cuuint32_t estride[2] = {1, 1};
    if (encode(&map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float*>(pw), gdim, gstride, box, estride,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return FCV_ERR_CUDA;

    int sms = 0;
    if (device_sm_count(&sms) != FCV_OK) return FCV_ERR_CUDA;
    auto kern = K == 9 ? tc::dwsep_conv1d_tc_kernel<9>
              : K == 3 ? tc::dwsep_conv1d_tc_kernel<3> : tc::dwsep_conv1d_tc_kernel<0>;
    const int grid = (int)(total < sms ? total : sms);
    return launch_cached(kern, (int)tc::SMEM_BYTES,
                         [&] { kern<<<grid, tc::NTHREADS, tc::SMEM_BYTES, stream>>>(prm, map); });
}

}  // namespace fcv
