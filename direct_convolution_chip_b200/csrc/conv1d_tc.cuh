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
// operand v is split as hi = rna_tf32(v), lo = rna_tf32(v - hi), and
//     d * pw ~= d_hi*pw_hi + d_hi*pw_lo + d_lo*pw_hi,
// dropping only d_lo*pw_lo (relative size ~2^-22), accumulated in fp32 in
// tensor memory (the error-corrected TF32 scheme of Ootomo & Yokota, 2022).
//
// B200 design (one CTA per SM, persistent over tiles of 128 times x 256
// output channels, K stepped in chunks of 32 channels = one 128-byte row):
//   * warps 0-7 (producers): stage the input halo x[n, c0:c0+32, t0-p : ...]
//     in shared memory, compute the depthwise tile with FP32 FMA (4 times x 4
//     channels per thread from a 16-sample register window; the depthwise
//     weights of all channels stay resident), split it into TF32 hi/lo and
//     write both as K-major, 128B-swizzled UMMA operands; the pw chunk
//     (256 x 32) is split the same way.  The global loads of the next chunk
//     are in flight while the current chunk is computed.
//   * warp 8: allocates 512 TMEM columns (two 128 x 256 fp32 accumulators);
//     one thread issues 12 tcgen05.mma (kind::tf32, M=128, N=256, K=8) per
//     chunk and commits them to the stage's "empty" barrier and, after the
//     last chunk of a tile, to the accumulator's "full" barrier.
//   * warps 9-12 (epilogue): drain one accumulator with tcgen05.ld while the
//     MMAs fill the other, add the bias and store along t (each warp store
//     covers 32 consecutive times of one output channel: 128 coalesced bytes).
//   * Every wait is bounded: a wait that runs out sets a CTA abort flag and
//     the device error word, every role then leaves its loop, outstanding
//     MMAs are drained (bounded) and TMEM is freed before the CTA exits.
#pragma once

#include "common.cuh"

namespace fcv {
namespace tc {

constexpr int TM = 128;        // times per tile (UMMA M)
constexpr int TN = 256;        // output channels per tile (UMMA N)
constexpr int KC = 32;         // channels per chunk: one 128-byte fp32 row
constexpr int STAGES = 2;
constexpr int NPROD = 256;     // producer threads, warps 0..7
constexpr int MMA_WARP = 8;
constexpr int NTHREADS = 13 * 32;
constexpr int KMAXW = 13;      // largest depthwise kernel (stride 1) of the register window
constexpr int XW_MAX = TM - 1 + KMAXW;  // 140 halo samples per channel at most
constexpr int XU = (XW_MAX + 31) / 32;  // halo samples per lane per channel
constexpr int XWP = 144;       // halo row pitch in floats (multiple of 8)
constexpr int XS_FLOATS = KC * XWP + 28;  // + skew of 4 floats per group of 4 channels
constexpr int DW_MAX = 4000;   // resident depthwise weights: C * K at most
constexpr uint32_t TMEM_COLS = 2 * TN;

constexpr uint32_t A_BYTES = TM * KC * 4;    // 16 KB
constexpr uint32_t B_BYTES = TN * KC * 4;    // 32 KB
constexpr uint32_t STAGE_BYTES = 2 * A_BYTES + 2 * B_BYTES;  // A_hi | A_lo | B_hi | B_lo
constexpr uint32_t OFF_XS = STAGES * STAGE_BYTES;
constexpr uint32_t OFF_DWS = OFF_XS + XS_FLOATS * 4;
constexpr uint32_t OFF_BAR = (OFF_DWS + DW_MAX * 4 + 7) & ~7u;
constexpr uint32_t NBAR = 9;   // full[2] empty[2] afull[2] aempty[2] drain
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
__device__ __forceinline__ bool wait_bounded(uint32_t bar, uint32_t parity, volatile uint32_t* abort_flag)
{
    if (mbar_try_wait(bar, parity)) return true;
    const unsigned long long t0 = globaltimer();
    for (uint32_t i = 1;; ++i) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((i & 255u) == 0) {
            if (*abort_flag) return false;
            if (globaltimer() - t0 > kWaitLimitNs) {
                *abort_flag = 1u;
                record_device_error(kErrTimeout);
                return false;
            }
        }
    }
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

__device__ __forceinline__ float tf32_rna(float v)
{
    uint32_t r;
    asm("cvt.rna.tf32.f32 %0, %1;\n" : "=r"(r) : "f"(v));
    return __uint_as_float(r);
}

__device__ __forceinline__ void split4(const float4 v, float4& hi, float4& lo)
{
    hi.x = tf32_rna(v.x); lo.x = tf32_rna(v.x - hi.x);
    hi.y = tf32_rna(v.y); lo.y = tf32_rna(v.y - hi.y);
    hi.z = tf32_rna(v.z); lo.z = tf32_rna(v.z - hi.z);
    hi.w = tf32_rna(v.w); lo.w = tf32_rna(v.w - hi.w);
}

__device__ __forceinline__ void sts128(uint32_t addr, float4 v)
{
    asm volatile("st.shared.v4.f32 [%0], {%1, %2, %3, %4};\n" ::"r"(addr), "f"(v.x), "f"(v.y), "f"(v.z), "f"(v.w)
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
    int pw_vec;  // pw rows 16-byte aligned (C % 4 == 0, aligned base)
};

struct TileCoord {
    int n, t0, o0;
};

__device__ __forceinline__ TileCoord decode_tile(const Params& p, int tile)
{
    TileCoord tc;
    const int o_tile = tile % p.tiles_o;
    const int rest = tile / p.tiles_o;
    tc.t0 = (rest % p.tiles_t) * TM;
    tc.n = rest / p.tiles_t;
    tc.o0 = o_tile * TN;
    return tc;
}

// KT: the depthwise kernel size when known at compile time, 0 for any K <= KMAXW.
template <int KT>
__global__ void __launch_bounds__(NTHREADS, 1) dwsep_conv1d_tc_kernel(const Params p)
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
    const int XW = TM - 1 + p.K;  // halo samples per channel (stride 1)

    // Depthwise weights of every channel stay resident: [C][K], row pitch K.
    for (int e = threadIdx.x; e < p.C * p.K; e += NTHREADS) dws[e] = __ldg(p.dw + e);
    __syncthreads();

    if (warp < 8) {
        // ------------------------------------------------------------ producers
        const int ptid = threadIdx.x;
        const int cg = lane & 7;               // depthwise: channel group of 4
        const int tq = (lane >> 3) + 4 * warp; // depthwise: times 4*tq .. 4*tq+3
        const int K = KT > 0 ? KT : p.K;
        float xr[4][XU];   // halo of channels 4*warp .. 4*warp+3, samples lane + 32*u
        float4 pr[8];      // pw chunk rows, 16 bytes each

        auto fetch = [&](int tile, int kc) {
            const TileCoord tcd = decode_tile(p, tile);
            const int c0 = kc * KC;
            const int tb = tcd.t0 - p.pad;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int c = c0 + 4 * warp + i;
                const float* xrow = p.x + ((size_t)tcd.n * p.C + (c < p.C ? c : 0)) * p.T;
#pragma unroll
                for (int u = 0; u < XU; ++u) {
                    const int ti = tb + lane + 32 * u;
                    xr[i][u] = (c < p.C && ti >= 0 && ti < p.T) ? __ldg(xrow + ti) : 0.f;
                }
            }
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int row = warp * 32 + i * 4 + (lane >> 3);
                const int o = tcd.o0 + row, c = c0 + 4 * (lane & 7);
                float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
                if (o < p.O) {
                    const float* src = p.pw + (size_t)o * p.C + c;
                    if (p.pw_vec) {
                        if (c < p.C) v = __ldg(reinterpret_cast<const float4*>(src));
                    } else {
                        if (c < p.C) v.x = __ldg(src);
                        if (c + 1 < p.C) v.y = __ldg(src + 1);
                        if (c + 2 < p.C) v.z = __ldg(src + 2);
                        if (c + 3 < p.C) v.w = __ldg(src + 3);
                    }
                }
                pr[i] = v;
            }
        };

        int seq = 0;
        int tile = blockIdx.x, kc = 0;
        if (tile < p.total_tiles) fetch(tile, kc);
        while (tile < p.total_tiles) {
            const int stage = seq & 1;
            const uint32_t parity = ((seq >> 1) & 1) ^ 1;
            if (ptid == 0 && !wait_bounded(bar_empty + 8 * stage, parity, abort_flag)) *prod_abort = 1u;
            asm volatile("bar.sync 1, 256;\n" ::: "memory");
            if (*prod_abort) break;

            const uint32_t a_hi = sbase + stage * STAGE_BYTES;
            const uint32_t a_lo = a_hi + A_BYTES;
            const uint32_t b_hi = a_lo + A_BYTES;
            const uint32_t b_lo = b_hi + B_BYTES;
            const int c0 = kc * KC;

            // Halo of this chunk into shared memory (rows skewed by 4 floats per channel group).
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int cl = 4 * warp + i;
                float* dst = xs + cl * XWP + 4 * ((cl >> 2) & 7);
#pragma unroll
                for (int u = 0; u < XU; ++u) {
                    const int j = lane + 32 * u;
                    if (j < XWP) dst[j] = xr[i][u];
                }
            }
            // pw chunk, split into TF32 hi/lo, as the K-major B operand.
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int row = warp * 32 + i * 4 + (lane >> 3);
                float4 hi, lo;
                split4(pr[i], hi, lo);
                const uint32_t off = sw128_off(row, lane & 7);
                sts128(b_hi + off, hi);
                sts128(b_lo + off, lo);
            }
            asm volatile("bar.sync 1, 256;\n" ::: "memory");  // halo visible to every producer

            // Issue the global loads of the next chunk now; they land while this one is computed.
            if (++kc == nk) {
                kc = 0;
                tile += gridDim.x;
            }
            if (tile < p.total_tiles) fetch(tile, kc);

            // Depthwise tile: 4 times x 4 channels per thread, then the TF32 split as the A operand.
            float dv[4][4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int cl = 4 * cg + i;
                const int c = c0 + cl;
                float d0 = 0.f, d1 = 0.f, d2 = 0.f, d3 = 0.f;
                if (c < p.C) {
                    const float* xrow = xs + cl * XWP + 4 * ((cl >> 2) & 7) + 4 * tq;
                    float win[16];
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const float4 v = *reinterpret_cast<const float4*>(xrow + 4 * q);
                        win[4 * q] = v.x; win[4 * q + 1] = v.y; win[4 * q + 2] = v.z; win[4 * q + 3] = v.w;
                    }
                    const float* wrow = dws + c * K;
                    if constexpr (KT > 0) {
#pragma unroll
                        for (int k = 0; k < KT; ++k) {
                            const float wk = wrow[k];
                            d0 = fmaf(win[k], wk, d0);
                            d1 = fmaf(win[k + 1], wk, d1);
                            d2 = fmaf(win[k + 2], wk, d2);
                            d3 = fmaf(win[k + 3], wk, d3);
                        }
                    } else {
#pragma unroll
                        for (int k = 0; k < KMAXW; ++k) {
                            if (k < K) {
                                const float wk = wrow[k];
                                d0 = fmaf(win[k], wk, d0);
                                d1 = fmaf(win[k + 1], wk, d1);
                                d2 = fmaf(win[k + 2], wk, d2);
                                d3 = fmaf(win[k + 3], wk, d3);
                            }
                        }
                    }
                }
                dv[i][0] = d0; dv[i][1] = d1; dv[i][2] = d2; dv[i][3] = d3;
            }
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                const int t = 4 * tq + r;
                float4 hi, lo;
                split4(make_float4(dv[0][r], dv[1][r], dv[2][r], dv[3][r]), hi, lo);
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
        if (lane == 0) {
            int seq = 0, local = 0;
            bool ok = true;
            for (int tile = blockIdx.x; ok && tile < p.total_tiles; tile += gridDim.x, ++local) {
                const int buf = local & 1;
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
        __syncwarp();
    } else {
        // ------------------------------------------------------------ epilogue
        const int q = warp & 3;  // TMEM lane quarter this warp may access
        int local = 0;
        for (int tile = blockIdx.x; tile < p.total_tiles; tile += gridDim.x, ++local) {
            const int buf = local & 1;
            int ok = 1;
            if (lane == 0) ok = wait_bounded(bar_afull + 8 * buf, (local >> 1) & 1, abort_flag) ? 1 : 0;
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) break;
            tc_fence_after();
            const TileCoord tcd = decode_tile(p, tile);
            const int t = tcd.t0 + 32 * q + lane;
            const bool t_ok = t < p.To;
            float* out_nt = p.out + (size_t)tcd.n * p.O * p.To + t;
            const uint32_t taddr = tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(buf * TN);
#pragma unroll 1
            for (int cb = 0; cb < TN / 16; ++cb) {
                uint32_t r[16];
                tmem_ld16(taddr + (uint32_t)(cb * 16), r);
                tmem_wait_ld();
                const int obase = tcd.o0 + cb * 16;
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    const int o = obase + j;
                    if (t_ok && o < p.O) {
                        const float bo = p.bias ? __ldg(p.bias + o) : 0.f;
                        out_nt[(size_t)o * p.To] = __uint_as_float(r[j]) + bo;
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar_aempty + 8 * buf);
        }
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
inline bool conv1d_tc_supported(int C, int O, int K, int stride)
{
    return stride == 1 && K >= 1 && K <= tc::KMAXW && C >= 1 && O >= 1 && (long long)C * K <= tc::DW_MAX;
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
    prm.pw_vec = ((C & 3) == 0 && (reinterpret_cast<uintptr_t>(pw) & 15) == 0) ? 1 : 0;
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return FCV_ERR_CUDA;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return FCV_ERR_CUDA;
    auto kern = K == 9 ? tc::dwsep_conv1d_tc_kernel<9>
              : K == 3 ? tc::dwsep_conv1d_tc_kernel<3> : tc::dwsep_conv1d_tc_kernel<0>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)tc::SMEM_BYTES) != cudaSuccess)
        return FCV_ERR_CUDA;
    const int grid = (int)(total < sms ? total : sms);
    kern<<<grid, tc::NTHREADS, tc::SMEM_BYTES, stream>>>(prm);
    return launch_status();
}

}  // namespace fcv
