// conv1d_tcx.cuh -- op B on tcgen05 tensor cores with the input halo staged by TMA.
//
// Same contraction, tiling, 3xTF32 split, MMA issuer and epilogue as the
// kernel in conv1d_tc.cuh (POPCORNBENCH trace "Kimi-K2.6__l2_p7", tile-GEMM
// formulation: depthwise tile on chip, pointwise contraction as a GEMM with
// M = time, N = output channels, K = input channels).  What changes is how the
// producers feed the A operand, because that kernel is bound by the shared
// memory pipe, not by the tensor cores: per 32-channel chunk its producers
// spent ~2,000 shared-memory wavefronts (halo stores, 4-fold redundant window
// reads) next to the 1,152 the MMAs themselves read.
//
//   * The TMA warp loads, next to the pw chunk, the input halo of the chunk
//     x[n, c0:c0+32, t0-pad-r : +148] as one 3-D box (time x channel x batch)
//     into the stage's A region, which the producers overwrite with the A
//     operand only after reading it.  Out-of-range times (the zero padding)
//     and channels read as zero, so there is no edge code at all.
//   * Producer thread = one channel (lane) x 16 consecutive times (warp): it
//     reads its window once (16 + K - 1 samples as 16-byte loads; the 148-float
//     row pitch makes a quarter-warp's loads hit distinct banks), runs the K
//     taps with packed FMA over time pairs, and writes its 16 A values as
//     32-bit stores that fill one 128-byte row per warp instruction.
//   * The pw operand's hi part is the raw fp32 chunk itself (the tensor core
//     ignores the 13 low mantissa bits); only lo = v - truncate(v) is written.
//   * r = (t0*s - pad) mod 4 (the same for every tile) keeps the box's first
//     time on a 16-byte boundary, as TMA requires; it is a template parameter
//     so the window indexing stays in registers.
//   * Stride s = 2 (the op's stride argument; output t reads x[2t + k - pad]):
//     a 128-output tile spans up to 2*127 + K + r = 270 input samples, more
//     than one TMA box can hold (256 per dimension), so the halo comes as two
//     boxes of 140 samples, the first into the A region, the second into the
//     B_lo region; the producers then write B_lo only after the barrier that
//     follows their window reads.  A thread's window covers 2*15 + K samples.
//
// Requirements beyond the register-staged kernel: stride 1 or 2, T % 4 == 0
// and a 16-byte aligned x (the TMA map's row strides are T*4 and C*T*4 bytes).
#pragma once

#include "conv1d_tc.cuh"

namespace fcv {
namespace tcx {

using namespace tc;

constexpr int XW = 148;                                     // halo box width = smem row pitch (floats), stride 1
constexpr uint32_t X_BYTES = (uint32_t)XW * KC * 4;         // 18,944 B per chunk
constexpr int XW2 = 140;                                    // stride 2: two boxes of this width (row pitch)
constexpr uint32_t X2_BYTES = (uint32_t)XW2 * KC * 4;       // 17,920 B per box
constexpr int DWX_MAX = 8192;                               // resident depthwise weights, [K][32*nk]

// Geometry per output-channel tile width TN_ (the UMMA N): 256 (two 96 KB
// stages) or 128 (three 64 KB stages; for O <= 128, where half of a 256-wide
// tile would be zero).  A stage is A_hi | A_lo | B_lo | B_hi: the halo boxes
// land from its start (stride 1: one box in the A region; stride 2: two boxes
// over the A and B_lo regions), never over B_hi, which the TMA fills at once.
template <int TN_>
struct Geo {
    static constexpr int TN = TN_;
    static constexpr int STAGES = TN_ == 256 ? 2 : 3;
    static constexpr uint32_t B_BYTES = (uint32_t)TN_ * KC * 4;
    static constexpr uint32_t OFF_BLO = 2 * A_BYTES;
    static constexpr uint32_t OFF_BHI = 2 * A_BYTES + B_BYTES;
    static constexpr uint32_t STAGE_BYTES = 2 * A_BYTES + 2 * B_BYTES;
    static constexpr uint32_t OFF_DWS = STAGES * STAGE_BYTES;
    static constexpr uint32_t OFF_BAR = OFF_DWS + DWX_MAX * 4;
    static constexpr uint32_t NBAR = 3 * STAGES + 6;  // full, empty, tma per stage; afull[2] aempty[2] drain gate
    static constexpr uint32_t OFF_MISC = OFF_BAR + NBAR * 8;
    static constexpr uint32_t SMEM_BYTES = OFF_MISC + 16 + 1024;  // slack to align the base to 1024 B
    static constexpr uint32_t TMEM_COLS = 2 * TN_;
    // Instruction descriptor: D fp32, A/B tf32, both K-major, N = TN, M = TM.
    static constexpr uint32_t IDESC = (1u << 4) | (2u << 7) | (2u << 10) | ((uint32_t)(TN_ >> 3) << 17) |
                                      ((uint32_t)(TM >> 4) << 24);
    static_assert(TN_ == 256 || TN_ == 128, "tile widths");
    static_assert(X_BYTES <= 2 * A_BYTES, "the stride-1 halo box must fit the stage's A region");
    static_assert(2 * X2_BYTES <= OFF_BHI, "the stride-2 halo boxes must stay below B_hi");
    static_assert(OFF_BHI % 1024 == 0 && STAGE_BYTES % 1024 == 0, "128B-swizzled operands on 1024-byte boundaries");
    static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");
};
static_assert((XW2 * 4) % 16 == 0 && XW2 % 4 == 0, "second stride-2 box starts 16-byte aligned");
static_assert((XW * 4) % 16 == 0, "TMA box inner extent must be a multiple of 16 bytes");

// 3-D tiled TMA load (no multicast) completing on `bar`.
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* map, int x0, int x1, int x2,
                                            uint32_t bar)
{
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], "
        "[%5];\n" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x0), "r"(x1), "r"(x2), "r"(bar)
        : "memory");
}

// Prefetch of one 3-D box into L2 (a hint: nothing waits for it).
__device__ __forceinline__ void tma_prefetch_3d(const CUtensorMap* map, int x0, int x1, int x2)
{
    asm volatile("cp.async.bulk.prefetch.tensor.3d.L2.global [%0, {%1, %2, %3}];\n" ::"l"(
                     reinterpret_cast<uint64_t>(map)),
                 "r"(x0), "r"(x1), "r"(x2)
                 : "memory");
}

// v - truncate_tf32(v) per component: the part of v below the TF32 mantissa, exact in fp32.
__device__ __forceinline__ float4 tf32_trunc_rest4(const float4 v)
{
    auto rest = [](float a) { return a - __uint_as_float(__float_as_uint(a) & 0xFFFFE000u); };
    return make_float4(rest(v.x), rest(v.y), rest(v.z), rest(v.w));
}

__device__ __forceinline__ void sts32(uint32_t addr, float v)
{
    asm volatile("st.shared.f32 [%0], %1;\n" ::"r"(addr), "f"(v) : "memory");
}

// tcgen05.mma kind::tf32 with the instruction descriptor as a parameter.
__device__ __forceinline__ void mma_tf32_id(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                            uint32_t accumulate)
{
    asm volatile(
        "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
        " tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n}\n" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Single-thread MMA issuer (the register-halo kernel's protocol, for G's
// stage count, stage layout and N): per tile wait until its accumulator buffer
// is drained; per chunk wait until the producers filled the stage, issue its
// 12 MMAs (4 K-steps x A_hi.B_hi + A_hi.B_lo + A_lo.B_hi) and commit them to
// the stage's "empty" barrier; after the last chunk commit "afull".  Finally
// drain every MMA issued (bounded) so TMEM can be freed.
template <class G>
__device__ __forceinline__ void mma_issuer_g(const Params& p, uint32_t tmem, uint32_t sbase, uint32_t bar_full,
                                             uint32_t bar_empty, uint32_t bar_afull, uint32_t bar_aempty,
                                             uint32_t bar_drain, volatile uint32_t* abort_flag, int nk, uint32_t gate)
{
    int seq = 0, local = 0;
    bool ok = true;
    for (int tile = blockIdx.x; ok && tile < p.total_tiles; tile += gridDim.x, ++local) {
        const int buf = local & 1;
        if (!stall_ok(p, 3, local, gate, abort_flag)) break;
        if (!wait_bounded(bar_aempty + 8 * buf, ((local >> 1) & 1) ^ 1, abort_flag)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem + (uint32_t)(buf * G::TN);
        for (int k = 0; k < nk; ++k, ++seq) {
            const int stage = seq % G::STAGES;
            if (!wait_bounded(bar_full + 8 * stage, (seq / G::STAGES) & 1, abort_flag)) {
                ok = false;
                break;
            }
            tc_fence_after();
            const uint32_t a_hi = sbase + stage * G::STAGE_BYTES;
            const uint32_t a_lo = a_hi + A_BYTES;
            const uint32_t b_lo = a_hi + G::OFF_BLO;
            const uint32_t b_hi = a_hi + G::OFF_BHI;
#pragma unroll
            for (int kk = 0; kk < KC / 8; ++kk) {
                const uint32_t koff = 32u * kk;
                const uint64_t dah = sw128_desc(a_hi + koff), dal = sw128_desc(a_lo + koff);
                const uint64_t dbh = sw128_desc(b_hi + koff), dbl = sw128_desc(b_lo + koff);
                mma_tf32_id(d_tmem, dah, dbh, G::IDESC, (k > 0 || kk > 0) ? 1u : 0u);
                mma_tf32_id(d_tmem, dah, dbl, G::IDESC, 1u);
                mma_tf32_id(d_tmem, dal, dbh, G::IDESC, 1u);
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

// KT: depthwise kernel size when fixed at compile time (0: any K <= KMAXW).
// R: (t0*S - pad) mod 4, the offset of the first needed sample inside the box.
// S: the stride, 1 or 2.  TN_: output channels per tile, 256 or 128.
template <int KT, int R, int S, int TN_>
__global__ void __launch_bounds__(NTHREADS, 1)
dwsep_conv1d_tcx_kernel(const Params p, const __grid_constant__ CUtensorMap pw_map,
                        const __grid_constant__ CUtensorMap x_map)
{
    using G = Geo<TN_>;
    constexpr int NS = G::STAGES;
    static_assert(S == 1 || S == 2, "stride 1 or 2");
    constexpr int KW = KT > 0 ? KT : KMAXW;              // taps the window must cover
    constexpr int NV = (R + S * 15 + KW + 3) / 4;        // 16-byte window loads per thread
    constexpr int PITCH = S == 1 ? XW : XW2;             // halo row pitch (floats)
    static_assert(S == 2 || 16 * 7 + 4 * NV <= XW, "window inside the halo box");
    static_assert(S == 1 || 32 * 7 + 4 * NV <= 2 * XW2, "window inside the two halo boxes");

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    const uint32_t sbase = smem_u32(smem);
    float* dws = reinterpret_cast<float*>(smem + G::OFF_DWS);
    const uint32_t bar_full = sbase + G::OFF_BAR;    // + 8 * stage
    const uint32_t bar_empty = bar_full + 8 * NS;    // + 8 * stage
    const uint32_t bar_tma = bar_full + 16 * NS;     // + 8 * stage
    const uint32_t bar_afull = bar_full + 24 * NS;   // + 8 * buf
    const uint32_t bar_aempty = bar_afull + 16;      // + 8 * buf
    const uint32_t bar_drain = bar_afull + 32;
    const uint32_t bar_gate = bar_afull + 40;        // never completed (failure-path test)
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + G::OFF_MISC);
    volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(smem + G::OFF_MISC + 4);
    volatile uint32_t* prod_abort = reinterpret_cast<volatile uint32_t*>(smem + G::OFF_MISC + 8);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int i = 0; i < NS; ++i) {
            mbar_init(bar_full + 8 * i, 8);    // one arrival per producer warp
            mbar_init(bar_empty + 8 * i, 1);   // tcgen05.commit
            mbar_init(bar_tma + 8 * i, 1);     // expect_tx arrival + TMA bytes
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(bar_afull + 8 * i, 1);   // tcgen05.commit
            mbar_init(bar_aempty + 8 * i, 4);  // one arrival per epilogue warp
        }
        mbar_init(bar_drain, 1);
        mbar_init(bar_gate, 1);
        *abort_flag = 0u;
        *prod_abort = 0u;
        asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
    }
    if (warp == MMA_WARP) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(smem_u32(tmem_holder)),
                     "r"(G::TMEM_COLS)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::: "memory");
    }

    const int nk = (p.C + KC - 1) / KC;
    // Depthwise weights of every channel stay resident, transposed to [K][CW]
    // with CW = 32 * nk (zero beyond C), so lane c of chunk kc reads its tap k
    // at dws[k * CW + 32 * kc + c]: 32 consecutive floats per warp load.
    const int CW = KC * nk;
    for (int e = threadIdx.x; e < p.K * CW; e += NTHREADS) {
        const int k = e / CW, c = e - (e / CW) * CW;
        dws[e] = c < p.C ? __ldg(p.dw + (size_t)c * p.K + k) : 0.f;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;

    if (warp < 8) {
        // ------------------------------------------------------------ producers
        const int ptid = threadIdx.x;
        const int K = KT > 0 ? KT : p.K;
        int seq = 0, local = 0;
        bool run = true;
        for (int tile = blockIdx.x; run && tile < p.total_tiles; tile += gridDim.x, ++local) {
            for (int kc = 0; kc < nk; ++kc, ++seq) {
                const int stage = seq % NS;
                const uint32_t parity = (seq / NS) & 1;
                if (ptid == 0 && kc == 0 && !stall_ok(p, 2, local, bar_gate, abort_flag)) *prod_abort = 1u;
                // The TMA copies of this stage (pw chunk and halo) have landed.
                if (ptid == 0 && !*prod_abort && !wait_bounded(bar_tma + 8 * stage, parity, abort_flag))
                    *prod_abort = 1u;
                asm volatile("bar.sync 1, 256;\n" ::: "memory");
                if (*prod_abort) {
                    run = false;
                    break;
                }
                // Thread 0 saw this phase complete, so this returns at once; it gives
                // every producer its own acquire of the TMA bytes.
                for (int spin = 0; !mbar_try_wait(bar_tma + 8 * stage, parity) && spin < (1 << 20); ++spin) {
                }

                const uint32_t a_hi = sbase + stage * G::STAGE_BYTES;
                const uint32_t a_lo = a_hi + A_BYTES;
                const uint32_t b_lo = a_hi + G::OFF_BLO;
                const uint32_t b_hi = a_hi + G::OFF_BHI;

                // pw chunk: B_hi stays the raw fp32 the TMA wrote, because the MMA
                // reads only the TF32 bits of an fp32 operand (the 13 low mantissa
                // bits are ignored, i.e. hi = truncate(v)); B_lo = v - truncate(v)
                // is exact and |B_lo| < 2^-10 |v|.  This saves the in-place rewrite.
                // At stride 2 the second halo box occupies the B_lo region, so
                // B_lo is written after the barrier below.
                auto split_pw = [&]() {
#pragma unroll
                    for (int i = 0; i < G::TN / 32; ++i) {
                        const int row = warp * (G::TN / 8) + i * 4 + (lane >> 3);
                        const uint32_t off = sw128_off(row, lane & 7);
                        sts128(b_lo + off, tf32_trunc_rest4(lds128(b_hi + off)));
                    }
                };
                if constexpr (S == 1) split_pw();

                // Depthwise: channel lane, times 16*warp .. 16*warp+15 of the tile.
                // Sample j of the halo is x[t0*S - pad - R + j]; output time
                // 16*warp + i takes samples S*(16*warp + i) + R + k, k < K.  At
                // stride 2, samples j >= XW2 sit in the second box (B_lo region).
                const float* xs0 = reinterpret_cast<const float*>(smem + stage * G::STAGE_BYTES) + lane * PITCH;
                const float* xs1 = xs0 + KC * XW2;  // the second stride-2 box follows the first
                float win[4 * NV];
#pragma unroll
                for (int q = 0; q < NV; ++q) {
                    const int j = S * 16 * warp + 4 * q;
                    const float* src = (S == 1 || j < XW2) ? xs0 + j : xs1 + (j - XW2);
                    const float4 v = *reinterpret_cast<const float4*>(src);
                    win[4 * q] = v.x;
                    win[4 * q + 1] = v.y;
                    win[4 * q + 2] = v.z;
                    win[4 * q + 3] = v.w;
                }
                float2 d2[8];
#pragma unroll
                for (int j = 0; j < 8; ++j) d2[j] = make_float2(0.f, 0.f);
                const float* wcol = dws + KC * kc + lane;
#pragma unroll
                for (int k = 0; k < KW; ++k) {
                    if (KT > 0 || k < K) {
                        const float w = wcol[k * CW];
                        const float2 w2 = make_float2(w, w);
#pragma unroll
                        for (int j = 0; j < 8; ++j)
                            d2[j] = __ffma2_rn(make_float2(win[R + 2 * S * j + k], win[R + 2 * S * j + S + k]), w2,
                                               d2[j]);
                    }
                }
                // Every producer has read its halo window before the A operand (and,
                // at stride 2, B_lo) overwrites it.
                asm volatile("bar.sync 1, 256;\n" ::: "memory");
                if constexpr (S == 2) split_pw();

                // A operand: row t = 16*warp + i, column = channel lane; one warp
                // store fills one 128-byte swizzled row.
                const uint32_t col = ((uint32_t)(lane & 3) << 2);
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const float v = (i & 1) ? d2[i >> 1].y : d2[i >> 1].x;
                    const float hi = tf32_round(v);
                    const uint32_t off = sw128_off(16 * warp + i, lane >> 2) + col;
                    sts32(a_hi + off, hi);
                    sts32(a_lo + off, v - hi);
                }
                // Make the generic-proxy writes visible to the tensor core, then signal the stage full.
                asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
                __syncwarp();
                if (lane == 0) mbar_arrive(bar_full + 8 * stage);
            }
        }
    } else if (warp == MMA_WARP) {
        // ---------------------------------------------------------- MMA issuer
        if (lane == 0)
            mma_issuer_g<G>(p, tmem, sbase, bar_full, bar_empty, bar_afull, bar_aempty, bar_drain, abort_flag, nk,
                            bar_gate);
        __syncwarp();
    } else if (warp == TMA_WARP) {
        // -------------------------------------------------------- TMA issuer
        if (lane == 0) {
            int seq = 0;
            bool pending[NS] = {};
            bool ok = true;
            int local = 0;
            for (int tile = blockIdx.x; ok && tile < p.total_tiles; tile += gridDim.x, ++local) {
                if (!stall_ok(p, 1, local, bar_gate, abort_flag)) break;
                const TileCoord tcd = decode_tile<TN_>(p, tile);
                const int x0 = tcd.t0 * S - p.pad - R;  // a multiple of 4: 16-byte aligned time coordinate
                // Pull the next tile's halo boxes into L2 now, so its TMA loads
                // wait on L2 rather than on DRAM latency.
                if (tile + (int)gridDim.x < p.total_tiles) {
                    const TileCoord nx = decode_tile<TN_>(p, tile + gridDim.x);
                    for (int k = 0; k < nk; ++k) {
                        tma_prefetch_3d(&x_map, nx.t0 * S - p.pad - R, k * KC, nx.n);
                        if (S == 2) tma_prefetch_3d(&x_map, nx.t0 * S - p.pad - R + XW2, k * KC, nx.n);
                    }
                }
                for (int k = 0; k < nk; ++k, ++seq) {
                    const int stage = seq % NS;
                    if (!wait_bounded(bar_empty + 8 * stage, ((seq / NS) & 1) ^ 1, abort_flag)) {
                        ok = false;
                        break;
                    }
                    pending[stage] = false;  // the producers consumed its previous loads before the MMA ran
                    const uint32_t st = sbase + stage * G::STAGE_BYTES;
                    mbar_arrive_expect_tx(bar_tma + 8 * stage, G::B_BYTES + (S == 1 ? X_BYTES : 2 * X2_BYTES));
                    tma_load_2d(st + G::OFF_BHI, &pw_map, k * KC, tcd.o0, bar_tma + 8 * stage);
                    tma_load_3d(st, &x_map, x0, k * KC, tcd.n, bar_tma + 8 * stage);
                    if (S == 2) tma_load_3d(st + X2_BYTES, &x_map, x0 + XW2, k * KC, tcd.n, bar_tma + 8 * stage);
                    pending[stage] = true;
                }
            }
            // Wait (bounded) for copies still in flight before the CTA can exit,
            // also when another role gave up and they were never consumed
            // (normally they have all landed and this returns at once).
            {
                for (int st = 0; st < NS; ++st) {
                    if (!pending[st]) continue;
                    const int last = seq - 1 - ((seq - 1 - st) % NS);  // latest sequence number on this stage
                    const unsigned long long t0 = globaltimer();
                    while (last >= 0 && !mbar_try_wait(bar_tma + 8 * st, (last / NS) & 1)) {
                        if (globaltimer() - t0 > kWaitLimitNs) break;
                    }
                }
            }
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ epilogue
        epilogue_warp<TN_>(p, tmem, bar_afull, bar_aempty, abort_flag, warp, lane, bar_gate);
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == MMA_WARP) {
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tmem), "r"(G::TMEM_COLS)
                     : "memory");
    }
}

}  // namespace tcx

// Shapes the TMA-halo tensor-core kernel covers.
inline bool conv1d_tcx_supported(int C, int T, int O, int K, int stride, const void* x, const void* pw)
{
    const long long cw = (long long)tc::KC * ((C + tc::KC - 1) / tc::KC);
    return (stride == 1 || stride == 2) && K >= 1 && K <= tc::KMAXW && C >= 1 && O >= 1 && T >= 1 && (C & 3) == 0 &&
           (T & 3) == 0 && (reinterpret_cast<uintptr_t>(x) & 15) == 0 &&
           (reinterpret_cast<uintptr_t>(pw) & 15) == 0 && cw * K <= tcx::DWX_MAX;
}

namespace tcx {
using KernelPtr = void (*)(const tc::Params, const CUtensorMap, const CUtensorMap);

// The instance for (K, r, stride) at tile width TN_: K = 9 with r = 0 and K = 3
// with r = 3 (the pages' kernel sizes with pad K/2) have their taps unrolled
// at 256 columns; every other K runs the generic K <= 13 loop.
template <int TN_>
inline KernelPtr select_kernel(int K, int r, int stride)
{
    if (stride == 1) {
        if constexpr (TN_ == 256) {
            if (K == 9 && r == 0) return dwsep_conv1d_tcx_kernel<9, 0, 1, TN_>;
            if (K == 3 && r == 3) return dwsep_conv1d_tcx_kernel<3, 3, 1, TN_>;
        }
        if (r == 0) return dwsep_conv1d_tcx_kernel<0, 0, 1, TN_>;
        if (r == 1) return dwsep_conv1d_tcx_kernel<0, 1, 1, TN_>;
        if (r == 2) return dwsep_conv1d_tcx_kernel<0, 2, 1, TN_>;
        return dwsep_conv1d_tcx_kernel<0, 3, 1, TN_>;
    }
    if constexpr (TN_ == 256) {
        if (K == 9 && r == 0) return dwsep_conv1d_tcx_kernel<9, 0, 2, TN_>;
        if (K == 3 && r == 3) return dwsep_conv1d_tcx_kernel<3, 3, 2, TN_>;
    }
    if (r == 0) return dwsep_conv1d_tcx_kernel<0, 0, 2, TN_>;
    if (r == 1) return dwsep_conv1d_tcx_kernel<0, 1, 2, TN_>;
    if (r == 2) return dwsep_conv1d_tcx_kernel<0, 2, 2, TN_>;
    return dwsep_conv1d_tcx_kernel<0, 3, 2, TN_>;
}
}  // namespace tcx

// Output channels per tile of the TMA-halo kernel: 128 when O fits in one such
// tile (a 256-wide tile would be half zero), else 256.
inline int conv1d_tcx_tile_n(int O) { return O <= 128 ? 128 : 256; }

inline int launch_dwsep_conv1d_tcx(const float* x, const float* dw, const float* pw, const float* bias, int N,
                                   int C, int T, int O, int K, int stride, int pad, int To, float* out,
                                   cudaStream_t stream, int stall_role = 0, int stall_at = 0,
                                   unsigned long long stall_ns = 0)
{
    const int tn = conv1d_tcx_tile_n(O);
    tc::Params prm;
    prm.stall_role = stall_role;
    prm.stall_at = stall_at;
    prm.stall_ns = stall_ns;
    prm.x = x; prm.dw = dw; prm.pw = pw; prm.bias = bias; prm.out = out;
    prm.C = C; prm.T = T; prm.O = O; prm.K = K; prm.pad = pad; prm.To = To;
    prm.tiles_t = (To + tc::TM - 1) / tc::TM;
    prm.tiles_o = (O + tn - 1) / tn;
    const long long total = (long long)N * prm.tiles_t * prm.tiles_o;
    if (total > 0x7fffffffLL) return FCV_ERR_UNSUPPORTED;
    prm.total_tiles = (int)total;
    prm.out_vec = ((To & 3) == 0 && (reinterpret_cast<uintptr_t>(out) & 15) == 0) ? 1 : 0;

    auto encode = tensor_map_encoder();
    if (!encode) return FCV_ERR_CUDA;
    // pw [O][C]: 32 channels x tn output channels per box, 128B-swizzled.
    CUtensorMap pw_map, x_map;
    {
        const cuuint64_t gdim[2] = {(cuuint64_t)C, (cuuint64_t)O};
        const cuuint64_t gstride[1] = {(cuuint64_t)C * sizeof(float)};
        const cuuint32_t box[2] = {(cuuint32_t)tc::KC, (cuuint32_t)tn};
        const cuuint32_t estride[2] = {1, 1};
        if (encode(&pw_map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float*>(pw), gdim, gstride, box, estride,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return FCV_ERR_CUDA;
    }
    // x [N][C][T]: 148 (stride 2: 140) times x 32 channels x 1 batch item per
    // box, rows packed (no swizzle); times and channels outside the tensor read
    // as zero.
    {
        const cuuint64_t gdim[3] = {(cuuint64_t)T, (cuuint64_t)C, (cuuint64_t)N};
        const cuuint64_t gstride[2] = {(cuuint64_t)T * sizeof(float), (cuuint64_t)C * T * sizeof(float)};
        const cuuint32_t box[3] = {(cuuint32_t)(stride == 1 ? tcx::XW : tcx::XW2), (cuuint32_t)tc::KC, 1};
        const cuuint32_t estride[3] = {1, 1, 1};
        if (encode(&x_map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<float*>(x), gdim, gstride, box, estride,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return FCV_ERR_CUDA;
    }

    int sms = 0;
    if (device_sm_count(&sms) != FCV_OK) return FCV_ERR_CUDA;
    const int r = (-pad) & 3;  // (t0*stride - pad) mod 4 with t0 a multiple of 128
    const tcx::KernelPtr kern = tn == 256 ? tcx::select_kernel<256>(K, r, stride) : tcx::select_kernel<128>(K, r, stride);
    const int smem = (int)(tn == 256 ? tcx::Geo<256>::SMEM_BYTES : tcx::Geo<128>::SMEM_BYTES);
    const int grid = (int)(total < sms ? total : sms);
    return launch_cached(kern, smem, [&] { kern<<<grid, tc::NTHREADS, smem, stream>>>(prm, pw_map, x_map); });
}

}  // namespace fcv
