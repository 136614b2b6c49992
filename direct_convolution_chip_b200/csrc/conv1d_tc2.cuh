// conv1d_tc2.cuh -- op B on a pair of SMs: the 2-CTA (cta_group::2) form of
// the tensor-core separable conv1d with the input halo staged by TMA.
//
// Same arithmetic as conv1d_tcx.cuh (depthwise on FP32 FMA into the A operand,
// pointwise as a 3xTF32 tcgen05 contraction with the pw hi part read raw,
// fp32 accumulation in TMEM).  What changes is the tiling: the two CTAs of a
// cluster compute one 256-time x 256-output-channel tile with
// tcgen05.mma.cta_group::2 (M = 256, N = 256, K = 8), at stride 1 or 2 (the
// stride-2 halo in two TMA boxes, as in the single-SM kernel).  Each CTA holds its own
// 128 rows of A (its times) and HALF of B (128 of the 256 pw rows), so per CTA
// the pw split work, the B stage and the MMA's shared-memory reads are halved,
// and three 64 KB stages fit where the single-SM kernel has two of 96 KB: the
// extra stage hides the TMA latency that bounds the single-SM pipeline.
//
// Roles per CTA (512 threads): warps 0-7 produce (depthwise from the
// TMA-staged halo, A split); warp 8 allocates TMEM (both CTAs) and, in the
// leader CTA only, one thread issues the MMAs for the pair; warps 9-12 drain
// this CTA's accumulator rows; warp 13 loads, per chunk, this CTA's half of
// the pw chunk and its input halo by TMA; warps 14-15 form the pw lo part
// beside the producers (taking that pass off the depthwise warps shortens
// their per-chunk chain; sixteen depthwise warps of 8 times each, or two
// groups of eight on alternate chunks, measured slower: the shared-memory
// data path, which the MMAs' operand reads also use, sets the pace, not the
// warps' latency).  The leader's "full" collects its own 10 producer and
// split warps and one forwarded arrival per chunk from the other CTA, whose
// warps arrive locally and whose warp-8 lane 0 relays
// (a cluster-scope release per producer warp cost ~1,600 cycles on the
// producers' path); the leader's "aempty" collects both CTAs' epilogues
// (remote arrives).  The producers stage the depthwise weights after the
// opening cluster barrier, so the TMA warp starts at once, and help drain the
// pair's last tile, which has no successor to overlap its drain with.  MMA completion is committed to both CTAs' "empty"/"afull"
// barriers with a multicast commit.  Every mbarrier wait is bounded and also
// watches the peer CTA's abort flag, so the pair gives up together; a cluster
// barrier follows initialisation and precedes exit, so no CTA leaves while
// its peer may still signal it.  No TMA multicast.
#pragma once

#include "conv1d_tcx.cuh"

namespace fcv {
namespace tc2 {

using tc::TileCoord;

constexpr int TM = 128;          // times per CTA (pair: 256)
constexpr int TN = 256;          // output channels per pair tile (UMMA N)
constexpr int TNH = TN / 2;      // pw rows held by each CTA
constexpr int KC = 32;
constexpr int STAGES = 3;
constexpr int NPW = 8;                  // depthwise producer warps
constexpr int TPW = TM / NPW;                // times per producer warp
constexpr int MMA_WARP = NPW, TMA_WARP = NPW + 5;
constexpr int SPLIT_WARP = NPW + 6, NSPLIT = 2;  // warps that form B_lo
constexpr int NTHREADS = (SPLIT_WARP + NSPLIT) * 32;
constexpr int FULL_ARRIVALS = NPW + NSPLIT;  // per CTA and chunk: producer and split warps
static_assert(TPW % 4 == 0 && TPW * NPW == TM, "16-byte window loads cover the CTA's times");
constexpr int KMAXW = tc::KMAXW;
constexpr int XW = 148;          // halo box width = smem row pitch (floats), stride 1
constexpr uint32_t X_BYTES = (uint32_t)XW * KC * 4;
constexpr int XW2 = tcx::XW2;    // stride 2: two boxes of this width
constexpr uint32_t X2_BYTES = tcx::X2_BYTES;
constexpr int DWX_MAX = 8192;    // resident depthwise weights, [K][32*nk]
constexpr uint32_t TMEM_COLS = 2 * TN;

constexpr uint32_t A_BYTES = TM * KC * 4;    // 16 KB
constexpr uint32_t B_BYTES = TNH * KC * 4;   // 16 KB
constexpr uint32_t STAGE_BYTES = 2 * A_BYTES + 2 * B_BYTES;
constexpr uint32_t OFF_DWS = STAGES * STAGE_BYTES;
constexpr uint32_t OFF_BAR = OFF_DWS + DWX_MAX * 4;
constexpr uint32_t NBAR = 19;    // full[3] empty[3] afull[2] aempty[2] drain tma[3] lfull[3] gate last
constexpr uint32_t OFF_MISC = OFF_BAR + 24 * 8;
constexpr uint32_t SMEM_BYTES = OFF_MISC + 16 + 1024;
static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");
// Stage: A_hi | A_lo | B_lo | B_hi.  The halo (one box at stride 1, two at
// stride 2) is staged from the stage's start; at stride 2 it reaches into B_lo,
// which the producers then form after their halo barrier (the split warps
// serve stride 1 only), and it never reaches B_hi, where the TMA puts pw.
constexpr uint32_t OFF_BLO = 2 * A_BYTES, OFF_BHI = 2 * A_BYTES + B_BYTES;
static_assert(X_BYTES <= 2 * A_BYTES, "the stride-1 halo box must fit the stage's A region");
static_assert(2 * X2_BYTES <= OFF_BHI, "the stride-2 halo boxes must stay below B_hi");

// D fp32, A/B tf32, K-major, N = 256, M = 256 (the pair).
constexpr uint32_t kIdesc2 = (1u << 4) | (2u << 7) | (2u << 10) | ((uint32_t)(TN >> 3) << 17) |
                             ((uint32_t)(256 >> 4) << 24);

__device__ __forceinline__ uint32_t cluster_rank()
{
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;\n" : "=r"(r));
    return r;
}

__device__ __forceinline__ void cluster_sync()
{
    asm volatile("barrier.cluster.arrive.release.aligned;\nbarrier.cluster.wait.acquire.aligned;\n" ::: "memory");
}

// Address of the same shared-memory location in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t mapa(uint32_t addr, uint32_t rank)
{
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;\n" : "=r"(r) : "r"(addr), "r"(rank));
    return r;
}

__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr)
{
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];\n" ::"r"(cluster_addr) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait_cluster(uint32_t bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n"
        " selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// Abort state of the pair: this CTA's flag and the peer CTA's (its
// shared::cluster address).  A wait gives up when either is set, so when one
// role of one CTA gives up the whole pair leaves its loops within microseconds
// instead of each wait running out on its own.
struct PairAbort {
    volatile uint32_t* local;
    uint32_t peer;
};

__device__ __forceinline__ bool pair_aborted(const PairAbort& a)
{
    if (*a.local) return true;
    uint32_t v;
    asm volatile("ld.relaxed.cluster.shared::cluster.u32 %0, [%1];\n" : "=r"(v) : "r"(a.peer) : "memory");
    if (v) *a.local = 1u;
    return v != 0;
}

// Bounded wait on a barrier of this CTA, with cluster-scope acquire (CLUSTER:
// barriers the peer CTA signals) or CTA-scope acquire.  After `limit_ns` it
// sets this CTA's abort flag and the device error word and returns false.
template <bool CLUSTER>
__device__ __forceinline__ bool pair_wait(uint32_t bar, uint32_t parity, const PairAbort& a,
                                          unsigned long long limit_ns = tc::kWaitLimitNs)
{
    auto test = [&] { return CLUSTER ? mbar_try_wait_cluster(bar, parity) : tc::mbar_try_wait(bar, parity); };
    if (test()) return true;
    const unsigned long long t0 = tc::globaltimer();
    for (uint32_t i = 1;; ++i) {
        if (test()) return true;
        if ((i & 255u) == 0) {
            if (pair_aborted(a)) return false;
            if (tc::globaltimer() - t0 > limit_ns) {
                *a.local = 1u;
                record_device_error(kErrTimeout);
                return false;
            }
        }
    }
}

__device__ __forceinline__ void mma2_tf32(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t accumulate)
{
    asm volatile(
        "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
        " tcgen05.mma.cta_group::2.kind::tf32 [%0], %1, %2, %3, p;\n}\n" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(kIdesc2), "r"(accumulate)
        : "memory");
}

// Commit all prior MMAs of this thread to `bar` in both CTAs of the pair.
__device__ __forceinline__ void commit2(uint32_t bar)
{
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;\n" ::"r"(bar),
        "h"((unsigned short)3)
        : "memory");
}

struct Params {
    const float* x;
    const float* dw;
    const float* pw;
    const float* bias;
    float* out;
    int C, T, O, K, pad, To;
    int tiles_t, tiles_o, total_tiles;  // pair tiles (256 times each)
    int out_vec;                         // output rows 16-byte aligned
    // Failure-path test (all 0 in normal calls): role stall_role (1 TMA warp,
    // 2 producers, 3 MMA issuer, 4 epilogue, 5 pw split, 6 relay) of the CTA
    // of rank stall_rank in every pair waits, before its stall_at-th tile, on a
    // barrier nothing completes, with limit stall_ns.
    int stall_role = 0, stall_at = 0, stall_rank = 0;
    unsigned long long stall_ns = 0;
};

// The failure-path test hook: true unless this role is to stall before its
// `local`-th tile in this CTA and its wait on `gate` ran out (which sets the
// abort flag and the device error word).
__device__ __forceinline__ bool stall_ok(const Params& p, int role, int local, uint32_t rank, uint32_t gate,
                                         const PairAbort& ab)
{
    if (p.stall_role != role || local != p.stall_at || (int)rank != p.stall_rank) return true;
    return pair_wait<false>(gate, 0, ab, p.stall_ns);
}

__device__ __forceinline__ TileCoord decode_pair_tile(const Params& p, int tile)
{
    TileCoord tc;
    tc.t0 = (tile % p.tiles_t) * (2 * TM);
    const int rest = tile / p.tiles_t;
    tc.o0 = (rest % p.tiles_o) * TN;
    tc.n = rest / p.tiles_o;
    return tc;
}

// Drains the 16-column blocks [cb0, cb1) (both even) of this warp's 32 TMEM
// lanes of a finished accumulator at `taddr` (times tw .. tw+31 of tile tcd):
// two blocks at a time, so that their eight 4x4 transposes overlap (lane 4k+j
// ends with times tw+4k..tw+4k+3 of channels 4j..4j+3), the bias added after
// the transpose, where a lane's four values belong to one output channel, then
// 16-byte streaming stores.
__device__ __forceinline__ void drain_blocks(const Params& p, const TileCoord& tcd, uint32_t taddr, int tw, int cb0,
                                             int cb1, int lane)
{
    const bool vec = tw + 32 <= p.To && p.out_vec;
    const int kq = lane >> 2, jq = lane & 3;
    auto bias_of = [&](int o) { return (p.bias && o < p.O) ? __ldg(p.bias + o) : 0.f; };
#pragma unroll 1
    for (int cb = cb0; cb < cb1; cb += 2) {
        uint32_t ra[16], rb[16];
        tc::tmem_ld16(taddr + (uint32_t)(cb * 16), ra);
        tc::tmem_ld16(taddr + (uint32_t)((cb + 1) * 16), rb);
        tc::tmem_wait_ld16(ra);
        tc::tmem_wait_ld16(rb);
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
                for (int m = 0; m < 4; ++m) tc::quad_transpose(x[h][m][0], x[h][m][1], x[h][m][2], x[h][m][3], jq);
#pragma unroll
            for (int h = 0; h < 2; ++h)
#pragma unroll
                for (int m = 0; m < 4; ++m) {
                    const int o = tcd.o0 + (cb + h) * 16 + 4 * jq + m;
                    if (o < p.O) {
                        float* dst = p.out + ((size_t)tcd.n * p.O + o) * p.To + tw + 4 * kq;
                        const float b = bv[h][m];
                        __stcs(reinterpret_cast<float4*>(dst),  // streaming store
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
    }
}

// The last tile of a pair has no successor to overlap its drain with, so the
// eight producer warps, idle by then, take blocks 6..11 (warps 0-3) and 12..15
// (warps 4-7) of their TMEM lane quarter while the epilogue warp takes 0..5.
constexpr int LAST_EPI_BLOCKS = 6, LAST_PROD_SPLIT = 12;
static_assert(LAST_EPI_BLOCKS % 2 == 0 && LAST_PROD_SPLIT % 2 == 0 && LAST_PROD_SPLIT < TN / 16,
              "blocks are drained in pairs");

// KT: depthwise kernel size when fixed at compile time (0: any K <= KMAXW).
// R: (t0*S - pad) mod 4, the offset of the first needed sample inside the box.
// S: stride (1 or 2).
template <int KT, int R, int S>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(NTHREADS, 1)
dwsep_conv1d_tc2_kernel(const Params p, const __grid_constant__ CUtensorMap pw_map,
                        const __grid_constant__ CUtensorMap x_map)
{
    using namespace tc;
    constexpr int KW = KT > 0 ? KT : KMAXW;            // taps the window must cover
    constexpr int NV = (R + S * (TPW - 1) + KW + 3) / 4;  // 16-byte window loads per thread
    static_assert(S == 1 || S == 2, "stride 1 or 2");
    static_assert(S * TPW * (NPW - 1) + 4 * NV <= (S == 1 ? XW : 2 * XW2), "window inside the halo boxes");
    constexpr int FULL_N = S == 1 ? FULL_ARRIVALS : NPW;  // producer (and, at stride 1, split) warps
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    const uint32_t sbase = smem_u32(smem);
    float* dws = reinterpret_cast<float*>(smem + OFF_DWS);
    const uint32_t bar_full = sbase + OFF_BAR;   // + 8 * stage (leader's collects both CTAs)
    const uint32_t bar_empty = bar_full + 24;    // + 8 * stage
    const uint32_t bar_afull = bar_full + 48;    // + 8 * buf
    const uint32_t bar_aempty = bar_full + 64;   // + 8 * buf (leader's collects both CTAs)
    const uint32_t bar_drain = bar_full + 80;
    const uint32_t bar_tma = bar_full + 88;      // + 8 * stage
    const uint32_t bar_lfull = bar_full + 112;   // + 8 * stage (rank 1: its producers, forwarded by the relay)
    const uint32_t bar_gate = bar_full + 136;    // never completed: the failure-path test's stall
    const uint32_t bar_last = bar_full + 144;    // the 4 epilogue warps have seen the last tile's accumulator
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + OFF_MISC);
    volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(smem + OFF_MISC + 4);
    volatile uint32_t* prod_abort = reinterpret_cast<volatile uint32_t*>(smem + OFF_MISC + 8);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_rank();
    const bool leader = rank == 0;
    const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;

    if (threadIdx.x == 0) {
        for (int i = 0; i < STAGES; ++i) {
            mbar_init(bar_full + 8 * i, FULL_N + 1);  // the leader's warps + the other CTA's relay
            mbar_init(bar_lfull + 8 * i, FULL_N);     // the other CTA's warps (used in rank 1)
            mbar_init(bar_empty + 8 * i, 1);   // multicast commit
            mbar_init(bar_tma + 8 * i, 1);     // expect_tx arrival + TMA bytes
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(bar_afull + 8 * i, 1);   // multicast commit
            mbar_init(bar_aempty + 8 * i, 8);  // 4 epilogue warps x 2 CTAs (used in the leader)
        }
        mbar_init(bar_drain, 1);
        mbar_init(bar_gate, 1);
        mbar_init(bar_last, 4);
        *abort_flag = 0u;
        *prod_abort = 0u;
        asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
    }
    if (warp == MMA_WARP) {
        asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(smem_u32(tmem_holder)),
                     "r"(TMEM_COLS)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;\n" ::: "memory");
    }
    const int nk = (p.C + KC - 1) / KC;
    const int CW = KC * nk;
    tc_fence_before();
    cluster_sync();  // barriers of both CTAs initialised, TMEM allocated
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;
    const PairAbort ab{abort_flag, mapa(smem_u32(const_cast<uint32_t*>(abort_flag)), rank ^ 1u)};

    if (warp < NPW) {
        // ------------------------------------------------------------ producers
        const int ptid = threadIdx.x;
        // Depthwise weights resident as [K][CW], CW = 32 * nk, zero beyond C,
        // staged by the producers (their only readers) while the TMA warp
        // already issues the first copies; the group barrier of the first
        // chunk orders these writes before any read.
        for (int e = ptid; e < p.K * CW; e += NPW * 32) {
            const int k = e / CW, c = e - (e / CW) * CW;
            dws[e] = c < p.C ? __ldg(p.dw + (size_t)c * p.K + k) : 0.f;
        }
        const int K = KT > 0 ? KT : p.K;
        int stage = 0;
        uint32_t phase = 0;
        bool run = true;
        int local = 0;
        for (int tile = pair; run && tile < p.total_tiles; tile += npairs, ++local) {
            for (int kc = 0; kc < nk; ++kc) {
                // The TMA copies of this stage (pw half and halo) have landed.
                if (ptid == 0 && ((kc == 0 && !stall_ok(p, 2, local, rank, bar_gate, ab)) ||
                                  !pair_wait<false>(bar_tma + 8 * stage, phase, ab)))
                    *prod_abort = 1u;
                asm volatile("bar.sync 1, %0;\n" ::"n"(NPW * 32) : "memory");
                if (*prod_abort) {
                    run = false;
                    break;
                }
                for (int spin = 0; !mbar_try_wait(bar_tma + 8 * stage, phase) && spin < (1 << 20); ++spin) {
                }
                const uint32_t a_hi = sbase + stage * STAGE_BYTES;
                const uint32_t a_lo = a_hi + A_BYTES;

                // Depthwise: channel lane, this CTA's times TPW*warp .. +TPW-1;
                // halo sample j is x[(t0 + 128*rank)*S - pad - R + j], output time
                // TPW*warp + i takes samples S*(TPW*warp + i) + R + k, k < K; at
                // stride 2, samples j >= XW2 sit in the second box.
                const float* xs0 = reinterpret_cast<const float*>(smem + stage * STAGE_BYTES) +
                                   lane * (S == 1 ? XW : XW2);
                const float* xs1 = xs0 + KC * XW2;
                float win[4 * NV];
#pragma unroll
                for (int q = 0; q < NV; ++q) {
                    const int j = S * TPW * warp + 4 * q;
                    const float* src = (S == 1 || j < XW2) ? xs0 + j : xs1 + (j - XW2);
                    const float4 v = *reinterpret_cast<const float4*>(src);
                    win[4 * q] = v.x;
                    win[4 * q + 1] = v.y;
                    win[4 * q + 2] = v.z;
                    win[4 * q + 3] = v.w;
                }
                float2 d2[TPW / 2];
#pragma unroll
                for (int j = 0; j < TPW / 2; ++j) d2[j] = make_float2(0.f, 0.f);
                const float* wcol = dws + KC * kc + lane;
#pragma unroll
                for (int k = 0; k < KW; ++k) {
                    if (KT > 0 || k < K) {
                        const float w = wcol[k * CW];
                        const float2 w2 = make_float2(w, w);
#pragma unroll
                        for (int j = 0; j < TPW / 2; ++j)
                            d2[j] = __ffma2_rn(make_float2(win[R + 2 * S * j + k], win[R + 2 * S * j + S + k]),
                                               w2, d2[j]);
                    }
                }
                // Every producer has read its halo window before the A operand (and,
                // at stride 2, B_lo) overwrites it.
                asm volatile("bar.sync 1, %0;\n" ::"n"(NPW * 32) : "memory");
                if constexpr (S == 2) {
                    // This CTA's half of the pw chunk: B_hi stays raw (the MMA reads
                    // its TF32 bits), B_lo = v - truncate(v); 16 rows per warp.
                    const uint32_t b_lo = a_hi + OFF_BLO, b_hi = a_hi + OFF_BHI;
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const uint32_t off = sw128_off(warp * 16 + i * 4 + (lane >> 3), lane & 7);
                        sts128(b_lo + off, tcx::tf32_trunc_rest4(lds128(b_hi + off)));
                    }
                }
                const uint32_t col = ((uint32_t)(lane & 3) << 2);
#pragma unroll
                for (int i = 0; i < TPW; ++i) {
                    const float v = (i & 1) ? d2[i >> 1].y : d2[i >> 1].x;
                    const float hi = tf32_round(v);
                    const uint32_t off = sw128_off(TPW * warp + i, lane >> 2) + col;
                    tcx::sts32(a_hi + off, hi);
                    tcx::sts32(a_lo + off, v - hi);
                }
                asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
                __syncwarp();
                // The leader's producers arrive at its "full" directly; the other
                // CTA's arrive locally and its relay thread forwards one cluster
                // arrival, so no producer warp waits out a cluster-scope release.
                if (lane == 0) mbar_arrive(leader ? bar_full + 8 * stage : bar_lfull + 8 * stage);
                if (++stage == STAGES) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
        }
        if (run) {
            // The last tile's drain, beside the epilogue warps, once they have
            // seen its accumulator complete (a barrier used once: no stale phase).
            int ok = 1;
            if (lane == 0) ok = pair_wait<false>(bar_last, 0, ab) ? 1 : 0;
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (ok) {
                tc_fence_after();
                const int last = local - 1, q = warp & 3;
                const TileCoord tcd = decode_pair_tile(p, pair + last * npairs);
                const uint32_t taddr = tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)((last & 1) * TN);
                const int cb0 = warp < 4 ? LAST_EPI_BLOCKS : LAST_PROD_SPLIT;
                const int cb1 = warp < 4 ? LAST_PROD_SPLIT : TN / 16;
                drain_blocks(p, tcd, taddr, tcd.t0 + (int)rank * TM + 32 * q, cb0, cb1, lane);
                tc_fence_before();
            }
        }
    } else if (warp == MMA_WARP) {
        // ---------------------------------------------------------- MMA issuer
        if (lane == 0 && leader) {
            int local = 0, stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            for (int tile = pair; ok && tile < p.total_tiles; tile += npairs, ++local) {
                const int buf = local & 1;
                if (!stall_ok(p, 3, local, rank, bar_gate, ab)) break;
                if (!pair_wait<true>(bar_aempty + 8 * buf, ((local >> 1) & 1) ^ 1, ab)) break;
                tc_fence_after();
                const uint32_t d_tmem = tmem + (uint32_t)(buf * TN);
                for (int k = 0; k < nk; ++k) {
                    if (!pair_wait<true>(bar_full + 8 * stage, phase, ab)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a_hi = sbase + stage * STAGE_BYTES;
                    const uint32_t a_lo = a_hi + A_BYTES;
                    const uint32_t b_lo = a_hi + OFF_BLO;
                    const uint32_t b_hi = a_hi + OFF_BHI;
#pragma unroll
                    for (int kk = 0; kk < KC / 8; ++kk) {
                        const uint32_t koff = 32u * kk;
                        const uint64_t dah = sw128_desc(a_hi + koff), dal = sw128_desc(a_lo + koff);
                        const uint64_t dbh = sw128_desc(b_hi + koff), dbl = sw128_desc(b_lo + koff);
                        mma2_tf32(d_tmem, dah, dbh, (k > 0 || kk > 0) ? 1u : 0u);
                        mma2_tf32(d_tmem, dah, dbl, 1u);
                        mma2_tf32(d_tmem, dal, dbh, 1u);
                    }
                    commit2(bar_empty + 8 * stage);  // both CTAs' stage free once these MMAs read it
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (ok) commit2(bar_afull + 8 * buf);  // both CTAs' accumulator rows complete
            }
            commit2(bar_drain);  // every MMA issued for the pair has completed once this fires
        }
        if (lane == 0 && !leader) {
            // Relay: once this CTA's 8 producer warps have filled a stage (local
            // barrier, CTA-scope release/acquire), one cluster-scope arrival
            // at the leader's "full" carries their writes to the leader's
            // issuer.  Bounded like every wait; after an abort the leader's
            // barrier is still alive (the closing cluster barrier).
            const uint32_t full_leader = mapa(bar_full, 0);
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            int local = 0;
            for (int tile = pair; ok && tile < p.total_tiles; tile += npairs, ++local) {
                for (int k = 0; k < nk; ++k) {
                    if ((k == 0 && !stall_ok(p, 6, local, rank, bar_gate, ab)) ||
                        !pair_wait<false>(bar_lfull + 8 * stage, phase, ab)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_cluster(full_leader + 8 * stage);
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
        }
        if (lane == 0) {
            const unsigned long long t0 = globaltimer();
            while (!mbar_try_wait_cluster(bar_drain, 0)) {
                if (globaltimer() - t0 > kWaitLimitNs) {
                    *abort_flag = 1u;
                    record_device_error(kErrTimeout);
                    break;
                }
            }
        }
        __syncwarp();
    } else if (warp >= SPLIT_WARP) {
        // ------------------------------------------------------ pw split
        // This CTA's half of each pw chunk, once its TMA copy has landed: B_hi
        // stays raw (the MMA reads its TF32 bits), B_lo = v - truncate(v).
        // Off the depthwise warps' path, so their chunk time is the
        // depthwise alone.
        const int sl = (warp - SPLIT_WARP) * 32 + lane;
        int stage = 0;
        uint32_t phase = 0;
        bool ok = S == 1;  // at stride 2 the producers form B_lo after their halo barrier
        int local = 0;
        for (int tile = pair; ok && tile < p.total_tiles; tile += npairs, ++local) {
            for (int k = 0; k < nk; ++k) {
                int good = 1;
                if (lane == 0)
                    good = ((k != 0 || stall_ok(p, 5, local, rank, bar_gate, ab)) &&
                            pair_wait<false>(bar_tma + 8 * stage, phase, ab)) ? 1 : 0;
                good = __shfl_sync(0xffffffffu, good, 0);
                if (!good) {
                    ok = false;
                    break;
                }
                for (int spin = 0; !mbar_try_wait(bar_tma + 8 * stage, phase) && spin < (1 << 20); ++spin) {
                }
                const uint32_t b_hi = sbase + stage * STAGE_BYTES + OFF_BHI;
                const uint32_t b_lo = sbase + stage * STAGE_BYTES + OFF_BLO;
                // 1024 16-byte slots (128 rows x 8), 16 per thread in two batches
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    float4 v[8];
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const int slot = (8 * h + i) * 32 * NSPLIT + sl;
                        v[i] = lds128(b_hi + sw128_off(slot >> 3, slot & 7));
                    }
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const int slot = (8 * h + i) * 32 * NSPLIT + sl;
                        sts128(b_lo + sw128_off(slot >> 3, slot & 7), tcx::tf32_trunc_rest4(v[i]));
                    }
                }
                asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
                __syncwarp();
                if (lane == 0) mbar_arrive(leader ? bar_full + 8 * stage : bar_lfull + 8 * stage);
                if (++stage == STAGES) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
        }
    } else if (warp == TMA_WARP) {
        // -------------------------------------------------------- TMA issuer
        // Per chunk: this CTA's half of the pw chunk into B_hi and its input
        // halo [32 channels][148 times] into the A region, once the MMAs that
        // last read the stage (in both CTAs) have completed.
        if (lane == 0) {
            int stage = 0, issued = 0;
            uint32_t phase = 0;
            bool pending[STAGES] = {false, false, false};
            bool ok = true;
            int local = 0;
            for (int tile = pair; ok && tile < p.total_tiles; tile += npairs, ++local) {
                if (!stall_ok(p, 1, local, rank, bar_gate, ab)) break;
                const TileCoord tcd = decode_pair_tile(p, tile);
                const int x0 = (tcd.t0 + (int)rank * TM) * S - p.pad - R;  // a multiple of 4
                // Pull the next tile's halo boxes into L2 now, so its TMA loads
                // wait on L2 rather than on DRAM latency.
                if (tile + npairs < p.total_tiles) {
                    const TileCoord nx = decode_pair_tile(p, tile + npairs);
                    const int nx0 = (nx.t0 + (int)rank * TM) * S - p.pad - R;
                    for (int k = 0; k < nk; ++k) {
                        tcx::tma_prefetch_3d(&x_map, nx0, k * KC, nx.n);
                        if (S == 2) tcx::tma_prefetch_3d(&x_map, nx0 + XW2, k * KC, nx.n);
                    }
                }
                for (int k = 0; k < nk; ++k) {
                    if (!pair_wait<true>(bar_empty + 8 * stage, phase ^ 1, ab)) {
                        ok = false;
                        break;
                    }
                    pending[stage] = false;
                    const uint32_t st = sbase + stage * STAGE_BYTES;
                    mbar_arrive_expect_tx(bar_tma + 8 * stage, B_BYTES + (S == 1 ? X_BYTES : 2 * X2_BYTES));
                    tma_load_2d(st + OFF_BHI, &pw_map, k * KC, tcd.o0 + (int)rank * TNH, bar_tma + 8 * stage);
                    tcx::tma_load_3d(st, &x_map, x0, k * KC, tcd.n, bar_tma + 8 * stage);
                    if (S == 2) tcx::tma_load_3d(st + X2_BYTES, &x_map, x0 + XW2, k * KC, tcd.n, bar_tma + 8 * stage);
                    pending[stage] = true;
                    ++issued;
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            {
                // Wait (bounded) for copies still in flight before the CTA can
                // exit, also when another role gave up and they were never
                // consumed (normally they have all landed): the latest use of
                // stage s is number u = issued-1-((issued-1-s) mod 3).
                for (int st = 0; st < STAGES; ++st) {
                    if (!pending[st]) continue;
                    const int u = issued - 1 - ((issued - 1 - st) % STAGES);
                    const unsigned long long t0 = globaltimer();
                    while (u >= 0 && !mbar_try_wait(bar_tma + 8 * st, (uint32_t)((u / STAGES) & 1))) {
                        if (globaltimer() - t0 > kWaitLimitNs) break;
                    }
                }
            }
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ epilogue
        const int q = warp & 3;
        const uint32_t aempty_leader = mapa(bar_aempty, 0);
        int local = 0;
        for (int tile = pair; tile < p.total_tiles; tile += npairs, ++local) {
            const int buf = local & 1;
            int ok = 1;
            if (lane == 0)
                ok = (stall_ok(p, 4, local, rank, bar_gate, ab) &&
                      pair_wait<true>(bar_afull + 8 * buf, (local >> 1) & 1, ab)) ? 1 : 0;
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) break;
            tc_fence_after();
            const TileCoord tcd = decode_pair_tile(p, tile);
            const int tw = tcd.t0 + (int)rank * TM + 32 * q;
            const uint32_t taddr = tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(buf * TN);
            const bool last = tile + npairs >= p.total_tiles;
            if (last && lane == 0) mbar_arrive(bar_last);  // the producers take the rest of this tile
            drain_blocks(p, tcd, taddr, tw, 0, last ? LAST_EPI_BLOCKS : TN / 16, lane);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(aempty_leader + 8 * buf);
        }
    }

    tc_fence_before();
    __syncthreads();
    cluster_sync();  // the peer no longer signals this CTA's barriers
    tc_fence_after();
    if (warp == MMA_WARP) {
        asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;\n" ::"r"(tmem), "r"(TMEM_COLS)
                     : "memory");
    }
}

using KernelPtr = decltype(&dwsep_conv1d_tc2_kernel<0, 0, 1>);

template <int S>
inline KernelPtr select_kernel(int K, int r)
{
    if (K == 9 && r == 0) return dwsep_conv1d_tc2_kernel<9, 0, S>;
    if (K == 3 && r == 3) return dwsep_conv1d_tc2_kernel<3, 3, S>;
    if (r == 0) return dwsep_conv1d_tc2_kernel<0, 0, S>;
    if (r == 1) return dwsep_conv1d_tc2_kernel<0, 1, S>;
    if (r == 2) return dwsep_conv1d_tc2_kernel<0, 2, S>;
    return dwsep_conv1d_tc2_kernel<0, 3, S>;
}

}  // namespace tc2

// The 2-SM path covers the shapes of the single-SM TMA-halo kernel.
inline bool conv1d_tc2_supported(int C, int T, int O, int K, int stride, const void* x, const void* pw)
{
    const long long cw = (long long)tc2::KC * ((C + tc2::KC - 1) / tc2::KC);
    return (stride == 1 || stride == 2) && K >= 1 && K <= tc::KMAXW && C >= 1 && O >= 1 && T >= 1 && (C & 3) == 0 &&
           (T & 3) == 0 && (reinterpret_cast<uintptr_t>(x) & 15) == 0 &&
           (reinterpret_cast<uintptr_t>(pw) & 15) == 0 && cw * K <= tc2::DWX_MAX;
}

// Where AUTO takes the SM pair over the single-SM TMA-halo kernel: at least
// eight 32-channel chunks per tile (C >= 256), so the pair's per-tile
// start-up and drain are amortised, and, at stride 1, O >= 256, so the
// 256-wide tile is not half empty.  Measured on B200 over the conv1d shape
// sweep: stride 1, 1.05-1.20x faster there, 0.80-0.98x at C = 64, about even
// at O = 128; stride 2 (where the depthwise window work, which the pair
// splits, is twice as large), 1.03-1.14x at C = 384 and O = 128 and
// 1.22-1.38x at O = 768, 0.82-0.96x at C = 64 and T = 16384.
inline bool conv1d_tc2_preferred(int C, int T, int O, int K, int stride, const void* x, const void* pw)
{
    return C >= 256 && (stride == 2 || O >= 256) && conv1d_tc2_supported(C, T, O, K, stride, x, pw);
}

inline int launch_dwsep_conv1d_tc2(const float* x, const float* dw, const float* pw, const float* bias, int N,
                                   int C, int T, int O, int K, int stride, int pad, int To, float* out,
                                   cudaStream_t stream,
                                   int stall_role = 0, int stall_at = 0, int stall_rank = 0,
                                   unsigned long long stall_ns = 0)
{
    tc2::Params prm;
    prm.stall_role = stall_role;
    prm.stall_at = stall_at;
    prm.stall_rank = stall_rank;
    prm.stall_ns = stall_ns;
    prm.x = x; prm.dw = dw; prm.pw = pw; prm.bias = bias; prm.out = out;
    prm.C = C; prm.T = T; prm.O = O; prm.K = K; prm.pad = pad; prm.To = To;
    prm.tiles_t = (To + 2 * tc2::TM - 1) / (2 * tc2::TM);
    prm.tiles_o = (O + tc2::TN - 1) / tc2::TN;
    const long long total = (long long)N * prm.tiles_t * prm.tiles_o;
    if (total > 0x7fffffffLL) return FCV_ERR_UNSUPPORTED;
    prm.total_tiles = (int)total;
    prm.out_vec = ((To & 3) == 0 && (reinterpret_cast<uintptr_t>(out) & 15) == 0) ? 1 : 0;

    auto encode = tensor_map_encoder();
    if (!encode) return FCV_ERR_CUDA;
    CUtensorMap pw_map, x_map;
    {   // pw [O][C]: 32 channels x 128 output channels per box (this CTA's half), 128B-swizzled
        const cuuint64_t gdim[2] = {(cuuint64_t)C, (cuuint64_t)O};
        const cuuint64_t gstride[1] = {(cuuint64_t)C * sizeof(float)};
        const cuuint32_t box[2] = {(cuuint32_t)tc2::KC, (cuuint32_t)tc2::TNH};
        const cuuint32_t estride[2] = {1, 1};
        if (encode(&pw_map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float*>(pw), gdim, gstride, box, estride,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return FCV_ERR_CUDA;
    }
    {   // x [N][C][T]: 148 (stride 2: 140) times x 32 channels x 1 batch item per box; outside reads 0
        const cuuint64_t gdim[3] = {(cuuint64_t)T, (cuuint64_t)C, (cuuint64_t)N};
        const cuuint64_t gstride[2] = {(cuuint64_t)T * sizeof(float), (cuuint64_t)C * T * sizeof(float)};
        const cuuint32_t box[3] = {(cuuint32_t)(stride == 1 ? tc2::XW : tc2::XW2), (cuuint32_t)tc2::KC, 1};
        const cuuint32_t estride[3] = {1, 1, 1};
        if (encode(&x_map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<float*>(x), gdim, gstride, box, estride,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return FCV_ERR_CUDA;
    }

    int sms = 0;
    if (device_sm_count(&sms) != FCV_OK) return FCV_ERR_CUDA;
    const int r = (-pad) & 3;  // (t0*stride - pad) mod 4 with t0 a multiple of 128
    const tc2::KernelPtr kern = stride == 1 ? tc2::select_kernel<1>(K, r) : tc2::select_kernel<2>(K, r);
    const long long pairs = total < sms / 2 ? total : sms / 2;
    dim3 grid((unsigned)(2 * pairs));
    return launch_cached(kern, (int)tc2::SMEM_BYTES,
                         [&] { kern<<<grid, tc2::NTHREADS, tc2::SMEM_BYTES, stream>>>(prm, pw_map, x_map); });
}

}  // namespace fcv
