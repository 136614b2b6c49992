// conv2d_tc.cuh -- op A on tcgen05 tensor cores: the direct 3x3 convolution of
// every pooled window as an implicit GEMM, fp32-accurate through a 3xTF32 split.
//
// What it computes (POPCORNBENCH trace of the fused Conv2d -> AvgPool -> Sigmoid
// -> Sum kernel; the trace notes cuDNN would run this convolution on TF32
// tensor cores): every conv output y[n, co, r, c] = b[co] + sum over (ci, ky, kx)
// of w[co, ci, ky, kx] * x[n, ci, r+ky, c+kx], averaged over P x P windows,
// passed through the sigmoid and summed per image.  Written as a GEMM per
// tile, D[m, co] = sum_k A[m, k] * B[co, k] with
//     m = one of 128 conv positions (P conv rows x 128/P conv columns),
//     k = (ci, ky, kx), chunks of 8 input channels = 72 K elements,
//     A = the im2col rows of x, B = w.
// Every conv output is computed (the same multiply-adds as the FMA kernel),
// only on the tensor cores; the P x P pooling is a sum over accumulator rows
// done in the epilogue.
//
// B200 design (one CTA per SM, persistent over tiles, 23 warps):
//   * warp 21 (TMA): one 4-D box per (tile, chunk) brings the input halo
//     [8 channels][P + 2 rows][128/P + 2 columns] into one of two shared
//     buffers (cp.async by the producers instead when rows are not 16-byte
//     aligned).
//   * warps 0-7 (producers, two per TMEM lane quarter): each thread owns one
//     conv position (= one TMEM lane) and half of its 72 im2col values: reads
//     them from the halo, splits them into TF32 hi/lo and writes them straight
//     into tensor memory with tcgen05.st (the A operand of the MMA is read from
//     TMEM, so A costs no shared-memory bandwidth).  Before a tile's first chunk
//     they also see its accumulator drained, so the MMA issuers wait on one
//     barrier per chunk.
//   * warps 8 and 22 (MMA issuers, even and odd tiles): one thread each issues
//     27 tcgen05.mma (kind::tf32, M = 128, N = Cout', K = 8, A from TMEM, B
//     from shared memory) per chunk: A_hi*B_hi + A_hi*B_lo + A_lo*B_hi, from
//     descriptors computed once.  Each owns one of the two A stages; while one
//     waits on a barrier the other keeps the tensor core busy.
//   * TMEM: 2 or 3 accumulators of Cout' columns, two A stages of 144.
//   * The weights, split into TF32 hi/lo once per CTA, stay in shared memory
//     in the K-major 128-byte-swizzled layout for the whole kernel.
//   * warps 9-12 (drain, one per lane quarter): copy a finished accumulator
//     with tcgen05.ld into one of two transposed shared buffers and release
//     it at once.
//   * warps 13-20 (pool): each thread sums the P x P conv outputs of its
//     (window, channel) values, adds the bias, applies the sigmoid and
//     accumulates; one atomic add per warp and image.  Pooling of one tile
//     overlaps the drain of the next.
//   * Every wait is bounded, as in the conv1d kernels.
//
// Sub-chunk variant (conv2d_tc4_kernel; used when the halo comes by TMA and
// Cout' <= 96): each chunk's nine K-steps are split into K-steps 0-4 and 5-8,
// TMEM holds four A stages of 80 columns (sub-chunk s of a tile with parity q
// in stage 2q + s), and the producers form two independent groups of four
// warps, one per sub-chunk, so a group refills its half of the next tile while
// the MMAs of the other half run.  Each MMA issuer commits a sub-chunk's stage
// as soon as its MMAs are issued.  With three accumulators of 64 columns that
// is exactly the 512 TMEM columns.
#pragma once

#include "conv1d_tc.cuh"
#include "conv2d_direct.cuh"

#include <type_traits>

namespace fcv {
namespace c2tc {

using tc::globaltimer;
using tc::kWaitLimitNs;
using tc::mbar_arrive;
using tc::mbar_init;
using tc::mbar_try_wait;
using tc::smem_u32;
using tc::sw128_desc;
using tc::sw128_off;
using tc::tc_commit;
using tc::tc_fence_after;
using tc::tc_fence_before;
using tc::tf32_round;
using tc::tmem_ld16;
using tc::tmem_wait_ld;
using tc::wait_bounded;

constexpr int MT = 128;           // conv positions per tile (UMMA M)
constexpr int CCH = 8;            // input channels per K chunk
constexpr int KCH = 9 * CCH;      // 72 K elements per chunk
constexpr int KST = KCH / 8;      // 9 MMA K-steps per chunk
constexpr int A_COLS = 2 * KCH;   // one A stage in TMEM: hi (72 columns) | lo (72 columns)
constexpr int NP_MAX = 112;       // padded Cout: 2 * NP + 2 * A_COLS <= 512 TMEM columns
constexpr int NPROD = 256;        // producer threads: warps 0-7, two per TMEM lane quarter
constexpr int MMA_WARP = 8;
constexpr int DRAIN_WARP0 = 9;    // epilogue drain: warps 9-12, one per TMEM lane quarter
constexpr int POOL_WARP0 = 13;    // epilogue pooling: warps 13-20
constexpr int NPOOL = 256;
constexpr int TMA_WARP = 21;
constexpr int MMA_WARP2 = 22;     // second MMA issuer (odd tiles)
constexpr int NTHREADS = 23 * 32;
constexpr int SUB0 = 5;           // sub-chunk kernel: K-steps 0-4 | 5-8 of a chunk
constexpr int SUB_LO = 8 * SUB0;  // lo half of a sub-chunk A stage (columns)
constexpr int SUB_COLS = 2 * SUB_LO;  // one sub-chunk A stage: hi (40) | lo (40); four of them
constexpr int NP_MAX_SUB = 96;    // sub-chunk kernel: 2 * NP + 4 * SUB_COLS <= 512
constexpr int TP = 132;           // pitch of the transposed accumulator buffer (floats)
constexpr uint32_t TMEM_COLS = 512;
constexpr int SMEM_LIMIT = 227 * 1024;

template <int P>
struct Geo {
    static constexpr int WC = MT / P;                                // conv columns per tile
    static constexpr int WPT = WC / P;                               // pooled windows per tile
    static constexpr int HR = P + 2;                                 // halo rows
    static constexpr int HW = WC + 2;                                // halo columns
    static constexpr int HP = P == 8 ? 48 : ((HW + 3) & ~3);         // halo row pitch (floats)
    static constexpr int CHS = HR * HP;                              // halo channel stride
    static constexpr int HALO = CCH * CHS;                           // floats per halo buffer
    static_assert(WC * P == MT && WPT * P == WC, "tile shape");
    static_assert(HP >= HW, "halo pitch");
};

struct Params {
    const float* x;
    const float* w;
    const float* b;
    float* out;       // sum mode: out[N]; tap mode: pooled[N, Cout, PH, PW]
    int Cin, H, W, Cout, PH, PW;
    int NP;           // Cout rounded up to 16 (MMA N)
    int nchunks;      // ceil(Cin / 8)
    int natoms;       // 128-byte-wide K blocks of the weight operand (3 per chunk)
    int tiles_x;      // tiles per pooled row
    int tiles_img;    // tiles per image
    int total_tiles;
    int use_tma;      // halo by one 4-D TMA box (W % 4 == 0, aligned x), else by cp.async
    int nacc;         // accumulator buffers in TMEM: 3 when they fit next to the kernel's A stages, else 2
};

// Shared-memory layout (bytes, from a 1024-aligned base).
struct Layout {
    uint32_t b_hi, b_lo, halo, tbuf, bias, bar, misc, total;
};

template <int P>
__host__ __device__ inline Layout make_layout(int NP, int natoms)
{
    Layout L;
    const uint32_t atoms_bytes = (uint32_t)natoms * (uint32_t)NP * 128u;
    L.b_hi = 0;
    L.b_lo = atoms_bytes;
    L.halo = 2 * atoms_bytes;
    L.tbuf = L.halo + 2u * Geo<P>::HALO * 4u;
    L.bias = L.tbuf + 2u * (uint32_t)NP * TP * 4u;  // two transposed accumulator buffers
    L.bar = (L.bias + (uint32_t)NP * 4u + 7u) & ~7u;
    L.misc = L.bar + 24u * 8u;
    L.total = L.misc + 16u;
    return L;
}

// D[tmem] (+)= A[tmem] * B[smem]^T, kind::tf32, A read from tensor memory.
__device__ __forceinline__ void mma_tf32_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                            uint32_t accumulate)
{
    asm volatile(
        "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
        " tcgen05.mma.cta_group::1.kind::tf32 [%0], [%1], %2, %3, p;\n}\n" ::"r"(d_tmem),
        "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// The same, always accumulating.
__device__ __forceinline__ void mma_tf32_ts_acc(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc)
{
    asm volatile("tcgen05.mma.cta_group::1.kind::tf32 [%0], [%1], %2, %3, 1;\n" ::"r"(d_tmem), "r"(a_tmem),
                 "l"(bdesc), "r"(idesc)
                 : "memory");
}

// 8 consecutive 32-bit TMEM columns of the warp's 32 lanes (one register each).
__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t (&r)[8])
{
    asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};\n" ::"r"(taddr),
                 "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]));
}

__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;\n" ::: "memory"); }

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

struct TileCoord {
    int n, py, tx;  // image, pooled row, tile column
};

__device__ __forceinline__ TileCoord decode(const Params& p, int tile)
{
    TileCoord t;
    t.n = tile / p.tiles_img;
    const int r = tile - t.n * p.tiles_img;
    t.py = r / p.tiles_x;
    t.tx = r - t.py * p.tiles_x;
    return t;
}

// Weights as the B operand, split into TF32 hi/lo, and the padded bias, into
// shared memory (all threads of the CTA; the caller fences and synchronises).
template <int P>
__device__ __forceinline__ void stage_weights(const Params& p, uint8_t* smem, const Layout& L, float* bias_s)
{
    const int NP = p.NP;
    // Element (co, k) with
    // k = 72 * chunk + e, e = 9 * (ci mod 8) + 3 * ky + kx, sits in 128-byte K
    // block 3 * chunk + e / 32 (blocks of NP rows), row co, swizzled 16-byte
    // chunk (e mod 32) / 4.  Every chunk starts a K block, so the descriptors of
    // chunk c are those of chunk 0 moved by c * 3 blocks.
    const int ktot = KCH * p.nchunks;
    for (int idx = threadIdx.x; idx < NP * ktot; idx += NTHREADS) {
        const int co = idx / ktot, k = idx - co * ktot;
        const int ch = k / KCH, e = k - ch * KCH;
        const int ci = ch * CCH + e / 9, t = e % 9;
        const float v = (co < p.Cout && ci < p.Cin) ? __ldg(p.w + ((size_t)co * p.Cin + ci) * 9 + t) : 0.f;
        const float hi = tf32_round(v);
        const int a = 3 * ch + (e >> 5), kin = e & 31;
        const uint32_t off = (uint32_t)a * NP * 128u + sw128_off(co, kin >> 2) + (uint32_t)(kin & 3) * 4u;
        *reinterpret_cast<float*>(smem + L.b_hi + off) = hi;
        *reinterpret_cast<float*>(smem + L.b_lo + off) = v - hi;
    }
    for (int i = threadIdx.x; i < NP; i += NTHREADS) bias_s[i] = i < p.Cout ? __ldg(p.b + i) : 0.f;
}

// TMA warp: one box [8 channels][P + 2 rows][HP columns] per (tile, chunk)
// into the two halo buffers, in the order the producers consume them.
template <int P>
__device__ __forceinline__ void tma_halo_warp(const Params& p, const CUtensorMap& x_map, float* halo,
                                              uint32_t bar_hfull, uint32_t bar_hempty,
                                              volatile uint32_t* abort_flag, int lane)
{
    using G = Geo<P>;
    // The box lands in the halo layout itself; rows, columns and channels
    // outside x read 0.
    if (p.use_tma && lane == 0) {
        int seq = 0;
        bool pending[2] = {false, false};
        bool ok = true;
        for (int tile = blockIdx.x; ok && tile < p.total_tiles; tile += gridDim.x) {
            const TileCoord tcd = decode(p, tile);
            for (int ch = 0; ch < p.nchunks; ++ch, ++seq) {
                const int b = seq & 1;
                if (!wait_bounded(bar_hempty + 8 * b, ((seq >> 1) & 1) ^ 1, abort_flag)) {
                    ok = false;
                    break;
                }
                pending[b] = false;  // the producers consumed its previous box
                tc::mbar_arrive_expect_tx(bar_hfull + 8 * b, (uint32_t)G::HALO * 4u);
                tma_load_4d(smem_u32(halo + b * G::HALO), &x_map, tcd.tx * G::WC, tcd.py * P, ch * CCH, tcd.n,
                            bar_hfull + 8 * b);
                pending[b] = true;
            }
        }
        {
            // Wait (bounded) for boxes still in flight before the CTA may leave,
            // also when another role gave up and they were never consumed
            // (normally they have all landed and this returns at once).
            for (int b = 0; b < 2; ++b) {
                if (!pending[b]) continue;
                const int last = seq - 1 - ((seq - 1 - b) & 1);  // latest sequence number on buffer b
                const unsigned long long t0 = globaltimer();
                while (last >= 0 && !mbar_try_wait(bar_hfull + 8 * b, (last >> 1) & 1)) {
                    if (globaltimer() - t0 > kWaitLimitNs) break;
                }
            }
        }
    }
    __syncwarp();
}

// Epilogue warps 9-20: drain (9-12) and pool (13-20), as described above.
template <int P, int MODE>
__device__ __forceinline__ void epilogue_warps(const Params& p, float* tbuf, const float* bias_s, uint32_t tmem,
                                               uint32_t bar_accfull, uint32_t bar_accempty, uint32_t bar_tfull,
                                               uint32_t bar_tempty, volatile uint32_t* abort_flag, int warp,
                                               int lane)
{
    using G = Geo<P>;
    const int NP = p.NP;
    // Drain warps (one per TMEM lane quarter) copy a finished accumulator
    // into one of two transposed buffers and release it at once; pool warps
    // then reduce that buffer.  Pooling of one tile overlaps the drain of
    // the next, so the epilogue's rate is the slower of the two halves.
    int abuf = 0, local = 0;
    uint32_t aphase = 0;
    if (warp >= DRAIN_WARP0 && warp < DRAIN_WARP0 + 4) {
        const int q = warp & 3;  // TMEM lane quarter of this warp
        const int mrow = 32 * q + lane;
        for (int tile = blockIdx.x; tile < p.total_tiles; tile += gridDim.x, ++local) {
            const int buf = abuf;
            const uint32_t bphase = aphase;
            if (++abuf == p.nacc) {
                abuf = 0;
                aphase ^= 1u;
            }
            const int tb = local & 1;
            const uint32_t tphase = (local >> 1) & 1;
            int ok = 1;
            if (lane == 0) {
                ok = wait_bounded(bar_accfull + 8 * buf, bphase, abort_flag) &&
                     wait_bounded(bar_tempty + 8 * tb, tphase ^ 1, abort_flag);
            }
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) break;
            tc_fence_after();  // TMEM loads after the MMAs lane 0 saw complete
            float* tbw = tbuf + tb * NP * TP;
            const uint32_t taddr = tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(buf * NP);
            for (int cb = 0; cb < NP / 16; cb += 2) {  // two TMEM loads per wait
                uint32_t v[16], u[16];
                const bool two = cb + 1 < NP / 16;
                tmem_ld16(taddr + (uint32_t)(16 * cb), v);
                if (two) tmem_ld16(taddr + (uint32_t)(16 * (cb + 1)), u);
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 16; ++j) tbw[(16 * cb + j) * TP + mrow] = __uint_as_float(v[j]);
                if (two) {
#pragma unroll
                    for (int j = 0; j < 16; ++j) tbw[(16 * (cb + 1) + j) * TP + mrow] = __uint_as_float(u[j]);
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(bar_accempty + 8 * buf);  // accumulator free for the MMA
                mbar_arrive(bar_tfull + 8 * tb);      // this quarter of the buffer is written
            }
        }
    } else {
        const int ptid = threadIdx.x - 32 * POOL_WARP0;  // 0..255
        const float inv_area = 1.f / (float)(P * P);
        const float inv_cout = 1.f / (float)p.Cout;
        float acc = 0.f;
        int cur = -1;
        auto flush = [&]() {
            float s = acc;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
            if (lane == 0 && cur >= 0) atomicAdd(p.out + cur, s);
            acc = 0.f;
        };
        for (int tile = blockIdx.x; tile < p.total_tiles; tile += gridDim.x, ++local) {
            const int tb = local & 1;
            const uint32_t tphase = (local >> 1) & 1;
            int ok = 1;
            if (lane == 0) ok = wait_bounded(bar_tfull + 8 * tb, tphase, abort_flag) ? 1 : 0;
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) break;
            // every lane acquires the drain warps' stores (returns at once)
            for (int spin = 0; !mbar_try_wait(bar_tfull + 8 * tb, tphase) && spin < (1 << 20); ++spin) {
            }
            const TileCoord tcd = decode(p, tile);
            if (MODE != kTap && tcd.n != cur) {
                flush();
                cur = tcd.n;
            }
            const float* tbr = tbuf + tb * NP * TP;
            const int nval = G::WPT * p.Cout;
#pragma unroll 2
            for (int v = ptid; v < nval; v += NPOOL) {
                // j = v / Cout exactly: (v + 1/2) / Cout is at least 1/(2 Cout) away
                // from an integer and v < 2^14, far inside fp32 precision.
                const int j = (int)(((float)v + 0.5f) * inv_cout), co = v - j * p.Cout;
                const int px = tcd.tx * G::WPT + j;
                if (px >= p.PW) continue;
                const float* tb4 = tbr + co * TP + j * P;
                float s = 0.f;
#pragma unroll
                for (int rr = 0; rr < P; ++rr) {
                    if constexpr (P % 4 == 0) {
#pragma unroll
                        for (int dc = 0; dc < P; dc += 4) {
                            const float4 f = *reinterpret_cast<const float4*>(tb4 + rr * G::WC + dc);
                            s += (f.x + f.y) + (f.z + f.w);
                        }
                    } else {
#pragma unroll
                        for (int dc = 0; dc < P; ++dc) s += tb4[rr * G::WC + dc];
                    }
                }
                const float pooled = s * inv_area + bias_s[co];
                if (MODE == kTap) {
                    p.out[(((size_t)tcd.n * p.Cout + co) * p.PH + tcd.py) * p.PW + px] = pooled;
                } else {
                    acc += __fdividef(1.f, 1.f + __expf(-pooled));  // sigmoid; 0 once exp overflows
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(bar_tempty + 8 * tb);  // this warp is done with the buffer
        }
        if (MODE != kTap) flush();
    }
}

template <int P, int MODE>
__global__ void __launch_bounds__(NTHREADS, 1) conv2d_tc_kernel(const Params p, const __grid_constant__ CUtensorMap x_map)
{
    using G = Geo<P>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    const uint32_t sbase = smem_u32(smem);
    const Layout L = make_layout<P>(p.NP, p.natoms);
    float* halo = reinterpret_cast<float*>(smem + L.halo);
    float* tbuf = reinterpret_cast<float*>(smem + L.tbuf);
    float* bias_s = reinterpret_cast<float*>(smem + L.bias);
    const uint32_t bar_afull = sbase + L.bar;         // + 8 * stage, 8 producer-warp arrivals
    const uint32_t bar_aempty = bar_afull + 16;       // + 8 * stage, tcgen05.commit
    const uint32_t bar_accfull = bar_afull + 32;      // + 8 * buf (up to 3), tcgen05.commit
    const uint32_t bar_accempty = bar_afull + 56;     // + 8 * buf (up to 3), 4 drain-warp arrivals
    const uint32_t bar_drain = bar_afull + 80;
    const uint32_t bar_hfull = bar_afull + 88;        // + 8 * buf, TMA halo landed
    const uint32_t bar_hempty = bar_afull + 104;      // + 8 * buf, 8 producer-warp arrivals
    const uint32_t bar_tfull = bar_afull + 120;       // + 8 * buf, 4 drain-warp arrivals
    const uint32_t bar_tempty = bar_afull + 136;      // + 8 * buf, 8 pool-warp arrivals
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + L.misc);
    volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(smem + L.misc + 4);
    volatile uint32_t* prod_abort = reinterpret_cast<volatile uint32_t*>(smem + L.misc + 8);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int NP = p.NP;

    if (threadIdx.x == 0) {
        for (int i = 0; i < 2; ++i) {
            mbar_init(bar_afull + 8 * i, 8);
            mbar_init(bar_aempty + 8 * i, 1);
        }
        for (int i = 0; i < 3; ++i) {
            mbar_init(bar_accfull + 8 * i, 1);
            mbar_init(bar_accempty + 8 * i, 4);
        }
        mbar_init(bar_drain, 2);  // one commit per MMA issuer
        mbar_init(bar_hfull, 1);
        mbar_init(bar_hfull + 8, 1);
        mbar_init(bar_hempty, 8);
        mbar_init(bar_hempty + 8, 8);
        mbar_init(bar_tfull, 4);
        mbar_init(bar_tfull + 8, 4);
        mbar_init(bar_tempty, 8);
        mbar_init(bar_tempty + 8, 8);
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

    stage_weights<P>(p, smem, L, bias_s);
    asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");  // weights visible to the tensor core
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;
    // Accumulators: p.nacc buffers of NP columns (3 when they fit next to the two
    // A stages, else 2), used round robin: buffer abuf, phase aphase.
    const uint32_t a_col0 = (uint32_t)(p.nacc * NP);  // first A-stage column

    if (warp < 8) {
        // ------------------------------------------------------------ producers
        const int tid = threadIdx.x;               // 0..255
        const int m = 32 * (warp & 3) + lane;      // conv position = TMEM lane
        const int half = warp >> 2;                // K groups 0-4 or 5-8 of the chunk
        const int r = m / G::WC, c = m - (m / G::WC) * G::WC;
        const uint32_t lane_base = (uint32_t)(32 * (warp & 3)) << 16;
        int pseq_tile = blockIdx.x, pseq_ch = 0;  // cp.async path: the (tile, chunk) being fetched

        // Halo of (tile, chunk) into buffer buf by cp.async, for rows that are
        // not 16-byte aligned (the TMA warp loads it otherwise).
        auto fetch = [&](int tile, int ch, int buf) {
            const TileCoord tcd = decode(p, tile);
            const int y0 = tcd.py * P, x0 = tcd.tx * G::WC, c0 = ch * CCH;
            float* dst = halo + buf * G::HALO;
            const float* src = p.x + ((size_t)tcd.n * p.Cin) * p.H * p.W;
            for (int i = tid; i < CCH * G::HR * G::HW; i += NPROD) {
                const int ci = i / (G::HR * G::HW);
                const int rem = i - ci * (G::HR * G::HW);
                const int hr = rem / G::HW, hc = rem - (rem / G::HW) * G::HW;
                const int gy = y0 + hr, gx = x0 + hc, gc = c0 + ci;
                const bool ok = gc < p.Cin && gy < p.H && gx < p.W;
                const float* s = ok ? src + ((size_t)gc * p.H + gy) * p.W + gx : p.x;
                cp_async4(dst + ci * G::CHS + hr * G::HP + hc, s, ok);
            }
            cp_async_commit();
        };

        if (!p.use_tma && pseq_tile < p.total_tiles) fetch(pseq_tile, 0, 0);
        int seq = 0, tile = blockIdx.x, ch = 0, abuf = 0, t = 0;
        uint32_t aphase = 0;
        for (; tile < p.total_tiles; ++seq) {
            // A stage = tile parity (each MMA issuer owns one stage); its use
            // number u counts the chunks written into it so far.  Halo buffers
            // alternate per chunk.
            const int stage = t & 1;
            const uint32_t upar = (uint32_t)(((t >> 1) * p.nchunks + ch) & 1);
            const int hbuf = seq & 1;
            const uint32_t par = (seq >> 1) & 1;
            // The MMAs that read this A stage last have completed, the halo has
            // landed and, for a tile's first chunk, the epilogue has drained the
            // accumulator this tile will use: the MMA issuers then wait on
            // "A full" alone.  One thread waits (bounded) before the barrier, so
            // the abort decision after it is the same for all.
            if (tid == 0 && !wait_bounded(bar_aempty + 8 * stage, upar ^ 1, abort_flag)) *prod_abort = 1u;
            if (tid == 0 && ch == 0 && !wait_bounded(bar_accempty + 8 * abuf, aphase ^ 1, abort_flag))
                *prod_abort = 1u;
            if (p.use_tma) {
                if (tid == 0 && !wait_bounded(bar_hfull + 8 * hbuf, par, abort_flag)) *prod_abort = 1u;
            } else {
                cp_async_wait<0>();
            }
            asm volatile("bar.sync 1, 256;\n" ::: "memory");  // halo landed, stage free
            if (*prod_abort) break;
            if (p.use_tma) {
                for (int spin = 0; !mbar_try_wait(bar_hfull + 8 * hbuf, par) && spin < (1 << 20); ++spin) {
                }
            }
            // tcgen05.fence::after_thread_sync behind the barrier orders this
            // thread's TMEM writes after the MMAs thread 0 saw complete.
            tc_fence_after();
            if (!p.use_tma) {
                // Fetch the next (tile, chunk) halo into the other buffer.
                if (++pseq_ch == p.nchunks) {
                    pseq_ch = 0;
                    pseq_tile += gridDim.x;
                }
                if (pseq_tile < p.total_tiles) fetch(pseq_tile, pseq_ch, hbuf ^ 1);
            }

            // im2col row of position (r, c): 72 values, 8 per TMEM store; the two
            // warps of a lane quarter take K groups 0-4 and 5-8.  A_hi is the raw
            // fp32 value (the MMA reads only its TF32 bits, i.e. truncates it);
            // A_lo = v - truncate(v) is exact.
            const float* hb = halo + hbuf * G::HALO + r * G::HP + c;
            const uint32_t a_hi = tmem + lane_base + a_col0 + (uint32_t)(stage * A_COLS);
            auto build = [&](auto g0c, auto g1c) {
                constexpr int g0 = decltype(g0c)::value, g1 = decltype(g1c)::value;
#pragma unroll
                for (int g = g0; g < g1; ++g) {
                    uint32_t hi[8], lo[8];
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        const int e = 8 * g + q;
                        const int ci = e / 9, t = e % 9;
                        const float v = hb[ci * G::CHS + (t / 3) * G::HP + (t % 3)];
                        hi[q] = __float_as_uint(v);
                        lo[q] = __float_as_uint(v - __uint_as_float(hi[q] & 0xFFFFE000u));
                    }
                    tmem_st8(a_hi + (uint32_t)(8 * g), hi);
                    tmem_st8(a_hi + (uint32_t)(KCH + 8 * g), lo);
                }
            };
            if (half == 0) build(std::integral_constant<int, 0>{}, std::integral_constant<int, 5>{});
            else build(std::integral_constant<int, 5>{}, std::integral_constant<int, KST>{});
            __syncwarp();
            if (p.use_tma && lane == 0) mbar_arrive(bar_hempty + 8 * hbuf);  // this warp is done with the halo
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar_afull + 8 * stage);
            if (++ch == p.nchunks) {
                ch = 0;
                tile += gridDim.x;
                ++t;
                if (++abuf == p.nacc) {
                    abuf = 0;
                    aphase ^= 1u;
                }
            }
        }
        cp_async_wait<0>();  // no copy may land after the CTA has left
    } else if (warp == TMA_WARP) {
        tma_halo_warp<P>(p, x_map, halo, bar_hfull, bar_hempty, abort_flag, lane);
    } else if (warp == MMA_WARP || warp == MMA_WARP2) {
        // --------------------------------------------------------- MMA issuers
        // Two issuing threads, one for the even and one for the odd tiles of this
        // CTA: while one waits on a barrier the other keeps the tensor core fed.
        // Each commit tracks the issuing thread's own MMAs, which is what every
        // barrier here needs (a stage or accumulator is used by one tile).
        if (lane == 0) {
            const int par = warp == MMA_WARP ? 0 : 1;
            const uint32_t idesc = (1u << 4) | (2u << 7) | (2u << 10) | ((uint32_t)(NP >> 3) << 17) |
                                   ((uint32_t)(MT >> 4) << 24);
            // B descriptors of chunk 0's nine K-steps, computed once: the issue
            // loop then spends a few instructions per MMA, so the tensor core,
            // not this thread, sets the pace.
            uint64_t bh0[KST], bl0[KST];
#pragma unroll
            for (int kk = 0; kk < KST; ++kk) {
                const uint32_t boff = (uint32_t)(kk >> 2) * NP * 128u + 32u * (uint32_t)(kk & 3);
                bh0[kk] = sw128_desc(sbase + L.b_hi + boff);
                bl0[kk] = sw128_desc(sbase + L.b_lo + boff);
            }
            const uint64_t chunk_step = (uint64_t)(3u * NP * 128u) >> 4;  // descriptor address units
            int abuf = par % p.nacc;
            bool ok = true;
            for (int t = par, tile = blockIdx.x + par * gridDim.x; ok && tile < p.total_tiles;
                 t += 2, tile += 2 * gridDim.x) {
                const int buf = abuf;  // drained: the producers saw it before "A full"
                abuf = (abuf + 2) % p.nacc;
                const uint32_t d_tmem = tmem + (uint32_t)(buf * NP);
                int seq = t * p.nchunks;
                const int stage = par;  // = t & 1
                for (int ch = 0; ch < p.nchunks; ++ch, ++seq) {
                    const uint32_t upar = (uint32_t)(((t >> 1) * p.nchunks + ch) & 1);
                    if (!wait_bounded(bar_afull + 8 * stage, upar, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t ah = tmem + a_col0 + (uint32_t)(stage * A_COLS), al = ah + (uint32_t)KCH;
                    const uint64_t cofs = chunk_step * (uint64_t)ch;
                    mma_tf32_ts(d_tmem, ah, bh0[0] + cofs, idesc, ch > 0 ? 1u : 0u);
                    mma_tf32_ts_acc(d_tmem, ah, bl0[0] + cofs, idesc);
                    mma_tf32_ts_acc(d_tmem, al, bh0[0] + cofs, idesc);
#pragma unroll
                    for (int kk = 1; kk < KST; ++kk) {
                        mma_tf32_ts_acc(d_tmem, ah + 8u * kk, bh0[kk] + cofs, idesc);
                        mma_tf32_ts_acc(d_tmem, ah + 8u * kk, bl0[kk] + cofs, idesc);
                        mma_tf32_ts_acc(d_tmem, al + 8u * kk, bh0[kk] + cofs, idesc);
                    }
                    tc_commit(bar_aempty + 8 * stage);  // A stage free once these MMAs are done
                }
                if (ok) tc_commit(bar_accfull + 8 * buf);
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
    } else {
        epilogue_warps<P, MODE>(p, tbuf, bias_s, tmem, bar_accfull, bar_accempty, bar_tfull, bar_tempty, abort_flag,
                                warp, lane);
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == MMA_WARP) {
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tmem), "r"(TMEM_COLS)
                     : "memory");
    }
}

template <int P, int MODE>
__global__ void __launch_bounds__(NTHREADS, 1) conv2d_tc4_kernel(const Params p, const __grid_constant__ CUtensorMap x_map)
{
    using G = Geo<P>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    const uint32_t sbase = smem_u32(smem);
    const Layout L = make_layout<P>(p.NP, p.natoms);
    float* halo = reinterpret_cast<float*>(smem + L.halo);
    float* tbuf = reinterpret_cast<float*>(smem + L.tbuf);
    float* bias_s = reinterpret_cast<float*>(smem + L.bias);
    const uint32_t bar_afull = sbase + L.bar;         // + 8 * stage (4), 4 producer-warp arrivals
    const uint32_t bar_aempty = bar_afull + 32;       // + 8 * stage (4), tcgen05.commit
    const uint32_t bar_accfull = bar_afull + 64;      // + 8 * buf (3), tcgen05.commit
    const uint32_t bar_accempty = bar_afull + 88;     // + 8 * buf (3), 4 drain-warp arrivals
    const uint32_t bar_drain = bar_afull + 112;
    const uint32_t bar_hfull = bar_afull + 120;       // + 8 * buf, TMA halo landed
    const uint32_t bar_hempty = bar_afull + 136;      // + 8 * buf, 8 producer-warp arrivals
    const uint32_t bar_tfull = bar_afull + 152;       // + 8 * buf, 4 drain-warp arrivals
    const uint32_t bar_tempty = bar_afull + 168;      // + 8 * buf, 8 pool-warp arrivals
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + L.misc);
    volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(smem + L.misc + 4);
    volatile uint32_t* prod_abort = reinterpret_cast<volatile uint32_t*>(smem + L.misc + 8);  // [2], one per group

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int NP = p.NP;

    if (threadIdx.x == 0) {
        for (int i = 0; i < 4; ++i) {
            mbar_init(bar_afull + 8 * i, 4);
            mbar_init(bar_aempty + 8 * i, 1);
        }
        for (int i = 0; i < 3; ++i) {
            mbar_init(bar_accfull + 8 * i, 1);
            mbar_init(bar_accempty + 8 * i, 4);
        }
        mbar_init(bar_drain, 2);  // one commit per MMA issuer
        mbar_init(bar_hfull, 1);
        mbar_init(bar_hfull + 8, 1);
        mbar_init(bar_hempty, 8);
        mbar_init(bar_hempty + 8, 8);
        mbar_init(bar_tfull, 4);
        mbar_init(bar_tfull + 8, 4);
        mbar_init(bar_tempty, 8);
        mbar_init(bar_tempty + 8, 8);
        *abort_flag = 0u;
        prod_abort[0] = 0u;
        prod_abort[1] = 0u;
        asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
    }
    if (warp == MMA_WARP) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(smem_u32(tmem_holder)),
                     "r"(TMEM_COLS)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::: "memory");
    }

    stage_weights<P>(p, smem, L, bias_s);
    asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");  // weights visible to the tensor core
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;
    // Accumulators: p.nacc buffers of NP columns (3 when they fit next to the
    // four sub-chunk A stages, else 2), used round robin: buffer abuf, phase aphase.
    const uint32_t a_col0 = (uint32_t)(p.nacc * NP);  // first A-stage column (4 stages of SUB_COLS)

    if (warp < 8) {
        // ------------------------------------------------------------ producers
        // Two independent groups of four warps, one per K sub-chunk (K-steps
        // 0-4 and 5-8 of every chunk); warp w of a group owns TMEM lane quarter
        // w & 3.  Sub-chunk s of a tile with parity q goes to A stage 2q + s, so a
        // group rebuilds its sub-stage as soon as the MMAs that read it are done,
        // whatever the other group is doing.
        const int grp = warp >> 2;                 // sub-chunk of this group
        const int gtid = threadIdx.x - 128 * grp;  // 0..127
        const int m = 32 * (warp & 3) + lane;      // conv position = TMEM lane
        const int r = m / G::WC, c = m - (m / G::WC) * G::WC;
        const uint32_t lane_base = (uint32_t)(32 * (warp & 3)) << 16;
        int seq = 0, tile = blockIdx.x, ch = 0, abuf = 0, t = 0;
        uint32_t aphase = 0;
        for (; tile < p.total_tiles; ++seq) {
            const int stage = 2 * (t & 1) + grp;
            const uint32_t upar = (uint32_t)(((t >> 1) * p.nchunks + ch) & 1);
            const int hbuf = seq & 1;
            const uint32_t hpar = (seq >> 1) & 1;
            // This sub-stage's last MMAs are done, the halo has landed and, for
            // sub-chunk 0 of a tile's first chunk, the accumulator the tile will
            // reset is drained.  The group's first thread waits (bounded) before
            // the group barrier, so the abort decision after it is the group's.
            if (gtid == 0) {
                if (!wait_bounded(bar_aempty + 8 * stage, upar ^ 1, abort_flag)) prod_abort[grp] = 1u;
                else if (!wait_bounded(bar_hfull + 8 * hbuf, hpar, abort_flag)) prod_abort[grp] = 1u;
                else if (grp == 0 && ch == 0 && !wait_bounded(bar_accempty + 8 * abuf, aphase ^ 1, abort_flag))
                    prod_abort[grp] = 1u;
            }
            if (grp == 0) asm volatile("bar.sync 1, 128;\n" ::: "memory");
            else asm volatile("bar.sync 3, 128;\n" ::: "memory");
            if (prod_abort[grp]) break;
            for (int spin = 0; !mbar_try_wait(bar_hfull + 8 * hbuf, hpar) && spin < (1 << 20); ++spin) {
            }
            tc_fence_after();
            // im2col values of position (r, c) for this sub-chunk's K groups, 8 per
            // TMEM store; A_hi is the raw fp32 value (the MMA reads its TF32
            // bits), A_lo = v - truncate(v) is exact.
            const float* hb = halo + hbuf * G::HALO + r * G::HP + c;
            const uint32_t a_st = tmem + lane_base + a_col0 + (uint32_t)(stage * SUB_COLS);
            auto build = [&](auto g0c, auto g1c) {
                constexpr int g0 = decltype(g0c)::value, g1 = decltype(g1c)::value;
#pragma unroll
                for (int g = g0; g < g1; ++g) {
                    uint32_t hi[8], lo[8];
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        const int e = 8 * g + q;
                        const int ci = e / 9, tt = e % 9;
                        const float v = hb[ci * G::CHS + (tt / 3) * G::HP + (tt % 3)];
                        hi[q] = __float_as_uint(v);
                        lo[q] = __float_as_uint(v - __uint_as_float(hi[q] & 0xFFFFE000u));
                    }
                    tmem_st8(a_st + (uint32_t)(8 * (g - g0)), hi);
                    tmem_st8(a_st + (uint32_t)(SUB_LO + 8 * (g - g0)), lo);
                }
            };
            if (grp == 0) build(std::integral_constant<int, 0>{}, std::integral_constant<int, SUB0>{});
            else build(std::integral_constant<int, SUB0>{}, std::integral_constant<int, KST>{});
            __syncwarp();
            if (lane == 0) mbar_arrive(bar_hempty + 8 * hbuf);  // this warp is done with the halo
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar_afull + 8 * stage);
            if (++ch == p.nchunks) {
                ch = 0;
                tile += gridDim.x;
                ++t;
                if (++abuf == p.nacc) {
                    abuf = 0;
                    aphase ^= 1u;
                }
            }
        }
    } else if (warp == TMA_WARP) {
        tma_halo_warp<P>(p, x_map, halo, bar_hfull, bar_hempty, abort_flag, lane);
    } else if (warp == MMA_WARP || warp == MMA_WARP2) {
        // --------------------------------------------------------- MMA issuers
        // Two issuing threads, one for the even and one for the odd tiles of this
        // CTA: while one waits on a barrier the other keeps the tensor core fed.
        // Each commit tracks the issuing thread's own MMAs, which is what every
        // barrier here needs (a stage or accumulator is used by one tile).
        if (lane == 0) {
            const int par = warp == MMA_WARP ? 0 : 1;
            const uint32_t idesc = (1u << 4) | (2u << 7) | (2u << 10) | ((uint32_t)(NP >> 3) << 17) |
                                   ((uint32_t)(MT >> 4) << 24);
            // B descriptors of chunk 0's nine K-steps, computed once: the issue
            // loop then spends a few instructions per MMA, so the tensor core,
            // not this thread, sets the pace.
            uint64_t bh0[KST], bl0[KST];
#pragma unroll
            for (int kk = 0; kk < KST; ++kk) {
                const uint32_t boff = (uint32_t)(kk >> 2) * NP * 128u + 32u * (uint32_t)(kk & 3);
                bh0[kk] = sw128_desc(sbase + L.b_hi + boff);
                bl0[kk] = sw128_desc(sbase + L.b_lo + boff);
            }
            const uint64_t chunk_step = (uint64_t)(3u * NP * 128u) >> 4;  // descriptor address units
            int abuf = par % p.nacc;
            bool ok = true;
            for (int t = par, tile = blockIdx.x + par * gridDim.x; ok && tile < p.total_tiles;
                 t += 2, tile += 2 * gridDim.x) {
                const int buf = abuf;  // drained: the producers saw it before "A full"
                abuf = (abuf + 2) % p.nacc;
                const uint32_t d_tmem = tmem + (uint32_t)(buf * NP);
                for (int ch = 0; ch < p.nchunks && ok; ++ch) {
                    const uint32_t upar = (uint32_t)(((t >> 1) * p.nchunks + ch) & 1);
                    const uint64_t cofs = chunk_step * (uint64_t)ch;
                    // sub-chunk 0: K-steps 0 .. SUB0-1, in A stage 2 * par
                    {
                        const int stage = 2 * par;
                        if (!wait_bounded(bar_afull + 8 * stage, upar, abort_flag)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        const uint32_t ah = tmem + a_col0 + (uint32_t)(stage * SUB_COLS), al = ah + (uint32_t)SUB_LO;
                        mma_tf32_ts(d_tmem, ah, bh0[0] + cofs, idesc, ch > 0 ? 1u : 0u);
                        mma_tf32_ts_acc(d_tmem, ah, bl0[0] + cofs, idesc);
                        mma_tf32_ts_acc(d_tmem, al, bh0[0] + cofs, idesc);
#pragma unroll
                        for (int j = 1; j < SUB0; ++j) {
                            mma_tf32_ts_acc(d_tmem, ah + 8u * j, bh0[j] + cofs, idesc);
                            mma_tf32_ts_acc(d_tmem, ah + 8u * j, bl0[j] + cofs, idesc);
                            mma_tf32_ts_acc(d_tmem, al + 8u * j, bh0[j] + cofs, idesc);
                        }
                        tc_commit(bar_aempty + 8 * stage);
                    }
                    // sub-chunk 1: K-steps SUB0 .. 8, in A stage 2 * par + 1
                    {
                        const int stage = 2 * par + 1;
                        if (!wait_bounded(bar_afull + 8 * stage, upar, abort_flag)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        const uint32_t ah = tmem + a_col0 + (uint32_t)(stage * SUB_COLS), al = ah + (uint32_t)SUB_LO;
#pragma unroll
                        for (int j = 0; j < KST - SUB0; ++j) {
                            mma_tf32_ts_acc(d_tmem, ah + 8u * j, bh0[SUB0 + j] + cofs, idesc);
                            mma_tf32_ts_acc(d_tmem, ah + 8u * j, bl0[SUB0 + j] + cofs, idesc);
                            mma_tf32_ts_acc(d_tmem, al + 8u * j, bh0[SUB0 + j] + cofs, idesc);
                        }
                        tc_commit(bar_aempty + 8 * stage);
                    }
                }
                if (ok) tc_commit(bar_accfull + 8 * buf);
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
    } else {
        epilogue_warps<P, MODE>(p, tbuf, bias_s, tmem, bar_accfull, bar_accempty, bar_tfull, bar_tempty, abort_flag,
                                warp, lane);
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == MMA_WARP) {
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tmem), "r"(TMEM_COLS)
                     : "memory");
    }
}

}  // namespace c2tc

inline bool conv2d_tc_pool_ok(int P) { return P == 1 || P == 2 || P == 4 || P == 8; }

template <int P>
inline uint32_t conv2d_tc_smem(int Cin, int Cout)
{
    const int NP = (Cout + 15) & ~15;
    const int nchunks = (Cin + c2tc::CCH - 1) / c2tc::CCH;
    const int natoms = 3 * nchunks;
    return c2tc::make_layout<P>(NP, natoms).total + 1024u;
}

// Shapes the tensor-core conv2d covers: pool 1, 2, 4 or 8, Cout <= 112 and a
// weight operand that fits shared memory next to the buffers.
inline bool conv2d_tc_supported(int Cin, int Cout, int P)
{
    if (!conv2d_tc_pool_ok(P) || Cout < 1 || Cout > c2tc::NP_MAX || Cin < 1) return false;
    uint32_t s = 0;
    switch (P) {
    case 1: s = conv2d_tc_smem<1>(Cin, Cout); break;
    case 2: s = conv2d_tc_smem<2>(Cin, Cout); break;
    case 4: s = conv2d_tc_smem<4>(Cin, Cout); break;
    default: s = conv2d_tc_smem<8>(Cin, Cout); break;
    }
    return s <= (uint32_t)c2tc::SMEM_LIMIT;
}

// What one launch of the tensor-core conv2d uses for given sizes: the kernel
// (the sub-chunk kernel when the halo comes by TMA and Cout' <= 96), its
// accumulator count, the TMEM columns it addresses of the 512 it allocates,
// and the dynamic shared memory it requests.
struct Conv2dTcPlan {
    int sub;          // 1: conv2d_tc4_kernel, 0: conv2d_tc_kernel
    int NP;           // Cout rounded up to 16 (MMA N)
    int nacc;         // accumulator buffers of NP columns
    int tmem_cols;    // accumulators + A stages
    uint32_t smem;    // bytes, including the 1 KB alignment slack
};

template <int P>
inline Conv2dTcPlan conv2d_tc_plan(int Cin, int Cout, bool use_tma)
{
    Conv2dTcPlan pl;
    pl.NP = (Cout + 15) & ~15;
    pl.sub = (use_tma && pl.NP <= c2tc::NP_MAX_SUB) ? 1 : 0;
    const int a_cols = pl.sub ? 4 * c2tc::SUB_COLS : 2 * c2tc::A_COLS;
    pl.nacc = (3 * pl.NP + a_cols <= (int)c2tc::TMEM_COLS) ? 3 : 2;
    pl.tmem_cols = pl.nacc * pl.NP + a_cols;
    // At least 120 KB, so that two CTAs never share an SM: each allocates all
    // 512 TMEM columns.
    pl.smem = conv2d_tc_smem<P>(Cin, Cout);
    if (pl.smem < 120u * 1024u) pl.smem = 120u * 1024u;
    return pl;
}

inline bool conv2d_tc_plan_for(int Cin, int Cout, int P, bool use_tma, Conv2dTcPlan* pl)
{
    switch (P) {
    case 1: *pl = conv2d_tc_plan<1>(Cin, Cout, use_tma); return true;
    case 2: *pl = conv2d_tc_plan<2>(Cin, Cout, use_tma); return true;
    case 4: *pl = conv2d_tc_plan<4>(Cin, Cout, use_tma); return true;
    case 8: *pl = conv2d_tc_plan<8>(Cin, Cout, use_tma); return true;
    default: return false;
    }
}

template <int P, int MODE>
inline int launch_conv2d_tc_p(c2tc::Params prm, int N, int grid, cudaStream_t stream)
{
    // x [N][Cin][H][W] as a 4-D tensor; one box is the halo of one (tile,
    // chunk): HP columns x (P + 2) rows x 8 channels x 1 image.  Needs 16-byte
    // row strides (W % 4 == 0) and an aligned x; otherwise cp.async stages it.
    CUtensorMap map;
    memset(&map, 0, sizeof(map));
    prm.use_tma = 0;
    if ((prm.W & 3) == 0 && (reinterpret_cast<uintptr_t>(prm.x) & 15) == 0) {
        auto encode = tensor_map_encoder();
        if (!encode) return FCV_ERR_CUDA;
        using G = c2tc::Geo<P>;
        const cuuint64_t gdim[4] = {(cuuint64_t)prm.W, (cuuint64_t)prm.H, (cuuint64_t)prm.Cin, (cuuint64_t)N};
        const cuuint64_t gstride[3] = {(cuuint64_t)prm.W * 4, (cuuint64_t)prm.H * prm.W * 4,
                                       (cuuint64_t)prm.Cin * prm.H * prm.W * 4};
        const cuuint32_t box[4] = {(cuuint32_t)G::HP, (cuuint32_t)G::HR, (cuuint32_t)c2tc::CCH, 1};
        const cuuint32_t estride[4] = {1, 1, 1, 1};
        if (encode(&map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, const_cast<float*>(prm.x), gdim, gstride, box, estride,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return FCV_ERR_CUDA;
        prm.use_tma = 1;
    }
    // With the halo by TMA and Cout <= 96, the sub-chunk kernel: four smaller A
    // stages let a producer group refill half a chunk while the MMAs of the
    // other half run.
    const Conv2dTcPlan pl = conv2d_tc_plan<P>(prm.Cin, prm.Cout, prm.use_tma != 0);
    prm.nacc = pl.nacc;
    auto kern = pl.sub ? c2tc::conv2d_tc4_kernel<P, MODE> : c2tc::conv2d_tc_kernel<P, MODE>;
    return launch_cached(kern, (int)pl.smem, [&] { kern<<<grid, c2tc::NTHREADS, pl.smem, stream>>>(prm, map); });
}

// MODE: kSumAtomic (out[N], zeroed by the caller) or kTap (pooled values).
template <int MODE>
inline int launch_conv2d_tc(const float* x, const float* w, const float* b, int N, int Cin, int H, int W, int Cout,
                            int P, int PH, int PW, float* out, cudaStream_t stream)
{
    if (!conv2d_tc_supported(Cin, Cout, P)) return FCV_ERR_UNSUPPORTED;
    c2tc::Params prm;
    prm.x = x; prm.w = w; prm.b = b; prm.out = out;
    prm.Cin = Cin; prm.H = H; prm.W = W; prm.Cout = Cout; prm.PH = PH; prm.PW = PW;
    prm.NP = (Cout + 15) & ~15;
    prm.nchunks = (Cin + c2tc::CCH - 1) / c2tc::CCH;
    prm.natoms = 3 * prm.nchunks;
    const int wpt = c2tc::MT / (P * P);
    prm.tiles_x = (PW + wpt - 1) / wpt;
    const long long per_img = (long long)PH * prm.tiles_x;
    const long long total = per_img * N;
    if (total > 0x7fffffffLL) return FCV_ERR_UNSUPPORTED;
    prm.tiles_img = (int)per_img;
    prm.total_tiles = (int)total;
    prm.use_tma = 0;
    prm.nacc = 2;  // set with the kernel choice in launch_conv2d_tc_p
    int sms = 0;
    if (device_sm_count(&sms) != FCV_OK) return FCV_ERR_CUDA;
    const int grid = (int)(total < sms ? total : sms);
    switch (P) {
    case 1: return launch_conv2d_tc_p<1, MODE>(prm, N, grid, stream);
    case 2: return launch_conv2d_tc_p<2, MODE>(prm, N, grid, stream);
    case 4: return launch_conv2d_tc_p<4, MODE>(prm, N, grid, stream);
    default: return launch_conv2d_tc_p<8, MODE>(prm, N, grid, stream);
    }
}

}  // namespace fcv
