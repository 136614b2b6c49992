// conv1d_fma.cuh -- op B on FP32 FMA: depthwise conv1d folded into the pointwise conv1d.
//
// Method (POPCORNBENCH trace "Kimi-K2.6__l2_p7", tile-GEMM formulation): for
// each chunk of input channels, compute the depthwise result d[c, t] of the
// output tile into shared memory, then accumulate the pointwise contraction
// out[o, t] += pw[o, c] * d[c, t] as a sum of rank-1 updates.  The depthwise
// value of each (c, t) is formed once per CTA (not once per output channel as
// in the trace's first per-channel-halo kernel) and never leaves the chip.
//
// Tiling: a CTA owns out[n, o0:o0+OT, t0:t0+TT]; each thread an RO x RT
// register block (RO output channels x RT consecutive times).  Per chunk of
// CC channels the CTA stages the input halo x[n, c, t0*s-p : ...] (zero
// outside [0, T)), the depthwise weights, and pw transposed to [c][o], so the
// inner loop is two 16-byte shared loads per RO*RT FMAs.
#pragma once

#include "common.cuh"

namespace fcv {

struct Conv1dFmaTile {
    static constexpr int OT = 128, TT = 128, CC = 16, RO = 8, RT = 8;
    static constexpr int NT = (OT / RO) * (TT / RT);  // 256 threads
    static constexpr int KMAX = 32, SMAX = 16;
};

template <int S_FIXED>
__global__ void __launch_bounds__(Conv1dFmaTile::NT, 2)
dwsep_conv1d_fma_kernel(const float* __restrict__ x, const float* __restrict__ dw,
                        const float* __restrict__ pw, const float* __restrict__ bias,
                        int C, int T, int O, int K, int s_rt, int pad, int To,
                        int tiles_t, int tiles_o, float* __restrict__ out)
{
    using G = Conv1dFmaTile;
    constexpr int OT = G::OT, TT = G::TT, CC = G::CC, RO = G::RO, RT = G::RT, NT = G::NT;
    const int s = S_FIXED > 0 ? S_FIXED : s_rt;
    const int XW = (TT - 1) * s + K;  // halo samples per channel
    const int XWP = (XW + 3) & ~3;

    extern __shared__ __align__(16) float smem[];
    float* pws = smem;                 // [CC][OT]  pw transposed
    float* ds = pws + CC * OT;         // [CC][TT]  depthwise result
    float* dws = ds + CC * TT;         // [CC][KMAX]
    float* xs = dws + CC * G::KMAX;    // [CC][XWP] input halo

    int blk = blockIdx.x;
    const int tt_tile = blk % tiles_t;
    blk /= tiles_t;
    const int to_tile = blk % tiles_o;
    const int n = blk / tiles_o;
    const int t0 = tt_tile * TT, o0 = to_tile * OT;
    const long long xbeg = (long long)t0 * s - pad;  // first input sample of the halo

    const int tid = threadIdx.x;
    const int tcol = tid % (TT / RT), orow = tid / (TT / RT);

    float acc[RO][RT];
#pragma unroll
    for (int i = 0; i < RO; ++i)
#pragma unroll
        for (int j = 0; j < RT; ++j) acc[i][j] = 0.f;

    const float* xn = x + (size_t)n * C * T;

    for (int c0 = 0; c0 < C; c0 += CC) {
        for (int i = tid; i < CC * XW; i += NT) {
            const int cl = i / XW, j = i - (i / XW) * XW;
            const int c = c0 + cl;
            const long long ti = xbeg + j;
            xs[cl * XWP + j] = (c < C && ti >= 0 && ti < T) ? __ldg(xn + (size_t)c * T + ti) : 0.f;
        }
        for (int i = tid; i < CC * G::KMAX; i += NT) {
            const int cl = i / G::KMAX, k = i % G::KMAX;
            const int c = c0 + cl;
            dws[i] = (c < C && k < K) ? __ldg(dw + (size_t)c * K + k) : 0.f;
        }
        for (int i = tid; i < CC * OT; i += NT) {
            const int cl = i % CC, ol = i / CC;  // consecutive threads read consecutive c
            const int c = c0 + cl, o = o0 + ol;
            pws[cl * OT + ol] = (c < C && o < O) ? __ldg(pw + (size_t)o * C + c) : 0.f;
        }
        __syncthreads();
        // Depthwise: each (c, t) of the tile once.
        for (int i = tid; i < CC * TT; i += NT) {
            const int cl = i / TT, tl = i % TT;
            const float* xr = xs + cl * XWP + tl * s;
            const float* wr = dws + cl * G::KMAX;
            float d = 0.f;
            for (int k = 0; k < K; ++k) d = fmaf(xr[k], wr[k], d);
            ds[i] = d;
        }
        __syncthreads();
        // Pointwise: rank-1 updates over the chunk.
#pragma unroll 4
        for (int cl = 0; cl < CC; ++cl) {
            float a[RO], bv[RT];
            const float4* ap = reinterpret_cast<const float4*>(pws + cl * OT + orow * RO);
            const float4* bp = reinterpret_cast<const float4*>(ds + cl * TT + tcol * RT);
#pragma unroll
            for (int q = 0; q < RO / 4; ++q) {
                const float4 v = ap[q];
                a[4 * q] = v.x; a[4 * q + 1] = v.y; a[4 * q + 2] = v.z; a[4 * q + 3] = v.w;
            }
#pragma unroll
            for (int q = 0; q < RT / 4; ++q) {
                const float4 v = bp[q];
                bv[4 * q] = v.x; bv[4 * q + 1] = v.y; bv[4 * q + 2] = v.z; bv[4 * q + 3] = v.w;
            }
#pragma unroll
            for (int i = 0; i < RO; ++i)
#pragma unroll
                for (int j = 0; j < RT; ++j) acc[i][j] = fmaf(a[i], bv[j], acc[i][j]);
        }
        __syncthreads();
    }

    // Epilogue: + bias, store along t.
#pragma unroll
    for (int i = 0; i < RO; ++i) {
        const int o = o0 + orow * RO + i;
        if (o >= O) continue;
        const float bo = bias ? __ldg(bias + o) : 0.f;
        float* orow_p = out + ((size_t)n * O + o) * To;
#pragma unroll
        for (int j = 0; j < RT; ++j) {
            const int t = t0 + tcol * RT + j;
            if (t < To) orow_p[t] = acc[i][j] + bo;
        }
    }
}

inline size_t conv1d_fma_smem_bytes(int K, int s)
{
    using G = Conv1dFmaTile;
    const int XW = (G::TT - 1) * s + K;
    const int XWP = (XW + 3) & ~3;
    return sizeof(float) * ((size_t)G::CC * G::OT + G::CC * G::TT + G::CC * G::KMAX + (size_t)G::CC * XWP);
}

inline int launch_dwsep_conv1d_fma(const float* x, const float* dw, const float* pw, const float* bias,
                                   int N, int C, int T, int O, int K, int s, int pad, int To,
                                   float* out, cudaStream_t stream)
{
    using G = Conv1dFmaTile;
    const int tiles_t = (To + G::TT - 1) / G::TT;
    const int tiles_o = (O + G::OT - 1) / G::OT;
    const long long nblk = (long long)N * tiles_t * tiles_o;
    if (nblk > 0x7fffffffLL) return FCV_ERR_UNSUPPORTED;
    const size_t smem = conv1d_fma_smem_bytes(K, s);
    auto kern = (s == 1) ? dwsep_conv1d_fma_kernel<1> : dwsep_conv1d_fma_kernel<0>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
        return FCV_ERR_CUDA;
    kern<<<(unsigned)nblk, G::NT, smem, stream>>>(x, dw, pw, bias, C, T, O, K, s, pad, To, tiles_t,
                                                  tiles_o, out);
    return launch_status();
}

}  // namespace fcv
