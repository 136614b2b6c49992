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
// inner loop is two 16-byte shared loads per RO*RT FMAs.  Chunks are double
// buffered: the cp.async copies of chunk i+1 are in flight while chunk i is
// computed.
//
// This is the FP32-FMA path; it covers every supported shape and serves as
// the fallback of the tensor-core path.
#pragma once

#include "common.cuh"

namespace fcv {

struct Conv1dFmaTile {
    static constexpr int OT = 128, TT = 128, CC = 16, RO = 8, RT = 8;
    static constexpr int NT = (OT / RO) * (TT / RT);  // 256 threads
    static constexpr int KMAX = 32, SMAX = 8;
};

struct Conv1dFmaSmem {
    int xwp;       // halo row pitch (floats)
    int buf;       // floats per staging buffer: pws + dws + xs
    size_t bytes;  // total dynamic shared memory
};

inline __host__ __device__ Conv1dFmaSmem conv1d_fma_smem(int K, int s)
{
    using G = Conv1dFmaTile;
    Conv1dFmaSmem m;
    m.xwp = (((G::TT - 1) * s + K) + 3) & ~3;
    m.buf = G::CC * G::OT + G::CC * G::KMAX + G::CC * m.xwp;
    m.bytes = sizeof(float) * ((size_t)2 * m.buf + (size_t)G::CC * G::TT);
    return m;
}

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
    const Conv1dFmaSmem L = conv1d_fma_smem(K, s);

    extern __shared__ __align__(16) float smem[];
    // staging buffer b: pws [CC][OT] (pw transposed) | dws [CC][KMAX] | xs [CC][xwp]
    float* ds = smem + 2 * L.buf;      // [CC][TT] depthwise result

    int blk = blockIdx.x;
    const int tt_tile = blk % tiles_t;
    blk /= tiles_t;
    const int to_tile = blk % tiles_o;
    const int n = blk / tiles_o;
    const int t0 = tt_tile * TT, o0 = to_tile * OT;
    const long long xbeg = (long long)t0 * s - pad;  // first input sample of the halo

    const int tid = threadIdx.x;
    const int tcol = tid % (TT / RT), orow = tid / (TT / RT);
    const float* xn = x + (size_t)n * C * T;

    auto stage = [&](int c0, int b) {
        float* pws = smem + b * L.buf;
        float* dws = pws + CC * OT;
        float* xs = dws + CC * G::KMAX;
        for (int i = tid; i < CC * XW; i += NT) {
            const int cl = i / XW, j = i - (i / XW) * XW;
            const int c = c0 + cl;
            const long long ti = xbeg + j;
            const bool in = c < C && ti >= 0 && ti < T;
            cp_async4(xs + cl * L.xwp + j, in ? xn + (size_t)c * T + ti : x, in);
        }
        for (int i = tid; i < CC * G::KMAX; i += NT) {
            const int cl = i / G::KMAX, k = i % G::KMAX;
            const int c = c0 + cl;
            const bool in = c < C && k < K;
            cp_async4(dws + i, in ? dw + (size_t)c * K + k : dw, in);
        }
        for (int i = tid; i < CC * OT; i += NT) {
            const int cl = i % CC, ol = i / CC;  // consecutive threads read consecutive c
            const int c = c0 + cl, o = o0 + ol;
            const bool in = c < C && o < O;
            cp_async4(pws + cl * OT + ol, in ? pw + (size_t)o * C + c : pw, in);
        }
        cp_async_commit();
    };

    float acc[RO][RT];
#pragma unroll
    for (int i = 0; i < RO; ++i)
#pragma unroll
        for (int j = 0; j < RT; ++j) acc[i][j] = 0.f;

    const int nchunks = (C + CC - 1) / CC;
    stage(0, 0);
    for (int k = 0; k < nchunks; ++k) {
        const int b = k & 1;
        if (k + 1 < nchunks) {
            stage((k + 1) * CC, b ^ 1);  // the buffer was released by the barrier ending chunk k-1
            cp_async_wait<1>();
        } else {
            cp_async_wait<0>();
        }
        __syncthreads();
        const float* pws = smem + b * L.buf;
        const float* dws = pws + CC * OT;
        const float* xs = dws + CC * G::KMAX;
        // Depthwise: each (c, t) of the tile once.
        for (int i = tid; i < CC * TT; i += NT) {
            const int cl = i / TT, tl = i % TT;
            const float* xr = xs + cl * L.xwp + tl * s;
            const float* wr = dws + cl * G::KMAX;
            float d = 0.f;
            for (int kk = 0; kk < K; ++kk) d = fmaf(xr[kk], wr[kk], d);
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
        __syncthreads();  // ds and staging buffer b are free again
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

inline int launch_dwsep_conv1d_fma(const float* x, const float* dw, const float* pw, const float* bias,
                                   int N, int C, int T, int O, int K, int s, int pad, int To,
                                   float* out, cudaStream_t stream)
{
    using G = Conv1dFmaTile;
    const int tiles_t = (To + G::TT - 1) / G::TT;
    const int tiles_o = (O + G::OT - 1) / G::OT;
    const long long nblk = (long long)N * tiles_t * tiles_o;
    if (nblk > 0x7fffffffLL) return FCV_ERR_UNSUPPORTED;
    const size_t smem = conv1d_fma_smem(K, s).bytes;
    auto kern = (s == 1) ? dwsep_conv1d_fma_kernel<1> : dwsep_conv1d_fma_kernel<0>;
    return launch_cached(kern, (int)smem, [&] {
        kern<<<(unsigned)nblk, G::NT, smem, stream>>>(x, dw, pw, bias, C, T, O, K, s, pad, To, tiles_t, tiles_o,
                                                      out);
    });
}

}  // namespace fcv
