// conv2d_poolfirst.cuh -- op A with the pooling applied to the input first.
//
// Identity (exact in real arithmetic; only the rounding differs from the
// direct method): the P x P mean of the conv outputs of a window is a 3x3 conv
// of box sums of the input,
//   sum_{dy,dx<P} conv[P*ph+dy][P*pw+dx]
//     = sum_{ic,ky,kx} w[c,ic,ky,kx] * S[ic,ky,kx],
//   S[ic,ky,kx] = sum_{dy,dx<P} x[ic][P*ph+dy+ky][P*pw+dx+kx],
// because pooling and convolution are both linear.  S (9 values per input
// channel and pooled position) does not depend on the output channel, so a
// pooled value costs 9*Cin MACs instead of 9*Cin*P*P -- at P = 4, 16x fewer.
// It is the pool-folded composite of the l2_p65 trace's tile-fusion design
// (the shared (P+2)x(P+2) input patch of a window, and the bias added once per
// pooled value), taken to its end: the conv output is never formed at all.
//
// Kernel: a CTA covers 8 x 16 pooled positions x 64 output channels of one
// image, in chunks of 4 input channels:
//   1. cp.async stages the input halo [4][8P+2][16P+2] and the weights
//      [4*9][64] (zero past the image / past Cin / past Cout);
//   2. each thread forms the box sums S of two (position, channel) pairs with
//      separable running sums over its (P+2)x(P+2) patch -> smem S[36][128];
//   3. the contraction out[pos][c] += sum_k S[k][pos] * W[k][c] runs as a
//      register-blocked FP32 GEMM: 4 positions x 8 channels per thread, packed
//      fma.rn.f32x2 over channel pairs.
// Epilogue as in the direct kernel: mean + bias, sigmoid, block sum, one
// atomicAdd per CTA (or the tap / the deterministic workspace sum).
#pragma once

#include "common.cuh"
#include "conv2d_direct.cuh"

namespace fcv {

template <int P>
struct PoolFirstGeom {
    static constexpr int TPH = 8, TPW = 16;          // pooled positions per CTA: 8 x 16
    static constexpr int NPOS = TPH * TPW;           // 128
    static constexpr int CB = 64;                    // output channels per CTA
    static constexpr int ICC = 4;                    // input channels per chunk
    static constexpr int NT = 256;
    static constexpr int KC = ICC * 9;               // contraction length per chunk
    static constexpr int HY = P * TPH + 2, HX = P * TPW + 2;
    static constexpr int HXP = HX + 1;               // odd pitch: patch rows of adjacent positions spread over banks
    static constexpr int RP = 4, RC = 8;             // per-thread register block: 4 positions x 8 channels
    static constexpr int HALO_FLOATS = ICC * HY * HXP;
    static constexpr int S_FLOATS = KC * NPOS;
    static constexpr int W_FLOATS = KC * CB;
    static constexpr size_t SMEM_BYTES = sizeof(float) * (HALO_FLOATS + S_FLOATS + W_FLOATS + NT / 32 + 4);
    static_assert((NPOS / RP) * (CB / RC) == NT, "thread layout");
};

template <int P, int MODE>
__global__ void __launch_bounds__(256, 2)
conv2d_poolfirst_kernel(const float* __restrict__ x, const float* __restrict__ w,
                        const float* __restrict__ bias, int Cin, int H, int W, int Cout,
                        int PH, int PW, int tiles_y, int tiles_x, float* __restrict__ out,
                        float* __restrict__ partials, unsigned int* __restrict__ counters)
{
    using G = PoolFirstGeom<P>;
    constexpr int NT = G::NT, NPOS = G::NPOS, CB = G::CB, ICC = G::ICC, KC = G::KC;
    constexpr int HY = G::HY, HX = G::HX, HXP = G::HXP, RP = G::RP, RC = G::RC;

    extern __shared__ __align__(16) float smem[];
    float* halo = smem;                       // [ICC][HY][HXP]
    float* Ss = halo + G::HALO_FLOATS;        // [KC][NPOS]   box sums, k = icl*9 + ky*3 + kx
    float* Ws = Ss + G::S_FLOATS;             // [KC][CB]
    float* red = Ws + G::W_FLOATS;            // [NT/32 + 4]

    int tile = blockIdx.x;
    const int tx_tile = tile % tiles_x;
    tile /= tiles_x;
    const int ty_tile = tile % tiles_y;
    const int n = tile / tiles_y;
    const int c_base = blockIdx.y * CB;
    const int ph0 = ty_tile * G::TPH, pw0 = tx_tile * G::TPW;
    const int y0 = ph0 * P, x0 = pw0 * P;
    const int tid = threadIdx.x;

    // GEMM thread block: positions 4*pg .. 4*pg+3, channels 8*cgi .. 8*cgi+7
    const int cgi = tid & 7, pg = tid >> 3;

    float2 acc[RP][RC / 2];
#pragma unroll
    for (int i = 0; i < RP; ++i)
#pragma unroll
        for (int j = 0; j < RC / 2; ++j) acc[i][j] = make_float2(0.f, 0.f);

    const float* xn = x + (size_t)n * Cin * H * W;
    for (int ic0 = 0; ic0 < Cin; ic0 += ICC) {
        for (int i = tid; i < ICC * HY * HX; i += NT) {
            const int icl = i / (HY * HX);
            const int rem = i - icl * (HY * HX);
            const int r = rem / HX, sc = rem - (rem / HX) * HX;
            const int ic = ic0 + icl, yy = y0 + r, xx = x0 + sc;
            const bool in = ic < Cin && yy < H && xx < W;
            cp_async4(halo + (icl * HY + r) * HXP + sc, in ? xn + ((size_t)ic * H + yy) * W + xx : x, in);
        }
        for (int i = tid; i < KC * CB; i += NT) {
            const int cl = i % CB, k = i / CB;
            const int icl = k / 9, tap = k - (k / 9) * 9;
            const int c = c_base + cl, ic = ic0 + icl;
            const bool in = c < Cout && ic < Cin;
            cp_async4(Ws + i, in ? w + ((size_t)c * Cin + ic) * 9 + tap : w, in);
        }
        cp_async_commit();
        cp_async_wait<0>();
        __syncthreads();

        // Box sums: (position, input channel) pairs, two per thread.
        for (int q = tid; q < NPOS * ICC; q += NT) {
            const int pos = q % NPOS, icl = q / NPOS;
            const int py = pos / G::TPW, px = pos % G::TPW;
            const float* hp = halo + (icl * HY + py * P) * HXP + px * P;
            // row sums over P columns at the 3 column offsets, for the P+2 rows
            float R[P + 2][3];
#pragma unroll
            for (int r = 0; r < P + 2; ++r) {
                float s0 = 0.f;
#pragma unroll
                for (int dx = 0; dx < P; ++dx) s0 += hp[r * HXP + dx];
                R[r][0] = s0;
                R[r][1] = s0 - hp[r * HXP] + hp[r * HXP + P];
                R[r][2] = R[r][1] - hp[r * HXP + 1] + hp[r * HXP + P + 1];
            }
#pragma unroll
            for (int kx = 0; kx < 3; ++kx) {
                float s = 0.f;
#pragma unroll
                for (int dy = 0; dy < P; ++dy) s += R[dy][kx];
                Ss[(icl * 9 + 0 * 3 + kx) * NPOS + pos] = s;
                s = s - R[0][kx] + R[P][kx];
                Ss[(icl * 9 + 1 * 3 + kx) * NPOS + pos] = s;
                s = s - R[1][kx] + R[P + 1][kx];
                Ss[(icl * 9 + 2 * 3 + kx) * NPOS + pos] = s;
            }
        }
        __syncthreads();

        // Contraction over this chunk's 36 (input channel, tap) pairs.
        const int kc = min(ICC, Cin - ic0) * 9;
#pragma unroll 4
        for (int k = 0; k < kc; ++k) {
            const float4 sv = *reinterpret_cast<const float4*>(Ss + k * NPOS + RP * pg);
            const float4 w0 = *reinterpret_cast<const float4*>(Ws + k * CB + RC * cgi);
            const float4 w1 = *reinterpret_cast<const float4*>(Ws + k * CB + RC * cgi + 4);
            const float2 wp[4] = {make_float2(w0.x, w0.y), make_float2(w0.z, w0.w), make_float2(w1.x, w1.y),
                                  make_float2(w1.z, w1.w)};
            const float s4[4] = {sv.x, sv.y, sv.z, sv.w};
#pragma unroll
            for (int i = 0; i < RP; ++i) {
                const float2 si = make_float2(s4[i], s4[i]);
#pragma unroll
                for (int j = 0; j < RC / 2; ++j) acc[i][j] = __ffma2_rn(si, wp[j], acc[i][j]);
            }
        }
        __syncthreads();
    }

    // Epilogue: mean + bias, sigmoid, block sum (or the tap / deterministic sum).
    float local = 0.f;
#pragma unroll
    for (int i = 0; i < RP; ++i) {
        const int pos = RP * pg + i;
        const int ph = ph0 + pos / G::TPW, pw = pw0 + pos % G::TPW;
        const bool valid = ph < PH && pw < PW;
#pragma unroll
        for (int j = 0; j < RC; ++j) {
            const int cc = c_base + RC * cgi + j;
            if (valid && cc < Cout) {
                const float a = (j & 1) ? acc[i][j / 2].y : acc[i][j / 2].x;
                const float avg = a / (float)(P * P) + __ldg(bias + cc);
                if (MODE == kTap) {
                    out[(((size_t)n * Cout + cc) * PH + ph) * PW + pw] = avg;
                } else {
                    local += 1.0f / (1.0f + expf(-avg));
                }
            }
        }
    }
    if (MODE == kSumAtomic) {
        const float total = block_sum<NT>(local, red);
        if (tid == 0) atomicAdd(out + n, total);
    } else if (MODE == kSumDet) {
        const float total = block_sum<NT>(local, red);
        const int per_image = tiles_y * tiles_x * (int)gridDim.y;
        const int slot = ((int)(blockIdx.x % (unsigned)(tiles_y * tiles_x))) * (int)gridDim.y + (int)blockIdx.y;
        volatile int* last = reinterpret_cast<volatile int*>(red + NT / 32);
        if (tid == 0) {
            partials[(size_t)n * per_image + slot] = total;
            __threadfence();
            const unsigned int prev = atomicAdd(counters + n, 1u);
            *last = (prev == (unsigned int)per_image - 1u) ? 1 : 0;
        }
        __syncthreads();
        if (*last) {
            __threadfence();
            double sacc = 0.0;
            for (int i = tid; i < per_image; i += NT) sacc += (double)__ldcg(partials + (size_t)n * per_image + i);
            __syncthreads();
            const double all = block_sum_d<NT>(sacc, reinterpret_cast<double*>(halo));
            if (tid == 0) out[n] = (float)all;
        }
    }
}

template <int P, int MODE>
int launch_conv2d_poolfirst_p(const float* x, const float* w, const float* b, int N, int Cin, int H, int W,
                              int Cout, int PH, int PW, float* out, float* partials, unsigned int* counters,
                              cudaStream_t stream)
{
    using G = PoolFirstGeom<P>;
    const int tiles_y = (PH + G::TPH - 1) / G::TPH;
    const int tiles_x = (PW + G::TPW - 1) / G::TPW;
    const long long nblk = (long long)N * tiles_y * tiles_x;
    const int cblk = (Cout + G::CB - 1) / G::CB;
    if (nblk > 0x7fffffffLL || cblk > 65535) return FCV_ERR_UNSUPPORTED;
    auto kern = conv2d_poolfirst_kernel<P, MODE>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)G::SMEM_BYTES) != cudaSuccess)
        return FCV_ERR_CUDA;
    dim3 grid((unsigned)nblk, (unsigned)cblk);
    kern<<<grid, G::NT, G::SMEM_BYTES, stream>>>(x, w, b, Cin, H, W, Cout, PH, PW, tiles_y, tiles_x, out,
                                                  partials, counters);
    return launch_status();
}

// Tiles per image and channel blocks of the pool-first kernel.
inline void conv2d_poolfirst_grid(int PH, int PW, int Cout, int* tiles_y, int* tiles_x, int* cblocks)
{
    *tiles_y = (PH + PoolFirstGeom<1>::TPH - 1) / PoolFirstGeom<1>::TPH;
    *tiles_x = (PW + PoolFirstGeom<1>::TPW - 1) / PoolFirstGeom<1>::TPW;
    *cblocks = (Cout + PoolFirstGeom<1>::CB - 1) / PoolFirstGeom<1>::CB;
}

// PH, PW >= 1 here.
template <int MODE>
int launch_conv2d_poolfirst(const float* x, const float* w, const float* b, int N, int Cin, int H, int W,
                            int Cout, int P, int PH, int PW, float* out, cudaStream_t stream,
                            float* partials = nullptr, unsigned int* counters = nullptr)
{
    switch (P) {
    case 1: return launch_conv2d_poolfirst_p<1, MODE>(x, w, b, N, Cin, H, W, Cout, PH, PW, out, partials, counters, stream);
    case 2: return launch_conv2d_poolfirst_p<2, MODE>(x, w, b, N, Cin, H, W, Cout, PH, PW, out, partials, counters, stream);
    case 3: return launch_conv2d_poolfirst_p<3, MODE>(x, w, b, N, Cin, H, W, Cout, PH, PW, out, partials, counters, stream);
    case 4: return launch_conv2d_poolfirst_p<4, MODE>(x, w, b, N, Cin, H, W, Cout, PH, PW, out, partials, counters, stream);
    case 5: return launch_conv2d_poolfirst_p<5, MODE>(x, w, b, N, Cin, H, W, Cout, PH, PW, out, partials, counters, stream);
    case 6: return launch_conv2d_poolfirst_p<6, MODE>(x, w, b, N, Cin, H, W, Cout, PH, PW, out, partials, counters, stream);
    case 7: return launch_conv2d_poolfirst_p<7, MODE>(x, w, b, N, Cin, H, W, Cout, PH, PW, out, partials, counters, stream);
    case 8: return launch_conv2d_poolfirst_p<8, MODE>(x, w, b, N, Cin, H, W, Cout, PH, PW, out, partials, counters, stream);
    default: return FCV_ERR_UNSUPPORTED;
    }
}

}  // namespace fcv
