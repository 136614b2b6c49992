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
// image, in chunks of ICC input channels (4; 2 from P = 5 on, so that two CTAs
// still fit an SM):
//   1. cp.async stages the input halo [ICC][8P+2][16P+2] (16-byte copies of
//      whole rows when W % 4 == 0 and x is 16-byte aligned, else 4-byte ones)
//      and the weights [ICC*9][64] (zero past the image / Cin / Cout);
//   2. the box sums S[ic][ky][kx][pos] in two separable passes, both with the
//      lanes of a warp on consecutive pooled columns: horizontal sums of P
//      samples at the three column offsets kx (one vector read of P+2 samples
//      per row and pooled column) into H[ic][kx][row][px], then vertical
//      running sums over P rows at the three row offsets ky.  H's row pitch
//      puts the two half-warps of the vertical pass (pooled rows 2j, 2j+1) in
//      opposite halves of the banks;
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
    static constexpr int ICC = P <= 4 ? 4 : 2;       // input channels per chunk
    static constexpr int NT = 256;
    static constexpr int KC = ICC * 9;               // contraction length per chunk
    static constexpr int HY = P * TPH + 2, HX = P * TPW + 2;
    static constexpr int HXP = (HX + 3) & ~3;        // halo row pitch: rows start 16-byte aligned
    static constexpr int NF4 = HXP / 4;              // 16-byte pieces per staged row
    // Row pitch of the horizontal sums H: (P * HRP) mod 32 == 16, so pooled
    // rows 2j and 2j+1 (the two half-warps of the vertical pass) use opposite
    // bank halves.
    static constexpr int HRP = (P & 1) ? 16 : (P == 4 ? 20 : (P == 8 ? 18 : 24));
    static constexpr int RP = 4, RC = 8;             // per-thread register block: 4 positions x 8 channels
    static constexpr int HALO_FLOATS = ICC * HY * HXP;
    static constexpr int H_FLOATS = ICC * 3 * HY * HRP;
    static constexpr int S_FLOATS = KC * NPOS;
    static constexpr int W_FLOATS = KC * CB;
    static constexpr size_t SMEM_BYTES =
        sizeof(float) * (HALO_FLOATS + H_FLOATS + S_FLOATS + W_FLOATS + NT / 32 + 4);
    static_assert((NPOS / RP) * (CB / RC) == NT, "thread layout");
    static_assert((P * HRP) % 32 == 16 && HRP >= TPW, "vertical-pass bank halves");
    static_assert(SMEM_BYTES * 2 <= 227 * 1024, "two CTAs per SM");
    static_assert(HALO_FLOATS % 4 == 0 && H_FLOATS % 4 == 0 && S_FLOATS % 4 == 0, "16-byte aligned smem arrays");
};

// The P + 2 consecutive samples v[0..P+1] at p, with the widest loads the
// alignment of p allows (p = row + P * px: 16 bytes when P % 4 == 0, 8 when P
// is even, else 4; lanes on consecutive px then read consecutive words).  For
// P % 4 == 0 the last two samples come with a 16-byte load too (at a 16-byte
// lane stride an 8-byte load would meet another lane's banks); it stays inside
// the row, whose pitch is 16P + 4 floats then.
template <int P>
__device__ __forceinline__ void load_run(const float* p, float (&v)[P + 2])
{
    if constexpr (P % 4 == 0) {
#pragma unroll
        for (int q = 0; q < P / 4; ++q) {
            const float4 t = *reinterpret_cast<const float4*>(p + 4 * q);
            v[4 * q] = t.x; v[4 * q + 1] = t.y; v[4 * q + 2] = t.z; v[4 * q + 3] = t.w;
        }
        const float4 t = *reinterpret_cast<const float4*>(p + P);
        v[P] = t.x; v[P + 1] = t.y;
    } else if constexpr (P % 2 == 0) {
#pragma unroll
        for (int q = 0; q < (P + 2) / 2; ++q) {
            const float2 t = *reinterpret_cast<const float2*>(p + 2 * q);
            v[2 * q] = t.x; v[2 * q + 1] = t.y;
        }
    } else {
#pragma unroll
        for (int q = 0; q < P + 2; ++q) v[q] = p[q];
    }
}

// VEC: the halo rows are staged as 16-byte copies (W % 4 == 0 and x 16-byte
// aligned), else as 4-byte ones.
template <int P, int MODE, bool VEC>
__global__ void __launch_bounds__(256, 2)
conv2d_poolfirst_kernel(const float* __restrict__ x, const float* __restrict__ w,
                        const float* __restrict__ bias, int Cin, int H, int W, int Cout,
                        int PH, int PW, int tiles_y, int tiles_x, float* __restrict__ out,
                        float* __restrict__ partials, unsigned int* __restrict__ counters)
{
    using G = PoolFirstGeom<P>;
    constexpr int NT = G::NT, NPOS = G::NPOS, CB = G::CB, ICC = G::ICC, KC = G::KC;
    constexpr int HY = G::HY, HX = G::HX, HXP = G::HXP, RP = G::RP, RC = G::RC, HRP = G::HRP;

    extern __shared__ __align__(16) float smem[];
    float* halo = smem;                       // [ICC][HY][HXP]
    float* Hs = halo + G::HALO_FLOATS;        // [ICC][3][HY][HRP]  horizontal sums at column offsets kx
    float* Ss = Hs + G::H_FLOATS;             // [KC][NPOS]   box sums, k = icl*9 + ky*3 + kx
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

    // GEMM thread block: positions 4*pg .. 4*pg+3, channels 4*cgi .. 4*cgi+3 and
    // 32+4*cgi .. 32+4*cgi+3 (a quarter-warp's weight loads then cover 128
    // contiguous bytes)
    const int cgi = tid & 7, pg = tid >> 3;

    float2 acc[RP][RC / 2];
#pragma unroll
    for (int i = 0; i < RP; ++i)
#pragma unroll
        for (int j = 0; j < RC / 2; ++j) acc[i][j] = make_float2(0.f, 0.f);

    const float* xn = x + (size_t)n * Cin * H * W;
    const int warp = tid >> 5, lane = tid & 31;
    for (int ic0 = 0; ic0 < Cin; ic0 += ICC) {
        if constexpr (VEC) {
            // one staged row per warp iteration: x0 is a multiple of 16 and W of
            // 4, so a 16-byte piece lies wholly inside or wholly outside the row
            for (int row = warp; row < ICC * HY; row += NT / 32) {
                const int icl = row / HY, r = row - (row / HY) * HY;
                const int ic = ic0 + icl, yy = y0 + r;
                const bool row_in = ic < Cin && yy < H;
                const float* src = xn + ((size_t)(row_in ? ic : 0) * H + (row_in ? yy : 0)) * W;
                for (int f = lane; f < G::NF4; f += 32) {
                    const int xx = x0 + 4 * f;
                    const bool in = row_in && xx < W;
                    cp_async16(halo + row * HXP + 4 * f, in ? src + xx : x, in ? 16 : 0);
                }
            }
        } else {
            for (int i = tid; i < ICC * HY * HX; i += NT) {
                const int icl = i / (HY * HX);
                const int rem = i - icl * (HY * HX);
                const int r = rem / HX, sc = rem - (rem / HX) * HX;
                const int ic = ic0 + icl, yy = y0 + r, xx = x0 + sc;
                const bool in = ic < Cin && yy < H && xx < W;
                cp_async4(halo + (icl * HY + r) * HXP + sc, in ? xn + ((size_t)ic * H + yy) * W + xx : x, in);
            }
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

        // Horizontal pass: for every staged row and pooled column px, the sums of
        // P samples starting at columns P*px + kx, kx = 0, 1, 2.
        for (int i = tid; i < ICC * HY * G::TPW; i += NT) {
            const int px = i % G::TPW, row = i / G::TPW;
            const int icl = row / HY, r = row - (row / HY) * HY;
            float v[P + 2];
            load_run<P>(halo + row * HXP + P * px, v);
            float h = 0.f;
#pragma unroll
            for (int dx = 0; dx < P; ++dx) h += v[dx];
            float* hd = Hs + ((icl * 3) * HY + r) * HRP + px;
            hd[0] = h;
            h = h - v[0] + v[P];
            hd[HY * HRP] = h;
            h = h - v[1] + v[P + 1];
            hd[2 * HY * HRP] = h;
        }
        __syncthreads();

        // Vertical pass: for every (input channel, kx) and pooled position, the
        // sums of P horizontal sums starting at rows P*py + ky, ky = 0, 1, 2:
        // the box sums S[ic][ky][kx][pos].
        for (int i = tid; i < ICC * 3 * NPOS; i += NT) {
            const int pos = i % NPOS, g = i / NPOS;
            const int icl = g / 3, kx = g - (g / 3) * 3;
            const int py = pos / G::TPW, px = pos % G::TPW;
            const float* hp = Hs + ((icl * 3 + kx) * HY + P * py) * HRP + px;
            float v[P + 2];
#pragma unroll
            for (int j = 0; j < P + 2; ++j) v[j] = hp[j * HRP];
            float s = 0.f;
#pragma unroll
            for (int dy = 0; dy < P; ++dy) s += v[dy];
            Ss[(icl * 9 + kx) * NPOS + pos] = s;
            s = s - v[0] + v[P];
            Ss[(icl * 9 + 3 + kx) * NPOS + pos] = s;
            s = s - v[1] + v[P + 1];
            Ss[(icl * 9 + 6 + kx) * NPOS + pos] = s;
        }
        __syncthreads();

        // Contraction over this chunk's 36 (input channel, tap) pairs.
        const int kc = min(ICC, Cin - ic0) * 9;
#pragma unroll 4
        for (int k = 0; k < kc; ++k) {
            const float4 sv = *reinterpret_cast<const float4*>(Ss + k * NPOS + RP * pg);
            const float4 w0 = *reinterpret_cast<const float4*>(Ws + k * CB + 4 * cgi);
            const float4 w1 = *reinterpret_cast<const float4*>(Ws + k * CB + CB / 2 + 4 * cgi);
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
            const int cc = c_base + (j < 4 ? 4 * cgi + j : CB / 2 + 4 * cgi + (j - 4));
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
    const bool vec = (W & 3) == 0 && (reinterpret_cast<uintptr_t>(x) & 15) == 0;
    auto kern = vec ? conv2d_poolfirst_kernel<P, MODE, true> : conv2d_poolfirst_kernel<P, MODE, false>;
    dim3 grid((unsigned)nblk, (unsigned)cblk);
    return launch_cached(kern, (int)G::SMEM_BYTES, [&] {
        kern<<<grid, G::NT, G::SMEM_BYTES, stream>>>(x, w, b, Cin, H, W, Cout, PH, PW, tiles_y, tiles_x, out,
                                                      partials, counters);
    });
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
