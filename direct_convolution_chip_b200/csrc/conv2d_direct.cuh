// conv2d_direct.cuh -- op A on FP32 FMA: conv2d 3x3 -> AvgPool2d(P) -> sigmoid -> sum.
//
// Method (POPCORNBENCH trace "Kimi-K2.6__l2_p65", tile-fusion design and final
// kernel): every pooled value is the mean of the P x P conv outputs of its
// window, and the windows do not overlap, so computing the conv only inside
// the windows does the same work as conv-then-pool while the conv output never
// leaves registers.  The bias is added once per pooled value (mean(conv + b) =
// mean(conv) + b, the bias-folding step of the same trace).  Rows and columns
// past PH*P / PW*P are never computed (floor pooling drops them).
//
// B200 design:
//   * One CTA covers a TPH x (TPW*RX) tile of pooled outputs for a block of
//     CB = CG*NCH output channels of one image.  Its input halo
//     [ICC][P*TPH+2][P*TPW*RX+2] is staged in shared memory (zero-filled past
//     the image) one chunk of ICC input channels at a time.
//   * The halo and weights arrive by cp.async, every copy of a chunk in flight
//     at once, so a CTA waits for one memory latency per chunk, not one per
//     element.
//   * Each thread owns RX adjacent pooled positions for CG channels.  It keeps
//     its (P+2) x (RX*P+2) input patch in registers and, per 3x3 tap, the CG
//     weights of that tap (a broadcast shared-memory read), then issues
//     P*P*RX*CG independent FMAs -- consecutive FMAs update different
//     accumulators, so the FMA pipe is not stalled on a dependency chain.
//     For P <= 4 the FMAs are packed (fma.rn.f32x2, two channels per
//     instruction): the FP32 pipe does the same 128 FMA/clk/SM either way, but
//     half the issue slots go to the FMAs, leaving room for loads and
//     addressing.
//   * Epilogue: mean + bias, sigmoid (CUDA expf), a warp-shuffle + shared
//     memory block sum, and one atomicAdd per CTA into out[n].
#pragma once

#include "common.cuh"

// Largest pool size that uses packed fma.rn.f32x2 (its register patch holds
// every input value twice).
#ifndef FCV_CONV2D_PACKED_MAX_P
#define FCV_CONV2D_PACKED_MAX_P 4
#endif

namespace fcv {

template <int P>
struct Conv2dTile;

// (RX, CG, TPH, TPW, NCH, ICC) per pool size: register patch + accumulators
// stay well under 128 registers; halo + weights stay under ~60 KB so several
// CTAs share an SM.
template <> struct Conv2dTile<1> { static constexpr int RX = 2, CG = 16, TPH = 16, TPW = 8,  NCH = 2, ICC = 8; };
template <> struct Conv2dTile<2> { static constexpr int RX = 2, CG = 16, TPH = 8,  TPW = 8,  NCH = 4, ICC = 8; };
template <> struct Conv2dTile<3> { static constexpr int RX = 1, CG = 16, TPH = 8,  TPW = 8,  NCH = 4, ICC = 8; };
template <> struct Conv2dTile<4> { static constexpr int RX = 1, CG = 16, TPH = 8,  TPW = 8,  NCH = 4, ICC = 8; };
template <> struct Conv2dTile<5> { static constexpr int RX = 1, CG = 8,  TPH = 4,  TPW = 8,  NCH = 4, ICC = 4; };
template <> struct Conv2dTile<6> { static constexpr int RX = 1, CG = 8,  TPH = 4,  TPW = 8,  NCH = 4, ICC = 4; };
template <> struct Conv2dTile<7> { static constexpr int RX = 1, CG = 8,  TPH = 4,  TPW = 8,  NCH = 4, ICC = 4; };
template <> struct Conv2dTile<8> { static constexpr int RX = 1, CG = 8,  TPH = 4,  TPW = 8,  NCH = 4, ICC = 2; };

// NARROW (layers with Cout <= 32 at P <= 4): half the channel groups and twice
// the pooled rows per CTA, so no thread computes channels that do not exist.
template <int P, bool NARROW = false>
struct Conv2dGeom {
    using T = Conv2dTile<P>;
    static constexpr bool NR = NARROW && P <= 4;
    static constexpr int RX = T::RX, CG = T::CG, TPW = T::TPW, ICC = T::ICC;
    static constexpr int TPH = NR ? 2 * T::TPH : T::TPH;
    static constexpr int NCH = NR ? T::NCH / 2 : T::NCH;
    static constexpr int NPOS = TPH * TPW;          // threads per channel group
    static constexpr int NT = NPOS * NCH;           // threads per CTA
    static constexpr int CB = CG * NCH;             // output channels per CTA
    static constexpr int TILE_PH = TPH;             // pooled rows per CTA
    static constexpr int TILE_PW = TPW * RX;        // pooled cols per CTA
    static constexpr int HY = P * TILE_PH + 2;      // halo rows
    static constexpr int HX = P * TILE_PW + 2;      // halo cols
    static constexpr int HXP = (HX + 3) & ~3;       // halo row pitch (16-byte rows)
    static constexpr int PY = P + 2;                // register patch rows
    static constexpr int PX = RX * P + 2;           // register patch cols
    static constexpr int HALO_FLOATS = ICC * HY * HXP;
    static constexpr int W_FLOATS = ICC * 9 * CB;
    static constexpr size_t SMEM_BYTES = sizeof(float) * (HALO_FLOATS + W_FLOATS + NT / 32 + 1);
};

// What the kernel produces.
enum Conv2dMode : int {
    kSumAtomic = 0,  // out[n] += one block sum per CTA (atomicAdd; out pre-zeroed)
    kTap = 1,        // pooled pre-sigmoid values, no sum
    kSumDet = 2,     // block sums to a workspace; the last CTA of each image sums them in a fixed order
};

// Sum of `v` (double) over a thread block, valid in thread 0; fixed order.
template <int NT>
__device__ __forceinline__ double block_sum_d(double v, double* scratch)
{
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if (lane == 0) scratch[warp] = v;
    __syncthreads();
    double s = 0.0;
    if (threadIdx.x < 32) {
        s = (lane < NT / 32) ? scratch[lane] : 0.0;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
    }
    return s;
}

// MODE is a Conv2dMode.  partials/counters are used by kSumDet only: the
// workspace holds one float per CTA ([N][per_image]) and one counter per image
// (zero at launch).
template <int P, int MODE, bool NARROW, bool PACKED = (P <= FCV_CONV2D_PACKED_MAX_P)>
__global__ void __launch_bounds__(Conv2dGeom<P, NARROW>::NT, 2)
conv2d_direct_kernel(const float* __restrict__ x, const float* __restrict__ w,
                     const float* __restrict__ bias, int Cin, int H, int W, int Cout,
                     int PH, int PW, int tiles_y, int tiles_x, float* __restrict__ out,
                     float* __restrict__ partials, unsigned int* __restrict__ counters, int vec16)
{
    constexpr bool TAP = MODE == kTap;
    using G = Conv2dGeom<P, NARROW>;
    constexpr int RX = G::RX, CG = G::CG, NPOS = G::NPOS, NT = G::NT, CB = G::CB;
    constexpr int HY = G::HY, HX = G::HX, HXP = G::HXP, PY = G::PY, PX = G::PX, ICC = G::ICC;

    extern __shared__ __align__(16) float smem[];
    float* halo = smem;                      // [ICC][HY][HXP]
    float* ws = smem + G::HALO_FLOATS;       // [ICC][9][CB]
    float* red = ws + G::W_FLOATS;           // [NT/32]

    int tile = blockIdx.x;
    const int tx_tile = tile % tiles_x;
    tile /= tiles_x;
    const int ty_tile = tile % tiles_y;
    const int n = tile / tiles_y;
    const int c_base = blockIdx.y * CB;
    const int ph0 = ty_tile * G::TILE_PH, pw0 = tx_tile * G::TILE_PW;
    const int y0 = ph0 * P, x0 = pw0 * P;

    const int tid = threadIdx.x;
    const int grp = tid / NPOS, pos = tid % NPOS;
    const int ty = pos / G::TPW, tx = pos % G::TPW;

    float2 acc2[RX][CG / 2];  // acc2[rx][c/2] holds channels c (x) and c+1 (y)
#pragma unroll
    for (int r = 0; r < RX; ++r)
#pragma unroll
        for (int c = 0; c < CG / 2; ++c) acc2[r][c] = make_float2(0.f, 0.f);

    const float* xn = x + (size_t)n * Cin * H * W;

    for (int ic0 = 0; ic0 < Cin; ic0 += ICC) {
        // Stage the halo of this input-channel chunk and its weights with
        // asynchronous copies, all in flight at once (zero past the image);
        // only the chunk's nic real channels are staged.  Weights as
        // [icl][tap][c_local] so a thread's CG channels of one tap are contiguous.
        const int nic = min(ICC, Cin - ic0);
        if (vec16) {
            // Rows are 16-byte aligned (W % 4 == 0, aligned x, x0 a multiple of 4):
            // HXP/4 copies of 16 bytes per halo row, zero-filled past the image.
            constexpr int CPR = HXP / 4;
            for (int i = tid; i < nic * HY * CPR; i += NT) {
                const int row = i / CPR, q = i - (i / CPR) * CPR;
                const int icl = row / HY, r = row - (row / HY) * HY;
                const int yy = y0 + r, xx = x0 + 4 * q;
                const int bytes = yy < H ? 4 * max(0, min(4, W - xx)) : 0;
                cp_async16(halo + (icl * HY + r) * HXP + 4 * q,
                           bytes ? xn + ((size_t)(ic0 + icl) * H + yy) * W + xx : x, bytes);
            }
        } else {
            for (int i = tid; i < nic * HY * HX; i += NT) {
                const int icl = i / (HY * HX);
                const int rem = i - icl * (HY * HX);
                const int r = rem / HX, sc = rem - (rem / HX) * HX;
                const int ic = ic0 + icl, yy = y0 + r, xx = x0 + sc;
                const bool in = ic < Cin && yy < H && xx < W;
                cp_async4(halo + (icl * HY + r) * HXP + sc, in ? xn + ((size_t)ic * H + yy) * W + xx : x, in);
            }
        }
        for (int i = tid; i < nic * 9 * CB; i += NT) {
            const int cl = i % CB;
            const int tap = (i / CB) % 9;
            const int icl = i / (9 * CB);
            const int c = c_base + cl, ic = ic0 + icl;
            const bool in = c < Cout && ic < Cin;
            cp_async4(ws + i, in ? w + ((size_t)c * Cin + ic) * 9 + tap : w, in);
        }
        cp_async_commit();
        cp_async_wait<0>();
        __syncthreads();

        for (int icl = 0; icl < nic; ++icl) {
            const float* hp = halo + (icl * HY + ty * P) * HXP + tx * (RX * P);
            const float* wp = ws + icl * 9 * CB + grp * CG;
            if constexpr (PACKED) {
                // Packed FP32 FMA: each fma.rn.f32x2 updates two adjacent
                // output channels; the input value is duplicated into both
                // halves of a register pair once per patch load.
                float2 patch[PY][PX];
#pragma unroll
                for (int r = 0; r < PY; ++r)
#pragma unroll
                    for (int sc = 0; sc < PX; ++sc) {
                        const float v = hp[r * HXP + sc];
                        patch[r][sc] = make_float2(v, v);
                    }
#pragma unroll
                for (int ky = 0; ky < 3; ++ky) {
#pragma unroll
                    for (int kx = 0; kx < 3; ++kx) {
                        float2 wr[CG / 2];
#pragma unroll
                        for (int c = 0; c < CG; c += 4) {
                            const float4 v = *reinterpret_cast<const float4*>(wp + (ky * 3 + kx) * CB + c);
                            wr[c / 2] = make_float2(v.x, v.y);
                            wr[c / 2 + 1] = make_float2(v.z, v.w);
                        }
#pragma unroll
                        for (int rx = 0; rx < RX; ++rx)
#pragma unroll
                            for (int dy = 0; dy < P; ++dy)
#pragma unroll
                                for (int dx = 0; dx < P; ++dx) {
                                    const float2 pv = patch[dy + ky][rx * P + dx + kx];
#pragma unroll
                                    for (int c = 0; c < CG / 2; ++c) acc2[rx][c] = __ffma2_rn(pv, wr[c], acc2[rx][c]);
                                }
                    }
                }
            } else {
                float patch[PY][PX];
#pragma unroll
                for (int r = 0; r < PY; ++r)
#pragma unroll
                    for (int sc = 0; sc < PX; ++sc) patch[r][sc] = hp[r * HXP + sc];
#pragma unroll
                for (int ky = 0; ky < 3; ++ky) {
#pragma unroll
                    for (int kx = 0; kx < 3; ++kx) {
                        float wr[CG];
#pragma unroll
                        for (int c = 0; c < CG; c += 4) {
                            const float4 v = *reinterpret_cast<const float4*>(wp + (ky * 3 + kx) * CB + c);
                            wr[c] = v.x; wr[c + 1] = v.y; wr[c + 2] = v.z; wr[c + 3] = v.w;
                        }
#pragma unroll
                        for (int rx = 0; rx < RX; ++rx)
#pragma unroll
                            for (int dy = 0; dy < P; ++dy)
#pragma unroll
                                for (int dx = 0; dx < P; ++dx) {
                                    const float pv = patch[dy + ky][rx * P + dx + kx];
#pragma unroll
                                    for (int c = 0; c < CG; ++c)
                                        acc2[rx][c / 2] = (c & 1) ? make_float2(acc2[rx][c / 2].x, fmaf(pv, wr[c], acc2[rx][c / 2].y))
                                                                  : make_float2(fmaf(pv, wr[c], acc2[rx][c / 2].x), acc2[rx][c / 2].y);
                                }
                    }
                }
            }
        }
        __syncthreads();
    }

    // Epilogue: mean of the window + bias, then sigmoid and the block sum.
    const int ph = ph0 + ty;
    float local = 0.f;
#pragma unroll
    for (int rx = 0; rx < RX; ++rx) {
        const int pw = pw0 + tx * RX + rx;
        const bool valid = ph < PH && pw < PW;
#pragma unroll
        for (int c = 0; c < CG; ++c) {
            const int cc = c_base + grp * CG + c;
            if (valid && cc < Cout) {
                const float a = (c & 1) ? acc2[rx][c / 2].y : acc2[rx][c / 2].x;
                const float avg = a / (float)(P * P) + __ldg(bias + cc);
                if (TAP) {
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
        // Deterministic: this CTA's block sum goes to its own workspace slot; the
        // CTA that finishes last for image n (seen through a counter, nothing
        // waits) adds the slots in a fixed order and writes out[n].
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
            __syncthreads();  // red is reused below
            const double all = block_sum_d<NT>(sacc, reinterpret_cast<double*>(halo));
            if (tid == 0) out[n] = (float)all;
        }
    }
}

inline bool conv2d_narrow(int P, int Cout) { return P <= 4 && Cout <= 32; }

// Grid of the direct kernel for pool size P: tiles per image and channel blocks.
template <int P, bool NARROW>
void conv2d_grid_p(int PH, int PW, int Cout, int* tiles_y, int* tiles_x, int* cblocks)
{
    using G = Conv2dGeom<P, NARROW>;
    *tiles_y = (PH + G::TILE_PH - 1) / G::TILE_PH;
    *tiles_x = (PW + G::TILE_PW - 1) / G::TILE_PW;
    *cblocks = (Cout + G::CB - 1) / G::CB;
}

template <int P>
void conv2d_grid_pp(int PH, int PW, int Cout, int* tiles_y, int* tiles_x, int* cblocks)
{
    if (conv2d_narrow(P, Cout)) conv2d_grid_p<P, true>(PH, PW, Cout, tiles_y, tiles_x, cblocks);
    else conv2d_grid_p<P, false>(PH, PW, Cout, tiles_y, tiles_x, cblocks);
}

inline bool conv2d_grid(int P, int PH, int PW, int Cout, int* tiles_y, int* tiles_x, int* cblocks)
{
    switch (P) {
    case 1: conv2d_grid_pp<1>(PH, PW, Cout, tiles_y, tiles_x, cblocks); return true;
    case 2: conv2d_grid_pp<2>(PH, PW, Cout, tiles_y, tiles_x, cblocks); return true;
    case 3: conv2d_grid_pp<3>(PH, PW, Cout, tiles_y, tiles_x, cblocks); return true;
    case 4: conv2d_grid_pp<4>(PH, PW, Cout, tiles_y, tiles_x, cblocks); return true;
    case 5: conv2d_grid_pp<5>(PH, PW, Cout, tiles_y, tiles_x, cblocks); return true;
    case 6: conv2d_grid_pp<6>(PH, PW, Cout, tiles_y, tiles_x, cblocks); return true;
    case 7: conv2d_grid_pp<7>(PH, PW, Cout, tiles_y, tiles_x, cblocks); return true;
    case 8: conv2d_grid_pp<8>(PH, PW, Cout, tiles_y, tiles_x, cblocks); return true;
    default: return false;
    }
}

template <int P, int MODE, bool NARROW>
int launch_conv2d_direct_pn(const float* x, const float* w, const float* b, int N, int Cin, int H,
                            int W, int Cout, int PH, int PW, float* out, float* partials,
                            unsigned int* counters, cudaStream_t stream)
{
    using G = Conv2dGeom<P, NARROW>;
    int tiles_y, tiles_x, cblk;
    conv2d_grid_p<P, NARROW>(PH, PW, Cout, &tiles_y, &tiles_x, &cblk);
    const long long nblk = (long long)N * tiles_y * tiles_x;
    if (nblk > 0x7fffffffLL || cblk > 65535) return FCV_ERR_UNSUPPORTED;
    auto kern = conv2d_direct_kernel<P, MODE, NARROW>;
    dim3 grid((unsigned)nblk, (unsigned)cblk);
    const int vec16 = ((W & 3) == 0 && (reinterpret_cast<uintptr_t>(x) & 15) == 0 && (P * G::TILE_PW) % 4 == 0) ? 1 : 0;
    auto go = [&] {
        kern<<<grid, G::NT, G::SMEM_BYTES, stream>>>(x, w, b, Cin, H, W, Cout, PH, PW, tiles_y, tiles_x, out,
                                                      partials, counters, vec16);
    };
    if (G::SMEM_BYTES > 48 * 1024) return launch_cached(kern, (int)G::SMEM_BYTES, go);
    go();
    return launch_status();
}

template <int P, int MODE>
int launch_conv2d_direct_p(const float* x, const float* w, const float* b, int N, int Cin, int H,
                           int W, int Cout, int PH, int PW, float* out, float* partials,
                           unsigned int* counters, cudaStream_t stream)
{
    if (conv2d_narrow(P, Cout))
        return launch_conv2d_direct_pn<P, MODE, true>(x, w, b, N, Cin, H, W, Cout, PH, PW, out, partials,
                                                      counters, stream);
    return launch_conv2d_direct_pn<P, MODE, false>(x, w, b, N, Cin, H, W, Cout, PH, PW, out, partials,
                                                   counters, stream);
}

// PH, PW >= 1 here; the caller handles the empty cases.
template <int MODE>
int launch_conv2d_direct(const float* x, const float* w, const float* b, int N, int Cin, int H,
                         int W, int Cout, int P, int PH, int PW, float* out, cudaStream_t stream,
                         float* partials = nullptr, unsigned int* counters = nullptr)
{
    switch (P) {
    case 1: return launch_conv2d_direct_p<1, MODE>(x, w, b, N, Cin, H, W, Cout, PH, PW, out, partials, counters, stream);
    case 2: return launch_conv2d_direct_p<2, MODE>(x, w, b, N, Cin, H, W, Cout, PH, PW, out, partials, counters, stream);
    case 3: return launch_conv2d_direct_p<3, MODE>(x, w, b, N, Cin, H, W, Cout, PH, PW, out, partials, counters, stream);
    case 4: return launch_conv2d_direct_p<4, MODE>(x, w, b, N, Cin, H, W, Cout, PH, PW, out, partials, counters, stream);
    case 5: return launch_conv2d_direct_p<5, MODE>(x, w, b, N, Cin, H, W, Cout, PH, PW, out, partials, counters, stream);
    case 6: return launch_conv2d_direct_p<6, MODE>(x, w, b, N, Cin, H, W, Cout, PH, PW, out, partials, counters, stream);
    case 7: return launch_conv2d_direct_p<7, MODE>(x, w, b, N, Cin, H, W, Cout, PH, PW, out, partials, counters, stream);
    case 8: return launch_conv2d_direct_p<8, MODE>(x, w, b, N, Cin, H, W, Cout, PH, PW, out, partials, counters, stream);
    default: return FCV_ERR_UNSUPPORTED;
    }
}

// Workspace of the deterministic sum: [N][per_image] floats, then N counters
// (16-byte aligned).  0 bytes when nothing is launched (PH or PW == 0).
inline size_t conv2d_det_workspace_bytes(int N, int Cout, int P, int PH, int PW)
{
    if (N <= 0 || PH <= 0 || PW <= 0) return 0;
    int ty, tx, cb;
    if (!conv2d_grid(P, PH, PW, Cout, &ty, &tx, &cb)) return 0;
    const size_t part = ((size_t)N * ty * tx * cb * sizeof(float) + 15) & ~(size_t)15;
    return part + (size_t)N * sizeof(unsigned int);
}

}  // namespace fcv
