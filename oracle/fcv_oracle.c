/*
 * fcv_oracle.c -- plain, slow, obviously-correct CPU oracle for the two fused
 * convolution operations.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path links, loads or calls
 * this file: only the tests, the package's smoke check and the benchmark's CPU
 * baseline leg do.  It shares no code, header, table or constant with the CUDA
 * library; it is written straight from the definitions on the pages:
 *
 *   POPCORNBENCH trace "Kimi-K2.6__l2_p65" (fused Conv2d -> AvgPool2d ->
 *     Sigmoid -> Sum), opening analysis: the conv formula
 *       out[i,j] = sum_{c,ky,kx} in[b,c,i+ky,j+kx] * w[oc,c,ky,kx] + bias[oc],
 *     the shapes [128,8,384,384] -> [128,64,382,382] -> [128,64,95,95] -> [128]
 *     (stride 1, no padding; AvgPool2d(4) with stride 4 and floor), sigmoid,
 *     and the sum over dims 1,2,3.
 *   POPCORNBENCH trace "Kimi-K2.6__l2_p7" (depthwise-separable Conv1d),
 *     opening analysis:
 *       out[b,o,t] = sum_c ( sum_k in[b,c,t*stride+k-padding] * dw[c,k] ) * pw[o,c] + bias[o]
 *     with zero padding outside [0,T) and T_out = (T + 2p - K)/s + 1.
 *
 * Every accumulation is in double.  Inputs are fp32 host arrays, contiguous,
 * row-major (NCHW / NCT).  OpenMP spreads independent (batch, channel) planes
 * over the host cores; each plane is computed by the same plain loops, and all
 * final sums are taken in a fixed order, so results do not depend on the thread
 * count.
 *
 * Return value of every entry point: 0 on success, 1 if the sizes lie outside
 * the operation's domain (nothing is written then).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define REF_OK 0
#define REF_BAD_SIZE 1

int fcvref_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* ------------------------------------------------------------------------- */
/* Op A: Conv2d(3x3, stride 1, no padding) -> AvgPool2d(P, stride P, floor)   */
/*       -> sigmoid -> sum over (C, PH, PW)                                  */
/* ------------------------------------------------------------------------- */

/* Output sizes of op A (l2_p65 trace, opening analysis: 384 -> 382 -> 95).
 * Conv output Ho = H - 3 + 1; pooled PH = floor(Ho / P). */
int fcvref_conv2d_out_dims(int H, int W, int P, int* Ho, int* Wo, int* PH, int* PW)
{
    if (H < 3 || W < 3 || P < 1) return REF_BAD_SIZE;
    *Ho = H - 3 + 1;
    *Wo = W - 3 + 1;
    *PH = *Ho / P;
    *PW = *Wo / P;
    return REF_OK;
}

static int conv2d_args_ok(int N, int Cin, int H, int W, int Cout, int P)
{
    return N >= 0 && Cin >= 1 && Cout >= 1 && H >= 3 && W >= 3 && P >= 1;
}

/* The full conv output plane of one (b, c): every Ho x Wo value, bias added to
 * each conv output exactly as the definition states it. */
static void conv2d_plane(const float* x, const float* w, const float* bias,
                         int b, int c, int Cin, int H, int W, double* plane)
{
    const int Ho = H - 2, Wo = W - 2;
    for (int y = 0; y < Ho; ++y)
        for (int xo = 0; xo < Wo; ++xo)
            plane[(size_t)y * Wo + xo] = (double)bias[c];
    for (int ic = 0; ic < Cin; ++ic) {
        const float* xin = x + ((size_t)b * Cin + ic) * (size_t)H * W;
        for (int ky = 0; ky < 3; ++ky) {
            for (int kx = 0; kx < 3; ++kx) {
                const double wv = (double)w[(((size_t)c * Cin + ic) * 3 + ky) * 3 + kx];
                for (int y = 0; y < Ho; ++y) {
                    const float* row = xin + (size_t)(y + ky) * W + kx;
                    double* prow = plane + (size_t)y * Wo;
                    for (int xo = 0; xo < Wo; ++xo)
                        prow[xo] += (double)row[xo] * wv;
                }
            }
        }
    }
}

/* Average of one P x P pooling window (stride P, no padding): the divisor is
 * always P*P because floor mode never creates a partial window. */
static double pool_window(const double* plane, int Wo, int P, int ph, int pw)
{
    double s = 0.0;
    for (int dy = 0; dy < P; ++dy)
        for (int dx = 0; dx < P; ++dx)
            s += plane[(size_t)(P * ph + dy) * Wo + (P * pw + dx)];
    return s / ((double)P * (double)P);
}

static double sigmoid(double v) { return 1.0 / (1.0 + exp(-v)); }

/* Pre-sigmoid pooled values pooled[N, Cout, PH, PW] (the "tap" of the fused
 * path).  Conv rows/cols past PH*P / PW*P are computed and then ignored, which
 * is the literal meaning of floor pooling. */
int fcvref_conv2d_pool_tap(const float* x, const float* w, const float* bias,
                           int N, int Cin, int H, int W, int Cout, int P,
                           double* pooled)
{
    if (!conv2d_args_ok(N, Cin, H, W, Cout, P)) return REF_BAD_SIZE;
    const int Ho = H - 2, Wo = W - 2, PH = Ho / P, PW = Wo / P;
    const long long planes = (long long)N * Cout;
    #pragma omp parallel
    {
        double* plane = (double*)malloc(sizeof(double) * (size_t)Ho * Wo);
        #pragma omp for schedule(dynamic, 1)
        for (long long bc = 0; bc < planes; ++bc) {
            const int b = (int)(bc / Cout), c = (int)(bc % Cout);
            conv2d_plane(x, w, bias, b, c, Cin, H, W, plane);
            double* dst = pooled + (size_t)bc * PH * PW;
            for (int ph = 0; ph < PH; ++ph)
                for (int pw = 0; pw < PW; ++pw)
                    dst[(size_t)ph * PW + pw] = pool_window(plane, Wo, P, ph, pw);
        }
        free(plane);
    }
    return REF_OK;
}

/* out[b] = sum_{c, ph, pw} sigmoid(avgpool(conv(x))[b, c, ph, pw]). */
int fcvref_conv2d_pool_sigmoid_sum(const float* x, const float* w, const float* bias,
                                   int N, int Cin, int H, int W, int Cout, int P,
                                   double* out)
{
    if (!conv2d_args_ok(N, Cin, H, W, Cout, P)) return REF_BAD_SIZE;
    const int Ho = H - 2, Wo = W - 2, PH = Ho / P, PW = Wo / P;
    const long long planes = (long long)N * Cout;
    double* partial = (double*)calloc((size_t)(planes > 0 ? planes : 1), sizeof(double));
    #pragma omp parallel
    {
        double* plane = (double*)malloc(sizeof(double) * (size_t)Ho * Wo);
        #pragma omp for schedule(dynamic, 1)
        for (long long bc = 0; bc < planes; ++bc) {
            const int b = (int)(bc / Cout), c = (int)(bc % Cout);
            conv2d_plane(x, w, bias, b, c, Cin, H, W, plane);
            double s = 0.0;
            for (int ph = 0; ph < PH; ++ph)
                for (int pw = 0; pw < PW; ++pw)
                    s += sigmoid(pool_window(plane, Wo, P, ph, pw));
            partial[bc] = s;
        }
        free(plane);
    }
    for (int b = 0; b < N; ++b) {
        double s = 0.0;
        for (int c = 0; c < Cout; ++c) s += partial[(size_t)b * Cout + c];
        out[b] = s;
    }
    free(partial);
    return REF_OK;
}

/* Selected pooled values, each evaluated on its own from the definition: the
 * P*P conv outputs of its window (each a 3x3xCin dot product plus bias), then
 * their mean.  idx holds n rows of (b, c, ph, pw).  Used where the full tensor
 * would take too long. */
int fcvref_conv2d_pool_tap_at(const float* x, const float* w, const float* bias,
                              int N, int Cin, int H, int W, int Cout, int P,
                              const int64_t* idx, int64_t n, double* vals)
{
    if (!conv2d_args_ok(N, Cin, H, W, Cout, P)) return REF_BAD_SIZE;
    const int Ho = H - 2, Wo = W - 2, PH = Ho / P, PW = Wo / P;
    for (int64_t i = 0; i < n; ++i) {
        const int64_t b = idx[4 * i], c = idx[4 * i + 1], ph = idx[4 * i + 2], pw = idx[4 * i + 3];
        if (b < 0 || b >= N || c < 0 || c >= Cout || ph < 0 || ph >= PH || pw < 0 || pw >= PW)
            return REF_BAD_SIZE;
    }
    #pragma omp parallel for schedule(dynamic, 16)
    for (int64_t i = 0; i < n; ++i) {
        const int64_t b = idx[4 * i], c = idx[4 * i + 1], ph = idx[4 * i + 2], pw = idx[4 * i + 3];
        double window = 0.0;
        for (int dy = 0; dy < P; ++dy) {
            for (int dx = 0; dx < P; ++dx) {
                const int64_t y = P * ph + dy, xo = P * pw + dx;
                double conv = (double)bias[c];
                for (int ic = 0; ic < Cin; ++ic)
                    for (int ky = 0; ky < 3; ++ky)
                        for (int kx = 0; kx < 3; ++kx)
                            conv += (double)x[(((size_t)b * Cin + ic) * H + (y + ky)) * (size_t)W + (xo + kx)]
                                  * (double)w[(((size_t)c * Cin + ic) * 3 + ky) * 3 + kx];
                window += conv;
            }
        }
        vals[i] = window / ((double)P * (double)P);
    }
    return REF_OK;
}

/* ------------------------------------------------------------------------- */
/* Op B: depthwise Conv1d(K, stride s, zero padding p, groups=C, no bias)     */
/*       -> pointwise Conv1d(1x1, C -> O) + bias[o]                          */
/* ------------------------------------------------------------------------- */

/* T_out = floor((T + 2p - K) / s) + 1 (l2_p7 trace, opening analysis:
 * (4096 + 2*4 - 9)/1 + 1 = 4096). */
int fcvref_conv1d_out_len(int T, int K, int s, int p, int* To)
{
    if (T < 1 || K < 1 || s < 1 || p < 0) return REF_BAD_SIZE;
    const long long span = (long long)T + 2LL * p - K;
    if (span < 0) return REF_BAD_SIZE;
    *To = (int)(span / s) + 1;
    return REF_OK;
}

static int conv1d_args_ok(int N, int C, int T, int O, int K, int s, int p, int* To)
{
    if (N < 0 || C < 1 || O < 1) return 0;
    return fcvref_conv1d_out_len(T, K, s, p, To) == REF_OK;
}

/* Input with zero padding: in[b, c, i] for 0 <= i < T, else 0. */
static double xpad(const float* xrow, int T, long long i)
{
    return (i >= 0 && i < T) ? (double)xrow[i] : 0.0;
}

/* The explicit two-stage definition: the depthwise conv output d[c, t] is
 * formed for every channel first, then the 1x1 conv mixes channels:
 *   d[b,c,t]   = sum_k xpad[b,c,t*s+k-p] * dw[c,k]
 *   out[b,o,t] = sum_c pw[o,c] * d[b,c,t] + bias[o]      (bias may be NULL)
 * Output out[N, O, To]. */
int fcvref_dwsep_conv1d(const float* x, const float* dw, const float* pw, const float* bias,
                        int N, int C, int T, int O, int K, int s, int p, double* out)
{
    int To;
    if (!conv1d_args_ok(N, C, T, O, K, s, p, &To)) return REF_BAD_SIZE;
    double* d = (double*)malloc(sizeof(double) * (size_t)C * To);
    for (int b = 0; b < N; ++b) {
        #pragma omp parallel for schedule(static)
        for (int c = 0; c < C; ++c) {
            const float* xrow = x + ((size_t)b * C + c) * T;
            for (int t = 0; t < To; ++t) {
                double acc = 0.0;
                for (int k = 0; k < K; ++k)
                    acc += xpad(xrow, T, (long long)t * s + k - p) * (double)dw[(size_t)c * K + k];
                d[(size_t)c * To + t] = acc;
            }
        }
        #pragma omp parallel for schedule(static)
        for (int o = 0; o < O; ++o) {
            double* orow = out + ((size_t)b * O + o) * To;
            const double bo = bias ? (double)bias[o] : 0.0;
            for (int t = 0; t < To; ++t) orow[t] = 0.0;
            for (int c = 0; c < C; ++c) {
                const double pv = (double)pw[(size_t)o * C + c];
                const double* drow = d + (size_t)c * To;
                for (int t = 0; t < To; ++t) orow[t] += pv * drow[t];
            }
            for (int t = 0; t < To; ++t) orow[t] += bo;
        }
    }
    free(d);
    return REF_OK;
}

/* Selected outputs, each evaluated on its own in the fused order of the page's
 * formula: sum over c of (the depthwise sum over k) times pw[o,c], plus bias.
 * idx holds n rows of (b, o, t). */
int fcvref_dwsep_conv1d_at(const float* x, const float* dw, const float* pw, const float* bias,
                           int N, int C, int T, int O, int K, int s, int p,
                           const int64_t* idx, int64_t n, double* vals)
{
    int To;
    if (!conv1d_args_ok(N, C, T, O, K, s, p, &To)) return REF_BAD_SIZE;
    for (int64_t i = 0; i < n; ++i) {
        const int64_t b = idx[3 * i], o = idx[3 * i + 1], t = idx[3 * i + 2];
        if (b < 0 || b >= N || o < 0 || o >= O || t < 0 || t >= To) return REF_BAD_SIZE;
    }
    #pragma omp parallel for schedule(dynamic, 16)
    for (int64_t i = 0; i < n; ++i) {
        const int64_t b = idx[3 * i], o = idx[3 * i + 1], t = idx[3 * i + 2];
        double acc = 0.0;
        for (int c = 0; c < C; ++c) {
            const float* xrow = x + ((size_t)b * C + c) * T;
            double dwsum = 0.0;
            for (int k = 0; k < K; ++k)
                dwsum += xpad(xrow, T, t * s + k - p) * (double)dw[(size_t)c * K + k];
            acc += dwsum * (double)pw[(size_t)o * C + c];
        }
        vals[i] = acc + (bias ? (double)bias[o] : 0.0);
    }
    return REF_OK;
}
