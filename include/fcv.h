/*
 * fcv.h -- C ABI of libfcv, fused small-channel direct convolution for
 * NVIDIA B200 (sm_100a).
 *
 * Two fused operations whose intermediate never reaches device memory:
 *
 *   A. conv2d 3x3 (stride 1, no padding) -> AvgPool2d(P, stride P, floor)
 *      -> sigmoid -> sum over (channels, pooled rows, pooled cols),
 *      one fp32 scalar per batch item.
 *      Defined on POPCORNBENCH trace "Kimi-K2.6__l2_p65" (fused Conv2d ->
 *      AvgPool2d -> Sigmoid -> Sum), opening analysis: the conv formula
 *      out[i,j] = sum_{c,ky,kx} in[b,c,i+ky,j+kx] * w[oc,c,ky,kx] + bias[oc],
 *      the shapes [128,8,384,384] -> [128,64,382,382] -> [128,64,95,95] -> [128],
 *      and the pool-semantics check (stride = kernel, floor, trailing rows and
 *      columns dropped).
 *
 *   B. depthwise conv1d (kernel K, stride s, zero padding p, no bias) folded
 *      into the pointwise 1x1 conv1d (C -> O) that consumes it, plus bias[o].
 *      Defined on POPCORNBENCH trace "Kimi-K2.6__l2_p7" (depthwise-separable
 *      Conv1d), opening analysis:
 *      out[b,o,t] = sum_c ( sum_k in[b,c,t*s+k-p] * dw[c,k] ) * pw[o,c] + bias[o],
 *      T_out = (T + 2p - K)/s + 1, input zero outside [0, T).
 *
 * Conventions for every compute entry point:
 *   - All tensor pointers are DEVICE pointers owned by the caller; fp32,
 *     contiguous, row-major (NCHW for op A, NCT for op B).  Inputs are read
 *     only.  Outputs must not alias inputs.  Pointers must be 4-byte aligned.
 *     A pointer may be NULL when its tensor has no elements, or when N == 0
 *     (nothing is then read or written); otherwise NULL is INVALID_ARG.
 *   - `stream` is a cudaStream_t passed as void*; NULL is the legacy default
 *     stream.  Calls are asynchronous on that stream: they never synchronize
 *     and never allocate memory.
 *   - Argument errors are reported synchronously, before anything is
 *     enqueued, with FCV_ERR_INVALID_ARG or FCV_ERR_UNSUPPORTED.  A launch
 *     failure reported by the CUDA runtime returns FCV_ERR_CUDA.  Device-side
 *     faults are never raised on purpose: a kernel whose bounded wait runs out
 *     records FCV_ERR_TIMEOUT in a device error word (fcv_device_error) and
 *     returns early.
 *   - N == 0 (an empty batch) is valid and enqueues nothing.
 *   - The library holds no per-call state; concurrent calls on different
 *     streams with disjoint outputs are safe.  Between calls it keeps, per
 *     device, the SM count and each kernel's raised shared-memory limit
 *     (looked up or set once, under a lock; set again after a failed launch,
 *     as after cudaDeviceReset).  The one exception is
 *     fcv_conv2d_pool_sigmoid_sum_noalloc: all its calls on a device share one
 *     library-owned 256 KiB array, so calls that overlap on the GPU race and
 *     must be serialised by the caller.
 */
#ifndef FCV_H
#define FCV_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    FCV_OK = 0,
    FCV_ERR_INVALID_ARG = 1, /* null pointer, size out of domain, misaligned pointer, overflow */
    FCV_ERR_UNSUPPORTED = 2, /* valid operation, but outside the shapes this build runs */
    FCV_ERR_CUDA = 3,        /* the CUDA runtime reported an error at launch */
    FCV_ERR_TIMEOUT = 4      /* a kernel's bounded wait ran out (see fcv_device_error) */
} fcv_status;

/* Algorithm selectors for the *_ex entry points.  FCV_ALGO_AUTO picks the
 * fastest path valid for the shape and pointers (fcv_conv2d_auto_algo and
 * fcv_dwsep_conv1d_auto_algo report which).  For op A it is always the direct
 * method (every conv output is computed): FCV_CONV2D_TC_SHIFT_3XTF32 where it
 * covers the shape, else FCV_CONV2D_TC_3XTF32 where that one does, except narrow
 * layers (Cin <= 4 and Cout <= 32) whose FP32-FMA grid has at least 128 CTAs
 * (there FP32 FMA measured faster), else FP32 FMA; the pool-first identity is
 * never chosen automatically.  The AUTO report for op A assumes a 16-byte
 * aligned x. */
typedef enum {
    FCV_ALGO_AUTO = 0,
    /* op A */
    FCV_CONV2D_DIRECT = 10,       /* direct 3x3 conv of every pooled window, FP32 FMA */
    FCV_CONV2D_POOLFIRST = 11,    /* pool the input first (exact identity, 9*Cin MACs per pooled
                                     value instead of 9*Cin*P*P), FP32 FMA; same results within
                                     rounding.  Never chosen by FCV_ALGO_AUTO, which keeps the
                                     direct method. */
    FCV_CONV2D_TC_3XTF32 = 12,    /* the direct method as an implicit GEMM on tcgen05 tensor
                                     cores (K = 9*Cin, N = Cout), fp32-accurate through a
                                     3xTF32 split; pool 1, 2, 4 or 8 and Cout <= 112 only,
                                     UNSUPPORTED otherwise */
    FCV_CONV2D_TC_SHIFT_3XTF32 = 13, /* the direct method on tcgen05 tensor cores with four images
                                     side by side in the MMA's N dimension, so that each of the
                                     nine taps reads the staged input rows in place (no im2col);
                                     M = 64 output channels x (TF32 hi | lo weights), fp32-accurate;
                                     Cin <= 16, pool 1, 2, 4 or 8 and a 16-byte aligned x only,
                                     UNSUPPORTED otherwise */
    /* op B */
    FCV_CONV1D_FMA = 20,          /* depthwise + pointwise on FP32 FMA */
    FCV_CONV1D_TC_3XTF32 = 21,    /* pointwise on tcgen05 tensor cores, 3xTF32 split, one SM per tile */
    FCV_CONV1D_TC2_3XTF32 = 22,   /* SM pairs (tcgen05 cta_group::2, 256x256 tiles), input halo
                                     and pw by TMA; stride 1 or 2, T % 4 == 0, 16-byte aligned x */
    FCV_CONV1D_TC_TMA_3XTF32 = 23 /* one SM per tile, input halo staged by TMA; stride 1 or 2,
                                     T % 4 == 0 and a 16-byte aligned x */
} fcv_algo;

/* ---------------------------------------------------------------- op A --- */

/* out[n] = sum_{c<Cout, ph<PH, pw<PW} sigmoid( avgpool_P( conv3x3(x, w) + b )[n,c,ph,pw] )
 *
 *   x    [N, Cin, H, W]     input
 *   w    [Cout, Cin, 3, 3]  conv weight
 *   b    [Cout]             conv bias (required)
 *   out  [N]                result; fully overwritten (the library zeroes it
 *                           on `stream` before accumulating)
 *   pool                    AvgPool2d kernel = stride, no padding, floor mode
 *
 * Ho = H - 2, Wo = W - 2, PH = floor(Ho / pool), PW = floor(Wo / pool).
 * PH == 0 or PW == 0 is valid and gives out = 0.
 * INVALID_ARG: x, w, b or out NULL while N > 0; N < 0; Cin, Cout < 1; H, W < 3; pool < 1;
 *              element counts beyond 2^31 * 2^31; misaligned pointers.
 * UNSUPPORTED: pool > 8.
 * The per-batch sum is accumulated with atomic adds (one per thread block and
 * image; one per warp and image on the im2col tensor-core path), so the last
 * bits may differ between runs. */
int fcv_conv2d_pool_sigmoid_sum(const float* x, const float* w, const float* b,
                                int N, int Cin, int H, int W, int Cout, int pool,
                                float* out, void* stream);

int fcv_conv2d_pool_sigmoid_sum_ex(const float* x, const float* w, const float* b,
                                   int N, int Cin, int H, int W, int Cout, int pool,
                                   float* out, int algo, void* stream);

/* Deterministic variant of fcv_conv2d_pool_sigmoid_sum: bitwise-identical
 * results from run to run.  Each thread block writes its partial sum to its
 * own slot of a caller-provided workspace; the block that finishes last for a
 * batch item (detected with a counter; nothing waits) adds that item's slots
 * in a fixed order and stores out[n].  Same result within rounding as the
 * atomic variant; the alternative the l2_p65 trace weighs in its
 * atomic-contention analysis (a per-tile workspace plus a fixed-order pass).
 *
 *   workspace        device memory owned by the caller, 16-byte aligned, at
 *                    least fcv_conv2d_workspace_bytes(...) bytes; its contents
 *                    on entry do not matter (the library clears what it needs
 *                    on `stream`).  Calls sharing a workspace must not overlap.
 *   workspace_bytes  its size.
 * INVALID_ARG additionally when the workspace is NULL, misaligned or too small
 * (a zero-byte requirement accepts NULL). */
int fcv_conv2d_pool_sigmoid_sum_det(const float* x, const float* w, const float* b,
                                    int N, int Cin, int H, int W, int Cout, int pool,
                                    float* out, void* workspace, size_t workspace_bytes,
                                    void* stream);

/* fcv_conv2d_pool_sigmoid_sum_det without a caller workspace and without any
 * allocation, for callers that may not allocate device memory while they run
 * (a plugin in an engine that owns all device memory, a loop that cannot take
 * the implicit synchronisation of cudaMalloc/cudaFree, a fixed memory budget).
 * The pages have no counterpart; this is a library facility.
 *
 * The workspace is a 256 KiB array in the library's own device memory (every
 * GPU that loads the library holds it until the process exits).  The first
 * call on each device looks up that array's address (cudaGetSymbolAddress) with
 * the device current and keeps it for later calls; make that first call before
 * any stream capture.  A failed lookup returns FCV_ERR_CUDA and is tried again
 * on the next call.  The kept address belongs to the device's context at the
 * time of the lookup: after cudaDeviceReset it is no longer valid, so do not
 * use this entry point in a process after resetting the device.  Sizes
 * whose workspace (fcv_conv2d_workspace_bytes) exceeds 256 KiB are rejected
 * with FCV_ERR_UNSUPPORTED before anything is enqueued.  All calls on a device
 * share the one array: calls that overlap on the GPU (other streams, other
 * host threads) race and must be serialised by the caller.  The array keeps
 * the previous call's contents; the call clears what must start at zero.
 * Otherwise the same arguments, results and errors as
 * fcv_conv2d_pool_sigmoid_sum_det; it calls no allocator. */
int fcv_conv2d_pool_sigmoid_sum_noalloc(const float* x, const float* w, const float* b,
                                        int N, int Cin, int H, int W, int Cout, int pool,
                                        float* out, void* stream);

/* Bytes of workspace fcv_conv2d_pool_sigmoid_sum_det needs for these sizes
 * (0 when nothing is launched, e.g. PH or PW == 0).  Host only, no CUDA call.
 * Same INVALID_ARG / UNSUPPORTED rules as the compute entry points. */
int fcv_conv2d_workspace_bytes(int N, int Cin, int H, int W, int Cout, int pool, size_t* bytes);

/* The pooled pre-sigmoid values of the same kernel, for checking the conv and
 * pool stages element by element:
 *   pooled [N, Cout, PH, PW]  = avgpool_P( conv3x3(x, w) + b ), fully overwritten.
 * Same arguments, errors and algorithms as fcv_conv2d_pool_sigmoid_sum_ex;
 * nothing is summed.  `pooled` may be NULL when PH or PW is 0. */
int fcv_conv2d_pool_tap(const float* x, const float* w, const float* b,
                        int N, int Cin, int H, int W, int Cout, int pool,
                        float* pooled, int algo, void* stream);

/* ---------------------------------------------------------------- op B --- */

/* out[n,o,t] = sum_{c<C} pw_w[o,c] * ( sum_{k<K} xpad[n,c,t*stride+k-pad] * dw_w[c,k] ) + bias[o]
 *
 *   x     [N, C, T]   input; xpad is x with zeros outside [0, T)
 *   dw_w  [C, K]      depthwise weight (the [C,1,K] tensor)
 *   pw_w  [O, C]      pointwise weight (the [O,C,1] tensor)
 *   bias  [O] or NULL (NULL: no bias)
 *   out   [N, O, To]  To = floor((T + 2*pad - K) / stride) + 1; fully overwritten
 *
 * The depthwise result lives only in on-chip memory.  Every algorithm is
 * fp32-accurate (FP32 FMA, or tensor cores through a 3xTF32 split); results
 * are deterministic run to run.
 * FCV_ALGO_AUTO takes FCV_CONV1D_TC2_3XTF32 when C >= 256 and either stride
 * is 2 or stride is 1 and O >= 256, with K <= 13, C % 4 == 0, T % 4 == 0, x
 * and pw_w 16-byte aligned and 32*ceil(C/32)*K <= 8192 (where the SM pair
 * measured faster); else
 * FCV_CONV1D_TC_TMA_3XTF32 when stride is 1 or 2, K <= 13, C % 4 == 0,
 * T % 4 == 0, x and pw_w are 16-byte aligned and 32*ceil(C/32)*K <= 8192;
 * else FCV_CONV1D_TC_3XTF32 when stride == 1, K <= 13, C % 4 == 0,
 * pw_w is 16-byte aligned and C*K <= 4000; else FCV_CONV1D_FMA.  An explicit
 * tensor-core algorithm outside its conditions returns UNSUPPORTED.
 * INVALID_ARG: x, dw_w, pw_w or out NULL while N > 0; N < 0; C, O, T, K, stride < 1;
 *              pad < 0; To < 1; sizes beyond the 64-bit index range;
 *              misaligned pointers.
 * UNSUPPORTED: K > 32, pad >= 2^20, stride > 8. */
int fcv_dwsep_conv1d(const float* x, const float* dw_w, const float* pw_w, const float* bias,
                     int N, int C, int T, int O, int K, int stride, int pad,
                     float* out, void* stream);

int fcv_dwsep_conv1d_ex(const float* x, const float* dw_w, const float* pw_w, const float* bias,
                        int N, int C, int T, int O, int K, int stride, int pad,
                        float* out, int algo, void* stream);

/* -------------------------------------------------------------- utility --- */

/* The algorithm FCV_ALGO_AUTO runs for these sizes, written to *algo; no CUDA
 * call is made.  Returns the status the compute call would return for invalid
 * or unsupported sizes (INVALID_ARG also when algo is NULL). */
int fcv_conv2d_auto_algo(int N, int Cin, int H, int W, int Cout, int pool, int* algo);

/* The same for op B; x and pw_w matter only through their 16-byte alignment
 * (they are not read). */
int fcv_dwsep_conv1d_auto_algo(const float* x, const float* pw_w, int N, int C, int T, int O, int K,
                               int stride, int pad, int* algo);

/* Diagnostic (layout may change between versions): what one launch of
 * FCV_CONV2D_TC_3XTF32 uses for these sizes.  use_tma says whether the input
 * halo comes by TMA (W % 4 == 0 and a 16-byte aligned x).  Writes the kernel
 * variant (1 = sub-chunk, 0 = full-chunk), the accumulator buffers, the tensor
 * memory columns the kernel addresses (of the 512 it allocates) and the dynamic
 * shared memory it requests.  FCV_ERR_UNSUPPORTED outside that kernel's
 * envelope, FCV_ERR_INVALID_ARG for a NULL output or sizes < 1.  No CUDA call. */
int fcv_conv2d_tc_plan(int Cin, int Cout, int pool, int use_tma, int* variant, int* nacc, int* tmem_cols,
                       unsigned int* smem_bytes);

/* Human-readable name of a status code (static storage). */
const char* fcv_status_string(int status);

/* Library version, major * 10000 + minor * 100 + patch. */
int fcv_version(void);

/* Synchronizes `stream`, then returns and clears the device error word of the
 * current device: FCV_OK, or FCV_ERR_TIMEOUT if a kernel gave up a bounded
 * wait since the last call.  Returns FCV_ERR_CUDA if the synchronization fails. */
int fcv_device_error(void* stream);

/* Self-test of the failure path (no counterpart on the pages): launches one
 * tiny kernel whose thread waits, with limit `limit_ns` (1 ns .. 10 s), on a
 * barrier that nothing completes.  The bounded wait gives up, records
 * FCV_ERR_TIMEOUT in the device error word and the kernel exits normally, so a
 * following fcv_device_error(stream) returns FCV_ERR_TIMEOUT and the context
 * stays usable.  Nothing faults, traps or hangs.  Asynchronous on `stream`. */
int fcv_selftest_wait_timeout(unsigned long long limit_ns, void* stream);

/* Test of the failure path of the shifted-operand tensor-core conv2d
 * (FCV_CONV2D_TC_SHIFT_3XTF32; no counterpart on the pages).  Runs that kernel
 * on op A's arguments, except that one role of every thread block waits, just
 * before its `at_unit`-th unit of work, on a barrier nothing completes, with a
 * wait limit of `limit_ns` (1 ns .. 10 s; the same limit then bounds that
 * block's other main-loop waits).  The wait gives up, records FCV_ERR_TIMEOUT
 * in the device error word and sets the block's abort flag; every role leaves
 * its loop, the copies and MMAs already issued are waited for, tensor memory
 * is freed and the kernel exits.  `out` is zeroed first and then holds a
 * partial sum.  role: 1 loader, 2 producers, 3 MMA issuer, 4 epilogue.
 * INVALID_ARG for a role outside 1..4, at_unit < 0 or limit_ns outside its
 * range, UNSUPPORTED where that kernel does not apply; otherwise as
 * fcv_conv2d_pool_sigmoid_sum.  Asynchronous on `stream`. */
int fcv_selftest_conv2d_stall(const float* x, const float* w, const float* b,
                              int N, int Cin, int H, int W, int Cout, int pool,
                              float* out, int role, int at_unit, unsigned long long limit_ns,
                              void* stream);

/* The same test for op B's TMA-halo tensor-core kernel (FCV_CONV1D_TC_TMA_3XTF32):
 * one role of every thread block (1 TMA warp, 2 producers, 3 MMA issuer, 4
 * epilogue) waits, before its `at_tile`-th output tile, on a barrier nothing
 * completes, with limit `limit_ns` (1 ns .. 10 s); the block then takes its
 * abort path and FCV_ERR_TIMEOUT is recorded.  `out` holds partial results.
 * INVALID_ARG / UNSUPPORTED as for fcv_selftest_conv2d_stall, with that
 * kernel's envelope; otherwise as fcv_dwsep_conv1d. */
int fcv_selftest_conv1d_stall(const float* x, const float* dw_w, const float* pw_w, const float* bias,
                              int N, int C, int T, int O, int K, int stride, int pad,
                              float* out, int role, int at_tile, unsigned long long limit_ns,
                              void* stream);

/* The same test for op B's SM-pair kernel (FCV_CONV1D_TC2_3XTF32): in the CTA
 * of rank `rank` (0 leads the pair, 1 is its peer) of every pair, role `role`
 * (1 TMA warp, 2 depthwise producers, 3 MMA issuer -- rank 0 only, 4 epilogue,
 * 5 pw split warps, 6 relay -- rank 1 only) waits, before its `at_tile`-th
 * pair tile, on a barrier nothing completes, with limit `limit_ns` (1 ns ..
 * 10 s).  That CTA takes its abort path, its peer sees the abort flag through
 * distributed shared memory and leaves as well, and FCV_ERR_TIMEOUT is
 * recorded; `out` holds partial results.  INVALID_ARG for a role, rank or
 * limit outside those ranges; UNSUPPORTED outside that kernel's envelope;
 * otherwise as fcv_dwsep_conv1d. */
int fcv_selftest_conv1d_pair_stall(const float* x, const float* dw_w, const float* pw_w, const float* bias,
                                   int N, int C, int T, int O, int K, int stride, int pad,
                                   float* out, int role, int at_tile, int rank, unsigned long long limit_ns,
                                   void* stream);

#ifdef __cplusplus
}
#endif

#endif /* FCV_H */
