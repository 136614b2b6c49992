// fcv_lib.cu -- the extern "C" boundary of libfcv (declared in include/fcv.h).
//
// Host side only: argument validation (synchronous, before anything is
// enqueued), output zeroing, algorithm dispatch and launch-status mapping.
// Every arithmetic step of both operations runs in the kernels included below.
#include <stdint.h>

#include "common.cuh"
#include "conv1d_fma.cuh"
#include "conv1d_tc.cuh"
#include "conv1d_tc2.cuh"
#include "conv1d_tcx.cuh"
#include "conv2d_direct.cuh"
#include "conv2d_poolfirst.cuh"
#include "conv2d_tc.cuh"
#include "conv2d_tcs.cuh"

#define FCV_VERSION_MAJOR 0
#define FCV_VERSION_MINOR 1
#define FCV_VERSION_PATCH 0

namespace {

bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

// a * b * c * d without int64 overflow (all factors >= 0).
bool mul_ok(long long a, long long b, long long c, long long d)
{
    const long long lim = (long long)1 << 62;
    long long v = a;
    for (long long f : {b, c, d}) {
        if (f != 0 && v > lim / f) return false;
        v *= f;
    }
    return true;
}

// A pointer may be NULL exactly when the tensor behind it has no elements or
// nothing is read or written (N == 0); otherwise it must be non-NULL and
// 4-byte aligned.
bool ptr_ok(const void* p, bool needed) { return needed ? (p != nullptr && aligned4(p)) : aligned4(p); }

int check_conv2d(const float* x, const float* w, const float* b, int N, int Cin, int H, int W,
                 int Cout, int pool, const float* out, bool tap)
{
    if (N < 0 || Cin < 1 || Cout < 1 || H < 3 || W < 3 || pool < 1) return FCV_ERR_INVALID_ARG;
    if (!mul_ok(N, Cin, H, W) || !mul_ok(Cout, Cin, 9, 1) || !mul_ok(N, Cout, H, W))
        return FCV_ERR_INVALID_ARG;
    const bool work = N > 0;
    const bool out_has_elems = work && (!tap || ((H - 2) / pool > 0 && (W - 2) / pool > 0));
    if (!ptr_ok(x, work) || !ptr_ok(w, work) || !ptr_ok(b, work) || !ptr_ok(out, out_has_elems))
        return FCV_ERR_INVALID_ARG;
    if (pool > 8) return FCV_ERR_UNSUPPORTED;
    return FCV_OK;
}

int check_conv1d(const float* x, const float* dw, const float* pw, const float* bias, int N, int C,
                 int T, int O, int K, int stride, int pad, const float* out, int* To)
{
    if (N < 0 || C < 1 || O < 1 || T < 1 || K < 1 || stride < 1 || pad < 0) return FCV_ERR_INVALID_ARG;
    const bool work = N > 0;
    if (!ptr_ok(x, work) || !ptr_ok(dw, work) || !ptr_ok(pw, work) || !ptr_ok(out, work) || !aligned4(bias))
        return FCV_ERR_INVALID_ARG;
    const long long span = (long long)T + 2LL * pad - K;
    if (span < 0) return FCV_ERR_INVALID_ARG;  // To < 1
    const long long to = span / stride + 1;
    if (to > 0x7fffffffLL) return FCV_ERR_INVALID_ARG;
    if (!mul_ok(N, C, T, 1) || !mul_ok(N, O, to, 1) || !mul_ok(O, C, 1, 1)) return FCV_ERR_INVALID_ARG;
    if (K > fcv::Conv1dFmaTile::KMAX || stride > fcv::Conv1dFmaTile::SMAX || pad >= (1 << 20))
        return FCV_ERR_UNSUPPORTED;
    *To = (int)to;
    return FCV_OK;
}

// Smallest FMA-kernel grid (CTAs) at which AUTO lets it take a narrow layer.
constexpr long long kConv2dFmaMinCtas = 128;

// What AUTO runs for op A.  Narrow layers (Cin <= 4 and Cout <= 32) whose FMA
// grid fills at least kConv2dFmaMinCtas CTAs stay on FP32 FMA: the tensor-core
// kernels pad Cin to 8 input channels and Cout to 64, so the FMA kernel, whose
// time scales with Cin * Cout, does less work there (x[16,3,509,509], Cout 32,
// pool 4: FMA 187 us, shifted-operand tensor cores 201 us; Cin 4: 240 against
// 214, Cout 48: 339 against 203).  Otherwise the shifted-operand tensor-core
// kernel where it applies (Cin <= 16, pool 1, 2, 4 or 8, 16-byte aligned x;
// it beat FMA by 1.7-3.2x at Cin 8 and 16 on 509 x 509 images), else the
// im2col tensor-core kernel where it applies, else FP32 FMA.
int conv2d_auto_algo_for(int N, int Cin, int Cout, int pool, int PH, int PW, bool x_aligned16)
{
    const bool tcs = fcv::conv2d_tcs_supported(Cin, pool, x_aligned16 ? reinterpret_cast<const void*>(16)
                                                                      : reinterpret_cast<const void*>(4));
    const bool tc = fcv::conv2d_tc_supported(Cin, Cout, pool);
    if (!tcs && !tc) return FCV_CONV2D_DIRECT;
    if (Cin <= 4 && Cout <= 32) {
        int ty = 0, tx = 0, cb = 0;
        if (fcv::conv2d_grid(pool, PH, PW, Cout, &ty, &tx, &cb) &&
            (long long)N * ty * tx * cb >= kConv2dFmaMinCtas)
            return FCV_CONV2D_DIRECT;
    }
    return tcs ? FCV_CONV2D_TC_SHIFT_3XTF32 : FCV_CONV2D_TC_3XTF32;
}

int conv2d_common(const float* x, const float* w, const float* b, int N, int Cin, int H, int W,
                  int Cout, int pool, float* out, int algo, bool tap, void* stream)
{
    int st = check_conv2d(x, w, b, N, Cin, H, W, Cout, pool, out, tap);
    if (st != FCV_OK) return st;
    if (algo != FCV_ALGO_AUTO && algo != FCV_CONV2D_DIRECT && algo != FCV_CONV2D_POOLFIRST &&
        algo != FCV_CONV2D_TC_3XTF32 && algo != FCV_CONV2D_TC_SHIFT_3XTF32)
        return FCV_ERR_INVALID_ARG;
    if (algo == FCV_CONV2D_TC_3XTF32 && !fcv::conv2d_tc_supported(Cin, Cout, pool)) return FCV_ERR_UNSUPPORTED;
    if (algo == FCV_CONV2D_TC_SHIFT_3XTF32 && !fcv::conv2d_tcs_supported(Cin, pool, x)) return FCV_ERR_UNSUPPORTED;
    if (N == 0) return FCV_OK;
    cudaStream_t s = fcv::as_stream(stream);
    const int PH = (H - 2) / pool, PW = (W - 2) / pool;
    if (!tap) {
        // The kernels accumulate atomic adds into out[n]; start from zero.
        if (cudaMemsetAsync(out, 0, sizeof(float) * (size_t)N, s) != cudaSuccess) return FCV_ERR_CUDA;
    }
    if (PH == 0 || PW == 0) return FCV_OK;  // empty sum: out stays 0; the tap has no elements
    if (algo == FCV_ALGO_AUTO)
        algo = conv2d_auto_algo_for(N, Cin, Cout, pool, PH, PW, (reinterpret_cast<uintptr_t>(x) & 15) == 0);
    switch (algo) {
    case FCV_CONV2D_TC_SHIFT_3XTF32:
        return tap ? fcv::launch_conv2d_tcs<fcv::kTap>(x, w, b, N, Cin, H, W, Cout, pool, PH, PW, out, s)
                   : fcv::launch_conv2d_tcs<fcv::kSumAtomic>(x, w, b, N, Cin, H, W, Cout, pool, PH, PW, out, s);
    case FCV_CONV2D_TC_3XTF32:
        return tap ? fcv::launch_conv2d_tc<fcv::kTap>(x, w, b, N, Cin, H, W, Cout, pool, PH, PW, out, s)
                   : fcv::launch_conv2d_tc<fcv::kSumAtomic>(x, w, b, N, Cin, H, W, Cout, pool, PH, PW, out, s);
    case FCV_CONV2D_POOLFIRST:
        return tap ? fcv::launch_conv2d_poolfirst<fcv::kTap>(x, w, b, N, Cin, H, W, Cout, pool, PH, PW, out, s)
                   : fcv::launch_conv2d_poolfirst<fcv::kSumAtomic>(x, w, b, N, Cin, H, W, Cout, pool, PH, PW, out, s);
    default:
        return tap ? fcv::launch_conv2d_direct<fcv::kTap>(x, w, b, N, Cin, H, W, Cout, pool, PH, PW, out, s)
                   : fcv::launch_conv2d_direct<fcv::kSumAtomic>(x, w, b, N, Cin, H, W, Cout, pool, PH, PW, out, s);
    }
}

}  // namespace

extern "C" {

int fcv_conv2d_workspace_bytes(int N, int Cin, int H, int W, int Cout, int pool, size_t* bytes)
{
    if (!bytes) return FCV_ERR_INVALID_ARG;
    if (N < 0 || Cin < 1 || Cout < 1 || H < 3 || W < 3 || pool < 1) return FCV_ERR_INVALID_ARG;
    if (!mul_ok(N, Cin, H, W) || !mul_ok(N, Cout, H, W)) return FCV_ERR_INVALID_ARG;
    if (pool > 8) return FCV_ERR_UNSUPPORTED;
    *bytes = fcv::conv2d_det_workspace_bytes(N, Cout, pool, (H - 2) / pool, (W - 2) / pool);
    return FCV_OK;
}

int fcv_conv2d_pool_sigmoid_sum_det(const float* x, const float* w, const float* b, int N, int Cin, int H,
                                    int W, int Cout, int pool, float* out, void* workspace,
                                    size_t workspace_bytes, void* stream)
{
    int st = check_conv2d(x, w, b, N, Cin, H, W, Cout, pool, out, false);
    if (st != FCV_OK) return st;
    const int PH = (H - 2) / pool, PW = (W - 2) / pool;
    const size_t need = fcv::conv2d_det_workspace_bytes(N, Cout, pool, PH, PW);
    if (need > 0 && (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 15) != 0 || workspace_bytes < need))
        return FCV_ERR_INVALID_ARG;
    if (N == 0) return FCV_OK;
    cudaStream_t s = fcv::as_stream(stream);
    if (PH == 0 || PW == 0) {
        return cudaMemsetAsync(out, 0, sizeof(float) * (size_t)N, s) == cudaSuccess ? FCV_OK : FCV_ERR_CUDA;
    }
    unsigned char* base = static_cast<unsigned char*>(workspace);
    unsigned int* counters = reinterpret_cast<unsigned int*>(base + need - sizeof(unsigned int) * (size_t)N);
    if (cudaMemsetAsync(counters, 0, sizeof(unsigned int) * (size_t)N, s) != cudaSuccess) return FCV_ERR_CUDA;
    return fcv::launch_conv2d_direct<fcv::kSumDet>(x, w, b, N, Cin, H, W, Cout, pool, PH, PW, out, s,
                                                   reinterpret_cast<float*>(base), counters);
}

int fcv_conv2d_pool_sigmoid_sum(const float* x, const float* w, const float* b, int N, int Cin, int H,
                                int W, int Cout, int pool, float* out, void* stream)
{
    return conv2d_common(x, w, b, N, Cin, H, W, Cout, pool, out, FCV_ALGO_AUTO, false, stream);
}

int fcv_conv2d_pool_sigmoid_sum_ex(const float* x, const float* w, const float* b, int N, int Cin,
                                   int H, int W, int Cout, int pool, float* out, int algo, void* stream)
{
    return conv2d_common(x, w, b, N, Cin, H, W, Cout, pool, out, algo, false, stream);
}

int fcv_conv2d_pool_tap(const float* x, const float* w, const float* b, int N, int Cin, int H, int W,
                        int Cout, int pool, float* pooled, int algo, void* stream)
{
    return conv2d_common(x, w, b, N, Cin, H, W, Cout, pool, pooled, algo, true, stream);
}

int fcv_dwsep_conv1d_ex(const float* x, const float* dw_w, const float* pw_w, const float* bias, int N,
                        int C, int T, int O, int K, int stride, int pad, float* out, int algo, void* stream)
{
    int To = 0;
    int st = check_conv1d(x, dw_w, pw_w, bias, N, C, T, O, K, stride, pad, out, &To);
    if (st != FCV_OK) return st;
    if (N == 0) return FCV_OK;
    cudaStream_t s = fcv::as_stream(stream);
    switch (algo) {
    case FCV_ALGO_AUTO:
        if (fcv::conv1d_tc2_preferred(C, T, O, K, stride, x, pw_w))
            return fcv::launch_dwsep_conv1d_tc2(x, dw_w, pw_w, bias, N, C, T, O, K, stride, pad, To, out, s);
        if (fcv::conv1d_tcx_supported(C, T, O, K, stride, x, pw_w))
            return fcv::launch_dwsep_conv1d_tcx(x, dw_w, pw_w, bias, N, C, T, O, K, stride, pad, To, out, s);
        if (fcv::conv1d_tc_supported(C, O, K, stride, pw_w)) {
            return fcv::launch_dwsep_conv1d_tc(x, dw_w, pw_w, bias, N, C, T, O, K, stride, pad, To, out, s);
        }
        return fcv::launch_dwsep_conv1d_fma(x, dw_w, pw_w, bias, N, C, T, O, K, stride, pad, To, out, s);
    case FCV_CONV1D_TC2_3XTF32:
        if (!fcv::conv1d_tc2_supported(C, T, O, K, stride, x, pw_w)) return FCV_ERR_UNSUPPORTED;
        return fcv::launch_dwsep_conv1d_tc2(x, dw_w, pw_w, bias, N, C, T, O, K, stride, pad, To, out, s);
    case FCV_CONV1D_FMA:
        return fcv::launch_dwsep_conv1d_fma(x, dw_w, pw_w, bias, N, C, T, O, K, stride, pad, To, out, s);
    case FCV_CONV1D_TC_3XTF32:
        if (!fcv::conv1d_tc_supported(C, O, K, stride, pw_w)) return FCV_ERR_UNSUPPORTED;
        return fcv::launch_dwsep_conv1d_tc(x, dw_w, pw_w, bias, N, C, T, O, K, stride, pad, To, out, s);
    case FCV_CONV1D_TC_TMA_3XTF32:
        if (!fcv::conv1d_tcx_supported(C, T, O, K, stride, x, pw_w)) return FCV_ERR_UNSUPPORTED;
        return fcv::launch_dwsep_conv1d_tcx(x, dw_w, pw_w, bias, N, C, T, O, K, stride, pad, To, out, s);
    default:
        return FCV_ERR_INVALID_ARG;
    }
}

int fcv_dwsep_conv1d(const float* x, const float* dw_w, const float* pw_w, const float* bias, int N,
                     int C, int T, int O, int K, int stride, int pad, float* out, void* stream)
{
    return fcv_dwsep_conv1d_ex(x, dw_w, pw_w, bias, N, C, T, O, K, stride, pad, out, FCV_ALGO_AUTO, stream);
}

int fcv_selftest_wait_timeout(unsigned long long limit_ns, void* stream)
{
    if (limit_ns == 0 || limit_ns > 10ull * 1000 * 1000 * 1000) return FCV_ERR_INVALID_ARG;
    fcv::tc::selftest_wait_timeout_kernel<<<1, 32, 0, fcv::as_stream(stream)>>>(limit_ns);
    return fcv::launch_status();
}

int fcv_selftest_conv2d_stall(const float* x, const float* w, const float* b, int N, int Cin, int H, int W,
                              int Cout, int pool, float* out, int role, int at_unit, unsigned long long limit_ns,
                              void* stream)
{
    int st = check_conv2d(x, w, b, N, Cin, H, W, Cout, pool, out, false);
    if (st != FCV_OK) return st;
    if (role < 1 || role > 4 || at_unit < 0 || limit_ns == 0 || limit_ns > 10ull * 1000 * 1000 * 1000)
        return FCV_ERR_INVALID_ARG;
    if (!fcv::conv2d_tcs_supported(Cin, pool, x)) return FCV_ERR_UNSUPPORTED;
    if (N == 0) return FCV_OK;
    cudaStream_t s = fcv::as_stream(stream);
    const int PH = (H - 2) / pool, PW = (W - 2) / pool;
    if (cudaMemsetAsync(out, 0, sizeof(float) * (size_t)N, s) != cudaSuccess) return FCV_ERR_CUDA;
    if (PH == 0 || PW == 0) return FCV_OK;
    return fcv::launch_conv2d_tcs<fcv::kSumAtomic>(x, w, b, N, Cin, H, W, Cout, pool, PH, PW, out, s, limit_ns, role,
                                                   at_unit);
}

int fcv_selftest_conv1d_stall(const float* x, const float* dw_w, const float* pw_w, const float* bias, int N, int C,
                              int T, int O, int K, int stride, int pad, float* out, int role, int at_tile,
                              unsigned long long limit_ns, void* stream)
{
    int To = 0;
    int st = check_conv1d(x, dw_w, pw_w, bias, N, C, T, O, K, stride, pad, out, &To);
    if (st != FCV_OK) return st;
    if (role < 1 || role > 4 || at_tile < 0 || limit_ns == 0 || limit_ns > 10ull * 1000 * 1000 * 1000)
        return FCV_ERR_INVALID_ARG;
    if (!fcv::conv1d_tcx_supported(C, T, O, K, stride, x, pw_w)) return FCV_ERR_UNSUPPORTED;
    if (N == 0) return FCV_OK;
    return fcv::launch_dwsep_conv1d_tcx(x, dw_w, pw_w, bias, N, C, T, O, K, stride, pad, To, out,
                                        fcv::as_stream(stream), role, at_tile, limit_ns);
}

int fcv_selftest_conv1d_pair_stall(const float* x, const float* dw_w, const float* pw_w, const float* bias, int N,
                                   int C, int T, int O, int K, int stride, int pad, float* out, int role,
                                   int at_tile, int rank, unsigned long long limit_ns, void* stream)
{
    int To = 0;
    int st = check_conv1d(x, dw_w, pw_w, bias, N, C, T, O, K, stride, pad, out, &To);
    if (st != FCV_OK) return st;
    if (role < 1 || role > 6 || rank < 0 || rank > 1 || (role == 3 && rank != 0) || (role == 6 && rank != 1) ||
        (role == 5 && stride != 1) || at_tile < 0 || limit_ns == 0 || limit_ns > 10ull * 1000 * 1000 * 1000)
        return FCV_ERR_INVALID_ARG;
    if (!fcv::conv1d_tc2_supported(C, T, O, K, stride, x, pw_w)) return FCV_ERR_UNSUPPORTED;
    if (N == 0) return FCV_OK;
    return fcv::launch_dwsep_conv1d_tc2(x, dw_w, pw_w, bias, N, C, T, O, K, stride, pad, To, out,
                                        fcv::as_stream(stream), role, at_tile, rank, limit_ns);
}

int fcv_conv2d_auto_algo(int N, int Cin, int H, int W, int Cout, int pool, int* algo)
{
    if (!algo) return FCV_ERR_INVALID_ARG;
    if (N < 0 || Cin < 1 || Cout < 1 || H < 3 || W < 3 || pool < 1) return FCV_ERR_INVALID_ARG;
    if (!mul_ok(N, Cin, H, W) || !mul_ok(N, Cout, H, W)) return FCV_ERR_INVALID_ARG;
    if (pool > 8) return FCV_ERR_UNSUPPORTED;
    const int PH = (H - 2) / pool, PW = (W - 2) / pool;
    *algo = conv2d_auto_algo_for(N, Cin, Cout, pool, PH, PW, true);
    return FCV_OK;
}

int fcv_conv2d_tc_plan(int Cin, int Cout, int pool, int use_tma, int* variant, int* nacc, int* tmem_cols,
                       unsigned int* smem_bytes)
{
    if (!variant || !nacc || !tmem_cols || !smem_bytes) return FCV_ERR_INVALID_ARG;
    if (Cin < 1 || Cout < 1 || pool < 1) return FCV_ERR_INVALID_ARG;
    if (!fcv::conv2d_tc_supported(Cin, Cout, pool)) return FCV_ERR_UNSUPPORTED;
    fcv::Conv2dTcPlan pl;
    if (!fcv::conv2d_tc_plan_for(Cin, Cout, pool, use_tma != 0, &pl)) return FCV_ERR_UNSUPPORTED;
    *variant = pl.sub;
    *nacc = pl.nacc;
    *tmem_cols = pl.tmem_cols;
    *smem_bytes = pl.smem;
    return FCV_OK;
}

int fcv_dwsep_conv1d_auto_algo(const float* x, const float* pw_w, int N, int C, int T, int O, int K, int stride,
                               int pad, int* algo)
{
    if (!algo) return FCV_ERR_INVALID_ARG;
    int To = 0;
    // Validation without reading any data: the pointers stand in for the
    // tensors only through their alignment.
    const float* dummy = reinterpret_cast<const float*>(16);
    float* odummy = reinterpret_cast<float*>(16);
    const int st = check_conv1d(N > 0 && !x ? dummy : x, dummy, N > 0 && !pw_w ? dummy : pw_w, nullptr, N, C, T, O,
                                K, stride, pad, odummy, &To);
    if (st != FCV_OK) return st;
    if (fcv::conv1d_tc2_preferred(C, T, O, K, stride, x, pw_w)) *algo = FCV_CONV1D_TC2_3XTF32;
    else if (fcv::conv1d_tcx_supported(C, T, O, K, stride, x, pw_w)) *algo = FCV_CONV1D_TC_TMA_3XTF32;
    else if (fcv::conv1d_tc_supported(C, O, K, stride, pw_w)) *algo = FCV_CONV1D_TC_3XTF32;
    else *algo = FCV_CONV1D_FMA;
    return FCV_OK;
}

const char* fcv_status_string(int status)
{
    switch (status) {
    case FCV_OK: return "FCV_OK";
    case FCV_ERR_INVALID_ARG: return "FCV_ERR_INVALID_ARG: invalid argument";
    case FCV_ERR_UNSUPPORTED: return "FCV_ERR_UNSUPPORTED: shape outside the supported envelope";
    case FCV_ERR_CUDA: return "FCV_ERR_CUDA: CUDA runtime error";
    case FCV_ERR_TIMEOUT: return "FCV_ERR_TIMEOUT: a kernel's bounded wait ran out";
    default: return "unknown fcv status";
    }
}

int fcv_version(void)
{
    return FCV_VERSION_MAJOR * 10000 + FCV_VERSION_MINOR * 100 + FCV_VERSION_PATCH;
}

int fcv_device_error(void* stream)
{
    if (cudaStreamSynchronize(fcv::as_stream(stream)) != cudaSuccess) return FCV_ERR_CUDA;
    unsigned int v = 0;
    if (cudaMemcpyFromSymbol(&v, fcv::g_device_error, sizeof(v)) != cudaSuccess) return FCV_ERR_CUDA;
    if (v != 0) {
        const unsigned int zero = 0;
        if (cudaMemcpyToSymbol(fcv::g_device_error, &zero, sizeof(zero)) != cudaSuccess) return FCV_ERR_CUDA;
    }
    return (v & fcv::kErrTimeout) ? FCV_ERR_TIMEOUT : FCV_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Allocation-free variant of the deterministic conv2d sum.
//
// Some callers cannot allocate device memory at the point where they run this
// operation: a plugin inside an inference engine or framework that owns every
// device allocation and forbids cudaMalloc while it executes, a latency-critical
// loop that cannot afford the implicit device synchronisation cudaMalloc and
// cudaFree may perform, or a deployment whose device-memory budget is fixed at
// start-up.  For them the workspace of fcv_conv2d_pool_sigmoid_sum_det lives in
// a fixed-size array that the library places in device memory when it is
// loaded; every GPU that loads the library keeps that array until the process
// exits.
// ---------------------------------------------------------------------------

#include <mutex>

namespace {

constexpr size_t kNoAllocScratchBytes = 256 * 1024;  // the largest workspace this variant serves

// One instance per device (per CUDA context).  In host code this name is only a
// host-side stand-in for the device array: its device address comes from
// cudaGetSymbolAddress below, never from taking the address here.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kNoAllocMaxDevices = 64;
std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kNoAllocMaxDevices];  // cached device address per device; NULL until a lookup succeeds

// Device address of g_noalloc_scratch on the current device, looked up with
// that device current the first time it is needed and then cached.  A failed
// lookup is not cached: the next call tries again.
int noalloc_scratch(void** ptr)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return FCV_ERR_CUDA;
    if (dev < 0 || dev >= kNoAllocMaxDevices) return FCV_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (g_noalloc_ptr[dev] == nullptr) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) {
            (void)cudaGetLastError();  // leave no sticky status behind for the caller's next call
            return FCV_ERR_CUDA;
        }
        g_noalloc_ptr[dev] = p;
    }
    *ptr = g_noalloc_ptr[dev];
    return FCV_OK;
}

}  // namespace

extern "C" int fcv_conv2d_pool_sigmoid_sum_noalloc(const float* x, const float* w, const float* b, int N,
                                                   int Cin, int H, int W, int Cout, int pool, float* out,
                                                   void* stream)
{
    int st = check_conv2d(x, w, b, N, Cin, H, W, Cout, pool, out, false);
    if (st != FCV_OK) return st;
    const int PH = (H - 2) / pool, PW = (W - 2) / pool;
    const size_t need = fcv::conv2d_det_workspace_bytes(N, Cout, pool, PH, PW);
    if (need > kNoAllocScratchBytes) return FCV_ERR_UNSUPPORTED;  // too large for the static scratch
    if (N == 0) return FCV_OK;
    cudaStream_t s = fcv::as_stream(stream);
    if (PH == 0 || PW == 0) {
        return cudaMemsetAsync(out, 0, sizeof(float) * (size_t)N, s) == cudaSuccess ? FCV_OK : FCV_ERR_CUDA;
    }
    void* scratch = nullptr;
    st = noalloc_scratch(&scratch);
    if (st != FCV_OK) return st;
    // The array keeps whatever the previous call left: clear the per-image
    // counters, which must start at zero (the partial-sum slots are always
    // written before they are read).
    unsigned char* base = static_cast<unsigned char*>(scratch);
    unsigned int* counters = reinterpret_cast<unsigned int*>(base + need - sizeof(unsigned int) * (size_t)N);
    if (cudaMemsetAsync(counters, 0, sizeof(unsigned int) * (size_t)N, s) != cudaSuccess) return FCV_ERR_CUDA;
    return fcv::launch_conv2d_direct<fcv::kSumDet>(x, w, b, N, Cin, H, W, Cout, pool, PH, PW, out, s,
                                                   reinterpret_cast<float*>(base), counters);
}
