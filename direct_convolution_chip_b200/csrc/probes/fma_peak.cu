// fma_peak.cu -- FP32 FMA throughput probe (scalar fma.rn.f32 and packed
// fma.rn.f32x2), used to measure the FMA-pipe roofline on the device the
// benchmark runs on.  Each thread runs NCHAIN independent FMA chains so the
// pipe, not latency, bounds the rate.  Built as libfcv_probes.so.
#include <cuda_runtime.h>

namespace {

constexpr int NCHAIN = 8;

__global__ void __launch_bounds__(256) fma_scalar_kernel(float* sink, int iters, float a, float b)
{
    float v[NCHAIN];
#pragma unroll
    for (int j = 0; j < NCHAIN; ++j) v[j] = threadIdx.x * 1e-3f + j;
    for (int i = 0; i < iters; ++i) {
#pragma unroll
        for (int u = 0; u < 16; ++u)
#pragma unroll
            for (int j = 0; j < NCHAIN; ++j) v[j] = fmaf(v[j], a, b);
    }
    float s = 0.f;
#pragma unroll
    for (int j = 0; j < NCHAIN; ++j) s += v[j];
    if (s == 1234.5f) sink[blockIdx.x] = s;  // keeps the chains live
}

__global__ void __launch_bounds__(256) fma_packed_kernel(float* sink, int iters, float a, float b)
{
    float2 v[NCHAIN];
#pragma unroll
    for (int j = 0; j < NCHAIN; ++j) v[j] = make_float2(threadIdx.x * 1e-3f + j, j * 0.5f);
    const float2 a2 = make_float2(a, a), b2 = make_float2(b, b);
    for (int i = 0; i < iters; ++i) {
#pragma unroll
        for (int u = 0; u < 16; ++u)
#pragma unroll
            for (int j = 0; j < NCHAIN; ++j) v[j] = __ffma2_rn(v[j], a2, b2);
    }
    float s = 0.f;
#pragma unroll
    for (int j = 0; j < NCHAIN; ++j) s += v[j].x + v[j].y;
    if (s == 1234.5f) sink[blockIdx.x] = s;
}

}  // namespace

extern "C" {

// Runs the chosen FMA kernel on every SM (blocks_per_sm CTAs of 256 threads
// each) and writes the achieved FP32 rate in FLOP/s (2 per FMA) to *flops and
// the elapsed device time in ms to *ms.  Synchronizes the device.  Returns 0 on
// success, 1 on bad arguments, 3 on a CUDA error.
int fcvprobe_fma_rate(int packed, int blocks_per_sm, int iters, double* flops, double* ms)
{
    if (blocks_per_sm < 1 || iters < 1 || !flops || !ms) return 1;
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 3;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 3;
    const int blocks = sms * blocks_per_sm;
    float* sink = nullptr;
    if (cudaMalloc(&sink, sizeof(float) * blocks) != cudaSuccess) return 3;
    cudaEvent_t e0, e1;
    cudaEventCreate(&e0);
    cudaEventCreate(&e1);
    // warm-up launch, then the timed one
    for (int rep = 0; rep < 2; ++rep) {
        cudaEventRecord(e0);
        if (packed) fma_packed_kernel<<<blocks, 256>>>(sink, iters, 0.999f, 1e-4f);
        else fma_scalar_kernel<<<blocks, 256>>>(sink, iters, 0.999f, 1e-4f);
        cudaEventRecord(e1);
    }
    int st = (cudaEventSynchronize(e1) == cudaSuccess && cudaGetLastError() == cudaSuccess) ? 0 : 3;
    float t = 0.f;
    cudaEventElapsedTime(&t, e0, e1);
    const double fma_per_thread = (double)iters * 16.0 * NCHAIN * (packed ? 2.0 : 1.0);
    *flops = 2.0 * fma_per_thread * 256.0 * blocks / (t * 1e-3);
    *ms = t;
    cudaEventDestroy(e0);
    cudaEventDestroy(e1);
    cudaFree(sink);
    return st;
}

}  // extern "C"
