// common.cuh -- internals shared by the libfcv kernels (one translation unit).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>
#include <mutex>
#include <vector>

#include "../../include/fcv.h"

namespace fcv {

// Device error word of the current device.  A kernel whose bounded wait runs
// out ORs a code in here and returns early; fcv_device_error() reads and
// clears it.  Nothing in the library traps or faults on purpose.
__device__ unsigned int g_device_error;

constexpr unsigned int kErrTimeout = 1u;

__device__ __forceinline__ void record_device_error(unsigned int code)
{
    atomicOr(&g_device_error, code);
}

// Sum of `v` over a thread block, valid in thread 0.  `scratch` holds one
// float per warp.
template <int NT>
__device__ __forceinline__ float block_sum(float v, float* scratch)
{
    static_assert(NT % 32 == 0, "block size must be a multiple of 32");
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if (lane == 0) scratch[warp] = v;
    __syncthreads();
    float s = 0.f;
    if (threadIdx.x < 32) {
        s = (lane < NT / 32) ? scratch[lane] : 0.f;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
    }
    return s;
}

// 4-byte asynchronous global->shared copy; when `pred` is false nothing is
// read and the destination is zero-filled (src-size 0).  `gsrc` must still be
// a valid global address, so callers pass a base pointer in that case.
__device__ __forceinline__ void cp_async4(void* smem_dst, const void* gsrc, bool pred)
{
    const unsigned s = (unsigned)__cvta_generic_to_shared(smem_dst);
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;\n" ::"r"(s), "l"(gsrc), "r"(pred ? 4 : 0)
                 : "memory");
}

// 16-byte asynchronous global->shared copy of `bytes` (0..16) valid bytes; the
// rest of the 16 destination bytes are zero-filled.  Both addresses must be
// 16-byte aligned (for bytes == 0 pass an aligned base pointer).
__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gsrc, int bytes)
{
    const unsigned s = (unsigned)__cvta_generic_to_shared(smem_dst);
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(s), "l"(gsrc), "r"(bytes) : "memory");
}

__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }

template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory"); }

inline cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

inline int launch_status()
{
    return cudaGetLastError() == cudaSuccess ? FCV_OK : FCV_ERR_CUDA;
}

// ---------------------------------------------------------------------------
// Host-side launch state kept between calls.  A call on a small problem
// should cost little more than its launch, so the SM count is looked up once
// per device and each kernel's dynamic shared-memory limit is raised once per
// device; a context reset (cudaDeviceReset) drops that limit, which shows as a
// failed launch, after which launch_cached sets it again and launches once
// more.

constexpr int kMaxCachedDevices = 64;

// Number of SMs of the current device.
inline int device_sm_count(int* sms)
{
    static std::atomic<int> cache[kMaxCachedDevices];  // static storage: zero until looked up
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return FCV_ERR_CUDA;
    const bool cached = dev >= 0 && dev < kMaxCachedDevices;
    if (cached) {
        const int v = cache[dev].load(std::memory_order_relaxed);
        if (v > 0) {
            *sms = v;
            return FCV_OK;
        }
    }
    int v = 0;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0) return FCV_ERR_CUDA;
    if (cached) cache[dev].store(v, std::memory_order_relaxed);
    *sms = v;
    return FCV_OK;
}

struct SmemLimit {
    const void* fn;
    int dev;
    int bytes;
};

inline std::mutex& smem_limit_mu()
{
    static std::mutex m;
    return m;
}

inline std::vector<SmemLimit>& smem_limits()
{
    static std::vector<SmemLimit> v;
    return v;
}

// Raise `fn`'s dynamic shared-memory limit to `bytes` on the current device
// unless an earlier call already did.
inline int ensure_smem_limit(const void* fn, int bytes)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return FCV_ERR_CUDA;
    std::lock_guard<std::mutex> lock(smem_limit_mu());
    for (const SmemLimit& e : smem_limits())
        if (e.fn == fn && e.dev == dev && e.bytes >= bytes) return FCV_OK;
    if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess) return FCV_ERR_CUDA;
    for (SmemLimit& e : smem_limits())
        if (e.fn == fn && e.dev == dev) {
            e.bytes = bytes;
            return FCV_OK;
        }
    smem_limits().push_back({fn, dev, bytes});
    return FCV_OK;
}

inline void forget_smem_limit(const void* fn)
{
    std::lock_guard<std::mutex> lock(smem_limit_mu());
    auto& v = smem_limits();
    for (size_t i = 0; i < v.size();)
        if (v[i].fn == fn) {
            v[i] = v.back();
            v.pop_back();
        } else {
            ++i;
        }
}

// Launch through `go` (a callable that issues the <<<...>>> launch) with the
// kernel's shared-memory limit raised; after a failed launch the limit is set
// again and the launch repeated once.
template <typename Kern, typename Go>
inline int launch_cached(Kern kern, int smem_bytes, Go&& go)
{
    const void* fn = reinterpret_cast<const void*>(kern);
    if (ensure_smem_limit(fn, smem_bytes) != FCV_OK) return FCV_ERR_CUDA;
    go();
    if (cudaGetLastError() == cudaSuccess) return FCV_OK;
    forget_smem_limit(fn);
    if (ensure_smem_limit(fn, smem_bytes) != FCV_OK) return FCV_ERR_CUDA;
    go();
    return launch_status();
}

}  // namespace fcv
