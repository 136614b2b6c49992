// tf32_mma_rate.cu -- tcgen05 TF32 MMA throughput probe: the tensor-core
// roofline of the 3xTF32 kernels, measured on the device instead of derived
// from the bf16 GEMM figure.  One CTA per SM; one thread issues `iters`
// back-to-back tcgen05.mma.cta_group::1.kind::tf32 (M = 128, K = 8, N = 64,
// 128 or 256) into 1, 2 or 4 TMEM accumulators, with A read from shared
// memory or from tensor memory, committing every 96 MMAs.  The operands are
// whatever the buffers hold: only the rate is measured.  Built into
// libfcv_probes.so.
#include <cuda_runtime.h>
#include <stdint.h>

namespace {

__device__ __forceinline__ uint32_t smem_u32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

__device__ __forceinline__ unsigned long long gtimer()
{
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;\n" : "=l"(t));
    return t;
}

// K-major operand, 128-byte swizzle, 8-row groups 1024 B apart.
__device__ __forceinline__ uint64_t desc_sw128(uint32_t saddr)
{
    return (uint64_t)((saddr & 0x3FFFFu) >> 4) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
           ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

__device__ __forceinline__ void mma_ss(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc)
{
    asm volatile("tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, 1;\n" ::"r"(d), "l"(a), "l"(b), "r"(idesc)
                 : "memory");
}

__device__ __forceinline__ void mma_ts(uint32_t d, uint32_t a, uint64_t b, uint32_t idesc)
{
    asm volatile("tcgen05.mma.cta_group::1.kind::tf32 [%0], [%1], %2, %3, 1;\n" ::"r"(d), "r"(a), "l"(b), "r"(idesc)
                 : "memory");
}

// The MMA sequence is a 3xTF32 contraction: for each of 4 K-steps (one
// 128-byte K block) A_hi*B_hi, A_hi*B_lo, A_lo*B_hi, K-step s going to
// accumulator s mod CHAINS.  Descriptors are computed once, so the issuing
// thread spends a few instructions per MMA and the tensor core sets the rate.
template <int N, bool A_TMEM, int CHAINS>
__global__ void __launch_bounds__(128, 1) mma_rate_kernel(int outer, int issuers, unsigned long long* cycles,
                                                          unsigned int* timeouts)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    const uint32_t a_hi_s = smem_u32(smem);            // 128 rows x 128 B
    const uint32_t a_lo_s = a_hi_s + 128 * 128;
    const uint32_t b_hi_s = a_lo_s + 128 * 128;        // N <= 256 rows x 128 B
    const uint32_t b_lo_s = b_hi_s + 256 * 128;
    const uint32_t bar = b_lo_s + 256 * 128;
    __shared__ uint32_t tmem_holder;
    const int ncommits = issuers * ((outer + 7) / 8);

    if (threadIdx.x == 0) {
        asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(bar), "r"(ncommits) : "memory");
        asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
    }
    if (threadIdx.x < 32) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 512;\n" ::"r"(smem_u32(&tmem_holder))
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::: "memory");
    }
    asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory");
    const uint32_t tmem = tmem_holder;

    // Issuer i (lane 0 of warp i) drives accumulator columns [i * CHAINS * N, ...).
    const int issuer = threadIdx.x >> 5;
    if ((threadIdx.x & 31) == 0 && issuer < issuers) {
        const uint32_t idesc = (1u << 4) | (2u << 7) | (2u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);
        const uint32_t dbase = tmem + (uint32_t)(issuer * CHAINS * N);
        uint64_t bh[4], bl[4], ah[4], al[4];
        uint32_t th[4], tl[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            bh[k] = desc_sw128(b_hi_s + 32u * k);
            bl[k] = desc_sw128(b_lo_s + 32u * k);
            ah[k] = desc_sw128(a_hi_s + 32u * k);
            al[k] = desc_sw128(a_lo_s + 32u * k);
            th[k] = tmem + 448u + 8u * k;  // A_hi in TMEM columns 448..479
            tl[k] = tmem + 480u + 8u * k;  // A_lo in TMEM columns 480..511
        }
        const unsigned long long c0 = clock64();
        for (int it = 0; it < outer; ++it) {
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const uint32_t d = dbase + (uint32_t)((k % CHAINS) * N);
                if (A_TMEM) {
                    mma_ts(d, th[k], bh[k], idesc);
                    mma_ts(d, th[k], bl[k], idesc);
                    mma_ts(d, tl[k], bh[k], idesc);
                } else {
                    mma_ss(d, ah[k], bh[k], idesc);
                    mma_ss(d, ah[k], bl[k], idesc);
                    mma_ss(d, al[k], bh[k], idesc);
                }
            }
            if ((it & 7) == 7 || it == outer - 1)
                asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n" ::"r"(bar)
                             : "memory");
        }
        // Every commit has arrived once all MMAs completed (bounded wait).
        const unsigned long long t0 = gtimer();
        uint32_t done = 0;
        while (!done) {
            asm volatile(
                "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], 0;\n selp.u32 %0, 1, 0, p;\n}\n"
                : "=r"(done)
                : "r"(bar)
                : "memory");
            if (!done && gtimer() - t0 > 2000000000ull) {
                atomicAdd(timeouts, 1u);
                break;
            }
        }
        if (issuer == 0) cycles[blockIdx.x] = clock64() - c0;
    }
    asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory");
    if (threadIdx.x < 32)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;\n" ::"r"(tmem) : "memory");
}

template <int N, bool A_TMEM, int CHAINS>
int run(int blocks, int outer, int issuers, unsigned long long* cycles, unsigned int* timeouts, float* ms)
{
    // Operand buffers take 97 KB; 160 KB keeps one CTA per SM (each allocates
    // all 512 TMEM columns).
    const int smem = 160 * 1024;
    auto k = mma_rate_kernel<N, A_TMEM, CHAINS>;
    if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess) return 3;
    cudaEvent_t e0, e1;
    cudaEventCreate(&e0);
    cudaEventCreate(&e1);
    for (int rep = 0; rep < 2; ++rep) {  // warm-up, then the timed launch
        cudaEventRecord(e0);
        k<<<blocks, 128, smem>>>(outer, issuers, cycles, timeouts);
        cudaEventRecord(e1);
    }
    const int st = (cudaEventSynchronize(e1) == cudaSuccess && cudaGetLastError() == cudaSuccess) ? 0 : 3;
    cudaEventElapsedTime(ms, e0, e1);
    cudaEventDestroy(e0);
    cudaEventDestroy(e1);
    return st;
}

template <int N, bool A_TMEM>
int run_chains(int chains, int blocks, int outer, int issuers, unsigned long long* cycles, unsigned int* timeouts,
               float* ms)
{
    if (chains == 1) return run<N, A_TMEM, 1>(blocks, outer, issuers, cycles, timeouts, ms);
    if (chains == 2) return run<N, A_TMEM, 2>(blocks, outer, issuers, cycles, timeouts, ms);
    return run<N, A_TMEM, 4>(blocks, outer, issuers, cycles, timeouts, ms);
}

}  // namespace

extern "C" {

// Runs the probe on every SM and reports the TF32 rate in FLOP/s (2 per MAC)
// over the whole device, the elapsed time, and the average SM cycles per MMA
// instruction.  n: 32, 64, 128 or 256; a_tmem: 0 (A in shared memory) or 1 (A in
// tensor memory); chains: 1, 2 or 4 independent accumulators per issuing
// thread; issuers: 1 or 2 threads (in different warps) issuing at once, with
// issuers * chains * n <= 448; iters: MMAs per issuer, a multiple of 12.  Synchronizes the
// device.  Returns 0 on success, 1 on bad arguments, 3 on a CUDA error, 4 if a
// wait timed out (the result is then meaningless).
int fcvprobe_tf32_mma_rate(int n, int a_tmem, int chains, int issuers, int iters, double* flops, double* ms,
                           double* cycles_per_mma)
{
    if ((n != 32 && n != 64 && n != 128 && n != 256) || (chains != 1 && chains != 2 && chains != 4) ||
        (issuers != 1 && issuers != 2) || issuers * chains * n > 448 || iters < 12 || iters % 12 != 0 ||
        iters / 96 > (1 << 18) || !flops || !ms || !cycles_per_mma)
        return 1;
    const int outer = iters / 12;
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 3;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 3;
    unsigned long long* cycles = nullptr;
    unsigned int* timeouts = nullptr;
    if (cudaMalloc(&cycles, sizeof(unsigned long long) * sms) != cudaSuccess) return 3;
    if (cudaMalloc(&timeouts, sizeof(unsigned int)) != cudaSuccess) {
        cudaFree(cycles);
        return 3;
    }
    cudaMemset(timeouts, 0, sizeof(unsigned int));
    float t = 0.f;
    int st;
    if (n == 32) st = a_tmem ? run_chains<32, true>(chains, sms, outer, issuers, cycles, timeouts, &t)
                             : run_chains<32, false>(chains, sms, outer, issuers, cycles, timeouts, &t);
    else if (n == 64) st = a_tmem ? run_chains<64, true>(chains, sms, outer, issuers, cycles, timeouts, &t)
                             : run_chains<64, false>(chains, sms, outer, issuers, cycles, timeouts, &t);
    else if (n == 128) st = a_tmem ? run_chains<128, true>(chains, sms, outer, issuers, cycles, timeouts, &t)
                                   : run_chains<128, false>(chains, sms, outer, issuers, cycles, timeouts, &t);
    else st = a_tmem ? run_chains<256, true>(chains, sms, outer, issuers, cycles, timeouts, &t)
                     : run_chains<256, false>(chains, sms, outer, issuers, cycles, timeouts, &t);
    unsigned long long* hc = new unsigned long long[sms];
    unsigned int to = 0;
    if (st == 0 && (cudaMemcpy(hc, cycles, sizeof(unsigned long long) * sms, cudaMemcpyDeviceToHost) != cudaSuccess ||
                    cudaMemcpy(&to, timeouts, sizeof(unsigned int), cudaMemcpyDeviceToHost) != cudaSuccess))
        st = 3;
    if (st == 0) {
        double c = 0.0;
        for (int i = 0; i < sms; ++i) c += (double)hc[i];
        *cycles_per_mma = c / sms / ((double)iters * issuers);
        *ms = t;
        *flops = 2.0 * 128.0 * n * 8.0 * (double)iters * issuers * sms / (t * 1e-3);
        if (to) st = 4;
    }
    delete[] hc;
    cudaFree(cycles);
    cudaFree(timeouts);
    return st;
}

}  // extern "C"
