// umma_layout.cu -- probes of the tcgen05.mma kind::tf32 operand layouts and
// costs that the shifted-operand conv2d kernel is built on.  Built into
// libfcv_probes.so; every probe is one kernel launch on host-built shared
// memory images, with bounded waits.
//
//   fcvprobe_umma_b_map   one MMA per K index k0 (M = 128, N = 256, K = 8): A is
//       1 in column k0 of every row (K-major, no swizzle: rows 16 bytes apart,
//       the second 4-element K half 128 bytes further, 8-row groups 256 bytes
//       apart), B holds the float index of each shared-memory word.  Row 0 of
//       D then shows, for every N index, the word the tensor core read for
//       (k0, n): the B address map of the given descriptor and major bit.
//   fcvprobe_umma_m64_rows  one M = 64, N = 64 MMA with A row m = m + 1 in
//       column 0 and B = 1: which TMEM lane holds which row of D (lanes the
//       MMA does not write keep the fill value -7).
//   fcvprobe_umma_cycles  one CTA per SM, one thread issuing `iters` MMAs
//       back to back (M = 64 or 128, N = 192 or 256, A from shared memory or
//       tensor memory, both K-major without swizzle); SM cycles per MMA.
//   fcvprobe_umma_b_map_ex  the B address map of a K-major descriptor with a
//       given layout type (none, 128/64/32-byte swizzle), leading and stride
//       byte offsets, start address offset from a 1024-byte aligned image and
//       descriptor base-offset field.
//   fcvprobe_umma_cycles_ex  the rate probe with such a B descriptor whose
//       start address cycles through 0, shift, 2*shift bytes (the three column
//       taps of a shifted-operand convolution).
#include <cuda_runtime.h>
#include <stdint.h>

namespace {

__device__ __forceinline__ uint32_t su32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

__device__ __forceinline__ uint64_t desc_none(uint32_t addr, uint32_t lbo, uint32_t sbo)
{
    return (uint64_t)((addr & 0x3FFFFu) >> 4) | ((uint64_t)(lbo >> 4) << 16) | ((uint64_t)(sbo >> 4) << 32) |
           ((uint64_t)1 << 46);
}

// Descriptor with a layout type (bits 61-63: 0 none, 2 SW128, 4 SW64, 6 SW32)
// and base-offset field (bits 49-51).
__device__ __forceinline__ uint64_t desc_gen(uint32_t addr, uint32_t lbo, uint32_t sbo, uint32_t layout,
                                             uint32_t base_off)
{
    return desc_none(addr, lbo, sbo) | ((uint64_t)(base_off & 7u) << 49) | ((uint64_t)(layout & 7u) << 61);
}

__device__ __forceinline__ uint32_t idesc_tf32(int m, int n, int b_major)
{
    return (1u << 4) | (2u << 7) | (2u << 10) | ((uint32_t)b_major << 16) | ((uint32_t)(n >> 3) << 17) |
           ((uint32_t)(m >> 4) << 24);
}

__device__ __forceinline__ bool wait_parity(uint32_t bar, uint32_t parity)
{
    uint32_t ok = 0;
    for (int it = 0; it < 4000000 && !ok; ++it)
        asm volatile(
            "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
            : "=r"(ok)
            : "r"(bar), "r"(parity)
            : "memory");
    return ok != 0;
}

__device__ __forceinline__ void fence_before() { asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory"); }
__device__ __forceinline__ void fence_after() { asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory"); }

// Shared memory: A image at 0 (16 KB), B image at 16 KB (48 KB); 64 KB dynamic.
constexpr int A_WORDS = 4096, B_WORDS = 12288;
constexpr uint32_t SMEM_BYTES = 65536;

// mode 0: B address map (k0 = 0..7, one MMA each, row 0 of D copied out per k0)
// mode 1: M = 64 row layout
__global__ void __launch_bounds__(128, 1) layout_kernel(int mode, int b_major, uint32_t lbo, uint32_t sbo,
                                                        uint32_t layout, uint32_t start_off, uint32_t base_off,
                                                        float* d_out, unsigned* status)
{
    extern __shared__ __align__(1024) uint8_t sm[];
    float* A = reinterpret_cast<float*>(sm);
    float* B = reinterpret_cast<float*>(sm + 16384);
    __shared__ __align__(8) unsigned long long bar;
    __shared__ uint32_t tmem_holder;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;\n" ::"r"(su32(&bar)) : "memory");
        asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
    }
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 256;\n" ::"r"(su32(&tmem_holder))
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::: "memory");
    }
    fence_before();
    __syncthreads();
    fence_after();
    const uint32_t tmem = tmem_holder;
    unsigned ok_all = 1;
    const int rounds = mode == 0 ? 8 : 1;
    for (int r = 0; r < rounds; ++r) {
        // operand images
        for (int i = threadIdx.x; i < A_WORDS; i += blockDim.x) A[i] = 0.f;
        for (int i = threadIdx.x; i < B_WORDS; i += blockDim.x)
            B[i] = mode == 0 ? (float)(i & 2047) : 0.f;  // word index (exact in TF32 below 2048)
        __syncthreads();
        for (int m = threadIdx.x; m < 128; m += blockDim.x) {
            const int k = mode == 0 ? r : 0;
            A[((m & 7) * 16 + (m >> 3) * 256 + (k >> 2) * 128 + (k & 3) * 4) / 4] = mode == 0 ? 1.f : (float)(m + 1);
        }
        if (mode == 1)
            for (int n = threadIdx.x; n < 64; n += blockDim.x) B[((n & 7) * 16 + (n >> 3) * 256) / 4] = 1.f;
        // D columns 0..255 filled with -7 so that lanes the MMA leaves alone show
        {
            uint32_t v[8];
            for (int j = 0; j < 8; ++j) v[j] = __float_as_uint(-7.f);
            for (int c = 0; c < 256; c += 8)
                asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};\n" ::"r"(
                                 tmem + ((uint32_t)(32 * warp) << 16) + (uint32_t)c),
                             "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]));
            asm volatile("tcgen05.wait::st.sync.aligned;\n" ::: "memory");
        }
        asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
        fence_before();
        __syncthreads();
        fence_after();
        if (threadIdx.x == 0) {
            const uint64_t ad = desc_none(su32(A), 128, 256);
            const uint64_t bd =
                mode == 0 ? desc_gen(su32(B) + start_off, lbo, sbo, layout, base_off) : desc_none(su32(B), 128, 256);
            const uint32_t id = mode == 0 ? idesc_tf32(128, 256, b_major) : idesc_tf32(64, 64, 0);
            asm volatile("tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, 0;\n" ::"r"(tmem), "l"(ad), "l"(bd),
                         "r"(id)
                         : "memory");
            asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n" ::"r"(
                             su32(&bar))
                         : "memory");
            ok_all &= wait_parity(su32(&bar), (uint32_t)(r & 1)) ? 1u : 0u;
        }
        fence_before();
        __syncthreads();
        fence_after();
        // copy out: mode 0 -> row 0 (lane 0) of D, 256 columns, per k0; mode 1 -> column 0 of all 128 lanes
        uint32_t v[8];
        if (mode == 0) {
            if (warp == 0) {
                for (int c = 0; c < 256; c += 8) {
                    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];\n"
                                 : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
                                   "=r"(v[7])
                                 : "r"(tmem + (uint32_t)c));
                    asm volatile("tcgen05.wait::ld.sync.aligned;\n" ::: "memory");
                    if (lane == 0)
                        for (int j = 0; j < 8; ++j) d_out[r * 256 + c + j] = __uint_as_float(v[j]);
                }
            }
        } else {
            asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];\n"
                         : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
                           "=r"(v[7])
                         : "r"(tmem + ((uint32_t)(32 * warp) << 16)));
            asm volatile("tcgen05.wait::ld.sync.aligned;\n" ::: "memory");
            d_out[32 * warp + lane] = __uint_as_float(v[0]);
        }
        fence_before();
        __syncthreads();
        fence_after();
    }
    if (threadIdx.x == 0) *status = ok_all;
    fence_before();
    __syncthreads();
    fence_after();
    if (warp == 0) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 256;\n" ::"r"(tmem) : "memory");
}

// Rate: one thread per CTA issues `iters` MMAs into one accumulator, then
// commits and waits (bounded); SM cycles from clock64.
__global__ void __launch_bounds__(128, 1) cycles_kernel(int m, int n, int a_tmem, int iters, uint32_t layout,
                                                        uint32_t lbo, uint32_t sbo, uint32_t shift,
                                                        unsigned long long* cycles, unsigned* status)
{
    extern __shared__ __align__(1024) uint8_t sm[];
    float* A = reinterpret_cast<float*>(sm);
    float* B = reinterpret_cast<float*>(sm + 16384);
    __shared__ __align__(8) unsigned long long bar;
    __shared__ uint32_t tmem_holder;
    const int warp = threadIdx.x >> 5;
    for (int i = threadIdx.x; i < A_WORDS; i += blockDim.x) A[i] = 1.f / 1024.f;
    for (int i = threadIdx.x; i < B_WORDS; i += blockDim.x) B[i] = 1.f / 1024.f;
    if (threadIdx.x == 0) {
        asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;\n" ::"r"(su32(&bar)) : "memory");
        asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
    }
    asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 512;\n" ::"r"(su32(&tmem_holder))
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::: "memory");
    }
    fence_before();
    __syncthreads();
    fence_after();
    const uint32_t tmem = tmem_holder;
    if (threadIdx.x == 0) {
        const uint64_t ad = desc_none(su32(A), 128, 256);
        const uint64_t bd0 = desc_gen(su32(B), lbo, sbo, layout, 0);
        const uint64_t bd1 = desc_gen(su32(B) + shift, lbo, sbo, layout, 0);
        const uint64_t bd2 = desc_gen(su32(B) + 2 * shift, lbo, sbo, layout, 0);
        const uint32_t id = idesc_tf32(m, n, 0);
        const uint32_t a_t = tmem + 256;  // A in tensor memory: columns 256..263 (contents do not matter)
        const long long t0 = clock64();
        for (int i = 0; i < iters; i += 3) {
            if (a_tmem) {
                asm volatile("tcgen05.mma.cta_group::1.kind::tf32 [%0], [%1], %2, %3, 1;\n" ::"r"(tmem), "r"(a_t),
                             "l"(bd0), "r"(id)
                             : "memory");
                asm volatile("tcgen05.mma.cta_group::1.kind::tf32 [%0], [%1], %2, %3, 1;\n" ::"r"(tmem), "r"(a_t),
                             "l"(bd1), "r"(id)
                             : "memory");
                asm volatile("tcgen05.mma.cta_group::1.kind::tf32 [%0], [%1], %2, %3, 1;\n" ::"r"(tmem), "r"(a_t),
                             "l"(bd2), "r"(id)
                             : "memory");
            } else {
                asm volatile("tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, 1;\n" ::"r"(tmem), "l"(ad),
                             "l"(bd0), "r"(id)
                             : "memory");
                asm volatile("tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, 1;\n" ::"r"(tmem), "l"(ad),
                             "l"(bd1), "r"(id)
                             : "memory");
                asm volatile("tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, 1;\n" ::"r"(tmem), "l"(ad),
                             "l"(bd2), "r"(id)
                             : "memory");
            }
        }
        asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n" ::"r"(
                         su32(&bar))
                     : "memory");
        const bool ok = wait_parity(su32(&bar), 0);
        if (blockIdx.x == 0) {
            *cycles = (unsigned long long)(clock64() - t0);
            *status = ok ? 1u : 0u;
        }
    }
    fence_before();
    __syncthreads();
    fence_after();
    if (warp == 0) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;\n" ::"r"(tmem) : "memory");
}

}  // namespace

extern "C" {

// B address map: out[k0 * 256 + n] = shared-memory word read for (k0, n).
// Returns 0, 1 (bad arguments), 2 (CUDA error) or 3 (an MMA did not complete).
int fcvprobe_umma_b_map(int b_major, unsigned lbo, unsigned sbo, float* out_host)
{
    if ((b_major != 0 && b_major != 1) || lbo > 512 || sbo > 512 || (lbo & 15) || (sbo & 15) || !out_host) return 1;
    float* d = nullptr;
    unsigned* st = nullptr;
    if (cudaMalloc(&d, 8 * 256 * sizeof(float)) != cudaSuccess) return 2;
    if (cudaMalloc(&st, sizeof(unsigned)) != cudaSuccess) {
        cudaFree(d);
        return 2;
    }
    cudaFuncSetAttribute(layout_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES);
    layout_kernel<<<1, 128, SMEM_BYTES>>>(0, b_major, lbo, sbo, 0, 0, 0, d, st);
    unsigned ok = 0;
    int rc = cudaDeviceSynchronize() == cudaSuccess ? 0 : 2;
    if (!rc && cudaMemcpy(out_host, d, 8 * 256 * sizeof(float), cudaMemcpyDeviceToHost) != cudaSuccess) rc = 2;
    if (!rc && cudaMemcpy(&ok, st, sizeof(unsigned), cudaMemcpyDeviceToHost) != cudaSuccess) rc = 2;
    cudaFree(d);
    cudaFree(st);
    return rc ? rc : (ok ? 0 : 3);
}

// M = 64 rows: out[lane] = row + 1 held by TMEM lane `lane` (-7: not written).
int fcvprobe_umma_m64_rows(float* out_host)
{
    if (!out_host) return 1;
    float* d = nullptr;
    unsigned* st = nullptr;
    if (cudaMalloc(&d, 128 * sizeof(float)) != cudaSuccess) return 2;
    if (cudaMalloc(&st, sizeof(unsigned)) != cudaSuccess) {
        cudaFree(d);
        return 2;
    }
    cudaFuncSetAttribute(layout_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES);
    layout_kernel<<<1, 128, SMEM_BYTES>>>(1, 0, 128, 256, 0, 0, 0, d, st);
    unsigned ok = 0;
    int rc = cudaDeviceSynchronize() == cudaSuccess ? 0 : 2;
    if (!rc && cudaMemcpy(out_host, d, 128 * sizeof(float), cudaMemcpyDeviceToHost) != cudaSuccess) rc = 2;
    if (!rc && cudaMemcpy(&ok, st, sizeof(unsigned), cudaMemcpyDeviceToHost) != cudaSuccess) rc = 2;
    cudaFree(d);
    cudaFree(st);
    return rc ? rc : (ok ? 0 : 3);
}

// SM cycles per MMA (CTA 0 of one CTA per SM) for M in {64, 128}, N in {192, 256}.
int fcvprobe_umma_cycles(int m, int n, int a_tmem, int iters, double* cycles_per_mma)
{
    if ((m != 64 && m != 128) || (n != 192 && n != 256) || iters < 1 || iters > 100000 || !cycles_per_mma) return 1;
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return 2;
    unsigned long long* c = nullptr;
    unsigned* st = nullptr;
    if (cudaMalloc(&c, sizeof(unsigned long long)) != cudaSuccess) return 2;
    if (cudaMalloc(&st, sizeof(unsigned)) != cudaSuccess) {
        cudaFree(c);
        return 2;
    }
    // 200 KB of shared memory: one CTA per SM (each allocates all 512 TMEM columns)
    cudaFuncSetAttribute(cycles_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
    cycles_kernel<<<sms, 128, 200 * 1024>>>(m, n, a_tmem ? 1 : 0, iters, 0, 128, 256, 0, c, st);
    unsigned long long cyc = 0;
    unsigned ok = 0;
    int rc = cudaDeviceSynchronize() == cudaSuccess ? 0 : 2;
    if (!rc && cudaMemcpy(&cyc, c, sizeof(cyc), cudaMemcpyDeviceToHost) != cudaSuccess) rc = 2;
    if (!rc && cudaMemcpy(&ok, st, sizeof(unsigned), cudaMemcpyDeviceToHost) != cudaSuccess) rc = 2;
    cudaFree(c);
    cudaFree(st);
    *cycles_per_mma = (double)cyc / (3 * ((iters + 2) / 3));  // the loop issues MMAs three at a time
    return rc ? rc : (ok ? 0 : 3);
}

// B address map of a K-major descriptor with layout type `layout` (0 none, 2
// SW128, 4 SW64, 6 SW32), byte offsets lbo/sbo, start address `start_off`
// bytes after a 1024-byte aligned image and base-offset field `base_off`;
// out_host[k * 256 + n] = index (mod 2048) of the word read for (k, n).
int fcvprobe_umma_b_map_ex(int layout, unsigned lbo, unsigned sbo, unsigned start_off, unsigned base_off,
                           float* out_host)
{
    if ((layout != 0 && layout != 2 && layout != 4 && layout != 6) || lbo > 8192 || sbo > 8192 || (lbo & 15) ||
        (sbo & 15) || start_off > 4096 || (start_off & 15) || base_off > 7 || !out_host)
        return 1;
    // N = 256 rows at most 32 * sbo + one 128-byte row past the start: inside the 48 KB B image
    if (start_off + 32u * sbo + lbo + 128u > (unsigned)(B_WORDS * 4)) return 1;
    float* d = nullptr;
    unsigned* st = nullptr;
    if (cudaMalloc(&d, 8 * 256 * sizeof(float)) != cudaSuccess) return 2;
    if (cudaMalloc(&st, sizeof(unsigned)) != cudaSuccess) {
        cudaFree(d);
        return 2;
    }
    cudaFuncSetAttribute(layout_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES);
    layout_kernel<<<1, 128, SMEM_BYTES>>>(0, 0, lbo, sbo, (uint32_t)layout, start_off, base_off, d, st);
    unsigned ok = 0;
    int rc = cudaDeviceSynchronize() == cudaSuccess ? 0 : 2;
    if (!rc && cudaMemcpy(out_host, d, 8 * 256 * sizeof(float), cudaMemcpyDeviceToHost) != cudaSuccess) rc = 2;
    if (!rc && cudaMemcpy(&ok, st, sizeof(unsigned), cudaMemcpyDeviceToHost) != cudaSuccess) rc = 2;
    cudaFree(d);
    cudaFree(st);
    return rc ? rc : (ok ? 0 : 3);
}

// SM cycles per MMA with a B descriptor of the given layout whose start
// address cycles through 0, shift, 2 * shift bytes.
int fcvprobe_umma_cycles_ex(int m, int n, int a_tmem, int layout, unsigned lbo, unsigned sbo, unsigned shift,
                            int iters, double* cycles_per_mma)
{
    if ((m != 64 && m != 128) || (n != 192 && n != 256) || iters < 3 || iters > 100000 || !cycles_per_mma ||
        (layout != 0 && layout != 2 && layout != 4 && layout != 6) || lbo > 8192 || sbo > 8192 || (lbo & 15) ||
        (sbo & 15) || shift > 1024 || (shift & 15))
        return 1;
    // B image: 200 KB - 16 KB for A; rows reach 2 * shift + (n / 8) * sbo + lbo + 128 bytes
    if (2u * shift + (unsigned)(n / 8) * sbo + lbo + 128u > 184u * 1024u) return 1;
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return 2;
    unsigned long long* c = nullptr;
    unsigned* st = nullptr;
    if (cudaMalloc(&c, sizeof(unsigned long long)) != cudaSuccess) return 2;
    if (cudaMalloc(&st, sizeof(unsigned)) != cudaSuccess) {
        cudaFree(c);
        return 2;
    }
    cudaFuncSetAttribute(cycles_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
    cycles_kernel<<<sms, 128, 200 * 1024>>>(m, n, a_tmem ? 1 : 0, iters, (uint32_t)layout, lbo, sbo, shift, c, st);
    unsigned long long cyc = 0;
    unsigned ok = 0;
    int rc = cudaDeviceSynchronize() == cudaSuccess ? 0 : 2;
    if (!rc && cudaMemcpy(&cyc, c, sizeof(cyc), cudaMemcpyDeviceToHost) != cudaSuccess) rc = 2;
    if (!rc && cudaMemcpy(&ok, st, sizeof(unsigned), cudaMemcpyDeviceToHost) != cudaSuccess) rc = 2;
    cudaFree(c);
    cudaFree(st);
    *cycles_per_mma = (double)cyc / (3 * ((iters + 2) / 3));
    return rc ? rc : (ok ? 0 : 3);
}

}  // extern "C"
