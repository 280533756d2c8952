// mma_rate.cu — diagnostics: the issue rate of the block-scaled MMA on one SM, the ceiling
// that the GEMM kernels' MMA phases are measured against.
//
// One CTA, one issuing thread, operands resident in shared memory (finite E2M1 bytes; unit
// UE4M3 scales), accumulator and scale factors in tensor memory.  Per K step of 256:
//   mode 0   4 x tcgen05.mma kind::mxf4nvf4 block16 (M = 128, N = n, K = 64), scale factors
//            copied into tensor memory once before the timed loop;
//   mode 1   the K step's scale-atom copies (tcgen05.cp .32x128b.warpx4: 4 for A, 4 per
//            128-row group of W) into one of four scale slots, then its 4 MMAs, all from the
//            same thread (the order a single producer of copies and MMAs would see).
// clock64 is read before the first instruction, after the last one is issued, and after a
// tcgen05.commit of all of them has arrived (bounded wait).  The operands hold no meaning;
// only the cycle counts are read.
#include <cuda_runtime.h>

#include "sm100.cuh"

namespace nvfp4 {

namespace {

constexpr int kRateCodes = 16384 + 32768;  // A: 128 rows x 128 B; W: up to 256 rows x 128 B
constexpr int kRateSf = 4 * 512 + 8 * 512;  // A's 4 atoms, W's 4 atoms per 128-row group (<= 2)
constexpr int kRateSmem = kRateCodes + kRateSf + 1024;

__device__ unsigned long long g_rate_out[3];

__device__ __forceinline__ void rate_copy_sf(uint32_t t_sf, uint32_t sf, int groups) {
#pragma unroll 1
    for (int kb = 0; kb < 4; ++kb) {
        tc_cp_32x128b_warpx4(t_sf + 4 * kb, desc_sf_32x128b(sf + kb * 512));
#pragma unroll 1
        for (int g = 0; g < groups; ++g)
            tc_cp_32x128b_warpx4(t_sf + 16 + 4 * (groups * kb + g), desc_sf_32x128b(sf + 2048 + (g * 4 + kb) * 512));
    }
}

__global__ void __launch_bounds__(128, 1) mma_rate_kernel(int n, int mode, int ksteps) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *s = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    __shared__ uint32_t tmem_base;
    __shared__ int abort_flag;
    __shared__ uint32_t wait_status;
    __shared__ __align__(8) uint64_t bar;
    for (int i = threadIdx.x; i < kRateCodes; i += blockDim.x) s[i] = static_cast<uint8_t>((i * 37) & 0x77);
    for (int i = threadIdx.x; i < kRateSf; i += blockDim.x) s[kRateCodes + i] = 0x38;  // UE4M3 1.0
    if (threadIdx.x == 0) {
        abort_flag = 0;
        wait_status = 0;
        mbar_init(smem_u32(&bar), 1);
        fence_mbar_init();
    }
    // the shared-memory operands are read by the tensor cores (async proxy)
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    if ((threadIdx.x >> 5) == 1) {
        tmem_alloc(smem_u32(&tmem_base), 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_base;
    const int groups = n > 128 ? 2 : 1;
    if (threadIdx.x == 0) {
        const uint32_t a = smem_u32(s), b = smem_u32(s + 16384), sf = smem_u32(s + kRateCodes);
        const uint32_t idesc = idesc_mxf4nvf4(128, n);
        // accumulator in columns [0, n); four scale slots of 64 columns from column 256
        if (mode == 0) rate_copy_sf(tmem + 256, sf, groups);
        const unsigned long long t0 = clock64();
#pragma unroll 1
        for (int it = 0; it < ksteps; ++it) {
            const uint32_t t_sf = tmem + 256 + (mode == 0 ? 0u : 64u * static_cast<uint32_t>(it & 3));
            if (mode == 1) rate_copy_sf(t_sf, sf, groups);
#pragma unroll
            for (int kb = 0; kb < 4; ++kb)
                tc_mma_mxf4nvf4(tmem, desc_kmajor_sw128(a + 32 * kb), desc_kmajor_sw128(b + 32 * kb), idesc,
                                t_sf + 4 * kb, t_sf + 16 + 4 * groups * kb, (it > 0 || kb > 0) ? 1u : 0u);
        }
        const unsigned long long t1 = clock64();
        tc_commit(smem_u32(&bar));
        const bool done = mbar_wait(smem_u32(&bar), 0, &abort_flag, &wait_status, kStatusTimeoutAccum);
        const unsigned long long t2 = clock64();
        g_rate_out[0] = t1 - t0;
        g_rate_out[1] = t2 - t0;
        g_rate_out[2] = done ? 0ull : 1ull;
    }
    tc_fence_before();
    __syncthreads();
    if ((threadIdx.x >> 5) == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

}  // namespace

cudaError_t run_mma_rate(int n, int mode, int ksteps, unsigned long long out[3]) {
    cudaError_t e = cudaFuncSetAttribute(mma_rate_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kRateSmem);
    if (e != cudaSuccess) return e;
    mma_rate_kernel<<<1, 128, kRateSmem>>>(n, mode, ksteps);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if ((e = cudaDeviceSynchronize()) != cudaSuccess) return e;
    return cudaMemcpyFromSymbol(out, g_rate_out, 3 * sizeof(unsigned long long));
}

}  // namespace nvfp4
