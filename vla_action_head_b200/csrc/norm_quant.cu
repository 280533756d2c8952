// norm_quant.cu — launchers of the norm -> NVFP4 front-end (the per-row code is in
// norm_row.cuh) and the offline weight quantizer.
#include <cuda_runtime.h>

#include "gemm.h"
#include "norm.h"
#include "norm_row.cuh"
#include "quant.cuh"
#include "sm100.cuh"

namespace nvfp4 {

// TPR threads per row, BPT blocks of 16 per thread, F32: fp32 input (else bf16).
template <int TPR, int BPT, bool F32>
__global__ void __launch_bounds__(128) norm_quant_kernel(const NormArgs p) {
    constexpr int kRowsPerCta = 128 / TPR;
    __shared__ double red[4];
    // Let the next kernel launch now (it prefetches its weights), then wait for our input,
    // which may be the previous kernel's output (programmatic dependent launch).
    pdl_launch_dependents();
    pdl_wait();
    norm_row<TPR, BPT, F32>(p, blockIdx.x * kRowsPerCta + threadIdx.x / TPR, threadIdx.x % TPR, red);
}

// Weight amax: max |w| over N x K bf16, folded into *amax_bits with an atomic max on the
// fp32 bit pattern (monotonic for non-negative floats).
__global__ void __launch_bounds__(256) weight_amax_kernel(const uint16_t *w, int N, int K, int ldw,
                                                          uint32_t *amax_bits) {
    const int kv = K >> 3;  // 16-byte vectors per row
    const size_t total = static_cast<size_t>(N) * kv;
    float a = 0.0f;
    for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < total;
         i += static_cast<size_t>(gridDim.x) * blockDim.x) {
        const size_t r = i / kv, c = i % kv;
        const uint4 u = __ldg(reinterpret_cast<const uint4 *>(w + r * ldw) + c);
        const uint32_t ws[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) a = fmaxf(a, fmaxf(fabsf(bf16lo(ws[j])), fabsf(bf16hi(ws[j]))));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
    __shared__ float red[8];
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = a;
    __syncthreads();
    if (threadIdx.x == 0) {
        for (int i = 1; i < 8; ++i) a = fmaxf(a, red[i]);
        atomicMax(amax_bits, __float_as_uint(a));
    }
}

// ---- launchers (host) ---------------------------------------------------------------------
template <int TPR, bool F32>
static cudaError_t launch_tpr(const NormArgs &a, int bpt, cudaStream_t s) {
    const dim3 grid((a.M + (128 / TPR) - 1) / (128 / TPR));
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(128);
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl_enabled() ? 1 : 0;
    switch (bpt) {
#define NVFP4_CASE(B) \
    case B: return cudaLaunchKernelEx(&cfg, norm_quant_kernel<TPR, B, F32>, a);
        NVFP4_CASE(1) NVFP4_CASE(2) NVFP4_CASE(3) NVFP4_CASE(4)
        NVFP4_CASE(5) NVFP4_CASE(6) NVFP4_CASE(7) NVFP4_CASE(8)
#undef NVFP4_CASE
    default:
        if constexpr (!F32) {
            if (bpt <= 12) return cudaLaunchKernelEx(&cfg, norm_quant_kernel<TPR, 12, F32>, a);
            if (bpt <= 16) return cudaLaunchKernelEx(&cfg, norm_quant_kernel<TPR, 16, F32>, a);
        }
        return cudaErrorInvalidValue;
    }
}

// Host entry used by the C ABI.  K % 16 == 0 and the size limits are checked by the caller.
// Few rows (up to about one per SM): a CTA per row, so each row's reductions are spread
// over 128 threads and the per-row latency is short.  Many rows: a warp per row.
cudaError_t launch_norm_quant(const NormArgs &a, bool f32_in, cudaStream_t s) {
    const int nblk = a.K >> 4;
    if (a.M <= 160 && nblk <= 128 * 8) {
        const int bpt = (nblk + 127) / 128;
        return f32_in ? launch_tpr<128, true>(a, bpt, s) : launch_tpr<128, false>(a, bpt, s);
    }
    if (nblk <= 32 * 8) {
        const int bpt = (nblk + 31) / 32;
        return f32_in ? launch_tpr<32, true>(a, bpt, s) : launch_tpr<32, false>(a, bpt, s);
    }
    const int bpt = (nblk + 127) / 128;
    return f32_in ? launch_tpr<128, true>(a, bpt, s) : launch_tpr<128, false>(a, bpt, s);
}

cudaError_t probe_norm_kernels() {
    cudaFuncAttributes fa;
    return cudaFuncGetAttributes(&fa, norm_quant_kernel<32, 1, false>);
}

cudaError_t launch_weight_amax(const uint16_t *w, int N, int K, int ldw, uint32_t *amax_bits,
                               cudaStream_t s) {
    cudaError_t e = cudaMemsetAsync(amax_bits, 0, sizeof(uint32_t), s);
    if (e != cudaSuccess) return e;
    const size_t vecs = static_cast<size_t>(N) * (K >> 3);
    size_t blocks = (vecs + 255) / 256;
    if (blocks > 148 * 8) blocks = 148 * 8;
    if (blocks == 0) blocks = 1;
    weight_amax_kernel<<<static_cast<unsigned>(blocks), 256, 0, s>>>(w, N, K, ldw, amax_bits);
    return cudaGetLastError();
}

}  // namespace nvfp4
