// norm.h — internal interface between the C ABI (api.cu) and the norm / quantizer kernels.
#pragma once

#include <cuda_runtime.h>

#include <cstdint>

namespace nvfp4 {

struct NormArgs {
    const void *x;
    int M, K, ldx;
    int kind;  // nvfp4_norm
    const uint16_t *gamma, *beta, *scale, *shift;
    float eps;
    float g;                    // global decode scale (activation path)
    const uint32_t *amax_bits;  // weight path: g = amax / (qmax * 448) computed from this word
    int qflags;                 // kQuantRotate | kQuantE0M3 (quant.cuh)
    int interleave;             // weight path: pairwise gate/up row interleave
    uint8_t *codes;
    uint8_t *sf;
    float *y_out;  // non-NULL: write the normalized fp32 y instead of quantizing
    // gated residual front-end (bf16 only): x is replaced by h = bf16(x + gate * d), which
    // is also stored to h_out; res_d == NULL: none
    const uint16_t *res_d;
    int ldd;
    const uint16_t *res_gate;  // NULL: 1
    uint16_t *h_out;
    int ldh;
};

cudaError_t launch_norm_quant(const NormArgs &a, bool f32_in, cudaStream_t s);
// max |w| (rotate: max over the Hadamard-rotated 16-element blocks along K) into *amax_bits.
cudaError_t launch_weight_amax(const uint16_t *w, int N, int K, int ldw, int rotate, uint32_t *amax_bits,
                               cudaStream_t s);
// MSE-searched block scales for an N x K bf16 weight (global scale from *amax_bits); rotate:
// the blocks are Hadamard-rotated first.
cudaError_t launch_weight_mse(const uint16_t *w, int N, int K, int ldw, int interleave, int rotate,
                              const uint32_t *amax_bits, uint8_t *codes, uint8_t *sf, cudaStream_t s);
cudaError_t probe_norm_kernels();
cudaError_t probe_gemm_kernels();

}  // namespace nvfp4
