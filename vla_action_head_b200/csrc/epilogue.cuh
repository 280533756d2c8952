// epilogue.cuh — the fused GEMM epilogue, shared by the standalone GEMM and the layer
// executor: v = acc * gA * gW (+ bias[n]) (+ residual[m, n]), then bf16 out, or tanh-GELU /
// GeGLU re-quantized to NVFP4 ("GROOT N1.7 update: Thor NVFP4 + FA4 performance tier",
// §What is in the tier; "Pi0.5 Thor NVFP4 End-to-End Results", §Half-Width Fused GeGLU
// Epilogue and §Fused GeGLU FFN in the Decoder: GELU on the fp32 accumulator, gate/up on
// adjacent columns, 16 values per output scale block).
#pragma once

#include <cuda_bf16.h>

#include <cstdint>

#include "gemm.h"
#include "quant.cuh"

namespace nvfp4 {

__device__ __forceinline__ float gelu_tanh_f(float z) {
    const float k0 = 0.7978845608028654f;  // sqrt(2/pi)
    const float z3 = z * z * z;
    return 0.5f * z * (1.0f + tanhf(k0 * (z + 0.044715f * z3)));
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t *>(&h);
}

// Epilogue of one 32-column chunk held by this thread (row m, columns n .. n + 31).
// Every field of p is read once into a local first: the byte stores of the FP4 outputs may
// alias any memory as far as the compiler knows, and p may live in global memory.
template <class P>
__device__ __forceinline__ void epilogue_chunk(const P &p, int m, int n, float *v) {
    const int epi = p.epi, N = p.N, ldr = p.ldr, ldo = p.ldo;
    const float alpha = p.alpha, g_out = p.g_out;
    const uint16_t *const bias = p.bias;
    const uint16_t *const residual = p.residual;
    uint16_t *const out = p.out;
    uint8_t *const out_codes = p.out_codes;
    uint8_t *const out_sf = p.out_sf;
    const bool has_bias = bias != nullptr &&
                          (epi == kEpiBias || epi == kEpiBiasResidual || epi == kEpiBiasGelu || epi == kEpiGeglu);
    const bool has_res = (epi == kEpiResidual || epi == kEpiBiasResidual);
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __fmul_rn(v[i], alpha);
    if (has_bias) {
        const uint4 *bq = reinterpret_cast<const uint4 *>(bias + n);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const uint4 u = __ldg(bq + j);
            const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
            for (int t = 0; t < 4; ++t) {
                v[8 * j + 2 * t] = __fadd_rn(v[8 * j + 2 * t], bf16lo(w[t]));
                v[8 * j + 2 * t + 1] = __fadd_rn(v[8 * j + 2 * t + 1], bf16hi(w[t]));
            }
        }
    }
    if (has_res) {
        const uint4 *rq = reinterpret_cast<const uint4 *>(residual + static_cast<size_t>(m) * ldr + n);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const uint4 u = __ldcg(rq + j);
            const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
            for (int t = 0; t < 4; ++t) {
                v[8 * j + 2 * t] = __fadd_rn(v[8 * j + 2 * t], bf16lo(w[t]));
                v[8 * j + 2 * t + 1] = __fadd_rn(v[8 * j + 2 * t + 1], bf16hi(w[t]));
            }
        }
    }
    if (epi == kEpiBiasGelu) {
        const float d6g = __fmul_rn(6.0f, g_out);
        const int k_atoms_out = (N + 63) >> 6;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            float y[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) y[i] = gelu_tanh_f(v[16 * h + i]);
            uint2 c;
            const uint32_t s = quantize_block16(y, g_out, d6g, c);
            const int col = n + 16 * h;
            *reinterpret_cast<uint2 *>(out_codes + static_cast<size_t>(m) * (N >> 1) + (col >> 1)) = c;
            out_sf[sf_offset(m, col >> 4, k_atoms_out)] = static_cast<uint8_t>(s);
        }
    } else if (epi == kEpiGeglu) {
        const float d6g = __fmul_rn(6.0f, g_out);
        const int n_out = N >> 1;
        const int k_atoms_out = (n_out + 63) >> 6;
        float y[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) y[j] = __fmul_rn(gelu_tanh_f(v[2 * j]), v[2 * j + 1]);
        uint2 c;
        const uint32_t s = quantize_block16(y, g_out, d6g, c);
        const int col = n >> 1;  // first output column of this block
        *reinterpret_cast<uint2 *>(out_codes + static_cast<size_t>(m) * (n_out >> 1) + (col >> 1)) = c;
        out_sf[sf_offset(m, col >> 4, k_atoms_out)] = static_cast<uint8_t>(s);
    } else {
        uint4 *oq = reinterpret_cast<uint4 *>(out + static_cast<size_t>(m) * ldo + n);
#pragma unroll
        for (int j = 0; j < 4; ++j)
            oq[j] = make_uint4(pack_bf16x2(v[8 * j], v[8 * j + 1]), pack_bf16x2(v[8 * j + 2], v[8 * j + 3]),
                               pack_bf16x2(v[8 * j + 4], v[8 * j + 5]), pack_bf16x2(v[8 * j + 6], v[8 * j + 7]));
    }
}

}  // namespace nvfp4
