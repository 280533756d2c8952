// epilogue.cuh — the fused GEMM epilogue, shared by the GEMM kernels (small-M, persistent,
// grouped): v = acc * gA * gW (+ bias[n]) (+ residual[m, n]), then bf16 out, or tanh-GELU /
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

// tanh-form GELU, 0.5 z (1 + tanh(u)) with u = sqrt(2/pi) (z + 0.044715 z^3), evaluated as
// z / (1 + exp(-2u)) since (1 + tanh(u)) / 2 = 1 / (1 + exp(-2u)): one exponential and one
// division (relative error a few fp32 ulp; large negative z gives -0 like the tanh form).
__device__ __forceinline__ float gelu_tanh_f(float z) {
    const float k2 = 1.5957691216057308f;  // 2 sqrt(2/pi)
    const float u2 = k2 * (z + 0.044715f * z * z * z);
    return __fdividef(z, 1.0f + __expf(-u2));
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t *>(&h);
}

// Epilogue of one chunk of W = 16 or 32 columns held by this thread (row m, columns
// n .. n + W - 1; GeGLU needs W = 32: 32 interleaved gate/up columns make one 16-value
// output block).  bw / rw: the bias of columns n.. and the residual of row m, columns n..,
// as W / 2 words of bf16 pairs each (NULL: none), already loaded.
// Every field of p is read once into a local first: the byte stores of the FP4 outputs may
// alias any memory as far as the compiler knows, and p may live in global memory.
// EPI >= 0 fixes the epilogue kind at compile time (only that path is generated).
// p.out_rotate: the FP4 epilogues rotate each 16-value output block by the 16-point
// Hadamard matrix before quantizing it ("Pi0.5 Thor NVFP4 End-to-End Results", §Full-INT4
// Decoder Activations + Hadamard Rotation: the GeGLU exit is one of the rotated exits).
template <int W, int EPI = -1, class P>
__device__ __forceinline__ void epilogue_chunk_w(const P &p, int m, int n, float *v, const uint32_t *bw,
                                                 const uint32_t *rw) {
    static_assert(W == 16 || W == 32, "chunk width");
    const int epi = EPI >= 0 ? EPI : p.epi;
    const int N = p.N, ldo = p.ldo;
    const float alpha = p.alpha, g_out = p.g_out;
    uint16_t *const out = p.out;
    uint8_t *const out_codes = p.out_codes;
    uint8_t *const out_sf = p.out_sf;
    const bool rot = p.out_rotate != 0;
    const bool has_bias = bw != nullptr &&
                          (epi == kEpiBias || epi == kEpiBiasResidual || epi == kEpiBiasGelu || epi == kEpiGeglu);
    const bool has_res = rw != nullptr && (epi == kEpiResidual || epi == kEpiBiasResidual);
#pragma unroll
    for (int i = 0; i < W; ++i) v[i] = __fmul_rn(v[i], alpha);
    if (has_bias) {
#pragma unroll
        for (int t = 0; t < W / 2; ++t) {
            v[2 * t] = __fadd_rn(v[2 * t], bf16lo(bw[t]));
            v[2 * t + 1] = __fadd_rn(v[2 * t + 1], bf16hi(bw[t]));
        }
    }
    if (has_res) {
#pragma unroll
        for (int t = 0; t < W / 2; ++t) {
            v[2 * t] = __fadd_rn(v[2 * t], bf16lo(rw[t]));
            v[2 * t + 1] = __fadd_rn(v[2 * t + 1], bf16hi(rw[t]));
        }
    }
    if (epi == kEpiBiasGelu) {
        const float d6g = __fmul_rn(6.0f, g_out);
        const int k_atoms_out = (N + 63) >> 6;
#pragma unroll
        for (int h = 0; h < W / 16; ++h) {
            float y[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) y[i] = gelu_tanh_f(v[16 * h + i]);
            if (rot) fwht16(y);
            uint2 c;
            const uint32_t s = quantize_block16(y, g_out, d6g, c);
            const int col = n + 16 * h;
            *reinterpret_cast<uint2 *>(out_codes + static_cast<size_t>(m) * (N >> 1) + (col >> 1)) = c;
            out_sf[sf_offset(m, col >> 4, k_atoms_out)] = static_cast<uint8_t>(s);
        }
    } else if (epi == kEpiGeglu) {
        if constexpr (W == 32) {
            const float d6g = __fmul_rn(6.0f, g_out);
            const int n_out = N >> 1;
            const int k_atoms_out = (n_out + 63) >> 6;
            float y[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) y[j] = __fmul_rn(gelu_tanh_f(v[2 * j]), v[2 * j + 1]);
            if (rot) fwht16(y);
            uint2 c;
            const uint32_t s = quantize_block16(y, g_out, d6g, c);
            const int col = n >> 1;  // first output column of this block
            *reinterpret_cast<uint2 *>(out_codes + static_cast<size_t>(m) * (n_out >> 1) + (col >> 1)) = c;
            out_sf[sf_offset(m, col >> 4, k_atoms_out)] = static_cast<uint8_t>(s);
        }
    } else {
        uint4 *oq = reinterpret_cast<uint4 *>(out + static_cast<size_t>(m) * ldo + n);
#pragma unroll
        for (int j = 0; j < W / 8; ++j)
            oq[j] = make_uint4(pack_bf16x2(v[8 * j], v[8 * j + 1]), pack_bf16x2(v[8 * j + 2], v[8 * j + 3]),
                               pack_bf16x2(v[8 * j + 4], v[8 * j + 5]), pack_bf16x2(v[8 * j + 6], v[8 * j + 7]));
    }
}

// Loads W bf16 (W / 2 words) from global or shared memory.
template <int W = 32>
__device__ __forceinline__ void load_bf16(const uint16_t *src, uint32_t *w) {
    const uint4 *q = reinterpret_cast<const uint4 *>(src);
#pragma unroll
    for (int j = 0; j < W / 8; ++j) {
        const uint4 u = q[j];
        w[4 * j] = u.x;
        w[4 * j + 1] = u.y;
        w[4 * j + 2] = u.z;
        w[4 * j + 3] = u.w;
    }
}

// The same, with bias_n / res_mn pointing to the bias of columns n.. and the residual of
// row m, columns n.. (global or shared memory; NULL: none).
template <int W = 32, int EPI = -1, class P>
__device__ __forceinline__ void epilogue_chunk_src(const P &p, int m, int n, float *v, const uint16_t *bias_n,
                                                   const uint16_t *res_mn) {
    uint32_t bw[W / 2], rw[W / 2];
    if (bias_n != nullptr) load_bf16<W>(bias_n, bw);
    if (res_mn != nullptr) load_bf16<W>(res_mn, rw);
    epilogue_chunk_w<W, EPI>(p, m, n, v, bias_n != nullptr ? bw : nullptr, res_mn != nullptr ? rw : nullptr);
}

// The same, reading bias and residual from the arguments' global pointers.
template <int W = 32, int EPI = -1, class P>
__device__ __forceinline__ void epilogue_chunk(const P &p, int m, int n, float *v) {
    const int epi = EPI >= 0 ? EPI : p.epi;
    const uint16_t *const bias =
        (epi == kEpiBias || epi == kEpiBiasResidual || epi == kEpiBiasGelu || epi == kEpiGeglu) ? p.bias : nullptr;
    const uint16_t *const residual = (epi == kEpiResidual || epi == kEpiBiasResidual) ? p.residual : nullptr;
    epilogue_chunk_src<W, EPI>(p, m, n, v, bias != nullptr ? bias + n : nullptr,
                       residual != nullptr ? residual + static_cast<size_t>(m) * p.ldr + n : nullptr);
}

}  // namespace nvfp4
