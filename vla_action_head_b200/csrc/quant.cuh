// quant.cuh — the per-16 NVFP4 block quantizer and the scale-factor layout, as device
// functions shared by the norm front-end, the weight quantizer and the GEMM epilogues.
//
// Block quantizer ("GROOT N1.7 update: Thor NVFP4 + FA4 performance tier", §What is in the
// tier: one UE4M3 scale per 16 elements computed at run time; "Pi0.5 Thor NVFP4 End-to-End
// Results", §Implemented Path: native E2M1 conversion, round-to-nearest-even):
//   a = max|y|;  t = a / (6 g);  s = E4M3_rn_satfinite(t);  S = dec(s) g
//   dec(s) == 0 -> all codes +0;  else  code_i = E2M1_rn_satfinite(y_i * (1 / S))
// Every step is one fp32 operation rounded to nearest even (explicit _rn intrinsics, so
// the compiler cannot contract or reassociate them).
#pragma once

#include <cstdint>

#include "sm100.cuh"

namespace nvfp4 {

// Scale-factor byte offset: 512-byte atoms of 128 rows x 4 blocks (K rounded up to 64
// elements), atoms ordered K fastest then 128-row group; inside an atom row r, block c at
// (r % 32) * 16 + ((r % 128) / 32) * 4 + c % 4 ("Pi0.5 ...", §Encoder Attention QKV NVFP4 +
// Scale-Factor Zero-Init: tile-interleaved layouts round K up to 64-element atoms).
__host__ __device__ __forceinline__ size_t sf_offset(int row, int kblk, int k_atoms) {
    const size_t atom = static_cast<size_t>(row >> 7) * k_atoms + (kblk >> 2);
    return atom * 512 + ((row & 31) << 4) + (((row >> 5) & 3) << 2) + (kblk & 3);
}

// Quantizes y[0..15]; d6g = 6 * g (fp32).  Writes 8 code bytes (element 0 in the low
// nibble of byte 0) and returns the scale byte.
__device__ __forceinline__ uint32_t quantize_block16(const float *y, float g, float d6g,
                                                     uint2 &codes) {
    float m8[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) m8[i] = fmaxf(fabsf(y[i]), fabsf(y[i + 8]));
#pragma unroll
    for (int w = 4; w > 0; w >>= 1)
#pragma unroll
        for (int i = 0; i < w; ++i) m8[i] = fmaxf(m8[i], m8[i + w]);
    const float a = fmaxf(0.0f, m8[0]);  // NaN inputs are ignored, as fmaxf does
    const float t = __fdiv_rn(a, d6g);
    const uint32_t s = cvt_e4m3_rn_satfinite(t);
    const float ds = e4m3_to_f32(s);
    if (ds == 0.0f) {
        codes = make_uint2(0u, 0u);
        return s;
    }
    const float S = __fmul_rn(ds, g);
    const float r = __frcp_rn(S);
    float v[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __fmul_rn(y[i], r);
    codes.x = cvt_e2m1x8(v);
    codes.y = cvt_e2m1x8(v + 8);
    return s;
}

// Quantizer options (the norm front-end, the weight quantizers and the FP4 epilogues):
//   kQuantRotate  each 16-element block is rotated by the orthonormal 16 x 16 Hadamard
//                 matrix before it is quantized ("Pi0.5 Thor NVFP4 End-to-End Results",
//                 §Full-INT4 Decoder Activations + Hadamard Rotation: both GEMM operands'
//                 blocks rotated, which leaves the GEMM unchanged);
//   kQuantE0M3    uniform INT4 elements (sign-magnitude, magnitudes 0..7) with amax / 7
//                 block scales instead of E2M1 with amax / 6 (same page, §E0M3 Uniform-INT4
//                 Decoder Weights).
enum : int { kQuantRotate = 1, kQuantE0M3 = 2 };

// Sylvester-ordered 16-point Hadamard rotation of one block in registers (the in-register
// fast Walsh-Hadamard transform): stages d = 1, 2, 4, 8 pair element i with i ^ d, the
// element with bit d clear taking a + b and the other a - b (a the lower-index value), each
// one fp32 add rounded to nearest even; then every element times 1/4 (H16 / 4 is
// orthonormal and its own inverse).
__device__ __forceinline__ void fwht16(float *y) {
#pragma unroll
    for (int d = 1; d < 16; d <<= 1)
#pragma unroll
        for (int i = 0; i < 16; ++i)
            if ((i & d) == 0) {
                const float a = y[i], b = y[i | d];
                y[i] = __fadd_rn(a, b);
                y[i | d] = __fsub_rn(a, b);
            }
#pragma unroll
    for (int i = 0; i < 16; ++i) y[i] = __fmul_rn(y[i], 0.25f);
}

// E0M3 element code of v: |v| rounded to the nearest integer, ties to even, saturated at 7;
// bit 3 = the sign bit of v (kept for values that round to 0, as the E2M1 conversion does).
__device__ __forceinline__ uint32_t e0m3_code(float v) {
    const uint32_t q = static_cast<uint32_t>(__float2int_rn(fminf(fabsf(v), 7.0f)));
    return q | ((__float_as_uint(v) >> 28) & 8u);
}

// The E0M3 block: the steps of quantize_block16 with 7 in place of 6 (d7g = 7 * g).
__device__ __forceinline__ uint32_t quantize_block16_e0m3(const float *y, float g, float d7g, uint2 &codes) {
    float a = 0.0f;
#pragma unroll
    for (int i = 0; i < 16; ++i) a = fmaxf(a, fabsf(y[i]));
    const float t = __fdiv_rn(a, d7g);
    const uint32_t s = cvt_e4m3_rn_satfinite(t);
    const float ds = e4m3_to_f32(s);
    if (ds == 0.0f) {
        codes = make_uint2(0u, 0u);
        return s;
    }
    const float r = __frcp_rn(__fmul_rn(ds, g));
    uint32_t w[2] = {0u, 0u};
#pragma unroll
    for (int i = 0; i < 16; ++i) w[i >> 3] |= e0m3_code(__fmul_rn(y[i], r)) << (4 * (i & 7));
    codes = make_uint2(w[0], w[1]);
    return s;
}

// The block quantizer under the options: y (modified in place when rotating) -> codes and
// the returned scale byte; dqg = (6 or 7) * g for the E2M1 or E0M3 grid.
__device__ __forceinline__ uint32_t quantize_block16_opt(float *y, float g, float dqg, int qflags, uint2 &codes) {
    if (qflags & kQuantRotate) fwht16(y);
    return (qflags & kQuantE0M3) ? quantize_block16_e0m3(y, g, dqg, codes) : quantize_block16(y, g, dqg, codes);
}
// Top grid magnitude of the elements (6 for E2M1, 7 for E0M3).
__device__ __forceinline__ float quant_qmax(int qflags) { return (qflags & kQuantE0M3) ? 7.0f : 6.0f; }

__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }
// Two fp32 -> bf16 (round to nearest even), lo in the low half.
__device__ __forceinline__ uint32_t pack_bf16x2_rn(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

}  // namespace nvfp4
