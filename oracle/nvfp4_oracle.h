/*
 * nvfp4_oracle.h — plain, single-threaded CPU oracle for the NVFP4 linear layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and bench.py's
 * cpu_baseline / reference arm may load this library.  It shares no code, header,
 * table or helper with the CUDA path in vla_action_head_b200/csrc/.
 *
 * What it computes (sources, cited as "page title, section"):
 *  - E2M1 element codes on the grid {0, .5, 1, 1.5, 2, 3, 4, 6} with a sign bit,
 *    round-to-nearest-even ("Pi0.5 Thor NVFP4 End-to-End Results", §Implemented Path:
 *    native FP4 conversion is round-to-nearest-even).
 *  - One unsigned E4M3 scale per 16 contiguous K elements plus an fp32 per-tensor
 *    global scale ("GROOT N1.7 update: Thor NVFP4 + FA4 performance tier",
 *    §What is in the tier: dynamic per-16-element activation quantization).
 *  - LayerNorm / RMSNorm / AdaLN / AdaRMSNorm front-ends that emit FP4 directly and
 *    are bit-identical to norm-then-quantize (same page, §What is in the tier;
 *    "Pi0.5 ...", §Vectorized SigLIP LayerNorms and §Implemented Path).
 *  - Scale-factor buffers in 128-row x 4-block tile-interleaved atoms, K rounded up to
 *    64-element atoms, padding zero ("Pi0.5 ...", §Encoder Attention QKV NVFP4 +
 *    Scale-Factor Zero-Init).
 *  - Offline weight quantization, optional pairwise gate/up row interleave
 *    ("Pi0.5 ...", §Implemented Path; §Fused GeGLU Epilogue for the P1 Encoder FFN).
 *  - The 16-point Hadamard block rotation and uniform INT4 (E0M3) elements ("Pi0.5 ...",
 *    §Full-INT4 Decoder Activations + Hadamard Rotation; §E0M3 Uniform-INT4 Decoder
 *    Weights), as options of the quantizers and of the FP4-output epilogues.
 *  - Block-scaled GEMM with bias / residual / tanh-GELU->FP4 / GeGLU->FP4 epilogues,
 *    GELU applied to the unrounded accumulator ("GROOT N1.7 ...", §What is in the tier;
 *    "Pi0.5 ...", §Fused GeGLU FFN in the Decoder), evaluated here in fp64.
 *
 * Readings where the pages are silent are listed beside each function in the .c file.
 * Parity status: every function is pinned by tests/test_oracle_*.py (no "parity
 * unpinned" function), except that the FP4-output GEMM epilogues use std tanh and
 * are compared statistically, as the tests state.
 */
#ifndef NVFP4_ORACLE_H
#define NVFP4_ORACLE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum { ORC_NORM_NONE = 0, ORC_NORM_LAYERNORM = 1, ORC_NORM_RMSNORM = 2, ORC_NORM_ADALN = 3,
       ORC_NORM_ADARMS = 4 };
enum { ORC_EPI_NONE = 0, ORC_EPI_BIAS = 1, ORC_EPI_RESIDUAL = 2, ORC_EPI_BIAS_RESIDUAL = 3,
       ORC_EPI_BIAS_GELU = 4, ORC_EPI_GEGLU = 5, ORC_EPI_BIAS_GELU_RHT = 6, ORC_EPI_GEGLU_RHT = 7 };
/* quantizer options: ROTATE = 16-point Hadamard rotation of each block before quantizing;
   E0M3 = uniform INT4 elements (magnitudes 0..7, block scale amax / 7) instead of E2M1 */
enum { ORC_Q_ROTATE = 1, ORC_Q_E0M3 = 2 };

/* element codecs */
float   orc_e2m1_decode(uint8_t code);
uint8_t orc_e2m1_encode(float v);
float   orc_e4m3_decode(uint8_t code);
uint8_t orc_e4m3_encode(float t);
void    orc_e2m1_encode_n(const float *v, size_t n, uint8_t *out);
void    orc_e4m3_encode_n(const float *v, size_t n, uint8_t *out);
void    orc_e4m3_decode_n(const uint8_t *c, size_t n, float *out);

/* scale-factor layout */
size_t orc_sf_bytes(int rows, int K);
size_t orc_sf_offset(int row, int kblk, int K);

/* one 16-element block: codes[8] packed (element 2j low nibble), returns the scale byte */
uint8_t orc_quantize_block16(const float *y, float g, uint8_t *codes8);

/* rows of fp32 y (row stride ldy) -> codes [rows, ceil(K/2)] and scale bytes.
   sf must be zeroed by the caller (padding stays zero). K % 16 != 0 is padded with zeros. */
void orc_quantize_rows(const float *y, int rows, int K, int ldy, float g,
                       uint8_t *codes, uint8_t *sf);

/* per-row norm of bf16 (in_fp32=0) or fp32 (in_fp32=1) x -> fp32 y [rows, K] (dense). */
void orc_norm_rows(const void *x, int in_fp32, int rows, int K, int ldx, int kind,
                   const uint16_t *gamma, const uint16_t *beta, const uint16_t *mod_scale,
                   const uint16_t *mod_shift, float eps, float *y);

/* fp32 -> bf16, round to nearest even (single value and array). */
uint16_t orc_f32_to_bf16(float v);
void orc_f32_to_bf16_array(const float *v, size_t n, uint16_t *out);

/* gated residual update: h = bf16(x + gate * d), fp32 product then fp32 sum; gate NULL = 1. */
void orc_gated_residual(const uint16_t *x, const uint16_t *d, const uint16_t *gate, int rows, int K,
                        uint16_t *h);

/* fused: norm then quantize, written as the two steps. */
void orc_quantize_norm(const void *x, int in_fp32, int rows, int K, int ldx, int kind,
                       const uint16_t *gamma, const uint16_t *beta, const uint16_t *mod_scale,
                       const uint16_t *mod_shift, float eps, float g,
                       uint8_t *codes, uint8_t *sf);

/* offline weight quantizer; returns the global scale. */
float orc_quantize_weight(const uint16_t *w, int N, int K, int ldw, int interleave_gate_up,
                          uint8_t *codes, uint8_t *sf);

/* MSE-searched block scales (weights): E(s) of one block with scale byte s (codes8 may be
 * NULL), the block quantizer that keeps the byte of least E, and the weight quantizer. */
double orc_block_sse(const float *y, float g, uint8_t s, uint8_t *codes8);
uint8_t orc_quantize_block16_mse(const float *y, float g, uint8_t *codes8);
float orc_quantize_weight_mse(const uint16_t *w, int N, int K, int ldw, int interleave_gate_up,
                              uint8_t *codes, uint8_t *sf);

/* 16-point Hadamard rotation (in place, fp32 butterfly), E0M3 codec and block quantizer,
 * and the quantizers / dequantizer under the options above. */
void    orc_hadamard16(float *y);
float   orc_e0m3_decode(uint8_t code);
uint8_t orc_e0m3_encode(float v);
uint8_t orc_quantize_block16_e0m3(const float *y, float g, uint8_t *codes8);
uint8_t orc_quantize_block16_ex(const float *y, float g, int flags, uint8_t *codes8);
void orc_quantize_rows_ex(const float *y, int rows, int K, int ldy, float g, int flags,
                          uint8_t *codes, uint8_t *sf);
void orc_quantize_norm_ex(const void *x, int in_fp32, int rows, int K, int ldx, int kind,
                          const uint16_t *gamma, const uint16_t *beta, const uint16_t *mod_scale,
                          const uint16_t *mod_shift, float eps, float g, int flags,
                          uint8_t *codes, uint8_t *sf);
float orc_quantize_weight_ex(const uint16_t *w, int N, int K, int ldw, int interleave_gate_up, int flags,
                             int mse, uint8_t *codes, uint8_t *sf);
void orc_dequantize_ex(const uint8_t *codes, const uint8_t *sf, float g, int rows, int K, int flags,
                       double *out);

/* dequantize rows -> fp64 [rows, K] */
void orc_dequantize(const uint8_t *codes, const uint8_t *sf, float g, int rows, int K,
                    double *out);

/* GEMM + epilogue, rows listed in m_idx (n_rows of them; NULL = all M rows in order).
   v_out [n_rows, N] receives acc*gA*gW + bias + residual in fp64 (before GELU/GeGLU).
   For BIAS_GELU / GEGLU, h_out [n_rows, N_out] receives the fp64 activation and, when
   out_codes / out_sf are non-NULL, its FP4 quantization with g_out is written at the
   listed rows' positions (out_sf zeroed by the caller; sized for M rows, K = N_out). */
void orc_gemm(const uint8_t *a_codes, const uint8_t *a_sf, float gA, int M,
              const uint8_t *w_codes, const uint8_t *w_sf, float gW, int N, int K,
              int epi, const uint16_t *bias, const uint16_t *residual, int ldr,
              const int *m_idx, int n_rows, double *v_out, double *h_out,
              float g_out, uint8_t *out_codes, uint8_t *out_sf);

double orc_gelu_tanh(double z);

#ifdef __cplusplus
}
#endif
#endif
