/*
 * nvfp4_oracle.c — plain, single-threaded CPU oracle for the NVFP4 linear layer.
 *
 * TEST INFRASTRUCTURE ONLY: loaded by tests/, __graft_entry__.smoke() and bench.py's
 * CPU baseline.  No product code path may call it.  It shares nothing with the CUDA
 * sources.  Build: gcc -O2 -std=c11 -ffp-contract=off -fno-fast-math (see build_oracle.py);
 * every fp32 operation below is one IEEE-754 binary32 operation rounded to nearest even
 * (x86-64 SSE arithmetic, no contraction into fused multiply-add).
 *
 * Sources are cited as "page title, section".  Where the pages leave a step open the
 * reading taken is stated as READING in the comment beside it.
 */
#include "nvfp4_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------------------ */
/* bf16 -> fp32 widening is exact: the bf16 bits are the top half of the fp32 bits.     */
static float bf16_to_f32(uint16_t h) {
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* ------------------------------------------------------------------------------------ */
/* E2M1: 1 sign bit, 2 exponent bits, 1 mantissa bit; magnitudes 0, .5, 1, 1.5, 2, 3, 4, 6
 * (the NVFP4 element grid).  Code bit 3 is the sign.                                      */
static const double kE2M1Mag[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};

float orc_e2m1_decode(uint8_t code) {
    double m = kE2M1Mag[code & 7u];
    return (float)((code & 8u) ? -m : m);
}

/* Round to nearest on the E2M1 grid, ties to the code with an even mantissa bit
 * ("Pi0.5 Thor NVFP4 End-to-End Results", §Implemented Path: native FP4 conversion is
 * round-to-nearest-even).  Magnitudes above 6 saturate to 6 (satfinite).
 * READING: the sign of the input is kept, so values that round to zero give +0 (0x0) or
 * -0 (0x8) by their sign, as an IEEE-style conversion does.  Inputs are finite.        */
uint8_t orc_e2m1_encode(float v) {
    uint8_t sign = signbit(v) ? 8u : 0u;
    double a = fabs((double)v);
    if (a >= 6.0) return (uint8_t)(sign | 7u); /* satfinite: everything from 6 up is 6 */
    int best = 0;
    double best_d = a; /* distance to magnitude 0 */
    for (int c = 1; c < 8; ++c) {
        double d = fabs(a - kE2M1Mag[c]);
        if (d < best_d || (d == best_d && (c & 1) == 0 && (best & 1) != 0)) {
            best = c;
            best_d = d;
        }
    }
    return (uint8_t)(sign | (uint8_t)best);
}

/* ------------------------------------------------------------------------------------ */
/* E4M3 (bias 7): normal (1 + m/8) * 2^(e-7) for e = 1..15, except e = 15, m = 7 which is
 * NaN; subnormal m * 2^-9; max finite 448 (0x7E).  The block scale is the unsigned form
 * (sign bit 0) ("Pi0.5 ...", §Encoder Attention QKV NVFP4 + Scale-Factor Zero-Init: the
 * bytes 0x7F/0xFF decode as NaN).                                                       */
float orc_e4m3_decode(uint8_t code) {
    int s = code >> 7, e = (code >> 3) & 15, m = code & 7;
    double mag;
    if (e == 15 && m == 7) return NAN;
    if (e == 0) mag = ldexp((double)m, -9);
    else mag = ldexp(1.0 + m / 8.0, e - 7);
    return (float)(s ? -mag : mag);
}

/* Round to nearest E4M3 value, ties to the even code, magnitudes above 448 saturate to
 * 448 (satfinite).  Finite codes 0x00..0x7E are strictly increasing in value, so the
 * two candidates are found by bisection.  Sign kept (the block scale is never negative). */
uint8_t orc_e4m3_encode(float t) {
    uint8_t sign = signbit(t) ? 0x80u : 0u;
    double a = fabs((double)t);
    if (isnan(t)) return (uint8_t)(sign | 0x7Fu);
    if (a >= 448.0) return (uint8_t)(sign | 0x7Eu);
    int lo = 0, hi = 0x7E; /* invariant: dec(lo) <= a < dec(hi) */
    while (hi - lo > 1) {
        int mid = (lo + hi) / 2;
        if ((double)orc_e4m3_decode((uint8_t)mid) <= a) lo = mid;
        else hi = mid;
    }
    double dl = a - (double)orc_e4m3_decode((uint8_t)lo);
    double dh = (double)orc_e4m3_decode((uint8_t)hi) - a;
    int c = (dl < dh) ? lo : (dh < dl) ? hi : ((lo & 1) == 0 ? lo : hi);
    return (uint8_t)(sign | (uint8_t)c);
}

/* Array forms of the codecs (one call per array instead of per element). */
void orc_e2m1_encode_n(const float *v, size_t n, uint8_t *out) {
    for (size_t i = 0; i < n; ++i) out[i] = orc_e2m1_encode(v[i]);
}
void orc_e4m3_encode_n(const float *v, size_t n, uint8_t *out) {
    for (size_t i = 0; i < n; ++i) out[i] = orc_e4m3_encode(v[i]);
}
void orc_e4m3_decode_n(const uint8_t *c, size_t n, float *out) {
    for (size_t i = 0; i < n; ++i) out[i] = orc_e4m3_decode(c[i]);
}

/* ------------------------------------------------------------------------------------ */
/* Scale-factor layout ("Pi0.5 ...", §Encoder Attention QKV NVFP4 + Scale-Factor
 * Zero-Init: tile-interleaved SFA/SFB layouts round K up to 64-element atoms; padding
 * entries must be zero).
 * READING: the tile atom is 128 rows x 4 scale blocks = 512 bytes; inside it, row r and
 * block c sit at (r % 32) * 16 + ((r % 128) / 32) * 4 + c % 4; atoms are ordered with the
 * K-atom index fastest, then the 128-row group.  Rows are padded to 128.                */
size_t orc_sf_bytes(int rows, int K) {
    size_t row_groups = ((size_t)rows + 127) / 128;
    size_t k_atoms = ((size_t)K + 63) / 64;
    return row_groups * k_atoms * 512;
}

size_t orc_sf_offset(int row, int kblk, int K) {
    size_t k_atoms = ((size_t)K + 63) / 64;
    size_t atom = (size_t)(row / 128) * k_atoms + (size_t)(kblk / 4);
    return atom * 512 + (size_t)(row % 32) * 16 + (size_t)((row % 128) / 32) * 4 + (size_t)(kblk % 4);
}

/* ------------------------------------------------------------------------------------ */
/* One block of 16 values ("GROOT N1.7 ...", §What is in the tier: one UE4M3 scale per
 * 16 elements, computed at run time; E2M1 codes; fp32 per-tensor global scale g).
 *   a = max|y|;  d = 6*g;  t = a/d;  s = E4M3(t);  S = dec(s)*g
 *   dec(s) == 0  -> every code is +0 and the scale byte is 0
 *   otherwise    r = 1/S;  code_i = E2M1(y_i * r)
 * READING: a/(6g) is one IEEE division, y*(1/S) one reciprocal then one multiply, every
 * step rounded to fp32 nearest-even (the pages fix no order; this one is reproducible).
 * Codes are packed two per byte, element 2j in the low nibble.                          */
uint8_t orc_quantize_block16(const float *y, float g, uint8_t *codes8) {
    float a = 0.0f;
    for (int i = 0; i < 16; ++i) {
        float m = fabsf(y[i]);
        if (m > a) a = m;
    }
    float d = 6.0f * g;
    float t = a / d;
    uint8_t s = orc_e4m3_encode(t);
    float ds = orc_e4m3_decode(s);
    if (ds == 0.0f) {
        memset(codes8, 0, 8);
        return s;
    }
    float S = ds * g;
    float r = 1.0f / S;
    for (int j = 0; j < 8; ++j) {
        float v0 = y[2 * j] * r;
        float v1 = y[2 * j + 1] * r;
        codes8[j] = (uint8_t)(orc_e2m1_encode(v0) | (orc_e2m1_encode(v1) << 4));
    }
    return s;
}

void orc_quantize_rows(const float *y, int rows, int K, int ldy, float g,
                       uint8_t *codes, uint8_t *sf) {
    int nblk = (K + 15) / 16;
    size_t row_bytes = (size_t)nblk * 8;
    float blk[16];
    for (int r = 0; r < rows; ++r) {
        for (int b = 0; b < nblk; ++b) {
            for (int i = 0; i < 16; ++i) {
                int k = b * 16 + i;
                blk[i] = (k < K) ? y[(size_t)r * ldy + k] : 0.0f;
            }
            uint8_t s = orc_quantize_block16(blk, g, codes + (size_t)r * row_bytes + (size_t)b * 8);
            sf[orc_sf_offset(r, b, K)] = s;
        }
    }
}

/* ------------------------------------------------------------------------------------ */
/* Norm front-ends, one row at a time ("GROOT N1.7 ...", §What is in the tier: AdaLN and
 * the pre-FFN LayerNorm emit FP4 directly; "Pi0.5 ...", §Implemented Path: AdaRMSNorm
 * before QKV and Gate+Up; §Vectorized SigLIP LayerNorms: LayerNorm to NVFP4).
 *   LayerNorm : n = (x - mu) * rstd;          y = n * gamma + beta
 *   RMSNorm   : y = (x * rstd_rms) * gamma
 *   AdaLN     : y = n * (1 + scale) + shift
 *   AdaRMSNorm: y = (x * rstd_rms) * (1 + scale) [+ shift]
 * READING: row statistics are accumulated in fp64 in index order (mean, then the
 * population variance about it; mean of squares for RMS), rounded once to fp32:
 * mu_f = (float)mu, rstd_f = (float)(1 / sqrt(var + eps)).  The elementwise steps are
 * fp32 operations in the order written, (1 + scale) formed first.  A NULL gamma reads
 * as 1, a NULL beta / scale / shift as 0.                                               */
static float ld_x(const void *x, int in_fp32, size_t i) {
    return in_fp32 ? ((const float *)x)[i] : bf16_to_f32(((const uint16_t *)x)[i]);
}

void orc_norm_rows(const void *x, int in_fp32, int rows, int K, int ldx, int kind,
                   const uint16_t *gamma, const uint16_t *beta, const uint16_t *mod_scale,
                   const uint16_t *mod_shift, float eps, float *y) {
    for (int r = 0; r < rows; ++r) {
        size_t base = (size_t)r * ldx;
        float *yr = y + (size_t)r * K;
        if (kind == ORC_NORM_NONE) {
            for (int k = 0; k < K; ++k) yr[k] = ld_x(x, in_fp32, base + k);
            continue;
        }
        float mu_f = 0.0f, rstd_f;
        if (kind == ORC_NORM_LAYERNORM || kind == ORC_NORM_ADALN) {
            double s = 0.0;
            for (int k = 0; k < K; ++k) s += (double)ld_x(x, in_fp32, base + k);
            double mu = s / K;
            double q = 0.0;
            for (int k = 0; k < K; ++k) {
                double dv = (double)ld_x(x, in_fp32, base + k) - mu;
                q += dv * dv;
            }
            double var = q / K;
            mu_f = (float)mu;
            rstd_f = (float)(1.0 / sqrt(var + (double)eps));
        } else {
            double q = 0.0;
            for (int k = 0; k < K; ++k) {
                double xv = (double)ld_x(x, in_fp32, base + k);
                q += xv * xv;
            }
            rstd_f = (float)(1.0 / sqrt(q / K + (double)eps));
        }
        for (int k = 0; k < K; ++k) {
            float xv = ld_x(x, in_fp32, base + k);
            float ga = gamma ? bf16_to_f32(gamma[k]) : 1.0f;
            float be = beta ? bf16_to_f32(beta[k]) : 0.0f;
            float sc = mod_scale ? bf16_to_f32(mod_scale[k]) : 0.0f;
            float sh = mod_shift ? bf16_to_f32(mod_shift[k]) : 0.0f;
            float out;
            switch (kind) {
            case ORC_NORM_LAYERNORM: {
                float n = (xv - mu_f) * rstd_f;
                float t = n * ga;
                out = t + be;
                break;
            }
            case ORC_NORM_ADALN: {
                float n = (xv - mu_f) * rstd_f;
                float opl = 1.0f + sc;
                float t = n * opl;
                out = t + sh;
                break;
            }
            case ORC_NORM_RMSNORM: {
                float n = xv * rstd_f;
                out = n * ga;
                break;
            }
            default: { /* ORC_NORM_ADARMS */
                float n = xv * rstd_f;
                float opl = 1.0f + sc;
                float t = n * opl;
                out = mod_shift ? t + sh : t;
                break;
            }
            }
            yr[k] = out;
        }
    }
}

/* fp32 -> bf16, round to nearest even at bit 16 (IEEE 754 roundTiesToEven applied to the
 * 8-bit significand of bfloat16); overflow goes to infinity; NaN stays a quiet NaN.       */
uint16_t orc_f32_to_bf16(float v) {
    uint32_t u;
    memcpy(&u, &v, 4);
    if ((u & 0x7FFFFFFFu) > 0x7F800000u) return (uint16_t)((u >> 16) | 0x0040u); /* NaN */
    uint32_t lsb = (u >> 16) & 1u;
    u += 0x7FFFu + lsb;
    return (uint16_t)(u >> 16);
}

void orc_f32_to_bf16_array(const float *v, size_t n, uint16_t *out) {
    for (size_t i = 0; i < n; ++i) out[i] = orc_f32_to_bf16(v[i]);
}

/* Gated residual update in front of a norm ("Pi0.5 Thor NVFP4 End-to-End Results",
 * §Implemented Path: gated residual update + Pi0.5 AdaRMSNorm + gate output + NVFP4/SFA in
 * one launch before Gate+Up and the next layer's QKV):
 *   h[r, k] = x[r, k] + gate[k] * d[r, k]
 * x is the residual stream, d the sublayer's output, gate the layer's modulation gate.
 * READING: one fp32 product, then one fp32 sum (no fused multiply-add), rounded once to
 * bf16 (the residual stream is bf16).  The norm that follows reads that bf16 h, so the
 * fused launch is the two-step chain "update, then norm -> FP4".  A NULL gate reads as 1.  */
void orc_gated_residual(const uint16_t *x, const uint16_t *d, const uint16_t *gate, int rows, int K,
                        uint16_t *h) {
    for (int r = 0; r < rows; ++r) {
        for (int k = 0; k < K; ++k) {
            size_t i = (size_t)r * K + k;
            float g = gate ? bf16_to_f32(gate[k]) : 1.0f;
            float t = g * bf16_to_f32(d[i]);
            float s = bf16_to_f32(x[i]) + t;
            h[i] = orc_f32_to_bf16(s);
        }
    }
}

/* Fused norm -> FP4 is, by the pages' contract, identical to the two-step chain
 * ("GROOT N1.7 ...", §What is in the tier: bit-identical to the two-step chain).
 * READING: the intermediate y is not rounded to bf16/fp16 between the steps.           */
void orc_quantize_norm(const void *x, int in_fp32, int rows, int K, int ldx, int kind,
                       const uint16_t *gamma, const uint16_t *beta, const uint16_t *mod_scale,
                       const uint16_t *mod_shift, float eps, float g,
                       uint8_t *codes, uint8_t *sf) {
    float *y = (float *)malloc(sizeof(float) * (size_t)K);
    size_t esz = in_fp32 ? 4 : 2;
    int nblk = (K + 15) / 16;
    for (int r = 0; r < rows; ++r) {
        const char *xr = (const char *)x + (size_t)r * ldx * esz;
        orc_norm_rows(xr, in_fp32, 1, K, ldx, kind, gamma, beta, mod_scale, mod_shift, eps, y);
        /* quantize this row as row r of the output */
        float blk[16];
        for (int b = 0; b < nblk; ++b) {
            for (int i = 0; i < 16; ++i) {
                int k = b * 16 + i;
                blk[i] = (k < K) ? y[k] : 0.0f;
            }
            uint8_t s = orc_quantize_block16(blk, g, codes + (size_t)r * nblk * 8 + (size_t)b * 8);
            sf[orc_sf_offset(r, b, K)] = s;
        }
    }
    free(y);
}

/* ------------------------------------------------------------------------------------ */
/* Offline weight quantization ("Pi0.5 ...", §Implemented Path: weights are quantized
 * once to NVFP4 E2M1 plus block scales).  Blocks run along K, as for activations.
 * READING: the per-tensor global scale is amax(|W|) / (6 * 448) so that the largest
 * block scale lands on the E4M3 maximum; an all-zero tensor takes g = 1.
 * Optional pairwise interleave ("Pi0.5 ...", §Fused GeGLU Epilogue for the P1 Encoder
 * FFN: gate and up rows pairwise interleaved along N): rows [0, N/2) are gate, rows
 * [N/2, N) are up; packed row 2j = gate row j, packed row 2j+1 = up row j.             */
float orc_quantize_weight(const uint16_t *w, int N, int K, int ldw, int interleave_gate_up,
                          uint8_t *codes, uint8_t *sf) {
    float amax = 0.0f;
    for (int n = 0; n < N; ++n)
        for (int k = 0; k < K; ++k) {
            float m = fabsf(bf16_to_f32(w[(size_t)n * ldw + k]));
            if (m > amax) amax = m;
        }
    float g = (amax == 0.0f) ? 1.0f : amax / 2688.0f;
    float *y = (float *)malloc(sizeof(float) * (size_t)K);
    int nblk = (K + 15) / 16;
    for (int r = 0; r < N; ++r) {
        int src = r;
        if (interleave_gate_up) src = (r % 2 == 0) ? r / 2 : N / 2 + r / 2;
        for (int k = 0; k < K; ++k) y[k] = bf16_to_f32(w[(size_t)src * ldw + k]);
        float blk[16];
        for (int b = 0; b < nblk; ++b) {
            for (int i = 0; i < 16; ++i) {
                int k = b * 16 + i;
                blk[i] = (k < K) ? y[k] : 0.0f;
            }
            uint8_t s = orc_quantize_block16(blk, g, codes + (size_t)r * nblk * 8 + (size_t)b * 8);
            sf[orc_sf_offset(r, b, K)] = s;
        }
    }
    free(y);
    return g;
}

/* ------------------------------------------------------------------------------------ */
/* MSE-searched block scales for weights ("Pi0.5 Thor NVFP4 End-to-End Results",
 * §E0M3 Uniform-INT4 Decoder Weights: the default decoder weights are NVFP4 "(MSE)";
 * §Fused GeGLU FFN in the Decoder: the gate/up weight is MSE-quantized like the other
 * decoder projections).  The pages name the criterion, not the search.
 * READING: per 16-element block every UE4M3 scale byte s = 0x00 .. 0x7E is a candidate.
 * The codes for s are those the amax quantizer writes once its scale is s: q_i =
 * E2M1_RNE(y_i * (1 / (dec(s) * g))) in fp32, all +0 when dec(s) = 0.  The block error
 *   E(s) = sum_i (y_i - val(q_i) * dec(s) * g)^2
 * is formed in fp64 (the product is exact; one rounded difference and one rounded
 * square-add per term, terms in index order).  The byte with the smallest E is kept, the
 * smaller byte on ties (so a zero block keeps s = 0).  g stays amax(|W|) / 2688.          */
double orc_block_sse(const float *y, float g, uint8_t s, uint8_t *codes8) {
    float ds = orc_e4m3_decode(s);
    uint8_t q[16];
    if (ds == 0.0f) {
        memset(q, 0, sizeof q);
    } else {
        float S = ds * g;
        float r = 1.0f / S;
        for (int i = 0; i < 16; ++i) q[i] = orc_e2m1_encode(y[i] * r);
    }
    if (codes8 != NULL)
        for (int j = 0; j < 8; ++j) codes8[j] = (uint8_t)(q[2 * j] | (q[2 * j + 1] << 4));
    double e = 0.0;
    for (int i = 0; i < 16; ++i) {
        double rec = (double)orc_e2m1_decode(q[i]) * (double)ds * (double)g;
        double d = (double)y[i] - rec;
        e = e + d * d;
    }
    return e;
}

uint8_t orc_quantize_block16_mse(const float *y, float g, uint8_t *codes8) {
    uint8_t best = 0;
    double best_e = orc_block_sse(y, g, 0, NULL);
    for (int s = 1; s <= 0x7E; ++s) {
        double e = orc_block_sse(y, g, (uint8_t)s, NULL);
        if (e < best_e) {
            best_e = e;
            best = (uint8_t)s;
        }
    }
    orc_block_sse(y, g, best, codes8);
    return best;
}

/* As orc_quantize_weight, with the block scales of orc_quantize_block16_mse. */
float orc_quantize_weight_mse(const uint16_t *w, int N, int K, int ldw, int interleave_gate_up,
                              uint8_t *codes, uint8_t *sf) {
    float amax = 0.0f;
    for (int n = 0; n < N; ++n)
        for (int k = 0; k < K; ++k) {
            float m = fabsf(bf16_to_f32(w[(size_t)n * ldw + k]));
            if (m > amax) amax = m;
        }
    float g = (amax == 0.0f) ? 1.0f : amax / 2688.0f;
    int nblk = (K + 15) / 16;
    float blk[16];
    for (int r = 0; r < N; ++r) {
        int src = r;
        if (interleave_gate_up) src = (r % 2 == 0) ? r / 2 : N / 2 + r / 2;
        for (int b = 0; b < nblk; ++b) {
            for (int i = 0; i < 16; ++i) {
                int k = b * 16 + i;
                blk[i] = (k < K) ? bf16_to_f32(w[(size_t)src * ldw + k]) : 0.0f;
            }
            uint8_t s = orc_quantize_block16_mse(blk, g, codes + (size_t)r * nblk * 8 + (size_t)b * 8);
            sf[orc_sf_offset(r, b, K)] = s;
        }
    }
    return g;
}

/* ------------------------------------------------------------------------------------ */
/* 16-point Hadamard rotation of one block ("Pi0.5 Thor NVFP4 End-to-End Results",
 * §Full-INT4 Decoder Activations + Hadamard Rotation: every 16-value block of both GEMM
 * operands is rotated by the orthonormal 16 x 16 Hadamard matrix before quantization;
 * lane-parallel kernels run it as a 4-stage shfl_xor butterfly, vectorized kernels as an
 * in-register fast Walsh-Hadamard transform; the rotation leaves the GEMM unchanged).
 * The matrix is Sylvester's H16, entry (i, j) = (-1)^popcount(i & j), times 1/4, which
 * makes it orthonormal and its own inverse.
 * READING: the four butterfly stages pair element i with element i ^ d for d = 1, 2, 4, 8
 * in that order; of each pair the element whose index has bit d clear becomes a + b and
 * the other a - b (a the lower-index value), each one fp32 addition or subtraction
 * rounded to nearest even; the 1/4 is applied last, one fp32 multiply per element (exact
 * unless the result is subnormal).                                                       */
void orc_hadamard16(float *y) {
    for (int d = 1; d < 16; d <<= 1)
        for (int i = 0; i < 16; ++i)
            if ((i & d) == 0) {
                float a = y[i], b = y[i | d];
                y[i] = a + b;
                y[i | d] = a - b;
            }
    for (int i = 0; i < 16; ++i) y[i] = y[i] * 0.25f;
}

/* The same rotation in fp64 (the reference value of a rotated fp64 activation). */
static void hadamard16_f64(double *y) {
    for (int d = 1; d < 16; d <<= 1)
        for (int i = 0; i < 16; ++i)
            if ((i & d) == 0) {
                double a = y[i], b = y[i | d];
                y[i] = a + b;
                y[i | d] = a - b;
            }
    for (int i = 0; i < 16; ++i) y[i] = y[i] * 0.25;
}

/* Uniform INT4 elements, E0M3 ("Pi0.5 ...", §E0M3 Uniform-INT4 Decoder Weights: a
 * sign-magnitude uniform INT4 grid, magnitudes 0..7, beside E2M1; per-16 UE4M3 block
 * scales computed as amax / 7).
 * READING: code bit 3 is the sign and bits 0..2 the magnitude, so code c decodes to
 * +-(c & 7); encoding rounds |v| to the nearest integer, ties to the even integer (the
 * rounding the E2M1 path uses), and saturates at 7; the sign of v is kept as in E2M1, so
 * a negative value that rounds to 0 gives 0x8.  Inputs are finite.                       */
float orc_e0m3_decode(uint8_t code) {
    double m = (double)(code & 7u);
    return (float)((code & 8u) ? -m : m);
}

uint8_t orc_e0m3_encode(float v) {
    uint8_t sign = signbit(v) ? 8u : 0u;
    double a = fabs((double)v);
    if (a >= 7.0) return (uint8_t)(sign | 7u);
    double fl = floor(a);
    double fr = a - fl; /* exact: a < 8 has at most 24 significant bits */
    int q = (int)fl;
    if (fr > 0.5 || (fr == 0.5 && (q & 1) != 0)) q += 1;
    return (uint8_t)(sign | (uint8_t)q);
}

/* One E0M3 block: the E2M1 block quantizer's steps with 7 in place of 6.
 *   a = max|y|;  d = 7*g;  t = a/d;  s = E4M3(t);  S = dec(s)*g
 *   dec(s) == 0 -> every code +0;  else r = 1/S, code_i = E0M3(y_i * r)
 * READING: one IEEE fp32 operation per step, as for E2M1.                                 */
uint8_t orc_quantize_block16_e0m3(const float *y, float g, uint8_t *codes8) {
    float a = 0.0f;
    for (int i = 0; i < 16; ++i) {
        float m = fabsf(y[i]);
        if (m > a) a = m;
    }
    float d = 7.0f * g;
    float t = a / d;
    uint8_t s = orc_e4m3_encode(t);
    float ds = orc_e4m3_decode(s);
    if (ds == 0.0f) {
        memset(codes8, 0, 8);
        return s;
    }
    float S = ds * g;
    float r = 1.0f / S;
    for (int j = 0; j < 8; ++j) {
        float v0 = y[2 * j] * r;
        float v1 = y[2 * j + 1] * r;
        codes8[j] = (uint8_t)(orc_e0m3_encode(v0) | (orc_e0m3_encode(v1) << 4));
    }
    return s;
}

/* A block under the quantizer options: rotated first if ORC_Q_ROTATE, then the E2M1 or
 * (ORC_Q_E0M3) the E0M3 block quantizer.  y is not modified.                             */
uint8_t orc_quantize_block16_ex(const float *y, float g, int flags, uint8_t *codes8) {
    float blk[16];
    memcpy(blk, y, sizeof blk);
    if (flags & ORC_Q_ROTATE) orc_hadamard16(blk);
    return (flags & ORC_Q_E0M3) ? orc_quantize_block16_e0m3(blk, g, codes8) : orc_quantize_block16(blk, g, codes8);
}

void orc_quantize_rows_ex(const float *y, int rows, int K, int ldy, float g, int flags,
                          uint8_t *codes, uint8_t *sf) {
    int nblk = (K + 15) / 16;
    size_t row_bytes = (size_t)nblk * 8;
    float blk[16];
    for (int r = 0; r < rows; ++r) {
        for (int b = 0; b < nblk; ++b) {
            for (int i = 0; i < 16; ++i) {
                int k = b * 16 + i;
                blk[i] = (k < K) ? y[(size_t)r * ldy + k] : 0.0f;
            }
            sf[orc_sf_offset(r, b, K)] =
                orc_quantize_block16_ex(blk, g, flags, codes + (size_t)r * row_bytes + (size_t)b * 8);
        }
    }
}

/* Norm then quantize under the options (the rotation applies to the normalized y). */
void orc_quantize_norm_ex(const void *x, int in_fp32, int rows, int K, int ldx, int kind,
                          const uint16_t *gamma, const uint16_t *beta, const uint16_t *mod_scale,
                          const uint16_t *mod_shift, float eps, float g, int flags,
                          uint8_t *codes, uint8_t *sf) {
    float *y = (float *)malloc(sizeof(float) * (size_t)K);
    size_t esz = in_fp32 ? 4 : 2;
    int nblk = (K + 15) / 16;
    for (int r = 0; r < rows; ++r) {
        const char *xr = (const char *)x + (size_t)r * ldx * esz;
        orc_norm_rows(xr, in_fp32, 1, K, ldx, kind, gamma, beta, mod_scale, mod_shift, eps, y);
        float blk[16];
        for (int b = 0; b < nblk; ++b) {
            for (int i = 0; i < 16; ++i) {
                int k = b * 16 + i;
                blk[i] = (k < K) ? y[k] : 0.0f;
            }
            sf[orc_sf_offset(r, b, K)] =
                orc_quantize_block16_ex(blk, g, flags, codes + (size_t)r * nblk * 8 + (size_t)b * 8);
        }
    }
    free(y);
}

/* Offline weight quantizer under the options.  The values quantized are the (optionally
 * rotated) 16-element blocks of W along K, rows optionally gate/up interleaved as in
 * orc_quantize_weight; with `mse` (E2M1 only) the block scales are the MSE search's.
 * READING: the global scale is amax over the values actually quantized (the rotated
 * blocks when rotating, since a rotated block's amax can reach 4x the original's) divided
 * by (top grid magnitude x 448): 6 x 448 = 2688 for E2M1, 7 x 448 = 3136 for E0M3, so the
 * largest block scale lands on the E4M3 maximum; an all-zero tensor takes g = 1.  The
 * pages give E0M3 weights amax/7 block scales only, so mse with E0M3 is not defined and
 * the E0M3 amax quantizer is used.                                                        */
float orc_quantize_weight_ex(const uint16_t *w, int N, int K, int ldw, int interleave_gate_up, int flags,
                             int mse, uint8_t *codes, uint8_t *sf) {
    int nblk = (K + 15) / 16;
    float *vals = (float *)malloc(sizeof(float) * (size_t)N * nblk * 16);
    float amax = 0.0f;
    for (int r = 0; r < N; ++r) {
        int src = r;
        if (interleave_gate_up) src = (r % 2 == 0) ? r / 2 : N / 2 + r / 2;
        for (int b = 0; b < nblk; ++b) {
            float *blk = vals + ((size_t)r * nblk + b) * 16;
            for (int i = 0; i < 16; ++i) {
                int k = b * 16 + i;
                blk[i] = (k < K) ? bf16_to_f32(w[(size_t)src * ldw + k]) : 0.0f;
            }
            if (flags & ORC_Q_ROTATE) orc_hadamard16(blk);
            for (int i = 0; i < 16; ++i) {
                float m = fabsf(blk[i]);
                if (m > amax) amax = m;
            }
        }
    }
    float g = (amax == 0.0f) ? 1.0f : amax / ((flags & ORC_Q_E0M3) ? 3136.0f : 2688.0f);
    for (int r = 0; r < N; ++r)
        for (int b = 0; b < nblk; ++b) {
            const float *blk = vals + ((size_t)r * nblk + b) * 16;
            uint8_t *c8 = codes + (size_t)r * nblk * 8 + (size_t)b * 8;
            uint8_t s;
            if (flags & ORC_Q_E0M3) s = orc_quantize_block16_e0m3(blk, g, c8);
            else if (mse) s = orc_quantize_block16_mse(blk, g, c8);
            else s = orc_quantize_block16(blk, g, c8);
            sf[orc_sf_offset(r, b, K)] = s;
        }
    free(vals);
    return g;
}

/* Dequantize under the element grid of `flags` (E0M3 or E2M1); a rotation is not undone:
 * the result is the (rotated) block the codes represent.                                  */
void orc_dequantize_ex(const uint8_t *codes, const uint8_t *sf, float g, int rows, int K, int flags,
                       double *out) {
    int nblk = (K + 15) / 16;
    for (int r = 0; r < rows; ++r)
        for (int k = 0; k < K; ++k) {
            uint8_t byte = codes[(size_t)r * nblk * 8 + (size_t)k / 2];
            uint8_t c = (k % 2 == 0) ? (byte & 15u) : (byte >> 4);
            double e = (flags & ORC_Q_E0M3) ? (double)orc_e0m3_decode(c) : (double)orc_e2m1_decode(c);
            out[(size_t)r * K + k] = e * (double)orc_e4m3_decode(sf[orc_sf_offset(r, k / 16, K)]) * (double)g;
        }
}

/* Dequantized value of element k of row `row`: val(code) * dec(scale) * g, exact in fp64. */
static double deq_elem(const uint8_t *codes, const uint8_t *sf, float g, int row, int k, int K) {
    int nblk = (K + 15) / 16;
    uint8_t byte = codes[(size_t)row * nblk * 8 + (size_t)k / 2];
    uint8_t c = (k % 2 == 0) ? (byte & 15u) : (byte >> 4);
    double s = (double)orc_e4m3_decode(sf[orc_sf_offset(row, k / 16, K)]);
    return (double)orc_e2m1_decode(c) * s * (double)g;
}

void orc_dequantize(const uint8_t *codes, const uint8_t *sf, float g, int rows, int K,
                    double *out) {
    for (int r = 0; r < rows; ++r)
        for (int k = 0; k < K; ++k) out[(size_t)r * K + k] = deq_elem(codes, sf, g, r, k, K);
}

/* ------------------------------------------------------------------------------------ */
/* tanh-form GELU, 0.5 z (1 + tanh(sqrt(2/pi) (z + 0.044715 z^3))), in fp64. */
double orc_gelu_tanh(double z) {
    const double k = sqrt(2.0 / 3.14159265358979323846);
    return 0.5 * z * (1.0 + tanh(k * (z + 0.044715 * z * z * z)));
}

/* Block-scaled GEMM with fused epilogue ("GROOT N1.7 ...", §What is in the tier: every
 * DiT GEMM is NVFP4 x NVFP4 with fused bf16 bias / bias+residual / bias+tanh-GELU+FP4
 * output epilogues; "Pi0.5 ...", §Half-Width Fused GeGLU Epilogue and §Fused GeGLU FFN
 * in the Decoder: gelu(gate) * up on pairwise-interleaved columns, quantized once, GELU
 * on the fp32 accumulator rather than on a rounded GEMM output).
 *   acc[m,n] = sum_k Adeq[m,k] * Wdeq[n,k]          (fp64, k ascending)
 *   v[m,n]   = acc + bias[n] + residual[m,n]        (terms present per epilogue)
 *   BIAS_GELU: h = gelu(v), N_out = N;   GEGLU: h[m,j] = gelu(v[m,2j]) * v[m,2j+1], N_out = N/2
 *   FP4 output = the block quantizer applied to (float)h along n with g_out.
 *   BIAS_GELU_RHT / GEGLU_RHT: the same, each 16-value block of (float)h rotated by
 *   orc_hadamard16 before the block quantizer ("Pi0.5 ...", §Full-INT4 Decoder Activations +
 *   Hadamard Rotation: the GeGLU exit is one of the rotated activation exits, so the next
 *   GEMM's rotated weights see a rotated input); h_out then holds the fp64 rotation of h.
 * Dequantized operands include their global scales, so acc already carries gA * gW.    */
void orc_gemm(const uint8_t *a_codes, const uint8_t *a_sf, float gA, int M,
              const uint8_t *w_codes, const uint8_t *w_sf, float gW, int N, int K,
              int epi, const uint16_t *bias, const uint16_t *residual, int ldr,
              const int *m_idx, int n_rows, double *v_out, double *h_out,
              float g_out, uint8_t *out_codes, uint8_t *out_sf) {
    if (!m_idx) n_rows = M;
    double *arows = (double *)malloc(sizeof(double) * (size_t)n_rows * K);
    double *wrow = (double *)malloc(sizeof(double) * (size_t)K);
    for (int i = 0; i < n_rows; ++i) {
        int m = m_idx ? m_idx[i] : i;
        for (int k = 0; k < K; ++k) arows[(size_t)i * K + k] = deq_elem(a_codes, a_sf, gA, m, k, K);
    }
    int rot = (epi == ORC_EPI_BIAS_GELU_RHT || epi == ORC_EPI_GEGLU_RHT);
    if (epi == ORC_EPI_BIAS_GELU_RHT) epi = ORC_EPI_BIAS_GELU;
    if (epi == ORC_EPI_GEGLU_RHT) epi = ORC_EPI_GEGLU;
    int use_bias = (epi == ORC_EPI_BIAS || epi == ORC_EPI_BIAS_RESIDUAL || epi == ORC_EPI_BIAS_GELU ||
                    epi == ORC_EPI_GEGLU) && bias != NULL;
    int use_res = (epi == ORC_EPI_RESIDUAL || epi == ORC_EPI_BIAS_RESIDUAL);
    for (int n = 0; n < N; ++n) {
        for (int k = 0; k < K; ++k) wrow[k] = deq_elem(w_codes, w_sf, gW, n, k, K);
        for (int i = 0; i < n_rows; ++i) {
            int m = m_idx ? m_idx[i] : i;
            const double *ar = arows + (size_t)i * K;
            double acc = 0.0;
            for (int k = 0; k < K; ++k) acc += ar[k] * wrow[k];
            if (use_bias) acc += (double)bf16_to_f32(bias[n]);
            if (use_res) acc += (double)bf16_to_f32(residual[(size_t)m * ldr + n]);
            v_out[(size_t)i * N + n] = acc;
        }
    }
    if (epi == ORC_EPI_BIAS_GELU || epi == ORC_EPI_GEGLU) {
        int n_out = (epi == ORC_EPI_GEGLU) ? N / 2 : N;
        float *hf = (float *)malloc(sizeof(float) * (size_t)n_out);
        int oblk = (n_out + 15) / 16;
        for (int i = 0; i < n_rows; ++i) {
            int m = m_idx ? m_idx[i] : i;
            const double *v = v_out + (size_t)i * N;
            for (int j = 0; j < n_out; ++j) {
                double h = (epi == ORC_EPI_GEGLU) ? orc_gelu_tanh(v[2 * j]) * v[2 * j + 1]
                                                   : orc_gelu_tanh(v[j]);
                if (h_out) h_out[(size_t)i * n_out + j] = h;
                hf[j] = (float)h;
            }
            if (h_out && rot)
                for (int b = 0; b + 16 <= n_out; b += 16) hadamard16_f64(h_out + (size_t)i * n_out + b);
            if (out_codes && out_sf) {
                float blk[16];
                for (int b = 0; b < oblk; ++b) {
                    for (int t = 0; t < 16; ++t) {
                        int j = b * 16 + t;
                        blk[t] = (j < n_out) ? hf[j] : 0.0f;
                    }
                    uint8_t s = orc_quantize_block16_ex(blk, g_out, rot ? ORC_Q_ROTATE : 0,
                                                        out_codes + (size_t)m * oblk * 8 + (size_t)b * 8);
                    out_sf[orc_sf_offset(m, b, n_out)] = s;
                }
            }
        }
        free(hf);
    }
    free(wrow);
    free(arows);
}
