// norm_row.cuh — one row of the norm -> NVFP4 front-end, shared by the standalone kernel
// and the layer executor (both must produce the same bytes).
//
// One row is owned by TPR threads.  Each thread loads whole 16-element blocks with 16-byte
// loads (block b of a row goes to thread b % TPR), keeps them in registers, reduces the row
// statistics with warp shuffles (and shared memory across warps), then normalizes,
// quantizes and stores each block from the same registers ("Pi0.5 Thor NVFP4 End-to-End
// Results", §Vectorized SigLIP LayerNorms: 16-byte loads, one 16-element block per thread,
// all stages from registers).
//
// Row statistics are fp64 sums (mean, then the population variance about it; mean of
// squares for RMS), rounded once to fp32: mu_f = (float)mu, rstd_f = (float)(1/sqrt(v+eps)).
// The elementwise steps are single fp32 operations in a fixed order (no contraction):
//   LayerNorm  y = ((x - mu_f) * rstd_f) * gamma + beta
//   RMSNorm    y = (x * rstd_f) * gamma
//   AdaLN      y = ((x - mu_f) * rstd_f) * (1 + scale) + shift
//   AdaRMSNorm y = (x * rstd_f) * (1 + scale) [+ shift]
// ("GROOT N1.7 update: Thor NVFP4 + FA4 performance tier", §What is in the tier: AdaLN and
// the pre-FFN LayerNorm emit FP4 directly, bit-identical to the two-step chain; "Pi0.5 ...",
// §Implemented Path: AdaRMSNorm + NVFP4/SFA in one launch.)
#pragma once

#include "norm.h"
#include "quant.cuh"

namespace nvfp4 {

enum { kNone = 0, kLayerNorm = 1, kRmsNorm = 2, kAdaLN = 3, kAdaRms = 4 };

template <int TPR>
__device__ __forceinline__ double row_sum(double v, double *red) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = __dadd_rn(v, __shfl_xor_sync(0xffffffffu, v, o));
    if constexpr (TPR == 32) {
        return v;
    } else {
        const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
        __syncthreads();
        if (lane == 0) red[warp] = v;
        __syncthreads();
        double s = 0.0;
#pragma unroll
        for (int w = 0; w < TPR / 32; ++w) s = __dadd_rn(s, red[w]);
        return s;
    }
}

// Loads the 16 params of block b (bf16) as fp32, or `dflt` when the pointer is NULL.
__device__ __forceinline__ void load_param16(const uint16_t *p, int b, float dflt, float *out) {
    if (p == nullptr) {
#pragma unroll
        for (int i = 0; i < 16; ++i) out[i] = dflt;
        return;
    }
    const uint4 *q = reinterpret_cast<const uint4 *>(p + static_cast<size_t>(b) * 16);
    const uint4 u0 = __ldg(q), u1 = __ldg(q + 1);
    const uint32_t w[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        out[2 * i] = bf16lo(w[i]);
        out[2 * i + 1] = bf16hi(w[i]);
    }
}

// Row `row` of p, handled by thread t of TPR (TPR = 32: one warp; TPR = 128: the CTA, with
// `red` four doubles of shared memory).  TPR, BPT (blocks of 16 per thread) and F32 (fp32
// input, else bf16) are compile-time; K <= 16 * TPR * BPT.
template <int TPR, int BPT, bool F32>
__device__ __forceinline__ void norm_row(const NormArgs &p, int row, int t, double *red) {
    constexpr int kWords = F32 ? 16 : 8;  // 32-bit words per 16-element block
    const int nblk = p.K >> 4;
    const int k_atoms = (p.K + 63) >> 6;
    const bool row_ok = row < p.M;
    int src_row = row;
    if (p.interleave) src_row = (row & 1) ? (p.M >> 1) + (row >> 1) : (row >> 1);

    uint32_t raw[BPT][kWords];
    const char *xrow = static_cast<const char *>(p.x) +
                       static_cast<size_t>(row_ok ? src_row : 0) * p.ldx * (F32 ? 4 : 2);
#pragma unroll
    for (int i = 0; i < BPT; ++i) {
        const int b = t + i * TPR;
        if (row_ok && b < nblk) {
            const uint4 *q = reinterpret_cast<const uint4 *>(xrow + static_cast<size_t>(b) * 16 * (F32 ? 4 : 2));
#pragma unroll
            for (int j = 0; j < kWords / 4; ++j) {
                const uint4 u = __ldg(q + j);
                raw[i][4 * j] = u.x;
                raw[i][4 * j + 1] = u.y;
                raw[i][4 * j + 2] = u.z;
                raw[i][4 * j + 3] = u.w;
            }
        } else {
#pragma unroll
            for (int j = 0; j < kWords; ++j) raw[i][j] = 0u;
        }
    }
    auto elem = [&](int i, int e) -> float {
        if constexpr (F32) return __uint_as_float(raw[i][e]);
        else return (e & 1) ? bf16hi(raw[i][e >> 1]) : bf16lo(raw[i][e >> 1]);
    };

    // ---- row statistics (fp64) ----
    float mu_f = 0.0f, rstd_f = 1.0f;
    const int kind = p.kind;
    if (kind == kLayerNorm || kind == kAdaLN) {
        double s = 0.0;
#pragma unroll
        for (int i = 0; i < BPT; ++i)
#pragma unroll
            for (int e = 0; e < 16; ++e) s = __dadd_rn(s, static_cast<double>(elem(i, e)));
        s = row_sum<TPR>(s, red);
        const double mu = __ddiv_rn(s, static_cast<double>(p.K));
        double q = 0.0;
#pragma unroll
        for (int i = 0; i < BPT; ++i) {
            if (t + i * TPR < nblk) {
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    const double dv = __dsub_rn(static_cast<double>(elem(i, e)), mu);
                    q = __dadd_rn(q, __dmul_rn(dv, dv));
                }
            }
        }
        q = row_sum<TPR>(q, red);
        mu_f = static_cast<float>(mu);
        rstd_f = static_cast<float>(
            __ddiv_rn(1.0, __dsqrt_rn(__dadd_rn(__ddiv_rn(q, static_cast<double>(p.K)), static_cast<double>(p.eps)))));
    } else if (kind == kRmsNorm || kind == kAdaRms) {
        double q = 0.0;
#pragma unroll
        for (int i = 0; i < BPT; ++i)
#pragma unroll
            for (int e = 0; e < 16; ++e) {
                const double xv = static_cast<double>(elem(i, e));
                q = __dadd_rn(q, __dmul_rn(xv, xv));
            }
        q = row_sum<TPR>(q, red);
        rstd_f = static_cast<float>(
            __ddiv_rn(1.0, __dsqrt_rn(__dadd_rn(__ddiv_rn(q, static_cast<double>(p.K)), static_cast<double>(p.eps)))));
    }
    if (!row_ok) return;

    float g = p.g;
    if (p.amax_bits != nullptr) {
        const float amax = __uint_as_float(*p.amax_bits);
        g = (amax == 0.0f) ? 1.0f : __fdiv_rn(amax, 2688.0f);
    }
    const float d6g = __fmul_rn(6.0f, g);

    // ---- normalize + quantize each block from registers ----
#pragma unroll
    for (int i = 0; i < BPT; ++i) {
        const int b = t + i * TPR;
        if (b >= nblk) break;
        float y[16];
        if (kind == kNone) {
#pragma unroll
            for (int e = 0; e < 16; ++e) y[e] = elem(i, e);
        } else {
            float pa[16], pb[16];
            const bool ln = (kind == kLayerNorm || kind == kAdaLN);
            const bool ada = (kind == kAdaLN || kind == kAdaRms);
            if (ada) {
                load_param16(p.scale, b, 0.0f, pa);
#pragma unroll
                for (int e = 0; e < 16; ++e) pa[e] = __fadd_rn(1.0f, pa[e]);
            } else {
                load_param16(p.gamma, b, 1.0f, pa);
            }
            const bool add_b = (kind == kLayerNorm) || (kind == kAdaLN) ||
                               (kind == kAdaRms && p.shift != nullptr);
            if (add_b) load_param16(kind == kLayerNorm ? p.beta : p.shift, b, 0.0f, pb);
#pragma unroll
            for (int e = 0; e < 16; ++e) {
                const float xv = elem(i, e);
                const float n = ln ? __fmul_rn(__fsub_rn(xv, mu_f), rstd_f) : __fmul_rn(xv, rstd_f);
                const float tt = __fmul_rn(n, pa[e]);
                y[e] = add_b ? __fadd_rn(tt, pb[e]) : tt;
            }
        }
        if (p.y_out != nullptr) {
            float4 *yo = reinterpret_cast<float4 *>(p.y_out + static_cast<size_t>(row) * p.K + b * 16);
#pragma unroll
            for (int j = 0; j < 4; ++j) yo[j] = make_float4(y[4 * j], y[4 * j + 1], y[4 * j + 2], y[4 * j + 3]);
            continue;
        }
        uint2 c;
        const uint32_t s = quantize_block16(y, g, d6g, c);
        *reinterpret_cast<uint2 *>(p.codes + static_cast<size_t>(row) * (p.K >> 1) + b * 8) = c;
        p.sf[sf_offset(row, b, k_atoms)] = static_cast<uint8_t>(s);
    }
}

}  // namespace nvfp4
