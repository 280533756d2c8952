// norm_row.cuh — one row of the norm -> NVFP4 front-end (the norm_quant_kernel launches: a
// warp per row for many rows, four warps per row for few).
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

// Sum of v over the TPR threads of a row (t = the thread's index among them).  TPR = 128:
// the CTA's four warps meet on named barrier 1, with `red` four doubles of shared memory.
template <int TPR>
__device__ __forceinline__ double row_sum(double v, double *red, int t) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = __dadd_rn(v, __shfl_xor_sync(0xffffffffu, v, o));
    if constexpr (TPR == 32) {
        return v;
    } else {
        static_assert(TPR == 128, "a row is one warp or four");
        const int warp = t >> 5, lane = t & 31;
        asm volatile("bar.sync 1, 128;" ::: "memory");
        if (lane == 0) red[warp] = v;
        asm volatile("bar.sync 1, 128;" ::: "memory");
        double s = 0.0;
#pragma unroll
        for (int w = 0; w < TPR / 32; ++w) s = __dadd_rn(s, red[w]);
        return s;
    }
}

// Pairwise fp64 sum of the 16 elements of one block (fp32 values, exact in fp64).
template <class Elem>
__device__ __forceinline__ double block_sum16(Elem elem) {
    double v[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) v[e] = __dadd_rn(static_cast<double>(elem(2 * e)), static_cast<double>(elem(2 * e + 1)));
#pragma unroll
    for (int w = 4; w > 0; w >>= 1)
#pragma unroll
        for (int e = 0; e < w; ++e) v[e] = __dadd_rn(v[e], v[e + w]);
    return v[0];
}

// Row `row` of p, handled by thread t of TPR (TPR = 32: one warp; TPR = 128: four warps on
// named barrier 1, with `red` four doubles of shared memory).  TPR, BPT (blocks of 16 per thread) and F32 (fp32
// input, else bf16) are compile-time; K <= 16 * TPR * BPT.
//
// Latency is what matters at tens of rows, so every global load of the row is issued
// first: the x blocks (ld.global.cg: x may have been written earlier in the same launch by
// other SMs), and the per-column parameters (bf16, read-only; in registers for BPT <= 4,
// else prefetched into L1).  The fp64 sums are pairwise trees per block, so the dependent
// chain is a few adds rather than one per element; fp64 keeps the rounded fp32 statistics
// independent of the summation order.
template <int TPR, int BPT, bool F32>
__device__ __forceinline__ void norm_row(const NormArgs &p, int row, int t, double *red) {
    constexpr int kWords = F32 ? 16 : 8;  // 32-bit words per 16-element block
    constexpr bool kParamRegs = BPT <= 4;
    // Every field is read once into a local: the byte stores below may alias any memory as
    // far as the compiler knows.
    const int M = p.M, K = p.K, ldx = p.ldx, kind = p.kind;
    const void *const x = p.x;
    const float eps = p.eps, g_arg = p.g;
    const uint32_t *const amax_bits = p.amax_bits;
    const int qflags = p.qflags;
    uint8_t *const codes_out = p.codes;
    uint8_t *const sf_out = p.sf;
    float *const y_out = p.y_out;
    const uint16_t *const res_d = F32 ? nullptr : p.res_d;
    const uint16_t *const res_gate = p.res_gate;
    uint16_t *const h_out = p.h_out;
    const int ldd = p.ldd, ldh = p.ldh;
    const int nblk = K >> 4;
    const int k_atoms = (K + 63) >> 6;
    const bool row_ok = row < M;
    int src_row = row;
    if (p.interleave) src_row = (row & 1) ? (M >> 1) + (row >> 1) : (row >> 1);

    const bool ln = (kind == kLayerNorm || kind == kAdaLN);
    const bool ada = (kind == kAdaLN || kind == kAdaRms);
    const bool has_a = kind != kNone;
    const bool add_b = (kind == kLayerNorm) || (kind == kAdaLN) || (kind == kAdaRms && p.shift != nullptr);
    // y = n * A + B with A = gamma (default 1) or 1 + scale (default scale 0), B = beta / shift
    const uint16_t *pa = ada ? p.scale : p.gamma;
    const uint16_t *pb = (kind == kLayerNorm) ? p.beta : p.shift;
    const uint32_t pa_dflt = ada ? 0u : 0x3F803F80u;  // bf16 pair (0, 0) or (1, 1)

    uint32_t raw[BPT][kWords];
    uint32_t wa[kParamRegs ? BPT : 1][8], wb[kParamRegs ? BPT : 1][8];
    const char *xrow = static_cast<const char *>(x) +
                       static_cast<size_t>(row_ok ? src_row : 0) * ldx * (F32 ? 4 : 2);
#pragma unroll
    for (int i = 0; i < BPT; ++i) {
        const int b = t + i * TPR;
        const bool ok = row_ok && b < nblk;
        if (ok) {
            const uint4 *q = reinterpret_cast<const uint4 *>(xrow + static_cast<size_t>(b) * 16 * (F32 ? 4 : 2));
#pragma unroll
            for (int j = 0; j < kWords / 4; ++j) {
                const uint4 u = __ldcg(q + j);
                raw[i][4 * j] = u.x;
                raw[i][4 * j + 1] = u.y;
                raw[i][4 * j + 2] = u.z;
                raw[i][4 * j + 3] = u.w;
            }
        } else {
#pragma unroll
            for (int j = 0; j < kWords; ++j) raw[i][j] = 0u;
        }
        if constexpr (!F32) {
            // gated residual front-end ("Pi0.5 Thor NVFP4 End-to-End Results", §Implemented
            // Path): h = x + gate * d, one fp32 product and one fp32 sum, rounded once to bf16;
            // h replaces x for the norm and is stored as the new residual stream
            if (res_d != nullptr && ok) {
                const uint4 *qd = reinterpret_cast<const uint4 *>(res_d + static_cast<size_t>(src_row) * ldd + b * 16);
                const uint4 d0 = __ldcg(qd), d1 = __ldcg(qd + 1);
                uint4 g0 = make_uint4(0x3F803F80u, 0x3F803F80u, 0x3F803F80u, 0x3F803F80u), g1 = g0;
                if (res_gate != nullptr) {
                    const uint4 *qg = reinterpret_cast<const uint4 *>(res_gate + b * 16);
                    g0 = __ldg(qg);
                    g1 = __ldg(qg + 1);
                }
                const uint32_t dw[8] = {d0.x, d0.y, d0.z, d0.w, d1.x, d1.y, d1.z, d1.w};
                const uint32_t gw[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const float lo = __fadd_rn(bf16lo(raw[i][j]), __fmul_rn(bf16lo(gw[j]), bf16lo(dw[j])));
                    const float hi = __fadd_rn(bf16hi(raw[i][j]), __fmul_rn(bf16hi(gw[j]), bf16hi(dw[j])));
                    raw[i][j] = pack_bf16x2_rn(lo, hi);
                }
                uint4 *qh = reinterpret_cast<uint4 *>(h_out + static_cast<size_t>(row) * ldh + b * 16);
                qh[0] = make_uint4(raw[i][0], raw[i][1], raw[i][2], raw[i][3]);
                qh[1] = make_uint4(raw[i][4], raw[i][5], raw[i][6], raw[i][7]);
            }
        }
        if constexpr (kParamRegs) {
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                wa[i][j] = pa_dflt;
                wb[i][j] = 0u;
            }
            if (ok && has_a && pa != nullptr) {
                const uint4 *q = reinterpret_cast<const uint4 *>(pa + static_cast<size_t>(b) * 16);
                const uint4 u0 = __ldg(q), u1 = __ldg(q + 1);
                wa[i][0] = u0.x; wa[i][1] = u0.y; wa[i][2] = u0.z; wa[i][3] = u0.w;
                wa[i][4] = u1.x; wa[i][5] = u1.y; wa[i][6] = u1.z; wa[i][7] = u1.w;
            }
            if (ok && add_b && pb != nullptr) {
                const uint4 *q = reinterpret_cast<const uint4 *>(pb + static_cast<size_t>(b) * 16);
                const uint4 u0 = __ldg(q), u1 = __ldg(q + 1);
                wb[i][0] = u0.x; wb[i][1] = u0.y; wb[i][2] = u0.z; wb[i][3] = u0.w;
                wb[i][4] = u1.x; wb[i][5] = u1.y; wb[i][6] = u1.z; wb[i][7] = u1.w;
            }
        } else {
            if (ok && has_a && pa != nullptr)
                asm volatile("prefetch.global.L1 [%0];" ::"l"(pa + static_cast<size_t>(b) * 16));
            if (ok && add_b && pb != nullptr)
                asm volatile("prefetch.global.L1 [%0];" ::"l"(pb + static_cast<size_t>(b) * 16));
        }
    }
    auto elem = [&](int i, int e) -> float {
        if constexpr (F32) return __uint_as_float(raw[i][e]);
        else return (e & 1) ? bf16hi(raw[i][e >> 1]) : bf16lo(raw[i][e >> 1]);
    };

    // ---- row statistics (fp64) ----
    float mu_f = 0.0f, rstd_f = 1.0f;
    if (ln) {
        double s = 0.0;
#pragma unroll
        for (int i = 0; i < BPT; ++i) s = __dadd_rn(s, block_sum16([&](int e) { return elem(i, e); }));
        s = row_sum<TPR>(s, red, t);
        const double mu = __ddiv_rn(s, static_cast<double>(K));
        double q = 0.0;
#pragma unroll
        for (int i = 0; i < BPT; ++i) {
            if (t + i * TPR < nblk) {
                double d[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    const double dv = __dsub_rn(static_cast<double>(elem(i, e)), mu);
                    d[e] = __dmul_rn(dv, dv);
                }
#pragma unroll
                for (int w = 8; w > 0; w >>= 1)
#pragma unroll
                    for (int e = 0; e < w; ++e) d[e] = __dadd_rn(d[e], d[e + w]);
                q = __dadd_rn(q, d[0]);
            }
        }
        q = row_sum<TPR>(q, red, t);
        mu_f = static_cast<float>(mu);
        rstd_f = static_cast<float>(
            __ddiv_rn(1.0, __dsqrt_rn(__dadd_rn(__ddiv_rn(q, static_cast<double>(K)), static_cast<double>(eps)))));
    } else if (kind == kRmsNorm || kind == kAdaRms) {
        double q = 0.0;
#pragma unroll
        for (int i = 0; i < BPT; ++i) {
            double d[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) {
                const double xv = static_cast<double>(elem(i, e));
                d[e] = __dmul_rn(xv, xv);
            }
#pragma unroll
            for (int w = 8; w > 0; w >>= 1)
#pragma unroll
                for (int e = 0; e < w; ++e) d[e] = __dadd_rn(d[e], d[e + w]);
            q = __dadd_rn(q, d[0]);
        }
        q = row_sum<TPR>(q, red, t);
        rstd_f = static_cast<float>(
            __ddiv_rn(1.0, __dsqrt_rn(__dadd_rn(__ddiv_rn(q, static_cast<double>(K)), static_cast<double>(eps)))));
    }
    if (!row_ok) return;

    float g = g_arg;
    const float qmax = quant_qmax(qflags);
    if (amax_bits != nullptr) {
        const float amax = __uint_as_float(*amax_bits);
        g = (amax == 0.0f) ? 1.0f : __fdiv_rn(amax, __fmul_rn(qmax, 448.0f));
    }
    const float dqg = __fmul_rn(qmax, g);

    // ---- normalize + quantize each block from registers ----
#pragma unroll
    for (int i = 0; i < BPT; ++i) {
        const int b = t + i * TPR;
        if (b >= nblk) break;
        float y[16];
        if (!has_a) {
#pragma unroll
            for (int e = 0; e < 16; ++e) y[e] = elem(i, e);
        } else {
            uint32_t ua[8], ub[8];
            if constexpr (kParamRegs) {
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    ua[j] = wa[i][j];
                    ub[j] = wb[i][j];
                }
            } else {
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    ua[j] = pa_dflt;
                    ub[j] = 0u;
                }
                if (pa != nullptr) {
                    const uint4 *q = reinterpret_cast<const uint4 *>(pa + static_cast<size_t>(b) * 16);
                    const uint4 u0 = __ldg(q), u1 = __ldg(q + 1);
                    ua[0] = u0.x; ua[1] = u0.y; ua[2] = u0.z; ua[3] = u0.w;
                    ua[4] = u1.x; ua[5] = u1.y; ua[6] = u1.z; ua[7] = u1.w;
                }
                if (add_b && pb != nullptr) {
                    const uint4 *q = reinterpret_cast<const uint4 *>(pb + static_cast<size_t>(b) * 16);
                    const uint4 u0 = __ldg(q), u1 = __ldg(q + 1);
                    ub[0] = u0.x; ub[1] = u0.y; ub[2] = u0.z; ub[3] = u0.w;
                    ub[4] = u1.x; ub[5] = u1.y; ub[6] = u1.z; ub[7] = u1.w;
                }
            }
#pragma unroll
            for (int e = 0; e < 16; ++e) {
                const float xv = elem(i, e);
                float av = (e & 1) ? bf16hi(ua[e >> 1]) : bf16lo(ua[e >> 1]);
                if (ada) av = __fadd_rn(1.0f, av);
                const float n = ln ? __fmul_rn(__fsub_rn(xv, mu_f), rstd_f) : __fmul_rn(xv, rstd_f);
                const float tt = __fmul_rn(n, av);
                y[e] = add_b ? __fadd_rn(tt, (e & 1) ? bf16hi(ub[e >> 1]) : bf16lo(ub[e >> 1])) : tt;
            }
        }
        if (y_out != nullptr) {
            float4 *yo = reinterpret_cast<float4 *>(y_out + static_cast<size_t>(row) * K + b * 16);
#pragma unroll
            for (int j = 0; j < 4; ++j) yo[j] = make_float4(y[4 * j], y[4 * j + 1], y[4 * j + 2], y[4 * j + 3]);
            continue;
        }
        uint2 c;
        const uint32_t s = quantize_block16_opt(y, g, dqg, qflags, c);
        *reinterpret_cast<uint2 *>(codes_out + static_cast<size_t>(row) * (K >> 1) + b * 8) = c;
        sf_out[sf_offset(row, b, k_atoms)] = static_cast<uint8_t>(s);
    }
}

}  // namespace nvfp4
