// api.cu — the C ABI declared in include/nvfp4.h: argument validation, schedule choice,
// TMA descriptor encoding and kernel launches.  No entry point allocates device memory,
// and only nvfp4_quantize_weight / nvfp4_get_device_status synchronise.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cmath>
#include <cstdint>
#include <cstring>

#include "../../include/nvfp4.h"
#include "gemm.h"
#include "norm.h"


using namespace nvfp4;

namespace {

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool scale_ok(float g) {
    return std::isfinite(g) && g >= std::ldexp(1.0f, -100) && g <= std::ldexp(1.0f, 100);
}

// Current device must be compute capability 10.0 (B200 / sm_100a).
nvfp4_status check_device(int *sms = nullptr) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return NVFP4_ERR_CUDA;
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
        return NVFP4_ERR_CUDA;
    if (major != 10 || minor != 0) return NVFP4_ERR_UNSUPPORTED_DEVICE;
    if (sms && cudaDeviceGetAttribute(sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return NVFP4_ERR_CUDA;
    return NVFP4_OK;
}

nvfp4_status from_cuda(cudaError_t e) { return e == cudaSuccess ? NVFP4_OK : NVFP4_ERR_CUDA; }

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (fn == nullptr) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    return fn;
}

// 2-D uint8 view [rows, row_bytes] of FP4 codes, box 128 bytes x box_rows, 128-byte swizzle.
bool make_code_map(CUtensorMap *m, const void *ptr, int rows, int row_bytes, int box_rows) {
    auto fn = encode_fn();
    if (fn == nullptr) return false;
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(row_bytes), static_cast<cuuint64_t>(rows)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(row_bytes)};
    cuuint32_t box[2] = {128u, static_cast<cuuint32_t>(box_rows)};
    cuuint32_t estr[2] = {1u, 1u};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(ptr), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

unsigned long long *g_trace = nullptr;  // diagnostics: per-CTA GEMM timestamps
size_t g_trace_words = 0;
size_t g_trace_cursor = 0;

struct Schedule {
    int block_n;
    int splits;
    int kt_per_split;
    bool cluster;  // split-K partials reduced over DSMEM inside a cluster (no workspace)
};

constexpr int kMaxClusterSplits = 8;  // portable cluster size

int sm_count_cached() {
    static int sms = 0;
    if (sms == 0) {
        int dev = 0;
        if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            sms = 148;
    }
    return sms;
}

// Normalises a (block_n, splits) request so that every split owns >= 1 K tile.  Split
// counts up to the portable cluster size reduce inside a cluster (`use_cluster`), larger
// ones through the caller's workspace.
Schedule finish(int block_n, int splits, int K, bool use_cluster = true) {
    const int k_tiles = (K + 255) / 256;
    if (splits < 1) splits = 1;
    if (splits > k_tiles) splits = k_tiles;
    const int per = (k_tiles + splits - 1) / splits;
    const int eff = (k_tiles + per - 1) / per;
    return Schedule{block_n, eff, per, use_cluster && eff > 1 && eff <= kMaxClusterSplits};
}

// Default schedule.  Small M streams the weights: pick the tile width and split factor
// (<= 8, reduced in a cluster) that put about one CTA on every SM, preferring wider tiles
// and fewer splits.  Large M is compute-bound: widest tile, no split.
Schedule choose(int M, int N, int K) {
    const int sms = sm_count_cached();
    const int k_tiles = (K + 255) / 256;
    const int m_tiles = (M + 127) / 128;
    if (M <= 128) {
        Schedule best{64, 1, k_tiles, false};
        double best_cost = 1e30;
        for (int bn : {128, 64}) {
            if (N % bn != 0) continue;
            const int n_tiles = N / bn * m_tiles;
            for (int s = 1; s <= kMaxClusterSplits && s <= k_tiles; ++s) {
                const Schedule c = finish(bn, s, K);
                const int ctas = n_tiles * c.splits;
                if (ctas > 2 * sms) continue;
                const double cost = std::fabs(static_cast<double>(ctas - sms)) / sms + 0.03 * c.splits +
                                    (bn == 64 ? 0.05 : 0.0);
                if (cost < best_cost) {
                    best_cost = cost;
                    best = c;
                }
            }
        }
        return best;
    }
    const int bn = (N % 256 == 0) ? 256 : (N % 128 == 0) ? 128 : 64;
    return finish(bn, 1, K);
}

// The workspace-reduced schedule (used by nvfp4_gemm_noalloc): enough (tile, split) CTAs
// to put every SM on the weight stream, partials through global memory.
Schedule choose_workspace(int M, int N, int K) {
    const int sms = sm_count_cached();
    const int k_tiles = (K + 255) / 256;
    if (M <= 128) {
        const int bn = (N % 128 == 0) ? 128 : 64;
        const int n_tiles = N / bn;
        int splits = (sms + n_tiles / 2) / n_tiles;
        if (splits > k_tiles) splits = k_tiles;
        return finish(bn, splits, K, false);
    }
    return choose(M, N, K);
}

size_t workspace_for(int M, int N, const Schedule &s) {
    if (s.splits <= 1 || s.cluster) return 0;
    const size_t tiles = static_cast<size_t>((M + 127) / 128) * (N / s.block_n);
    const size_t tickets = (tiles * 4 + 255) / 256 * 256;
    return tickets + static_cast<size_t>(s.splits) * M * N * sizeof(float);
}

nvfp4_status gemm_impl(const nvfp4_tensor *A, const nvfp4_tensor *W, int M, int N, int K, nvfp4_epilogue epi,
                       const void *bias, const void *residual, int ldr, void *out_bf16, int ldo, uint8_t *out_codes,
                       uint8_t *out_sf, float out_global_scale, void *workspace, size_t ws_bytes, int block_n,
                       int splits, cudaStream_t stream) {
    if (A == nullptr || W == nullptr) return NVFP4_ERR_INVALID_ARG;
    if (M < 0 || N <= 0 || K <= 0) return NVFP4_ERR_INVALID_ARG;
    if (A->rows != M || W->rows != N || A->K != K || W->K != K) return NVFP4_ERR_INVALID_ARG;
    if (static_cast<int>(epi) < 0 || static_cast<int>(epi) > 5) return NVFP4_ERR_INVALID_ARG;
    if (K % 32 != 0 || N % 64 != 0) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (!scale_ok(A->global_scale) || !scale_ok(W->global_scale)) return NVFP4_ERR_INVALID_ARG;
    if (M == 0) return NVFP4_OK;  // nothing to read or write
    const bool fp4_out = (epi == NVFP4_EPI_BIAS_GELU || epi == NVFP4_EPI_GEGLU);
    const bool need_bias = (epi == NVFP4_EPI_BIAS || epi == NVFP4_EPI_BIAS_RESIDUAL || epi == NVFP4_EPI_BIAS_GELU);
    const bool need_res = (epi == NVFP4_EPI_RESIDUAL || epi == NVFP4_EPI_BIAS_RESIDUAL);
    if (need_bias && bias == nullptr) return NVFP4_ERR_INVALID_ARG;
    if (need_res && (residual == nullptr || ldr < N)) return NVFP4_ERR_INVALID_ARG;
    if (need_res && ldr % 8 != 0) return NVFP4_ERR_MISALIGNED;
    if (fp4_out) {
        if (out_codes == nullptr || out_sf == nullptr || !scale_ok(out_global_scale)) return NVFP4_ERR_INVALID_ARG;
        if (!aligned16(out_codes) || !aligned16(out_sf)) return NVFP4_ERR_MISALIGNED;
    } else {
        if (out_bf16 == nullptr || ldo < N) return NVFP4_ERR_INVALID_ARG;
        if (ldo % 8 != 0 || !aligned16(out_bf16)) return NVFP4_ERR_MISALIGNED;
    }
    if (A->codes == nullptr || A->sf == nullptr || W->codes == nullptr || W->sf == nullptr)
        return NVFP4_ERR_INVALID_ARG;
    if (!aligned16(A->codes) || !aligned16(A->sf) || !aligned16(W->codes) || !aligned16(W->sf))
        return NVFP4_ERR_MISALIGNED;
    if ((bias && !aligned16(bias)) || (need_res && !aligned16(residual))) return NVFP4_ERR_MISALIGNED;
    nvfp4_status st = check_device();
    if (st != NVFP4_OK) return st;

    Schedule sc;
    if (block_n == 0 && splits == 0) {
        sc = choose(M, N, K);
    } else if (block_n == 0 && splits == -1) {
        sc = choose_workspace(M, N, K);
    } else {
        if (block_n != 64 && block_n != 128 && block_n != 256) return NVFP4_ERR_INVALID_ARG;
        if (N % block_n != 0 || splits == 0) return NVFP4_ERR_UNSUPPORTED_SHAPE;
        // splits < 0: reduce -splits partials through the workspace instead of a cluster
        sc = finish(block_n, splits < 0 ? -splits : splits, K, splits > 0);
        if (sc.cluster && M > 128) sc = finish(block_n, sc.splits, K, false);
    }
    const size_t need = workspace_for(M, N, sc);
    if (need > 0) {
        if (workspace == nullptr || ws_bytes < need) return NVFP4_ERR_WORKSPACE;
        if (!aligned16(workspace)) return NVFP4_ERR_MISALIGNED;
    }

    GemmArgs p = {};
    p.M = M;
    p.N = N;
    p.K = K;
    p.k_atoms = (K + 63) / 64;
    p.k_tiles = (K + 255) / 256;
    p.kt_per_split = sc.kt_per_split;
    p.splits = sc.splits;
    p.cluster = sc.cluster ? 1 : 0;
    p.n_tiles = N / sc.block_n;
    p.a_box_rows = static_cast<uint32_t>(M >= 128 ? 128 : (M + 7) / 8 * 8);
    p.sfa = A->sf;
    p.sfb = W->sf;
    p.alpha = A->global_scale * W->global_scale;
    p.epi = static_cast<int>(epi);
    p.bias = static_cast<const uint16_t *>(bias);
    p.residual = static_cast<const uint16_t *>(residual);
    p.ldr = ldr;
    p.out = static_cast<uint16_t *>(out_bf16);
    p.ldo = ldo;
    p.out_codes = out_codes;
    p.out_sf = out_sf;
    p.g_out = out_global_scale;
    if (need > 0) {
        const size_t tiles = static_cast<size_t>((M + 127) / 128) * p.n_tiles;
        p.tickets = static_cast<uint32_t *>(workspace);
        p.partials = reinterpret_cast<float *>(static_cast<uint8_t *>(workspace) + (tiles * 4 + 255) / 256 * 256);
    }
    const size_t ctas = static_cast<size_t>(p.n_tiles) * ((M + 127) / 128) * p.splits;
    if (g_trace != nullptr && g_trace_cursor + 8 * ctas <= g_trace_words) {
        p.trace = g_trace + g_trace_cursor;
        g_trace_cursor += 8 * ctas;
    }
    CUtensorMap ta, tb;
    if (!make_code_map(&ta, A->codes, M, K / 2, static_cast<int>(p.a_box_rows)) ||
        !make_code_map(&tb, W->codes, N, K / 2, sc.block_n))
        return NVFP4_ERR_CUDA;
    cudaError_t e = launch_gemm(ta, tb, p, sc.block_n, stream);
    if (e == cudaSuccess) e = cudaGetLastError();
    return from_cuda(e);
}

nvfp4_status norm_impl(const void *x, nvfp4_in_dtype dt, int M, int K, int ldx, nvfp4_norm kind, const void *gamma,
                       const void *beta, const void *mod_scale, const void *mod_shift, float eps, float g,
                       uint8_t *codes, uint8_t *sf, float *y_out, cudaStream_t stream) {
    if (M < 0 || K <= 0) return NVFP4_ERR_INVALID_ARG;
    if (dt != NVFP4_IN_BF16 && dt != NVFP4_IN_FP32) return NVFP4_ERR_INVALID_ARG;
    if (static_cast<int>(kind) < 0 || static_cast<int>(kind) > 4) return NVFP4_ERR_INVALID_ARG;
    if (K % 16 != 0 || K > (dt == NVFP4_IN_FP32 ? 16384 : 32768)) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (M == 0) return NVFP4_OK;  // nothing to read or write
    if (x == nullptr || ldx < K) return NVFP4_ERR_INVALID_ARG;
    if (!(eps >= 0.0f) || !std::isfinite(eps)) return NVFP4_ERR_INVALID_ARG;
    if (y_out == nullptr) {
        if (codes == nullptr || sf == nullptr || !scale_ok(g)) return NVFP4_ERR_INVALID_ARG;
        if (!aligned16(codes) || !aligned16(sf)) return NVFP4_ERR_MISALIGNED;
    } else if (!aligned16(y_out)) {
        return NVFP4_ERR_MISALIGNED;
    }
    if (!aligned16(x) || ldx % (dt == NVFP4_IN_FP32 ? 4 : 8) != 0) return NVFP4_ERR_MISALIGNED;
    for (const void *pp : {gamma, beta, mod_scale, mod_shift})
        if (pp != nullptr && !aligned16(pp)) return NVFP4_ERR_MISALIGNED;
    nvfp4_status st = check_device();
    if (st != NVFP4_OK) return st;
    NormArgs a = {};
    a.x = x;
    a.M = M;
    a.K = K;
    a.ldx = ldx;
    a.kind = static_cast<int>(kind);
    a.gamma = static_cast<const uint16_t *>(gamma);
    a.beta = static_cast<const uint16_t *>(beta);
    a.scale = static_cast<const uint16_t *>(mod_scale);
    a.shift = static_cast<const uint16_t *>(mod_shift);
    a.eps = eps;
    a.g = g;
    a.codes = codes;
    a.sf = sf;
    a.y_out = y_out;
    cudaError_t e = launch_norm_quant(a, dt == NVFP4_IN_FP32, stream);
    if (e == cudaSuccess) e = cudaGetLastError();
    return from_cuda(e);
}

}  // namespace

extern "C" {

nvfp4_status nvfp4_probe(void) {
    nvfp4_status st = check_device();
    if (st != NVFP4_OK) return st;
    // the kernels of this library must load on the device
    if (probe_norm_kernels() != cudaSuccess || probe_gemm_kernels() != cudaSuccess) {
        cudaGetLastError();
        return NVFP4_ERR_UNSUPPORTED_DEVICE;
    }
    return encode_fn() != nullptr ? NVFP4_OK : NVFP4_ERR_CUDA;
}

const char *nvfp4_status_string(nvfp4_status s) {
    switch (s) {
    case NVFP4_OK: return "ok";
    case NVFP4_ERR_INVALID_ARG: return "invalid argument";
    case NVFP4_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
    case NVFP4_ERR_MISALIGNED: return "misaligned pointer or leading dimension";
    case NVFP4_ERR_WORKSPACE: return "workspace missing or too small";
    case NVFP4_ERR_UNSUPPORTED_DEVICE: return "unsupported device (needs sm_100)";
    case NVFP4_ERR_CUDA: return "CUDA error";
    case NVFP4_ERR_TIMEOUT: return "device wait timed out";
    }
    return "unknown status";
}

size_t nvfp4_sf_bytes(int rows, int K) {
    if (rows < 0 || K < 0) return 0;
    return static_cast<size_t>((rows + 127) / 128) * ((K + 63) / 64) * 512;
}

size_t nvfp4_sf_offset(int row, int kblk, int K) {
    const size_t k_atoms = static_cast<size_t>((K + 63) / 64);
    const size_t atom = static_cast<size_t>(row / 128) * k_atoms + static_cast<size_t>(kblk / 4);
    return atom * 512 + static_cast<size_t>(row % 32) * 16 + static_cast<size_t>((row % 128) / 32) * 4 +
           static_cast<size_t>(kblk % 4);
}

nvfp4_status nvfp4_sf_zero(uint8_t *sf, int rows, int K, nvfp4_stream_t stream) {
    if (sf == nullptr || rows < 0 || K < 0) return NVFP4_ERR_INVALID_ARG;
    return from_cuda(cudaMemsetAsync(sf, 0, nvfp4_sf_bytes(rows, K), stream));
}

size_t nvfp4_gemm_workspace_bytes(int M, int N, int K) {
    if (M <= 0 || N <= 0 || K <= 0 || N % 64 != 0) return 0;
    return workspace_for(M, N, choose(M, N, K));
}

size_t nvfp4_gemm_workspace_bytes_ex(int M, int N, int K, int block_n, int splits) {
    if (M <= 0 || N <= 0 || K <= 0) return 0;
    if (block_n == 0 && splits == 0) return nvfp4_gemm_workspace_bytes(M, N, K);
    if (block_n == 0 && splits == -1) return N % 64 ? 0 : workspace_for(M, N, choose_workspace(M, N, K));
    if (block_n <= 0 || N % block_n != 0 || splits == 0) return 0;
    Schedule sc = finish(block_n, splits < 0 ? -splits : splits, K, splits > 0);
    if (sc.cluster && M > 128) sc = finish(block_n, sc.splits, K, false);
    return workspace_for(M, N, sc);
}

nvfp4_status nvfp4_set_gemm_trace(unsigned long long *buf, size_t words) {
    g_trace = buf;
    g_trace_words = buf ? words : 0;
    g_trace_cursor = 0;
    return NVFP4_OK;
}

nvfp4_status nvfp4_get_device_status(nvfp4_stream_t stream) {
    uint32_t v = 0;
    if (read_and_clear_device_status(stream, &v) != cudaSuccess) return NVFP4_ERR_CUDA;
    return v == 0 ? NVFP4_OK : NVFP4_ERR_TIMEOUT;
}

nvfp4_status nvfp4_quantize_norm(const void *x, nvfp4_in_dtype dt, int M, int K, int ldx, nvfp4_norm kind,
                                 const void *gamma, const void *beta, const void *mod_scale, const void *mod_shift,
                                 float eps, float global_scale, uint8_t *codes, uint8_t *sf, nvfp4_stream_t stream) {
    return norm_impl(x, dt, M, K, ldx, kind, gamma, beta, mod_scale, mod_shift, eps, global_scale, codes, sf,
                     nullptr, stream);
}

nvfp4_status nvfp4_norm_f32(const void *x, nvfp4_in_dtype dt, int M, int K, int ldx, nvfp4_norm kind, const void *gamma,
                        const void *beta, const void *mod_scale, const void *mod_shift, float eps, float *y,
                        nvfp4_stream_t stream) {
    if (y == nullptr) return NVFP4_ERR_INVALID_ARG;
    return norm_impl(x, dt, M, K, ldx, kind, gamma, beta, mod_scale, mod_shift, eps, 1.0f, nullptr, nullptr, y,
                     stream);
}

nvfp4_status nvfp4_quantize_weight(const void *w_bf16, int N, int K, int ldw, int interleave_gate_up, uint8_t *codes,
                                   uint8_t *sf, float *global_scale_out, void *scratch, nvfp4_stream_t stream) {
    if (w_bf16 == nullptr || codes == nullptr || sf == nullptr || global_scale_out == nullptr || scratch == nullptr)
        return NVFP4_ERR_INVALID_ARG;
    if (N <= 0 || K <= 0 || ldw < K) return NVFP4_ERR_INVALID_ARG;
    if (K % 16 != 0 || K > 32768) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (interleave_gate_up && N % 2 != 0) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (!aligned16(w_bf16) || !aligned16(codes) || !aligned16(sf) || !aligned16(scratch) || ldw % 8 != 0)
        return NVFP4_ERR_MISALIGNED;
    nvfp4_status st = check_device();
    if (st != NVFP4_OK) return st;
    uint32_t *amax = static_cast<uint32_t *>(scratch);
    cudaError_t e = launch_weight_amax(static_cast<const uint16_t *>(w_bf16), N, K, ldw, amax, stream);
    if (e != cudaSuccess) return NVFP4_ERR_CUDA;
    NormArgs a = {};
    a.x = w_bf16;
    a.M = N;
    a.K = K;
    a.ldx = ldw;
    a.kind = NVFP4_NORM_NONE;
    a.eps = 0.0f;
    a.g = 1.0f;
    a.amax_bits = amax;
    a.interleave = interleave_gate_up ? 1 : 0;
    a.codes = codes;
    a.sf = sf;
    e = launch_norm_quant(a, false, stream);
    if (e == cudaSuccess) e = cudaGetLastError();
    if (e != cudaSuccess) return NVFP4_ERR_CUDA;
    uint32_t bits = 0;
    e = cudaMemcpyAsync(&bits, amax, sizeof(bits), cudaMemcpyDeviceToHost, stream);
    if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
    if (e != cudaSuccess) return NVFP4_ERR_CUDA;
    float am;
    std::memcpy(&am, &bits, sizeof am);
    *global_scale_out = (am == 0.0f) ? 1.0f : am / 2688.0f;
    return NVFP4_OK;
}

nvfp4_status nvfp4_gemm(const nvfp4_tensor *A, const nvfp4_tensor *W, int M, int N, int K, nvfp4_epilogue epi,
                        const void *bias, const void *residual, int ldr, void *out_bf16, int ldo, uint8_t *out_codes,
                        uint8_t *out_sf, float out_global_scale, void *workspace, size_t ws_bytes,
                        nvfp4_stream_t stream) {
    return gemm_impl(A, W, M, N, K, epi, bias, residual, ldr, out_bf16, ldo, out_codes, out_sf, out_global_scale,
                     workspace, ws_bytes, 0, 0, stream);
}

nvfp4_status nvfp4_gemm_noalloc(const nvfp4_tensor *A, const nvfp4_tensor *W, int M, int N, int K,
                                nvfp4_epilogue epi, const void *bias, const void *residual, int ldr,
                                void *out_bf16, int ldo, uint8_t *out_codes, uint8_t *out_sf,
                                float out_global_scale, nvfp4_stream_t stream) {
    size_t need = 0;
    if (A != nullptr && W != nullptr && M > 0 && N > 0 && K > 0 && N % 64 == 0)
        need = workspace_for(M, N, choose_workspace(M, N, K));
    void *ws = nullptr;
    size_t ws_bytes = 0;
    if (need > 0) {
        const nvfp4_status st = check_device();
        if (st != NVFP4_OK) return st;
        if (noalloc_scratch(&ws, &ws_bytes) != cudaSuccess) return NVFP4_ERR_CUDA;
        if (need > ws_bytes) return NVFP4_ERR_WORKSPACE;  // shape needs more than the fixed scratch
        // the split-K tickets must start at zero; the previous call's contents are still there
        const size_t tiles = static_cast<size_t>((M + 127) / 128) * (N / choose_workspace(M, N, K).block_n);
        if (cudaMemsetAsync(ws, 0, (tiles * 4 + 255) / 256 * 256, stream) != cudaSuccess) return NVFP4_ERR_CUDA;
    }
    return gemm_impl(A, W, M, N, K, epi, bias, residual, ldr, out_bf16, ldo, out_codes, out_sf, out_global_scale, ws,
                     ws_bytes, 0, -1, stream);
}

nvfp4_status nvfp4_gemm_ex(const nvfp4_tensor *A, const nvfp4_tensor *W, int M, int N, int K, nvfp4_epilogue epi,
                           const void *bias, const void *residual, int ldr, void *out_bf16, int ldo,
                           uint8_t *out_codes, uint8_t *out_sf, float out_global_scale, void *workspace,
                           size_t ws_bytes, int block_n, int splits, nvfp4_stream_t stream) {
    return gemm_impl(A, W, M, N, K, epi, bias, residual, ldr, out_bf16, ldo, out_codes, out_sf, out_global_scale,
                     workspace, ws_bytes, block_n, splits, stream);
}

}  // extern "C"
