// api.cu — the C ABI declared in include/nvfp4.h: argument validation, schedule choice,
// TMA descriptor encoding and kernel launches.  No entry point allocates device memory,
// and only nvfp4_quantize_weight / nvfp4_get_device_status synchronise.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <vector>

#include "../../include/nvfp4.h"
#include "gemm.h"
#include "norm.h"

namespace nvfp4 {
// mma_rate.cu: one CTA issues `ksteps` K steps of block-scaled MMAs (mode 0) or of scale
// copies + MMAs (mode 1) at width n; out = issue cycles, completion cycles, timeout flag.
cudaError_t run_mma_rate(int n, int mode, int ksteps, unsigned long long out[3]);
}  // namespace nvfp4

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

thread_local cudaError_t g_last_cuda_error = cudaSuccess;  // for nvfp4_last_cuda_error_string

nvfp4_status from_cuda(cudaError_t e) {
    if (e == cudaSuccess) return NVFP4_OK;
    g_last_cuda_error = e;
    return NVFP4_ERR_CUDA;
}

// The driver's tensor-map encoder, looked up once (host threads racing on the first call
// each look it up and store the same pointer).
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static std::atomic<PFN_cuTensorMapEncodeTiled_v12000> fn{nullptr};
    PFN_cuTensorMapEncodeTiled_v12000 f = fn.load(std::memory_order_acquire);
    if (f == nullptr) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess) {
            f = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
            fn.store(f, std::memory_order_release);
        }
    }
    return f;
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

// Device address of the library's status word on the current device (looked up once).
uint32_t *status_word() {
    static std::atomic<uint32_t *> addr[kMaxDevices];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    uint32_t *a = addr[dev].load(std::memory_order_acquire);
    if (a == nullptr) {
        if (device_status_address(&a) != cudaSuccess) return nullptr;
        addr[dev].store(a, std::memory_order_release);
    }
    return a;
}

// SM count of the current device (148 on a B200), looked up once per device.
int sm_count_cached() {
    static std::atomic<int> sms[kMaxDevices];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 148;
    int n = sms[dev].load(std::memory_order_acquire);
    if (n == 0) {
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
        sms[dev].store(n, std::memory_order_release);
    }
    return n;
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

// Default schedule: the tile width and split factor (<= 8, reduced in a cluster) of least
// modelled time.  Small M is a chain of latencies; the cost is a latency model (us) fitted to schedule
// sweeps of the DiT (M = 41) and action-expert (M = 50) GEMMs on B200:
//   0.3 per K tile a CTA walks, + 0.3 + 0.004 * block_n for a split-K exchange (two cluster
//   barriers and the partial rows pushed to their owners), + the operand bytes streamed at
//   30 GB/s per CTA (up to one CTA per SM), + 2e-4 per element of a re-quantizing epilogue
//   (bias+GELU or GeGLU -> FP4) on the owner CTA.  Grids above 1.35 CTAs per SM (1.5 for a
//   re-quantizing epilogue), or above what one wave of the kernel holds, measured slow and
//   are not used; with 16 or more K tiles a grid stays within one CTA per SM (measured in
//   the DiT chain at 41 x 1536 x 6144: 6 splits on 144 CTAs 30.92 us per layer against 8
//   splits on 192 CTAs 31.24, the model's own pick).
Schedule choose(int M, int N, int K, bool fp4_out) {
    const int sms = sm_count_cached();
    const int k_tiles = (K + 255) / 256;
    const int m_tiles = (M + 127) / 128;
    if (M <= 128) {
        Schedule best{64, 1, k_tiles, false};
        double best_cost = 1e30;
        const double bytes = static_cast<double>(N) * K * (0.5 + 1.0 / 16) + static_cast<double>(M) * K * 0.5;
        for (int bn : {128, 64}) {
            if (N % bn != 0) continue;
            const int n_tiles = N / bn * m_tiles;
            for (int s = 1; s <= kMaxClusterSplits && s <= k_tiles; ++s) {
                const Schedule c = finish(bn, s, K);
                const int ctas = n_tiles * c.splits;
                if (20 * ctas > 27 * sms) continue;
                // M > 64 runs one CTA per SM: more CTAs than one wave holds (clusters must fit in
                // a GPC) run as two waves.  (At M <= 64, two CTAs share an SM; the occupancy API
                // under-counts those waves, and the measured grids fit.)
                const int wave = M > 64 ? gemm_wave_ctas(false, bn, c.splits) : 0;
                if (wave > 0 && ctas > wave) continue;
                if (fp4_out && 2 * ctas > 3 * sms) continue;
                if (k_tiles >= 16 && ctas > sms) continue;
                const int owner_rows = (std::min(M, 128) + c.splits - 1) / c.splits;
                const double cost = 0.3 * c.kt_per_split + (c.splits > 1 ? 0.3 + 0.004 * bn : 0.0) +
                                    bytes / (std::min(ctas, sms) * 30e3) +
                                    (fp4_out ? 2e-4 * owner_rows * bn : 0.0);
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

// The many-row schedule: block_n 256 or 128 = the one-CTA persistent kernel with that tile
// width and `splits` (1 or 2) K splits (through the workspace).  Cost (us): waves x K tiles
// per unit x the measured time of a K tile (0.82 at 256 columns, 0.70 at 128: the wider
// tile does twice the work for 1.17x the time), + 2.5 for the partial's round trip; splits
// must divide the K tiles.  (Four splits of the 968 x 2048 x 16384 down projection measured
// slower than two: 41.5 against 36.6 us.)
// K tiles of the first of two splits: half, plus up to 3 so that the second split (its
// partial published ~3 us after its accumulator is complete, ~0.6-0.8 us per K tile) is
// usually done before the first arrives.
int persistent_k0(int k_tiles) { return (k_tiles + 1) / 2 + std::min(3, (k_tiles - 2) / 4); }

struct ManyRows {
    int block_n;  // 0: not applicable
    int splits;
};
ManyRows choose_persistent(int M, int N, int K) {
    const int sms = sm_count_cached();
    const int m_tiles = (M + 127) / 128;
    const int k_tiles = (K + 255) / 256;
    ManyRows best{0, 1};
    double best_cost = 1e30;
    for (int bn : {256, 128}) {
        if (N % bn != 0) continue;
        const int tiles = m_tiles * (N / bn);
        for (int s : {1, 2}) {
            if (s == 2 && k_tiles < 2) continue;
            const int units = tiles * s;
            const double cost = ((units + sms - 1) / sms) * (s == 2 ? persistent_k0(k_tiles) : k_tiles) *
                                    (bn == 256 ? 0.82 : 0.70) +
                                (s > 1 ? 2.5 : 0.0);
            if (cost < best_cost) {
                best_cost = cost;
                best = ManyRows{bn, s};
            }
        }
    }
    return best;
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
    return choose(M, N, K, false);
}

// Workspace layout: a fixed region of tile counters, then the fp32 partials.  One-tile
// kernel: one ticket per tile, splits x M x N partials.  Persistent kernel (`persistent`):
// an arrival ticket and a published count per tile, splits x whole 128-row tiles x N
// partials.  The counters of every schedule sit in the same fixed region, which no
// schedule's partials overlap: a workspace reused across shapes keeps its counters zero
// (every kernel returns the counters it used to zero), so no call finds another shape's
// partial values where it expects counters.
constexpr size_t kTicketRegion = 16384;
size_t ticket_words_bytes(size_t tiles, bool persistent) { return tiles * (persistent ? 8 : 4); }

size_t workspace_for(int M, int N, const Schedule &s, bool persistent = false) {
    if (s.splits <= 1 || s.cluster) return 0;
    const size_t rows = persistent ? static_cast<size_t>((M + 127) / 128) * 128 : static_cast<size_t>(M);
    return kTicketRegion + static_cast<size_t>(s.splits) * rows * N * sizeof(float);
}

// Kernel epilogue kind of an ABI epilogue, and whether its FP4 output blocks are rotated:
// the *_RHT kinds are BIAS_GELU / GEGLU with each output block Hadamard-rotated first.
int kernel_epi(nvfp4_epilogue e) {
    return e == NVFP4_EPI_BIAS_GELU_RHT ? kEpiBiasGelu : e == NVFP4_EPI_GEGLU_RHT ? kEpiGeglu : static_cast<int>(e);
}
int epi_rotates(nvfp4_epilogue e) { return (e == NVFP4_EPI_BIAS_GELU_RHT || e == NVFP4_EPI_GEGLU_RHT) ? 1 : 0; }

// Argument checks shared by nvfp4_gemm* and the GEMM op of a program (no device access).
nvfp4_status validate_gemm(const nvfp4_tensor *A, const nvfp4_tensor *W, int M, int N, int K, nvfp4_epilogue epi,
                           const void *bias, const void *residual, int ldr, void *out_bf16, int ldo,
                           uint8_t *out_codes, uint8_t *out_sf, float out_global_scale) {
    if (A == nullptr || W == nullptr) return NVFP4_ERR_INVALID_ARG;
    if (M < 0 || N <= 0 || K <= 0) return NVFP4_ERR_INVALID_ARG;
    if (A->rows != M || W->rows != N || A->K != K || W->K != K) return NVFP4_ERR_INVALID_ARG;
    if (static_cast<int>(epi) < 0 || static_cast<int>(epi) > 7) return NVFP4_ERR_INVALID_ARG;
    if (K % 32 != 0 || N % 64 != 0) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (!scale_ok(A->global_scale) || !scale_ok(W->global_scale)) return NVFP4_ERR_INVALID_ARG;
    if (M == 0) return NVFP4_OK;
    const bool fp4_out = (kernel_epi(epi) == kEpiBiasGelu || kernel_epi(epi) == kEpiGeglu);
    const bool need_bias = (epi == NVFP4_EPI_BIAS || epi == NVFP4_EPI_BIAS_RESIDUAL || kernel_epi(epi) == kEpiBiasGelu);
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
    return NVFP4_OK;
}

nvfp4_status gemm_impl(const nvfp4_tensor *A, const nvfp4_tensor *W, int M, int N, int K, nvfp4_epilogue epi,
                       const void *bias, const void *residual, int ldr, void *out_bf16, int ldo, uint8_t *out_codes,
                       uint8_t *out_sf, float out_global_scale, void *workspace, size_t ws_bytes, int block_n,
                       int splits, cudaStream_t stream) {
    nvfp4_status st = validate_gemm(A, W, M, N, K, epi, bias, residual, ldr, out_bf16, ldo, out_codes, out_sf,
                                    out_global_scale);
    if (st != NVFP4_OK || M == 0) return st;  // M == 0: nothing to read or write
    st = check_device();
    if (st != NVFP4_OK) return st;

    Schedule sc;
    int persistent_bn = 0;  // > 0: the persistent kernel with this tile width
    ManyRows many{0, 1};
    if (block_n == 0 && splits == 0 && M > 128 && (many = choose_persistent(M, N, K)).block_n > 0) {
        persistent_bn = many.block_n;
        sc = finish(persistent_bn, many.splits, K, false);
    } else if (block_n == 0 && splits == 0) {
        sc = choose(M, N, K, kernel_epi(epi) == kEpiBiasGelu || kernel_epi(epi) == kEpiGeglu);
    } else if (block_n == 0 && splits == -1) {
        sc = choose_workspace(M, N, K);
    } else {
        if (block_n != 64 && block_n != 128 && block_n != 256) return NVFP4_ERR_INVALID_ARG;
        if (N % block_n != 0 || splits == 0) return NVFP4_ERR_UNSUPPORTED_SHAPE;
        // splits < 0: reduce -splits partials through the workspace instead of a cluster
        sc = finish(block_n, splits < 0 ? -splits : splits, K, splits > 0);
        if (sc.cluster && M > 128) sc = finish(block_n, sc.splits, K, false);
    }
    const size_t need = workspace_for(M, N, sc, persistent_bn > 0);
    if (need > 0) {
        const size_t tiles = static_cast<size_t>((M + 127) / 128) * (N / sc.block_n);
        if (ticket_words_bytes(tiles, persistent_bn > 0) > kTicketRegion) return NVFP4_ERR_UNSUPPORTED_SHAPE;
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
    if (persistent_bn > 0) {
        p.splits = many.splits;
        p.kt_per_split = many.splits == 2 ? persistent_k0(p.k_tiles) : p.k_tiles;
    }
    p.cluster = sc.cluster ? 1 : 0;
    p.n_tiles = N / sc.block_n;
    p.a_box_rows = static_cast<uint32_t>(M >= 128 ? 128 : (M + 7) / 8 * 8);
    p.sfa = A->sf;
    p.sfb = W->sf;
    p.alpha = A->global_scale * W->global_scale;
    p.epi = kernel_epi(epi);
    p.out_rotate = epi_rotates(epi);
    p.bias = static_cast<const uint16_t *>(bias);
    p.residual = static_cast<const uint16_t *>(residual);
    p.ldr = ldr;
    p.out = static_cast<uint16_t *>(out_bf16);
    p.ldo = ldo;
    p.out_codes = out_codes;
    p.out_sf = out_sf;
    p.g_out = out_global_scale;
    if (need > 0) {
        p.tickets = static_cast<uint32_t *>(workspace);
        p.partials = reinterpret_cast<float *>(static_cast<uint8_t *>(workspace) + kTicketRegion);
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
    // default schedule for many rows: the persistent kernel; an explicit (block_n, splits)
    // request runs the one-tile-per-CTA kernel
    const bool persistent = persistent_bn > 0;
    if (persistent && (p.status = status_word()) == nullptr) return NVFP4_ERR_CUDA;
    cudaError_t e = persistent ? launch_gemm_persistent(ta, tb, p, persistent_bn, stream)
                               : launch_gemm(ta, tb, p, sc.block_n, stream);
    if (e == cudaSuccess) e = cudaGetLastError();
    return from_cuda(e);
}

struct Residual {
    const void *d = nullptr;
    int ldd = 0;
    const void *gate = nullptr;
    void *h = nullptr;
    int ldh = 0;
};

nvfp4_status norm_impl(const void *x, nvfp4_in_dtype dt, int M, int K, int ldx, nvfp4_norm kind, const void *gamma,
                       const void *beta, const void *mod_scale, const void *mod_shift, float eps, float g,
                       uint8_t *codes, uint8_t *sf, float *y_out, cudaStream_t stream, const Residual &res = {},
                       int qflags = 0) {
    if (M < 0 || K <= 0) return NVFP4_ERR_INVALID_ARG;
    if ((qflags & ~(NVFP4_QUANT_ROTATE | NVFP4_QUANT_E0M3)) != 0) return NVFP4_ERR_INVALID_ARG;
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
    if (res.d != nullptr) {
        if (dt != NVFP4_IN_BF16 || res.h == nullptr || res.ldd < K || res.ldh < K) return NVFP4_ERR_INVALID_ARG;
        if (!aligned16(res.d) || !aligned16(res.h) || res.ldd % 8 != 0 || res.ldh % 8 != 0 ||
            (res.gate != nullptr && !aligned16(res.gate)))
            return NVFP4_ERR_MISALIGNED;
    }
    nvfp4_status st = check_device();
    if (st != NVFP4_OK) return st;
    NormArgs a = {};
    a.res_d = static_cast<const uint16_t *>(res.d);
    a.ldd = res.ldd;
    a.res_gate = static_cast<const uint16_t *>(res.gate);
    a.h_out = static_cast<uint16_t *>(res.h);
    a.ldh = res.ldh;
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
    a.qflags = qflags;
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
    if (probe_norm_kernels() != cudaSuccess || probe_gemm_kernels() != cudaSuccess ||
        probe_gemm_persistent() != cudaSuccess ||
        probe_gemm_grouped() != cudaSuccess) {
        cudaGetLastError();
        return NVFP4_ERR_UNSUPPORTED_DEVICE;
    }
    return encode_fn() != nullptr ? NVFP4_OK : NVFP4_ERR_CUDA;
}

const char *nvfp4_last_cuda_error_string(void) { return cudaGetErrorString(g_last_cuda_error); }

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
    if (M > 128) {
        const ManyRows many = choose_persistent(M, N, K);
        if (many.block_n > 0) return workspace_for(M, N, finish(many.block_n, many.splits, K, false), true);
    }
    return workspace_for(M, N, choose(M, N, K, false));
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

size_t nvfp4_gemm_trace_words(int M, int N, int K, nvfp4_epilogue epi) {
    if (M <= 0 || N <= 0 || K <= 0 || N % 64 != 0) return 0;
    if (static_cast<int>(epi) < 0 || static_cast<int>(epi) > 7) return 0;
    const size_t m_tiles = static_cast<size_t>((M + 127) / 128);
    if (M > 128) {
        const ManyRows many = choose_persistent(M, N, K);
        if (many.block_n > 0) return 8 * m_tiles * static_cast<size_t>(N / many.block_n) * many.splits;
    }
    const Schedule sc = choose(M, N, K, kernel_epi(epi) == kEpiBiasGelu || kernel_epi(epi) == kEpiGeglu);
    return 8 * m_tiles * static_cast<size_t>(N / sc.block_n) * sc.splits;
}

nvfp4_status nvfp4_set_gemm_trace(unsigned long long *buf, size_t words) {
    g_trace = buf;
    g_trace_words = buf ? words : 0;
    g_trace_cursor = 0;
    return NVFP4_OK;
}

nvfp4_status nvfp4_mma_rate(int n, int mode, int ksteps, double *issue_cycles, double *complete_cycles) {
    if ((n != 64 && n != 128 && n != 256) || (mode != 0 && mode != 1) || ksteps < 1 || ksteps > 4096 ||
        issue_cycles == nullptr || complete_cycles == nullptr)
        return NVFP4_ERR_INVALID_ARG;
    nvfp4_status st = check_device();
    if (st != NVFP4_OK) return st;
    unsigned long long out[3] = {0, 0, 0};
    const cudaError_t e = run_mma_rate(n, mode, ksteps, out);
    if (e != cudaSuccess) return from_cuda(e);
    if (out[2] != 0) return NVFP4_ERR_TIMEOUT;
    *issue_cycles = static_cast<double>(out[0]) / ksteps;
    *complete_cycles = static_cast<double>(out[1]) / ksteps;
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

nvfp4_status nvfp4_quantize_norm_ex(const void *x, nvfp4_in_dtype dt, int M, int K, int ldx, nvfp4_norm kind,
                                    const void *gamma, const void *beta, const void *mod_scale, const void *mod_shift,
                                    float eps, float global_scale, int flags, uint8_t *codes, uint8_t *sf,
                                    nvfp4_stream_t stream) {
    return norm_impl(x, dt, M, K, ldx, kind, gamma, beta, mod_scale, mod_shift, eps, global_scale, codes, sf,
                     nullptr, stream, Residual{}, flags);
}

nvfp4_status nvfp4_residual_quantize_norm_ex(const void *x, const void *d, const void *gate, int M, int K, int ldx,
                                             int ldd, int ldh, nvfp4_norm kind, const void *gamma, const void *beta,
                                             const void *mod_scale, const void *mod_shift, float eps,
                                             float global_scale, int flags, void *h_out, uint8_t *codes, uint8_t *sf,
                                             nvfp4_stream_t stream) {
    if (M > 0 && d == nullptr) return NVFP4_ERR_INVALID_ARG;
    Residual r;
    r.d = d;
    r.ldd = ldd;
    r.gate = gate;
    r.h = h_out;
    r.ldh = ldh;
    return norm_impl(x, NVFP4_IN_BF16, M, K, ldx, kind, gamma, beta, mod_scale, mod_shift, eps, global_scale, codes,
                     sf, nullptr, stream, r, flags);
}

nvfp4_status nvfp4_residual_quantize_norm(const void *x, const void *d, const void *gate, int M, int K, int ldx,
                                          int ldd, int ldh, nvfp4_norm kind, const void *gamma, const void *beta,
                                          const void *mod_scale, const void *mod_shift, float eps, float global_scale,
                                          void *h_out, uint8_t *codes, uint8_t *sf, nvfp4_stream_t stream) {
    if (M > 0 && d == nullptr) return NVFP4_ERR_INVALID_ARG;
    Residual r;
    r.d = d;
    r.ldd = ldd;
    r.gate = gate;
    r.h = h_out;
    r.ldh = ldh;
    return norm_impl(x, NVFP4_IN_BF16, M, K, ldx, kind, gamma, beta, mod_scale, mod_shift, eps, global_scale, codes,
                     sf, nullptr, stream, r);
}

nvfp4_status nvfp4_norm_f32(const void *x, nvfp4_in_dtype dt, int M, int K, int ldx, nvfp4_norm kind, const void *gamma,
                        const void *beta, const void *mod_scale, const void *mod_shift, float eps, float *y,
                        nvfp4_stream_t stream) {
    if (y == nullptr) return NVFP4_ERR_INVALID_ARG;
    return norm_impl(x, dt, M, K, ldx, kind, gamma, beta, mod_scale, mod_shift, eps, 1.0f, nullptr, nullptr, y,
                     stream);
}

static nvfp4_status quantize_weight_impl(const void *w_bf16, int N, int K, int ldw, int interleave_gate_up,
                                         uint8_t *codes, uint8_t *sf, float *global_scale_out, void *scratch,
                                         int flags, cudaStream_t stream) {
    if ((flags & ~(NVFP4_QUANT_ROTATE | NVFP4_QUANT_E0M3 | NVFP4_QUANT_MSE)) != 0) return NVFP4_ERR_INVALID_ARG;
    // E0M3 weights take amax / 7 block scales; an MSE search is defined for E2M1 only
    if ((flags & NVFP4_QUANT_E0M3) && (flags & NVFP4_QUANT_MSE)) return NVFP4_ERR_INVALID_ARG;
    const bool mse = (flags & NVFP4_QUANT_MSE) != 0;
    const int rotate = (flags & NVFP4_QUANT_ROTATE) ? 1 : 0;
    const int qflags = flags & (NVFP4_QUANT_ROTATE | NVFP4_QUANT_E0M3);
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
    cudaError_t e = launch_weight_amax(static_cast<const uint16_t *>(w_bf16), N, K, ldw, rotate, amax, stream);
    if (e != cudaSuccess) return NVFP4_ERR_CUDA;
    if (mse) {
        e = launch_weight_mse(static_cast<const uint16_t *>(w_bf16), N, K, ldw, interleave_gate_up ? 1 : 0, rotate,
                              amax, codes, sf, stream);
        if (e != cudaSuccess) return NVFP4_ERR_CUDA;
    }
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
    a.qflags = qflags;
    if (!mse) {
        e = launch_norm_quant(a, false, stream);
        if (e == cudaSuccess) e = cudaGetLastError();
        if (e != cudaSuccess) return NVFP4_ERR_CUDA;
    }
    uint32_t bits = 0;
    e = cudaMemcpyAsync(&bits, amax, sizeof(bits), cudaMemcpyDeviceToHost, stream);
    if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
    if (e != cudaSuccess) return NVFP4_ERR_CUDA;
    float am;
    std::memcpy(&am, &bits, sizeof am);
    *global_scale_out = (am == 0.0f) ? 1.0f : am / ((qflags & NVFP4_QUANT_E0M3) ? 3136.0f : 2688.0f);
    return NVFP4_OK;
}

nvfp4_status nvfp4_quantize_weight(const void *w_bf16, int N, int K, int ldw, int interleave_gate_up, uint8_t *codes,
                                   uint8_t *sf, float *global_scale_out, void *scratch, nvfp4_stream_t stream) {
    return quantize_weight_impl(w_bf16, N, K, ldw, interleave_gate_up, codes, sf, global_scale_out, scratch, 0,
                                stream);
}

nvfp4_status nvfp4_quantize_weight_ex(const void *w_bf16, int N, int K, int ldw, int interleave_gate_up, int flags,
                                      uint8_t *codes, uint8_t *sf, float *global_scale_out, void *scratch,
                                      nvfp4_stream_t stream) {
    return quantize_weight_impl(w_bf16, N, K, ldw, interleave_gate_up, codes, sf, global_scale_out, scratch, flags,
                                stream);
}

nvfp4_status nvfp4_quantize_weight_mse(const void *w_bf16, int N, int K, int ldw, int interleave_gate_up,
                                       uint8_t *codes, uint8_t *sf, float *global_scale_out, void *scratch,
                                       nvfp4_stream_t stream) {
    return quantize_weight_impl(w_bf16, N, K, ldw, interleave_gate_up, codes, sf, global_scale_out, scratch,
                                NVFP4_QUANT_MSE, stream);
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
    // A call that is rejected touches nothing on the device: the arguments are checked
    // before the shared buffer's tickets are cleared.
    nvfp4_status st = validate_gemm(A, W, M, N, K, epi, bias, residual, ldr, out_bf16, ldo, out_codes, out_sf,
                                    out_global_scale);
    if (st != NVFP4_OK || M == 0) return st;
    const size_t need = workspace_for(M, N, choose_workspace(M, N, K));
    void *ws = nullptr;
    size_t ws_bytes = 0;
    if (need > 0) {
        st = check_device();
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

// ---- grouped GEMM programs -------------------------------------------------------------------
size_t nvfp4_program_bytes(int n_ops) {
    if (n_ops <= 0) return 0;
    const size_t maps = static_cast<size_t>(n_ops) * 2 * sizeof(CUtensorMap);
    const size_t probs = (static_cast<size_t>(n_ops) * sizeof(GemmArgs) + 255) / 256 * 256;
    const size_t tab = ((static_cast<size_t>(4 * n_ops + 1)) * sizeof(int) + 255) / 256 * 256;  // the tile table
    return maps + probs + tab;
}

static bool build_grouped(const nvfp4_op *ops, int n_ops, uint8_t *base, size_t maps_off, size_t ops_off,
                          size_t tab_off, nvfp4_program *prog, nvfp4_status *st);

nvfp4_status nvfp4_program_build(const nvfp4_op *ops, int n_ops, void *buffer, size_t bytes, nvfp4_program *prog) {
    if (ops == nullptr || n_ops <= 0 || buffer == nullptr || prog == nullptr) return NVFP4_ERR_INVALID_ARG;
    if (n_ops > kGroupedMaxProblems) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (bytes < nvfp4_program_bytes(n_ops)) return NVFP4_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(buffer) & 255u) != 0) return NVFP4_ERR_MISALIGNED;
    for (int i = 0; i < n_ops; ++i) {
        const nvfp4_op &o = ops[i];
        if (o.type != NVFP4_OP_GEMM) return NVFP4_ERR_UNSUPPORTED_SHAPE;  // norm ops: nvfp4_quantize_norm
        if (o.dep != NVFP4_DEP_NONE) return NVFP4_ERR_UNSUPPORTED_SHAPE;  // dependent ops: a launch chain
        if (o.epi != ops[0].epi || o.N % 128 != 0) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    }
    nvfp4_status st = check_device();
    if (st != NVFP4_OK) return st;
    const size_t maps_b = static_cast<size_t>(n_ops) * 2 * sizeof(CUtensorMap);
    const size_t probs_b = (static_cast<size_t>(n_ops) * sizeof(GemmArgs) + 255) / 256 * 256;
    nvfp4_status gst = NVFP4_OK;
    build_grouped(ops, n_ops, static_cast<uint8_t *>(buffer), 0, maps_b, maps_b + probs_b, prog, &gst);
    if (gst != NVFP4_OK) return gst;
    prog->buffer = buffer;
    prog->bytes = bytes;
    prog->n_ops = n_ops;
    prog->cluster = 1;
    prog->maps_offset = 0;
    prog->ops_offset = maps_b;
    prog->done_offset = maps_b + probs_b;
    return NVFP4_OK;
}

// A grouped GEMM (independent GEMM ops, one epilogue kind, N % 128 == 0) for the grouped
// persistent kernel: one split per tile, the weight stream kept running across problem
// boundaries.  Writes the problems' GemmArgs, their tensor maps and the tile table.
static bool build_grouped(const nvfp4_op *ops, int n_ops, uint8_t *base, size_t maps_off, size_t ops_off,
                          size_t tab_off, nvfp4_program *prog, nvfp4_status *st) {
    for (int i = 0; i < n_ops; ++i) {
        const nvfp4_op &o = ops[i];
        *st = validate_gemm(&o.A, &o.W, o.M, o.N, o.K, o.epi, o.bias, o.residual, o.ldr, o.out_bf16, o.ldo,
                            o.out_codes, o.out_sf, o.out_global_scale);
        if (*st == NVFP4_OK && o.M <= 0) *st = NVFP4_ERR_UNSUPPORTED_SHAPE;
        if (*st != NVFP4_OK) return true;
    }
    uint32_t *status = status_word();
    if (status == nullptr) {
        *st = NVFP4_ERR_CUDA;
        return true;
    }
    std::vector<GemmArgs> probs(static_cast<size_t>(n_ops));
    std::vector<CUtensorMap> maps(static_cast<size_t>(n_ops) * 2);
    std::vector<int> tab(static_cast<size_t>(4 * n_ops + 1));
    int total = 0;
    for (int i = 0; i < n_ops; ++i) {
        const nvfp4_op &o = ops[i];
        GemmArgs &p = probs[i];
        p = GemmArgs{};
        p.M = o.M;
        p.N = o.N;
        p.K = o.K;
        p.k_atoms = (o.K + 63) / 64;
        p.k_tiles = (o.K + 255) / 256;
        p.kt_per_split = p.k_tiles;
        p.splits = 1;
        p.n_tiles = o.N / 128;
        p.a_box_rows = static_cast<uint32_t>(o.M >= 128 ? 128 : (o.M + 7) / 8 * 8);
        p.sfa = o.A.sf;
        p.sfb = o.W.sf;
        p.alpha = o.A.global_scale * o.W.global_scale;
        p.epi = kernel_epi(o.epi);
        p.out_rotate = epi_rotates(o.epi);
        p.bias = static_cast<const uint16_t *>(o.bias);
        p.residual = static_cast<const uint16_t *>(o.residual);
        p.ldr = o.ldr;
        p.out = static_cast<uint16_t *>(o.out_bf16);
        p.ldo = o.ldo;
        p.out_codes = o.out_codes;
        p.out_sf = o.out_sf;
        p.g_out = o.out_global_scale;
        p.status = status;
        if (!make_code_map(&maps[2 * i], o.A.codes, o.M, o.K / 2, static_cast<int>(p.a_box_rows)) ||
            !make_code_map(&maps[2 * i + 1], o.W.codes, o.N, o.K / 2, 128)) {
            *st = NVFP4_ERR_CUDA;
            return true;
        }
        const int m_tiles = (o.M + 127) / 128;
        tab[i] = total;
        tab[n_ops + 1 + i] = m_tiles;
        tab[2 * n_ops + 1 + i] = p.k_tiles;
        tab[3 * n_ops + 1 + i] = p.k_atoms;
        total += m_tiles * p.n_tiles;
    }
    tab[n_ops] = total;
    if (cudaMemcpy(base + maps_off, maps.data(), maps.size() * sizeof(CUtensorMap), cudaMemcpyHostToDevice) !=
            cudaSuccess ||
        cudaMemcpy(base + ops_off, probs.data(), probs.size() * sizeof(GemmArgs), cudaMemcpyHostToDevice) !=
            cudaSuccess ||
        cudaMemcpy(base + tab_off, tab.data(), tab.size() * sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess) {
        *st = NVFP4_ERR_CUDA;
        return true;
    }
    const int sms = sm_count_cached();
    prog->grid = total < sms ? total : sms;
    prog->kind = 1;
    prog->epi = kernel_epi(ops[0].epi);
    prog->tiles = total;
    prog->waits = 0;
    *st = NVFP4_OK;
    return true;
}

nvfp4_status nvfp4_program_run(const nvfp4_program *prog, nvfp4_stream_t stream) {
    if (prog == nullptr || prog->buffer == nullptr || prog->n_ops <= 0) return NVFP4_ERR_INVALID_ARG;
    uint8_t *base = static_cast<uint8_t *>(prog->buffer);
    if (prog->kind == 1) {
        GroupedParams g;
        g.probs = reinterpret_cast<const GemmArgs *>(base + prog->ops_offset);
        g.maps = reinterpret_cast<const CUtensorMap *>(base + prog->maps_offset);
        g.tab = reinterpret_cast<const int *>(base + prog->done_offset);
        g.n_probs = prog->n_ops;
        g.total_tiles = prog->tiles;
        g.status = status_word();
        if (g.status == nullptr) return NVFP4_ERR_CUDA;
        g.trace = (g_trace != nullptr && g_trace_words >= static_cast<size_t>(prog->grid) * 8) ? g_trace : nullptr;
        cudaError_t e = launch_gemm_grouped(g, prog->epi, prog->grid, stream);
        if (e == cudaSuccess) e = cudaGetLastError();
        return from_cuda(e);
    }
    return NVFP4_ERR_INVALID_ARG;  // not a program this library built
}

}  // extern "C"
