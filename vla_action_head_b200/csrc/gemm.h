// gemm.h — internal interface between the C ABI (api.cu) and the GEMM kernel (gemm.cu).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cstddef>
#include <cstdint>

namespace nvfp4 {

// Host-side caches that hold per-device state (addresses, function attributes) have one
// entry per device index below this bound.
constexpr int kMaxDevices = 64;

// Raises `func`'s dynamic shared-memory limit to `bytes` on the current device, once per
// device (the attribute belongs to the device's context; `done` has kMaxDevices entries).
// Safe to call from several host threads: a race only repeats the idempotent call.
cudaError_t set_smem_limit_once(const void *func, int bytes, std::atomic<bool> *done);

enum { kEpiNone = 0, kEpiBias = 1, kEpiResidual = 2, kEpiBiasResidual = 3, kEpiBiasGelu = 4, kEpiGeglu = 5 };

struct GemmArgs {
    int M, N, K;
    int k_atoms;       // ceil(K / 64): scale atoms per 128-row group
    int k_tiles;       // ceil(K / 256): pipeline K tiles
    int kt_per_split;  // K tiles per split (persistent kernel with 2 splits: K tiles of split 0)
    int splits;
    int cluster;       // 1: the splits of a tile form a cluster and reduce over DSMEM
    int n_tiles;
    uint32_t a_box_rows;  // rows per A TMA box (min(128, M rounded up to 8))
    const uint8_t *sfa;
    const uint8_t *sfb;
    float alpha;  // gA * gW
    int epi;
    const uint16_t *bias;
    const uint16_t *residual;
    int ldr;
    uint16_t *out;
    int ldo;
    uint8_t *out_codes;
    uint8_t *out_sf;
    float g_out;
    int out_rotate;     // FP4 epilogues: Hadamard-rotate each output block before quantizing
    float *partials;    // split-K: [splits, M, N] fp32 (persistent kernel: [2, tiles, 128 x BN])
    uint32_t *tickets;  // split-K: one word per output tile (persistent kernel: two)
    unsigned long long *trace;  // optional per-CTA timestamps (diagnostics), 8 words per CTA
    uint32_t *status;           // the library's device status word (persistent kernel)
};

cudaError_t launch_gemm(const CUtensorMap &ta, const CUtensorMap &tb, const GemmArgs &p, int block_n,
                        cudaStream_t s);
// CTAs that one wave of the one-tile kernel holds for the given A rows class (small: M <= 64),
// tile width and cluster size (1: no cluster), from the occupancy API; 0 if unknown.
int gemm_wave_ctas(bool small, int block_n, int cluster);

// Persistent 128 x block_n tile kernel for many rows (gemm_persistent.cu): block_n 256 or
// 128, one split or two (through the workspace).  Grid: min(tiles x splits, SMs) CTAs.
int gemm_persistent_grid(int M, int n_tiles, int splits);
cudaError_t launch_gemm_persistent(const CUtensorMap &ta, const CUtensorMap &tb, const GemmArgs &p, int block_n,
                                   cudaStream_t s);
cudaError_t probe_gemm_persistent();

// Grouped kernel (gemm_grouped.cu): independent problems, one epilogue kind, 128 x 128 tiles
// numbered problem by problem, one CTA per SM.  probs[n] and maps[2n] (A with a_box_rows-row
// boxes, W with 128-row boxes) and tab[4n + 1] (first tile of each problem and the total,
// then m_tiles, k_tiles, k_atoms of each) in device memory.
constexpr int kGroupedMaxProblems = 256;
struct GroupedParams {
    const GemmArgs *probs;
    const CUtensorMap *maps;
    const int *tab;
    int n_probs;
    int total_tiles;
    uint32_t *status;
    unsigned long long *trace;
};
cudaError_t launch_gemm_grouped(const GroupedParams &p, int epi, int grid, cudaStream_t s);
cudaError_t probe_gemm_grouped();

// Device address and size of the library-owned split-K workspace used by
// nvfp4_gemm_noalloc (looked up once per device; allocation-free).
cudaError_t noalloc_scratch(void **ptr, size_t *bytes);

// Programmatic dependent launch for this library's kernels: on unless NVFP4_PDL=0.
bool pdl_enabled();

// Device address of the library's status word (for kernels in other translation units).
cudaError_t device_status_address(uint32_t **p);

// Reads the device status word and clears it (after synchronising `s`).
cudaError_t read_and_clear_device_status(cudaStream_t s, uint32_t *out);

}  // namespace nvfp4
