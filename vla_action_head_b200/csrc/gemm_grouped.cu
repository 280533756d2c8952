// gemm_grouped.cu — grouped block-scaled NVFP4 GEMM: many independent problems (each its own
// A, W, epilogue arguments and output; one epilogue kind for all) in one persistent launch
// ("GROOT N1.7 update: Thor NVFP4 + FA4 performance tier", §What is in the tier: the 32
// per-frame cross-attention K/V projections run as NVFP4 GEMMs).
//
//   acc[m, n] = sum_k e(A_p)[m, k] sA_p[m, k/16] e(W_p)[n, k] sW_p[n, k/16]     (fp32, TMEM)
//   v = acc * gA_p * gW_p (+ bias_p[n]) (+ residual_p[m, n])  ->  bf16, or GELU/GeGLU -> FP4
//
// The problems' 128 x 128 output tiles are numbered problem by problem (m-tile fastest); one
// CTA per SM walks tiles blockIdx.x, blockIdx.x + gridDim.x, ...  The walk is one stream of
// K steps through a 6-stage ring, so a CTA's next tile (often another problem's) loads while
// the current one computes, and the epilogue of a tile overlaps the next tile's MMAs: the
// weight stream never stops for a problem boundary.  At M <= 64 per problem (the cross-KV
// projections of a 41-token context) the A box covers only the valid rows; the rows the M =
// 128 MMA reads beyond them hold finite stale bytes whose scales are the zero padding of the
// 128-row scale atom, so they add nothing.
//
// Roles (384 threads), as in gemm_persistent.cu: warp 0 producer (scale atoms on their own
// per-stage barrier, ahead of the codes), warp 1 MMA issuer, warps 2..9 epilogue, warps 10
// and 11 scale copiers (two TMEM scale slots).  A tile's problem is found by binary search in
// a shared-memory table of the problems' first tile indices.  Every wait is bounded.
#include <cuda.h>
#include <cuda_runtime.h>

#include "epilogue.cuh"
#include "gemm.h"
#include "sm100.cuh"

namespace nvfp4 {

namespace {

constexpr int kThreads = 384;
constexpr int kCopiers = 2;  // warps 10, 11
constexpr int kSfAtom = 512;
constexpr int kBN = 128;
constexpr int kStageA = 128 * 128;
constexpr int kStageB = kBN * 128;
constexpr int kOffB = kStageA;
constexpr int kOffSfa = kOffB + kStageB;
constexpr int kOffSfb = kOffSfa + 4 * kSfAtom;
constexpr int kStage = kOffSfb + 4 * kSfAtom;  // 36 KB
constexpr int kStages = 6;
constexpr int kSlots = 2;
constexpr int kOffTab = kStages * kStage;  // first[n + 1], m_tiles[n], k_tiles[n], k_atoms[n]
constexpr int kOffBar = kOffTab + (4 * kGroupedMaxProblems + 4) * 4;
// barriers: full[kStages], sf_full[kStages], empty[kStages], acc_full, acc_empty,
// sf_ready[kSlots], sf_free[kSlots]
constexpr int kOffMisc = kOffBar + (3 * kStages + 2 + 2 * kSlots) * 8;
constexpr int kSmemBytes = kOffMisc + 16 + 1024;
constexpr int kColSf = kBN;
constexpr int kSfSlot = 16 + 16;
constexpr int kTmemCols = 256;
static_assert(kStage % 1024 == 0, "stage alignment (128-byte swizzle atoms)");
static_assert(kSmemBytes <= 232448, "shared memory per CTA");
static_assert(kColSf + kSlots * kSfSlot <= kTmemCols, "tensor memory columns");

__device__ __forceinline__ bool bar_epi_and(bool v) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.and.pred q, 1, 256, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"(static_cast<uint32_t>(v))
        : "memory");
    return r != 0;
}

__device__ __forceinline__ bool drain_wait(uint32_t bar, uint32_t parity, uint32_t *status) {
    int dummy = 0;
    return mbar_wait(bar, parity, &dummy, status, kStatusTimeoutDrain);
}

// A tile of the walk: its problem, position and K extent.
struct TileRef {
    int p, m_tile, n_tile, k_tiles, k_atoms;
};

// The tables in shared memory: first[n + 1] (first tile index of each problem, then the
// total), m_tiles[n], k_tiles[n], k_atoms[n].
__device__ __forceinline__ TileRef tile_ref(const int *tab, int n, int t) {
    const int *first = tab;
    int lo = 0, hi = n - 1;  // the last problem whose first tile is <= t
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (first[mid] <= t) lo = mid;
        else hi = mid - 1;
    }
    const int local = t - first[lo], mt = tab[n + 1 + lo];
    return TileRef{lo, local % mt, local / mt, tab[2 * n + 1 + lo], tab[3 * n + 1 + lo]};
}

// Walks this CTA's K steps in order: tile i (blockIdx.x + i * gridDim.x), K tile kt.
struct StepWalk {
    const int *tab;
    int n, total, i = 0, kt = -1;
    TileRef cur{};
    __device__ bool next() {
        if (kt >= 0 && kt + 1 < cur.k_tiles) {
            ++kt;
            return true;
        }
        if (kt >= 0) ++i;
        const int t = static_cast<int>(blockIdx.x) + i * static_cast<int>(gridDim.x);
        if (t >= total) return false;
        cur = tile_ref(tab, n, t);
        kt = 0;
        return true;
    }
};

template <int EPI>
__global__ void __launch_bounds__(kThreads, 1) gemm_grouped_kernel(const GroupedParams P) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    int *tab = reinterpret_cast<int *>(smem + kOffTab);
    const uint32_t bar_full = sbase + kOffBar;
    const uint32_t bar_sfl = bar_full + 8 * kStages;
    const uint32_t bar_empty = bar_sfl + 8 * kStages;
    const uint32_t bar_accf = bar_empty + 8 * kStages;
    const uint32_t bar_acce = bar_accf + 8;
    const uint32_t bar_sfr = bar_acce + 8;
    const uint32_t bar_sff = bar_sfr + 8 * kSlots;
    volatile uint32_t *misc = reinterpret_cast<volatile uint32_t *>(smem + kOffMisc);  // [0] TMEM base, [1] abort
    volatile int *abort_flag = reinterpret_cast<volatile int *>(misc + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n = P.n_probs, total = P.total_tiles;
    const int my_tiles = static_cast<int>(blockIdx.x) < total ? (total - 1 - static_cast<int>(blockIdx.x)) / gridDim.x + 1 : 0;
    unsigned long long *trace = P.trace != nullptr ? P.trace + 8ull * blockIdx.x : nullptr;
    if (trace != nullptr && threadIdx.x == 0) trace[0] = globaltimer_ns();

    for (int j = threadIdx.x; j < 4 * n + 1; j += kThreads) tab[j] = P.tab[j];
    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(bar_full + 8 * s, 1);
            mbar_init(bar_sfl + 8 * s, 1);
            mbar_init(bar_empty + 8 * s, 1);
        }
        mbar_init(bar_accf, 1);
        mbar_init(bar_acce, 1);
        for (int j = 0; j < kSlots; ++j) {
            mbar_init(bar_sfr + 8 * j, kCopiers);
            mbar_init(bar_sff + 8 * j, 1);
        }
        misc[1] = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(const_cast<uint32_t *>(misc)), kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = misc[0];
    pdl_launch_dependents();

    if (warp == 0) {
        // ------------------------------ producer (whole warp) ------------------------------
        const uint64_t pol_w = policy_evict_first(), pol_a = policy_evict_last();
        StepWalk ww{tab, n, total}, wa{tab, n, total};
        auto nkb_of = [](const TileRef &r, int kt) { return min(4, r.k_atoms - 4 * kt); };
        auto expect_and_w = [&](int st) {
            const int s = st % kStages;
            const TileRef &r = ww.cur;
            const GemmArgs *a = P.probs + r.p;
            const uint32_t nkb = static_cast<uint32_t>(nkb_of(r, ww.kt));
            const uint32_t full = bar_full + 8 * s, sfl = bar_sfl + 8 * s, base = sbase + s * kStage;
            if (lane == 0) {
                mbar_arrive_expect_tx(sfl, 2 * nkb * kSfAtom);
                mbar_arrive_expect_tx(full, __ldg(&a->a_box_rows) * 128u + kStageB);
                const uint8_t *sfb = a->sfb;
                bulk_load(base + kOffSfb, sfb + (static_cast<size_t>(r.n_tile) * r.k_atoms + 4 * ww.kt) * kSfAtom,
                          nkb * kSfAtom, sfl, pol_w);
                tma_load_2d(base + kOffB, P.maps + 2 * r.p + 1, ww.kt * 128, r.n_tile * kBN, full, pol_w);
            }
            __syncwarp();
        };
        auto issue_a = [&](int st) {
            const int s = st % kStages;
            const TileRef &r = wa.cur;
            const GemmArgs *a = P.probs + r.p;
            const uint32_t nkb = static_cast<uint32_t>(nkb_of(r, wa.kt));
            const uint32_t full = bar_full + 8 * s, sfl = bar_sfl + 8 * s, base = sbase + s * kStage;
            if (lane == 0) {
                const uint8_t *sfa = a->sfa;
                bulk_load(base + kOffSfa, sfa + (static_cast<size_t>(r.m_tile) * r.k_atoms + 4 * wa.kt) * kSfAtom,
                          nkb * kSfAtom, sfl, pol_a);
                tma_load_2d(base, P.maps + 2 * r.p, wa.kt * 128, r.m_tile * 128, full, pol_a);
            }
            __syncwarp();
        };
        int pre = 0;
        while (pre < kStages && ww.next()) expect_and_w(pre++);
        pdl_wait();  // A and its scales may come from the previous kernel
        for (int st = 0; st < pre; ++st) {
            wa.next();
            issue_a(st);
        }
        int issued = pre;
        for (int st = pre;; ++st) {
            if (!ww.next()) break;
            wa.next();
            const int s = st % kStages, use = st / kStages;
            bool ok = true;
            if (lane == 0)
                ok = mbar_wait(bar_empty + 8 * s, (use - 1) & 1, abort_flag, P.status, kStatusTimeoutEmpty);
            if (!__shfl_sync(0xffffffffu, ok ? 1 : 0, 0)) break;
            expect_and_w(st);
            issue_a(st);
            issued = st + 1;
        }
        if (lane == 0)
            for (int st = max(0, issued - kStages); st < issued; ++st) {
                drain_wait(bar_full + 8 * (st % kStages), (st / kStages) & 1, P.status);
                drain_wait(bar_sfl + 8 * (st % kStages), (st / kStages) & 1, P.status);
            }
    } else if (warp == 1) {
        if (lane == 0) {
            // ------------------------------ MMA issuer ------------------------------
            constexpr uint32_t idesc = idesc_mxf4nvf4(128, kBN);
            int st = 0;
            for (int i = 0; i < my_tiles; ++i) {
                const TileRef r = tile_ref(tab, n, static_cast<int>(blockIdx.x) + i * static_cast<int>(gridDim.x));
                if (i > 0 && !mbar_wait(bar_acce, (i - 1) & 1, abort_flag, P.status, kStatusTimeoutAccum)) break;
                tc_fence_after();
                bool ok = true;
                for (int kt = 0; kt < r.k_tiles; ++kt, ++st) {
                    const int s = st % kStages, slot = st % kSlots;
                    if (!mbar_wait(bar_full + 8 * s, (st / kStages) & 1, abort_flag, P.status, kStatusTimeoutFull) ||
                        !mbar_wait(bar_sfr + 8 * slot, (st / kSlots) & 1, abort_flag, P.status, kStatusTimeoutFull)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const int nkb = min(4, r.k_atoms - 4 * kt);
                    const uint32_t base = sbase + s * kStage;
                    const uint32_t t_sf = tmem + kColSf + slot * kSfSlot;
                    for (int kb = 0; kb < nkb; ++kb)
                        tc_mma_mxf4nvf4(tmem, desc_kmajor_sw128(base + 32 * kb), desc_kmajor_sw128(base + kOffB + 32 * kb),
                                        idesc, t_sf + 4 * kb, t_sf + 16 + 4 * kb, (kt > 0 || kb > 0) ? 1u : 0u);
                    tc_commit(bar_empty + 8 * s);
                    tc_commit(bar_sff + 8 * slot);
                }
                tc_commit(bar_accf);  // always: completion of every MMA issued above
                if (!ok) break;
            }
        }
    } else if (warp >= 10) {
        if (lane == 0) {
            // --------------------------- scale copiers (warps 10, 11) ---------------------------
            // copier c copies k-blocks 2c and 2c + 1 of each stage (A and W atoms)
            const int c = warp - 10;
            StepWalk w{tab, n, total};
            for (int st = 0; w.next(); ++st) {
                const int s = st % kStages, slot = st % kSlots;
                if (!mbar_wait(bar_sfl + 8 * s, (st / kStages) & 1, abort_flag, P.status, kStatusTimeoutFull))
                    break;
                if (st >= kSlots && !mbar_wait(bar_sff + 8 * slot, (st / kSlots - 1) & 1, abort_flag, P.status,
                                               kStatusTimeoutFull))
                    break;
                tc_fence_after();
                const int nkb = min(4, w.cur.k_atoms - 4 * w.kt);
                const uint32_t base = sbase + s * kStage;
                const uint32_t t_sf = tmem + kColSf + slot * kSfSlot;
                for (int kb = 2 * c; kb < 2 * c + 2 && kb < nkb; ++kb) {
                    tc_cp_32x128b_warpx4(t_sf + 4 * kb, desc_sf_32x128b(base + kOffSfa + kb * kSfAtom));
                    tc_cp_32x128b_warpx4(t_sf + 16 + 4 * kb, desc_sf_32x128b(base + kOffSfb + kb * kSfAtom));
                }
                tc_commit(bar_sfr + 8 * slot);
            }
        }
    } else {
        // ------------------------------ epilogue (warps 2..9) ------------------------------
        const int q = warp & 3;
        const int half = (warp - 2) >> 2;  // which 64 of the 128 columns
        const int row = q * 32 + lane;
        const int e = threadIdx.x - 64;
        pdl_wait();  // residuals may come from the previous kernel
        for (int i = 0; i < my_tiles; ++i) {
            const TileRef r = tile_ref(tab, n, static_cast<int>(blockIdx.x) + i * static_cast<int>(gridDim.x));
            const bool got = e != 0 || mbar_wait(bar_accf, i & 1, abort_flag, P.status, kStatusTimeoutAccum);
            if (!bar_epi_and(got && *abort_flag == 0)) break;
            tc_fence_after();
            uint32_t acc[2][32];
            const uint32_t t_row = tmem + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(half * 64);
#pragma unroll
            for (int c = 0; c < 2; ++c) tmem_ld_32x32b_x32(t_row + 32 * c, acc[c]);
            tmem_ld_wait();
            tc_fence_before();
            bar_epi_and(true);
            if (e == 0) mbar_arrive(bar_acce);  // the MMA warp may start the next tile
            const GemmArgs &a = P.probs[r.p];
            const int m = r.m_tile * 128 + row;
            if (m < a.M) {
                const int n0 = r.n_tile * kBN + half * 64;
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                    float v[32];
#pragma unroll
                    for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(acc[c][j]);
                    epilogue_chunk<32, EPI>(a, m, n0 + 32 * c, v);
                }
            }
        }
    }

    // teardown
    __syncwarp();
    if (*abort_flag) {
        const uint64_t t0 = globaltimer_ns();
        while (globaltimer_ns() - t0 < 200000ull) {
        }
    }
    tc_fence_before();
    __syncthreads();
    if (trace != nullptr && threadIdx.x == 0) trace[6] = globaltimer_ns();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

template <int EPI>
cudaError_t launch_epi(const GroupedParams &p, int grid, cudaStream_t s) {
    static std::atomic<bool> attr_set[kMaxDevices];
    const cudaError_t e =
        set_smem_limit_once(reinterpret_cast<const void *>(gemm_grouped_kernel<EPI>), kSmemBytes, attr_set);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(grid));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = kSmemBytes;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl_enabled() ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, gemm_grouped_kernel<EPI>, p);
}

}  // namespace

cudaError_t launch_gemm_grouped(const GroupedParams &p, int epi, int grid, cudaStream_t s) {
    switch (epi) {
    case kEpiNone: return launch_epi<kEpiNone>(p, grid, s);
    case kEpiBias: return launch_epi<kEpiBias>(p, grid, s);
    case kEpiResidual: return launch_epi<kEpiResidual>(p, grid, s);
    case kEpiBiasResidual: return launch_epi<kEpiBiasResidual>(p, grid, s);
    case kEpiBiasGelu: return launch_epi<kEpiBiasGelu>(p, grid, s);
    case kEpiGeglu: return launch_epi<kEpiGeglu>(p, grid, s);
    default: return cudaErrorInvalidValue;
    }
}

cudaError_t probe_gemm_grouped() {
    cudaFuncAttributes fa;
    return cudaFuncGetAttributes(&fa, gemm_grouped_kernel<kEpiNone>);
}

}  // namespace nvfp4
