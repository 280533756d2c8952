// gemm_pair.cu — block-scaled NVFP4 GEMM on CTA pairs for many rows (the compute-bound
// regime, e.g. a prefill layer's gate/up projection at M = 968).
//
//   acc[m, n] = sum_k e(A)[m, k] sA[m, k/16] e(W)[n, k] sW[n, k/16]      (fp32, in TMEM)
//   v = acc * gA * gW (+ bias[n]) (+ residual[m, n])  ->  bf16, or tanh-GELU / GeGLU -> FP4
// ("GROOT N1.7 update: Thor NVFP4 + FA4 performance tier", §What is in the tier;
// "Pi0.5 Thor NVFP4 End-to-End Results", §Fused GeGLU FFN in the Decoder.)
//
// Why pairs: with one CTA per 128 x 256 tile, every K step moves 48 KB of codes through
// the SM's shared memory twice -- written by TMA, read by the tensor core -- which at the
// FP4 MMA rate is more than shared memory delivers.  A 2-CTA cluster computes a 256 x 256
// tile with tcgen05.mma.cta_group::2 (M = 256): each CTA stages its own 128 rows of A and
// one half (128 rows) of the W tile, and the MMA reads both CTAs' halves, so each SM moves
// 32 KB of codes per step for the same tensor work.
//
// Roles per CTA (512 threads, four warpgroups):
//   warp 0      producer (both CTAs): TMA loads of this CTA's A rows, its half of the W
//               rows and the scale atoms (its A rows; all 256 W rows) into a 5-stage ring.
//               Completion is counted on the LEADER's barriers; only the leader sets the
//               expected byte counts (both CTAs' bytes).
//   warp 1      TMEM allocation (both CTAs, cta_group::2); on the leader also the MMA
//               issuer: 4 x tcgen05.mma.cta_group::2 kind::mxf4nvf4 block16 per 256-wide K
//               tile; stage release and accumulator-full commits multicast to both CTAs.
//   warps 2, 3, scale copiers (leader): tcgen05.cp.cta_group::2 32x128b.warpx4, which fills
//   12..15      both CTAs' scale slots from their own shared memory.  A copy issued from one
//               thread completes ~200 cycles after the previous one (it writes both CTAs'
//               tensor memory), so a stage's 12 copies are spread over six warps.
//   warps 4..11 epilogue (both CTAs): each CTA drains its own 128 accumulator rows, hands the
//               accumulator back to the leader (one arrival per CTA), then runs the fused
//               epilogue from registers while the next tile's MMAs run.
// The copiers, producer and MMA warps need few registers: setmaxnreg moves 40 per thread
// from their two warpgroups to the two epilogue warpgroups.  The kernel is instantiated per
// epilogue kind.  Every wait is bounded (sm100.cuh).
#include <cuda.h>
#include <cuda_runtime.h>

#include "epilogue.cuh"
#include "gemm.h"
#include "sm100.cuh"

namespace nvfp4 {

namespace {

constexpr int kThreads = 512;
constexpr int kCopiers = 6;  // warps 2, 3, 12..15 of the leader
constexpr int kSfAtom = 512;
constexpr int kStageA = 128 * 128;      // this CTA's 128 A rows x 256 FP4
constexpr int kStageB = 128 * 128;      // this CTA's 128 of the tile's 256 W rows
constexpr int kStageSfa = 4 * kSfAtom;  // A scale atoms, 4 k-blocks
constexpr int kStageSfb = 8 * kSfAtom;  // W scale atoms, 2 groups of 128 rows x 4 k-blocks
constexpr int kOffB = kStageA;
constexpr int kOffSfa = kOffB + kStageB;
constexpr int kOffSfb = kOffSfa + kStageSfa;
constexpr int kStage = kOffSfb + kStageSfb;  // 38 KB
constexpr int kStages = (216 * 1024) / kStage;
constexpr int kOffBar = kStages * kStage;
constexpr int kSlots = 2;
// barriers: full[kStages], sf_full[kStages], empty[kStages], acc_full, acc_empty,
// sf_ready[kSlots], sf_free[kSlots]
constexpr int kOffMisc = kOffBar + (3 * kStages + 2 + 2 * kSlots) * 8;
constexpr int kSmemBytes = kOffMisc + 16 + 1024;  // + alignment slack
// tensor memory: accumulator columns 0..255, then kSlots scale slots of
// [A: 4 k-blocks x 4 | W: 4 k-blocks x 2 groups x 4]
constexpr int kColSf = 256;
constexpr int kSfSlot = 16 + 32;
constexpr int kTmemCols = 512;
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

// Bounded wait with cluster-scope acquire (arrivals from the peer CTA).
__device__ __forceinline__ bool mbar_wait_cluster(uint32_t bar, uint32_t parity, volatile int *abort_flag,
                                                  uint32_t *status, uint32_t why) {
    const uint64_t t0 = globaltimer_ns();
    while (true) {
        if (mbar_try_wait_cluster(bar, parity)) return true;
        if (*abort_flag) return false;
        if (globaltimer_ns() - t0 > kWaitLimitNs) {
            atomicCAS(status, static_cast<uint32_t>(kStatusOk), why);
            *abort_flag = 1;
            return false;
        }
    }
}

template <int EPI>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                     const __grid_constant__ CUtensorMap tmSa, const __grid_constant__ CUtensorMap tmSb,
                     const GemmArgs p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const uint32_t bar_full = sbase + kOffBar;
    const uint32_t bar_sfl = bar_full + 8 * kStages;
    const uint32_t bar_empty = bar_sfl + 8 * kStages;
    const uint32_t bar_accf = bar_empty + 8 * kStages;
    const uint32_t bar_acce = bar_accf + 8;
    const uint32_t bar_sfr = bar_acce + 8;          // kSlots: slot copied (an arrival per copier)
    const uint32_t bar_sff = bar_sfr + 8 * kSlots;  // kSlots: slot read by its MMAs
    volatile uint32_t *misc = reinterpret_cast<volatile uint32_t *>(smem + kOffMisc);  // [0] TMEM base, [1] abort
    volatile int *abort_flag = reinterpret_cast<volatile int *>(misc + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;
    const int pair = static_cast<int>(blockIdx.x) >> 1, pairs = static_cast<int>(gridDim.x) >> 1;
    const int m_tiles = (p.M + 255) / 256;
    const int tiles = m_tiles * p.n_tiles;
    const int k_tiles = p.k_tiles;
    const int my_tiles = pair < tiles ? (tiles - 1 - pair) / pairs + 1 : 0;
    const int steps = my_tiles * k_tiles;
    unsigned long long *trace = p.trace != nullptr ? p.trace + 8ull * blockIdx.x : nullptr;
    if (trace != nullptr && threadIdx.x == 0) trace[0] = globaltimer_ns();

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(bar_full + 8 * s, 1);
            mbar_init(bar_sfl + 8 * s, 1);
            mbar_init(bar_empty + 8 * s, 1);
        }
        mbar_init(bar_accf, 1);
        mbar_init(bar_acce, 2);  // one arrival from each CTA's epilogue
        for (int j = 0; j < kSlots; ++j) {
            mbar_init(bar_sfr + 8 * j, kCopiers);
            mbar_init(bar_sff + 8 * j, 1);
        }
        misc[1] = 0;
        fence_mbar_init();
        prefetch_tmap(&tmA);
        prefetch_tmap(&tmB);
        prefetch_tmap(&tmSa);
        prefetch_tmap(&tmSb);
    }
    if (warp == 1) {
        tmem_alloc_pair(smem_u32(const_cast<uint32_t *>(misc)), kTmemCols);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync_all();  // both CTAs' barriers exist before any remote arrival
    tc_fence_after();
    const uint32_t tmem = misc[0];
    pdl_launch_dependents();

    auto tile_of = [&](int i) { return pair + i * pairs; };

    // Registers: the epilogue warpgroups (1 and 2) take 168 per thread, the others give theirs
    // up (88): 128 x (2 x 168 + 2 x 88) = 65536, the launch's total.
    if ((warp >> 2) == 1 || (warp >> 2) == 2) {
        asm volatile("setmaxnreg.inc.sync.aligned.u32 168;" ::: "memory");
        // ------------------------------ epilogue (warps 4..11) ------------------------------
        const int q = warp & 3;            // TMEM sub-partition this warp may read
        const int half = (warp - 4) >> 2;  // which half of the 256 columns
        const int row = q * 32 + lane;
        const int e = threadIdx.x - 128;
        const uint32_t lead_acce = mapa_shared(bar_acce, 0);
        pdl_wait();  // residuals may come from the previous kernel
        for (int i = 0; i < my_tiles; ++i) {
            const int t = tile_of(i);
            const int m_tile = t % m_tiles, n_tile = t / m_tiles;
            const bool got = e != 0 || mbar_wait(bar_accf, i & 1, abort_flag, p.status, kStatusTimeoutAccum);
            if (!bar_epi_and(got && *abort_flag == 0)) break;
            tc_fence_after();
            uint32_t r[4][32];
            const uint32_t t_row = tmem + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(half * 128);
#pragma unroll
            for (int c = 0; c < 4; ++c) tmem_ld_32x32b_x32(t_row + 32 * c, r[c]);
            tmem_ld_wait();
            tc_fence_before();
            bar_epi_and(true);
            if (e == 0) mbar_arrive_remote(lead_acce);  // this CTA's rows are out of the accumulator
            const int m = m_tile * 256 + static_cast<int>(rank) * 128 + row;
            if (m < p.M) {
                const int n = n_tile * 256 + half * 128;
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    float v[32];
#pragma unroll
                    for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[c][j]);
                    epilogue_chunk<32, EPI>(p, m, n + 32 * c, v);
                }
            }
        }
    } else {
        asm volatile("setmaxnreg.dec.sync.aligned.u32 88;" ::: "memory");
        if (warp == 0) {
            // ------------------------------ producer (whole warp) ------------------------------
            const uint64_t pol = policy_evict_last();  // A and W both fit in L2 and are re-read
            const uint32_t lead_full = mapa_shared(bar_full, 0), lead_sfl = mapa_shared(bar_sfl, 0);
            auto expect = [&](int st) {
                if (leader && lane == 0) {
                    const int s = st % kStages;
                    mbar_arrive_expect_tx(bar_sfl + 8 * s, 2u * (kStageSfa + kStageSfb));
                    mbar_arrive_expect_tx(bar_full + 8 * s, 2u * (kStageA + kStageB));
                }
                __syncwarp();
            };
            // W: the scale atoms of both 128-row groups of the tile, then this CTA's half of the codes
            auto issue_w = [&](int st) {
                const int s = st % kStages, t = tile_of(st / k_tiles), kt = st % k_tiles;
                const int n_tile = t / m_tiles;
                const uint32_t base = sbase + s * kStage;
                if (lane < 2)
                    tma_load_2d_pair(base + kOffSfb + lane * 4 * kSfAtom, &tmSb, 0, (n_tile * 2 + lane) * p.k_atoms + 4 * kt,
                                     lead_sfl + 8 * s, pol);
                __syncwarp();
                if (lane == 0)
                    tma_load_2d_pair(base + kOffB, &tmB, kt * 128, n_tile * 256 + static_cast<int>(rank) * 128,
                                     lead_full + 8 * s, pol);
            };
            // A: this CTA's 128 rows (scale atoms, then codes)
            auto issue_a = [&](int st) {
                const int s = st % kStages, t = tile_of(st / k_tiles), kt = st % k_tiles;
                const int group = (t % m_tiles) * 2 + static_cast<int>(rank);
                const uint32_t base = sbase + s * kStage;
                if (lane == 0) {
                    tma_load_2d_pair(base + kOffSfa, &tmSa, 0, group * p.k_atoms + 4 * kt, lead_sfl + 8 * s, pol);
                    tma_load_2d_pair(base, &tmA, kt * 128, group * 128, lead_full + 8 * s, pol);
                }
            };
            const int pre = min(kStages, steps);
            for (int st = 0; st < pre; ++st) {
                expect(st);
                issue_w(st);
            }
            pdl_wait();  // A and its scales come from the previous kernel
            for (int st = 0; st < pre; ++st) issue_a(st);
            int issued = pre;
            for (int st = pre; st < steps; ++st) {
                const int s = st % kStages, use = st / kStages;
                bool ok = true;
                if (lane == 0)  // the stage is free in this CTA once the leader's MMAs have read it
                    ok = mbar_wait(bar_empty + 8 * s, (use - 1) & 1, abort_flag, p.status, kStatusTimeoutEmpty);
                if (!__shfl_sync(0xffffffffu, ok ? 1 : 0, 0)) break;
                expect(st);
                issue_w(st);
                issue_a(st);
                issued = st + 1;
            }
            // the leader's barriers count both CTAs' bytes: every issued stage must have landed
            // before either CTA may exit (the teardown's cluster barrier holds the peer)
            if (leader && lane == 0)
                for (int st = max(0, issued - kStages); st < issued; ++st) {
                    int dummy = 0;
                    mbar_wait(bar_full + 8 * (st % kStages), (st / kStages) & 1, &dummy, p.status, kStatusTimeoutDrain);
                    mbar_wait(bar_sfl + 8 * (st % kStages), (st / kStages) & 1, &dummy, p.status, kStatusTimeoutDrain);
                }
        } else if (warp == 1) {
            if (leader && lane == 0) {
                // ------------------------------ MMA issuer (leader) ------------------------------
                constexpr uint32_t idesc = idesc_mxf4nvf4(256, 256);
                int st = 0;
                for (int i = 0; i < my_tiles; ++i) {
                    // both CTAs' epilogues have drained the accumulator
                    if (i > 0 && !mbar_wait_cluster(bar_acce, (i - 1) & 1, abort_flag, p.status, kStatusTimeoutAccum))
                        break;
                    tc_fence_after();
                    bool ok = true;
                    for (int kt = 0; kt < k_tiles; ++kt, ++st) {
                        const int s = st % kStages, slot = st % kSlots;
                        if (!mbar_wait(bar_full + 8 * s, (st / kStages) & 1, abort_flag, p.status, kStatusTimeoutFull) ||
                            !mbar_wait(bar_sfr + 8 * slot, (st / kSlots) & 1, abort_flag, p.status, kStatusTimeoutFull)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        const uint32_t base = sbase + s * kStage;
                        const uint32_t t_sf = tmem + kColSf + slot * kSfSlot;
                        const int nkb = min(4, p.k_atoms - 4 * kt);
                        for (int kb = 0; kb < nkb; ++kb)
                            tc_mma_mxf4nvf4_pair(tmem, desc_kmajor_sw128(base + 32 * kb),
                                                 desc_kmajor_sw128(base + kOffB + 32 * kb), idesc, t_sf + 4 * kb,
                                                 t_sf + 16 + 8 * kb, (kt > 0 || kb > 0) ? 1u : 0u);
                        tc_commit_pair_mc(bar_empty + 8 * s, 0x3);  // frees the stage in both CTAs
                        tc_commit_pair(bar_sff + 8 * slot);          // and the leader's scale slot
                    }
                    tc_commit_pair_mc(bar_accf, 0x3);  // always: completion of every MMA issued above
                    if (!ok) break;
                }
            }
        } else {  // warps 2, 3, 12..15
            if (leader && lane == 0) {
                // ------------------------------ scale copiers (leader) ------------------------------
                // A stage's 12 atoms (4 k-blocks x [A, W group 0, W group 1]), numbered
                // kb * 3 + w; copier c takes the numbers c and c + 6.
                const int c = warp < 4 ? warp - 2 : warp - 10;
                for (int st = 0; st < steps; ++st) {
                    const int s = st % kStages, slot = st % kSlots, kt = st % k_tiles;
                    if (!mbar_wait(bar_sfl + 8 * s, (st / kStages) & 1, abort_flag, p.status, kStatusTimeoutFull))
                        break;
                    if (st >= kSlots && !mbar_wait(bar_sff + 8 * slot, (st / kSlots - 1) & 1, abort_flag, p.status,
                                                   kStatusTimeoutFull))
                        break;
                    tc_fence_after();
                    const int nkb = min(4, p.k_atoms - 4 * kt);
                    const uint32_t base = sbase + s * kStage;
                    const uint32_t t_sf = tmem + kColSf + slot * kSfSlot;
                    for (int u = c; u < 3 * nkb; u += kCopiers) {
                        const int kb = u / 3, w = u % 3;
                        if (w == 0)
                            tc_cp_32x128b_warpx4_pair(t_sf + 4 * kb, desc_sf_32x128b(base + kOffSfa + kb * kSfAtom));
                        else
                            tc_cp_32x128b_warpx4_pair(t_sf + 16 + 8 * kb + 4 * (w - 1),
                                                      desc_sf_32x128b(base + kOffSfb + (w - 1) * 4 * kSfAtom + kb * kSfAtom));
                    }
                    tc_commit_pair(bar_sfr + 8 * slot);  // arrives when this warp's copies have landed
                }
            }
        }
    }

    // teardown: neither CTA leaves while the other may still use its shared or tensor memory
    __syncwarp();
    if (*abort_flag) {
        // an abandoned run may leave copies or MMAs in flight: give them time to land before
        // shared and tensor memory are released
        const uint64_t t0 = globaltimer_ns();
        while (globaltimer_ns() - t0 < 200000ull) {
        }
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync_all();
    if (trace != nullptr && threadIdx.x == 0) trace[6] = globaltimer_ns();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem, kTmemCols);
    }
}

int pair_clusters() {
    static int n = 0;
    if (n == 0) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(2);
        cfg.blockDim = dim3(kThreads);
        cfg.dynamicSmemBytes = kSmemBytes;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 2;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int c = 0;
        if (cudaFuncSetAttribute(gemm_pair_kernel<kEpiNone>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 kSmemBytes) == cudaSuccess &&
            cudaOccupancyMaxActiveClusters(&c, gemm_pair_kernel<kEpiNone>, &cfg) == cudaSuccess && c > 0)
            n = c;
        else
            n = 64;
    }
    return n;
}

}  // namespace

int gemm_pair_clusters() { return pair_clusters(); }

template <int EPI>
static cudaError_t launch_epi(const CUtensorMap &ta, const CUtensorMap &tb, const CUtensorMap &tsa,
                              const CUtensorMap &tsb, const GemmArgs &p, cudaStream_t s) {
    static bool attr_set = false;
    if (!attr_set) {
        cudaError_t e =
            cudaFuncSetAttribute(gemm_pair_kernel<EPI>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
        if (e != cudaSuccess) return e;
        attr_set = true;
    }
    const int tiles = ((p.M + 255) / 256) * p.n_tiles;
    const int pairs = tiles < pair_clusters() ? tiles : pair_clusters();
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * pairs);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = kSmemBytes;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl_enabled() ? 2 : 1;
    return cudaLaunchKernelEx(&cfg, gemm_pair_kernel<EPI>, ta, tb, tsa, tsb, p);
}

cudaError_t launch_gemm_pair(const CUtensorMap &ta, const CUtensorMap &tb, const CUtensorMap &tsa,
                             const CUtensorMap &tsb, const GemmArgs &p, cudaStream_t s) {
    switch (p.epi) {
    case kEpiNone: return launch_epi<kEpiNone>(ta, tb, tsa, tsb, p, s);
    case kEpiBias: return launch_epi<kEpiBias>(ta, tb, tsa, tsb, p, s);
    case kEpiResidual: return launch_epi<kEpiResidual>(ta, tb, tsa, tsb, p, s);
    case kEpiBiasResidual: return launch_epi<kEpiBiasResidual>(ta, tb, tsa, tsb, p, s);
    case kEpiBiasGelu: return launch_epi<kEpiBiasGelu>(ta, tb, tsa, tsb, p, s);
    case kEpiGeglu: return launch_epi<kEpiGeglu>(ta, tb, tsa, tsb, p, s);
    default: return cudaErrorInvalidValue;
    }
}

cudaError_t probe_gemm_pair() {
    cudaFuncAttributes fa;
    return cudaFuncGetAttributes(&fa, gemm_pair_kernel<kEpiNone>);
}

}  // namespace nvfp4
