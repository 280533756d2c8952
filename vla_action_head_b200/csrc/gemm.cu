// gemm.cu — block-scaled NVFP4 GEMM on sm_100a tensor cores with fused epilogues.
//
//   acc[m, n] = sum_k e(A)[m, k] sA[m, k/16] e(W)[n, k] sW[n, k/16]      (fp32, in TMEM)
//   v = acc * gA * gW (+ bias[n]) (+ residual[m, n])  ->  bf16, or tanh-GELU / GeGLU -> FP4
// ("GROOT N1.7 update: Thor NVFP4 + FA4 performance tier", §What is in the tier: every DiT
// GEMM block-scaled NVFP4 with fused bf16 bias / bias+residual / bias+tanh-GELU+FP4
// epilogues; "Pi0.5 Thor NVFP4 End-to-End Results", §Half-Width Fused GeGLU Epilogue and
// §Fused GeGLU FFN in the Decoder: gelu(gate)*up on pairwise-interleaved columns, 16
// values per output scale block, GELU on the fp32 accumulator.)
//
// One CTA computes a 128 x BN output tile over one K range (split-K for small M, where the
// GEMM streams weights and needs every SM pulling them).  Warp roles:
//   warp 0      TMA producer: 2-D tiled loads of the A / W code tiles (128-byte swizzle) and
//               1-D bulk loads of their scale-factor atoms into a STAGES-deep ring; the
//               weight half of the first stages is issued before the programmatic-launch
//               wait because weights never depend on the previous kernel.
//   warp 1      tensor-memory allocation; one thread issues tcgen05.mma kind::mxf4nvf4
//               block16 (M = 128, N = BN, K = 64 each).
//   warps 2..5  until the accumulator is ready: tcgen05.cp of the scale atoms (smem -> TMEM),
//               one k-block per warp, into two scale slots; then the epilogue:
//               tcgen05.ld of the fp32 accumulator (one row per thread), then
//               either the fused epilogue directly, or split-K partials to the workspace
//               with an arrival ticket; the last CTA of a tile reduces the partials in
//               split order (deterministic) and runs the epilogue.
// Every wait is bounded (see sm100.cuh); an expired wait records a status and the CTA
// unwinds: copies and MMAs in flight are drained, tensor memory is freed.
#include <cuda.h>
#include <cuda_bf16.h>
#include <atomic>
#include <cstdlib>
#include <type_traits>
#include <cuda_runtime.h>

#include "epilogue.cuh"
#include "gemm.h"
#include "norm.h"
#include "quant.cuh"
#include "sm100.cuh"

namespace nvfp4 {

__device__ uint32_t g_device_status = 0;

// Split-K workspace of nvfp4_gemm_noalloc: lives in the library's own device memory, so
// that entry point never allocates.  Every GPU that loads the library keeps these bytes
// until the process exits.
constexpr size_t kNoAllocScratchBytes = size_t(4) << 20;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

namespace {

constexpr int kThreads = 192;
constexpr int kSfAtom = 512;        // 128 rows x 4 scale blocks

template <int BN>
struct Cfg {
    static constexpr int kSfbGroups = BN >= 128 ? BN / 128 : 1;
    static constexpr int kBBytes = BN * 128;
    static constexpr int kSfaBytes = 4 * kSfAtom;
    static constexpr int kSfbBytes = kSfbGroups * 4 * kSfAtom;
    // tensor-memory columns: the accumulator, then kSlots scale slots of [A: 4 k-blocks x 4 |
    // W: 4 k-blocks x groups x 4]; K tile j uses slot j % kSlots.  Up to 128 columns wide, as
    // many slots as fit in 256 columns (6 at BN 64, 4 at BN 128): a CTA with that many K
    // tiles or fewer never waits for a slot, so the copies of every tile start as soon as it
    // lands.  (256 columns keep two CTAs per SM: the next kernel's CTAs allocate while this
    // one runs.)
    static constexpr int kColSf = BN;
    static constexpr int kSfSlot = 16 + 16 * kSfbGroups;
    static constexpr int kSlots = BN <= 128 ? (256 - BN) / kSfSlot : 2;
    static constexpr int kColsUsed = BN + kSlots * kSfSlot;
    static constexpr int kTmemCols = kColsUsed <= 32 ? 32 : kColsUsed <= 64 ? 64 : kColsUsed <= 128 ? 128
                                     : kColsUsed <= 256 ? 256 : 512;
};

// Shared-memory plan: STAGES x [A tile] then STAGES x [W tile], then the scale atoms.
// SMALL_A (M <= 64): an A stage holds 64 rows (8 KB).  The M = 128 MMA still reads a 16 KB
// window from the stage base; its rows 64..127 fall on the next buffer (finite E2M1 bytes),
// and their scales are the zero padding of the 128-row scale atom, so they add nothing.
template <int BN, int STAGES, bool SMALL_A>
struct Smem {
    static constexpr int kA = SMALL_A ? 8192 : 16384;
    static constexpr int kOffA = 0;
    static constexpr int kOffB = kOffA + STAGES * kA;
    static constexpr int kOffSfa = kOffB + STAGES * Cfg<BN>::kBBytes;
    static constexpr int kOffSfb = kOffSfa + STAGES * Cfg<BN>::kSfaBytes;
    // split-K partial rows for the cluster reduction (owner slots: S x ceil(rows / S) rows,
    // S <= 8).  At SMALL_A and BN 64 they have a region of their own, so a CTA may push its
    // partials while its peers' MMAs still read their stages; otherwise they reuse the stages.
    static constexpr int kRedLd = BN + 4;  // floats per row (padded against bank conflicts)
    static constexpr bool kSepRed = SMALL_A && BN == 64;
    static constexpr int kRedBytes = ((SMALL_A ? 64 : 128) + 8) * kRedLd * 4;
    static constexpr int kOffRed = kSepRed ? kOffSfb + STAGES * Cfg<BN>::kSfbBytes : 0;
    static constexpr int kOffBar = kOffSfb + STAGES * Cfg<BN>::kSfbBytes + (kSepRed ? kRedBytes : 0);
    // barriers: full[STAGES], empty[STAGES], acc, sf_ready[kSlots], sf_free[kSlots]
    static constexpr int kOffMisc = kOffBar + (2 * STAGES + 1 + 2 * Cfg<BN>::kSlots) * 8;
    static constexpr int kBytes = kOffMisc + 16 + 1024;  // + alignment slack
    static_assert(kSepRed || kRedBytes <= kOffBar, "reduction slots must fit the stages");
    static_assert(!SMALL_A || kBytes <= 113 * 1024, "two CTAs per SM");
    static_assert(Cfg<BN>::kBBytes >= 8192, "SMALL_A window overlaps the W tile");
};

__device__ __forceinline__ void named_barrier_epi() {
    asm volatile("bar.sync 1, 128;" ::: "memory");
}

// bounded wait that ignores the abort flag (used while draining before teardown)
__device__ __forceinline__ bool drain_wait(uint32_t bar, uint32_t parity) {
    int dummy = 0;
    return mbar_wait(bar, parity, &dummy, &g_device_status, kStatusTimeoutDrain);
}

// SMALL_A kernels are sized (shared memory, TMEM, registers) for two resident CTAs per SM.
template <int BN, int STAGES, bool SMALL_A>
__global__ void __launch_bounds__(kThreads, SMALL_A ? 2 : 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                const GemmArgs p) {
    using C = Cfg<BN>;
    using S = Smem<BN, STAGES, SMALL_A>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const uint32_t bar_full = sbase + S::kOffBar;             // STAGES barriers
    const uint32_t bar_empty = bar_full + STAGES * 8;         // STAGES barriers
    const uint32_t bar_acc = bar_empty + STAGES * 8;          // 1 barrier
    const uint32_t bar_sfr = bar_acc + 8;                     // kSlots: scale slot copied (4 arrivals)
    const uint32_t bar_sff = bar_sfr + 8 * C::kSlots;         // kSlots: scale slot read by its MMAs
    volatile uint32_t *misc = reinterpret_cast<volatile uint32_t *>(smem + S::kOffMisc);
    // misc[0] = tensor-memory base, misc[1] = abort flag, misc[2] = split-K ticket,
    // misc[3] = accumulator-valid decision of the epilogue warps
    volatile int *abort_flag = reinterpret_cast<volatile int *>(misc + 1);

    const unsigned long long t_entry = globaltimer_ns();
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int n_tile = blockIdx.x, m_tile = blockIdx.y, split = blockIdx.z;
    // diagnostics (globaltimer ns): [0] entry, [1] split-K epilogue items done, [2] set-up
    // done, [3] first stage landed, [4] last MMA issued, [5] accumulator ready, [6] exit,
    // [7] split-K partials visible
    unsigned long long *trace = nullptr;
    if (p.trace != nullptr)
        trace = p.trace + 8ull * ((static_cast<unsigned long long>(blockIdx.z) * gridDim.y + blockIdx.y) *
                                  gridDim.x + blockIdx.x);
    const int n0 = n_tile * BN, m0 = m_tile * 128;
    const int kt_begin = split * p.kt_per_split;
    const int kt_end = min(p.k_tiles, kt_begin + p.kt_per_split);
    const int nkt = kt_end - kt_begin;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(bar_full + 8 * s, 1);
            mbar_init(bar_empty + 8 * s, 1);
        }
        mbar_init(bar_acc, 1);
        for (int j = 0; j < C::kSlots; ++j) {
            mbar_init(bar_sfr + 8 * j, 4);
            mbar_init(bar_sff + 8 * j, 1);
        }
        misc[1] = 0;
        misc[2] = 0;
        fence_mbar_init();
        prefetch_tmap(&tmA);
        prefetch_tmap(&tmB);
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(const_cast<uint32_t *>(misc)), C::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = misc[0];
    // With a separate reduction region the only cluster-wide requirement before the partial
    // rows are pushed is that every peer has started (its shared memory exists): a cluster
    // barrier here, while the previous kernel still runs (programmatic launch), covers it.
    if constexpr (S::kSepRed) {
        if (p.cluster) cluster_sync_all();
    }
    if (trace != nullptr && threadIdx.x == 0) {
        trace[0] = t_entry;
        trace[2] = globaltimer_ns();
    }
    // Let the next kernel in the stream start its own weight prefetch.
    pdl_launch_dependents();

    auto nkb_of = [&](int kt) { return min(4, p.k_atoms - 4 * kt); };
    auto stage_bytes = [&](int kt) {
        return p.a_box_rows * 128u + static_cast<uint32_t>(C::kBBytes) +
               static_cast<uint32_t>(nkb_of(kt)) * kSfAtom * (1 + C::kSfbGroups);
    };

    if (warp == 0) {
        if (lane == 0) {
            // ------------------------------ producer ------------------------------
            const uint64_t pol_w = policy_evict_first();
            const uint64_t pol_a = policy_evict_last();
            auto load_w = [&](int j) {
                const int s = j % STAGES, kt = kt_begin + j;
                const uint32_t full = bar_full + 8 * s;
                const uint32_t nb = static_cast<uint32_t>(nkb_of(kt)) * kSfAtom;
                tma_load_2d(sbase + S::kOffB + s * C::kBBytes, &tmB, kt * 128, n0, full, pol_w);
#pragma unroll
                for (int gi = 0; gi < C::kSfbGroups; ++gi) {
                    const size_t grp = static_cast<size_t>(n0 / 128 + gi);
                    bulk_load(sbase + S::kOffSfb + s * C::kSfbBytes + gi * 4 * kSfAtom,
                              p.sfb + (grp * p.k_atoms + 4 * kt) * kSfAtom, nb, full, pol_w);
                }
            };
            auto load_a = [&](int j) {
                const int s = j % STAGES, kt = kt_begin + j;
                const uint32_t full = bar_full + 8 * s;
                const uint32_t nb = static_cast<uint32_t>(nkb_of(kt)) * kSfAtom;
                tma_load_2d(sbase + S::kOffA + s * S::kA, &tmA, kt * 128, m0, full, pol_a);
                bulk_load(sbase + S::kOffSfa + s * C::kSfaBytes,
                          p.sfa + (static_cast<size_t>(m_tile) * p.k_atoms + 4 * kt) * kSfAtom, nb, full, pol_a);
            };
            const int pre = min(STAGES, nkt);
            for (int j = 0; j < pre; ++j) {
                mbar_arrive_expect_tx(bar_full + 8 * (j % STAGES), stage_bytes(kt_begin + j));
                load_w(j);
            }
            pdl_wait();  // A and its scales come from the previous kernel
            for (int j = 0; j < pre; ++j) load_a(j);
            int issued = pre;
            for (int j = pre; j < nkt; ++j) {
                const int s = j % STAGES;
                if (!mbar_wait(bar_empty + 8 * s, ((j / STAGES) - 1) & 1, abort_flag, &g_device_status, kStatusTimeoutEmpty)) break;
                mbar_arrive_expect_tx(bar_full + 8 * s, stage_bytes(kt_begin + j));
                load_w(j);
                load_a(j);
                issued = j + 1;
            }
            // drain: every issued stage must have landed before the CTA may exit
            for (int j = max(0, issued - STAGES); j < issued; ++j)
                drain_wait(bar_full + 8 * (j % STAGES), (j / STAGES) & 1);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ------------------------------ MMA issuer ------------------------------
            constexpr uint32_t idesc = idesc_mxf4nvf4(128, BN);
            const uint32_t t_acc = tmem;
            const uint32_t sfb_sub = (BN == 64) ? static_cast<uint32_t>((n0 & 127) >> 5) : 0u;
            for (int j = 0; j < nkt; ++j) {
                const int s = j % STAGES, kt = kt_begin + j, slot = j % C::kSlots;
                if (!mbar_wait(bar_full + 8 * s, (j / STAGES) & 1, abort_flag, &g_device_status, kStatusTimeoutFull) ||
                    !mbar_wait(bar_sfr + 8 * slot, (j / C::kSlots) & 1, abort_flag, &g_device_status,
                               kStatusTimeoutFull))
                    break;
                tc_fence_after();
                if (trace != nullptr && j == 0) trace[3] = globaltimer_ns();
                const int nkb = nkb_of(kt);
                const uint32_t a_s = sbase + S::kOffA + s * S::kA;
                const uint32_t b_s = sbase + S::kOffB + s * C::kBBytes;
                const uint32_t t_sf = tmem + C::kColSf + slot * C::kSfSlot;
                for (int kb = 0; kb < nkb; ++kb) {
                    tc_mma_mxf4nvf4(t_acc, desc_kmajor_sw128(a_s + 32 * kb), desc_kmajor_sw128(b_s + 32 * kb),
                                    idesc, t_sf + 4 * kb, t_sf + 16 + 4 * C::kSfbGroups * kb + sfb_sub,
                                    (j > 0 || kb > 0) ? 1u : 0u);
                }
                tc_commit(bar_empty + 8 * s);   // frees the stage once these MMAs finished reading it
                tc_commit(bar_sff + 8 * slot);  // and the scale slot
            }
            if (trace != nullptr) trace[4] = globaltimer_ns();
            tc_commit(bar_acc);  // always: completion of every MMA issued above
        }
    } else {
        // ------------------------------ epilogue ------------------------------
        const int q = warp & 3;  // tensor-memory sub-partition this warp may read
        const int row = q * 32 + lane;
        const int m = m0 + row;
        const bool row_ok = m < p.M;
        // Until the accumulator is ready these warps copy the scale atoms (tcgen05.cp from one
        // thread complete one after another; from four warps they overlap): warp w copies
        // k-block w of each stage into the stage's scale slot.
        if (lane == 0) {
            const int w = warp - 2;
            const uint32_t sfa_s0 = sbase + S::kOffSfa, sfb_s0 = sbase + S::kOffSfb;
            for (int j = 0; j < nkt; ++j) {
                const int s = j % STAGES, kt = kt_begin + j, slot = j % C::kSlots;
                if (!mbar_wait(bar_full + 8 * s, (j / STAGES) & 1, abort_flag, &g_device_status, kStatusTimeoutFull))
                    break;
                if (j >= C::kSlots && !mbar_wait(bar_sff + 8 * slot, (j / C::kSlots - 1) & 1, abort_flag,
                                                 &g_device_status, kStatusTimeoutFull))
                    break;
                tc_fence_after();
                const uint32_t t_sf = tmem + C::kColSf + slot * C::kSfSlot;
                if (w < nkb_of(kt)) {
                    tc_cp_32x128b_warpx4(t_sf + 4 * w, desc_sf_32x128b(sfa_s0 + s * C::kSfaBytes + w * kSfAtom));
#pragma unroll
                    for (int gi = 0; gi < C::kSfbGroups; ++gi)
                        tc_cp_32x128b_warpx4(t_sf + 16 + 4 * C::kSfbGroups * w + 4 * gi,
                                             desc_sf_32x128b(sfb_s0 + s * C::kSfbBytes + gi * 4 * kSfAtom + w * kSfAtom));
                }
                tc_commit(bar_sfr + 8 * slot);  // arrives when this warp's copies have landed
            }
        }
        __syncwarp();
        const bool done = drain_wait(bar_acc, 0);
        // one decision for all four epilogue warps (tcgen05.ld and the named barriers below
        // must be reached uniformly)
        named_barrier_epi();
        if (threadIdx.x == 64) misc[3] = (done && !*abort_flag) ? 1u : 0u;
        named_barrier_epi();
        const bool acc_ok = misc[3] != 0u;
        if (trace != nullptr && threadIdx.x == 64) trace[5] = globaltimer_ns();
        tc_fence_after();
        pdl_wait();
        if (acc_ok) {
            const uint32_t t_row = tmem + (static_cast<uint32_t>(q * 32) << 16);
            if (p.splits == 1) {
                for (int c0 = 0; c0 < BN; c0 += 32) {
                    uint32_t r[32];
                    tmem_ld_32x32b_x32(t_row + c0, r);
                    tmem_ld_wait();
                    if (row_ok) {
                        float v[32];
#pragma unroll
                        for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
                        epilogue_chunk(p, m, n0 + c0, v);
                    }
                }
            } else if (p.cluster) {
                // split-K across the cluster: pushed to the owners after the cluster barrier
            } else {
                // split-K: partial tile to the workspace, then an arrival ticket
                float *part = p.partials + (static_cast<size_t>(split) * p.M) * p.N;
                for (int c0 = 0; c0 < BN; c0 += 32) {
                    uint32_t r[32];
                    tmem_ld_32x32b_x32(t_row + c0, r);
                    tmem_ld_wait();
                    if (row_ok) {
                        float4 *dst = reinterpret_cast<float4 *>(part + static_cast<size_t>(m) * p.N + n0 + c0);
#pragma unroll
                        for (int j = 0; j < 8; ++j)
                            __stcg(dst + j, make_float4(__uint_as_float(r[4 * j]), __uint_as_float(r[4 * j + 1]),
                                                        __uint_as_float(r[4 * j + 2]), __uint_as_float(r[4 * j + 3])));
                    }
                }
                __threadfence();
                named_barrier_epi();
                uint32_t *ticket = p.tickets + (static_cast<size_t>(m_tile) * p.n_tiles + n_tile);
                if (threadIdx.x == 64) misc[2] = atomicAdd(ticket, 1u);
                named_barrier_epi();
                if (misc[2] == static_cast<uint32_t>(p.splits - 1)) {
                    __threadfence();
                    if (trace != nullptr && threadIdx.x == 64) trace[7] = globaltimer_ns();
                    if (row_ok) {
                        for (int c0 = 0; c0 < BN; c0 += 32) {
                            float v[32];
#pragma unroll
                            for (int i = 0; i < 32; ++i) v[i] = 0.0f;
                            for (int sp = 0; sp < p.splits; ++sp) {
                                const float4 *src = reinterpret_cast<const float4 *>(
                                    p.partials + (static_cast<size_t>(sp) * p.M + m) * p.N + n0 + c0);
#pragma unroll
                                for (int j = 0; j < 8; ++j) {
                                    const float4 u = __ldcg(src + j);
                                    v[4 * j] = __fadd_rn(v[4 * j], u.x);
                                    v[4 * j + 1] = __fadd_rn(v[4 * j + 1], u.y);
                                    v[4 * j + 2] = __fadd_rn(v[4 * j + 2], u.z);
                                    v[4 * j + 3] = __fadd_rn(v[4 * j + 3], u.w);
                                }
                            }
                            epilogue_chunk(p, m, n0 + c0, v);
                        }
                    }
                    if (threadIdx.x == 64) *ticket = 0u;  // ready for the next call
                }
            }
        }
    }

    if (p.cluster) {
        // Deterministic split-K reduction over distributed shared memory.  CTA `rank` of the
        // cluster (= its split) owns local rows rank, rank + S, ...  (1) a cluster barrier
        // (only where the partial slots reuse the stages): every CTA's MMAs are done with its
        // stage buffers, which now hold partials; (2) every
        // CTA pushes each of its accumulator rows into slot [split][row / S] of the row's
        // owner (remote stores, nothing waits on them); (3) a cluster barrier: all partials
        // landed; (4) all threads of each owner add its rows' S partials from its own shared
        // memory in split order 0..S-1 and run the epilogue on chunks of W columns (16; 32 for
        // GeGLU).  Nothing reads a peer after (3).  The bias and residual of each thread's
        // first chunk are loaded before (1).
        const int S_ = p.splits;
        const int rank = static_cast<int>(cluster_ctarank());
        const int rows_valid = min(SMALL_A ? 64 : 128, p.M - m0);
        const int R = (rows_valid + S_ - 1) / S_;  // rows per owner
        float *part = reinterpret_cast<float *>(smem + S::kOffRed);
        if (warp < 2) pdl_wait();  // the residual may come from the previous kernel
        auto reduce = [&](auto width) {
            constexpr int W = decltype(width)::value;
            constexpr int kChunks = BN / W;
            const int e = threadIdx.x;
            const int i0 = rank + (e / kChunks) * S_, ch0 = e % kChunks;
            uint32_t bw0[W / 2], rw0[W / 2];
            const bool has_bias = p.bias != nullptr, has_res = p.residual != nullptr;
            if (i0 < rows_valid) {
                if (has_bias) load_bf16<W>(p.bias + n0 + ch0 * W, bw0);
                if (has_res) load_bf16<W>(p.residual + static_cast<size_t>(m0 + i0) * p.ldr + n0 + ch0 * W, rw0);
            }
            __syncwarp();
            // (1): the stages become partial slots; with a region of their own only this CTA's
            // threads need to meet (every one reads the accumulator-valid word below)
            if constexpr (!S::kSepRed) cluster_sync_all();
            else __syncthreads();
            const bool acc_ok = misc[3] != 0u;
            if (warp >= 2 && acc_ok) {
                const int q = warp & 3;
                const int row = q * 32 + lane;
                if (q * 32 < rows_valid) {  // warp-uniform: tcgen05.ld is .sync.aligned
                    const uint32_t t_row = tmem + (static_cast<uint32_t>(q * 32) << 16);
                    const uint32_t dst = mapa_shared(smem_u32(part + ((split * R + row / S_) * S::kRedLd)),
                                                     static_cast<uint32_t>(row % S_));
                    for (int c0 = 0; c0 < BN; c0 += 32) {
                        uint32_t r[32];
                        tmem_ld_32x32b_x32(t_row + c0, r);
                        tmem_ld_wait();
                        if (row < rows_valid) {
#pragma unroll
                            for (int j = 0; j < 8; ++j)
                                st_dsmem_f4(dst + 4 * (c0 + 4 * j),
                                            make_float4(__uint_as_float(r[4 * j]), __uint_as_float(r[4 * j + 1]),
                                                        __uint_as_float(r[4 * j + 2]), __uint_as_float(r[4 * j + 3])));
                        }
                    }
                }
            }
            __syncwarp();
            cluster_sync_all();  // (3)
            if (trace != nullptr && threadIdx.x == 64) trace[7] = globaltimer_ns();
            if (!acc_ok) return;
            for (int item = e;; item += kThreads) {
                const int li = item / kChunks, ch = item % kChunks;
                const int i = rank + li * S_;
                if (i >= rows_valid) break;
                float v[W];
#pragma unroll
                for (int t = 0; t < W; ++t) v[t] = 0.0f;
                for (int sp = 0; sp < S_; ++sp) {
                    const float4 *src4 = reinterpret_cast<const float4 *>(part + (sp * R + li) * S::kRedLd + ch * W);
#pragma unroll
                    for (int j = 0; j < W / 4; ++j) {
                        const float4 u = src4[j];
                        v[4 * j] = __fadd_rn(v[4 * j], u.x);
                        v[4 * j + 1] = __fadd_rn(v[4 * j + 1], u.y);
                        v[4 * j + 2] = __fadd_rn(v[4 * j + 2], u.z);
                        v[4 * j + 3] = __fadd_rn(v[4 * j + 3], u.w);
                    }
                }
                if (item == e)
                    epilogue_chunk_w<W>(p, m0 + i, n0 + ch * W, v, has_bias ? bw0 : nullptr, has_res ? rw0 : nullptr);
                else
                    epilogue_chunk<W>(p, m0 + i, n0 + ch * W, v);
            }
        };
        if (p.epi == kEpiGeglu)
            reduce(std::integral_constant<int, 32>());
        else
            reduce(std::integral_constant<int, 16>());
        if (trace != nullptr && threadIdx.x == 64) trace[1] = globaltimer_ns();
    }

    tc_fence_before();
    __syncthreads();
    if (trace != nullptr && threadIdx.x == 0) trace[6] = globaltimer_ns();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, C::kTmemCols);
    }
}

template <int BN, int STAGES, bool SMALL_A>
cudaError_t launch_bn(const CUtensorMap &ta, const CUtensorMap &tb, const GemmArgs &p, cudaStream_t s) {
    using S = Smem<BN, STAGES, SMALL_A>;
    static std::atomic<bool> attr_set[kMaxDevices];
    const cudaError_t e =
        set_smem_limit_once(reinterpret_cast<const void *>(gemm_kernel<BN, STAGES, SMALL_A>), S::kBytes, attr_set);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(p.n_tiles, (p.M + 127) / 128, p.splits);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = S::kBytes;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    int n = 0;
    if (pdl_enabled()) {
        attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[n].val.programmaticStreamSerializationAllowed = 1;
        ++n;
    }
    if (p.cluster) {
        attr[n].id = cudaLaunchAttributeClusterDimension;
        attr[n].val.clusterDim.x = 1;
        attr[n].val.clusterDim.y = 1;
        attr[n].val.clusterDim.z = static_cast<unsigned>(p.splits);
        ++n;
    }
    cfg.attrs = attr;
    cfg.numAttrs = n;
    return cudaLaunchKernelEx(&cfg, gemm_kernel<BN, STAGES, SMALL_A>, ta, tb, p);
}

}  // namespace

// Device address of g_noalloc_scratch for the current device.  Host code only sees a
// host-side stand-in under that name, so the address is looked up once per device (with
// that device current) and cached; no allocation is involved.  The cache entries are
// atomics: host threads making their first calls at once each look the address up and
// store the same value.
cudaError_t noalloc_scratch(void **ptr, size_t *bytes) {
    static std::atomic<void *> addr[kMaxDevices];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    void *a = addr[dev].load(std::memory_order_acquire);
    if (a == nullptr) {
        e = cudaGetSymbolAddress(&a, g_noalloc_scratch);
        if (e != cudaSuccess) return e;
        addr[dev].store(a, std::memory_order_release);
    }
    *ptr = a;
    *bytes = kNoAllocScratchBytes;
    return cudaSuccess;
}

cudaError_t set_smem_limit_once(const void *func, int bytes, std::atomic<bool> *done) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    if (done[dev].load(std::memory_order_acquire)) return cudaSuccess;
    e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess) done[dev].store(true, std::memory_order_release);
    return e;
}

bool pdl_enabled() {
    static int on = -1;
    if (on < 0) {
        const char *e = getenv("NVFP4_PDL");
        on = (e != nullptr && e[0] == '0') ? 0 : 1;
    }
    return on == 1;
}

cudaError_t probe_gemm_kernels() {
    cudaFuncAttributes fa;
    return cudaFuncGetAttributes(&fa, gemm_kernel<128, 5, false>);
}

cudaError_t device_status_address(uint32_t **p) {
    void *a = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&a, g_device_status);
    *p = static_cast<uint32_t *>(a);
    return e;
}

cudaError_t read_and_clear_device_status(cudaStream_t s, uint32_t *out) {
    cudaError_t e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return e;
    e = cudaMemcpyFromSymbol(out, g_device_status, sizeof(uint32_t));
    if (e != cudaSuccess) return e;
    const uint32_t zero = 0;
    return cudaMemcpyToSymbol(g_device_status, &zero, sizeof(uint32_t));
}

template <int BN, int STAGES, bool SMALL_A>
static int wave_ctas_of(int cluster) {
    using S = Smem<BN, STAGES, SMALL_A>;
    if (cudaFuncSetAttribute(gemm_kernel<BN, STAGES, SMALL_A>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             S::kBytes) != cudaSuccess)
        return 0;
    if (cluster <= 1) {
        int per_sm = 0, dev = 0, sms = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, gemm_kernel<BN, STAGES, SMALL_A>, kThreads,
                                                          S::kBytes) != cudaSuccess ||
            cudaGetDevice(&dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return 0;
        return per_sm * sms;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(cluster));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = S::kBytes;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = static_cast<unsigned>(cluster);
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, gemm_kernel<BN, STAGES, SMALL_A>, &cfg) != cudaSuccess) return 0;
    return n * cluster;
}

int gemm_wave_ctas(bool small, int block_n, int cluster) {
    if (cluster < 1 || cluster > 8) return 0;
    static int cache[2][3][9] = {};  // [small][64, 128, 256][cluster]; 0 = not yet asked
    const int w = block_n == 64 ? 0 : block_n == 128 ? 1 : block_n == 256 ? 2 : -1;
    if (w < 0) return 0;
    int &c = cache[small ? 1 : 0][w][cluster];
    if (c == 0) {
        int v = 0;
        switch (block_n) {
        case 64: v = small ? wave_ctas_of<64, 4, true>(cluster) : wave_ctas_of<64, 6, false>(cluster); break;
        case 128: v = small ? wave_ctas_of<128, 3, true>(cluster) : wave_ctas_of<128, 5, false>(cluster); break;
        default: v = small ? wave_ctas_of<256, 2, true>(cluster) : wave_ctas_of<256, 3, false>(cluster); break;
        }
        cudaGetLastError();
        c = v > 0 ? v : -1;
    }
    return c > 0 ? c : 0;
}

cudaError_t launch_gemm(const CUtensorMap &ta, const CUtensorMap &tb, const GemmArgs &p, int block_n,
                        cudaStream_t s) {
    const bool small = p.a_box_rows <= 64;
    // M <= 64: ~100 KB of shared memory and <= 256 TMEM columns, so two CTAs share an SM and
    // the next GEMM prefetches its weights while this one finishes.  Larger M: deep pipelines.
    switch (block_n) {
    case 64: return small ? launch_bn<64, 4, true>(ta, tb, p, s) : launch_bn<64, 6, false>(ta, tb, p, s);
    case 128: return small ? launch_bn<128, 3, true>(ta, tb, p, s) : launch_bn<128, 5, false>(ta, tb, p, s);
    case 256: return small ? launch_bn<256, 2, true>(ta, tb, p, s) : launch_bn<256, 3, false>(ta, tb, p, s);
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace nvfp4
