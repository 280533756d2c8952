// gemm_persistent.cu — block-scaled NVFP4 GEMM for many rows (the compute-bound regime,
// e.g. a prefill layer at M = 968), as a persistent kernel: one CTA per SM walks 128 x 256
// output tiles, m-tile fastest, so the 8 CTAs that share a weight tile read it close together
// and it is fetched from HBM once (the activations stay in L2).
//
//   acc[m, n] = sum_k e(A)[m, k] sA[m, k/16] e(W)[n, k] sW[n, k/16]      (fp32, in TMEM)
//   v = acc * gA * gW (+ bias[n]) (+ residual[m, n])  ->  bf16, or tanh-GELU / GeGLU -> FP4
// ("GROOT N1.7 update: Thor NVFP4 + FA4 performance tier", §What is in the tier;
// "Pi0.5 Thor NVFP4 End-to-End Results", §Fused GeGLU FFN in the Decoder.)
//
// Roles (384 threads):
//   warp 0      producer: TMA loads of the A (128 rows) and W (256 rows) code tiles and bulk
//               loads of their scale atoms into a 4-stage ring; the weights of the first
//               stages are issued before the programmatic-launch wait.
//   warps 10-11 scale copiers: tcgen05.cp (32x128b.warpx4) of the stage's scale atoms into
//               one of two TMEM scale slots, signalled to the MMA warp by tcgen05.commit.
//   warp 1      MMA issuer: 4 x tcgen05.mma kind::mxf4nvf4 block16 (M = 128, N = BN, K = 64)
//               per 256-wide K tile.
//   warps 2..9  epilogue: two warps per TMEM sub-partition, each draining 128 of the 256
//               accumulator columns of its 32 rows into registers; the accumulator is handed
//               back to the MMA warp right after the drain, so the fused epilogue of one tile
//               runs while the next tile's MMAs do.  The kernel is instantiated per epilogue
//               kind, so each instance holds one path (and fits its registers without spills).
//
// Scale copies: tcgen05.cp instructions from one thread complete one after another (about
// 90 cycles each, measured), which made them, not the MMAs, bound a single issuing thread.
// From separate warps they overlap (48 copies: 4490 cycles from one thread, 1011 from eight
// warps), so two copier warps issue them and the MMA warp only issues MMAs.
//
// Split K in two (when a GEMM has fewer 128 x BN tiles than SMs, e.g. the prefill down
// projection: 64 tiles of K = 16384): the CTAs walk (tile, split) units.  Each split of a
// tile takes an arrival ticket when its accumulator is complete; the second to arrive
// reduces, the first publishes its fp32 partial through the workspace (2 counters per tile
// + tiles x 128 x BN floats per split).
//
// Every wait is bounded (sm100.cuh); an expired wait records a status and the CTA unwinds.
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

// Shared-memory and TMEM plan for a tile width BN (256, or 128 when 256-wide tiles would
// leave SMs idle): as many stages of [A 128 x 256 FP4 | W BN x 256 FP4 | A scale atoms of
// the 4 k-blocks | W scale atoms, per 128-row group] as fit in 216 KB.
template <int BN>
struct PCfg {
    static constexpr int kGroups = BN / 128;  // 128-row scale groups of a W tile
    static constexpr int kStageA = 128 * 128;
    static constexpr int kStageB = BN * 128;
    static constexpr int kStageSfa = 4 * kSfAtom;
    static constexpr int kStageSfb = kGroups * 4 * kSfAtom;
    static constexpr int kOffB = kStageA;
    static constexpr int kOffSfa = kOffB + kStageB;
    static constexpr int kOffSfb = kOffSfa + kStageSfa;
    static constexpr int kStage = kOffSfb + kStageSfb;  // 54 KB (BN 256) / 36 KB (BN 128)
    static constexpr int kStages = (216 * 1024) / kStage;
    // per epilogue warp, 1 KB to stage 16 rows x 64 bytes of bf16 output / residual
    static constexpr int kOffStaging = kStages * kStage;
    static constexpr int kOffBar = kOffStaging + 8 * 1024;
    // scale columns: kSlots slots (step modulo kSlots) of [A: 4 k-blocks x 4 | W: 4 k-blocks x
    // groups x 4]; the copies of a step may run up to kSlots - 1 steps ahead of its MMAs
    static constexpr int kSlots = 2;
    static constexpr int kColSf = BN;
    static constexpr int kSfSlot = 16 + 16 * kGroups;
    static constexpr int kTmemCols = (kColSf + kSlots * kSfSlot) <= 256 ? 256 : 512;
    // barriers: full[kStages], empty[kStages], acc_full, acc_empty, sf_ready[kSlots],
    // sf_free[kSlots], sf_full[kStages]
    static constexpr int kOffMisc = kOffBar + (3 * kStages + 2 + 2 * kSlots) * 8;
    static constexpr int kSmemBytes = kOffMisc + 16 + 1024;  // + alignment slack
    static_assert(kStage % 1024 == 0, "stage alignment (128-byte swizzle atoms)");
    static_assert(kColSf + kSlots * kSfSlot <= kTmemCols, "tensor memory columns");
    static_assert(kSmemBytes <= 232448, "shared memory per CTA");
};

// Barrier of the 256 epilogue threads that also ANDs a flag across them (every decision to
// abandon the work is taken by all eight warps together).
// Bounded wait until the published count at p reaches target (split K: the reducer of a tile
// waits for the splits that arrived before it; they wait on nothing, so this ends unless one
// of them aborted).
__device__ bool wait_published(const unsigned int *p, unsigned int target, volatile int *abort_flag, uint32_t *status) {
    if (ld_acquire_gpu(p) >= target) return true;
    const uint64_t t0 = globaltimer_ns();
    while (true) {
        __nanosleep(32);
        if (ld_acquire_gpu(p) >= target) return true;
        if (*abort_flag) return false;
        if (globaltimer_ns() - t0 > kWaitLimitNs) {
            atomicCAS(status, static_cast<uint32_t>(kStatusOk), static_cast<uint32_t>(kStatusTimeoutPeer));
            *abort_flag = 1;
            return false;
        }
    }
}

// bf16 epilogue of one 32-column chunk of a warp's 32 rows (lane l holds row m0 + l, values
// v of columns n .. n + 31): v * alpha (+ bias) (+ residual), rounded to bf16, the same
// arithmetic as epilogue_chunk.  The residual is read and the output written through a 1 KB
// shared-memory buffer, 16 rows at a time, so that 4 lanes move the 64 bytes of one row
// (8 rows per warp access) instead of 32 lanes each touching a different row.  16-byte piece
// q of staged row r sits at r * 64 + 16 * (q ^ ((r >> 1) & 3)): both access patterns are
// free of bank conflicts.  Every lane of the warp must call it (rows >= M are not touched).
template <int EPI>
__device__ __forceinline__ void bf16_chunk_staged(const GemmArgs &p, int m0, int lane, int n, float *v,
                                                  uint8_t *stage) {
    const float alpha = p.alpha;
    const int M = p.M;
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __fmul_rn(v[i], alpha);
    if constexpr (EPI == kEpiBias || EPI == kEpiBiasResidual) {
        uint32_t bw[16];
        load_bf16<32>(p.bias + n, bw);
#pragma unroll
        for (int t = 0; t < 16; ++t) {
            v[2 * t] = __fadd_rn(v[2 * t], bf16lo(bw[t]));
            v[2 * t + 1] = __fadd_rn(v[2 * t + 1], bf16hi(bw[t]));
        }
    }
    auto slot = [&](int r, int q) { return reinterpret_cast<uint4 *>(stage + r * 64 + 16 * (q ^ ((r >> 1) & 3))); };
    const int q = lane & 3;
    if constexpr (EPI == kEpiResidual || EPI == kEpiBiasResidual) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
#pragma unroll
            for (int k = 0; k < 2; ++k) {
                const int r = (lane >> 2) + 8 * k, row = m0 + 16 * h + r;
                uint4 u = make_uint4(0u, 0u, 0u, 0u);
                if (row < M) u = *reinterpret_cast<const uint4 *>(p.residual + static_cast<size_t>(row) * p.ldr + n + 8 * q);
                *slot(r, q) = u;
            }
            __syncwarp();
            if ((lane >> 4) == h) {
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const uint4 u = *slot(lane & 15, j);
                    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                    for (int t = 0; t < 4; ++t) {
                        v[8 * j + 2 * t] = __fadd_rn(v[8 * j + 2 * t], bf16lo(w[t]));
                        v[8 * j + 2 * t + 1] = __fadd_rn(v[8 * j + 2 * t + 1], bf16hi(w[t]));
                    }
                }
            }
            __syncwarp();
        }
    }
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        if ((lane >> 4) == h) {
#pragma unroll
            for (int j = 0; j < 4; ++j)
                *slot(lane & 15, j) = make_uint4(pack_bf16x2(v[8 * j], v[8 * j + 1]), pack_bf16x2(v[8 * j + 2], v[8 * j + 3]),
                                                 pack_bf16x2(v[8 * j + 4], v[8 * j + 5]),
                                                 pack_bf16x2(v[8 * j + 6], v[8 * j + 7]));
        }
        __syncwarp();
#pragma unroll
        for (int k = 0; k < 2; ++k) {
            const int r = (lane >> 2) + 8 * k, row = m0 + 16 * h + r;
            const uint4 u = *slot(r, q);
            if (row < M) *reinterpret_cast<uint4 *>(p.out + static_cast<size_t>(row) * p.ldo + n + 8 * q) = u;
        }
        __syncwarp();
    }
}

// One 32-column chunk of the epilogue: bf16 kinds through the staging buffer (every lane),
// FP4 kinds per row.
template <int EPI>
__device__ __forceinline__ void chunk_out(const GemmArgs &p, int m0, int lane, int n, float *v, uint8_t *stage) {
    if constexpr (EPI == kEpiBiasGelu || EPI == kEpiGeglu) {
        if (m0 + lane < p.M) epilogue_chunk<32, EPI>(p, m0 + lane, n, v);
    } else {
        bf16_chunk_staged<EPI>(p, m0, lane, n, v, stage);
    }
}

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

// SPLIT: K split in two (p.splits == 2); a separate instance, so the unsplit kernel carries
// none of the split epilogue.
template <int BN, int EPI, bool SPLIT>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_persistent_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                           const GemmArgs p) {
    using Cf = PCfg<BN>;
    constexpr int kStages = Cf::kStages, kStage = Cf::kStage, kStageA = Cf::kStageA, kStageB = Cf::kStageB;
    constexpr int kOffB = Cf::kOffB, kOffSfa = Cf::kOffSfa, kOffSfb = Cf::kOffSfb, kGroups = Cf::kGroups;
    constexpr int kColSf = Cf::kColSf, kSfSlot = Cf::kSfSlot, kTmemCols = Cf::kTmemCols, kSlots = Cf::kSlots;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const uint32_t bar_full = sbase + Cf::kOffBar;
    const uint32_t bar_empty = bar_full + 8 * kStages;
    const uint32_t bar_accf = bar_empty + 8 * kStages;
    const uint32_t bar_acce = bar_accf + 8;
    const uint32_t bar_sfr = bar_acce + 8;            // kSlots: slot copied (an arrival per copier)
    const uint32_t bar_sff = bar_sfr + 8 * kSlots;    // kSlots: slot read by its MMAs
    const uint32_t bar_sfl = bar_sff + 8 * kSlots;    // kStages: the stage's scale atoms have landed
    // misc: [0] TMEM base, [1] abort flag, [2] split-K arrival ticket of the current unit
    volatile uint32_t *misc = reinterpret_cast<volatile uint32_t *>(smem + Cf::kOffMisc);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(misc + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int m_tiles = (p.M + 127) / 128;
    const int tiles = m_tiles * p.n_tiles;
    // work units: (tile, split); unit u is tile u % tiles, split u / tiles.  Split 0 covers K
    // tiles [0, k0), split 1 [k0, k_tiles), k0 = p.kt_per_split (k_tiles without a split).
    // The host makes split 0 a few K tiles longer, so that split 1 has usually published its
    // partial by the time split 0 arrives and the reducer does not wait.
    constexpr int n_splits = SPLIT ? 2 : 1;
    const int k0 = SPLIT ? p.kt_per_split : p.k_tiles;
    auto kt_begin_of = [&](int split) { return split != 0 ? k0 : 0; };
    auto kt_count_of = [&](int split) { return split != 0 ? p.k_tiles - k0 : k0; };
    const int units = tiles * n_splits;
    const int my_tiles = static_cast<int>(blockIdx.x) < units ? (units - 1 - static_cast<int>(blockIdx.x)) / gridDim.x + 1 : 0;
    int steps = my_tiles * k0;
    if constexpr (SPLIT) {
        steps = 0;
        for (int i = 0; i < my_tiles; ++i)
            steps += kt_count_of((static_cast<int>(blockIdx.x) + i * static_cast<int>(gridDim.x)) / tiles);
    }
    unsigned long long *trace = p.trace != nullptr ? p.trace + 8ull * blockIdx.x : nullptr;
    if (trace != nullptr && threadIdx.x == 0) trace[0] = globaltimer_ns();

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(bar_full + 8 * s, 1);
            mbar_init(bar_empty + 8 * s, 1);
            mbar_init(bar_sfl + 8 * s, 1);
        }
        mbar_init(bar_accf, 1);
        mbar_init(bar_acce, 1);
        for (int j = 0; j < kSlots; ++j) {
            mbar_init(bar_sfr + 8 * j, kCopiers);
            mbar_init(bar_sff + 8 * j, 1);
        }
        misc[1] = 0;
        fence_mbar_init();
        prefetch_tmap(&tmA);
        prefetch_tmap(&tmB);
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

    auto nkb_of = [&](int kt) { return min(4, p.k_atoms - 4 * kt); };
    auto unit_of = [&](int i) { return static_cast<int>(blockIdx.x) + i * static_cast<int>(gridDim.x); };
    auto tile_of = [&](int i) { return unit_of(i) % tiles; };
    // A walk over this CTA's steps: unit i, its tile t, step j of the unit's n K tiles = global
    // K tile kt0 + j.  Advancing costs an increment; the divisions run once per unit.
    struct Walk {
        int i, j, t, kt0, n;
    };
    auto walk_unit = [&](Walk &w) {
        const int u = unit_of(w.i);
        w.t = u % tiles;
        w.kt0 = kt_begin_of(u / tiles);
        w.n = kt_count_of(u / tiles);
    };
    auto walk_next = [&](Walk &w) {
        if (++w.j == w.n) {
            w.j = 0;
            ++w.i;
            walk_unit(w);
        }
    };
    auto walk_start = [&]() {
        Walk w{0, 0, 0, 0, 0};
        walk_unit(w);
        return w;
    };

    if (warp == 0) {
        // ------------------------------ producer (whole warp) ------------------------------
        const uint64_t pol = policy_evict_last();  // A and W both fit in L2 and are re-read
        // The scale atoms complete on their own barrier (sf_full) and are issued before the code
        // tiles: the copiers move them into tensor memory while the 48 KB of codes still land.
        auto expect = [&](int st, const Walk &w) {
            const int nkb = nkb_of(w.kt0 + w.j);
            if (lane == 0) {
                mbar_arrive_expect_tx(bar_sfl + 8 * (st % kStages), static_cast<uint32_t>(nkb) * (1u + kGroups) * kSfAtom);
                mbar_arrive_expect_tx(bar_full + 8 * (st % kStages), kStageA + kStageB);
            }
            __syncwarp();
        };
        auto issue_w = [&](int st, const Walk &w) {
            const int s = st % kStages, t = w.t, kt = w.kt0 + w.j;
            const int n_tile = t / m_tiles, nkb = nkb_of(kt);
            const uint32_t full = bar_full + 8 * s, sfl = bar_sfl + 8 * s, base = sbase + s * kStage;
            if (lane < kGroups) {  // the k-blocks' atoms of each 128-row group are contiguous
                const size_t grp = static_cast<size_t>(n_tile) * kGroups + lane;
                bulk_load(base + kOffSfb + lane * 4 * kSfAtom, p.sfb + (grp * p.k_atoms + 4 * kt) * kSfAtom,
                          static_cast<uint32_t>(nkb) * kSfAtom, sfl, pol);
            }
            __syncwarp();
            if (lane == 0) tma_load_2d(base + kOffB, &tmB, kt * 128, n_tile * BN, full, pol);
        };
        auto issue_a = [&](int st, const Walk &w) {
            const int s = st % kStages, t = w.t, kt = w.kt0 + w.j;
            const int m_tile = t % m_tiles, nkb = nkb_of(kt);
            const uint32_t full = bar_full + 8 * s, sfl = bar_sfl + 8 * s, base = sbase + s * kStage;
            if (lane == 0) {
                bulk_load(base + kOffSfa, p.sfa + (static_cast<size_t>(m_tile) * p.k_atoms + 4 * kt) * kSfAtom,
                          static_cast<uint32_t>(nkb) * kSfAtom, sfl, pol);
                tma_load_2d(base, &tmA, kt * 128, m_tile * 128, full, pol);
            }
        };
        const int pre = min(kStages, steps);
        Walk wk = walk_start();
        for (int st = 0; st < pre; ++st, walk_next(wk)) {
            expect(st, wk);
            issue_w(st, wk);
        }
        pdl_wait();  // A and its scales come from the previous kernel
        {
            Walk wa = walk_start();
            for (int st = 0; st < pre; ++st, walk_next(wa)) issue_a(st, wa);
        }
        int issued = pre;
        for (int st = pre; st < steps; ++st) {
            const int s = st % kStages, use = st / kStages;
            bool ok = true;
            if (lane == 0)
                ok = mbar_wait(bar_empty + 8 * s, (use - 1) & 1, abort_flag, p.status, kStatusTimeoutEmpty);
            if (!__shfl_sync(0xffffffffu, ok ? 1 : 0, 0)) break;
            expect(st, wk);
            issue_w(st, wk);
            issue_a(st, wk);
            issued = st + 1;
            walk_next(wk);
        }
        // every issued stage must have landed before the CTA may exit
        if (lane == 0)
            for (int st = max(0, issued - kStages); st < issued; ++st) {
                drain_wait(bar_full + 8 * (st % kStages), (st / kStages) & 1, p.status);
                drain_wait(bar_sfl + 8 * (st % kStages), (st / kStages) & 1, p.status);
            }
    } else if (warp == 1) {
        if (lane == 0) {
            // ------------------------------ MMA issuer ------------------------------
            constexpr uint32_t idesc = idesc_mxf4nvf4(128, BN);
            int st = 0;
            for (int i = 0; i < my_tiles; ++i) {
                if (i > 0 && !mbar_wait(bar_acce, (i - 1) & 1, abort_flag, p.status, kStatusTimeoutAccum))
                    break;
                tc_fence_after();
                bool ok = true;
                const int kt0 = kt_begin_of(unit_of(i) / tiles), cnt = kt_count_of(unit_of(i) / tiles);
                for (int j = 0; j < cnt; ++j, ++st) {
                    const int s = st % kStages, slot = st % kSlots, kt = kt0 + j;
                    if (!mbar_wait(bar_full + 8 * s, (st / kStages) & 1, abort_flag, p.status, kStatusTimeoutFull) ||
                        !mbar_wait(bar_sfr + 8 * slot, (st / kSlots) & 1, abort_flag, p.status, kStatusTimeoutFull)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const int nkb = nkb_of(kt);
                    const uint32_t base = sbase + s * kStage;
                    const uint32_t t_sf = tmem + kColSf + slot * kSfSlot;
                    for (int kb = 0; kb < nkb; ++kb)
                        tc_mma_mxf4nvf4(tmem, desc_kmajor_sw128(base + 32 * kb), desc_kmajor_sw128(base + kOffB + 32 * kb),
                                        idesc, t_sf + 4 * kb, t_sf + 16 + 4 * kGroups * kb,
                                        (j > 0 || kb > 0) ? 1u : 0u);
                    tc_commit(bar_empty + 8 * s);     // frees the stage once these MMAs have read it
                    tc_commit(bar_sff + 8 * slot);    // and the scale slot
                }
                tc_commit(bar_accf);  // always: completion of every MMA issued above
                if (!ok) break;
            }
        }
    } else if (warp >= 10) {
        if (lane == 0) {
            // --------------------------- scale copiers (warps 10, 11) ---------------------------
            // tcgen05.cp issued from one thread run one after another; spread over two warps they
            // overlap, and with two scale slots they overlap the MMAs of the previous stage too.
            // Copier c takes k-blocks 2c and 2c + 1 of every stage.
            const int c = warp - 10;
            Walk wk = walk_start();
            for (int st = 0; st < steps; ++st, walk_next(wk)) {
                const int s = st % kStages, slot = st % kSlots, kt = wk.kt0 + wk.j;
                if (!mbar_wait(bar_sfl + 8 * s, (st / kStages) & 1, abort_flag, p.status, kStatusTimeoutFull))
                    break;
                if (st >= kSlots && !mbar_wait(bar_sff + 8 * slot, (st / kSlots - 1) & 1, abort_flag, p.status,
                                          kStatusTimeoutFull))
                    break;
                tc_fence_after();
                const int nkb = nkb_of(kt);
                const uint32_t base = sbase + s * kStage;
                const uint32_t t_sf = tmem + kColSf + slot * kSfSlot;
                for (int kb = 2 * c; kb < 2 * c + 2 && kb < nkb; ++kb) {
                    tc_cp_32x128b_warpx4(t_sf + 4 * kb, desc_sf_32x128b(base + kOffSfa + kb * kSfAtom));
#pragma unroll
                    for (int g = 0; g < kGroups; ++g)
                        tc_cp_32x128b_warpx4(t_sf + 16 + 4 * kGroups * kb + 4 * g,
                                             desc_sf_32x128b(base + kOffSfb + g * 4 * kSfAtom + kb * kSfAtom));
                }
                tc_commit(bar_sfr + 8 * slot);  // arrives when this warp's copies have landed
            }
        }
    } else {
        // ------------------------------ epilogue (warps 2..9) ------------------------------
        const int q = warp & 3;            // TMEM sub-partition this warp may read
        const int half = (warp - 2) >> 2;  // which half of the BN columns
        constexpr int kChunks = BN / 64;   // 32-column chunks per thread
        const int row = q * 32 + lane;
        const int e = threadIdx.x - 64;
        uint8_t *const stage = smem + Cf::kOffStaging + (warp - 2) * 1024;
        pdl_wait();  // residuals may come from the previous kernel
        for (int i = 0; i < my_tiles; ++i) {
            const int t = tile_of(i);
            const int m_tile = t % m_tiles, n_tile = t / m_tiles;
            const bool got =
                e != 0 || mbar_wait(bar_accf, i & 1, abort_flag, p.status, kStatusTimeoutAccum);
            if (!bar_epi_and(got && *abort_flag == 0)) break;
            tc_fence_after();
            const uint32_t t_row =
                tmem + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(half * (BN / 2));
            const int m = m_tile * 128 + row;
            const int n = n_tile * BN + half * (BN / 2);
            if constexpr (!SPLIT) {
                if (i + 1 < my_tiles) {
                    // another tile follows: drain the accumulator at once and hand it back, so
                    // this epilogue runs under the next tile's MMAs
                    uint32_t r[kChunks][32];
#pragma unroll
                    for (int c = 0; c < kChunks; ++c) tmem_ld_32x32b_x32(t_row + 32 * c, r[c]);
                    tmem_ld_wait();
                    tc_fence_before();
                    bar_epi_and(true);
                    if (e == 0) mbar_arrive(bar_acce);  // the MMA warp may start the next tile
                    if (m < p.M) {
#pragma unroll
                        for (int c = 0; c < kChunks; ++c) {
                            float v[32];
#pragma unroll
                            for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[c][j]);
                            epilogue_chunk<32, EPI>(p, m, n + 32 * c, v);
                        }
                    }
                } else {
                    // the CTA's last tile: nothing runs under its epilogue, which is the launch's
                    // tail; read the accumulator a chunk at a time (few registers live) and
                    // store through the staging buffer
#pragma unroll 1
                    for (int c = 0; c < kChunks; ++c) {
                        uint32_t a[32];
                        tmem_ld_32x32b_x32(t_row + 32 * c, a);
                        tmem_ld_wait();
                        float v[32];
#pragma unroll
                        for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(a[j]);
                        chunk_out<EPI>(p, m - lane, lane, n + 32 * c, v, stage);
                    }
                    tc_fence_before();
                    bar_epi_and(true);
                    if (e == 0) mbar_arrive(bar_acce);
                }
                continue;
            }
            // Split K in two, arrive then publish: a split takes the tile's arrival ticket first.
            // The first to arrive copies its fp32 partial to the workspace in the threads' own
            // order (float4 (c, j) of epilogue thread e at ((split * tiles + t) * 8 kChunks +
            // 8 c + j) * 256 + e: a warp's store covers 512 contiguous bytes) and counts itself
            // published.  The second reduces: it waits (bounded) for that count, which the first
            // sets without waiting on anything, and adds the partial to its own accumulator read
            // straight from tensor memory.
            const int split = unit_of(i) / tiles;
            constexpr int kVec = kChunks * 8;  // float4 per thread
            float4 *part = reinterpret_cast<float4 *>(p.partials) + static_cast<size_t>(t) * kVec * 256 + e;
            const size_t split_stride = static_cast<size_t>(tiles) * kVec * 256;
            if (e == 0) misc[2] = atomicAdd(p.tickets + 2 * t, 1u);
            bar_epi_and(true);
            if (misc[2] == 0u) {  // first to arrive: publish
                uint32_t r[kChunks][32];
#pragma unroll
                for (int c = 0; c < kChunks; ++c) tmem_ld_32x32b_x32(t_row + 32 * c, r[c]);
                tmem_ld_wait();
                tc_fence_before();
                bar_epi_and(true);
                if (e == 0) mbar_arrive(bar_acce);  // the MMA warp may start the next tile
                if (m < p.M) {
#pragma unroll
                    for (int c = 0; c < kChunks; ++c)
#pragma unroll
                        for (int j = 0; j < 8; ++j)
                            __stcg(part + split * split_stride + (8 * c + j) * 256,
                                   make_float4(__uint_as_float(r[c][4 * j]), __uint_as_float(r[c][4 * j + 1]),
                                               __uint_as_float(r[c][4 * j + 2]), __uint_as_float(r[c][4 * j + 3])));
                }
                __threadfence();
                bar_epi_and(true);
                if (e == 0) atomicAdd(p.tickets + 2 * t + 1, 1u);  // published
                continue;
            }
            // the reducer
            const bool pub = e != 0 || wait_published(p.tickets + 2 * t + 1, 1u, abort_flag, p.status);
            if (!bar_epi_and(pub && *abort_flag == 0)) break;
            __threadfence();
            {
                // Every line of the other split's partial this thread will read is prefetched
                // into L1 first, so the chunks' loads do not each wait a round trip to L2.  The
                // prefetches follow the acquire of the published count, and no older copy of a
                // partial line can sit in L1: L1 does not keep global data across launches, and
                // within a launch each line is read once, here.
                const float4 *oth = part + (1 - split) * split_stride;
                if (m < p.M) {
#pragma unroll
                    for (int j = 0; j < kVec; ++j) prefetch_l1(oth + j * 256);
                }
#pragma unroll 1
                for (int c = 0; c < kChunks; ++c) {
                    uint32_t own[32];
                    tmem_ld_32x32b_x32(t_row + 32 * c, own);
                    tmem_ld_wait();
                    float v[32];  // p0 + p1 (IEEE addition commutes: the same bits either way)
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const float4 w = m < p.M ? oth[(8 * c + j) * 256] : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
                        v[4 * j] = __fadd_rn(__uint_as_float(own[4 * j]), w.x);
                        v[4 * j + 1] = __fadd_rn(__uint_as_float(own[4 * j + 1]), w.y);
                        v[4 * j + 2] = __fadd_rn(__uint_as_float(own[4 * j + 2]), w.z);
                        v[4 * j + 3] = __fadd_rn(__uint_as_float(own[4 * j + 3]), w.w);
                    }
                    chunk_out<EPI>(p, m - lane, lane, n + 32 * c, v, stage);
                }
            }
            tc_fence_before();
            bar_epi_and(true);
            if (e == 0) {
                mbar_arrive(bar_acce);  // the MMA warp may start the next tile
                p.tickets[2 * t] = 0u;  // ready for the next call
                p.tickets[2 * t + 1] = 0u;
            }
        }
    }

    // teardown
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
    if (trace != nullptr && threadIdx.x == 0) trace[6] = globaltimer_ns();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

}  // namespace

int gemm_persistent_grid(int M, int n_tiles, int splits) {
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        sms = 148;
    const int units = ((M + 127) / 128) * n_tiles * (splits > 1 ? splits : 1);
    return units < sms ? units : sms;
}

template <int BN, int EPI, bool SPLIT>
static cudaError_t launch_split(const CUtensorMap &ta, const CUtensorMap &tb, const GemmArgs &p, cudaStream_t s) {
    static std::atomic<bool> attr_set[kMaxDevices];
    const cudaError_t e = set_smem_limit_once(reinterpret_cast<const void *>(gemm_persistent_kernel<BN, EPI, SPLIT>),
                                              PCfg<BN>::kSmemBytes, attr_set);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(gemm_persistent_grid(p.M, p.n_tiles, p.splits));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = PCfg<BN>::kSmemBytes;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl_enabled() ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, gemm_persistent_kernel<BN, EPI, SPLIT>, ta, tb, p);
}

template <int BN, int EPI>
static cudaError_t launch_epi(const CUtensorMap &ta, const CUtensorMap &tb, const GemmArgs &p, cudaStream_t s) {
    return p.splits > 1 ? launch_split<BN, EPI, true>(ta, tb, p, s) : launch_split<BN, EPI, false>(ta, tb, p, s);
}

template <int BN>
static cudaError_t launch_bn(const CUtensorMap &ta, const CUtensorMap &tb, const GemmArgs &p, cudaStream_t s) {
    switch (p.epi) {
    case kEpiNone: return launch_epi<BN, kEpiNone>(ta, tb, p, s);
    case kEpiBias: return launch_epi<BN, kEpiBias>(ta, tb, p, s);
    case kEpiResidual: return launch_epi<BN, kEpiResidual>(ta, tb, p, s);
    case kEpiBiasResidual: return launch_epi<BN, kEpiBiasResidual>(ta, tb, p, s);
    case kEpiBiasGelu: return launch_epi<BN, kEpiBiasGelu>(ta, tb, p, s);
    case kEpiGeglu: return launch_epi<BN, kEpiGeglu>(ta, tb, p, s);
    default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_gemm_persistent(const CUtensorMap &ta, const CUtensorMap &tb, const GemmArgs &p, int block_n,
                                   cudaStream_t s) {
    // 1 split of all K tiles, or 2 of k0 and k_tiles - k0 >= 1; a split run needs its tickets
    // and partials
    if (p.splits < 1 || p.splits > 2) return cudaErrorInvalidValue;
    if (p.splits == 1 ? p.kt_per_split != p.k_tiles : (p.kt_per_split < 1 || p.kt_per_split >= p.k_tiles))
        return cudaErrorInvalidValue;
    if (p.splits > 1 && (p.tickets == nullptr || p.partials == nullptr)) return cudaErrorInvalidValue;
    if (block_n == 256) return launch_bn<256>(ta, tb, p, s);
    if (block_n == 128) return launch_bn<128>(ta, tb, p, s);
    return cudaErrorInvalidValue;
}

cudaError_t probe_gemm_persistent() {
    cudaFuncAttributes fa;
    return cudaFuncGetAttributes(&fa, gemm_persistent_kernel<256, kEpiNone, false>);
}

}  // namespace nvfp4
