// executor.cu — the layer executor: a whole program of norm -> NVFP4 and block-scaled GEMM
// ops (e.g. a stack of DiT layers) in ONE persistent cooperative launch.
//
// At M <= 64 tokens a linear layer is a chain of small dependent steps (norm, QKV GEMM,
// attention-output GEMM, norm, FFN up, FFN down).  As separate kernels each step pays a
// grid completion and a launch boundary; here every CTA walks the same program, ops are
// ordered by per-op completion counters in global memory (one release reduction per
// finishing CTA, an acquire poll by the consumers), and the weight tiles of later ops stream
// into each CTA's shared-memory ring while the current op waits for its input -- weights
// never depend on activations.
//
// Roles (256 threads):
//   warp 0      weight producer: TMA loads of W code tiles + bulk loads of their scale atoms,
//               for every GEMM unit of this CTA in program order, as far ahead as the ring
//               allows; they land on the stage's weight barrier.
//   warp 7      weight-scale copier: tcgen05.cp of each stage's W scale atoms into the stage's
//               TMEM scale slot as soon as the weights land (ahead of the activations).
//   warp 2      activation producer: waits until the op's input is complete, TMA loads the A
//               code tiles + scale atoms of the unit (activation barrier), then copies the A
//               scale atoms into the slots as each stage lands.
//   warp 1      MMA issuer: tcgen05.mma kind::mxf4nvf4 block16 into one of two TMEM
//               accumulators once a stage's weights, activations and both scale copies are in.
//   warps 3..6  workers: GEMM epilogues and norm rows.  Split-K partials are pushed to the
//               CTA that owns each column slice (distributed shared memory), which adds them
//               in split order (deterministic) and runs the fused epilogue; a tile that is not
//               split runs its epilogue straight from the accumulator.  A norm op runs one row
//               per CTA on all 128 workers.
// GEMM work: the grid is a set of clusters of C CTAs; for an op split S ways (S | C), the
// S CTAs that share a tile are cluster neighbours.  At start each CTA marks, in a shared-memory
// bit set, the ops it has work in; the roles walk only those (a grouped GEMM of many small
// independent ops gives each CTA a few of them).
// Every wait is bounded (2 s); an expired wait records a device status and unwinds.
#include <cuda.h>
#include <cuda_runtime.h>

#include "epilogue.cuh"
#include "exec.h"
#include "gemm.h"
#include "norm_row.cuh"
#include "quant.cuh"
#include "sm100.cuh"

namespace nvfp4 {

namespace {

constexpr int kThreads = 256;
constexpr int kRing = 6;        // stages; the TMEM scale slot of a stage is the stage's own
constexpr int kStageA = 8192;   // 64 rows x 128 bytes (M <= 64)
constexpr int kStageW = 16384;  // 128 rows x 128 bytes (block_n <= 128)
constexpr int kStageSfa = 2048;
constexpr int kStageSfb = 2048;
constexpr int kStage = kStageA + kStageW + kStageSfa + kStageSfb;
// split-K partials received as a slice owner: S slices x 64 rows x (bn / S + 4) floats
constexpr int kRedBytes = 64 * (128 + 16) * 4;
constexpr int kOffRed = kRing * kStage;
// staged epilogue inputs of this CTA's column slice: residual rows (bf16) and bias
constexpr int kStgLd = 128 + 8;
constexpr int kOffStg = kOffRed + kRedBytes;
constexpr int kStgBytes = 64 * kStgLd * 2;
constexpr int kOffStgBias = kOffStg + kStgBytes;
constexpr int kOffBar = kOffStgBias + 256;
// barriers: full_w[R], full_a[R], empty[R], sf_ready[R], acc_full[2], acc_empty[2]
constexpr int kOffMisc = kOffBar + (4 * kRing + 4) * 8;
// misc words: [0] TMEM base, [1] abort flag, [2] red_in (partial slices received as an
// owner), [3] red_free (owners done with this CTA's partials), [4..11] four doubles (norm rows)
constexpr int kOffMask = kOffMisc + 64;  // one bit per op: this CTA has work in it
constexpr int kSmemBytes = kOffMask + kExecMaxOps / 8 + 1024;
constexpr int kTmemCols = 512;  // two 128-column accumulators + kRing scale slots
constexpr int kColSf = 256;     // scale slot j: A atoms at kColSf + 32 j, W atoms 16 columns on
constexpr int kSfSlot = 32;
constexpr int kSfAtom = 512;
static_assert(kSmemBytes <= 232448, "shared memory per CTA");
static_assert(kColSf + kRing * kSfSlot <= kTmemCols, "tensor memory columns");

__device__ __forceinline__ unsigned int ld_acquire_cluster_smem(uint32_t addr) {
    unsigned int v;
    asm volatile("ld.acquire.cluster.shared::cta.u32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
    return v;
}
__device__ __forceinline__ void red_add_release_cluster(uint32_t cluster_addr, unsigned int v) {
    asm volatile("red.release.cluster.shared::cluster.add.u32 [%0], %1;" ::"r"(cluster_addr), "r"(v) : "memory");
}
// Completion of an op by this CTA: one release reduction at GPU scope (it orders the CTA's
// earlier stores, which the named barrier before it made visible to this thread).
__device__ __forceinline__ void red_add_release_gpu(unsigned int *p, unsigned int v) {
    asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ void fence_proxy_async_global() {
    asm volatile("fence.proxy.async.global;" ::: "memory");
}
__device__ __forceinline__ void bar_epi() { asm volatile("bar.sync 1, 128;" ::: "memory"); }
// Barrier of the 128 worker threads that also ANDs a flag across them: every decision to
// abandon the work is taken by all four warps together (a named barrier has no timeout, so
// no warp may leave while the others still expect it).
__device__ __forceinline__ bool bar_epi_and(bool v) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.and.pred q, 1, 128, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"(static_cast<uint32_t>(v))
        : "memory");
    return r != 0;
}

// Bounded wait until *p >= target (acquire, gpu scope): a tight poll first, then a short
// back-off.
__device__ bool wait_counter(const unsigned int *p, unsigned int target, volatile int *abort_flag, uint32_t *status) {
    for (int i = 0; i < 256; ++i)
        if (ld_acquire_gpu(p) >= target) return true;
    const uint64_t t0 = globaltimer_ns();
    while (true) {
        __nanosleep(32);
        if (ld_acquire_gpu(p) >= target) return true;
        if (*abort_flag) return false;
        if (globaltimer_ns() - t0 > kWaitLimitNs) {
            atomicCAS(status, static_cast<uint32_t>(kStatusOk), static_cast<uint32_t>(kStatusTimeoutOp));
            *abort_flag = 1;
            return false;
        }
    }
}
// Bounded wait until the local shared-memory counter at `addr` >= target (acquire, cluster).
__device__ bool wait_smem_counter(uint32_t addr, unsigned int target, volatile int *abort_flag, uint32_t *status) {
    if (ld_acquire_cluster_smem(addr) >= target) return true;
    const uint64_t t0 = globaltimer_ns();
    while (true) {
        if (ld_acquire_cluster_smem(addr) >= target) return true;
        if (*abort_flag) return false;
        if (globaltimer_ns() - t0 > kWaitLimitNs) {
            atomicCAS(status, static_cast<uint32_t>(kStatusOk), static_cast<uint32_t>(kStatusTimeoutPeer));
            *abort_flag = 1;
            return false;
        }
    }
}

struct Unit {
    int tile, split, kt0, kt1, owner_rank;
};

__device__ __forceinline__ int op_rounds(const ExecOp &op, int teams, int C) {
    const int per_round = teams * (C / op.splits);
    return (op.n_tiles + per_round - 1) / per_round;
}
// The GEMM unit of (team, rank) in round r, if any.  owner_rank: the cluster rank of the
// group's split 0 (the group's CTAs are owner_rank .. owner_rank + splits - 1).
__device__ __forceinline__ bool op_unit(const ExecOp &op, int team, int rank, int teams, int C, int r, Unit &u) {
    const int per_team = C / op.splits;
    const int t = team >= op.team0 ? team - op.team0 : team - op.team0 + teams;  // rotated team index
    const int tile = (r * teams + t) * per_team + rank / op.splits;
    if (tile >= op.n_tiles) return false;
    u.tile = tile;
    u.split = rank % op.splits;
    u.kt0 = u.split * op.kt_per_split;
    u.kt1 = min(op.k_tiles, u.kt0 + op.kt_per_split);
    u.owner_rank = (rank / op.splits) * op.splits;
    return true;
}

// Whether CTA (team, rank) has any work in op i: a norm row, or a GEMM unit in round 0
// (later rounds only add tiles to CTAs that have one in round 0).
__device__ __forceinline__ bool has_work(const ExecOp &op, int team, int rank, int teams, int C) {
    if (op.type == kOpNorm) return static_cast<int>(blockIdx.x) < op.norm.M;
    Unit u;
    return op_unit(op, team, rank, teams, C, 0, u);
}
// The first op after op i that this CTA has work in (n_ops if none).
__device__ __forceinline__ int next_op(const uint32_t *mask, int n_ops, int i) {
    for (int j = i + 1; j < n_ops; j = (j | 31) + 1) {
        const uint32_t bits = mask[j >> 5] >> (j & 31);
        if (bits != 0u) return j + __ffs(static_cast<int>(bits)) - 1;
    }
    return n_ops;
}

// One norm row on the 128 workers (thread e of them), kept out of line: the norm path has its
// own register allocation, apart from the epilogue's.
template <int BPT>
__device__ __noinline__ void norm_row_bpt(const NormArgs &a, int row, int e, double *red) {
    norm_row<128, BPT, false>(a, row, e, red);
}
__device__ void norm_row_any(const NormArgs &a, int bpt, int row, int e, double *red) {
    switch (bpt) {
    case 1: norm_row_bpt<1>(a, row, e, red); break;
    case 2: norm_row_bpt<2>(a, row, e, red); break;
    case 3: norm_row_bpt<3>(a, row, e, red); break;
    case 4: norm_row_bpt<4>(a, row, e, red); break;
    case 5: norm_row_bpt<5>(a, row, e, red); break;
    case 6: norm_row_bpt<6>(a, row, e, red); break;
    case 7: norm_row_bpt<7>(a, row, e, red); break;
    default: norm_row_bpt<8>(a, row, e, red); break;
    }
}

__global__ void __launch_bounds__(kThreads, 1) exec_kernel(const ExecParams P) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const uint32_t bar_fw = sbase + kOffBar;         // R: the stage's weights + weight scales landed
    const uint32_t bar_fa = bar_fw + 8 * kRing;      // R: the stage's activations + their scales landed
    const uint32_t bar_empty = bar_fa + 8 * kRing;   // R: the stage's MMAs are done with it (and its slot)
    const uint32_t bar_sfr = bar_empty + 8 * kRing;  // R: both scale copies of the stage are in TMEM
    const uint32_t bar_accf = bar_sfr + 8 * kRing;
    const uint32_t bar_acce = bar_accf + 16;
    uint32_t *opmask = reinterpret_cast<uint32_t *>(smem + kOffMask);
    volatile uint32_t *misc = reinterpret_cast<volatile uint32_t *>(smem + kOffMisc);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(misc + 1);
    const uint32_t red_in_addr = sbase + kOffMisc + 8;
    const uint32_t red_free_addr = sbase + kOffMisc + 12;
    double *norm_red = reinterpret_cast<double *>(smem + kOffMisc + 16);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int C = P.cluster;
    const int rank = static_cast<int>(cluster_ctarank());
    const int team = blockIdx.x / C;
    const int teams = gridDim.x / C;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kRing; ++s) {
            mbar_init(bar_fw + 8 * s, 1);
            mbar_init(bar_fa + 8 * s, 1);
            mbar_init(bar_empty + 8 * s, 1);
            mbar_init(bar_sfr + 8 * s, 2);  // the weight-scale copier and the activation producer
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(bar_accf + 8 * b, 1);
            mbar_init(bar_acce + 8 * b, 1);
        }
        misc[1] = 0;
        misc[2] = 0;
        misc[3] = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(const_cast<uint32_t *>(misc)), kTmemCols);
        tmem_relinquish();
    }
    // the ops this CTA has work in: one bit per op, 32 ops per warp ballot
    for (int w = warp; w < (P.n_ops + 31) / 32; w += kThreads / 32) {
        const int i = 32 * w + lane;
        const bool mine = i < P.n_ops && has_work(P.ops[i], team, rank, teams, C);
        const uint32_t bits = __ballot_sync(0xffffffffu, mine);
        if (lane == 0) opmask[w] = bits;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    cluster_sync_all();  // every CTA's counters are initialised before any remote update
    const uint32_t tmem = misc[0];

    auto nkb_of = [&](const ExecOp &op, int kt) { return min(4, op.k_atoms - 4 * kt); };
    // diagnostics: per (op, CTA) [0] W issued first tile, [1] A dependency seen, [2] first
    // stage full (MMA), [3] last MMA issued, [4] accumulator ready, [5] partials in (split
    // groups), [6] op signalled, [7] norm rows done / accumulator drained (GEMM)
    auto stamp = [&](int op_i, int k) {
        if (P.trace != nullptr) P.trace[(static_cast<size_t>(op_i) * gridDim.x + blockIdx.x) * 8 + k] = globaltimer_ns();
    };

    if (warp == 0 && lane == 0) {
        // ---------------------------- weight producer ----------------------------
        const uint64_t pol = policy_evict_first();
        int step = 0;
        for (int i = next_op(opmask, P.n_ops, -1); i < P.n_ops; i = next_op(opmask, P.n_ops, i)) {
            const ExecOp &op = P.ops[i];  // read in place: a local copy would live in (L1-starved) local memory
            if (op.type != kOpGemm) continue;
            const CUtensorMap *tmB = P.maps + op.tm_b;
            const int rounds = op_rounds(op, teams, C);
            for (int r = 0; r < rounds; ++r) {
                Unit u;
                if (!op_unit(op, team, rank, teams, C, r, u)) continue;
                for (int kt = u.kt0; kt < u.kt1; ++kt, ++step) {
                    const int slot = step % kRing, use = step / kRing;
                    if (use > 0 && !mbar_wait(bar_empty + 8 * slot, (use - 1) & 1, abort_flag, P.status,
                                              kStatusTimeoutEmpty))
                        goto done_w;
                    const uint32_t nb = static_cast<uint32_t>(nkb_of(op, kt)) * kSfAtom;
                    const uint32_t full = bar_fw + 8 * slot;
                    const uint32_t st = sbase + slot * kStage;
                    if (kt == u.kt0) stamp(i, 0);
                    mbar_arrive_expect_tx(full, static_cast<uint32_t>(op.bn) * 128u + nb);
                    tma_load_2d(st + kStageA, tmB, kt * 128, u.tile * op.bn, full, pol);
                    const size_t grp = static_cast<size_t>((u.tile * op.bn) / 128);
                    bulk_load(st + kStageA + kStageW + kStageSfa, op.sfb + (grp * op.k_atoms + 4 * kt) * kSfAtom, nb,
                              full, pol);
                }
            }
        }
    done_w:;
    } else if (warp == 7 && lane == 0) {
        // ---------------------------- weight-scale copier ----------------------------
        // The W scale atoms of a stage go into the stage's TMEM slot as soon as they land.  The
        // slot is free then: the stage was released (its MMAs done) before these weights were
        // loaded into it.
        int step = 0;
        for (int i = next_op(opmask, P.n_ops, -1); i < P.n_ops; i = next_op(opmask, P.n_ops, i)) {
            const ExecOp &op = P.ops[i];  // read in place: a local copy would live in (L1-starved) local memory
            if (op.type != kOpGemm) continue;
            const int rounds = op_rounds(op, teams, C);
            for (int r = 0; r < rounds; ++r) {
                Unit u;
                if (!op_unit(op, team, rank, teams, C, r, u)) continue;
                for (int kt = u.kt0; kt < u.kt1; ++kt, ++step) {
                    const int slot = step % kRing, use = step / kRing;
                    if (!mbar_wait(bar_fw + 8 * slot, use & 1, abort_flag, P.status, kStatusTimeoutFull))
                        goto done_c;
                    tc_fence_after();
                    const int nkb = nkb_of(op, kt);
                    const uint32_t st = sbase + slot * kStage;
                    const uint32_t t_sf = tmem + kColSf + slot * kSfSlot;
                    for (int kb = 0; kb < nkb; ++kb)
                        tc_cp_32x128b_warpx4(t_sf + 16 + 4 * kb,
                                             desc_sf_32x128b(st + kStageA + kStageW + kStageSfa + kb * kSfAtom));
                    tc_commit(bar_sfr + 8 * slot);  // arrives once the copies have landed
                }
            }
        }
    done_c:;
    } else if (warp == 2 && lane == 0) {
        // ---------------------------- activation producer ----------------------------
        // Per unit: every A stage is requested at once, then each stage's A scale atoms are
        // copied into its TMEM slot as it lands.
        const uint64_t pol = policy_evict_last();
        int step = 0;
        for (int i = next_op(opmask, P.n_ops, -1); i < P.n_ops; i = next_op(opmask, P.n_ops, i)) {
            const ExecOp &op = P.ops[i];  // read in place: a local copy would live in (L1-starved) local memory
            if (op.type != kOpGemm) continue;
            const CUtensorMap *tmA = P.maps + op.tm_a;
            bool ready = false;
            const int rounds = op_rounds(op, teams, C);
            for (int r = 0; r < rounds; ++r) {
                Unit u;
                if (!op_unit(op, team, rank, teams, C, r, u)) continue;
                if (!ready) {
                    if (op.dep >= 0 && !wait_counter(P.done + op.dep, P.ops[op.dep].units, abort_flag, P.status)) goto done_a;
                    fence_proxy_async_global();  // the input was written through the generic proxy
                    ready = true;
                    stamp(i, 1);
                }
                // batches of at most kRing stages: a stage is reused only after its MMAs, which
                // wait for the scale copies this thread makes after the batch's loads
                for (int kb0 = u.kt0; kb0 < u.kt1; kb0 += kRing) {
                    const int kb1 = min(u.kt1, kb0 + kRing), step0 = step;
                    for (int kt = kb0; kt < kb1; ++kt, ++step) {
                        const int slot = step % kRing, use = step / kRing;
                        if (use > 0 && !mbar_wait(bar_empty + 8 * slot, (use - 1) & 1, abort_flag, P.status,
                                                  kStatusTimeoutEmpty))
                            goto done_a;
                        const uint32_t nb = static_cast<uint32_t>(nkb_of(op, kt)) * kSfAtom;
                        const uint32_t full = bar_fa + 8 * slot;
                        const uint32_t st = sbase + slot * kStage;
                        mbar_arrive_expect_tx(full, op.a_box_rows * 128u + nb);
                        tma_load_2d(st, tmA, kt * 128, 0, full, pol);
                        bulk_load(st + kStageA + kStageW, op.sfa + static_cast<size_t>(4 * kt) * kSfAtom, nb, full,
                                  pol);
                    }
                    step = step0;
                    for (int kt = kb0; kt < kb1; ++kt, ++step) {
                        const int slot = step % kRing, use = step / kRing;
                        if (!mbar_wait(bar_fa + 8 * slot, use & 1, abort_flag, P.status, kStatusTimeoutFull))
                            goto done_a;
                        tc_fence_after();
                        const int nkb = nkb_of(op, kt);
                        const uint32_t st = sbase + slot * kStage;
                        const uint32_t t_sf = tmem + kColSf + slot * kSfSlot;
                        for (int kb = 0; kb < nkb; ++kb)
                            tc_cp_32x128b_warpx4(t_sf + 4 * kb, desc_sf_32x128b(st + kStageA + kStageW + kb * kSfAtom));
                        tc_commit(bar_sfr + 8 * slot);
                    }
                }
            }
        }
    done_a:;
    } else if (warp == 1 && lane == 0) {
        // ---------------------------- MMA issuer ----------------------------
        int step = 0, unit_idx = 0;
        for (int i = next_op(opmask, P.n_ops, -1); i < P.n_ops; i = next_op(opmask, P.n_ops, i)) {
            const ExecOp &op = P.ops[i];  // read in place: a local copy would live in (L1-starved) local memory
            if (op.type != kOpGemm) continue;
            const uint32_t idesc = idesc_mxf4nvf4(128, op.bn);
            const int rounds = op_rounds(op, teams, C);
            for (int r = 0; r < rounds; ++r) {
                Unit u;
                if (!op_unit(op, team, rank, teams, C, r, u)) continue;
                const int b = unit_idx & 1, acc_use = unit_idx >> 1;
                if (acc_use > 0 && !mbar_wait(bar_acce + 8 * b, (acc_use - 1) & 1, abort_flag, P.status,
                                              kStatusTimeoutAccum))
                    goto done_m;
                tc_fence_after();
                const uint32_t t_acc = tmem + static_cast<uint32_t>(b * 128);
                // a 64-row W tile reads its half of the 128-row scale atom
                const uint32_t sub = (op.bn == 64) ? static_cast<uint32_t>(((u.tile * op.bn) & 127) >> 5) : 0u;
                for (int kt = u.kt0; kt < u.kt1; ++kt, ++step) {
                    const int slot = step % kRing, use = step / kRing;
                    if (!mbar_wait(bar_fw + 8 * slot, use & 1, abort_flag, P.status, kStatusTimeoutFull) ||
                        !mbar_wait(bar_fa + 8 * slot, use & 1, abort_flag, P.status, kStatusTimeoutFull) ||
                        !mbar_wait(bar_sfr + 8 * slot, use & 1, abort_flag, P.status, kStatusTimeoutFull))
                        goto done_m;
                    tc_fence_after();
                    if (kt == u.kt0) stamp(i, 2);
                    const int nkb = nkb_of(op, kt);
                    const uint32_t st = sbase + slot * kStage;
                    const uint32_t t_sf = tmem + kColSf + slot * kSfSlot;
                    for (int kb = 0; kb < nkb; ++kb)
                        tc_mma_mxf4nvf4(t_acc, desc_kmajor_sw128(st + 32 * kb), desc_kmajor_sw128(st + kStageA + 32 * kb),
                                        idesc, t_sf + 4 * kb, t_sf + 16 + 4 * kb + sub, (kt > u.kt0 || kb > 0) ? 1u : 0u);
                    tc_commit(bar_empty + 8 * slot);  // the stage and its scale slot, once these MMAs are done
                }
                stamp(i, 3);
                tc_commit(bar_accf + 8 * b);
                ++unit_idx;
            }
        }
    done_m:;
    } else if (warp >= 3 && warp <= 6) {
        // ---------------------------- workers: epilogues and norm rows ----------------------------
        const int e = threadIdx.x - 96;  // 0..127
        const int q = warp & 3;          // TMEM sub-partition this warp reads
        const int row = q * 32 + lane;
        int unit_idx = 0;
        unsigned int in_expected = 0, free_expected = 0;  // split-group signals expected so far
        for (int i = next_op(opmask, P.n_ops, -1); i < P.n_ops; i = next_op(opmask, P.n_ops, i)) {
            const ExecOp &op = P.ops[i];  // read in place: a local copy would live in (L1-starved) local memory
            if (op.type == kOpNorm) {
                // one row at a time on all 128 workers: rows blockIdx.x, blockIdx.x + grid, ...
                const bool ok = (e != 0) || op.dep < 0 || wait_counter(P.done + op.dep, P.ops[op.dep].units, abort_flag, P.status);
                if (!bar_epi_and(ok)) goto done_e;
                if (e == 0) stamp(i, 1);
                for (int rr = blockIdx.x; rr < op.norm.M; rr += gridDim.x) norm_row_any(op.norm, op.bpt, rr, e, norm_red);
                bar_epi();
                if (e == 0) {
                    if (op.signal) red_add_release_gpu(P.done + i, 1u);
                    stamp(i, 7);
                }
                continue;
            }
            // GEMM op.  CTA k of a split group owns column slice k (bn / S columns, a multiple of
            // 32) of the group's tile: every CTA pushes its partial of slice k to CTA k, which
            // adds the S partials in split order and runs the epilogue of its slice.
            const int rounds = op_rounds(op, teams, C);
            const int S = op.splits;
            const int slice = op.bn / S;
            const int chunks = slice / 32;
            const int red_ld = slice + 4;
            const bool has_bias = op.bias != nullptr && (op.epi == kEpiBias || op.epi == kEpiBiasResidual ||
                                                         op.epi == kEpiBiasGelu || op.epi == kEpiGeglu);
            const bool has_res = op.residual != nullptr && (op.epi == kEpiResidual || op.epi == kEpiBiasResidual);
            const int rows_valid = min(64, op.M);
            uint16_t *stg = reinterpret_cast<uint16_t *>(smem + kOffStg);
            uint16_t *stg_bias = reinterpret_cast<uint16_t *>(smem + kOffStgBias);
            float *red = reinterpret_cast<float *>(smem + kOffRed);
            bool dep_seen = false;
            for (int r = 0; r < rounds; ++r) {
                Unit u;
                if (!op_unit(op, team, rank, teams, C, r, u)) continue;
                if (!dep_seen) {
                    // the epilogue reads residuals written by earlier ops: acquire here too
                    const bool ok =
                        (e != 0) || op.dep < 0 || wait_counter(P.done + op.dep, P.ops[op.dep].units, abort_flag, P.status);
                    if (!bar_epi_and(ok)) goto done_e;
                    dep_seen = true;
                }
                const int n0 = u.tile * op.bn;
                const int c0 = u.split * slice;  // first column of this CTA's slice, in the tile
                // stage the slice's residual rows and bias while the MMAs run
                if (has_res) {
                    const int per_row = slice / 8;
                    for (int idx = e; idx < rows_valid * per_row; idx += 128) {
                        const int rr = idx / per_row, c8 = idx % per_row;
                        const uint4 val = __ldcg(reinterpret_cast<const uint4 *>(
                            op.residual + static_cast<size_t>(rr) * op.ldr + n0 + c0 + 8 * c8));
                        *reinterpret_cast<uint4 *>(stg + rr * kStgLd + 8 * c8) = val;
                    }
                }
                if (has_bias && e < slice / 8)
                    *reinterpret_cast<uint4 *>(stg_bias + 8 * e) =
                        __ldg(reinterpret_cast<const uint4 *>(op.bias + n0 + c0 + 8 * e));
                // before pushing into the group's buffers: every owner is done with this CTA's
                // previous partials (one thread waits; the barrier orders the others after it)
                if (!bar_epi_and(e != 0 || S == 1 || free_expected == 0 ||
                                 wait_smem_counter(red_free_addr, free_expected, abort_flag, P.status)))
                    goto done_e;
                const int b = unit_idx & 1, acc_use = unit_idx >> 1;
                const bool got = mbar_wait(bar_accf + 8 * b, acc_use & 1, abort_flag, P.status,
                                           kStatusTimeoutAccum);
                if (!bar_epi_and(got)) goto done_e;
                tc_fence_after();
                if (e == 0) stamp(i, 4);
                const uint32_t t_row = tmem + static_cast<uint32_t>(b * 128) + (static_cast<uint32_t>(q * 32) << 16);
                if (S == 1) {
                    // the whole tile is this CTA's: the epilogue straight from the accumulator
                    if (q * 32 < rows_valid) {  // warp-uniform: tcgen05.ld is .sync.aligned
                        for (int cc = 0; cc < op.bn; cc += 32) {
                            uint32_t rg[32];
                            tmem_ld_32x32b_x32(t_row + cc, rg);
                            tmem_ld_wait();
                            if (row < rows_valid) {
                                float v[32];
#pragma unroll
                                for (int t = 0; t < 32; ++t) v[t] = __uint_as_float(rg[t]);
                                epilogue_chunk_src(op, row, n0 + cc, v, has_bias ? stg_bias + cc : nullptr,
                                                   has_res ? stg + row * kStgLd + cc : nullptr);
                            }
                        }
                    }
                    tc_fence_before();
                    bar_epi();
                    if (e == 0) {
                        mbar_arrive(bar_acce + 8 * b);  // the accumulator is free again
                        stamp(i, 7);
                    }
                } else {
                    // push: chunk cc goes to slice owner owner_rank + cc / slice, as split u.split
                    if (q * 32 < rows_valid) {
                        for (int cc = 0; cc < op.bn; cc += 32) {
                            uint32_t rg[32];
                            tmem_ld_32x32b_x32(t_row + cc, rg);
                            tmem_ld_wait();
                            if (row < rows_valid) {
                                const int k = cc / slice;
                                const uint32_t dst = mapa_shared(
                                    smem_u32(red + (u.split * 64 + row) * red_ld + (cc - k * slice)),
                                    static_cast<uint32_t>(u.owner_rank + k));
#pragma unroll
                                for (int j = 0; j < 8; ++j)
                                    st_dsmem_f4(dst + 16 * j,
                                                make_float4(__uint_as_float(rg[4 * j]), __uint_as_float(rg[4 * j + 1]),
                                                            __uint_as_float(rg[4 * j + 2]),
                                                            __uint_as_float(rg[4 * j + 3])));
                            }
                        }
                    }
                    tc_fence_before();
                    bar_epi();
                    if (e == 0) {
                        mbar_arrive(bar_acce + 8 * b);  // the accumulator is free again
                        stamp(i, 7);
                        for (int k = 0; k < S; ++k)
                            red_add_release_cluster(mapa_shared(red_in_addr, static_cast<uint32_t>(u.owner_rank + k)), 1u);
                    }
                    in_expected += static_cast<unsigned>(S);
                    if (!bar_epi_and(e != 0 || wait_smem_counter(red_in_addr, in_expected, abort_flag, P.status)))
                        goto done_e;
                    if (e == 0) stamp(i, 5);
                    for (int item = e;; item += 128) {
                        const int i_row = item / chunks, ch = item % chunks;
                        if (i_row >= rows_valid) break;
                        float v[32];
#pragma unroll
                        for (int t = 0; t < 32; ++t) v[t] = 0.0f;
                        for (int sp = 0; sp < S; ++sp) {
                            const float4 *src4 = reinterpret_cast<const float4 *>(red + (sp * 64 + i_row) * red_ld + 32 * ch);
#pragma unroll
                            for (int j = 0; j < 8; ++j) {
                                const float4 w4 = src4[j];
                                v[4 * j] = __fadd_rn(v[4 * j], w4.x);
                                v[4 * j + 1] = __fadd_rn(v[4 * j + 1], w4.y);
                                v[4 * j + 2] = __fadd_rn(v[4 * j + 2], w4.z);
                                v[4 * j + 3] = __fadd_rn(v[4 * j + 3], w4.w);
                            }
                        }
                        epilogue_chunk_src(op, i_row, n0 + c0 + 32 * ch, v, has_bias ? stg_bias + 32 * ch : nullptr,
                                           has_res ? stg + i_row * kStgLd + 32 * ch : nullptr);
                    }
                    bar_epi();
                    if (e == 0)  // this CTA is done with the group's partials of this unit
                        for (int k = 0; k < S; ++k)
                            red_add_release_cluster(mapa_shared(red_free_addr, static_cast<uint32_t>(u.owner_rank + k)),
                                                    1u);
                    free_expected += static_cast<unsigned>(S);
                }
                if (e == 0) {
                    if (op.signal) red_add_release_gpu(P.done + i, 1u);  // only ops a later op waits for
                    stamp(i, 6);
                }
                ++unit_idx;
            }
        }
    done_e:;
    }

    // teardown: peers may still write this CTA's shared memory until everyone is done
    __syncwarp();
    if (*abort_flag) {
        // an abandoned run may leave copies or MMAs in flight: give them time to land
        // before shared and tensor memory are released
        const uint64_t t0 = globaltimer_ns();
        while (globaltimer_ns() - t0 < 200000ull) {
        }
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync_all();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

}  // namespace

cudaError_t exec_grid(int cluster, int *grid) {
    cudaError_t e = cudaFuncSetAttribute(exec_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(cluster);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = kSmemBytes;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = static_cast<unsigned>(cluster);
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    e = cudaOccupancyMaxActiveClusters(&n, exec_kernel, &cfg);
    if (e != cudaSuccess) return e;
    *grid = n * cluster;
    return n > 0 ? cudaSuccess : cudaErrorInvalidConfiguration;
}

cudaError_t exec_launch(const ExecParams &p, int grid, cudaStream_t s) {
    cudaError_t e = cudaFuncSetAttribute(exec_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = kSmemBytes;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = static_cast<unsigned>(p.cluster);
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeCooperative;  // CTAs wait on one another: all must be resident
    attr[1].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, exec_kernel, p);
}

cudaError_t probe_exec_kernel() {
    cudaFuncAttributes fa;
    return cudaFuncGetAttributes(&fa, exec_kernel);
}

}  // namespace nvfp4
