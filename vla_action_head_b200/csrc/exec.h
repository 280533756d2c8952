// exec.h — internal interface of the layer executor (executor.cu): one persistent
// cooperative launch that runs a whole program of norm->FP4 and GEMM ops.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "norm.h"

namespace nvfp4 {

enum { kOpNorm = 0, kOpGemm = 1 };

// One op of a program, in device memory.  Ops run in program order: op i starts consuming
// its inputs once done[i - 1] reached ops[i - 1].units (every op depends on the previous one).
// Most ops a program may hold (the executor keeps one bit per op in shared memory).
constexpr int kExecMaxOps = 4096;

struct ExecOp {
    int type;
    int dep;             // index of the op whose completion this op waits for, -1 for none
    int signal;          // 1 if a later op waits for this one (its units count into done[i])
    unsigned int units;  // done[i] value when the op is complete (norm: rows; GEMM: tiles)
    // ---- norm -> FP4 (one warp per row) ----
    NormArgs norm;
    int bpt;  // 16-element blocks per lane, 1..8
    // ---- GEMM ----
    int tm_a, tm_b;  // indices into the tensor-map table
    int M, N, K, k_atoms, k_tiles;
    int bn, splits, kt_per_split, n_tiles;
    int team0;  // the team that takes the op's first tile (ops start where the last left off)
    uint32_t a_box_rows;
    const uint8_t *sfa, *sfb;
    float alpha;
    int epi;
    const uint16_t *bias, *residual;
    int ldr;
    uint16_t *out;
    int ldo;
    uint8_t *out_codes, *out_sf;
    float g_out;
    int out_rotate;  // FP4 epilogues: Hadamard-rotate each output block before quantizing
};

struct ExecParams {
    const ExecOp *ops;
    const CUtensorMap *maps;
    unsigned int *done;  // one counter per op, zeroed before each run
    int n_ops;
    int cluster;       // CTAs per cluster (the split-K reduction group size limit)
    uint32_t *status;  // the library's device status word
    unsigned long long *trace;  // optional: 8 globaltimer stamps per (op, CTA)
};

// Largest grid (multiple of `cluster`) whose CTAs are all co-resident.
cudaError_t exec_grid(int cluster, int *grid);
cudaError_t exec_launch(const ExecParams &p, int grid, cudaStream_t s);
cudaError_t probe_exec_kernel();

}  // namespace nvfp4
