/*
 * nvfp4.h — C ABI of libnvfp4.so: the NVFP4 linear layer of a VLA action head on B200
 * (sm_100a): bf16 -> {LayerNorm | RMSNorm | AdaLN | AdaRMSNorm} -> dynamic NVFP4 quantize,
 * offline NVFP4 weight quantize, and a block-scaled NVFP4 GEMM (tcgen05 kind::mxf4nvf4)
 * with fused bias / residual / tanh-GELU->FP4 / GeGLU->FP4 epilogues.
 *
 * Sources are cited as "page title, section":
 *   [GROOT]  "GROOT N1.7 update: Thor NVFP4 + FA4 performance tier"
 *   [PI05]   "Pi0.5 Thor NVFP4 End-to-End Results"
 *
 * Formats (shared by every entry point):
 *   FP4 tensor of `rows` x K elements:
 *     codes : uint8 [rows, K/2], row stride K/2 bytes; element 2j of a row in the low
 *             nibble of byte j, element 2j+1 in the high nibble; E2M1 code, bit 3 = sign,
 *             magnitudes {0, .5, 1, 1.5, 2, 3, 4, 6}.
 *     sf    : uint8 UE4M3 block scales, one per (row, 16-element K block), in 512-byte
 *             atoms of 128 rows x 4 blocks; atoms ordered K fastest, then 128-row group;
 *             inside an atom row r, block c is at (r%32)*16 + ((r%128)/32)*4 + c%4.
 *             Rows are padded to 128 and K to 64 elements; nvfp4_sf_bytes() gives the size.
 *             Padding bytes must be zero ([PI05] §Encoder Attention QKV NVFP4 +
 *             Scale-Factor Zero-Init): zero the buffer once at allocation (nvfp4_sf_zero);
 *             the quantizers write only real entries.
 *     global_scale g (fp32): an element decodes as val(code) * dec(sf) * g.
 *   bf16 tensors are row-major with the stated leading dimension (in elements).
 *
 * Conventions:
 *   - Every pointer inside a call is a DEVICE pointer unless marked "host".  The caller
 *     allocates and owns every buffer.  Device pointers must be 16-byte aligned and leading
 *     dimensions multiples of 8 elements.
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy default stream),
 *     allocate nothing and never synchronise, except nvfp4_quantize_weight (returns the
 *     global scale to the host) and nvfp4_get_device_status.
 *   - Errors are returned as nvfp4_status; nothing throws across the ABI and no call falls
 *     back to another precision or a host path ([PI05] §Implemented Path: unsupported
 *     shapes, missing kernels or failed launches raise; none selects another tier).
 *   - Global scales must be finite and within [2^-100, 2^100].
 */
#ifndef NVFP4_H
#define NVFP4_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *nvfp4_stream_t; /* same type as cudaStream_t */

typedef enum {
    NVFP4_OK = 0,
    NVFP4_ERR_INVALID_ARG = 1,       /* NULL pointer, bad enum, bad scale, ld < K ...     */
    NVFP4_ERR_UNSUPPORTED_SHAPE = 2, /* K or N outside the documented constraints        */
    NVFP4_ERR_MISALIGNED = 3,        /* pointer not 16-byte aligned / ld not a multiple of 8 */
    NVFP4_ERR_WORKSPACE = 4,         /* workspace NULL or smaller than required          */
    NVFP4_ERR_UNSUPPORTED_DEVICE = 5,/* current device is not sm_100                     */
    NVFP4_ERR_CUDA = 6,              /* a CUDA runtime/driver call or launch failed      */
    NVFP4_ERR_TIMEOUT = 7            /* a kernel's bounded wait expired (device status)  */
} nvfp4_status;

typedef enum {
    NVFP4_NORM_NONE = 0,      /* y = x (plain quantizer)                               */
    NVFP4_NORM_LAYERNORM = 1, /* y = (x - mu) * rstd * gamma + beta                    */
    NVFP4_NORM_RMSNORM = 2,   /* y = (x * rstd_rms) * gamma                            */
    NVFP4_NORM_ADALN = 3,     /* y = (x - mu) * rstd * (1 + scale) + shift             */
    NVFP4_NORM_ADARMS = 4     /* y = (x * rstd_rms) * (1 + scale) [+ shift]            */
} nvfp4_norm;

typedef enum {
    NVFP4_EPI_NONE = 0,          /* out = acc * gA * gW                       -> bf16   */
    NVFP4_EPI_BIAS = 1,          /* + bias[n]                                 -> bf16   */
    NVFP4_EPI_RESIDUAL = 2,      /* + residual[m, n]                          -> bf16   */
    NVFP4_EPI_BIAS_RESIDUAL = 3, /* + bias[n] + residual[m, n]                -> bf16   */
    NVFP4_EPI_BIAS_GELU = 4,     /* gelu_tanh(acc*gA*gW + bias[n])            -> FP4    */
    NVFP4_EPI_GEGLU = 5,         /* gelu_tanh(v[m,2j]) * v[m,2j+1], v = acc*gA*gW (+bias) -> FP4, width N/2 */
    /* BIAS_GELU / GEGLU with each 16-value output block rotated by the 16-point Hadamard
     * matrix before it is quantized (NVFP4_QUANT_ROTATE below): the rotated activation
     * exit that feeds a GEMM whose weights were quantized with NVFP4_QUANT_ROTATE
     * ([PI05] §Full-INT4 Decoder Activations + Hadamard Rotation). */
    NVFP4_EPI_BIAS_GELU_RHT = 6,
    NVFP4_EPI_GEGLU_RHT = 7
} nvfp4_epilogue;

/* Quantizer options (bit flags) of the *_ex quantizers:
 *   NVFP4_QUANT_ROTATE  rotate each 16-element block by the orthonormal Sylvester Hadamard
 *                       matrix H16 / 4 before quantizing it ([PI05] §Full-INT4 Decoder
 *                       Activations + Hadamard Rotation).  Rotating the blocks of both GEMM
 *                       operands leaves the product unchanged (H16 H16^T = 16 I), so the
 *                       block-scaled GEMM consumes rotated operands as they are.  The
 *                       rotation is the in-register butterfly: stages d = 1, 2, 4, 8 pair
 *                       element i with i ^ d (a + b at the lower index, a - b at the upper),
 *                       each one fp32 add, then each element times 1/4.
 *   NVFP4_QUANT_E0M3    uniform INT4 elements instead of E2M1 ([PI05] §E0M3 Uniform-INT4
 *                       Decoder Weights): code bit 3 = sign, bits 0..2 = round-half-even of
 *                       |y| / S saturated at 7; block scale s = E4M3(amax / (7 g)).  These
 *                       codes are a storage format: nvfp4_gemm reads E2M1 codes only (the
 *                       tensor-core E0M3 element format is not documented for sm_100a).
 *   NVFP4_QUANT_MSE     weights only: MSE-searched block scales (as
 *                       nvfp4_quantize_weight_mse); not with E0M3. */
typedef enum {
    NVFP4_QUANT_DEFAULT = 0,
    NVFP4_QUANT_ROTATE = 1,
    NVFP4_QUANT_E0M3 = 2,
    NVFP4_QUANT_MSE = 4
} nvfp4_quant_flags;

typedef enum { NVFP4_IN_BF16 = 0, NVFP4_IN_FP32 = 1 } nvfp4_in_dtype;

/* An FP4 operand: device codes / sf in the formats above, host-side global scale. */
typedef struct {
    const uint8_t *codes;
    const uint8_t *sf;
    float global_scale;
    int rows;
    int K;
} nvfp4_tensor;

/* ---- helpers ----------------------------------------------------------------------- */

/* NVFP4_OK if the current device is sm_100 and this library's kernels load on it;
 * NVFP4_ERR_UNSUPPORTED_DEVICE otherwise.  Call once before capture ([GROOT] §Shared-code
 * changes: the frontend probes its bindings up front instead of failing inside capture). */
nvfp4_status nvfp4_probe(void);

/* Static, never NULL. */
const char *nvfp4_status_string(nvfp4_status s);

/* The CUDA runtime's message for the last CUDA error behind an NVFP4_ERR_CUDA returned to
 * this thread ("no error" if there was none).  Static storage; never NULL. */
const char *nvfp4_last_cuda_error_string(void);

/* Bytes of a scale-factor buffer for rows x K elements: ceil(rows/128)*ceil(K/64)*512. */
size_t nvfp4_sf_bytes(int rows, int K);

/* Byte offset of the scale of (row, K block kblk) in that buffer (layout above). */
size_t nvfp4_sf_offset(int row, int kblk, int K);

/* Zeroes a scale-factor buffer (cudaMemsetAsync); once per allocation is enough. */
nvfp4_status nvfp4_sf_zero(uint8_t *sf, int rows, int K, nvfp4_stream_t stream);

/* Workspace bytes nvfp4_gemm needs for this shape; 0 if none.  For M <= 128 the default
 * schedule reduces split-K partials inside a thread-block cluster (distributed shared
 * memory) and needs no workspace; schedules that reduce through global memory (more than 8
 * splits, the ones selected by negative `splits` in nvfp4_gemm_ex, and the many-row (M > 128)
 * schedule when it splits K in two because the shape has fewer output tiles than SMs, e.g.
 * 968 x 2048 x 16384) need a fixed 16 KiB region of tile counters followed by the fp32
 * partials (splits x M x N x 4 bytes; the many-row schedule rounds M up to whole 128-row
 * tiles).  A workspace must be zeroed once at allocation; every call leaves its counters
 * zero again, and no call's partials overlap the counter region, so one workspace may serve
 * GEMMs of different shapes one after another (after NVFP4_ERR_TIMEOUT, zero it again).
 * Schedules whose counters exceed the region (more than 4096 tiles, 2048 for the many-row
 * kernel) return NVFP4_ERR_UNSUPPORTED_SHAPE. */
size_t nvfp4_gemm_workspace_bytes(int M, int N, int K);

/* Reads and clears the library's device status word after synchronising `stream`:
 * NVFP4_OK, or NVFP4_ERR_TIMEOUT if a kernel's bounded wait expired since the last read. */
nvfp4_status nvfp4_get_device_status(nvfp4_stream_t stream);

/* Diagnostics (tracing): while `buf` (device, `words` 64-bit words) is set, each
 * nvfp4_gemm launch takes the next free slice of it (8 words per CTA, CTA index
 * (split * m_tiles + m_tile) * n_tiles + n_tile) and writes globaltimer ns at: entry,
 * split-K epilogue items done, set-up done, first operand stage landed, last MMA issued,
 * accumulator ready, exit, split-K partials visible (words 1 and 7 stay 0 without
 * split-K).  Launches that no longer fit are not traced.  Setting
 * a buffer (or NULL, which turns tracing off) rewinds the cursor.  Host-side state, not
 * thread safe; captured launches keep the slice they got at capture.
 * nvfp4_program_run (grouped GEMM), when the buffer holds grid * 8 words, writes per CTA
 * at cta * 8: entry, first stage landed, last MMA issued, exit and per-tile stamps (see
 * gemm_grouped.cu). */
nvfp4_status nvfp4_set_gemm_trace(unsigned long long *buf, size_t words);

/* Diagnostics: the issue rate of the block-scaled MMA on one SM.  One CTA, one issuing
 * thread, operands resident in shared memory, accumulator and scale factors in tensor
 * memory, runs `ksteps` K steps of 256, each four tcgen05.mma kind::mxf4nvf4 block16
 * (M = 128, N = n, K = 64) -- mode 0 -- or each its scale-atom copies (tcgen05.cp: 4 for A,
 * 4 per 128-row group of W) followed by its four MMAs -- mode 1.  Writes SM clock cycles
 * per K step until the last instruction was issued (*issue_cycles) and until all of them
 * completed (*complete_cycles; host pointers).  n: 64, 128 or 256; mode 0 or 1;
 * 1 <= ksteps <= 4096 (else NVFP4_ERR_INVALID_ARG).  Uses 512 tensor-memory columns and
 * ~57 KB of shared memory on one SM; synchronises the device.  The data are meaningless;
 * only the cycle counts are. */
nvfp4_status nvfp4_mma_rate(int n, int mode, int ksteps, double *issue_cycles, double *complete_cycles);

/* Trace words one nvfp4_gemm launch of this shape and epilogue takes under the default
 * schedule (8 per CTA of its grid); 0 for a shape nvfp4_gemm does not accept. */
size_t nvfp4_gemm_trace_words(int M, int N, int K, nvfp4_epilogue epi);

/* ---- norm -> NVFP4 quantize (fused front-end) --------------------------------------- */

/* Per row of x [M, K] (leading dimension ldx, bf16 or fp32): the norm `kind`, then the
 * per-16 block quantizer with global scale `global_scale`, emitting codes [M, K/2] and
 * sf (nvfp4_sf_bytes(M, K), pre-zeroed).  ([GROOT] §What is in the tier: AdaLN and the
 * pre-FFN LayerNorm emit FP4 directly, bit-identical to the two-step chain; dynamic
 * per-16 activation quantization with no calibration pass.  [PI05] §Vectorized SigLIP
 * LayerNorms: register-resident single pass with 16-byte loads; §Implemented Path:
 * AdaRMSNorm + NVFP4/SFA in one launch, dynamic quantization of the attention output.)
 *
 * Per block of 16 normalized values y:  a = max|y|, s = E4M3_rn_satfinite(a / (6 g)),
 * S = dec(s) g; dec(s) == 0 -> all codes +0; else code_i = E2M1_rn_satfinite(y_i * (1/S)).
 * Row statistics: fp64 sums, mean and 1/sqrt(var + eps) rounded once to fp32.
 * gamma/beta/mod_scale/mod_shift: bf16 [K] or NULL (gamma NULL reads 1, others 0).
 * Constraints: M >= 0 (M == 0 is a no-op), 16 <= K <= 32768, K % 16 == 0, ldx >= K. */
nvfp4_status nvfp4_quantize_norm(const void *x, nvfp4_in_dtype dt, int M, int K, int ldx,
                                 nvfp4_norm kind, const void *gamma, const void *beta,
                                 const void *mod_scale, const void *mod_shift, float eps,
                                 float global_scale, uint8_t *codes, uint8_t *sf,
                                 nvfp4_stream_t stream);

/* The first step of the two-step chain alone: the same norm, written as fp32 y [M, K]
 * (dense).  nvfp4_quantize_norm(y, NVFP4_IN_FP32, ..., NVFP4_NORM_NONE, ...) is the second
 * step; the fused call equals the chain bit for bit. */
nvfp4_status nvfp4_norm_f32(const void *x, nvfp4_in_dtype dt, int M, int K, int ldx,
                            nvfp4_norm kind, const void *gamma, const void *beta,
                        const void *mod_scale, const void *mod_shift, float eps, float *y,
                        nvfp4_stream_t stream);

/* Gated residual front-end, one launch ([PI05] §Implemented Path: gated residual update +
 * Pi0.5 AdaRMSNorm + gate output + NVFP4/SFA in one launch before Gate+Up and the next
 * layer's QKV).  Per element of the bf16 residual stream x [M, K] (ldx) and the sublayer
 * output d [M, K] (ldd), with the bf16 gate [K] (NULL reads 1):
 *   h = bf16_rn(x + gate * d)      (one fp32 product, one fp32 sum, one rounding)
 * h is stored to h_out [M, K] (ldh, bf16, device) as the new residual stream, and the norm
 * `kind` + block quantizer of nvfp4_quantize_norm run on that bf16 h, so the result equals
 * nvfp4_quantize_norm(h, ...) bit for bit.  h_out may alias x (each element is read before
 * it is written, by the same thread); it must not overlap d.  Same constraints as
 * nvfp4_quantize_norm, bf16 only; ldd, ldh multiples of 8 and >= K. */
nvfp4_status nvfp4_residual_quantize_norm(const void *x, const void *d, const void *gate, int M, int K,
                                          int ldx, int ldd, int ldh, nvfp4_norm kind, const void *gamma,
                                          const void *beta, const void *mod_scale, const void *mod_shift,
                                          float eps, float global_scale, void *h_out, uint8_t *codes,
                                          uint8_t *sf, nvfp4_stream_t stream);

/* nvfp4_quantize_norm and nvfp4_residual_quantize_norm with quantizer options `flags`
 * (NVFP4_QUANT_ROTATE | NVFP4_QUANT_E0M3; other bits: NVFP4_ERR_INVALID_ARG).  The rotation
 * applies to the normalized y; with E0M3 the block scale is E4M3(amax / (7 g)).  Otherwise
 * the arguments, constraints and results are those of the calls without _ex. */
nvfp4_status nvfp4_quantize_norm_ex(const void *x, nvfp4_in_dtype dt, int M, int K, int ldx,
                                    nvfp4_norm kind, const void *gamma, const void *beta,
                                    const void *mod_scale, const void *mod_shift, float eps,
                                    float global_scale, int flags, uint8_t *codes, uint8_t *sf,
                                    nvfp4_stream_t stream);
nvfp4_status nvfp4_residual_quantize_norm_ex(const void *x, const void *d, const void *gate, int M,
                                             int K, int ldx, int ldd, int ldh, nvfp4_norm kind,
                                             const void *gamma, const void *beta,
                                             const void *mod_scale, const void *mod_shift,
                                             float eps, float global_scale, int flags, void *h_out,
                                             uint8_t *codes, uint8_t *sf, nvfp4_stream_t stream);

/* ---- offline weight quantize --------------------------------------------------------- */

/* W bf16 [N, K] (ldw) -> codes [N, K/2] + sf (nvfp4_sf_bytes(N, K), pre-zeroed) with the
 * per-tensor global scale g = amax(|W|) / (6 * 448) (1 if W is all zero), returned in
 * *global_scale_out (host).  interleave_gate_up = 1 packs rows [0, N/2) (gate) and
 * [N/2, N) (up) pairwise: output row 2j = gate row j, row 2j+1 = up row j ([PI05]
 * §Fused GeGLU Epilogue for the P1 Encoder FFN).  `scratch`: device, >= 256 bytes.
 * Synchronises `stream`.  ([PI05] §Implemented Path: weights quantized once at load.) */
nvfp4_status nvfp4_quantize_weight(const void *w_bf16, int N, int K, int ldw,
                                   int interleave_gate_up, uint8_t *codes, uint8_t *sf,
                                   float *global_scale_out, void *scratch,
                                   nvfp4_stream_t stream);

/* As nvfp4_quantize_weight, with MSE-searched block scales ([PI05] §E0M3 Uniform-INT4
 * Decoder Weights: the default decoder weights are NVFP4 "(MSE)"; §Fused GeGLU FFN in the
 * Decoder: the interleaved gate/up weight is MSE-quantized too).  Per 16-element block,
 * every UE4M3 scale byte 0x00..0x7E is tried with the codes the amax quantizer would write
 * at that scale; the byte whose block squared error (fp64, terms in index order) is least
 * is kept, the smaller byte on ties.  The global scale is the same amax / 2688.  Same
 * arguments and constraints as nvfp4_quantize_weight. */
nvfp4_status nvfp4_quantize_weight_mse(const void *w_bf16, int N, int K, int ldw,
                                       int interleave_gate_up, uint8_t *codes, uint8_t *sf,
                                       float *global_scale_out, void *scratch,
                                       nvfp4_stream_t stream);

/* The weight quantizer with options `flags` (NVFP4_QUANT_ROTATE | NVFP4_QUANT_E0M3 |
 * NVFP4_QUANT_MSE; E0M3 with MSE or other bits: NVFP4_ERR_INVALID_ARG).  The values
 * quantized are W's 16-element blocks along K, Hadamard-rotated with NVFP4_QUANT_ROTATE,
 * and the global scale is their amax over (top grid magnitude x 448): amax / 2688 for E2M1,
 * amax / 3136 for E0M3 (1 for an all-zero W) -- a rotated block's amax can be up to 4x the
 * original's, so the amax is taken after the rotation.  ([PI05] §Full-INT4 Decoder
 * Activations + Hadamard Rotation; §E0M3 Uniform-INT4 Decoder Weights: per-16 UE4M3 scales,
 * amax / 7.)  Arguments otherwise as nvfp4_quantize_weight; synchronises `stream`. */
nvfp4_status nvfp4_quantize_weight_ex(const void *w_bf16, int N, int K, int ldw,
                                      int interleave_gate_up, int flags, uint8_t *codes,
                                      uint8_t *sf, float *global_scale_out, void *scratch,
                                      nvfp4_stream_t stream);

/* ---- block-scaled NVFP4 GEMM with fused epilogue ------------------------------------ */

/* acc[m, n] = sum_k dec(A)[m, k] * dec(W)[n, k] over the E2M1 codes and UE4M3 block scales
 * (tcgen05.mma kind::mxf4nvf4, fp32 accumulation in tensor memory), then the epilogue
 * `epi` on v = acc * gA * gW (+ bias[n]) (+ residual[m, n]) ([GROOT] §What is in the tier:
 * fused bf16 bias / bias+residual / bias+tanh-GELU+FP4-output epilogues; [PI05] §Fused
 * GeGLU FFN in the Decoder: GELU on the fp32 accumulator, gate/up interleaved pairwise).
 *   A: M x K activations, W: N x K weights (A->rows == M, W->rows == N, both ->K == K).
 *   bias: bf16 [N] or NULL; residual: bf16 [M, ldr] (RESIDUAL / BIAS_RESIDUAL only).
 *   bf16 epilogues write out_bf16 [M, ldo]; FP4 epilogues (BIAS_GELU, GEGLU, and their
 *   rotated *_RHT forms) write
 *   out_codes [M, N_out/2] and out_sf (nvfp4_sf_bytes(M, N_out), pre-zeroed) quantized
 *   with out_global_scale, N_out = N (BIAS_GELU[_RHT]) or N/2 (GEGLU[_RHT]).
 *   workspace: >= nvfp4_gemm_workspace_bytes(M, N, K) bytes, zeroed once at allocation;
 *   used by one GEMM at a time (GEMMs that may run concurrently, e.g. on two streams, each
 *   need their own).
 * Launch overlap: the kernel starts while the previous kernel of `stream` still runs when
 * that kernel is one of this library's (programmatic dependent launch), and may read W, its
 * scales and bias before waiting for it; A, its scales and residual are read after.  So W
 * and bias must not be written by the library call immediately before on the same stream.
 * Constraints: M >= 0 (0 is a no-op), K % 32 == 0 (TMA 16-byte rows; a K % 64 tail is
 * covered by the zero scale padding, [PI05] §Encoder Attention QKV NVFP4 + Scale-Factor
 * Zero-Init), N % 64 == 0. */
nvfp4_status nvfp4_gemm(const nvfp4_tensor *A, const nvfp4_tensor *W, int M, int N, int K,
                        nvfp4_epilogue epi, const void *bias, const void *residual, int ldr,
                        void *out_bf16, int ldo, uint8_t *out_codes, uint8_t *out_sf,
                        float out_global_scale, void *workspace, size_t ws_bytes,
                        nvfp4_stream_t stream);

/* nvfp4_gemm for callers that cannot allocate device memory: no workspace argument.  None
 * of the source pages describes such an entry point; it is this library's own addition, and
 * it has no counterpart there to cite.  It serves code that is not allowed to
 * call cudaMalloc (or any allocator) once it is running -- for example a plugin inside a
 * host runtime that owns every device allocation, or a real-time control loop that must
 * not allocate after start-up.  The split-K workspace instead comes from a fixed 4 MiB
 * buffer inside this library's own device memory, which every GPU that loads the library
 * keeps until the process exits.  The call allocates nothing; it zeroes the buffer's
 * ticket words with cudaMemsetAsync on `stream` before the GEMM.
 *   - It runs the workspace-reduced schedule (nvfp4_gemm_ex with block_n = 0, splits = -1).
 *     Shapes for which that needs more than 4 MiB return NVFP4_ERR_WORKSPACE;
 *     nvfp4_gemm_workspace_bytes_ex(M, N, K, 0, -1) tells the need in advance.
 *   - The first call on each device looks the buffer's address up; make that first call
 *     before any stream capture.
 *   - Every call shares the one buffer, which keeps the previous call's contents: calls that
 *     may overlap on the GPU (other streams, other host threads) race on it; serialise them.
 *   - A call that fails the argument checks returns before it touches the buffer.
 * Otherwise the contract and results are those of nvfp4_gemm. */
nvfp4_status nvfp4_gemm_noalloc(const nvfp4_tensor *A, const nvfp4_tensor *W, int M, int N, int K,
                                nvfp4_epilogue epi, const void *bias, const void *residual, int ldr,
                                void *out_bf16, int ldo, uint8_t *out_codes, uint8_t *out_sf,
                                float out_global_scale, nvfp4_stream_t stream);

/* Schedule-pinned variant of nvfp4_gemm for tuning sweeps and tests: block_n in
 * {64, 128, 256} output columns per CTA and |splits| K partitions (each a whole number of
 * 256-element K tiles).  splits > 0 reduces the partials inside a cluster when splits <= 8
 * and M <= 128, otherwise through the workspace; splits < 0 always uses the workspace.
 * block_n = 0 with splits = 0 takes the default schedule, with splits = -1 the default
 * workspace-reduced schedule.  The default schedule for M > 128 with N % 128 == 0 runs a
 * persistent kernel (one CTA per SM walks 128 x 256 or 128 x 128 output tiles); a pinned
 * schedule always runs one tile per CTA.  Same contract otherwise; the workspace must hold
 * nvfp4_gemm_workspace_bytes_ex(M, N, K, block_n, splits) bytes. */
nvfp4_status nvfp4_gemm_ex(const nvfp4_tensor *A, const nvfp4_tensor *W, int M, int N, int K,
                           nvfp4_epilogue epi, const void *bias, const void *residual, int ldr,
                           void *out_bf16, int ldo, uint8_t *out_codes, uint8_t *out_sf,
                           float out_global_scale, void *workspace, size_t ws_bytes,
                           int block_n, int splits, nvfp4_stream_t stream);

size_t nvfp4_gemm_workspace_bytes_ex(int M, int N, int K, int block_n, int splits);

/* ---- grouped GEMM (a program of independent GEMMs in one launch) -------------------- */

/* A grouped GEMM runs many independent NVFP4 GEMMs -- e.g. the 32 per-frame cross-attention
 * K / V projections of a DiT ([GROOT] §What is in the tier) -- in ONE launch of the grouped
 * persistent kernel: one CTA per SM walks all the problems' 128 x 128 output tiles through
 * one TMA / tensor-core pipeline, so the weight stream does not stop at problem
 * boundaries.  Results are those of nvfp4_gemm on each problem (one split per tile).
 * Each op is described by an nvfp4_op of type NVFP4_OP_GEMM with dep = NVFP4_DEP_NONE; the
 * norm fields and other dep values belong to an earlier interface of this struct and are
 * rejected (NVFP4_ERR_UNSUPPORTED_SHAPE). */
typedef enum { NVFP4_OP_QUANTIZE_NORM = 0, NVFP4_OP_GEMM = 1 } nvfp4_op_type;

typedef struct {
    nvfp4_op_type type;  /* NVFP4_OP_GEMM */
    int M, N, K;
    /* unused (must describe no work): */
    const void *x;
    int ldx;
    nvfp4_norm norm;
    const void *gamma, *beta, *mod_scale, *mod_shift;
    float eps;
    /* A (M x K) times W (N x K)^T, epilogue as nvfp4_gemm */
    nvfp4_tensor A, W;
    nvfp4_epilogue epi;
    const void *bias, *residual;
    int ldr;
    void *out_bf16;
    int ldo;
    /* FP4 output of a BIAS_GELU / GEGLU epilogue (and their rotated forms) */
    uint8_t *out_codes, *out_sf;
    float out_global_scale;
    int dep;  /* NVFP4_DEP_NONE: the op's inputs are ready before the launch */
} nvfp4_op;

#define NVFP4_DEP_PREVIOUS 0
#define NVFP4_DEP_NONE (-1)

/* Host-side handle of a built grouped GEMM; the device data lives in `buffer`. */
typedef struct {
    void *buffer;
    size_t bytes;
    int n_ops;
    int grid;
    int cluster;
    size_t ops_offset, maps_offset, done_offset;
    int waits;  /* 0 */
    int kind;   /* 1: the grouped GEMM kernel */
    int epi;    /* the epilogue of every op */
    int tiles;  /* output tiles over all ops */
} nvfp4_program;

/* Device bytes a grouped GEMM of n_ops problems needs. */
size_t nvfp4_program_bytes(int n_ops);

/* Builds a grouped GEMM of 1..256 GEMM ops that all have dep = NVFP4_DEP_NONE, the same
 * epilogue and N % 128 == 0 (else NVFP4_ERR_UNSUPPORTED_SHAPE).  Validates each op by the
 * rules of nvfp4_gemm, encodes the TMA descriptors and copies the problems and their tile
 * table into `buffer` (device, >= nvfp4_program_bytes(n_ops), 256-byte aligned).
 * Synchronous (set-up time); the buffers the ops name must stay valid for every later run. */
nvfp4_status nvfp4_program_build(const nvfp4_op *ops, int n_ops, void *buffer, size_t bytes,
                                 nvfp4_program *prog);

/* Runs the grouped GEMM on `stream`: one launch.  Allocates nothing; capturable in a CUDA
 * graph.  Runs of the same program must not overlap. */
nvfp4_status nvfp4_program_run(const nvfp4_program *prog, nvfp4_stream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* NVFP4_H */
