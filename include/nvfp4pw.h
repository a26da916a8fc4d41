/*
 * nvfp4pw.h -- C ABI of the B200 (sm_100a) NVFP4 GPTQ + Schur Replay layer solve.
 *
 * Method: "Replay the Curvature: Accurate and Scalable NVFP4 Quantization for
 * Large Language Model Inference" (arXiv 2609.36654v1), Abstract:
 *   - NVFP4: every 16 consecutive E2M1 weights share one E4M3 block scale
 *     (Abstract, sentence defining NVFP4); a per-tensor fp32 global scale sits
 *     on top (s_g = amax|W| / (6 * 448)).
 *   - GPTQ: quantizing one column updates the columns that follow it (Abstract,
 *     sentence on why the scale choice is hard); second-order state H = X^T X
 *     is accumulated from calibration activations (Abstract, sentence on
 *     second-order state).
 *   - Schur Replay: each candidate block scale is scored by replaying the
 *     in-block GPTQ updates it causes and measuring the block error left after
 *     compensation from the still-unquantized columns (Abstract, sentence
 *     introducing Schur Replay).
 *
 * Conventions for every call
 *   - All array pointers are DEVICE pointers unless the argument says "host".
 *     The caller owns every buffer; the library allocates no device memory
 *     (scratch comes from a caller-provided workspace whose size the
 *     *_workspace_size() calls return).
 *   - Matrices are row-major and densely packed (leading dimension = columns).
 *   - Every call is asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *     default stream) and returns a host-side status at once.  Conditions that
 *     only the GPU can see (non-finite input, a non-positive pivot) are written
 *     to a sticky status word at the start of the workspace; read it with
 *     nvfp4_workspace_status() after the stream's work is done.  No kernel
 *     traps or spins without a bound.
 *   - Sizes are int64_t; negative sizes are NVFP4_ERR_INVALID_ARG.  The
 *     quantized dimension (d, d_in) must be a multiple of 16.
 *   - Alignment: W and dequant's `out` 16 bytes, packed codes 8 bytes,
 *     workspaces 256 bytes (NVFP4_ERR_INVALID_ARG / _WORKSPACE otherwise).
 */
#ifndef NVFP4PW_H
#define NVFP4PW_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Status codes returned by every call and stored in the device status word. */
typedef enum {
  NVFP4_OK = 0,
  NVFP4_ERR_INVALID_ARG = 1, /* null pointer, negative size, bad enum        */
  NVFP4_ERR_SHAPE = 2,       /* d or d_in not a multiple of 16, or too large */
  NVFP4_ERR_WORKSPACE = 3,   /* workspace null or smaller than required      */
  NVFP4_ERR_NONFINITE = 4,   /* NaN/Inf met in W or H (device-detected)      */
  NVFP4_ERR_NOT_PD = 5,      /* damped H not positive definite (device)      */
  NVFP4_ERR_TIMEOUT = 6,     /* a bounded device wait ran out (device)       */
  NVFP4_ERR_CUDA = 7,        /* a CUDA runtime call or launch failed         */
  NVFP4_ERR_UNSUPPORTED = 8, /* parameter value this build does not support  */
  NVFP4_ERR_BOUNDS = 9       /* debug build only: a kernel's tile or index
                                left its array; the access was skipped (device) */
} nvfp4_status;

/* Element type of an input or output array. */
typedef enum { NVFP4_BF16 = 0, NVFP4_F32 = 1 } nvfp4_dtype;

/* Opaque stream handle, layout-compatible with cudaStream_t / CUstream. */
typedef struct CUstream_st* nvfp4_stream_t;

/* Block-scale rule of the GPTQ sweep.
 *
 * NVFP4_RULE_SCHUR_REPLAY (default): every candidate scale of a block is
 *   scored by replaying the in-block GPTQ updates it causes and summing
 *   delta_j^2 = (v_j - q_j)^2 / U_jj^2, the block error left after
 *   compensation by the still-unquantized columns; the lowest score wins
 *   ("Replay the Curvature", Abstract, sentence introducing Schur Replay).
 * The two rules below evaluate a block on its own, which can misestimate its
 * final error once GPTQ updates the columns after each quantized one (the
 * Abstract's sentence on why scale choice is hard in GPTQ); they exist for
 * comparison (same sweep, same block amax and window, only the decision
 * differs):
 * NVFP4_RULE_AMAX: the centre code k0, which maps the block amax to 6.
 * NVFP4_RULE_BLOCK_MSE: the window code minimising sum_j (v_j - q_j)^2 with
 *   every v_j rounded on its own, before any in-block update; ties to the
 *   lower code. */
typedef enum {
  NVFP4_RULE_SCHUR_REPLAY = 0,
  NVFP4_RULE_AMAX = 1,
  NVFP4_RULE_BLOCK_MSE = 2
} nvfp4_scale_rule;

/* Arithmetic of the solve (nvfp4_solve_params.precision).
 * NVFP4_PRECISION_FP64_REPLAY (the default and the only value this build
 *   supports): the working copy W~ and the Schur Replay are fp64, the
 *   trailing-update products 3xTF32 on the tensor cores (fp32-level
 *   products, accumulated into the fp64 W~), the factor U fp64-accurate and
 *   stored fp32.  The codes are discrete decisions taken on values every
 *   earlier column's update has moved, so an fp32 working copy or replay flips
 *   decisions that are not near ties; this is the cheapest arithmetic measured
 *   to keep them on the exact solve's. */
typedef enum { NVFP4_PRECISION_FP64_REPLAY = 0 } nvfp4_precision;

/* Solve parameters.  n_candidates, cand_lo, lazy_batch and precision support
 * only the defaults below (n_candidates = 16, cand_lo = -8, lazy_batch = 128,
 * precision = NVFP4_PRECISION_FP64_REPLAY); other values, or a scale_rule
 * outside nvfp4_scale_rule, return NVFP4_ERR_UNSUPPORTED.  The candidate
 * window is the n_candidates consecutive E4M3 codes starting at
 * k0 + cand_lo, shifted into 1..126, where k0 = e4m3_rn(amax_block / (6 s_g))
 * (at least 1). */
typedef struct {
  int n_candidates; /* 16 */
  int cand_lo;      /* -8 */
  int lazy_batch;   /* 128: columns per batch of the trailing update */
  int scale_rule;   /* nvfp4_scale_rule, default NVFP4_RULE_SCHUR_REPLAY */
  int precision;    /* nvfp4_precision, default NVFP4_PRECISION_FP64_REPLAY */
} nvfp4_solve_params;

/* Fills *p with the defaults above. */
void nvfp4_default_params(nvfp4_solve_params* p);

/* Human-readable name of a status code (static storage, never NULL). */
const char* nvfp4_status_string(nvfp4_status s);

/* Synchronizes `stream`, then returns the device status word that the
 * prepare / quantize calls keep at the start of their workspace `ws`
 * (NVFP4_OK if nothing was flagged).  Returns NVFP4_ERR_CUDA if the copy
 * fails.  The word is sticky: it is cleared at the start of the next call
 * that uses the same workspace. */
nvfp4_status nvfp4_workspace_status(const void* ws, nvfp4_stream_t stream);

/* ------------------------------------------------------------------------ */
/* a1  Hessian: H (+)= X^T X over calibration tokens                          */
/* "Replay the Curvature", Abstract (second-order state from calibration     */
/* activations).                                                             */
/* ------------------------------------------------------------------------ */
/* H     : d x d fp32, full symmetric matrix (both triangles written).
 * X     : n_tok x d, bf16 or fp32 (x_dtype), one token per row.
 * beta  : 0 -> H = X^T X, 1 -> H += X^T X (accumulate over token chunks).
 * d must be a multiple of 16; n_tok >= 0 (0 with beta = 0 zeroes H).
 * bf16 products are exact in fp32 and are summed in fp32 on the tensor cores
 * (tcgen05, when d >= 256, n_tok >= 64 and X is 16-byte aligned; otherwise on
 * the CUDA cores); fp32 inputs are multiplied and summed in fp32 on the CUDA
 * cores.  With beta = 1 the existing H must be symmetric (as this call writes
 * it).  No workspace.  The tensor-core kernel's waits are bounded; if one runs
 * out it sets a library status word that nvfp4_hessian_status() reports. */
nvfp4_status nvfp4_hessian_accumulate(float* H, const void* X, nvfp4_dtype x_dtype,
                                      int64_t n_tok, int64_t d, int beta,
                                      nvfp4_stream_t stream);

/* The same accumulation with the tokens in HOST memory, streamed through the
 * device chunk by chunk ("Replay the Curvature", Abstract, infrastructure
 * sentence: calibration activations are tiered across device, host and disk;
 * this is the device/host tier for the Hessian).
 * X_host    : n_tok x d host array (bf16 or fp32), page-locked for the copies
 *             to overlap the compute (pageable memory works, without overlap).
 *             It is read asynchronously: keep it unchanged until `stream`
 *             has passed this call.
 * chunk_tok : tokens per chunk (>= 1); two device staging buffers of that
 *             many tokens live in ws.
 * ws        : device workspace of nvfp4_hessian_host_workspace_size() bytes,
 *             256-byte aligned.
 * The copy of chunk c + 1 runs on a library copy stream while the Hessian of
 * chunk c runs on `stream`; H accumulates the chunks in fp32 (beta applies to
 * the first chunk).  Host-side errors return at once: NVFP4_ERR_INVALID_ARG,
 * NVFP4_ERR_SHAPE (d % 16), NVFP4_ERR_WORKSPACE. */
size_t nvfp4_hessian_host_workspace_size(int64_t d, int64_t chunk_tok, nvfp4_dtype x_dtype);
nvfp4_status nvfp4_hessian_accumulate_host(float* H, const void* X_host, nvfp4_dtype x_dtype,
                                           int64_t n_tok, int64_t d, int beta,
                                           int64_t chunk_tok, void* ws, size_t ws_bytes,
                                           nvfp4_stream_t stream);

/* The same accumulation kept to fp64 accuracy, into an fp64 H: every product
 * of two token values and their sums are exact to fp64 rounding (the tokens
 * are transposed into fp64 channel rows, zero-padded, and the product runs on
 * the int8-slice tensor-core GEMM of the factorisation: channel rows scaled
 * by powers of two, cut into 7-bit slices, slice products exact in int32,
 * levels summed in fp64; 8192 tokens per pass, passes added in fp64).
 * For layers with fewer calibration tokens than channels: their damped
 * Hessian's condition number (1e4 and more) amplifies the fp32 rounding of H
 * (relative 6e-8) into factor errors that move decisions beyond near ties;
 * with this H and nvfp4_gptq_prepare_f64 the factor is as accurate as for a
 * well-conditioned layer.  About ten times the work of the bf16 tensor-core
 * Hessian.
 * H   : d x d fp64, full symmetric (both triangles written).
 * ws  : nvfp4_hessian_f64_workspace_size(n_tok, d) bytes, 256-byte aligned;
 *       a timed-out wait sets NVFP4_ERR_TIMEOUT in its status word
 *       (nvfp4_workspace_status).
 * Other arguments, layouts and errors as nvfp4_hessian_accumulate. */
size_t nvfp4_hessian_f64_workspace_size(int64_t n_tok, int64_t d);
nvfp4_status nvfp4_hessian_accumulate_f64(double* H, const void* X, nvfp4_dtype x_dtype,
                                          int64_t n_tok, int64_t d, int beta, void* ws,
                                          size_t ws_bytes, nvfp4_stream_t stream);

/* Synchronizes `stream` and returns, then clears, the status word of the
 * Hessian calls on the current device: NVFP4_ERR_TIMEOUT if a tensor-core
 * Hessian kernel gave up on a bounded wait since the last query, NVFP4_OK
 * otherwise (NVFP4_ERR_CUDA if the word could not be read). */
nvfp4_status nvfp4_hessian_status(nvfp4_stream_t stream);

/* ------------------------------------------------------------------------ */
/* a2-a4  damping + upper Cholesky factor of the damped inverse              */
/* "Replay the Curvature", Abstract, sentence on why the scale choice is     */
/* hard in GPTQ: quantizing a column updates the columns after it; the       */
/* update weights are the rows of U, the upper factor of the damped inverse  */
/* Hessian (H_d^-1 = U^T U), and 1 / U_jj^2 is the Schur complement that the  */
/* Schur Replay score weights each column's error with (Abstract, sentence   */
/* introducing Schur Replay).                                                */
/* ------------------------------------------------------------------------ */
/* Bytes of workspace nvfp4_gptq_prepare needs for dimension d. */
size_t nvfp4_prepare_workspace_size(int64_t d);

/* H       : d x d fp32 symmetric (read only).
 * damp    : lambda = damp * mean(diag H) is added to the diagonal (0.01).
 *           A column with H_ii == 0 is dead: H_ii := 1 before damping.
 * U       : d x d fp32 out; upper triangular with positive diagonal and
 *           (H + lambda I)^-1 = U^T U; the strict lower triangle is written 0.
 * dead    : optional (may be NULL) d bytes out, 1 where column i is dead.
 * lambda_out : optional (may be NULL) device fp32 scalar out, lambda.
 * ws/ws_bytes : workspace of at least nvfp4_prepare_workspace_size(d) bytes,
 *           256-byte aligned.  A non-positive pivot sets NVFP4_ERR_NOT_PD and
 *           a non-finite H sets NVFP4_ERR_NONFINITE in the status word; U is
 *           then unspecified. */
nvfp4_status nvfp4_gptq_prepare(const float* H, int64_t d, float damp, float* U,
                                uint8_t* dead, float* lambda_out, void* ws,
                                size_t ws_bytes, nvfp4_stream_t stream);

/* nvfp4_gptq_prepare from an fp64 H (as nvfp4_hessian_accumulate_f64 writes
 * it): the same factorisation, which runs in fp64 throughout, reads H without
 * rounding it to fp32 first.  Same workspace size and errors. */
nvfp4_status nvfp4_gptq_prepare_f64(const double* H, int64_t d, float damp, float* U,
                                    uint8_t* dead, float* lambda_out, void* ws,
                                    size_t ws_bytes, nvfp4_stream_t stream);

/* ------------------------------------------------------------------------ */
/* a5-a8  GPTQ with Schur Replay block-scale selection                       */
/* "Replay the Curvature", Abstract: the NVFP4 sentence (16 E2M1 codes per   */
/* block under one E4M3 scale), the sentence on why the scale choice is hard */
/* in GPTQ (column-sequential updates) and the sentence introducing Schur    */
/* Replay (each candidate scale scored by replaying the in-block GPTQ        */
/* updates it causes, after compensation by the unquantized columns).        */
/* ------------------------------------------------------------------------ */
/* Bytes of workspace nvfp4_gptq_schur_replay_quantize needs. */
size_t nvfp4_quantize_workspace_size(int64_t d_out, int64_t d_in,
                                     const nvfp4_solve_params* params);

/* W       : d_out x d_in, bf16 or fp32 (w_dtype), read only.
 * U       : d_in x d_in fp32 upper factor from nvfp4_gptq_prepare (several
 *           weight matrices with the same input, e.g. q/k/v, share one U).
 * params  : NULL for the defaults.
 * dead    : optional d_in bytes from nvfp4_gptq_prepare; dead columns of W
 *           are treated as zero.
 * codes   : d_out x d_in/2 bytes out; byte c of a row packs column 2c in the
 *           low nibble and column 2c+1 in the high nibble; nibble bit 3 is the
 *           sign, bits 2..0 index {0, 0.5, 1, 1.5, 2, 3, 4, 6}; zero is +0.
 * scales  : d_out x d_in/16 bytes out, E4M3 (fn) codes; 0 for an all-zero
 *           block.
 * global_scale : device fp32 scalar out, s_g = amax|W| / 2688 (1 if W == 0).
 * err_out : optional (may be NULL) device fp64 scalar out, sum of delta^2 =
 *           tr((W-Q)(H + lambda I)(W-Q)^T) up to rounding.
 * ws/ws_bytes : workspace (256-byte aligned) of at least
 *           nvfp4_quantize_workspace_size() bytes; holds the fp64 working copy
 *           of W (8 bytes per weight) and the fp64 deltas of one lazy batch.
 *           Non-finite W sets NVFP4_ERR_NONFINITE in its status word.
 * d_out is at most 2^22 and d_in at most 2^17 (NVFP4_ERR_SHAPE beyond).
 * The working copy and the replay are fp64: the codes are discrete decisions
 * taken on values that every earlier column's update has moved, so they need
 * more than fp32 precision to match an exact-arithmetic solve. */
nvfp4_status nvfp4_gptq_schur_replay_quantize(
    const void* W, nvfp4_dtype w_dtype, int64_t d_out, int64_t d_in, const float* U,
    const nvfp4_solve_params* params, const uint8_t* dead, uint8_t* codes,
    uint8_t* scales, float* global_scale, double* err_out, void* ws, size_t ws_bytes,
    nvfp4_stream_t stream);

/* Allocation-free form of nvfp4_gptq_schur_replay_quantize (the paper has no
 * counterpart; it serves callers that cannot allocate device memory when they
 * quantize, e.g. an engine that owns all GPU memory through its own fixed pool
 * and forbids allocations outside it, or a host loop that must not take the
 * implicit device synchronisation of cudaMalloc/cudaFree).
 *
 * Same arguments and results as nvfp4_gptq_schur_replay_quantize, without the
 * workspace: the scratch is one fixed 16 MiB device array inside the library,
 * present on every GPU that loads it until the process exits.  The call does
 * not allocate (no cudaMalloc, cudaFree or allocating library routine).
 *   - Size limit: the layer must satisfy
 *     nvfp4_quantize_workspace_size(d_out, d_in, params) <= 16 MiB (about one
 *     million weights, e.g. 1024 x 1024); larger layers return
 *     NVFP4_ERR_WORKSPACE without launching anything.
 *   - status_out: optional device int out; receives the device status word of
 *     this call (what nvfp4_workspace_status reports for the workspace form).
 *   - The device current on the calling thread must be the stream's device.
 *     The first call on a device looks up the array's device address (once
 *     per device, under a lock); make that first call before any stream
 *     capture.  Under CUDA's lazy module loading (the default) that first
 *     call is also when the library's module holding the array is loaded on
 *     the device, i.e. when the driver reserves its 16 MiB there; later calls
 *     reserve nothing.
 *   - All calls on one device share the array and it keeps the previous
 *     call's contents (the call clears what must start at zero itself).  Calls
 *     whose GPU work overlaps, e.g. on two streams without ordering, race and
 *     give undefined results: order them on one stream. */
nvfp4_status nvfp4_gptq_schur_replay_quantize_noalloc(
    const void* W, nvfp4_dtype w_dtype, int64_t d_out, int64_t d_in, const float* U,
    const nvfp4_solve_params* params, const uint8_t* dead, uint8_t* codes,
    uint8_t* scales, float* global_scale, double* err_out, int* status_out,
    nvfp4_stream_t stream);

/* ------------------------------------------------------------------------ */
/* Row shards: one layer's output rows split over calls (e.g. one per GPU)   */
/* ------------------------------------------------------------------------ */
/* "Replay the Curvature", Abstract, infrastructure sentence: independent
 * output rows are distributed across tensor-parallel ranks.  Given U the rows
 * of the solve are independent; only the global scale is shared.  So each
 * shard computes its max |W| with nvfp4_weight_amax, the shards' values are
 * reduced with MAX (a collective of the caller's, e.g. an NCCL all-reduce),
 * and every shard quantizes its rows with nvfp4_gptq_schur_replay_quantize_rows
 * from that layer amax: the codes and scales of the shards then equal the
 * whole-layer call's rows bit for bit.
 *
 * nvfp4_weight_amax: max |W| of a d_out x d_in block (dead columns, if given,
 * count as 0), written to the device fp32 scalar amax_out (0 for an empty
 * block).  Non-finite weights are not reported here (the quantize call flags
 * them). */
nvfp4_status nvfp4_weight_amax(const void* W, nvfp4_dtype w_dtype, int64_t d_out, int64_t d_in,
                               const uint8_t* dead, float* amax_out, nvfp4_stream_t stream);

/* As nvfp4_gptq_schur_replay_quantize for the rows W (d_out x d_in, a block
 * of rows of a larger layer), except that the global scale is computed from
 * the device fp32 scalar `amax` (the layer's max |W|) with the same formula,
 * s_g = fp32(amax / 2688) (1 when amax == 0), instead of from this block. */
nvfp4_status nvfp4_gptq_schur_replay_quantize_rows(
    const void* W, nvfp4_dtype w_dtype, int64_t d_out, int64_t d_in, const float* U,
    const nvfp4_solve_params* params, const uint8_t* dead, const float* amax,
    uint8_t* codes, uint8_t* scales, float* global_scale, double* err_out, void* ws,
    size_t ws_bytes, nvfp4_stream_t stream);

/* ------------------------------------------------------------------------ */
/* a9  dequantization: Q = e2m1(code) * e4m3(scale) * s_g                    */
/* "Replay the Curvature", Abstract (NVFP4 format).                          */
/* ------------------------------------------------------------------------ */
/* codes/scales/global_scale as written by the quantize call.
 * out     : d_out x d_in, fp32 or bf16 (out_dtype).  The product
 *           e2m1 * e4m3 is exact; the result is the exactly rounded
 *           (round-to-nearest-even) value of the full product in out_dtype. */
nvfp4_status nvfp4_dequant(const uint8_t* codes, const uint8_t* scales,
                           const float* global_scale, int64_t d_out, int64_t d_in,
                           void* out, nvfp4_dtype out_dtype, nvfp4_stream_t stream);

/* ------------------------------------------------------------------------ */
/* Export to the block-scaled FP4 GEMM operand layout                         */
/* ------------------------------------------------------------------------ */
/* "Replay the Curvature", Abstract, infrastructure sentence: each layer is
 * exported before its full-precision weights are retired.  The codes already
 * have the K-major data layout of an FP4 GEMM operand (two E2M1 nibbles per
 * byte, low nibble = even column); the E4M3 block scales are re-tiled here
 * into the layout in which block-scaled tensor-core GEMMs read the scale
 * operand of 16-element FP4 blocks: rows and scale columns padded (code 0) to
 * multiples of 128 and 4, tiles of 128 rows x 4 scale columns stored as 512
 * contiguous bytes in row-major tile order, and inside a tile the scale of row
 * r, column c at byte (r % 32) * 16 + (r / 32) * 4 + c.  The global scale s_g
 * is the GEMM's output scale.
 * out: device buffer of nvfp4_export_scales_size(d_out, d_in) bytes. */
size_t nvfp4_export_scales_size(int64_t d_out, int64_t d_in);
nvfp4_status nvfp4_export_scales(const uint8_t* scales, int64_t d_out, int64_t d_in,
                                 uint8_t* out, nvfp4_stream_t stream);

/* ------------------------------------------------------------------------ */
/* a10  layer error tr((W - Q) H (W - Q)^T) (measurement)                   */
/* ------------------------------------------------------------------------ */
size_t nvfp4_layer_error_workspace_size(int64_t d_out, int64_t d_in);

/* W, w_dtype : the original weights (dead columns contribute 0 because their
 *           H row is 0).  codes/scales/global_scale from the quantize call.
 * H       : d_in x d_in fp32, undamped, symmetric (the Hessian X^T X).  The
 *           error is evaluated as <H, E^T E> with E = W - Q: the Gram matrix
 *           E^T E is formed on its 128 x 128 tiles on or below the diagonal
 *           (3xTF32 on the tensor cores), and only those tiles of H are read.
 * err_out : device fp64 scalar out.
 * ws      : at least nvfp4_layer_error_workspace_size() bytes. */
nvfp4_status nvfp4_layer_error(const void* W, nvfp4_dtype w_dtype, const uint8_t* codes,
                               const uint8_t* scales, const float* global_scale,
                               const float* H, int64_t d_out, int64_t d_in,
                               double* err_out, void* ws, size_t ws_bytes,
                               nvfp4_stream_t stream);

/* ------------------------------------------------------------------------ */
/* Batched forms: `count` independent problems per call                      */
/* ("Replay the Curvature", Abstract: a layer's solve is independent of the  */
/* other layers' and, in a mixture-of-experts layer, every expert is its own */
/* linear layer with its own Hessian).                                       */
/* ------------------------------------------------------------------------ */
/* Every array argument is a HOST array of length count holding the per-problem
 * value of the argument of the same name in the single-problem call (device
 * pointers and sizes); the per-problem rules and layouts are those of the
 * single-problem call, and every result equals the single call's bit for bit.
 * Optional per-problem pointers (dead, lambda_out, err_out) may be given as a
 * NULL array.
 *
 * Problems of equal shape (d; or d_out and d_in) are solved together: each
 * kernel launch of the call covers all problems of one shape (up to 256; a
 * larger set makes one group per 256), so the number of launches grows with
 * the number of distinct shapes, not with count.  Problems are grouped in
 * their order of appearance.
 *
 * Scratch: ONE device workspace for the whole call (256-byte aligned), of
 * nvfp4_prepare_batched_workspace_size() / nvfp4_quantize_batched_workspace_
 * size() bytes for the same count and sizes -- the sum of the problems'
 * single-call workspaces, so split a call whose total does not fit.  It
 * starts with a status header: nvfp4_workspace_status() on it returns the
 * first non-OK status of any problem, nvfp4_batched_workspace_status() also
 * each problem's own (a timed-out wait inside a launch that serves several
 * problems is reported for each of them).
 *
 * Every argument is checked on the host before anything is launched: the
 * first problem that fails a check decides the returned status and then
 * nothing is queued.  count == 0 is a no-op; count < 0 or a NULL required
 * array is NVFP4_ERR_INVALID_ARG. */
size_t nvfp4_prepare_batched_workspace_size(int count, const int64_t* d);
size_t nvfp4_quantize_batched_workspace_size(int count, const int64_t* d_out,
                                             const int64_t* d_in,
                                             const nvfp4_solve_params* params);

/* Synchronizes `stream`, writes problem i's status word to status[i] (host
 * array of count ints, may be NULL) and returns the first non-OK status of
 * any problem of the batched call that last used ws. */
nvfp4_status nvfp4_batched_workspace_status(const void* ws, int count, int* status,
                                            nvfp4_stream_t stream);

/* Tensor-core problems (bf16 tokens, d >= 256, n_tok >= 64, 16-byte aligned)
 * of one d run in one launch per 128 problems, heaviest token counts first;
 * any other problem runs on its own.  No workspace. */
nvfp4_status nvfp4_hessian_accumulate_batched(int count, float* const* H, const void* const* X,
                                              nvfp4_dtype x_dtype, const int64_t* n_tok,
                                              const int64_t* d, int beta,
                                              nvfp4_stream_t stream);

nvfp4_status nvfp4_gptq_prepare_batched(int count, const float* const* H, const int64_t* d,
                                        float damp, float* const* U, uint8_t* const* dead,
                                        float* const* lambda_out, void* ws, size_t ws_bytes,
                                        nvfp4_stream_t stream);

nvfp4_status nvfp4_gptq_schur_replay_quantize_batched(
    int count, const void* const* W, nvfp4_dtype w_dtype, const int64_t* d_out,
    const int64_t* d_in, const float* const* U, const nvfp4_solve_params* params,
    const uint8_t* const* dead, uint8_t* const* codes, uint8_t* const* scales,
    float* const* global_scale, double* const* err_out, void* ws, size_t ws_bytes,
    nvfp4_stream_t stream);

/* The layer error of every problem (H: each problem's undamped d_in x d_in
 * Hessian; err_out: each problem's device fp64 scalar).  Scratch: one
 * workspace of nvfp4_layer_error_batched_workspace_size() bytes; a timed-out
 * wait of a launch is reported for every problem of that launch's shape. */
size_t nvfp4_layer_error_batched_workspace_size(int count, const int64_t* d_out,
                                                const int64_t* d_in);
nvfp4_status nvfp4_layer_error_batched(int count, const void* const* W, nvfp4_dtype w_dtype,
                                       const uint8_t* const* codes, const uint8_t* const* scales,
                                       const float* const* global_scale, const float* const* H,
                                       const int64_t* d_out, const int64_t* d_in,
                                       double* const* err_out, void* ws, size_t ws_bytes,
                                       nvfp4_stream_t stream);

/* No workspace. */
nvfp4_status nvfp4_dequant_batched(int count, const uint8_t* const* codes,
                                   const uint8_t* const* scales,
                                   const float* const* global_scale, const int64_t* d_out,
                                   const int64_t* d_in, void* const* out, nvfp4_dtype out_dtype,
                                   nvfp4_stream_t stream);

/* ------------------------------------------------------------------------ */
/* Diagnostics: launch accounting and per-phase device timing                */
/* (measurement support; the paper has no counterpart)                       */
/* ------------------------------------------------------------------------ */
/* The factorisation's fp32 GEMM building block, exposed so that it can be
 * tested on its own (the paper has no counterpart):
 *   C = beta C + alpha P Q^T   on the tensor cores, 3xTF32 (fp32 accuracy),
 * P: M x K (ldp), Q: N x K (ldq), C: M x N (ldc), fp32 row-major device
 * arrays; P and Q 16-byte aligned with ldp, ldq multiples of 4.  lower != 0
 * (M == N): only the 128 x 128 tiles on or below the diagonal are written.
 * status: device int, 0 on entry; a timed-out wait inside the kernel sets it
 * to NVFP4_ERR_TIMEOUT. */
nvfp4_status nvfp4_gemm_nt_f32(int64_t M, int64_t N, int64_t K, float alpha, const float* P,
                               int64_t ldp, const float* Q, int64_t ldq, float beta, float* C,
                               int64_t ldc, int lower, int* status, nvfp4_stream_t stream);

/* Number of kernels this library has launched since it was loaded (all
 * threads, all devices).  Host-only; never fails. */
long long nvfp4_launch_count(void);

/* Debugging support (the paper has no counterpart; it stands in for a memory
 * checker).  The library is also built as libnvfp4pw_debug.so with
 * NVFP4_DEBUG defined: there every kernel checks the tile and index
 * arithmetic it derives from the call's shapes (a tile decomposition that
 * leaves its output, a row or column past the array) before each access; a
 * failed check skips the access and records NVFP4_ERR_BOUNDS in the call's
 * status word (for the tensor-core Hessian: the status nvfp4_hessian_status
 * reads).  Results are otherwise identical to the release build.  Returns 1
 * in the debug build, 0 in the release build.  Host-only; never fails. */
int nvfp4_debug_build(void);

/* Failure-detection support (the paper has no counterpart).  Sets, for the
 * current device, how long a pipeline wait inside the library's tensor-core
 * kernels (a TMA copy to land, an MMA stage or accumulator to be released)
 * may spin before the kernel gives up: ns nanoseconds of wall time, 0 for the
 * default of 4 s.  A wait that runs out records NVFP4_ERR_TIMEOUT in the
 * call's status word; the kernel then waits (always with the 4 s bound) for
 * the copies and MMAs it has already issued, frees its tensor memory and
 * returns, so the context stays usable.  A limit shorter than a kernel's
 * normal waits makes it time out: that is how the timeout path is tested;
 * with ns = 1 a wait gives up as soon as one non-blocking probe finds that
 * what it waits for has not happened yet (the first copy of a kernel always
 * takes longer), so every tensor-core kernel then times out.
 * Synchronous (it writes the limit to device memory); returns NVFP4_ERR_CUDA
 * if that write fails.  Not for use while library kernels run. */
nvfp4_status nvfp4_set_wait_limit_ns(unsigned long long ns);

/* Phases reported by nvfp4_profile_end, in this order. */
enum {
  NVFP4_PHASE_HESSIAN = 0, /* nvfp4_hessian_accumulate                      */
  NVFP4_PHASE_PREPARE = 1, /* nvfp4_gptq_prepare                            */
  NVFP4_PHASE_REPLAY = 2,  /* Schur Replay batch kernels of the quantize call */
  NVFP4_PHASE_UPDATE = 3,  /* trailing-update GEMMs of the quantize call    */
  NVFP4_PHASE_DEQUANT = 4, /* nvfp4_dequant                                 */
  NVFP4_PHASE_OTHER = 5,   /* everything else (prologues, reductions)       */
  NVFP4_PHASE_FACTOR_GEMM = 6, /* inside PREPARE: its fp64 mma.sync GEMMs   */
  NVFP4_PHASE_PANEL = 7,   /* inside PREPARE: its Cholesky panel launches  */
  NVFP4_PHASE_FACTOR_I8 = 8, /* inside PREPARE: its int8-slice GEMMs (with
                                their slicing launches); work = fp64 flops */
  NVFP4_NUM_PHASES = 9
};

/* Starts a profiling window: from now on every phase above records a CUDA
 * event pair on its launching stream.  Resets the per-phase launch counts. */
nvfp4_status nvfp4_profile_begin(void);

/* Ends the window: waits for the recorded events and writes, for phases
 * 0..n_phases-1, the summed device time in ms (ms[]) and the number of kernel
 * launches (launches[]; a launch counts in the innermost phase open, so the
 * PREPARE count excludes its FACTOR_GEMM and PANEL launches while its time
 * includes them).  NVFP4_OTHER's time is not measured (0).  Returns
 * NVFP4_ERR_CUDA if an event could not be read. */
nvfp4_status nvfp4_profile_end(double* ms, long long* launches, int n_phases);

/* Algorithmic work the launches of each phase did inside the last profiling
 * window, counted by the launchers from their shapes: for FACTOR_GEMM the
 * flops a triangular-aware GEMM must do (2 M N K, halved where only a
 * triangle of C is wanted or P is triangular), for PANEL the flops of the
 * panel's Cholesky, inverse and slice solve.  Other phases report 0.  Call
 * after nvfp4_profile_end. */
nvfp4_status nvfp4_profile_work(double* work, int n_phases);

#ifdef __cplusplus
}
#endif
#endif /* NVFP4PW_H */
