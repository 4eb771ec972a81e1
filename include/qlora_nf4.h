/*
 * qlora_nf4.h -- C ABI of the B200 (sm_100a) QLoRA NF4 linear library.
 *
 * The library implements the hot path of a QLoRA linear layer:
 *
 *   1. NF4 blockwise quantization of a frozen fp32 weight W0 [rows, cols]
 *      (absolute maximum per block of 64 consecutive weights of the row-major
 *      flattening, nearest of the 16 NF4 levels, two 4-bit codes per byte with
 *      the even element in the low nibble).
 *      Source: "QLoRA: NF4 storage, gradients and local integration",
 *      sections "NF4: nonuniform reconstruction levels" and "Exact CPU
 *      teaching quantizer and adapter gradient path".
 *   2. Double quantization of the fp32 block scales: a per-tensor fp32 mean
 *      offset, int8 codes in chunks of 256 scales, one fp32 second-level
 *      absmax per chunk (about 4.127 bits per weight in total).
 *      Source: same page, section "Double quantization: correct the scale
 *      arithmetic"; "QLoRA Deep Dive: 4-bit NormalFloat & Double Quantization
 *      Internals", section "2. Squeezing More Memory: Double Quantization (DQ)".
 *   3. Dequantization to bf16 or fp32, and the LoRA linear forward and backward
 *         Y  = X W^T + s (X A^T) B^T
 *         dX = dY W + s (dY B) A,  dA = s (dY B)^T X,  dB = s dY^T (X A^T)
 *      with W the dequantized weight.
 *      Source: "QLoRA: NF4 storage, gradients and local integration", the
 *      gradient paragraph after the teaching program; "FT-02: QLoRA --
 *      Fine-Tuning with Quantization", section "4. The LoRA mechanics the API
 *      wraps" (LoRALinear, scaling = alpha / r).
 *
 * Conventions for every entry point:
 *   - Every pointer argument except host descriptor structs points to DEVICE
 *     memory owned by the caller.  The library allocates and frees nothing;
 *     scratch space is a caller-provided workspace whose size the matching
 *     *_ws_bytes function returns.
 *   - bf16 tensors are passed as uint16_t bit patterns, row-major.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  All work is
 *     enqueued on it and the call returns without waiting, except where a
 *     status must be read back (see qlora_nf4_quantize).
 *   - Alignment: fp32 weights to quantize and dense dequantize outputs 32
 *     bytes; packed codes, scale codes, bf16 activations and outputs 16 bytes;
 *     fp32 scalars and gradients 4.
 *     A misaligned pointer returns QLORA_ERR_ALIGNMENT.
 *   - Argument checks run on the host before anything is enqueued; a failed
 *     check returns an error status and enqueues nothing.
 *   - A CUDA launch or runtime error is returned as QLORA_ERR_CUDA.
 *   - Calls that share a workspace must not run concurrently on the GPU.
 *     Calls on different streams with different workspaces may overlap; the
 *     results do not depend on the overlap (every kernel sums in a fixed
 *     order), bit for bit.
 *   - Every call launches on the calling thread's current device; all its
 *     pointers must be that device's memory.  One process may use several
 *     devices (kernel attributes are set per device) and several host
 *     threads.
 */
#ifndef QLORA_NF4_H
#define QLORA_NF4_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum qlora_status {
  QLORA_OK = 0,
  QLORA_ERR_INVALID_ARG = 1,  /* null pointer, bad shape, bad rank, bad dtype  */
  QLORA_ERR_ALIGNMENT = 2,    /* a device pointer is not 16-byte aligned      */
  QLORA_ERR_NONFINITE = 3,    /* the weight to quantize holds NaN or Inf      */
  QLORA_ERR_WORKSPACE = 4,    /* workspace missing or smaller than required   */
  QLORA_ERR_CUDA = 5,         /* a CUDA runtime/launch error                  */
  QLORA_ERR_TIMEOUT = 6,      /* a device-side wait ran past its time limit   */
  QLORA_ERR_UNSUPPORTED = 7,  /* no sm_100 device, or a size beyond limits    */
  QLORA_ERR_CHECK = 8         /* a debug-build (QLORA_CHECKS) index or
                                 alignment test failed; the access was skipped */
} qlora_status;

/*
 * 4-bit codebooks.
 *   NF4: the 16 NormalFloat levels, ascending with the code ("QLoRA: NF4
 *        storage, gradients and local integration", section "Exact CPU
 *        teaching quantizer and adapter gradient path").
 *   FP4: the E2M1 grid of "FT-02: QLoRA -- Fine-Tuning with Quantization",
 *        section "Exercise 3: NF4 vs FP4 at equal memory": code bit 3 is the
 *        sign, bits 2..0 select the magnitude k/12, k = 0, 1/16, 2, 3, 4, 6,
 *        8, 12 (fp32-rounded).  Quantization never emits code 8 (-0).
 * Both quantize to the nearest level (fp32 distances), the lowest code on a
 * tie.
 */
typedef enum qlora_codebook { QLORA_CODEBOOK_NF4 = 0, QLORA_CODEBOOK_FP4 = 1 } qlora_codebook;

/*
 * Storage of the per-block scales.
 *   DQ_INT8 : double quantization, int8 codes q in [-127, 127] per block,
 *             t = fp32(q / 127) (4.127 bits per weight in all).
 *   DQ_FP8  : double quantization, E4M3 codes per block (stored in the same
 *             int8 array as bit patterns), q = E4M3(fp32(d / c2)) rounded to
 *             nearest even, t = the E4M3 value ("QLoRA Deep Dive: 4-bit
 *             NormalFloat & Double Quantization Internals", section "2.
 *             Squeezing More Memory: Double Quantization (DQ)": normalize by
 *             the chunk absmax, quantize to 8-bit floats).
 *   FP32    : no double quantization, the fp32 block absmax itself (4.5 bits
 *             per weight; same page, "Memory Savings Analysis").
 * Double-quantized scales decode as a = fp32(fp32(t * c2) + mu).
 */
typedef enum qlora_scale_format {
  QLORA_SCALES_DQ_INT8 = 0,
  QLORA_SCALES_DQ_FP8 = 1,
  QLORA_SCALES_FP32 = 2
} qlora_scale_format;

/* Element type of the dense weight given to the quantizer. */
typedef enum qlora_input_dtype { QLORA_INPUT_FP32 = 0, QLORA_INPUT_BF16 = 1, QLORA_INPUT_FP16 = 2 } qlora_input_dtype;

/*
 * One quantized tensor.  The struct itself lives in host memory; its pointers
 * are device memory owned by the caller.
 *   rows, cols   : W0 is [rows, cols] row-major (rows = d_out, cols = d_in);
 *                  cols must be a multiple of 64 so every block lies in one row.
 *   packed       : rows*cols/2 bytes; byte i holds code 2i (low nibble) and
 *                  code 2i+1 (high nibble).
 *   qscale       : rows*cols/64 scale codes, one per block (DQ formats):
 *                  int8 in [-127, 127] (DQ_INT8) or E4M3 bit patterns (DQ_FP8).
 *   c2           : ceil(rows*cols/16384) fp32 second-level scales, one per
 *                  chunk of 256 consecutive blocks (DQ formats).
 *   mu           : one fp32, the per-tensor mean of the block absmax values
 *                  (DQ formats).
 *   codebook     : qlora_codebook (0 = NF4).
 *   scale_format : qlora_scale_format (0 = DQ_INT8).
 *   absmax       : rows*cols/64 fp32 block scales (FP32 format only; 16-byte
 *                  aligned).  qscale, c2 and mu are unused (may be NULL) with
 *                  FP32 scales; absmax is unused (may be NULL) otherwise.
 * The weight decodes as fp32(L[code] * a), a the block scale (bf16 outputs
 * round that to nearest even).  A zero-initialized codebook / scale_format /
 * absmax is the NF4 double-quantized (int8) format.
 */
typedef struct qlora_nf4_weight {
  int64_t rows;
  int64_t cols;
  uint8_t *packed;
  int8_t *qscale;
  float *c2;
  float *mu;
  int32_t codebook;
  int32_t scale_format;
  float *absmax;
} qlora_nf4_weight;

/* Human-readable name of a status code (static string). */
const char *qlora_status_string(qlora_status status);

/*
 * Sizes of the quantized state of a [rows, cols] tensor and the workspace
 * qlora_nf4_quantize needs for it.  Any output pointer may be NULL.
 * n_blocks is also the length of the fp32 absmax array of QLORA_SCALES_FP32.
 * Errors: INVALID_ARG if rows < 1, cols < 64 or cols % 64 != 0.
 */
qlora_status qlora_nf4_sizes(int64_t rows, int64_t cols, size_t *packed_bytes, size_t *n_blocks,
                             size_t *n_chunks, size_t *ws_bytes);

/*
 * Quantize + double-quantize one fp32 tensor W [out->rows, out->cols]
 * (steps: block absmax, normalisation, nearest level of out->codebook,
 * packing; then, by out->scale_format, mean offset, second-level absmax per
 * 256-block chunk and int8 or E4M3 scale codes, or the fp32 absmax alone).
 * Results are bit-identical to the definition: fp32 IEEE division and
 * comparisons, fp64 strictly sequential mean (per chunk, then over chunks).
 *   W        : device fp32 input, not modified.
 *   out      : host struct describing the caller's output buffers.
 *   ws       : device workspace of at least qlora_nf4_sizes(...).ws_bytes.
 *   d_status : device int32 or NULL.  If non-NULL the call does not wait: the
 *              device writes 0 or QLORA_ERR_NONFINITE there when the work
 *              completes.  If NULL the call synchronizes `stream` and returns
 *              QLORA_ERR_NONFINITE itself when W holds NaN/Inf (the outputs are
 *              then unspecified).
 */
qlora_status qlora_nf4_quantize(const float *W, const qlora_nf4_weight *out, void *ws, size_t ws_bytes,
                                int32_t *d_status, void *stream);

/*
 * Quantize `count` independent tensors in one pass (same per-tensor results
 * as qlora_nf4_quantize on each; every tensor has its own mean offset).
 *   W    : host array of `count` device pointers.
 *   outs : host array of `count` descriptors.
 *   ws   : at least qlora_nf4_quantize_batched_ws_bytes(...) bytes.
 *   d_status, stream : as qlora_nf4_quantize (one status for the batch).
 */
size_t qlora_nf4_quantize_batched_ws_bytes(const qlora_nf4_weight *outs, int32_t count);
qlora_status qlora_nf4_quantize_batched(const float *const *W, const qlora_nf4_weight *outs, int32_t count,
                                        void *ws, size_t ws_bytes, int32_t *d_status, void *stream);

/*
 * Quantize dense weights given as fp32, bf16 or fp16 (qlora_input_dtype;
 * "FT-02: QLoRA -- Fine-Tuning with Quantization", section "3.
 * BitsAndBytesConfig in practice": checkpoints are 16-bit and are converted
 * at load time).  16-bit weights are widened to fp32 exactly and then
 * quantized as fp32 weights, so the result equals qlora_nf4_quantize of the
 * widened tensor.  Pointers, workspace and status as qlora_nf4_quantize /
 * qlora_nf4_quantize_batched; W is 32-byte aligned for fp32 and 16-byte
 * aligned for bf16 / fp16.  The codebook and scale format of the outputs
 * select the stored format; one call takes one format (every output of a
 * batch has the same codebook and scale_format, else QLORA_ERR_INVALID_ARG).
 */
qlora_status qlora_nf4_quantize_ex(const void *W, int32_t in_dtype, const qlora_nf4_weight *out, void *ws,
                                   size_t ws_bytes, int32_t *d_status, void *stream);
qlora_status qlora_nf4_quantize_batched_ex(const void *const *W, int32_t in_dtype, const qlora_nf4_weight *outs,
                                           int32_t count, void *ws, size_t ws_bytes, int32_t *d_status,
                                           void *stream);

/*
 * Quantize + double-quantize one tensor exactly as qlora_nf4_quantize does,
 * without a workspace.  (The pages have no counterpart: this is an interface
 * for callers, not a step of the method.)
 *
 * Some callers cannot allocate device memory or hand over a workspace: a
 * serving engine or framework plugin whose host reserves all device memory in
 * its own pool up front and forbids allocation while it runs, or a plain C
 * caller that owns no device allocator.  This entry point takes its scratch
 * from a fixed array inside the library instead: about 4.1 MB of device
 * memory that every GPU which loads the library holds until the process
 * exits.  It calls no cudaMalloc, cudaFree or other allocating routine.
 *   W, out, d_status, stream : as qlora_nf4_quantize.
 *   Limit: rows * cols <= 67,108,864 (2^26) weights; larger tensors return
 *   QLORA_ERR_UNSUPPORTED before anything is enqueued.
 * The first call on each device resolves the array's device address
 * (cudaGetSymbolAddress) for that device; make that first call before any
 * stream capture.  All calls on a device share the one array and it keeps
 * the previous call's contents (each call clears the parts that must start
 * at zero), so calls that overlap on the GPU -- on different streams or from
 * several host threads -- race and give wrong results: serialize them.
 */
qlora_status qlora_nf4_quantize_noalloc(const float *W, const qlora_nf4_weight *out, int32_t *d_status,
                                        void *stream);

/*
 * Dequantize to a dense [rows, cols] tensor.
 *   out_dtype : 0 = bf16 (uint16_t bit patterns), 1 = fp32.
 *   transpose : 0 = out is [rows, cols]; 1 = out is [cols, rows] (the
 *               transposed weight, bf16 only).
 * Bit-identical to the decode formula above.  No workspace.
 */
qlora_status qlora_nf4_dequantize(const qlora_nf4_weight *w, void *out, int32_t out_dtype, int32_t transpose,
                                  void *stream);
qlora_status qlora_nf4_dequantize_batched(const qlora_nf4_weight *weights, void *const *outs, int32_t count,
                                          int32_t out_dtype, void *stream);

/*
 * Merged dense weight of a LoRA-adapted layer:
 *     out = W + scale * B A          ([rows, cols], W the dequantized weight)
 * The dense layer that computes the same output as the two-branch forward
 * (Y = X out^T up to rounding).  Requantizing a merged layer is this call
 * with out_dtype = 1 followed by qlora_nf4_quantize on `out`.
 * Source: "FT-02: QLoRA -- Fine-Tuning with Quantization", section "4. The
 * LoRA mechanics the API wraps" (merge of W0 + (alpha / r) B A);
 * "QLoRA: NF4 storage, gradients and local integration", section "Merge
 * changes the operator: test it explicitly" (the merge uses the dequantized
 * weight; requantizing the merge moves it by Qhat(M) - M).
 *   w         : quantized weight, rows = N (d_out), cols = K (d_in).
 *   A         : bf16 [r, K].   B : bf16 [N, r] (both 2-byte aligned).
 *   r         : 1..64.  scale : s = alpha / r (finite).
 *   out       : [N, K] output, 16-byte aligned; out_dtype 0 = bf16, 1 = fp32.
 * Arithmetic: W[n][k] is the fp32 decode (bit-identical to
 * qlora_nf4_dequantize with out_dtype = 1); sum_j B[n][j] A[j][k] is a
 * tensor-core product of the bf16 operands with fp32 accumulation;
 * out = fma(scale, sum, W) in fp32, rounded to nearest-even for bf16.
 * No workspace.
 */
qlora_status qlora_merge(const qlora_nf4_weight *w, const uint16_t *A, const uint16_t *B, int32_t r, float scale,
                         void *out, int32_t out_dtype, void *stream);

/*
 * Device-side status of a linear-layer workspace.  Kernels record the first
 * device-detected error (QLORA_ERR_TIMEOUT: a barrier wait ran past its one
 * second limit, the kernel gave up and returned) in the first word of the
 * workspace; it stays set until read.
 *   qlora_workspace_reset  : zero the status word (enqueued on `stream`); call
 *                            once after allocating a workspace.
 *   qlora_workspace_status : synchronize `stream`, return the recorded status
 *                            (QLORA_OK if none) and clear it.
 */
qlora_status qlora_workspace_reset(void *ws, size_t ws_bytes, void *stream);
qlora_status qlora_workspace_status(void *ws, size_t ws_bytes, void *stream);

/*
 * Workspace bytes for qlora_linear_fwd / qlora_linear_bwd at tokens M,
 * weight [N, K] and rank r (the larger of the two needs; one workspace may
 * serve both) under the weight path in force (qlora_linear_set_weight_path).
 * Returns 0 for sizes the linear calls refuse: M < 1, N not a
 * positive multiple of 8, K not a positive multiple of 64, r outside 1..64,
 * or beyond the limits M <= 2^25, N and K < 2^31, N * K <= 2^40 (for
 * which the calls return QLORA_ERR_UNSUPPORTED).
 */
size_t qlora_linear_ws_bytes(int64_t M, int64_t N, int64_t K, int32_t r);

/*
 * Weight path of the tensor-core linear calls (M > 16).
 *   QLORA_WEIGHT_PATH_FUSED (default): the GEMM decodes the packed 4-bit
 *     weight and its block scales straight into its shared-memory operand
 *     tiles ("QLoRA Deep Dive: 4-bit NormalFloat & Double Quantization
 *     Internals", section "The Quantization Process in QLoRA": a block is
 *     multiplied back by its constant and used in the computation; "FT-02:
 *     QLoRA -- Fine-Tuning with Quantization", section "Reading the result:
 *     the three lines that decide memory": the weight stays in 4 bits and is
 *     dequantized on the fly).  No dense copy of the weight is written.
 *   QLORA_WEIGHT_PATH_DENSE: the ablation arm.  Each tensor-core call first
 *     dequantizes the whole weight to bf16 in the workspace (N * K * 2 more
 *     workspace bytes) and then runs a GEMM that reads that copy.
 * Both paths decode the same bf16 values and accumulate in the same order,
 * so their outputs are bit-identical.  The setting is process-wide; each
 * call reads it once.  qlora_linear_ws_bytes answers for the path in force
 * when it is called: a call on the dense path with a workspace sized for the
 * fused path returns QLORA_ERR_WORKSPACE.  A fused call on a device where
 * its kernel cannot be scheduled returns QLORA_ERR_UNSUPPORTED.
 *   qlora_linear_set_weight_path : INVALID_ARG for an unknown value.
 *   qlora_linear_weight_path     : the path in force.
 */
typedef enum qlora_weight_path { QLORA_WEIGHT_PATH_FUSED = 0, QLORA_WEIGHT_PATH_DENSE = 1 } qlora_weight_path;
qlora_status qlora_linear_set_weight_path(int32_t path);
int32_t qlora_linear_weight_path(void);

/*
 * LoRA linear forward:  Y = X W^T + scale * (X A^T) B^T.
 *   w     : quantized weight, rows = N (d_out), cols = K (d_in).
 *   X     : bf16 [M, K].   A : bf16 [r, K].   B : bf16 [N, r].
 *   r     : 1..64.  scale : s = alpha / r (finite).
 *   ws    : 256-byte aligned workspace of qlora_linear_ws_bytes(M, N, K, r).
 *   Y     : bf16 [M, N] output (overwritten).
 *   U_out : fp32 [M, r] output U = X A^T (keep it for the backward), or NULL.
 * M <= 16 runs the decode-shaped dequant-GEMV; larger M the tensor-core path.
 * Accumulation is fp32.  N must be a multiple of 8.
 */
qlora_status qlora_linear_fwd(const qlora_nf4_weight *w, const uint16_t *X, int64_t M, const uint16_t *A,
                              const uint16_t *B, int32_t r, float scale, uint16_t *Y, float *U_out, void *ws,
                              size_t ws_bytes, void *stream);

/*
 * Diagnostic of the bounded device waits (the pages have no counterpart: it
 * checks this library's failure detection, not a step of the method).
 * Runs the tensor-core forward of qlora_linear_fwd (M > 16, the fused weight
 * path) with the GEMM's MMA issuer first waiting on a barrier that nothing
 * arrives at, and every pipeline wait of the GEMM limited to wait_limit_us
 * microseconds (1 .. 1,000,000).  That wait runs out; the GEMM records
 * QLORA_ERR_TIMEOUT in the workspace status, every warp leaves its loop,
 * the copies already issued are waited for, tensor memory is freed and the
 * kernel returns, so the device and the stream stay usable.  Y is left
 * unspecified.  Returns QLORA_OK once enqueued (INVALID_ARG for M <= 16 or a
 * limit out of range); read the outcome with qlora_workspace_status.  The
 * other arguments are those of qlora_linear_fwd (no U output).
 */
qlora_status qlora_linear_fwd_stall_diagnostic(const qlora_nf4_weight *w, const uint16_t *X, int64_t M,
                                               const uint16_t *A, const uint16_t *B, int32_t r, float scale,
                                               uint16_t *Y, void *ws, size_t ws_bytes, int32_t wait_limit_us,
                                               void *stream);

/*
 * Self-test of the shared-memory barrier ring that the pipelined kernels use
 * (the pages have no counterpart: it checks this library's synchronisation,
 * not a step of the method).  One CTA: a producer thread writes the values
 * 1 .. iters into a ring of `stages` shared slots; one thread in each of
 * `consumers` warps reads every value in order.  A slot is published by an
 * mbarrier of one arrival and handed back by one of `consumers` arrivals.
 * Every wait takes the phase parity of its pass over the ring, as the GEMM
 * and side-product rings do, and gives up after wait_limit_us.
 *   stages     : 1 .. 8.   consumers : 0 .. 4 (0: nothing hands a slot back,
 *                so the producer's wait on its second pass runs out).
 *   iters      : 1 .. 2^24.   wait_limit_us : 1 .. 1,000,000.
 *   d_result   : device int32[3], 4-byte aligned, overwritten: [0] values a
 *                consumer read wrong, [1] values read (iters * consumers when
 *                every wait succeeded), [2] QLORA_ERR_TIMEOUT if a wait ran
 *                out, else 0.
 * Returns QLORA_OK once enqueued (INVALID_ARG for an argument out of range).
 */
qlora_status qlora_selftest_mbarrier_ring(int32_t stages, int32_t consumers, int32_t iters, int32_t wait_limit_us,
                                          int32_t *d_result, void *stream);

/*
 * Whether the debug checks are live in this library's device code (the pages
 * have no counterpart).  A library built with QLORA_CHECKS
 * (libqlora_nf4_checks.so) tests index and alignment conditions before the
 * accesses they guard and records QLORA_ERR_CHECK in the call's status word
 * when one fails, skipping the access.  This call runs one such test that
 * always fails, on no memory but the result word.
 *   d_result : device int32, 4-byte aligned, overwritten: QLORA_ERR_CHECK in
 *              the checks library, 0 in the default one.
 * Returns QLORA_OK once enqueued.
 */
qlora_status qlora_selftest_checks(int32_t *d_result, void *stream);

/*
 * LoRA linear backward for upstream gradient dY of Y.
 *   X, dY      : bf16 [M, K] and [M, N].
 *   U          : fp32 [M, r] = X A^T as saved by qlora_linear_fwd, or NULL to
 *                recompute it from X and A (one more pass over X).
 *   dX         : bf16 [M, K] output, or NULL to skip.  dX = dY W + s (dY B) A.
 *   accumulate : 0 overwrites dX, 1 adds into it (dX += ...; the sum is
 *                formed in fp32 and rounded once).
 *   dA         : fp32 [r, K] output, or NULL.   dA = s (dY B)^T X.
 *   dB         : fp32 [N, r] output, or NULL.   dB = s dY^T U.
 * dA and dB are overwritten, never accumulated.  No gradient is produced for
 * the frozen weight.
 */
qlora_status qlora_linear_bwd(const qlora_nf4_weight *w, const uint16_t *X, const uint16_t *dY, int64_t M,
                              const uint16_t *A, const uint16_t *B, int32_t r, float scale, const float *U,
                              uint16_t *dX, int32_t accumulate, float *dA, float *dB, void *ws, size_t ws_bytes,
                              void *stream);

/*
 * Kernel timing (instrumentation for benchmarks; off by default).
 * While enabled, every kernel the library enqueues is bracketed by CUDA
 * events recorded on the launching stream, grouped by family:
 *   "quantize" (quantize + double quant), "dequant", "gemv", "side" (rank-r
 *   products, gradient column sums, padding), "gemm" (tensor-core GEMM),
 *   "merge" (qlora_merge).
 *   qlora_timing_enable : 1 starts recording (clearing earlier records), 0 stops.
 *   qlora_timing_read   : waits for the recorded events of `family` and returns
 *                         the summed device time in milliseconds and the number
 *                         of launches since enabling; INVALID_ARG for an unknown
 *                         family name; CUDA if an event could not be read (the
 *                         other records are still summed and every record read
 *                         is consumed).
 * Host threads may enqueue concurrently while timing is enabled.  The events
 * belong to the device current at their creation: time one device per process.
 */
qlora_status qlora_timing_enable(int32_t enable);
qlora_status qlora_timing_read(const char *family, double *total_ms, int64_t *launches);

#ifdef __cplusplus
}
#endif

#endif /* QLORA_NF4_H */
