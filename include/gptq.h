/*
 * gptq.h -- C ABI of the B200 (sm_100a) GPTQ per-layer solve.
 *
 * The operations follow the GPTQ descriptions on these pages:
 *   [Tutorial]  "GPTQ：一键量化大模型压缩": §二阶信息 (H = 2 sum x x^T),
 *               §逐层量化 (layer objective ||W X - W^ X||_F^2), §误差补偿 (OBS
 *               compensation), §分组方案 (min-max scale/zero, groups).
 *   [Survey]    "LLM 量化技术" blog: §1.2 (x_q = round(x/s + z), s(x_q - z)),
 *               §2.3 (fixed column order, blocks of B = 128, Cholesky rows of H^-1).
 *   [Card]      "GPTQ: Accurate Post-Training Quantization for Generative
 *               Pre-trained Transformers" reading card, 方法适配 (lazy batch
 *               updates, Cholesky reformulation with mild damping).
 *   [Explainer] "一文读懂GPTQ" §三 (codes packed into int32 arrays; bits,
 *               group_size, desc_act).
 *
 * Conventions for every entry point
 *   - Matrices are row-major.  Device pointers are CUDA global memory owned by
 *     the caller; the library keeps no pointer after a call returns and
 *     allocates no device memory (scratch comes from the caller's workspace).
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  Work is
 *     enqueued on it; what a call synchronises is stated per call.
 *   - Arguments are validated on the host before anything is enqueued; a bad
 *     argument returns GPTQ_ERR_INVALID_ARG and touches no memory.
 *   - No kernel traps.  Every wait inside a kernel is bounded (about one
 *     second); a wait that runs out records GPTQ_ERR_TIMEOUT in a device status
 *     word that the synchronising calls (and gptq_check_device_status) report.
 *   - Return value: a gptq_status (int).
 */
#ifndef GPTQ_B200_GPTQ_H
#define GPTQ_B200_GPTQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same object as cudaStream_t. */
typedef struct CUstream_st *gptq_stream_t;

typedef enum {
  GPTQ_OK = 0,
  GPTQ_ERR_INVALID_ARG = 1, /* an argument failed validation; nothing was enqueued  */
  GPTQ_ERR_NOT_PD = 2,      /* damped H has a non-positive pivot (not positive definite) */
  GPTQ_ERR_CUDA = 3,        /* a CUDA runtime call failed                           */
  GPTQ_ERR_NO_MEMORY = 4,   /* workspace smaller than the size query returned       */
  GPTQ_ERR_TIMEOUT = 5      /* a bounded in-kernel wait ran out                     */
} gptq_status;

/* Static English text for a status code (never NULL). */
const char *gptq_status_string(int status);

/*
 * gptq_hessian_accumulate -- H += 2 X^T X   ([Tutorial] §二阶信息, H = 2 sum_i x_i x_i^T)
 *
 *   X    device, fp16 (IEEE binary16 bits), [n x d] row-major with leading
 *        dimension ldx (elements): row t is the activation vector of token t.
 *        16-byte aligned; ldx >= d and ldx % 8 == 0.
 *   n    number of tokens, n >= 0 (n == 0 enqueues nothing; X may then be NULL).
 *   d    input features, d > 0 and d % 32 == 0.
 *   H    device, fp32 [d x d] row-major (leading dimension d), 16-byte aligned.
 *        On return (stream order) H = sym(upper(H_in) + 2 X^T X): the upper
 *        triangle accumulates, and the lower triangle is written with the
 *        mirror of the new upper triangle.  Pass H = 0 for a fresh Hessian;
 *        calling repeatedly over token chunks sums them.
 *   Products of fp16 values are exact in fp32; the fp32 sums are folded out of
 *   the tensor-core accumulator every 512 tokens to bound rounding growth.
 *   Asynchronous: returns after enqueueing one kernel.
 */
int gptq_hessian_accumulate(const void *X, int64_t n, int64_t d, int64_t ldx, float *H,
                            gptq_stream_t stream);

/*
 * Options of the layer solve: a bit field, 0 for the plain solve.  Unknown bits
 * are invalid arguments.
 *   GPTQ_ACT_ORDER      quantise columns in order of descending diag(H)
 *                       ([Explainer] §三, desc_act).
 *   GPTQ_SYMMETRIC      the symmetric quantiser ("LLM 量化技术" §1.2): zero point 0,
 *                       s = max|x| / (2^(bits-1) - 1) over the group (1 for an
 *                       all-zero group), signed codes in [-2^(bits-1),
 *                       2^(bits-1) - 1] stored as code + 2^(bits-1) (so every
 *                       zero point is 2^(bits-1)).
 *   GPTQ_STATIC_GROUPS  each group's parameters come from the original W over
 *                       the layer's own column groups [k*group, (k+1)*group),
 *                       fixed before the sweep, instead of from the compensated
 *                       W when the sweep reaches the group; under act-order the
 *                       groups stay contiguous, g_idx[c] = c / group.  No effect
 *                       with group = -1.
 */
#define GPTQ_ACT_ORDER 1
#define GPTQ_SYMMETRIC 2
#define GPTQ_STATIC_GROUPS 4

/*
 * gptq_quantize_workspace_bytes -- device workspace needed by gptq_quantize_layer
 * for these arguments (0 if the arguments are invalid).  The workspace must be
 * 256-byte aligned.
 */
size_t gptq_quantize_workspace_bytes(int64_t r, int64_t d, int bits, int group, int block,
                                     int options);

/*
 * gptq_quantize_layer -- GPTQ solve of one linear layer
 *   ([Card] 方法适配; [Survey] §2.3; [Tutorial] §误差补偿, §分组方案)
 *
 * Steps, all on the GPU in stream order:
 *   1. lambda = damp * mean(diag H); H_d = H + lambda I.
 *   2. GPTQ_ACT_ORDER: perm = stable argsort of -diag(H) (ties keep the lower
 *      index); columns of W and rows/columns of H_d are taken in that order.
 *   3. U = upper Cholesky factor of H_d^-1 (U^T U = H_d^-1), computed as the
 *      "reverse" Cholesky H_d = R R^T (R upper) and U = R^-1.
 *   4. For j = 0..d-1 in blocks of `block` columns: at a group start, per-row
 *      s = (xmax - xmin)/(2^bits - 1) and z = rint(-xmin/s) over the current
 *      group columns (xmin <= 0 <= xmax; s = 1 if the range is empty); for
 *      group = -1 once per row from the original W (GPTQ_SYMMETRIC and
 *      GPTQ_STATIC_GROUPS change these parameters, see above).  q = clamp(rint(w_j/s) + z,
 *      0, 2^bits - 1), w^_j = s (q - z), e_j = (w_j - w^_j)/U_jj, and the
 *      later columns of the block move by -e_j U[j, j+1:].  Later blocks are
 *      moved once per block (lazy batch) or once per 1024 columns, an exact
 *      reordering of the same updates.
 *   5. loss = ||(W - W^) X^T||_F^2 = 1/2 tr(D H D^T) with D = W - W^ and the
 *      undamped H, evaluated as sum_j 1/2 e_j^2 - lambda/2 ||D||_F^2.
 *   6. Codes are returned in the original column order and packed.
 *
 *   W         device fp32 [r x d], read only.  W, H, W_hat and g_idx must be
 *             16-byte aligned; codes, qweight, scales and zeros 4-byte aligned.
 *   r, d      r >= 0 (r == 0: returns GPTQ_OK with *loss = 0, enqueues nothing),
 *             d > 0, d % 32 == 0.
 *   H         device fp32 [d x d], full symmetric (as written by
 *             gptq_hessian_accumulate).  CONSUMED: overwritten with the
 *             factorisation (U in the upper triangle without GPTQ_ACT_ORDER;
 *             the contents are unspecified with it).
 *   bits      2, 3, 4 or 8.
 *   group     -1 (one scale/zero per row) or a multiple of 32 that divides d
 *             with block % group == 0 or group % block == 0.
 *   block     32, 64 or 128 (the lazy-batch width B; the pages use 128).
 *   damp      relative damping >= 0 (the pages' "mild damping"; 0.01 typical).
 *   options   0 or a combination of GPTQ_ACT_ORDER, GPTQ_SYMMETRIC and
 *             GPTQ_STATIC_GROUPS.
 *   W_hat     device fp32 [r x d] or NULL: dequantised weights s(q - z) in the
 *             original column order.  May alias W.
 *   qweight   device int32 [r x d*bits/32]: per row, the codes of columns
 *             0..d-1 as an LSB-first bit stream (code c at stream bits
 *             [c*bits, (c+1)*bits), stream bit k = bit k%32 of word k/32).
 *   scales    device fp32 [r x G], G = d/group (G = 1 for group = -1).
 *             Column k belongs to quantisation group k (permuted positions
 *             [k*group, (k+1)*group) under act-order; original columns
 *             [k*group, (k+1)*group) with GPTQ_STATIC_GROUPS).
 *   zeros     device int32 [r x G], integer zero points in [0, 2^bits - 1].
 *   g_idx     device int32 [d] or NULL: group of each original column.
 *   codes     device uint8 [r x d] or NULL: unpacked codes, original order.
 *   loss      host double or NULL: the layer loss of step 5.
 *   workspace device scratch of at least gptq_quantize_workspace_bytes(...)
 *             bytes, 256-byte aligned; contents on entry are ignored.
 *   Synchronises `stream` once, at the end, to read the status and the loss.
 *   Returns GPTQ_ERR_NOT_PD if the damped H is not positive definite (outputs
 *   are then unspecified), GPTQ_ERR_NO_MEMORY if workspace_bytes is too small.
 */
int gptq_quantize_layer(const float *W, int64_t r, int64_t d, float *H, int bits, int group,
                        int block, float damp, int options, float *W_hat, int32_t *qweight,
                        float *scales, int32_t *zeros, int32_t *g_idx, uint8_t *codes,
                        double *loss, void *workspace, size_t workspace_bytes,
                        gptq_stream_t stream);

/*
 * gptq_factor / gptq_quantize_with_factor -- the solve in two halves, so that
 * one factor serves several sweeps: rows of one layer spread over several
 * GPUs, or several layers that read the same inputs and so share H.  The
 * inverse-Hessian information does not depend on W ([Card] 方法适配: every row
 * is quantised in the same order with the same factor).
 *
 * gptq_factor: steps 1-3 of gptq_quantize_layer.
 *   H        device fp32 [d x d], full symmetric, 16-byte aligned.  On return
 *            its upper triangle holds U in sweep order (the factor of the
 *            permuted H_d under GPTQ_ACT_ORDER); the strictly lower triangle is
 *            scratch.
 *   options  GPTQ_ACT_ORDER is used; the other bits are accepted and ignored.
 *   perm     device int32 [d] (GPTQ_ACT_ORDER; may be NULL otherwise): column
 *            perm[j] of W is quantised j-th.
 *   lambda   device fp32 [1]: the damping added to the diagonal (the loss
 *            needs it).
 *   workspace  gptq_factor_workspace_bytes(d, options) bytes, 256-byte aligned.
 *   Synchronises `stream` once, at the end; returns GPTQ_ERR_NOT_PD if H_d is
 *   not positive definite.
 *
 * gptq_quantize_with_factor: steps 4-6 of gptq_quantize_layer from a factor
 *   made by gptq_factor with the same d and GPTQ_ACT_ORDER bit (U, perm and
 *   lambda are read only, so they can serve any number of calls).  Other
 *   arguments as gptq_quantize_layer; the workspace is
 *   gptq_quantize_with_factor_workspace_bytes(r, d, bits, group, block) bytes.
 *   A perm that is not a permutation of 0..d-1 is found on the device before
 *   anything uses it and returns GPTQ_ERR_INVALID_ARG (outputs unspecified).
 *   Synchronises `stream` once, at the end, to read the status and the loss.
 */
size_t gptq_factor_workspace_bytes(int64_t d, int options);
int gptq_factor(float *H, int64_t d, float damp, int options, int32_t *perm, float *lambda,
                void *workspace, size_t workspace_bytes, gptq_stream_t stream);
size_t gptq_quantize_with_factor_workspace_bytes(int64_t r, int64_t d, int bits, int group,
                                                 int block);
int gptq_quantize_with_factor(const float *W, int64_t r, int64_t d, const float *U,
                              const int32_t *perm, const float *lambda, int bits, int group,
                              int block, int options, float *W_hat, int32_t *qweight,
                              float *scales, int32_t *zeros, int32_t *g_idx, uint8_t *codes,
                              double *loss, void *workspace, size_t workspace_bytes,
                              gptq_stream_t stream);

/*
 * gptq_pack -- pack codes into int32 words   ([Explainer] §三, int32 storage of 3/4-bit codes)
 *
 *   codes   device uint8 [r x d], values < 2^bits (higher bits are masked off).
 *   d       d > 0, d % 32 == 0.   bits: 2, 3, 4 or 8.
 *   qweight device int32 [r x d*bits/32], layout as in gptq_quantize_layer.
 *   Asynchronous.
 */
int gptq_pack(const uint8_t *codes, int64_t r, int64_t d, int bits, int32_t *qweight,
              gptq_stream_t stream);

/*
 * gptq_dequant_gemv -- y = x W^^T straight from a packed layer
 *   ([Card] §计算设置: the quantised layers run through a dequantising
 *   matrix-vector kernel at inference; [Explainer] §三: int32 packing,
 *   group_size and desc_act)
 *
 *   W^[row, c] = scales[row, gi(c)] * (q[row, c] - zeros[row, gi(c)]), with q the
 *   bits-bit code of column c unpacked from qweight (the layout gptq_quantize_layer
 *   and gptq_pack write) and gi(c) = g_idx[c] if g_idx is given, else c / group
 *   (0 for group = -1).
 *
 *   qweight device int32 [r x d*bits/32];  scales device fp32 [r x G];
 *   zeros   device int32 [r x G], G = 1 (group = -1) or d / group;
 *   g_idx   device int32 [d] or NULL (entries outside [0, G) are clamped to it);
 *   x       device fp32 [m x d] row-major, 16-byte aligned;
 *   y       device fp32 [m x r] row-major, written.
 *   d % 32 == 0; bits 2, 3, 4 or 8; group -1 or a multiple of 32 dividing d;
 *   0 <= m <= GPTQ_GEMV_MAX_M.  r == 0 or m == 0: nothing to do.  Invalid
 *   arguments return GPTQ_ERR_INVALID_ARG before anything is launched.
 *   Accumulation in fp32.  Asynchronous.
 */
#define GPTQ_GEMV_MAX_M 8
int gptq_dequant_gemv(const int32_t *qweight, const float *scales, const int32_t *zeros,
                      const int32_t *g_idx, int64_t r, int64_t d, int bits, int group,
                      const float *x, int64_t m, float *y, gptq_stream_t stream);

/*
 * gptq_dequant_fp16 / gptq_linear_fp16 -- run a quantised layer forward on
 * calibration tokens, to calibrate the next layer on what this one outputs
 *   ([Card] §计算设置: each block is quantised, then run to produce the next
 *   block's inputs; [Concept] §3 技術原理: the codes are dequantised to FP16
 *   and multiplied in floating point)
 *
 * gptq_dequant_fp16: W16[row, c] = fp16(scales[row, gi(c)] * (q[row, c] -
 *   zeros[row, gi(c)])) from the packed layer (arguments as gptq_dequant_gemv;
 *   W16 device fp16 [r x d], 16-byte aligned, written).  Asynchronous.
 * gptq_linear_fp16: Y = fp16(X W16^T) -- X device fp16 [n x d] (tokens x
 *   features), W16 device fp16 [r x d], Y device fp16 [n x r], all row-major and
 *   16-byte aligned; d % 32 == 0, r % 32 == 0.  fp32 accumulation on the tensor
 *   cores, folded every 512 features, one rounding to fp16 per output (values
 *   beyond the fp16 range become +-inf).  n == 0 or r == 0: nothing to do.
 *   Asynchronous; a bounded in-kernel wait that runs out is reported by
 *   gptq_check_device_status.
 * Both return GPTQ_ERR_INVALID_ARG before launching anything when an argument
 * is out of range.
 */
int gptq_dequant_fp16(const int32_t *qweight, const float *scales, const int32_t *zeros,
                      const int32_t *g_idx, int64_t r, int64_t d, int bits, int group, void *W16,
                      gptq_stream_t stream);
int gptq_linear_fp16(const void *X, int64_t n, int64_t d, const void *W16, int64_t r, void *Y,
                     gptq_stream_t stream);

/*
 * gptq_quantize_layer_noalloc -- gptq_quantize_layer for callers that cannot
 * allocate device memory.  (The GPTQ pages have no counterpart: this is a
 * deployment convenience of this library, not a step of the method.)
 *
 * Some callers cannot call cudaMalloc -- they run inside a memory pool that
 * forbids side allocations, or their runtime has reserved the whole device in
 * advance, or they can hand over only inputs and outputs.  This entry point
 * takes its scratch from a fixed array of GPTQ_NOALLOC_SCRATCH_BYTES bytes in
 * the library's own device memory instead of a workspace argument; every GPU
 * that loads the library holds that array until the process exits.  It calls
 * no allocator of any kind and creates no stream, event or graph (phase timing,
 * gptq_set_phase_timing, does not apply to this path).
 *
 *   Arguments, results and synchronisation are those of gptq_quantize_layer
 *   without the workspace pair.
 *   Arguments are checked first (GPTQ_ERR_INVALID_ARG as for
 *   gptq_quantize_layer); then the limit: returns GPTQ_ERR_NO_MEMORY (nothing enqueued) when
 *   gptq_quantize_workspace_bytes(r, d, bits, group, block, options) exceeds
 *   GPTQ_NOALLOC_SCRATCH_BYTES -- e.g. r = d = 2048 fits, r = d = 4096 does not.
 *   The first call on a device looks up the array's device address (once per
 *   device, with that device current); make that first call before any stream
 *   capture.  All calls share the one array, and each call leaves its contents
 *   behind; the next call clears what it needs cleared.  Calls whose work may
 *   overlap on the GPU (different streams or threads without ordering) race on
 *   the array: serialise them.
 */
#define GPTQ_NOALLOC_SCRATCH_BYTES ((size_t)64 << 20)
int gptq_quantize_layer_noalloc(const float *W, int64_t r, int64_t d, float *H, int bits,
                                int group, int block, float damp, int options, float *W_hat,
                                int32_t *qweight, float *scales, int32_t *zeros, int32_t *g_idx,
                                uint8_t *codes, double *loss, gptq_stream_t stream);

/*
 * gptq_layer_host_workspace_bytes / gptq_solve_layer_host -- the whole layer
 * from HOST buffers: copy X and W to the device, H = 2 X^T X, quantise, pack,
 * and copy qweight, scales, zeros, g_idx and the loss back.
 *
 *   X_host   host fp16 bits [n x d] (pinned memory gives full copy bandwidth).
 *   W_host   host fp32 [r x d].
 *   outputs  host buffers with the shapes of gptq_quantize_layer (g_idx_host
 *            may be NULL).
 *   dev_workspace  device scratch of gptq_layer_host_workspace_bytes(...) bytes,
 *            256-byte aligned; it holds the device copies of X, W, H and the
 *            outputs plus the quantiser's workspace.
 *   X is copied in chunks of max(32768, ceil(n/64)) tokens on a second stream
 *   (created once per device) and H is accumulated chunk by chunk as the chunks
 *   land -- the same H as gptq_hessian_accumulate called once per chunk -- so
 *   the Hessian overlaps the upload.
 *   Synchronous: returns when the outputs are in the host buffers.
 */
size_t gptq_layer_host_workspace_bytes(int64_t r, int64_t d, int64_t n, int bits, int group,
                                       int block, int options);
int gptq_solve_layer_host(const uint16_t *X_host, int64_t n, const float *W_host, int64_t r,
                          int64_t d, int bits, int group, int block, float damp, int options,
                          int32_t *qweight_host, float *scales_host, int32_t *zeros_host,
                          int32_t *g_idx_host, double *loss, void *dev_workspace,
                          size_t dev_workspace_bytes, gptq_stream_t stream);

/*
 * gptq_check_device_status -- synchronise `stream`, then return and clear the
 * library's device status word (GPTQ_ERR_TIMEOUT if an asynchronous kernel,
 * such as the Hessian, gave up on a bounded wait; GPTQ_OK otherwise).
 */
int gptq_check_device_status(gptq_stream_t stream);

/*
 * Text describing the last CUDA failure seen by this thread ("" if none):
 * source location, the failing call and the CUDA error name.  Valid until the
 * next failure on the same thread.
 */
const char *gptq_last_error(void);

/* Number of kernels this library has launched in this process (all devices). */
uint64_t gptq_launch_count(void);

/*
 * Phase timing for gptq_quantize_layer (off by default, process-wide, not
 * thread-safe).  When on, each call records CUDA events on its stream between
 * phases; gptq_last_phase_ms writes up to `n` durations in ms of the last call:
 *   [0] damping + act-order permutation
 *   [1] Cholesky factor and triangular inverse (U)
 *   [2] working copy of W and column sweep (in-block kernels and
 *       trailing-update GEMMs)
 *   [3] unpermute, loss and packing
 * and returns the number written.
 */
int gptq_set_phase_timing(int enable);
int gptq_last_phase_ms(float *ms, int n);

/*
 * gptq_selftest_timeout -- exercises the failure path of the kernels' bounded
 * waits (no page counterpart: a check of this library's error handling).
 * Launches one tensor-core GEMM of 128 x 128 x 256 on `stream` whose operand
 * loads stop after two of its eight K steps, so its waits for the missing
 * stages run out after about one second; the kernel then records
 * GPTQ_ERR_TIMEOUT in the library's device status word, waits (bounded) for its
 * own tensor-core work, frees its tensor memory and returns.  Nothing faults
 * and the context stays usable; gptq_check_device_status(stream) afterwards
 * returns GPTQ_ERR_TIMEOUT once (and clears it).
 *
 *   buf   device scratch of 81920 floats (320 KB), 16-byte aligned; its
 *         contents are read and partly overwritten.
 * Returns GPTQ_OK once launched, GPTQ_ERR_INVALID_ARG for a bad buffer.
 */
int gptq_selftest_timeout(float *buf, gptq_stream_t stream);

/*
 * gptq_gemm_pair_form -- which launch form the library's two-CTA tensor-core
 * product (the trailing updates and the factorisation's products with two or
 * more 128-row tiles) runs in on the current device; a diagnostic with no page
 * counterpart.  Before its first such product on a device the library tries,
 * with launches that return at once, the forms
 *   0  CTA pairs along y, cluster shape, priority and programmatic
 *      serialisation given at launch;   1  the same, cluster shape only;
 *   2  pairs along x, as 0;              3  pairs along x, as 1;
 *   4  pairs along x with a compile-time cluster shape, priority and
 *      programmatic serialisation;       5  the same as a plain launch;
 * and keeps the first the driver accepts; 6 = none was accepted and every
 * product runs on the one-CTA kernel.  The probe runs only while the pairs
 * are enabled (gptq_set_gemm_pair).
 *
 *   log, log_bytes  optional: receives the last probe's record, "form:result"
 *                   per form tried (NUL-terminated, truncated to log_bytes).
 * Returns the form (0 .. 6), or -1 when no product has probed this device yet
 * (or no device is current).
 */
int gptq_gemm_pair_form(char *log, size_t log_bytes);

/*
 * gptq_set_gemm_pair -- chooses the kernel of the library's products with two
 * or more 128-row tiles (trailing updates, factorisation products): nonzero =
 * CTA pairs (tcgen05.mma.cta_group::2, M = 256, each CTA loading half of B) in
 * the launch form gptq_gemm_pair_form reports; 0 = one CTA per 128 x 128 tile
 * (the default, measured faster on the 4096- and 49152-wide layers).  Both
 * give the same results up to the order of fp32 additions within a K step.
 * Process-wide; takes effect for later calls (cached CUDA graphs are keyed by
 * the setting).  Returns the previous setting (0 or 1).
 */
int gptq_set_gemm_pair(int enable);

/*
 * gptq_factor_plan -- a host-only diagnostic of the factorisation's schedule
 * (the Cholesky and inverse steps of gptq_quantize_layer): writes, without
 * touching a GPU, one text line per kernel the factorisation of a d x d H_d
 * would launch and per stream event it would record or wait on, in program
 * order.  The schedule is a blocked right-looking Cholesky taken from the
 * bottom-right corner with U assembled over a merge tree (the "LLM 量化技术"
 * blog §2.3 item 3 and the GPTQ reading card, 方法适配, call for a Cholesky in
 * place of an explicit inverse); the plan lets a test replay it in any order
 * its streams and events allow.
 *
 *   d             matrix size (a multiple of 32, at most 65536).
 *   outer_cols    outer block width S (a multiple of 128, or d); 0 = the width
 *                 gptq_quantize_layer uses for this d.
 *   side_streams  nonzero: the schedule with side streams (as in
 *                 gptq_quantize_layer); 0: everything on one stream.
 *   buf, buf_bytes  output text (NUL-terminated; may be NULL to query the size).
 *
 * Line formats (pointers as a buffer name and a float offset: A = the d x d
 * matrix, row stride d; T = the factorisation scratch):
 *   P d=<d> S=<S> T=<scratch floats> side=<0|1>
 *   L s=<stream> A=<ptr> ld=<ld> nb=<nb>                  leaf: block -> its U
 *   G s=<stream> M= N= K= A= lda= B= ldb= C= ldc= alpha= beta= flags= tb= prio=
 *                                                         C = alpha A op(B) + beta C
 *   C s=<stream> dst= ldd= src= lds= rows= cols=          2-D copy
 *   E s=<stream> e=<id>                                   record event id on a stream
 *   W s=<stream> e=<id>                                   the stream waits for the event
 * GEMM flags: 1 = A upper (k from the row tile), 2 = op(B) lower (k from the
 * column tile), 4 = B upper (k to the column tile), 8 = output tiles on or
 * above the diagonal only; tiles are 128 x 128.
 * Returns the bytes the full text needs (including the NUL), or 0 for invalid
 * arguments.
 */
size_t gptq_factor_plan(int64_t d, int64_t outer_cols, int side_streams, char *buf,
                        size_t buf_bytes);

#ifdef __cplusplus
}
#endif

#endif /* GPTQ_B200_GPTQ_H */
