/*
 * gq.h -- C ABI of libgq.so: layer-wise 4-bit post-training weight
 * quantization (GPTQ and round-to-nearest) on NVIDIA B200 (sm_100a).
 *
 * Sources (page title -- section):
 *   "GPTQ: Post-Training INT4" -- "OBQ Foundation", "Hessian-Based Weight
 *       Update", "The GPTQ Algorithm", "Group Quantization", "Running GPTQ
 *       with AutoGPTQ".
 *   "Model Quantization Mechanics: Precision Reduction and Weight
 *       Formatting" -- section 1 (affine and group-wise quantization),
 *       section 2.1 (GPTQ objective; Cholesky factor of the inverse Hessian).
 *   "GPT-2 Quantization Reconstruction Error" -- "What this project does"
 *       (4-bit symmetric per-channel RTN with 15 levels; per-layer MSE).
 *
 * Conventions shared by every entry point:
 *   - Every array pointer is a DEVICE pointer owned by the caller, except
 *     the ones whose name ends in _host.  Arrays are dense and row-major.
 *   - The library allocates no device memory.  Entry points that need
 *     scratch take a caller-owned workspace (ws, ws_bytes) whose minimum
 *     size the matching gq_*_workspace_size() returns; ws must be 256-byte
 *     aligned.  Workspace contents need not be initialised.
 *   - Work is enqueued asynchronously on `stream` (a cudaStream_t; NULL is
 *     the legacy default stream).  An entry point returns before the GPU
 *     work finishes unless it documents a synchronisation.
 *   - Argument errors are detected on the host and returned before any
 *     launch; nothing is written then.  GQ_ERR_CUDA reports a launch or
 *     runtime error (gq_last_error() gives the text).
 *   - Device-side failures: every wait inside a kernel (on a tensor-memory
 *     accelerator copy or a tensor-core result) gives up after 2 s instead
 *     of spinning forever and records GQ_ERR_TIMEOUT (7) in the call's
 *     device status word, the first int32 of its workspace (0 = no failure;
 *     the call resets it).  Calls that synchronise (the Cholesky call with
 *     info_host, the reconstruction error with sse_host or mse_host, the
 *     scaling search) read that word and return GQ_ERR_TIMEOUT; an
 *     asynchronous caller reads it with gq_workspace_status() after the
 *     work, before reusing the workspace.  The Hessian and reconstruction
 *     error write NaN into their result when a wait gave up.
 *   - Shapes: W is d_out x d_in; X (calibration activations) is
 *     n_tok x d_in in bf16.  d_in must be a positive multiple of 8;
 *     d_out >= 1; n_tok >= 0 (an empty calibration batch adds nothing).
 *   - Code width `bits`: 4 (the pages' INT4), or 2, 3 or 8 ("GPT-2
 *     Quantization Reconstruction Error", "Possible extensions": 4-bit
 *     against 8-bit; "Quantization sweep: perplexity vs compression": INT8
 *     and INT4).  Widths other than 4 need d_in and the group size to be
 *     multiples of 32, and GPTQ block_size 128.
 *   - Packed codes: each row is one little-endian bit stream along d_in in
 *     which column k occupies bits `bits`*k .. `bits`*k + bits - 1, cut into
 *     uint32 words: qpacked is [d_out][bits * d_in / 32].  At 4 bits nibble
 *     k of word j is column 8j+k; at 8 bits byte k of word j is column 4j+k.
 *     Symmetric codes -q..q (q = 2^(bits-1) - 1: 15 levels at 4 bits) are
 *     stored as c + 2^(bits-1); affine codes 0..2^bits - 1 as they are.
 *   - Scales and zeros are IEEE fp16 bit patterns (uint16), [d_out][n_groups]
 *     with n_groups = d_in / group_size, or 1 for group_size -1 and 0.  Zeros
 *     hold the integer zero-point 0..2^bits - 1 (0 for symmetric).
 *   - group_size is -1 (one group per output row), 0 (one scale for the
 *     whole matrix -- "GPT-2 Quantization Reconstruction Error", "Possible
 *     extensions": per-tensor scaling -- stored once per row, so the output
 *     has the per-row layout and every consumer treats it like -1) or a
 *     multiple of 8 that divides d_in; for GPTQ it is -1, 0, 32, 64 or 128
 *     and divides block_size.  A per-tensor GPTQ scale comes from the whole
 *     initial matrix, as a per-row one comes from the initial row.
 *   - Inputs must be finite; non-finite values give unspecified codes.
 */
#ifndef GQ_H
#define GQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef int32_t gq_status;
enum {
  GQ_OK = 0,
  GQ_ERR_ARG = 1,         /* null pointer, bad flag or unsupported option   */
  GQ_ERR_SHAPE = 2,       /* sizes violate the rules above                  */
  GQ_ERR_DTYPE = 3,       /* unknown gq_dtype                               */
  GQ_ERR_WORKSPACE = 4,   /* ws too small or misaligned                     */
  GQ_ERR_NOT_PD = 5,      /* damped Hessian not positive definite           */
  GQ_ERR_NONFINITE = 6,   /* a non-finite value where one is not allowed    */
  GQ_ERR_TIMEOUT = 7,     /* a bounded device-side wait gave up             */
  GQ_ERR_CUDA = 8         /* CUDA runtime / launch error                    */
};

typedef int32_t gq_dtype;
enum { GQ_F32 = 0, GQ_F16 = 1, GQ_BF16 = 2 };

/* Human-readable name of a status code (static string). */
const char *gq_status_string(gq_status s);

/* Detail of the last error returned on the calling host thread (static,
 * thread-local; empty string if none). */
const char *gq_last_error(void);

/* Number of kernels this library has launched in the process so far. */
uint64_t gq_launch_count(void);

/* ------------------------------------------------------------------------
 * Hessian accumulation.
 * "GPTQ: Post-Training INT4", "Hessian-Based Weight Update": the Hessian
 * of the layer-wise objective is H = 2 X X^T, the same for every output
 * row; with X stored tokens x d_in (the orientation of the listing in "The
 * GPTQ Algorithm") this is H = 2 X^T X.  The call is additive, so a
 * calibration set larger than memory is fed in several calls.
 *
 *   X   [n_tok][d_in] bf16 (device, read only, 16-byte aligned)
 *   H   [d_in][d_in] fp32 (device, in/out): on return
 *       H := sym(H) + 2 X^T X, where sym(H) takes the upper triangle
 *       (i <= j) of the incoming H and mirrors it; the result is exactly
 *       symmetric.
 *   ws  >= gq_hessian_workspace_size(n_tok, d_in) bytes.
 * Accumulates in fp32 on the tensor cores (bf16 x bf16 products are exact
 * in fp32), in fixed token chunks whose partial sums are added in a fixed
 * order: results are deterministic run to run.
 * ---------------------------------------------------------------------- */
size_t gq_hessian_workspace_size(int64_t n_tok, int64_t d_in);
gq_status gq_hessian_accumulate(const void *X_bf16, int64_t n_tok, int64_t d_in,
                                float *H, void *ws, size_t ws_bytes, void *stream);
/* As gq_hessian_accumulate, but H := 2 X^T X: the incoming contents of H
 * are neither read nor needed (no separate clearing of H). */
gq_status gq_hessian_compute(const void *X_bf16, int64_t n_tok, int64_t d_in, float *H,
                             void *ws, size_t ws_bytes, void *stream);

/* ------------------------------------------------------------------------
 * Damping, act-order and the upper Cholesky factor of the inverse Hessian.
 * "GPTQ: Post-Training INT4", "Running GPTQ with AutoGPTQ" (damp_percent,
 * desc_act) and "The GPTQ Algorithm" (Cholesky of H, then its inverse);
 * "Model Quantization Mechanics", section 2.1 (GPTQ uses a Cholesky
 * decomposition of the inverse Hessian).
 *
 * Steps, in order:
 *   1. dead columns: where H_jj == 0, set H_jj := 1 and mark the column
 *      (dead_out[j] = 1, else 0); GPTQ zeroes those weight columns;
 *   2. H_jj += damp_percent * mean_j(H_jj);
 *   3. act_order != 0: perm = the columns by descending H_jj, ties by lower
 *      index first (written to perm_out), and H := H[perm][:, perm];
 *   4. U := the upper-triangular matrix with positive diagonal such that
 *      H^-1 = U^T U (written to U; the strictly lower part is zero).
 *
 *   H          [d_in][d_in] fp32, exactly symmetric (device, in, 16-byte
 *              aligned; used as scratch: contents unspecified on return)
 *   perm_out   [d_in] int32 (device, out) -- required iff act_order != 0
 *   dead_out   [d_in] uint8 (device, out) or NULL
 *   U          [d_in][d_in] fp32 (device, out, 16-byte aligned)
 *   info_dev   int32 (device, out) or NULL: -1 on success, else a column
 *              (in processing order) at which the factorisation met a
 *              non-positive or non-finite pivot.
 *   info_host  int32 (host, out) or NULL.  If non-NULL the call
 *              synchronises the stream once at its end, stores the info
 *              value there and returns GQ_ERR_NOT_PD on failure.
 *   ws         >= gq_damp_cholesky_workspace_size(d_in) bytes.
 * Computed in fp32: a blocked Cholesky of the index-reversed matrix, whose
 * reversed inverse is U (no separate inverse of H is formed).  The
 * inverse's block steps run on a second stream forked from and joined back
 * to `stream` with events; that helper stream is created on first use for
 * each (device, caller stream) pair and kept until the process exits (none
 * is created while `stream` is being captured into a graph: the whole call
 * then stays on `stream`).  Callers that create many short-lived streams
 * should reuse a few instead.
 * ---------------------------------------------------------------------- */
size_t gq_damp_cholesky_workspace_size(int64_t d_in);
gq_status gq_damp_cholesky_inverse(float *H, int64_t d_in, float damp_percent,
                                   int act_order, int32_t *perm_out, uint8_t *dead_out,
                                   float *U, int32_t *info_dev, int32_t *info_host,
                                   void *ws, size_t ws_bytes, void *stream);

/* ------------------------------------------------------------------------
 * gq_damp_cholesky_inverse without a workspace.
 * The pages have no counterpart to this entry point; it exists for callers
 * that cannot allocate device memory and so cannot supply `ws`: code whose
 * device memory is all owned by a host framework's pool or fixed budget
 * (an extra cudaMalloc would bypass its accounting, or fail because the
 * memory is already reserved), and code that must not stall on cudaMalloc /
 * cudaFree, which can synchronise the whole device.
 *
 * Arguments and results are those of gq_damp_cholesky_inverse without
 * (ws, ws_bytes).  Limit: d_in <= 4096; larger d_in returns GQ_ERR_SHAPE
 * before any launch.  The scratch is a fixed ~2 MiB array in device memory
 * that every GPU using this library holds until the process exits; the
 * call allocates nothing.  The first call on a device looks up that
 * array's device address (once per device, for the current device); make
 * that first call before any stream capture.  All calls share the one
 * array: calls whose GPU work may overlap (other streams, other host
 * threads on the same device) race on it and must be serialised by the
 * caller.
 * ---------------------------------------------------------------------- */
gq_status gq_damp_cholesky_inverse_noalloc(float *H, int64_t d_in, float damp_percent,
                                           int act_order, int32_t *perm_out,
                                           uint8_t *dead_out, float *U, int32_t *info_dev,
                                           int32_t *info_host, void *stream);

/* ------------------------------------------------------------------------
 * GPTQ on one layer.
 * "GPTQ: Post-Training INT4", "The GPTQ Algorithm": columns in a fixed
 * left-to-right order (the act-order permutation if given) in blocks of
 * block_size columns; for column j of a block the code q of the current
 * weight w, the scaled error delta = (w - q) / U_jj, the in-block update
 * w[j+1:end] -= delta * U[j, j+1:end]; after the block the lazy trailing
 * update W[:, end:] -= Err * U[blk, end:].  A group's scale (and zero) is
 * taken from that group's current (already updated) weights when its first
 * column is reached ("Group Quantization"); per-channel (group_size == -1)
 * scales come from the initial row.  Symmetric grid: s = absmax / q, codes
 * -q..q (q = 7 at 4 bits); affine ("Model Quantization Mechanics", section
 * 1): s = (max' - min') / m with the range widened to contain 0, z =
 * rint(-min'/s), codes 0..m (m = 15 at 4 bits).  The fp16-rounded scale is
 * the one used; a scale that is 0
 * in fp16 becomes 1 (and z = 0); codes are rint(w / s) + z clamped, with
 * IEEE division and round-half-to-even, in fp32.
 *
 *   W          [d_out][d_in] in w_dtype (device, read only; not modified)
 *   U          [d_in][d_in] fp32 upper factor from gq_damp_cholesky_inverse
 *              (in processing order)
 *   bits       2, 3, 4 or 8 (see the conventions above)
 *   group_size -1, 0 (per tensor), 32, 64 or 128, dividing d_in and block_size
 *   block_size 32, 64 or 128 (the pages' value is 128; 128 unless bits is 4)
 *   sym        1 symmetric, 0 affine
 *   perm       [d_in] int32 processing order (act-order) or NULL
 *   dead       [d_in] uint8 dead-column mask or NULL
 *   qpacked    [d_out][bits*d_in/32] uint32 (out), original column order
 *   scales     [d_out][n_groups] fp16 bits (out); with perm, group k holds
 *              processing positions k*g .. k*g+g-1
 *   zeros      [d_out][n_groups] fp16 bits (out) or NULL (sym)
 *   g_idx      [d_in] int32 (out) or NULL: the group of each original
 *              column (position in perm / group_size)
 *   ws         >= gq_gptq_workspace_size(d_out, d_in, block_size) bytes;
 *              holds the fp32 working copy of W (4 d_out d_in bytes) and
 *              the scaled errors of one super-block (4 d_out S bytes).
 * The lazy update is applied on two levels with the same terms: after a
 * block, to the rest of its super-block of S columns (S = block_size times
 * a power of two near sqrt(d_in / block_size)); after a super-block, to all
 * columns beyond it at once.  Only the order of the fp32 sums differs from
 * the one-level form.
 * ---------------------------------------------------------------------- */
size_t gq_gptq_workspace_size(int64_t d_out, int64_t d_in, int block_size);
gq_status gq_gptq_quantize_layer(const void *W, gq_dtype w_dtype, int64_t d_out, int64_t d_in,
                                 const float *U, int bits, int group_size, int block_size,
                                 int sym, const int32_t *perm, const uint8_t *dead,
                                 uint32_t *qpacked, uint16_t *scales, uint16_t *zeros,
                                 int32_t *g_idx, void *ws, size_t ws_bytes, void *stream);

/* ------------------------------------------------------------------------
 * Round-to-nearest baseline with packing (int4, and the other widths).
 * "GPT-2 Quantization Reconstruction Error", "What this project does"
 * (per output row scale, 15 levels), "Model Quantization Mechanics",
 * section 1 (affine; groups of g consecutive weights), "GPTQ: Post-Training
 * INT4", "Group Quantization" (4 + 16/g (+16/g) bits per weight).  Same
 * grid, rounding and storage as gq_gptq_quantize_layer, on the raw weights
 * with no feedback.  Bit-exact and deterministic.
 *
 *   W        [d_out][d_in] in w_dtype (device, read only, 16-byte aligned)
 *   bits     2, 3, 4 or 8
 *   qpacked  [d_out][bits*d_in/32] uint32 (out)
 *   scales   [d_out][n_groups] fp16 bits (out)
 *   zeros    [d_out][n_groups] fp16 bits (out) or NULL (written with 0
 *            when sym and non-NULL)
 * ---------------------------------------------------------------------- */
gq_status gq_rtn_quantize_pack(const void *W, gq_dtype w_dtype, int64_t d_out, int64_t d_in,
                               int bits, int group_size, int sym, uint32_t *qpacked,
                               uint16_t *scales, uint16_t *zeros, void *stream);

/* ------------------------------------------------------------------------
 * Layer reconstruction error.
 * "Model Quantization Mechanics", section 2.1 and "GPTQ: Post-Training
 * INT4", "OBQ Foundation": the objective ||W X - W^ X||^2 (here with X
 * tokens x d_in: ||(W - W^) X^T||_F^2); "GPT-2 Quantization Reconstruction
 * Error" reports it per layer as an MSE over the layer's outputs.
 *
 *   W, w_dtype         original weights [d_out][d_in] (device)
 *   qpacked, scales,   the quantised layer (device), as produced above;
 *   zeros, g_idx       zeros NULL when sym; g_idx NULL unless act-order
 *   bits, group_size,  as the layer was quantised with
 *   sym
 *   X                  [n_tok][d_in] bf16 (device, 16-byte aligned)
 *   sse_dev            double (device, out): SSE = ||(W - W^) X^T||_F^2
 *   sse_host, mse_host double (host, out) or NULL; if either is non-NULL
 *                      the call synchronises the stream once at its end.
 *                      MSE = SSE / (n_tok * d_out).
 *   ws                 >= gq_recon_workspace_size(d_out, d_in, n_tok) bytes
 * W - W^ is formed in fp32 and fed to the tensor cores as a bf16 hi + lo
 * pair (X is exactly bf16); squares are summed in fp32 per tile and in
 * fp64 across tiles in a fixed order (deterministic).
 * ---------------------------------------------------------------------- */
size_t gq_recon_workspace_size(int64_t d_out, int64_t d_in, int64_t n_tok);
gq_status gq_recon_error(const void *W, gq_dtype w_dtype, const uint32_t *qpacked,
                         const uint16_t *scales, const uint16_t *zeros, const int32_t *g_idx,
                         int64_t d_out, int64_t d_in, int bits, int group_size, int sym,
                         const void *X_bf16, int64_t n_tok, double *sse_dev,
                         double *sse_host, double *mse_host, void *ws, size_t ws_bytes,
                         void *stream);

/* ------------------------------------------------------------------------
 * Layer reconstruction error from the Hessian (the same SSE by a second
 * route).  With H0 = 2 X^T X (undamped, as gq_hessian_accumulate returns
 * it), ||(W - W^) X^T||_F^2 = tr((W - W^) X^T X (W - W^)^T) = tr(dW H0
 * dW^T) / 2 ("GPTQ: Post-Training INT4", "Hessian-Based Weight Update": the
 * layer-wise objective is the quadratic form of H).  Costs 2 d_out d_in^2
 * flops instead of 2 n_tok d_out d_in, so it is the cheaper route whenever
 * the calibration set has more tokens than the layer has inputs.
 *
 *   W, ..., sym     as for gq_recon_error
 *   H0              [d_in][d_in] fp32 (device, read only, 16-byte aligned),
 *                   exactly symmetric, undamped
 *   n_tok           the number of calibration tokens H0 was accumulated
 *                   over (only for mse_host)
 *   sse_dev, sse_host, mse_host   as for gq_recon_error
 *   ws              >= gq_recon_error_hessian_workspace_size(d_out, d_in)
 *                   bytes (holds dW in fp32: 4 d_out d_in bytes)
 * dW is formed in fp32; the product dW H0 runs in fp32 accuracy on the
 * tensor cores (three TF32 products per term) and is never stored: each
 * output tile's sum of (dW H0) .* dW is kept in fp64 and the tiles are
 * added in a fixed order (deterministic).
 * ---------------------------------------------------------------------- */
size_t gq_recon_error_hessian_workspace_size(int64_t d_out, int64_t d_in);
gq_status gq_recon_error_hessian(const void *W, gq_dtype w_dtype, const uint32_t *qpacked,
                                 const uint16_t *scales, const uint16_t *zeros,
                                 const int32_t *g_idx, int64_t d_out, int64_t d_in, int bits,
                                 int group_size, int sym, const float *H0, int64_t n_tok,
                                 double *sse_dev, double *sse_host, double *mse_host, void *ws,
                                 size_t ws_bytes, void *stream);

/* ------------------------------------------------------------------------
 * Products with a quantised layer: consumers of the packed format.
 * "GPTQ: Post-Training INT4", "Group Quantization" and "Running GPTQ with
 * AutoGPTQ": the packed codes with 16-bit scales (and zeros) are what a
 * quantised model is served from.  Both calls multiply them with bf16
 * activations, Y = W^ X^T with W^ = s (c - z) per group, in one tensor-core
 * kernel that reads the packed codes and forms W^ in shared memory as it
 * goes (no dequantised copy of W in device memory).  W^ is exact as a bf16
 * hi + lo pair (an fp16 scale times a small integer), so the only error is
 * the fp32 accumulation over d_in terms.
 *
 *   qpacked, scales, zeros, g_idx, d_out, d_in, bits, group_size, sym
 *              the quantised layer as produced by the calls above
 *   X          [n_tok][d_in] bf16 (device, 16-byte aligned)
 *   ws         >= gq_w4a16_workspace_size(d_out, d_in, n_tok) bytes (the
 *              device status word only)
 *
 * gq_w4a16_matmul: Y [d_out][n_tok] fp32 (device, out, 16-byte aligned;
 * n_tok a multiple of 4), feature-major.
 *
 * gq_qlinear_bf16: the layer applied to X for the next layer's input,
 * token-major: Z[t][j] = act((X W^T)[t][j]) + R[t][j], rounded once to bf16.
 *   W_dense, w_dtype  used instead of the packed codes when qpacked is NULL
 *              (the layer before quantisation: [d_out][d_in], 16-byte
 *              aligned), else ignored
 *   act        GQ_ACT_NONE, GQ_ACT_RELU or GQ_ACT_GELU (the tanh form,
 *              0.5 x (1 + tanh(sqrt(2/pi) (x + 0.044715 x^3))))
 *   R          [n_tok][d_out] bf16 residual (device) or NULL
 *   Z          [n_tok][d_out] bf16 (device, out)
 * ---------------------------------------------------------------------- */
enum { GQ_ACT_NONE = 0, GQ_ACT_RELU = 1, GQ_ACT_GELU = 2 };
size_t gq_w4a16_workspace_size(int64_t d_out, int64_t d_in, int64_t n_tok);
gq_status gq_w4a16_matmul(const uint32_t *qpacked, const uint16_t *scales,
                          const uint16_t *zeros, const int32_t *g_idx, int64_t d_out,
                          int64_t d_in, int bits, int group_size, int sym, const void *X_bf16,
                          int64_t n_tok, float *Y, void *ws, size_t ws_bytes, void *stream);
gq_status gq_qlinear_bf16(const uint32_t *qpacked, const uint16_t *scales,
                          const uint16_t *zeros, const int32_t *g_idx, const void *W_dense,
                          gq_dtype w_dtype, int64_t d_out, int64_t d_in, int bits,
                          int group_size, int sym, const void *X_bf16, int64_t n_tok, int act,
                          const void *R_bf16, void *Z_bf16, void *ws, size_t ws_bytes,
                          void *stream);

/* ------------------------------------------------------------------------
 * Sequential quantisation of a chain of layers, each calibrated on the input
 * it actually receives: the output of the already quantised layers before
 * it ("GPT-2 Quantization Reconstruction Error", "Key findings": the
 * per-layer errors there were measured with the whole model running, so
 * upstream quantisation error reaches every later layer).
 *
 * For l = 0 .. n_layers - 1, on `stream`:
 *   H0 = 2 X_l^T X_l; dead columns, damping, U (no act-order); GPTQ of W_l
 *   into the layer's outputs; sse_dev[l] = ||(W_l - W^_l) X_l^T||_F^2 (by
 *   the Hessian route); X_{l+1}[t][j] = act_l((X_l W^_l^T)[t][j]) +
 *   X_r[t][j] if the layer names an earlier input r, rounded to bf16.
 *
 *   X0         [n_tok][layers[0].d_in] bf16 (device), the first input
 *   layers     host array of n_layers descriptors; layers[l].d_in must equal
 *              layers[l-1].d_out; a residual input X_r (0 <= r <= l) must
 *              have d_out columns
 *   bits, group_size, block_size, sym, damp_percent
 *              as for gq_gptq_quantize_layer / gq_damp_cholesky_inverse
 *   sse_dev    [n_layers] double (device, out)
 *   X_all_out  bf16 (device, out) or NULL: receives every input X_0 .. X_n
 *              (X_n is the chain's output), one after another, X_l taking
 *              n_tok * d_l elements with d_l = layers[l].d_in (d_n =
 *              layers[n-1].d_out)
 *   ws         >= gq_gptq_sequential_workspace_size(...) bytes: every input
 *              X_0 .. X_n (bf16), three d x d fp32 matrices for the widest
 *              layer, and the largest scratch of the steps
 * ---------------------------------------------------------------------- */
typedef struct {
  const void *W;          /* [d_out][d_in] (device, 16-byte aligned)          */
  gq_dtype w_dtype;
  int64_t d_out, d_in;
  int act;                /* GQ_ACT_* applied to the layer's output           */
  int residual_from;      /* -1, or r <= l: X_r is added to the output        */
  uint32_t *qpacked;      /* GPTQ outputs (device), as gq_gptq_quantize_layer */
  uint16_t *scales;
  uint16_t *zeros;        /* NULL when sym                                    */
} gq_seq_layer;

size_t gq_gptq_sequential_workspace_size(const gq_seq_layer *layers, int n_layers,
                                         int64_t n_tok, int block_size);
gq_status gq_gptq_sequential(const void *X0_bf16, int64_t n_tok, const gq_seq_layer *layers,
                             int n_layers, int bits, int group_size, int block_size, int sym,
                             float damp_percent, double *sse_dev, void *X_all_out_bf16,
                             void *ws, size_t ws_bytes, void *stream);

/* ------------------------------------------------------------------------
 * Activation-aware per-channel scaling before RTN.
 * "Model Quantization Mechanics", section 2.2: a per-channel factor s
 * multiplies the weights of input channels whose activations are large and
 * divides those activations, so the layer's output is unchanged while its
 * salient weights lose less to rounding; "GPT-2 Quantization Reconstruction
 * Error", "Possible extensions": scale important channels, chosen by
 * activation magnitude, before quantising.  The pages give no formula; this
 * call takes s_c = (H_cc / H_bar)^(alpha / 2) from the diagonal of the
 * undamped Hessian H = 2 X^T X (the channel RMS over its geometric mean,
 * to the power alpha; s_c = 1 where H_cc <= 0), tries alpha = k / n_grid
 * for k = 0 .. n_grid - 1, measures each as the layer error
 * ||(W - W^) X^T||^2 with W^ = dequant(RTN(W diag(s))) diag(s)^-1, and
 * quantises the layer with the alpha of the smallest error (the first on
 * ties).  alpha = 0 is plain RTN.
 *
 *   W, w_dtype   [d_out][d_in] (device, read only, 16-byte aligned)
 *   H            [d_in][d_in] fp32 undamped Hessian (device; only the
 *                diagonal is read), e.g. from gq_hessian_accumulate
 *   X            [n_tok][d_in] bf16 calibration inputs (device, 16-byte
 *                aligned), n_tok >= 1
 *   bits, group_size, sym   as for gq_rtn_quantize_pack
 *   n_grid       1 .. 256 (20 tries alpha = 0, 0.05, .., 0.95)
 *   qpacked, scales, zeros  (out) RTN of W diag(s) for the chosen alpha, in
 *                the layout of gq_rtn_quantize_pack; the dequantised
 *                weights must be divided by col_scale per input column
 *   col_scale    [d_in] fp32 (device, out) s of the chosen alpha, or NULL
 *   mse_host     [n_grid] double (host, out) the error per alpha divided by
 *                n_tok * d_out, or NULL
 *   best_host    int32 (host, out) the chosen k, or NULL
 *   ws           >= gq_awq_workspace_size(d_out, d_in, n_tok, group_size,
 *                sym) bytes, 256-byte aligned
 * Synchronises the stream once (the choice of alpha is made on the host).
 * ---------------------------------------------------------------------- */
size_t gq_awq_workspace_size(int64_t d_out, int64_t d_in, int64_t n_tok, int bits,
                             int group_size, int sym);
gq_status gq_awq_rtn_search(const void *W, gq_dtype w_dtype, int64_t d_out, int64_t d_in,
                            const float *H, const void *X_bf16, int64_t n_tok, int bits,
                            int group_size, int sym, int n_grid, uint32_t *qpacked,
                            uint16_t *scales, uint16_t *zeros, float *col_scale,
                            double *mse_host, int32_t *best_host, void *ws, size_t ws_bytes,
                            void *stream);

/* ------------------------------------------------------------------------
 * Device status of a call (a facility of this library; the pages have no
 * counterpart).
 *
 *   gq_workspace_status(ws, status_host, stream)
 *       synchronises `stream`, reads the device status word (the first
 *       int32 of the workspace `ws` that a call on that stream was given)
 *       into *status_host (if non-NULL) and returns GQ_OK, GQ_ERR_TIMEOUT
 *       if a device-side wait of that call gave up, or GQ_ERR_CUDA.
 *   gq_selftest_bounded_wait(arrive, limit_ns, ws, ws_bytes, stream)
 *       exercises the bounded wait itself: one thread waits on a
 *       shared-memory barrier (no copy, no tensor-core work); with arrive
 *       != 0 it arrives on the barrier first, else nothing ever arrives and
 *       the wait gives up after limit_ns (at most 1 s).  Records the result
 *       in word 0 of ws (>= 256 bytes, 256-byte aligned), synchronises, and
 *       returns GQ_OK or GQ_ERR_TIMEOUT like gq_workspace_status.
 * ---------------------------------------------------------------------- */
gq_status gq_workspace_status(const void *ws, int32_t *status_host, void *stream);
gq_status gq_selftest_bounded_wait(int arrive, uint64_t limit_ns, void *ws, size_t ws_bytes,
                                   void *stream);

/* ------------------------------------------------------------------------
 * Per-launch kernel timing (a measurement aid; the pages describe no such
 * facility).  A throughput figure for one kernel needs that kernel's own
 * duration, which events around a whole entry point (several kernels) do
 * not give.
 *
 *   gq_kernel_timer_start(mask, capacity)
 *       creates `capacity` CUDA event pairs on the current device.  From
 *       then on, every launch of a kernel whose bit (1 << gq_kernel) is set
 *       in `mask` is bracketed by an event pair recorded on the launch's
 *       own stream, together with the launch's algorithmic work, until
 *       `capacity` launches have been recorded or the timer is stopped.
 *       Inside a stream capture the pair is captured as external event
 *       nodes: every replay of the graph records it again, so a read after
 *       the replays gives the last replay's durations.  Launches on other
 *       devices are not recorded.  GQ_ERR_ARG if a session is active or
 *       capacity <= 0; GQ_ERR_CUDA if the events cannot be created.
 *   gq_kernel_timer_stop()
 *       no further launches are recorded (the records stay readable).
 *   gq_kernel_timer_read(kind, ms, work, max)
 *       after the recorded work has completed: fills up to `max` entries of
 *       the host arrays (the gq_kernel of the launch, its duration in ms,
 *       its algorithmic work) and returns the number of records, or -1 if
 *       an event cannot be read (the work has not run or not finished).
 *   gq_kernel_timer_release()
 *       destroys the events and ends the session.
 * The algorithmic work is counted in flops (2 per multiply-add) for
 * HESSIAN_MMA (symmetric half of X^T X), POTRF_TRSM, BLOCK_INVERSE,
 * GEMM_TF32X3 (the fp32 product; lower-triangle calls count the triangle),
 * RECON_MMA (one product (W - W^) X^T), QLINEAR (one product W^ X^T:
 * 2 n_tok d_out d_in) and SYRK_BF16 (the lower triangle of dW^T dW in the
 * error from the Hessian, three bf16 products: d_in (d_in + 1) d_out),
 * and in bytes that must cross
 * HBM for GPTQ_BLOCK (the block's working weights read, Err written, the U
 * block, codes and scales) and RTN (W read, codes, scales and zeros
 * written).  One session at a time per process; the calls are thread safe.
 * ---------------------------------------------------------------------- */
typedef enum {
  GQ_KERNEL_HESSIAN_MMA = 0,
  GQ_KERNEL_POTRF_TRSM = 1,
  GQ_KERNEL_BLOCK_INVERSE = 2,
  GQ_KERNEL_GEMM_TF32X3 = 3,
  GQ_KERNEL_GPTQ_BLOCK = 4,
  GQ_KERNEL_RTN = 5,
  GQ_KERNEL_RECON_MMA = 6,
  GQ_KERNEL_QLINEAR = 7,
  GQ_KERNEL_SYRK_BF16 = 8,
  GQ_KERNEL_COUNT = 9
} gq_kernel;

gq_status gq_kernel_timer_start(uint32_t mask, int32_t capacity);
gq_status gq_kernel_timer_stop(void);
int32_t gq_kernel_timer_read(int32_t *kind, float *ms, double *work, int32_t max);
gq_status gq_kernel_timer_release(void);

#ifdef __cplusplus
}
#endif
#endif /* GQ_H */
