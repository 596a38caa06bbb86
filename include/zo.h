/*
 * zo.h -- C ABI of libzo.so: the data-parallel hot path of 1SPSA / 1.5-SPSA
 * zero-order training on one B200 (sm_100a).
 *
 * The method (cited by page title and section):
 *   [HOW] "Stanford's 1.5-SPSA Trains OPT-30B Without Backpropagation", section
 *         "How 1.5-SPSA Works": each step draws n_pert Rademacher probes z_i in
 *         {-1,+1}^M, evaluates the loss at theta + eps*z_i and theta - eps*z_i, and
 *         averages (L+ - L-)/(2 eps) * z_i over the probes.
 *   [PSP] same page, section "Probe-Space Preconditioning": one extra clean loss
 *         L0 per step gives a per-probe curvature; probes are weighted by
 *         |c_i|^alpha (alpha = 0.1) so that high-curvature directions are
 *         down-weighted.  The preconditioner lives in probe space (O(n_pert)).
 *   [ABS] "Probe-Space Preconditioning for Fast and Stable Zero-Order Training",
 *         abstract: training runs in inference mode with no stored activations,
 *         gradients or optimizer state; probes come from a packed (8 signs per byte)
 *         random generator and are applied by fused unpack/apply kernels.
 *   [LOOP] "Pretraining Transformers Without Backprop: What Two Zero-Order Papers
 *         Actually Measure", section "Backprop's memory tax", loop flowchart:
 *         directions -> forward passes (loss only) -> preconditioned estimate ->
 *         update -> repeat.
 *
 * Readings fixed by this library where the pages are silent:
 *   - Probe bits, 8 signs per byte with a byte holding one element's signs under 8
 *     consecutive probes: Philox4x32-10 (Salmon et al., SC'11), key = (seed lo,
 *     seed hi), counter = (g lo, g hi, i >> 3, step) with g = j >> 4; element j of
 *     probe i takes bit (i & 7) of byte (j & 15) of the little-endian 16-byte block
 *     (word (j >> 2) & 3, bits 8 (j & 3)..); bit 1 means z_ij = -1.  Probes are
 *     regenerated, never stored.  zo_pack_probe exports one probe with 8 elements per
 *     byte: byte q holds elements 8q..8q+7, bit t <-> element 8q+t.
 *   - Perturbed value P_j = rd(theta_j + s*eps*z_j): one fp32 add (RNE); bf16 weights
 *     are widened, added in fp32 and rounded to bf16 (RNE).
 *   - g_i = (L+_i - L-_i)/(2 eps); c_i = (L+_i + L-_i - 2 L0)/eps^2;
 *     w_i = (|c_i| + damping)^(-alpha) (1SPSA: w_i = 1); a_i = lr*w_i*g_i/n, all in
 *     fp64, a_i rounded once to fp32.
 *   - theta' = rd(theta - sum_i a_i z_i) with a fixed fp32 order: probes in octets of
 *     8 (each octet summed left to right from its first signed term), octet sums
 *     added left to right, one fp32 subtraction, one rounding to the storage type.
 *   - "In place" and "exact restore": theta is written only by zo_step/zo_update.
 *     A perturbation is a state of the context; kernels that need perturbed values
 *     compute them on load or materialise them into a scratch window (the whole
 *     vector when a live buffer is enabled, one decoder layer at a time otherwise).
 *     zo_restore therefore returns theta bit-exactly, with no pass over memory.
 *
 * Conventions for every call:
 *   - Pointers documented as "device" must be device memory of the current device
 *     (e.g. torch CUDA tensors); "host" pointers are ordinary host memory.
 *   - Calls enqueue work on the context's stream and return without synchronising,
 *     unless documented otherwise.  The step counter lives in device memory, so a
 *     whole step is enqueued without a host synchronisation.
 *   - Every call returns a zo_status; on failure zo_last_error(ctx) describes it.
 *     No call throws, aborts or prints.  A context is not thread-safe.
 */
#ifndef ZO_H
#define ZO_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct zo_ctx zo_ctx;

typedef enum { ZO_F32 = 0, ZO_BF16 = 1 } zo_dtype;

typedef enum {
  ZO_OK = 0,
  ZO_ERR_INVALID = 1,     /* bad argument (size, sign, eps, pointer alignment, dtype) */
  ZO_ERR_STATE = 2,       /* call not allowed in the context's perturbation state */
  ZO_ERR_CUDA = 3,        /* a CUDA runtime call or kernel launch failed */
  ZO_ERR_OOM = 4,         /* device allocation failed */
  ZO_ERR_NONFINITE = 5,   /* a loss was NaN/Inf: the step was skipped (theta unchanged) */
  ZO_ERR_UNSUPPORTED = 6, /* valid request this library does not support */
  ZO_ERR_TIMEOUT = 7      /* a kernel gave up a bounded wait (see ZO_FLAG_TIMEOUT) */
} zo_status;

/* Device-side status flags reported by zo_sync. */
#define ZO_FLAG_NONFINITE 0x1u /* a loss was not finite; that step was skipped */
#define ZO_FLAG_TIMEOUT 0x2u   /* a tensor-core kernel's pipeline wait expired (about 2 s);
                                  its output is invalid */

/* Largest n_pert accepted by zo_step / zo_update (the update keeps a 1 KB table per
 * group of 8 probes in shared memory: 128 KB at this limit). */
#define ZO_MAX_PROBES 1024

/* ------------------------------------------------------------------ context */

/* Create a context over the flat parameter vector theta [ABS: the weights are the only
 * training state].
 *   params  device, caller-owned, M elements of `dtype`, 16-byte aligned; must outlive
 *           the context.  The library writes it only in zo_step / zo_update.
 *   M       number of parameters, 1 <= M < 2^39.
 *   dtype   ZO_F32 or ZO_BF16.
 *   seed    64-bit probe seed (Philox key).
 *   stream  cudaStream_t to enqueue on (NULL = legacy default stream).
 * Allocates small device buffers (step counter, coefficients, reduction scratch).
 * Errors: ZO_ERR_INVALID (null out/params, M out of range, misaligned params, dtype),
 *         ZO_ERR_OOM, ZO_ERR_CUDA.  The step counter starts at 0. */
zo_status zo_create(zo_ctx **out, void *params, int64_t M, int dtype, uint64_t seed,
                    void *stream);

/* Free the context and everything it allocated (synchronises its stream first).
 * NULL is accepted.  theta is not touched. */
zo_status zo_destroy(zo_ctx *ctx);

/* Text of the last error on this context ("" if none); valid until the next call. */
const char *zo_last_error(const zo_ctx *ctx);

/* Constant name of a status code, e.g. "ZO_ERR_STATE". */
const char *zo_status_name(int status);

/* Exponent alpha of the probe-space weights (default 0.1 [PSP]); must be finite, >= 0. */
zo_status zo_set_alpha(zo_ctx *ctx, float alpha);

/* Enable (1) or disable (0) the full-size live buffer: while perturbed, a device copy
 * P = rd(theta + s*eps*z_i) of all M parameters is materialised by zo_perturb and
 * returned by zo_live_params.  Costs M elements of device memory.  Only allowed in the
 * clean state.  Errors: ZO_ERR_STATE, ZO_ERR_OOM. */
zo_status zo_set_live_buffer(zo_ctx *ctx, int enable);

/* The parameters a loss evaluation should read now: theta when clean (or when no live
 * buffer is enabled), else the live buffer.  NULL on a NULL context. */
const void *zo_live_params(const zo_ctx *ctx);

/* Synchronise the context's stream and return the sticky device flags (ZO_FLAG_*)
 * raised since the last call, clearing them; *flags may be NULL.  Returns
 * ZO_ERR_TIMEOUT if ZO_FLAG_TIMEOUT was raised, else ZO_ERR_NONFINITE if
 * ZO_FLAG_NONFINITE was raised, else ZO_OK. */
zo_status zo_sync(zo_ctx *ctx, uint32_t *flags);

/* Read (synchronising) or set (enqueued) the device-resident step counter, which keys
 * the probes of the current step.  Setting it is how a run resumes from a checkpoint
 * of (theta, seed, step): the method keeps no other state [ABS]. */
zo_status zo_get_step(zo_ctx *ctx, uint32_t *step);
zo_status zo_set_step(zo_ctx *ctx, uint32_t step);

/* Element offset for a context that holds a slice of a larger parameter vector: params[j]
 * is element first_element + j of that vector (first_element >= 0, a multiple of 16, so
 * that slices keep whole 16-element sign groups).  Every sign the context generates
 * (zo_perturb, zo_perturb_range, zo_gemm_bf16_perturbed, zo_pack_probe, the quadratic
 * losses, zo_update, zo_step) is
 * then the sign of the global element index, so contexts with the same seed and step on
 * disjoint slices perturb and update exactly as one context on the whole vector would,
 * element by element; a separable loss (the diagonal quadratic) is the sum of the slices'
 * losses.  Default 0.  The MLP, low-rank and decoder entry points, whose losses are not sums
 * over parameter slices, return ZO_ERR_UNSUPPORTED while the offset is not 0.  Errors:
 * ZO_ERR_INVALID (negative or not a multiple of 16), ZO_ERR_STATE (perturbed). */
zo_status zo_set_element_offset(zo_ctx *ctx, int64_t first_element);

/* ------------------------------------------------------------------ tracing */

/* Phase timing of the step drivers (zo_quad_step, zo_mlp_step, zo_model_step): the next
 * n_steps driver calls record CUDA events on the context's stream at four points (step
 * start, after the clean loss, after the last perturbed loss, step end); n_steps = 0
 * disables recording.  At most 4096 steps.  Errors: ZO_ERR_INVALID, ZO_ERR_CUDA. */
zo_status zo_enable_phase_timing(zo_ctx *ctx, int32_t n_steps);

/* After the recorded steps, synchronise and write ms (host, n_steps x 3 floats):
 * per step the clean-loss, perturbed-losses and preconditioner+update times in
 * milliseconds.  Errors: ZO_ERR_INVALID (n_steps outside what was recorded). */
zo_status zo_phase_times(zo_ctx *ctx, int32_t n_steps, float *ms);

/* Per-class kernel timing, for measuring kernels inside a running step.  While enabled,
 * every launch of a timed class is bracketed by two CUDA events on the context's stream and
 * recorded with its algorithmic work: ZO_KT_GEMM (the tcgen05 projections; work = 2 M N K
 * flops, N counting both halves of a SwiGLU tile), ZO_KT_ATTENTION (causal attention; work =
 * 4 hd B H S (S + 1) / 2 flops: Q K^T and P V over the causal pairs), ZO_KT_PERTURB (the
 * unpack/apply kernel writing a perturbed window; work = 2 b count bytes: theta read, window
 * written) and ZO_KT_UPDATE (work = 2 b M bytes: theta read and written once); b is the bytes
 * per parameter.  The events cost a few microseconds per launch and break the programmatic
 * launch overlap of the update.  At most 65,536 launches are recorded between two
 * zo_kernel_times calls; later ones are counted as dropped.  Errors: ZO_ERR_INVALID. */
#define ZO_KT_GEMM 0
#define ZO_KT_ATTENTION 1
#define ZO_KT_PERTURB 2
#define ZO_KT_UPDATE 3
#define ZO_KT_COUNT 4

typedef struct {
  double ms;         /* summed launch durations, milliseconds */
  int64_t launches;  /* launches recorded */
  double work;       /* summed algorithmic flops (GEMM, attention) or bytes (perturb, update) */
} zo_kernel_time;

zo_status zo_enable_kernel_timing(zo_ctx *ctx, int enable);

/* Synchronise the context's stream, write the totals of the launches recorded since the
 * last call into out[ZO_KT_COUNT] (host), the number of launches not recorded into *dropped
 * (host, may be NULL), and start over.  Errors: ZO_ERR_INVALID (null out), ZO_ERR_CUDA. */
zo_status zo_kernel_times(zo_ctx *ctx, zo_kernel_time *out, int64_t *dropped);

/* Number of kernels this context has launched since it was created (every entry point that
 * enqueues work counts its launches; memory copies are not counted).  Errors: ZO_ERR_INVALID. */
zo_status zo_launch_count(zo_ctx *ctx, int64_t *count);

/* ------------------------------------------------------------------ zo_rng */

/* Write packed probe bytes [first_byte, first_byte + nbytes) of probe `probe` of step
 * `step` (any step: the probes are a pure function of (seed, step, probe, element), so no
 * state is read) into dev_out (device, nbytes bytes), 8 elements of the one probe per byte
 * (byte q: elements 8q..8q+7, bit t <-> element 8q+t).  Bits of
 * elements >= M are 0.  For tests and inspection: the training path regenerates probe
 * bits in registers and never stores them.
 * Errors: ZO_ERR_INVALID (probe < 0, range outside ceil(M/8) bytes, null dev_out). */
zo_status zo_pack_probe(zo_ctx *ctx, uint32_t step, int32_t probe, int64_t first_byte,
                        int64_t nbytes, uint8_t *dev_out);

/* ------------------------------------------------------------------ zo_perturb */

/* Enter the perturbed state theta + sign*eps*z_probe [HOW].  If the live buffer is
 * enabled this launches the fused unpack/apply kernel that writes all M perturbed
 * values into it; otherwise it only records (sign, eps, probe) for the loss kernels.
 *   sign  +1 or -1;  eps > 0 and finite;  probe >= 0.
 * Errors: ZO_ERR_INVALID, ZO_ERR_STATE (already perturbed), ZO_ERR_CUDA. */
zo_status zo_perturb(zo_ctx *ctx, int sign, float eps, int32_t probe);

/* Return to the clean state.  theta was never written, so this is exact and moves no
 * memory.  Errors: ZO_ERR_STATE (not perturbed). */
zo_status zo_restore(zo_ctx *ctx);

/* Materialise P = rd(theta + s*eps*z) (perturbed state) or theta (clean state) for
 * elements [first, first + count) into dev_out (device, count elements of the
 * context's dtype; 16-byte alignment and first % 8 == 0 give the vectorised path).
 * This is the per-window form of the unpack/apply kernel.
 * Errors: ZO_ERR_INVALID (range outside [0, M), null dev_out), ZO_ERR_CUDA. */
zo_status zo_perturb_range(zo_ctx *ctx, int64_t first, int64_t count, void *dev_out);

/* ------------------------------------------------------------------ losses (zo_forward) */

/* Diagonal quadratic L = 1/2 sum_j D_j P_j^2 at the current state, perturbation applied
 * on load (theta is read, never written), every term and sum in fp64, fixed reduction
 * order (deterministic).  Requires an ZO_F32 context.
 *   D         device, M floats.
 *   loss_out  device, one double: *loss_out = L, or += L when accumulate != 0.
 * Uses the context's reduction scratch; calls on one context must not overlap.
 * Errors: ZO_ERR_INVALID, ZO_ERR_UNSUPPORTED (bf16 context), ZO_ERR_CUDA. */
zo_status zo_quad_loss(zo_ctx *ctx, const float *D, double *loss_out, int accumulate);

/* Both losses of probe `probe`, L(theta + eps z) -> *loss_plus and L(theta - eps z) ->
 * *loss_minus (device doubles), from one pass over theta and D: the two perturbed vectors
 * share every load.  Each loss is the sum over all M elements of its own perturbed terms in
 * the same order as zo_quad_loss, so the results are bit-identical to perturb(+1) /
 * zo_quad_loss / restore / perturb(-1) / zo_quad_loss / restore.  Requires the clean state
 * (it does not change it); uses the current step counter.  The probe-parallel driver
 * evaluates probes this way.  Errors: as zo_quad_loss, ZO_ERR_STATE if perturbed. */
zo_status zo_quad_loss_pair(zo_ctx *ctx, const float *D, int32_t probe, float eps,
                            double *loss_plus, double *loss_minus);

/* The 2*count losses of the probes first_probe .. first_probe+count-1 (first_probe a
 * multiple of 8, count 1..64: the probes of up to eight octets; an octet's signs share one
 * generator block) from ONE pass over theta and D: L(theta + eps z_i) -> loss_plus[i - first_probe],
 * L(theta - eps z_i) -> loss_minus[i - first_probe] (device doubles).  Each element has
 * two perturbed values, rd(theta_j + eps) and rd(theta_j - eps), and each loss takes one of
 * them per element: L+_i is the fp64 sum of its M terms, and L-_i, which takes the other
 * term of every element, is formed as sum_j (t_a + t_b)_j - L+_i from one common sum.  The
 * results equal zo_quad_loss_pair's to fp64 rounding (not bit for bit: the grid and the
 * L- formula differ).  loss_clean (device double, or NULL) receives the clean loss L(theta)
 * from the same pass.  zo_quad_step evaluates its probes this way (and its clean loss in
 * the first pass).  Clean state required.  Errors: as zo_quad_loss_pair, ZO_ERR_INVALID for
 * a bad first_probe / count. */
zo_status zo_quad_loss_octet(zo_ctx *ctx, const float *D, int32_t first_probe, int32_t count,
                             float eps, double *loss_plus, double *loss_minus,
                             double *loss_clean);

/* Cross-entropy of an MLP classifier in -> hidden (ReLU) -> out evaluated at
 * zo_live_params(ctx) (fp32 CUDA-core arithmetic, no TF32), flat parameter order
 * W1[hidden][in], b1[hidden], W2[out][hidden], b2[out] (M must match).
 *   X        device, batch x n_in floats (row-major);  labels: device, batch int32 in
 *            [0, n_out).
 *   scale    multiplies the summed per-sample losses (1/batch gives the mean; 1/B_eff
 *            accumulates micro-batches into an effective-batch mean).
 *   loss_out device double: = scale*sum (accumulate == 0) or += scale*sum.
 * Requires a ZO_F32 context with the live buffer enabled when perturbed.
 * Limits: 1 <= n_in <= 1024, 1 <= n_hidden <= 1024, 1 <= n_out <= 1024, batch >= 1.
 * Errors: ZO_ERR_INVALID, ZO_ERR_STATE (perturbed without a live buffer),
 *         ZO_ERR_UNSUPPORTED, ZO_ERR_CUDA. */
zo_status zo_mlp_loss(zo_ctx *ctx, const float *X, const int32_t *labels, int batch,
                      int n_in, int n_hidden, int n_out, double scale, double *loss_out,
                      int accumulate);

/* Largest batch accepted by zo_mlp_loss_noalloc: its static scratch holds one fp64
 * partial per sample (32 KB) plus the reduction's ticket counter. */
#define ZO_NOALLOC_MAX_BATCH 4096

/* zo_mlp_loss without a context and without any device allocation.  The pages have no
 * counterpart: this entry point exists for callers that must not call cudaMalloc, e.g.
 * code running inside a host framework that owns every device allocation through its own
 * pool and memory budget.  Such callers pass inputs and
 * outputs only; the reduction scratch is a static device array of libzo.so, which every GPU
 * that loads the library holds (about 32 KB) until the process exits.
 *   P          device, M = n_hidden*n_in + n_hidden + n_out*n_hidden + n_out floats,
 *              flat order W1[hidden][in], b1[hidden], W2[out][hidden], b2[out] (the
 *              parameters to evaluate: theta, or a perturbed copy the caller made).
 *   X, labels, batch, n_in, n_hidden, n_out, scale, loss_out, accumulate: as zo_mlp_loss.
 *   stream     cudaStream_t to enqueue on (NULL = legacy default stream).
 * The first call on a device looks up the scratch array's device address (once per
 * device and CUDA context, with that device current).  The address is kept for the life of
 * the process: after cudaDeviceReset of a
 * device, whose context may come back with the same handle, the kept address is stale, so a
 * process that resets a device must not call this entry point on it again.
 * Every call clears the scratch's counter before its kernel.  All calls in the process
 * share the one scratch array, which keeps the last call's contents: calls that overlap
 * on the GPU (other streams, other threads) race and must be serialised by the caller.
 * Allocates nothing: no cudaMalloc, no cudaFree, no allocating library routine.
 * Errors (returned; there is no context to hold a message): ZO_ERR_INVALID for null
 * pointers, sizes outside the zo_mlp_loss limits, or batch > ZO_NOALLOC_MAX_BATCH;
 * ZO_ERR_CUDA if the scratch lookup, the counter reset or the launch fails. */
zo_status zo_mlp_loss_noalloc(const float *P, const float *X, const int32_t *labels,
                              int batch, int n_in, int n_hidden, int n_out, double scale,
                              double *loss_out, int accumulate, void *stream);

/* ------------------------------------------------------------------ zo_precond + zo_update */

/* One optimizer step from the losses of the current step [HOW][PSP]:
 *   loss_plus, loss_minus  device, n_pert doubles each (L(theta +- eps z_i));
 *   loss0                  device double (clean loss) for 1.5-SPSA, NULL for 1SPSA;
 *   lr, eps, damping       eps must be the one the losses were taken with.
 * Launches the probe-space preconditioner (one CTA, warp-shuffle reductions) and the
 * single-pass update that regenerates every probe in registers: theta is read once and
 * written once.  If any loss is not finite, theta and the step counter are left
 * unchanged and ZO_FLAG_NONFINITE is raised (seen by zo_sync); otherwise the step
 * counter advances by one.  No host synchronisation.
 * Errors: ZO_ERR_INVALID (n_pert outside [1, ZO_MAX_PROBES], eps <= 0, non-finite lr or
 *         damping < 0), ZO_ERR_STATE (perturbed), ZO_ERR_CUDA. */
zo_status zo_step(zo_ctx *ctx, const double *loss_plus, const double *loss_minus,
                  int32_t n_pert, const double *loss0, float lr, float eps, float damping);

/* Where zo_step reads its losses [LOOP: the losses feed the estimate wherever they were
 * produced]: on_device = 1 (the default) takes device pointers, which keeps a step free of
 * host synchronisation; on_device = 0 takes host pointers: zo_step copies the 2 n_pert (+1)
 * losses into the context's scratch on its stream and waits for the copies, so the host
 * arrays may be reused when it returns.  The step drivers always pass device losses and are
 * not affected.  Errors: ZO_ERR_INVALID (null context). */
zo_status zo_set_loss_location(zo_ctx *ctx, int on_device);

/* The update alone: theta <- rd(theta - sum_i coef_i z_i) with coef (device, n_pert
 * floats) at the current step, in the fixed fp32 order above.  Does not advance the
 * step counter.  Errors as zo_step. */
zo_status zo_update(zo_ctx *ctx, const float *coef, int32_t n_pert);

/* Copy the last zo_step's fp64 g_i, c_i, w_i (host arrays of n doubles each, any may be
 * NULL) and fp32 coefficients a_i (host, n floats, may be NULL).  Synchronises.
 * Errors: ZO_ERR_INVALID (n outside [1, last n_pert]). */
zo_status zo_get_precond(zo_ctx *ctx, int32_t n, double *g, double *c, double *w,
                         float *a);

/* ------------------------------------------------------------------ step driver */

/* One full step on the diagonal quadratic [LOOP]: the losses at +eps and -eps of up to 64
 * probes per pass over theta and D (perturbation on load: zo_quad_loss_octet), the clean
 * loss (1.5-SPSA) fused into the first pass, then zo_step.
 *   D           device, M floats;  losses_out device, 2*n_pert+1 doubles receiving
 *               [L0, L+_0..L+_{n-1}, L-_0..L-_{n-1}] (L0 = 0 for 1SPSA).
 *   preconditioned  1 = 1.5-SPSA, 0 = 1SPSA.
 * Errors: as zo_quad_loss and zo_step. */
zo_status zo_quad_step(zo_ctx *ctx, const float *D, int32_t n_pert, float eps, float lr,
                       float damping, int preconditioned, double *losses_out);

/* The same step with host buffers: copies D (host, M floats) to the device, runs the
 * step, and copies the 2*n_pert+1 losses back to losses_host (host).  Synchronises.
 * Device staging memory for D is owned by the context (allocated on first use). */
zo_status zo_quad_step_host(zo_ctx *ctx, const float *D_host, int32_t n_pert, float eps,
                            float lr, float damping, int preconditioned,
                            double *losses_host);

/* The same step without the final synchronisation, for pipelining: the copy of D (host,
 * M floats, pinned) runs on the context's own copy stream into one of two device staging
 * slots, so the next call's copy overlaps this step's kernels; the losses are copied back
 * to losses_host (pinned) on the context's stream.  D_host and losses_host must stay valid,
 * and losses_host unread, until the context's stream has been synchronised (zo_sync or the
 * caller's stream synchronisation).  Staging slots are owned by the context. */
zo_status zo_quad_step_host_async(zo_ctx *ctx, const float *D_host, int32_t n_pert, float eps,
                                  float lr, float damping, int preconditioned,
                                  double *losses_host);

/* Every loss of one MLP step from two launches: L(theta + eps z_i) -> loss_plus[i],
 * L(theta - eps z_i) -> loss_minus[i] for i < n_pert, and the clean loss L(theta) ->
 * *loss_clean unless it is NULL (device doubles; each = scale * sum of the batch's
 * per-sample losses).  Each evaluation's block stages rd(theta + s eps z_i) in shared memory
 * and runs zo_mlp_loss's per-sample arithmetic and batch sum in the same order, so every
 * value equals the corresponding zo_perturb / zo_mlp_loss / zo_restore result bit for bit.
 * Requires an fp32 context in the clean state with M = the MLP's parameter count and
 * M + n_hidden <= 49152 (the staged parameters, W1's rows padded by one); uses the current step counter.  X, labels, batch,
 * n_in, n_hidden, n_out as zo_mlp_loss; 1 <= n_pert <= ZO_MAX_PROBES, eps > 0.  Scratch of
 * (2 n_pert + 1) * batch doubles is owned by the context.  Errors: ZO_ERR_INVALID,
 * ZO_ERR_STATE, ZO_ERR_UNSUPPORTED (bf16 context or M above the limit), ZO_ERR_OOM,
 * ZO_ERR_CUDA. */
zo_status zo_mlp_losses(zo_ctx *ctx, const float *X, const int32_t *labels, int batch,
                        int n_in, int n_hidden, int n_out, int32_t n_pert, float eps,
                        double scale, double *loss_plus, double *loss_minus,
                        double *loss_clean);

/* One full MLP step [LOOP]: the clean loss (1.5-SPSA) and the 2*n_pert perturbed losses
 * (zo_mlp_losses when M + n_hidden <= 49152; otherwise one perturb / loss / restore per evaluation
 * through the live buffer, enabled by the call if needed), then zo_step.  Arguments as
 * zo_mlp_loss; losses_out as zo_quad_step. */
zo_status zo_mlp_step(zo_ctx *ctx, const float *X, const int32_t *labels, int batch,
                      int n_in, int n_hidden, int n_out, int32_t n_pert, float eps,
                      float lr, float damping, int preconditioned, double *losses_out);

/* ------------------------------------------------------------------ conditioning study */

/* The low-rank-plus-diagonal quadratic, a synthetic loss whose curvature differs from probe
 * to probe (on the diagonal quadratic every probe sees z^T D z = tr D, so 1.5-SPSA's
 * weights are all equal; "Stanford's 1.5-SPSA Trains OPT-30B Without Backpropagation",
 * section "Probe-Space Preconditioning", is about losses where they are not):
 *   L = 1/2 sum_j D_j P_j^2 + 1/2 sum_{k < rank} (lam[k] / M) (v_k . P)^2,
 * with v_k in {-1,+1}^M the generator's probe k at step 0 under seed vseed (so each adds
 * the eigenvalue lam[k] along v_k / sqrt(M)).  fp32 context, D device fp32 [M] 16-byte
 * aligned; every sum in fp64; the perturbation as in zo_quad_loss. */
typedef struct {
  int32_t rank;    /* 1..4 */
  float lam[4];    /* eigenvalue of each direction (entries past rank ignored) */
  uint64_t vseed;  /* seed of the directions */
} zo_lowrank;

/* L at the context's current state (clean or perturbed) into *loss_out (device fp64);
 * accumulate adds to it. */
zo_status zo_lowrank_loss(zo_ctx *ctx, const float *D, const zo_lowrank *q, double *loss_out,
                          int accumulate);

/* L(theta + eps z_probe) and L(theta - eps z_probe) from one pass (clean state only). */
zo_status zo_lowrank_loss_pair(zo_ctx *ctx, const float *D, const zo_lowrank *q, int32_t probe,
                               float eps, double *loss_plus, double *loss_minus);

/* One full step on this loss, as zo_quad_step. */
zo_status zo_lowrank_step(zo_ctx *ctx, const float *D, const zo_lowrank *q, int32_t n_pert,
                          float eps, float lr, float damping, int preconditioned,
                          double *losses_out);

/* ------------------------------------------------------------------ decoder (zo_forward) */

/* Two decoder families share this interface (cfg.family):
 * OPT (ZO_FAMILY_OPT), described next, and Qwen3 (ZO_FAMILY_QWEN3): pre-RMSNorm layers
 * (eps norm_eps), grouped-query attention (n_heads query heads of head_dim, n_kv_heads
 * key/value heads) with per-head RMSNorm on queries and keys followed by rotary embeddings
 * (rotate-half convention, base rope_theta), no projection biases, SwiGLU feed-forward
 * silu(x Wg^T) * (x Wu^T) Wd^T, final RMSNorm, head tied to the token embedding; the same
 * 2-class last-position loss.  Qwen3 flat parameter order (bf16; H, Hk, e = head_dim):
 *   E[V][d], then per layer: in_norm[d], Wqkv[(H+2Hk)e][d] (rows q, k, v), q_norm[e],
 *   k_norm[e], Wo[d][H e], post_norm[d], Wgu[2f][d] (rows gate, up), Wd[d][f];
 *   then final_norm[d]. */

/* Loss-only forward of an OPT-shaped decoder: pre-LN, learned positions (table of max_pos+2
 * rows, position s uses row s+2), ReLU FFN, biases on every projection, LayerNorm eps
 * 1e-5, final LayerNorm, head tied to the token embedding.  The loss is the 2-class
 * cross-entropy of the last position's logits restricted to class_ids[0..1] (label 0 or
 * 1 per sequence): the prompt-classification shape of the pages' fine-tuning benchmarks
 * ("Probe-Space Preconditioning for Fast and Stable Zero-Order Training", abstract:
 * OPT and Qwen3 post-training in inference mode).
 * Flat parameter order, all bf16 (d = d_model, f = d_ffn, V = vocab, P = max_pos + 2):
 *   E[V][d], Pos[P][d], then per layer: ln1.g[d], ln1.b[d], Wqkv[3d][d] (rows q, k, v),
 *   bqkv[3d], Wo[d][d], bo[d], ln2.g[d], ln2.b[d], W1[f][d], b1[f], W2[d][f], b2[d];
 *   then lnf.g[d], lnf.b[d].  Linear weights are [out][in] (row-major, in contiguous). */
/* Model families of zo_model_cfg.family. */
#define ZO_FAMILY_OPT 0
#define ZO_FAMILY_QWEN3 1

typedef struct {
  int32_t n_layers;
  int32_t d_model;      /* multiple of 64 */
  int32_t n_heads;      /* OPT: d_model / n_heads must be 64 or 128 */
  int32_t d_ffn;        /* multiple of 8 */
  int32_t vocab;
  int32_t max_pos;      /* longest sequence */
  int32_t class_ids[2]; /* token ids whose last-position logits are the two classes */
  int32_t family;       /* ZO_FAMILY_OPT or ZO_FAMILY_QWEN3 */
  int32_t n_kv_heads;   /* Qwen3: key/value heads, dividing n_heads (OPT: ignored) */
  int32_t head_dim;     /* Qwen3: 64 or 128 (OPT: ignored, d_model / n_heads) */
  float rope_theta;     /* Qwen3: rotary base (OPT: ignored) */
  float norm_eps;       /* Qwen3: RMSNorm epsilon (OPT: ignored, LayerNorm uses 1e-5) */
} zo_model_cfg;

typedef struct zo_model zo_model;

/* Number of parameters M of the layout above.  Errors: ZO_ERR_INVALID (bad config). */
zo_status zo_model_param_count(const zo_model_cfg *cfg, int64_t *M_out);

/* Bind a decoder to a bf16 context whose params hold the flat layout (ctx M must equal
 * zo_model_param_count).  Allocates, owned by the model: the layer window (one layer's
 * perturbed parameters) and activations for up to max_tokens = batch*seq tokens (fp32
 * residual stream [T][d], bf16 [T][d] x2, [T][3d], [T][f]).  The context must outlive
 * the model.  Errors: ZO_ERR_INVALID, ZO_ERR_OOM. */
zo_status zo_model_create(zo_model **out, zo_ctx *ctx, const zo_model_cfg *cfg,
                          int64_t max_tokens);
zo_status zo_model_destroy(zo_model *m);

/* Loss of one micro-batch at the context's current state (clean or perturbed):
 *   tokens  device int32 [batch][seq], ids in [0, vocab) (an id outside that range makes
 *           the loss NaN, so the step is skipped);  labels device int32 [batch] in {0, 1}.
 *   loss_out device double: = scale * sum of per-sequence losses (accumulate == 0) or +=.
 * With a perturbed context each layer's parameters are first materialised into the
 * layer window by the unpack/apply kernel (theta is not written); embeddings, the final
 * LayerNorm and the head rows are perturbed on load.
 * Errors: ZO_ERR_INVALID (seq > max_pos, batch*seq > max_tokens, batch > 4096, nulls),
 *         ZO_ERR_CUDA. */
zo_status zo_model_loss(zo_model *m, const int32_t *tokens, const int32_t *labels,
                        int32_t batch, int32_t seq, double scale, double *loss_out,
                        int accumulate);

/* Loss-only forwards (zo_model_loss, zo_model_step) run the last layer pruned to what the
 * loss reads: keys and values for every position, everything else (queries, attention,
 * output projection, feed-forward) for the last position of each sequence only.  On by
 * default; enabled = 0 runs the full last layer (for comparisons).  Batches above
 * min(max_tokens, 512) sequences and single-token sequences always run the full layer. */
zo_status zo_model_set_pruning(zo_model *m, int enabled);

/* Embedding plus the first n_layers_run layers of one micro-batch at the current state;
 * copies the fp32 residual stream [batch*seq][d_model] into h_out (device).  For
 * layer-by-layer parity checks. */
zo_status zo_model_hidden(zo_model *m, const int32_t *tokens, int32_t batch, int32_t seq,
                          int32_t n_layers_run, float *h_out);

/* One full step [LOOP][BUD]: the effective batch is n_micro micro-batches of
 * batch x seq (tokens device [n_micro][batch][seq], labels device [n_micro][batch]);
 * each loss is the mean over the effective batch, accumulated micro-batch by micro-batch.
 * Order: clean loss (1.5-SPSA), then for each probe the +eps and -eps losses, then
 * zo_step.  losses_out: device, 2*n_pert+1 doubles [L0, L+..., L-...]. */
zo_status zo_model_step(zo_model *m, const int32_t *tokens, const int32_t *labels,
                        int32_t batch, int32_t seq, int32_t n_micro, int32_t n_pert,
                        float eps, float lr, float damping, int preconditioned,
                        double *losses_out);

/* zo_model_step with host buffers: copies tokens_host [n_micro][batch][seq] and labels_host
 * [n_micro][batch] (host int32; pinned memory makes the copies asynchronous DMA) to device
 * staging owned by the model (allocated on first use, grown if a call needs more), runs
 * zo_model_step on them, copies the 2*n_pert+1 losses [L0, L+..., L-...] back to losses_host
 * (host doubles) and synchronises the context's stream.  Device flags (a skipped non-finite
 * step) are reported by the next zo_sync.  Errors: as zo_model_step, ZO_ERR_OOM. */
zo_status zo_model_step_host(zo_model *m, const int32_t *tokens_host, const int32_t *labels_host,
                             int32_t batch, int32_t seq, int32_t n_micro, int32_t n_pert,
                             float eps, float lr, float damping, int preconditioned,
                             double *losses_host);

/* ------------------------------------------------------------------ decoder components */

/* Epilogues of zo_gemm_bf16. */
#define ZO_EPI_BIAS_BF16 0  /* out bf16 = A.B^T + bias */
#define ZO_EPI_RELU_BF16 1  /* out bf16 = max(A.B^T + bias, 0) */
#define ZO_EPI_RESID_F32 2  /* out fp32 += A.B^T + bias (residual add) */
#define ZO_EPI_SWIGLU_BF16 3 /* out bf16 [M][N] = silu(A.Bg^T) * (A.Bu^T), B = [Bg; Bu] [2N][K],
                              * no bias (the Qwen3 gate and up projections in one GEMM) */

/* out[M][ldo] = epilogue(A[M][K] . B[N][K]^T + bias[N]) on the tcgen05 tensor cores:
 * bf16 operands (device, row-major, K contiguous), fp32 accumulation in TMEM, bias bf16
 * (device, may be NULL).  K % 8 == 0, ldo % 8 == 0, ldo >= N, all pointers 16-byte
 * aligned; ragged M, N, K are handled (zero fill).  With ZO_EPI_SWIGLU_BF16, B holds 2N
 * rows (gate rows, then up rows), N is the output width and bias must be NULL; the gate
 * and up products of a tile share one TMEM accumulator and are combined in fp32 before the
 * single bf16 rounding.  Enqueued on ctx's stream; a
 * pipeline stall beyond the bounded wait raises ZO_FLAG_TIMEOUT (seen by zo_sync). */
zo_status zo_gemm_bf16(zo_ctx *ctx, const void *A, const void *B, const void *bias, void *out,
                       int32_t M, int32_t N, int32_t K, int32_t ldo, int32_t epilogue);

/* zo_gemm_bf16 with B = the context's own bf16 parameters, read under its current
 * perturbation with the perturbation fused into the GEMM's operand path ("Probe-Space
 * Preconditioning for Fast and Stable Zero-Order Training", abstract: the probes are applied
 * by fused unpack/apply kernels; here the apply runs inside the GEMM instead of into a
 * window): B[n][k] = P at flat index w_offset + n K + k of the context, P = rd(theta + s eps
 * z_i) as zo_perturb set it (theta itself when the context is clean), computed per weight
 * tile in shared memory with no copy in HBM.  The product equals zo_gemm_bf16 on the
 * zo_perturb_range window of the same weights, element for element, when both use the same
 * single-CTA kernel form.  Every row tile of A regenerates the signs of the weight tiles it
 * reads (M / 128 times per weight).  ctx must be bf16 with first_element % 16 == 0;
 * w_offset % 16 == 0, K % 16 == 0, [w_offset, w_offset + N K) inside the context; epilogue
 * ZO_EPI_BIAS_BF16, ZO_EPI_RELU_BF16 or ZO_EPI_RESID_F32 (else ZO_ERR_UNSUPPORTED); A, bias,
 * out as zo_gemm_bf16.  Enqueued on ctx's stream; bounded waits as zo_gemm_bf16. */
zo_status zo_gemm_bf16_perturbed(zo_ctx *ctx, const void *A, int64_t w_offset, const void *bias,
                                 void *out, int32_t M, int32_t N, int32_t K, int32_t ldo,
                                 int32_t epilogue);

/* Test hook for the bounded waits of the tensor-core pipeline: runs zo_gemm_bf16 (no
 * bias, bf16 output) with the first stage's expected transaction count 16 bytes larger than
 * what its loads deliver, so that stage's barrier is never satisfied.  Every waiter gives
 * up after about 2 s, the kernel raises ZO_FLAG_TIMEOUT, lets its own loads land, waits for
 * issued MMAs, frees its TMEM and returns; out is left unspecified.  zo_sync then reports
 * ZO_ERR_TIMEOUT and the context remains usable.  No fault, trap or unbounded wait. */
zo_status zo_debug_gemm_timeout(zo_ctx *ctx, const void *A, const void *B, void *out, int32_t M,
                                int32_t N, int32_t K);

/* Causal multi-head attention: qkv device bf16 [batch*seq][3*d_model] (q, k, v at column
 * offsets 0, d, 2d; head h at +h*hd), out device bf16 [batch*seq][d_model];
 * softmax(q.k^T / sqrt(hd)) over keys <= query, hd = d_model/n_heads in {64, 128}.  Runs on
 * the tcgen05 tensor cores: fp32 scores, probabilities rounded to bf16 for P V, fp32
 * accumulation, one bf16 rounding of the output. */
zo_status zo_attention(zo_ctx *ctx, const void *qkv, void *out, int32_t batch, int32_t seq,
                       int32_t n_heads, int32_t d_model);

/* Grouped-query causal attention (the Qwen3 layer): qkv device bf16
 * [batch*seq][(n_heads + 2 n_kv_heads) head_dim] with the n_heads query heads first, then
 * the key heads, then the value heads; query head h reads key/value head
 * h / (n_heads / n_kv_heads).  out device bf16 [batch*seq][n_heads head_dim].
 * n_heads % n_kv_heads == 0, head_dim in {64, 128}, buffers 16-byte aligned. */
zo_status zo_attention_gqa(zo_ctx *ctx, const void *qkv, void *out, int32_t batch, int32_t seq,
                           int32_t n_heads, int32_t n_kv_heads, int32_t head_dim);

/* out bf16 [rows][d] = x / sqrt(mean(x^2) + eps) * w (x fp32 [rows][d], w bf16 [d]), the
 * Qwen3 RMSNorm; d <= 8192, d % 8 == 0, pointers 16-byte aligned. */
zo_status zo_rmsnorm(zo_ctx *ctx, const float *x, const void *w, void *out, int32_t rows,
                     int32_t d, float eps);

/* out bf16 [rows][d] = LayerNorm(x fp32 [rows][d]) * gamma + beta (bf16 [d]), eps 1e-5,
 * d <= 8192, d % 8 == 0, pointers 16-byte aligned. */
zo_status zo_layernorm(zo_ctx *ctx, const float *x, const void *gamma, const void *beta,
                       void *out, int32_t rows, int32_t d);

#ifdef __cplusplus
}
#endif

#endif /* ZO_H */
