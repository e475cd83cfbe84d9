/*
 * gptlayer.h — C ABI of the B200 (sm_100a) library for one GPT transformer
 * layer's training step with Megatron-style tensor parallelism on one GPU.
 *
 * What the step computes (sources are the Megatron-LM pages):
 *   - the GPT layer (pre-LayerNorm; QKV column split; causal attention with
 *     fused scale-mask-softmax; row-split output projection; column-split
 *     h->4h GEMM with fused bias+GeLU; row-split 4h->h GEMM):
 *     "Training GPT-2 with Megatron-LM" §4.1 (layer shapes) and §6.2
 *     (fused_softmax, fused_bias_gelu); "Megatron-LM 3D parallelism" §1
 *     (column split owns output columns, row split sums partial products);
 *     "Megatron-LM overview" §2.2 (FFN column split, QKV split by device);
 *   - mixed precision with FP32 master weights and dynamic loss scaling:
 *     "Megatron-LM overview" §3.1; Adam with lr 6e-5: same page, §4.2.
 *
 * The tp_size shards all live on the calling GPU.  The partial sums that a
 * multi-GPU run would all-reduce after each row-split GEMM (forward) and each
 * column-split input-gradient GEMM (backward) are summed inside the GEMM's
 * K loop here, so no collective exists on this path.
 *
 * Conventions shared by every entry point:
 *   - All device pointers are caller-owned CUDA device memory; the library
 *     allocates no device memory.  Every pointer must be 16-byte aligned.
 *   - All work is enqueued asynchronously on `stream`; no call synchronises
 *     the host with the device, except gptl_read_device_error().
 *   - Return value: 0 on success, a negative GPTL_E_* code otherwise.  Input
 *     validation happens before any launch: on error nothing is enqueued.
 *   - Kernels never trap.  A device-side failure (a bounded wait that timed
 *     out, an internal consistency check) sets a library-wide device error
 *     word, read with gptl_read_device_error().
 *   - Activations are row-major [T, h] with token row r = j*seq + p (batch j,
 *     position p), T = batch*seq.  Weights are [out][in] row-major, stored
 *     shard-major (layouts below).
 */
#ifndef GPTLAYER_H
#define GPTLAYER_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

struct CUstream_st;
typedef struct CUstream_st *gptl_stream_t;   /* same type as cudaStream_t */

enum {
  GPTL_OK = 0,
  GPTL_E_NULL = -1,    /* a required pointer is NULL                         */
  GPTL_E_SHAPE = -2,   /* unsupported or inconsistent sizes                  */
  GPTL_E_ALIGN = -3,   /* a pointer is not 16-byte aligned                   */
  GPTL_E_DTYPE = -4,   /* dtype is neither GPTL_FP16 nor GPTL_BF16           */
  GPTL_E_ARCH = -5,    /* the current device is not compute capability 10.x  */
  GPTL_E_CUDA = -6,    /* a CUDA runtime/driver call or a launch failed      */
  GPTL_E_DEVICE = -7,  /* the device error word is set (see below)           */
  GPTL_E_ARG = -8,     /* an invalid scalar argument (hyper-parameter)       */
  GPTL_E_TOO_LARGE = -9 /* the sizes exceed a fixed internal capacity         */
};

typedef enum { GPTL_FP16 = 0, GPTL_BF16 = 1 } gptl_dtype;

/* Sizes of one layer.  Requirements (GPTL_E_SHAPE otherwise): every field
 * > 0; heads | hidden; tp | heads; tp | ffn; head_dim = hidden/heads is a
 * multiple of 16 and at most 256; hidden % 64 == 0; (ffn/tp) % 64 == 0;
 * seq % 16 == 0; batch*seq < 2^31.  ln_eps > 0 (the pages do not state it;
 * 1e-5 is the usual GPT-2 value).
 * recompute_gelu (0 or 1): selective recompute of the FFN activation
 * ("Training GPT-2 with Megatron-LM", troubleshooting: activation
 * recomputation; "Megatron-LM overview" §3.3).  With 1, A = GeLU(Z) is not
 * kept in the saved workspace (batch*seq*ffn*2 bytes less): the forward writes
 * it into scratch for FFN2, and the backward writes it again from the saved Z
 * in the epilogue of the FFN2 input-gradient GEMM, which reads Z anyway.
 * The results are bit-identical to recompute_gelu = 0. */
typedef struct {
  int batch, seq, hidden, heads, ffn, tp;
  gptl_dtype dtype;
  float ln_eps;
  int recompute_gelu;
} gptl_shape;

/* Layer parameters in the compute dtype (fp16 or bf16), read-only here.
 * Column-split tensors: shard i owns output rows; row-split tensors: shard
 * i owns input columns ("Megatron-LM 3D parallelism" §1).
 *   ln1_g, ln1_b, ln2_g, ln2_b : [h]
 *   w_qkv : [t][3h/t][h]  rows of shard i = [Q_i; K_i; V_i], Q_i the rows of
 *           heads i*a/t .. (i+1)*a/t-1, head-major, head_dim rows each
 *   b_qkv : [t][3h/t]
 *   w_o   : [t][h][h/t]   b_o : [h]   (added once, after the shard sum)
 *   w_1   : [t][f/t][h]   b_1 : [t][f/t]
 *   w_2   : [t][h][f/t]   b_2 : [h]   (added once, after the shard sum)   */
typedef struct {
  const void *ln1_g, *ln1_b;
  const void *w_qkv, *b_qkv;
  const void *w_o, *b_o;
  const void *ln2_g, *ln2_b;
  const void *w_1, *b_1;
  const void *w_2, *b_2;
  /* Optional (all four or none): the four weight matrices transposed shard
   * by shard, as gpt_layer_adam_step and gpt_layer_transpose_weights write
   * them: w_qkv_t [t][h][3h/t], w_o_t [t][h/t][h], w_1_t [t][h][f/t],
   * w_2_t [t][f/t][h].  The backward's input-gradient products read these;
   * when they are NULL the backward transposes the weights itself into its
   * scratch.  The forward ignores them. */
  const void *w_qkv_t, *w_o_t, *w_1_t, *w_2_t;
} gptl_weights;

/* FP32 gradients, same layouts as gptl_weights, multiplied by the loss scale
 * (they are the gradients of the scaled loss).  gpt_layer_bwd OVERWRITES
 * them.  Normally these point into the flat gradient arena that
 * adam_step_fp32_master consumes (see gpt_layer_param_layout); to accumulate
 * over micro-batches, write each into a second arena and add it with
 * gptl_grad_accumulate. */
typedef struct {
  float *ln1_g, *ln1_b, *w_qkv, *b_qkv, *w_o, *b_o,
        *ln2_g, *ln2_b, *w_1, *b_1, *w_2, *b_2;
} gptl_grads;

/* Dynamic loss-scale state, in DEVICE memory, caller-initialised to
 * {scale = initial scale (65536), growth_tracker = 0, found_inf = 0,
 *  step = 0, error = 0}. */
typedef struct {
  float scale;          /* current loss scale S                              */
  int growth_tracker;   /* clean steps since the last scale change           */
  int found_inf;        /* written by adam_step_fp32_master (or by           */
                        /* gpt_layer_bwd_checked)                            */
  int step;             /* Adam steps taken (skipped steps not counted)      */
  int error;            /* reserved; 0                                       */
} gptl_scaler_state;

/* Bytes of device workspace the caller provides.
 *  saved   : activations written by gpt_layer_fwd and read by gpt_layer_bwd;
 *            must stay untouched between the two calls.
 *  scratch : temporaries of gpt_layer_bwd (and, with recompute_gelu, of
 *            gpt_layer_fwd); may be reused freely between calls on the same
 *            stream.
 * Returns GPTL_E_NULL / GPTL_E_SHAPE / GPTL_E_DTYPE on bad arguments. */
int gpt_layer_workspace_bytes(const gptl_shape *shape, size_t *saved_bytes,
                              size_t *scratch_bytes);

/* Offsets (in elements) of the 12 parameter tensors inside one flat arena, in
 * the order ln1_g, ln1_b, w_qkv, b_qkv, w_o, b_o, ln2_g, ln2_b, w_1, b_1, w_2,
 * b_2, each 64-element aligned, and the arena length n_params (a multiple of
 * 64).  The same offsets index the fp32 master / m / v / grad arenas and the
 * 16-bit weight arena.  Padding elements must be zero in the grad arena (the
 * overflow check scans the whole arena). */
int gpt_layer_param_layout(const gptl_shape *shape, size_t offsets[12], size_t *n_params);

/* Forward pass.  x: [T,h] input; y: [T,h] output (cdt).  saved: workspace of
 * saved_bytes; scratch: scratch_bytes of workspace with recompute_gelu (else
 * unused, may be NULL).  x, y, saved and scratch must not overlap. */
int gpt_layer_fwd(const gptl_shape *shape, const gptl_weights *w, const void *x, void *y,
                  void *saved, void *scratch, gptl_stream_t stream);

/* Backward pass.  dy: [T,h] gradient of the scaled loss w.r.t. y (cdt);
 * dx: [T,h] output (cdt); g: fp32 gradients, overwritten; saved: as written
 * by the matching gpt_layer_fwd; scratch: scratch_bytes of workspace. */
int gpt_layer_bwd(const gptl_shape *shape, const gptl_weights *w, const void *x,
                  const void *saved, const void *dy, void *dx, const gptl_grads *g,
                  void *scratch, gptl_stream_t stream);

/* Overflow check + fused unscale/Adam/cast over flat arenas of n_params
 * elements ("Megatron-LM overview" §3.1 and §4.2).
 *   1. st->found_inf <- 1 if any grad element is inf or NaN, else 0;
 *   2. if !found_inf, per element with t = st->step + 1 and S = st->scale:
 *        g = grad/S; m = b1*m + (1-b1)*g; v = b2*v + (1-b2)*g*g;
 *        p -= lr*( (m/(1-b1^t)) / (sqrt(v/(1-b2^t)) + eps) + wd*p );
 *        w16 = round-to-nearest-even(p) in dtype;
 *      if found_inf, master, m, v and w16 are left bit-unchanged.
 * master/m/v: [n] fp32 in/out; grad: [n] fp32 in; w16: [n] fp16/bf16 out.
 * Decisions are made on the device; st is read and written there.
 * GPTL_E_ARG if lr < 0, beta not in [0,1), eps < 0 or n_params % 4 != 0. */
int adam_step_fp32_master(size_t n_params, float *master, float *m, float *v,
                          const float *grad, void *w16, gptl_dtype dtype, float lr,
                          float beta1, float beta2, float eps, float weight_decay,
                          gptl_scaler_state *st, gptl_stream_t stream);

/* The step's overflow check folded into the backward ("Megatron-LM
 * overview" §3.1, dynamic loss scaling; the fused kernels of "Training GPT-2
 * with Megatron-LM" §6.2 taken to the optimizer side).  gpt_layer_bwd_checked
 * is gpt_layer_bwd that also sets st->found_inf (DEVICE) to 1 if any
 * gradient value it writes is inf or NaN, else 0: the kernels that write the
 * 12 gradients (the fp32 weight-gradient GEMMs' epilogues or their split-K
 * sums, and the column-sum reductions of the biases and LayerNorm
 * parameters) each test the values they store, so no pass re-reads the
 * arena.  adam_step_fp32_master_prechecked is adam_step_fp32_master without
 * step 1: it takes st->found_inf as it stands.  Used as a pair, with the
 * gradient arena holding exactly what gpt_layer_bwd_checked wrote and zero
 * padding, they make the same decision, bit for bit, as
 * gpt_layer_bwd + adam_step_fp32_master, at 4 bytes per parameter less HBM
 * traffic.  If anything else writes the arena in between (accumulation,
 * an injected value), use adam_step_fp32_master, which scans it.
 * Arguments and errors as gpt_layer_bwd / adam_step_fp32_master; also
 * GPTL_E_NULL if st is NULL and GPTL_E_ALIGN if it is not 4-byte aligned. */
int gpt_layer_bwd_checked(const gptl_shape *shape, const gptl_weights *w, const void *x,
                          const void *saved, const void *dy, void *dx, const gptl_grads *g,
                          void *scratch, gptl_scaler_state *st, gptl_stream_t stream);
int adam_step_fp32_master_prechecked(size_t n_params, float *master, float *m, float *v,
                                     const float *grad, void *w16, gptl_dtype dtype, float lr,
                                     float beta1, float beta2, float eps, float weight_decay,
                                     gptl_scaler_state *st, gptl_stream_t stream);

/* Dynamic loss-scale update (one device thread), after adam_step_fp32_master:
 *   found_inf: scale = max(scale*backoff_factor, min_scale); tracker = 0;
 *   else: tracker += 1; if tracker == growth_interval: scale *= growth_factor,
 *         tracker = 0; step += 1.
 * GPTL_E_ARG if growth_interval < 1, growth_factor < 1, backoff_factor not in
 * (0,1] or min_scale <= 0. */
int loss_scale_update(gptl_scaler_state *st, int growth_interval, float growth_factor,
                      float backoff_factor, float min_scale, gptl_stream_t stream);

/* Stacks of n_layers layers of one shape ("Training GPT-2 with Megatron-LM"
 * §4.1: --num-layers 32).  Layer l has its own weights w[l] and gradients
 * g[l] (normally layer l's block of one arena holding every layer's
 * parameters back to back, n_params of gpt_layer_param_layout apart, which
 * one adam_step_fp32_master call over n_layers * n_params then updates).
 *  saved_bytes  : n_layers per-layer saved workspaces (256-byte multiples);
 *  scratch_bytes: the layer scratch plus two [T,h] buffers for the input
 *                 gradients handed between layers.
 * GPTL_E_ARG if n_layers < 1; otherwise as gpt_layer_workspace_bytes. */
int gpt_stack_workspace_bytes(const gptl_shape *shape, int n_layers, size_t *saved_bytes,
                              size_t *scratch_bytes);

/* Forward through layers 0..n_layers-1: layer 0 reads x, layer l > 0 reads
 * layer l-1's output.  acts: n_layers [T,h] outputs (cdt) back to back,
 * layer l's at acts + l*T*h elements; the stack's output is the last one.
 * w: n_layers gptl_weights; saved: gpt_stack_workspace_bytes' saved bytes,
 * untouched until gpt_stack_bwd; scratch: its scratch bytes when the shape
 * has recompute_gelu (else may be NULL).  x, acts, saved and scratch must not
 * overlap.  All arguments are checked before the first launch. */
int gpt_stack_fwd(const gptl_shape *shape, int n_layers, const gptl_weights *w, const void *x,
                  void *acts, void *saved, void *scratch, gptl_stream_t stream);

/* Backward through layers n_layers-1..0: the last layer reads dy (gradient
 * of the scaled loss w.r.t. the stack's output), layer l < n_layers-1 reads
 * layer l+1's input gradient, and layer 0 writes dx.  x, acts and saved as
 * passed to / written by gpt_stack_fwd; g: n_layers gptl_grads, each
 * OVERWRITTEN; scratch: gpt_stack_workspace_bytes' scratch bytes.  All
 * arguments are checked before the first launch. */
int gpt_stack_bwd(const gptl_shape *shape, int n_layers, const gptl_weights *w, const void *x,
                  const void *acts, const void *saved, const void *dy, void *dx,
                  const gptl_grads *g, void *scratch, gptl_stream_t stream);

/* The optimizer step for n_layers layers of one shape whose parameters lie
 * back to back in one arena (n_layers * n_params elements, n_params and the
 * offsets of gpt_layer_param_layout), that also writes the transposed 16-bit
 * copy of every layer's four weight matrices into w16t: for the matrix at
 * offset o of the layout, shard i ([rows][cols] at o + i*rows*cols) goes
 * transposed to w16t + o + i*rows*cols as [cols][rows].  Elements of w16t
 * outside the four matrices are not written.  Point gptl_weights' *_t
 * fields of layer l at w16t + l*n_params + o, and the next backward reads
 * these copies instead of transposing the weights (at h = 10240, t = 4 that
 * is 2.5 GB per step written here instead of 5 GB moved there).
 *   prechecked = 0: overflow check of grad first, as adam_step_fp32_master;
 *   prechecked = 1: the flag gpt_layer_bwd_checked left in st->found_inf, as
 *                   adam_step_fp32_master_prechecked.
 * master, m, v, w16 and w16t are updated exactly as adam_step_fp32_master
 * updates master, m, v and w16 (the same arithmetic, bit for bit); on a
 * skipped step nothing is written.  w16t must not overlap the other arrays.
 * Errors as gpt_layer_workspace_bytes and adam_step_fp32_master, and
 * GPTL_E_ARG if n_layers < 1 or prechecked is not 0 or 1. */
int gpt_layer_adam_step(const gptl_shape *shape, int n_layers, float *master, float *m, float *v,
                        const float *grad, void *w16, void *w16t, float lr, float beta1,
                        float beta2, float eps, float weight_decay, int prechecked,
                        gptl_scaler_state *st, gptl_stream_t stream);

/* The transposed copies alone, from the 16-bit weights w16 (n_layers arenas
 * as above) into w16t: for the first backward, or after the weights were
 * changed by anything other than gpt_layer_adam_step. */
int gpt_layer_transpose_weights(const gptl_shape *shape, int n_layers, const void *w16, void *w16t,
                                gptl_stream_t stream);

/* Bytes of device workspace adam_step_fp32_master_clip takes (clip_ws). */
#define GPTL_CLIP_WORKSPACE_BYTES 16384

/* adam_step_fp32_master with gradient clipping by global norm ("Training
 * GPT-2 with Megatron-LM", troubleshooting: --clip-grad 1.0 against NaN
 * losses; "Megatron-LM overview" §5.1: too strong a clip slows convergence).
 *   1. one pass over grad: st->found_inf as in adam_step_fp32_master, and
 *      float64 partial sums of grad^2 (fixed order, so the result is
 *      bit-reproducible on a given GPU);
 *   2. with S = st->scale, into clip_ws:
 *        float at byte 0: norm = sqrt(sum_i (grad_i / S)^2), the L2 norm of
 *                         the unscaled gradient over the whole arena;
 *        float at byte 4: coef = max_norm / (norm + 1e-6) if that is < 1,
 *                         else exactly 1;
 *   3. if !found_inf: the Adam update of adam_step_fp32_master with the
 *      unscaled gradient taken as grad / (S / coef), i.e. (grad / S) * coef
 *      up to one fp32 rounding; with coef == 1 the update is bit-identical
 *      to adam_step_fp32_master's.
 * clip_ws: GPTL_CLIP_WORKSPACE_BYTES of DEVICE memory, 16-byte aligned, owned
 * by the caller, overlapping none of the arenas or st; norm and coef stay
 * there after the call (read them after the stream has reached this point).
 * Calls that share one clip_ws must be ordered on the device.  On overflow the step is skipped as in
 * adam_step_fp32_master, and norm / coef are whatever the inf or NaN give.
 * Other arguments and errors as adam_step_fp32_master; also GPTL_E_NULL if
 * clip_ws is NULL, GPTL_E_ALIGN if it is not 16-byte aligned, GPTL_E_ARG if
 * max_norm is not a finite positive number. */
int adam_step_fp32_master_clip(size_t n_params, float *master, float *m, float *v,
                               const float *grad, void *w16, gptl_dtype dtype, float lr,
                               float beta1, float beta2, float eps, float weight_decay,
                               float max_norm, void *clip_ws, gptl_scaler_state *st,
                               gptl_stream_t stream);

/* Gradient accumulation over micro-batches ("Training GPT-2 with
 * Megatron-LM" §4.3, --gradient-accumulation-steps): acc[i] += grad[i] for
 * i < n, in fp32 with one rounding per element.  Typical use: gpt_layer_bwd
 * writes each micro-batch's gradients into a second arena, which is added to
 * the accumulating arena; the sum is the gradient of the summed loss (scale
 * dOut by 1/micro-batches for the mean).  acc, grad: DEVICE, 16-byte
 * aligned, not overlapping.  GPTL_E_NULL / GPTL_E_ALIGN; GPTL_E_ARG if n is
 * 0 or not a multiple of 4, or the ranges overlap. */
int gptl_grad_accumulate(size_t n, float *acc, const float *grad, gptl_stream_t stream);

/* Standalone overflow check (step 1 of adam_step_fp32_master). */
int gptl_check_overflow(size_t n, const float *grad, gptl_scaler_state *st,
                        gptl_stream_t stream);

/* Human-readable text of a GPTL_E_* code (static storage). */
const char *gptl_strerror(int code);

/* Synchronises the current device, then reads (and with clear != 0 resets)
 * the library's device error word: 0 = no device-side error; otherwise a
 * bit mask (1 = a pipeline wait timed out in a GEMM, 2 = an internal index
 * check failed).  Test helper; returns GPTL_E_CUDA if the copy fails. */
int gptl_read_device_error(int *word, int clear);

#ifdef __cplusplus
}
#endif
#endif /* GPTLAYER_H */
