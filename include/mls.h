/*
 * mls.h -- C ABI of libmls: the Matryoshka LM-suite junction and the
 * multi-exit LM-head loss with online distillation, on NVIDIA B200 (sm_100a).
 *
 * The method ("Matryoshka Language Model Suites", Godey & Artzi, 2026) stacks
 * M blocks of strictly increasing width D_1 < ... < D_M.  Block m+1's input is
 * the junction of block m's output with a fresh residual embedding, and every
 * block ends in an exit with its own LM head.  This library implements the
 * data-parallel hot path of one training step on those pieces:
 *
 *   mls_junction_fwd / mls_junction_bwd       -- the parameter-free junction
 *   mls_multiexit_loss_fwd / _bwd             -- per-exit logits, next-token CE,
 *                                                distillation from the largest
 *                                                exit, and their gradients
 *
 * Conventions shared by every entry point
 *   - All tensors are row-major with tokens outermost, on the current CUDA
 *     device, and owned by the caller.  The library keeps no pointer after a
 *     call returns and allocates no device memory: scratch space is a caller
 *     buffer sized by the matching *_workspace query.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  Every call is
 *     asynchronous on that stream; results are valid once the stream has
 *     reached the end of the call.
 *   - Argument errors (NULL pointers, non-positive sizes, widths that do not
 *     increase, unsupported shapes or dtypes, misaligned pointers, workspace
 *     too small) are reported synchronously and nothing is launched.
 *   - Data errors found on the device (a token id or target outside [0, V))
 *     never cause an out-of-range access: the affected token's outputs are
 *     written as zeros and bit MLS_DEVFLAG_BAD_ID is OR-ed into *dev_status.
 *     A device-side wait that runs past its limit sets MLS_DEVFLAG_TIMEOUT and
 *     the kernel returns.  `dev_status` may be NULL (then nothing is recorded);
 *     mls_status_read() collects it.
 *   - Dtypes: MLS_F32 or MLS_BF16 inputs; accumulation is always fp32.
 *   - Reentrant: no global mutable state besides one-time kernel attributes.
 */
#ifndef MLS_H_
#define MLS_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MLS_OK = 0,
  MLS_ERR_INVALID_ARG = 1,     /* NULL pointer, size <= 0, widths not increasing   */
  MLS_ERR_UNSUPPORTED = 2,     /* shape/dtype/alignment outside the supported set */
  MLS_ERR_WORKSPACE = 3,       /* workspace NULL or smaller than the query result */
  MLS_ERR_CUDA = 4,            /* a CUDA runtime call or launch failed            */
  MLS_ERR_BAD_ID = 5,          /* reported by mls_status_read: id/target not in [0,V) */
  MLS_ERR_DEVICE_TIMEOUT = 6,  /* reported by mls_status_read: a device wait gave up */
  MLS_ERR_NO_DEVICE = 7        /* no sm_100 device is current                       */
} mls_status;

typedef enum { MLS_F32 = 0, MLS_BF16 = 1 } mls_dtype;

/* Bits of the device status word. */
#define MLS_DEVFLAG_BAD_ID  1
#define MLS_DEVFLAG_TIMEOUT 2

/* ------------------------------------------------------------------------ */
/* Junction                                                                  */
/* ------------------------------------------------------------------------ */

/*
 * mls_junction_fwd -- block m output -> block m+1 input.
 *
 * Defined by "Visualizing the core idea of Matryoshka LM Suites" (How to read
 * it, bottom panel: the junction) and "Matryoshka Language Model Suites"
 * (agihunt.info summary, junction paragraph): the block output is rescaled to
 * the L2 norm of the fresh residual embedding of the same token and the two
 * are concatenated along channels; the junction has no parameters.  The
 * residual table e_{m+1} has width delta = D_{m+1} - D_m and is indexed by the
 * original token ids ("Editing the methods of sub-models are made of blocks",
 * Modeling paragraph, after version).
 *
 * For every token t:
 *   s_t = ||e_next[x_t]||_2 / max(||o_m[t]||_2, 1e-12)           (fp32)
 *   y[t, 0:D_m]          = s_t * o_m[t]        (rounded to dt, nearest-even)
 *   y[t, D_m:D_m+delta]  = e_next[x_t]         (bit-exact copy)
 *
 *   x         device int32 [T]           token ids, each in [0, V)
 *   o_m       device dt [T, D_m]          block-m output
 *   e_next    device dt [V, delta]        residual table of block m+1
 *   y         device dt [T, D_m+delta]    output (must not alias the inputs)
 *   scale_out device f32 [T] or NULL      s_t
 *   Supported: D_m and delta multiples of 8 (bf16) or 4 (f32); every pointer
 *   16-byte aligned.  Otherwise MLS_ERR_UNSUPPORTED.
 */
mls_status mls_junction_fwd(const int32_t* x, int64_t T,
                            const void* o_m, int64_t D_m,
                            const void* e_next, int64_t V, int64_t delta,
                            void* y, float* scale_out,
                            mls_dtype dt, int32_t* dev_status, void* stream);

/*
 * mls_junction_bwd -- gradients of mls_junction_fwd (derived from its
 * definition; the pages give no gradient).  With u = o/||o||, e_hat = e/||e||
 * (e_hat = 0 when ||e|| = 0), s as above and dy = [g_o ; g_e]:
 *   do_m[t]    = s_t (g_o - u (u . g_o))
 *   de_rows[t] = g_e + (u . g_o) e_hat
 *   dE_table[v] (+)= sum over t with x_t = v of de_rows[t], summed in
 *                    ascending t (deterministic; no floating-point atomics)
 *
 *   dy        device dt [T, D_m+delta]    gradient w.r.t. y
 *   do_m      device dt [T, D_m]          output
 *   de_rows   device dt [T, delta] or NULL
 *   dE_table  device f32 [V, delta] or NULL;  accumulate_dE != 0 adds into it,
 *             0 overwrites every row (rows of unused ids become 0)
 *   workspace device, >= mls_junction_bwd_workspace(T, V) bytes when dE_table
 *             is non-NULL (may be NULL otherwise)
 * Supported shapes as for the forward pass.
 */
mls_status mls_junction_bwd(const int32_t* x, int64_t T,
                            const void* o_m, int64_t D_m,
                            const void* e_next, int64_t V, int64_t delta,
                            const void* dy, void* do_m, void* de_rows,
                            float* dE_table, int accumulate_dE,
                            void* workspace, size_t ws_bytes,
                            mls_dtype dt, int32_t* dev_status, void* stream);

/*
 * Junction variants (bit flags, combinable) for the ablations the pages
 * report: "Visualizing Core ideas", bullet (c) -- dropping the rescaling, and
 * filling the new channels with zeros instead of the fresh embedding -- and
 * "Is nesting the cheapest way to build a model suite?", section 5 (B) --
 * stop-gradient at every junction, so each block learns only from its own exit.
 *   MLS_JUNCTION_NO_RESCALE  s_t := 1:            y = [o ; e],   do = g_o, de = g_e
 *   MLS_JUNCTION_ZERO_FILL   new channels zero:   y = [s o ; 0], de = (u . g_o) e_hat
 *                            (the rescale still uses the fresh embedding's norm)
 *   MLS_JUNCTION_STOP_GRAD   forward unchanged;   do = 0, de as for the variant without it
 * Unknown bits return MLS_ERR_INVALID_ARG.  The _variant entry points take the
 * same arguments as mls_junction_fwd / mls_junction_bwd plus `variant`;
 * variant 0 is exactly the standard junction.
 */
typedef enum {
  MLS_JUNCTION_STANDARD = 0,
  MLS_JUNCTION_NO_RESCALE = 1,
  MLS_JUNCTION_ZERO_FILL = 2,
  MLS_JUNCTION_STOP_GRAD = 4
} mls_junction_variant;

mls_status mls_junction_fwd_variant(const int32_t* x, int64_t T,
                                    const void* o_m, int64_t D_m,
                                    const void* e_next, int64_t V, int64_t delta,
                                    void* y, float* scale_out, uint32_t variant,
                                    mls_dtype dt, int32_t* dev_status, void* stream);

mls_status mls_junction_bwd_variant(const int32_t* x, int64_t T,
                                    const void* o_m, int64_t D_m,
                                    const void* e_next, int64_t V, int64_t delta,
                                    const void* dy, void* do_m, void* de_rows,
                                    float* dE_table, int accumulate_dE,
                                    void* workspace, size_t ws_bytes, uint32_t variant,
                                    mls_dtype dt, int32_t* dev_status, void* stream);

/* Scratch bytes mls_junction_bwd needs for the dE_table scatter. */
mls_status mls_junction_bwd_workspace(int64_t T, int64_t V, size_t* bytes);

/*
 * Every junction of a suite in one call: J junctions (1 <= J <= 3) that share
 * the token ids x, T and V, with widths D (HOST int64 [J+1], strictly
 * increasing).  Junction k maps o[k] (dt [T, D[k]]) and e_next[k]
 * (dt [V, D[k+1] - D[k]]) to y[k] (dt [T, D[k+1]]), exactly as
 * mls_junction_fwd; the arrays o, e_next, y and scale_out are HOST arrays of
 * J device pointers (scale_out may be NULL, or hold NULL entries).  In a
 * training step the junctions' inputs come from different blocks, so this
 * call fits where all of them are at hand (recomputation, the benchmark's
 * hot-path step); the results equal J separate calls.  MLS_BF16 runs every
 * junction in one launch whose blocks are divided among the junctions.
 * Standard junction only (no variant bits).
 */
mls_status mls_junction_fwd_multi(const int32_t* x, int64_t T, int64_t V, int J, const int64_t* D,
                                  const void* const* o, const void* const* e_next,
                                  void* const* y, float* const* scale_out,
                                  mls_dtype dt, int32_t* dev_status, void* stream);

/*
 * The backward pass of mls_junction_fwd_multi: results equal J calls of
 * mls_junction_bwd with the same accumulate_dE.  dy, do_m: HOST arrays of J
 * device pointers; de_rows and dE_table: HOST arrays of J device pointers
 * (NULL entries allowed) or NULL.  The tokens are grouped by id once for all
 * table gradients.  workspace >= mls_junction_bwd_multi_workspace(T, V, J)
 * when any dE_table entry is non-NULL.
 */
mls_status mls_junction_bwd_multi_workspace(int64_t T, int64_t V, int J, size_t* bytes);

mls_status mls_junction_bwd_multi(const int32_t* x, int64_t T, int64_t V, int J, const int64_t* D,
                                  const void* const* o, const void* const* e_next,
                                  const void* const* dy, void* const* do_m, void* const* de_rows,
                                  float* const* dE_table, int accumulate_dE,
                                  void* workspace, size_t ws_bytes,
                                  mls_dtype dt, int32_t* dev_status, void* stream);

/*
 * mls_junction_bwd_noalloc -- mls_junction_bwd without a workspace argument.
 * The paper has no counterpart: this is a convenience of this library.
 *
 * For callers that cannot allocate device memory where they call the junction
 * backward pass: programs whose device memory is all handed out up front by
 * another allocator (a framework's caching allocator, a fixed pool), and
 * latency-critical code that must not call cudaMalloc/cudaFree, which can
 * synchronise the whole device.  The table-gradient scratch comes from a
 * fixed 4 MiB array in the library's own device memory, held by every GPU
 * that loads the library until the process exits; nothing is allocated.
 *
 * Arguments, results and errors are those of mls_junction_bwd, checked in the
 * same order.  Additionally:
 *   - with dE_table non-NULL, (T, V) must satisfy
 *     mls_junction_bwd_workspace(T, V) <= 4 MiB (for example T <= 65536 with
 *     V <= 262144); larger sizes return MLS_ERR_UNSUPPORTED (after the
 *     argument checks) and launch nothing;
 *   - every call on a device shares the one array and leaves its contents
 *     behind (each call re-initialises what it reads): calls whose work
 *     overlaps on the GPU (different streams, or different host threads,
 *     without ordering between them) race on it and give undefined results;
 *   - the first call on each device looks the array's device address up
 *     (cudaGetSymbolAddress, with that device current) and must come before
 *     any stream capture on that device.  The lookup is repeated on the first
 *     call after the device's context has been destroyed and re-created
 *     (cudaDeviceReset); that call must likewise come before any capture.
 */
mls_status mls_junction_bwd_noalloc(const int32_t* x, int64_t T,
                                    const void* o_m, int64_t D_m,
                                    const void* e_next, int64_t V, int64_t delta,
                                    const void* dy, void* do_m, void* de_rows,
                                    float* dE_table, int accumulate_dE,
                                    mls_dtype dt, int32_t* dev_status, void* stream);

/* ------------------------------------------------------------------------ */
/* Multi-exit LM-head loss                                                   */
/* ------------------------------------------------------------------------ */

/*
 * Loss definition.  Logits per exit l_m = W^m h_m with W^m in R^{V x D_m}
 * ("Editing the methods of sub-models are made of blocks", Modeling
 * paragraph); next-token cross-entropy at every exit; the largest exit's
 * softmax p_M teaches every smaller exit through a token-level cross-entropy
 * mixed with weight alpha_d ("Matryoshka Language Model Suites", agihunt.info
 * summary, distillation paragraph) as (1 - alpha_d) CE_LM + alpha_d CE_KD
 * ("Is nesting the cheapest way to build a model suite?", section 4: 0.7 and
 * 0.3); per-exit losses summed with equal weight (same summary, limitations
 * paragraph).  Each term is a mean over the T tokens; the teacher is
 * stop-gradient; the distillation temperature is 1.
 *
 *   CE_LM,m = mean_t ( lse_m,t - l_m,t,y_t )
 *   CE_KD,m = mean_t ( lse_m,t - S_m,t ),  S_m,t = sum_v p_M,t,v l_m,t,v   (m < M)
 *   L = sum_{m<M} [(1 - alpha_d) CE_LM,m + alpha_d CE_KD,m] + CE_LM,M
 *
 * The T x V logits are never written to memory.
 *
 * Common arguments
 *   M          number of exits, 1 <= M <= 4
 *   D          HOST int64 [M], strictly increasing widths
 *   y_targets  device int32 [T] next-token targets in [0, V)
 *   h          HOST array of M device pointers, h[m] is dt [T, D[m]]
 *   W          HOST array of M device pointers, W[m] is dt [V, D[m]]
 *   Supported: MLS_BF16 needs every D[m] % 64 == 0 and V % 128 == 0 (tensor
 *   core path); MLS_F32 accepts any positive sizes (CUDA-core path).  All
 *   device pointers 16-byte aligned.
 */

/*
 * Workspace bytes for the forward and backward calls of this shape.
 *
 * MLS_BF16 backward: the dense logit gradient G' is formed and consumed one
 * block of tokens x one chunk of the vocabulary at a time, so its workspace
 * does not grow with T x V.  *bwd_bytes is the workspace of the split chosen
 * for a 1.5 GiB budget (or of the whole problem in one piece, when that is
 * smaller); mls_multiexit_loss_bwd accepts any workspace of at least
 * mls_multiexit_loss_bwd_plan's minimum and splits the work to fit the size
 * it is given (a larger workspace means fewer, larger pieces).
 */
mls_status mls_multiexit_loss_workspace(int M, int64_t T, const int64_t* D, int64_t V,
                                        mls_dtype dt, size_t* fwd_bytes, size_t* bwd_bytes);

/*
 * How mls_multiexit_loss_bwd (MLS_BF16) splits its work for a workspace of
 * ws_bytes: token blocks of *Tb tokens and vocabulary chunks of *Vc columns
 * (the last block and chunk may be shorter; *Tb = T and *Vc = V is one
 * piece), and *min_bytes, the smallest workspace the call accepts.  With
 * ws_bytes below *min_bytes, *Tb = *Vc = 0.  Host-only; no device is needed.
 * MLS_F32 has no split: *Tb = T, *Vc = V, *min_bytes = its bwd_bytes.
 */
mls_status mls_multiexit_loss_bwd_plan(int M, int64_t T, const int64_t* D, int64_t V, mls_dtype dt,
                                       size_t ws_bytes, int64_t* Tb, int64_t* Vc, size_t* min_bytes);

/*
 * mls_multiexit_loss_fwd
 *   losses  device f32 [2M]: CE_LM[0..M-1], CE_KD[0..M-2], L
 *   stats   device f32 [3M-1, T]: rows 0..M-1 lse_m, rows M..2M-1 the target
 *           logits l_m,y, rows 2M..3M-2 S_m (the _opts form: the statistic of
 *           the chosen distillation, and for Jensen-Shannon or acceptance with
 *           the teacher gradient 4M-2 rows, see mls_loss_options).  Kept for the
 *           backward pass.
 */
mls_status mls_multiexit_loss_fwd(int M, int64_t T, int64_t V, const int64_t* D,
                                  const int32_t* y_targets,
                                  const void* const* h, const void* const* W,
                                  float alpha_d, mls_dtype dt,
                                  float* losses, float* stats,
                                  void* workspace, size_t ws_bytes,
                                  int32_t* dev_status, void* stream);

/*
 * mls_multiexit_loss_bwd -- gradients of L times grad_scale.  With
 * q_m = softmax(l_m):
 *   G_m = grad_scale/T (q_m - (1 - alpha_d) onehot(y) - alpha_d p_M),  m < M
 *   G_M = grad_scale/T (q_M - onehot(y))
 *   dh[m] = G_m W^m           device dt [T, D[m]], overwritten
 *   dW[m] (+)= G_m^T h_m      device f32 [V, D[m]]; accumulate_dW != 0 adds
 *   stats is the forward call's output for the same inputs.
 * MLS_BF16: the logits are computed again tile by tile (never stored) and
 * the dense part of G (q_m - alpha_d p_M, or p_M for the largest exit) is
 * written in fp16 (11-bit significand; entries beyond +-65504, which finite
 * logits do not produce, saturate) for one token block x vocabulary chunk at
 * a time into the workspace (see mls_multiexit_loss_bwd_plan), then
 * multiplied on the tensor cores with fp16 copies of the block's h rows and
 * the chunk's W rows (exact for values in fp16's normal range; a tensor whose
 * largest magnitude is 2^15 or more, or below 2^-10, is copied scaled by a
 * power of two that the result undoes); the one-hot part is applied exactly
 * in fp32 from the bf16 inputs.  dh rows of a block are summed over the
 * chunks in fp32 (fixed order), dW rows of a chunk over the blocks in fp32
 * (fixed order): results are deterministic for a given workspace size.
 */
mls_status mls_multiexit_loss_bwd(int M, int64_t T, int64_t V, const int64_t* D,
                                  const int32_t* y_targets,
                                  const void* const* h, const void* const* W,
                                  float alpha_d, mls_dtype dt,
                                  const float* stats, float grad_scale,
                                  void* const* dh, float* const* dW, int accumulate_dW,
                                  void* workspace, size_t ws_bytes,
                                  int32_t* dev_status, void* stream);

/* Distillation term of the smaller exits. */
typedef enum {
  MLS_DISTILL_CE = 0,          /* token-level cross-entropy to the largest exit's softmax (default) */
  MLS_DISTILL_REVERSE_KL = 1,  /* KL(q_m || p_M), an alternative the pages' follow-ups propose   */
  MLS_DISTILL_JS = 2,          /* Jensen-Shannon divergence of q_m and p_M                         */
  MLS_DISTILL_ACCEPT = 3       /* 1 - sum_v min(q_m, p_M): acceptance of a drafted token           */
} mls_distill;

/*
 * Options of the _opts variants of the loss entry points (NULL = defaults).
 *   distill       MLS_DISTILL_CE (the pages' method) or MLS_DISTILL_REVERSE_KL
 *                 ("Is nesting the cheapest way to build a model suite?",
 *                 section 4, proposes swapping in reverse KL):
 *                   KD_m = mean_t sum_v q_m,v (log q_m,v - log p_M,v),
 *                   student gradient (teacher still stop-gradient)
 *                   G_m = grad_scale/T ((1 - alpha_d)(q_m - onehot(y))
 *                                       + alpha_d q_m (log q_m - log p_M - KL_t)).
 *                 With it, losses[M..2M-2] hold the mean KL and stats rows
 *                 2M..3M-2 hold R_m,t = sum_v q_m,t,v (l_m,t,v - l_M,t,v), so
 *                 KL_t = R_m,t - lse_m,t + lse_M,t; the backward call must get
 *                 the same option.
 *                 MLS_DISTILL_JS (same section): with mu = (q_m + p_M)/2,
 *                   KD_m = mean_t (KL(q_m || mu) + KL(p_M || mu)) / 2  (<= ln 2),
 *                   G_m = grad_scale/T ((1 - alpha_d)(q_m - onehot(y))
 *                                       + alpha_d q_m (log(q_m/mu)/2 - K_t)),
 *                 K_t = KL(q_m || mu)/2, stored by the forward call in stats
 *                 rows 2M..3M-2.  Its forward takes a second pass over the
 *                 logits (the divergence needs the final normalisers); the
 *                 backward call must get the same option.
 *                 MLS_DISTILL_ACCEPT (same section; the acceptance probability
 *                 of a drafted token as the objective): KD_m = mean_t (1 - beta_t), beta = sum_v
 *                 min(q_m, p_M), the total variation distance; student
 *                 (sub)gradient G_m = grad_scale/T ((1 - alpha_d)(q_m - onehot(y))
 *                 + alpha_d q_m (A_t - [q_m < p_M])), A_t = sum over q < p of q,
 *                 stored by the forward call in stats rows 2M..3M-2.  Its
 *                 forward takes a second pass like Jensen-Shannon.
 *                 Other values return MLS_ERR_INVALID_ARG.
 *   teacher_grad  0 (default): the largest exit's softmax in the distillation
 *                 terms is a constant (stop-gradient).  1: it is not, and the
 *                 largest exit's logit gradient gains, for every smaller exit m,
 *                 lambda_m alpha_d dKD_m/dl_M:
 *                   MLS_DISTILL_CE:         -p_M (l_m - S_m),  S_m = sum_v p_M l_m
 *                   MLS_DISTILL_REVERSE_KL:  p_M - q_m
 *                   MLS_DISTILL_JS:          p_M (log(p_M/mu)/2 - KL(p_M || mu)/2)
 *                   MLS_DISTILL_ACCEPT:      p_M (B_t - [q_m >= p_M]), B_t = sum over q >= p of p.
 *                 Pass the same options to both calls.  With MLS_DISTILL_JS
 *                 or MLS_DISTILL_ACCEPT the forward call then also writes the
 *                 teacher-side statistic (KL(p_M || mu)/2, or B_t) per token
 *                 into stats rows 3M-1 .. 4M-3, so stats must have 4M-2 rows
 *                 (otherwise 3M-1).  The pages leave the teacher's gradient
 *                 open.
 *   exit_weights  HOST float [M] or NULL: per-exit loss weights lambda_m,
 *                 L = sum_{m<M} lambda_m [(1 - alpha_d) CE_LM,m + alpha_d CE_KD,m]
 *                     + lambda_M CE_LM,M,
 *                 and every exit's gradient is scaled by its lambda_m.  NULL
 *                 means 1 for every exit, the pages' equal weights; the same
 *                 summary's limitations paragraph ("Matryoshka Language Model
 *                 Suites") reports that reweighting closes much of the gap.
 *                 Non-finite weights return MLS_ERR_INVALID_ARG.
 * The per-exit CE_LM and CE_KD in `losses` are unweighted; L is weighted.
 */
typedef struct {
  const float* exit_weights;
  int distill;                 /* mls_distill */
  int teacher_grad;            /* 0: teacher stop-gradient (default); 1: see above */
} mls_loss_options;

mls_status mls_multiexit_loss_fwd_opts(int M, int64_t T, int64_t V, const int64_t* D,
                                       const int32_t* y_targets,
                                       const void* const* h, const void* const* W,
                                       float alpha_d, mls_dtype dt,
                                       float* losses, float* stats,
                                       void* workspace, size_t ws_bytes,
                                       const mls_loss_options* opts,
                                       int32_t* dev_status, void* stream);

mls_status mls_multiexit_loss_bwd_opts(int M, int64_t T, int64_t V, const int64_t* D,
                                       const int32_t* y_targets,
                                       const void* const* h, const void* const* W,
                                       float alpha_d, mls_dtype dt,
                                       const float* stats, float grad_scale,
                                       void* const* dh, float* const* dW, int accumulate_dW,
                                       void* workspace, size_t ws_bytes,
                                       const mls_loss_options* opts,
                                       int32_t* dev_status, void* stream);

/*
 * mls_exit_agreement -- how well every smaller exit agrees with the largest
 * one, per token, from the same logits (computed again, never stored) and the
 * normalisers in `stats` from mls_multiexit_loss_fwd.  Measures named by the
 * pages: the acceptance probability of a drafted token, beta = sum_v min(q, p)
 * with draft q and verifier p ("Is nesting the cheapest way to build a model
 * suite?", section 4), and pairwise KL and top-1 next-token agreement between
 * exits ("Matryoshka Language Model Suites", alignment paragraph).  For each
 * smaller exit m (draft q = q_m) against the largest exit (verifier p = p_M):
 *   beta_m,t  = sum_v min(q_m,t,v, p_M,t,v)
 *   KL_m,t    = sum_v p_M,t,v (log p_M,t,v - log q_m,t,v)
 *   agree_m,t = [argmax_v l_m,t,v == argmax_v l_M,t,v], first maximum on ties
 *
 *   M >= 2; h, W, D, V, dt as for the loss; no targets are needed
 *   stats      device f32 [3M-1, T] from mls_multiexit_loss_fwd (lse rows used)
 *   metrics    device f32 [3(M-1)]: mean beta_m, mean KL_m, mean agree_m (m < M)
 *   per_token  device f32 [3(M-1), T] or NULL: the per-token rows, same order
 *   top1       device int32 [M, T] or NULL: argmax of every exit's logits
 *   workspace  >= mls_exit_agreement_workspace(...) bytes
 */
mls_status mls_exit_agreement_workspace(int M, int64_t T, const int64_t* D, int64_t V,
                                        mls_dtype dt, size_t* bytes);

mls_status mls_exit_agreement(int M, int64_t T, int64_t V, const int64_t* D,
                              const void* const* h, const void* const* W, mls_dtype dt,
                              const float* stats, float* metrics, float* per_token,
                              int32_t* top1, void* workspace, size_t ws_bytes,
                              int32_t* dev_status, void* stream);

/* ------------------------------------------------------------------------ */
/* Status                                                                    */
/* ------------------------------------------------------------------------ */

/*
 * Synchronises `stream`, copies *dev_status to *host_out and clears the device
 * word.  Returns MLS_ERR_BAD_ID or MLS_ERR_DEVICE_TIMEOUT when the matching
 * flag was set (timeout wins), MLS_OK when the word was 0.
 */
mls_status mls_status_read(int32_t* dev_status, void* stream, int32_t* host_out);

/*
 * mls_selftest_wait_timeout -- exercises the bounded device-side waits; not
 * part of the method (the pages have no counterpart).  It launches the
 * tensor-core statistics kernel of mls_multiexit_loss_fwd on the given
 * problem (MLS_BF16 only, arguments as for that call) with two changes: the
 * kernel's load warp issues no loads, so the barriers the other warps wait on
 * never complete, and every wait gives up after wait_limit_ns nanoseconds
 * (1e3 <= wait_limit_ns <= 4e9) instead of the library's 4 s.  The kernel
 * then sets MLS_DEVFLAG_TIMEOUT in *dev_status (required, non-NULL) and
 * returns with nothing in flight; the merge and reduction kernels that follow
 * still run, so `losses` and `stats` hold meaningless values.  The stream
 * stays usable: mls_status_read() reports MLS_ERR_DEVICE_TIMEOUT and clears
 * the flag, and later calls on the same stream behave normally.
 */
mls_status mls_selftest_wait_timeout(int M, int64_t T, int64_t V, const int64_t* D,
                                     const int32_t* y_targets,
                                     const void* const* h, const void* const* W,
                                     float* losses, float* stats,
                                     void* workspace, size_t ws_bytes,
                                     uint64_t wait_limit_ns,
                                     int32_t* dev_status, void* stream);

/* Static English text for a status code. */
const char* mls_status_string(mls_status s);

/* Library version as MAJOR*10000 + MINOR*100 + PATCH. */
int mls_version(void);

/* Number of CUDA kernels this library has launched in this process (all
 * devices, all threads).  Diagnostics only; the count never resets. */
uint64_t mls_kernel_launches(void);

#ifdef __cplusplus
}
#endif
#endif /* MLS_H_ */
