/*
 * onela.h -- C ABI of the shared-state Gated DeltaNet beam-decode library.
 *
 * One decode step of a Gated DeltaNet (GDN) layer for W beams that all grow
 * out of one shared prompt-derived state S0 per (request, head), following
 * "OneLA: Scaling Linear-Attention Decoding to Large Beams in Generative
 * Recommendation" (abstract; evolve.pub review, Summary and key claims on
 * section 3.2, equations 2-4).  Per head, with S_{t-1} the state of the beam's
 * parent,
 *
 *     S_t     = alpha_t S_{t-1} + delta_t k_t^T
 *     delta_t = beta_t (v_t - alpha_t S_{t-1} k_t),   alpha_t = exp(g_t)
 *     o_t     = S_t q_t = alpha_t S_{t-1} q_t + delta_t (k_t . q_t)
 *
 * No per-beam state is ever formed.  Every beam is a chain of small
 * transition records (alpha, delta, k), written once and never moved, that
 * an index of parent pointers ties together (review, Summary; abstract).
 * S_{t-1} x for x in {k_t, q_t} is computed as
 *     G (S0 x) + sum_j w_j (k_j . x) delta_j
 * over the beam's ancestor records j (w_j: product of the gates of the
 * records after j, G: product of all of them), with S0 read once per head and
 * used for every beam (the abstract's fused kernel shares S0 across beams).
 *
 * Conventions for every entry point
 *   - All tensor pointers are DEVICE pointers on the handle's device unless a
 *     comment says otherwise; tensors are dense, row-major, no padding.
 *   - Streams are CUDA streams passed as opaque pointers (NULL = the legacy
 *     default stream).  Work is enqueued on the stream; no entry point on the
 *     decode path synchronises the host, so the calls can be captured in a
 *     CUDA graph.
 *   - Inputs are borrowed for the stream-ordered duration of the call; the
 *     library keeps no pointer to caller memory beyond it (one exception,
 *     opt-in: ONELA_FLAG_PDL, below).  The library owns its
 *     copy of S0, the record store and the ancestry index and frees them in
 *     onela_destroy.
 *   - Return value: ONELA_OK or one of the ONELA_ERR_* codes below.  A call
 *     that returns an error has enqueued no work.
 */
#ifndef ONELA_H
#define ONELA_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define ONELA_API __attribute__((visibility("default")))
#else
#define ONELA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct onela_handle onela_handle;
typedef void *onela_stream; /* a cudaStream_t */

/* Element types. */
enum { ONELA_F32 = 0, ONELA_BF16 = 1 };

/* Return codes. */
enum {
  ONELA_OK = 0,
  ONELA_ERR_ARG = 1,         /* null pointer, bad size or dtype, bad W_prev  */
  ONELA_ERR_STATE = 2,       /* decode before onela_set_prompt_state         */
  ONELA_ERR_CAPACITY = 3,    /* W beyond W_max, or unfolded depths beyond T_max */
  ONELA_ERR_PARENT = 4,      /* the device saw a parent index outside
                                [0, W_prev); reported by the next call or by
                                onela_status                                 */
  ONELA_ERR_CUDA = 5,        /* a CUDA call failed (allocation, launch ...)  */
  ONELA_ERR_UNSUPPORTED = 6, /* the requested kernel cannot run this shape   */
  ONELA_ERR_SCRATCH = 7,     /* onela_decode_step_noalloc: the decode does not
                                fit in its fixed 32 MiB device array         */
  ONELA_ERR_TIMEOUT = 8      /* a bounded wait inside a kernel ran out (bit 1
                                of the error word): the outputs of that call
                                are void; reported by the next call or by
                                onela_status                                 */
};

/* onela_config.flags bits.
 *   ONELA_FLAG_PDL  launch decode steps t >= 2 of the tensor-core kernel as
 *                   programmatic dependents of the kernel before them in the
 *                   stream: step t starts while step t-1 still runs, does
 *                   all its work that needs no delta of an earlier step
 *                   (S0 products, ancestry, key products, gate weights), and
 *                   waits for step t-1 only before it stages the ancestors'
 *                   deltas.  For that it reads the k, gate and parent_idx
 *                   arrays of the earlier steps of the decode again (at
 *                   most the last T_max).  Set
 *                   it only when (a) the kernel before step t in the stream
 *                   produces no input of step t (q, k, v, g, beta,
 *                   parent_idx), and (b) the k, gate and parent_idx arrays of
 *                   the last T_max steps before t stay unchanged and
 *                   allocated until step t has completed -- e.g. back-to-back
 *                   decode steps whose inputs were all written before the
 *                   first of them, as in a CUDA graph of a whole decode, or
 *                   the verification of a tree of drafted tokens.  Step 1
 *                   never overlaps. */
enum { ONELA_FLAG_PDL = 1 };
/*   ONELA_FLAG_NVTX  mark every decode step, fold and prefill call on the
 *                   host with an NVTX range ("onela step t", ...) for
 *                   timeline profilers; off by default (the ranges cost a
 *                   little host time per call, nothing on the device). */
enum { ONELA_FLAG_NVTX = 4 };


/* Which decode kernel runs.  AUTO picks the tensor-core kernel when the
 * shape allows it (bf16 q/k/v, d_k = d_v in {64, 128, 256}; T_max <= 32,
 * W_max <= 4096) and the SIMT kernel otherwise. */
enum { ONELA_KERNEL_AUTO = 0, ONELA_KERNEL_SIMT = 1, ONELA_KERNEL_TC = 2 };

/* Handle configuration.
 *   R, H            requests and heads (each (request, head) pair has its own
 *                   S0 and its own records).
 *   d_k, d_v        key and value widths, 1 <= d <= 256.
 *   W_max           most beams per step.
 *   T_max           depths the record store keeps: a decode may run T_max
 *                   steps, and deeper when onela_fold keeps every step's
 *                   unfolded depths (t - 1 - D_r) below T_max.
 *   s0_dtype        ONELA_F32 or ONELA_BF16: element type of S0.
 *   qkv_dtype       ONELA_F32 or ONELA_BF16: element type of q, k, v (and of
 *                   the k stored in the records).
 *   kernel          ONELA_KERNEL_*.
 *   s0_split        fp32 S0 on the tensor-core kernel only: number of bf16
 *                   terms S0 is split into (2 or 3; 0 means 2).  Ignored
 *                   otherwise.
 *   device          CUDA device ordinal the handle lives on.
 *   flags           ONELA_FLAG_* bits (0: none): ONELA_FLAG_PDL,
 *                   ONELA_FLAG_NVTX.
 */
typedef struct {
  int32_t R, H, d_k, d_v, W_max, T_max;
  int32_t s0_dtype;
  int32_t qkv_dtype;
  int32_t kernel;
  int32_t s0_split;
  int32_t device;
  int32_t flags;
} onela_config;

/* Create a handle: validates cfg and allocates, on cfg->device, the S0 copy,
 * the record store (alpha fp32 [T_max][R][H][W_max], delta fp32
 * [T_max][R][H][W_max][d_v], k [T_max][R][H][W_max][d_k] in qkv_dtype; the
 * tensor-core kernel also keeps each step's parents, int32 [T_max][R][W_max],
 * and the bf16 operand image of S0), the
 * ancestry index (int32 [T_max][R][W_max][T_max]) and an error word in
 * mapped, pinned host memory that the kernels write and the host reads.
 * The store is a ring over depths: depth t uses slot (t - 1) mod T_max, and
 * an ancestry row holds the ancestor at depth j + 1 in entry j mod T_max.
 * Host-side allocation only; no kernel runs.  *out receives the handle.
 * Errors: ONELA_ERR_ARG (null pointer or invalid field), ONELA_ERR_CUDA. */
ONELA_API int onela_create(const onela_config *cfg, onela_handle **out);

/* Install the state that every beam of a request starts from (the one state
 * built from the prompt, abstract) and rewind the decode to step 0.
 *   S0  device pointer, [R][H][d_v][d_k] in cfg.s0_dtype.  Copied on `stream`
 *       (and, for the tensor-core kernel, converted once into the bf16
 *       operand layout); S0 may be freed once the stream has passed the call.
 * Errors: ONELA_ERR_ARG, ONELA_ERR_CUDA. */
ONELA_API int onela_set_prompt_state(onela_handle *h, const void *S0, onela_stream stream);

/* Build the state every beam of a request starts from out of the request's
 * prompt, on the device, and install it as onela_set_prompt_state does (the
 * one prompt-derived state of the abstract).  For every (request, head), the
 * GDN recurrence of the review's section 3.2 (equation 2) from the zero state
 * over the L prompt tokens,
 *     S_l = alpha_l S_{l-1} + delta_l k_l^T,
 *     delta_l = beta_l (v_l - alpha_l S_{l-1} k_l),   alpha_l = exp(g_l),
 * in fp32, rounded to cfg.s0_dtype once at the end.
 *   L        prompt tokens, L >= 1.
 *   k        [R][L][H][d_k] in qkv_dtype.
 *   v        [R][L][H][d_v] in qkv_dtype.
 *   g        [R][L][H] fp32, the log of the decay gate.
 *   beta     [R][L][H] fp32.
 * Rewinds the decode to step 0.  The inputs may be freed once the stream has
 * passed the call.
 * Tensor-core handles with bf16 k and v, d_k = d_v in {64, 128} and k, v on
 * 16-byte boundaries take the prompt in chunks of 64 tokens: per chunk the
 * intra-chunk system (I + A) Delta = Z of the delta rule is solved once from
 * the keys and gates, and the state advances by three tensor-core products
 * (operands split into bf16 terms, fp32 accumulation: the same result as
 * the token-by-token recurrence up to rounding order); the prompt is cut
 * into segments that run side by side and are combined through their
 * transition matrices (onela_set_prefill_segments).  This path keeps a
 * workspace of about 25 KB per (request, head, chunk) on the handle, which
 * the first call that needs more allocates (cudaMalloc, synchronous: not
 * inside a stream capture).  Every other handle runs the recurrence token by
 * token.
 * Errors: ONELA_ERR_ARG, ONELA_ERR_CUDA. */
ONELA_API int onela_prefill(onela_handle *h, int32_t L, const void *k, const void *v,
                            const float *g, const float *beta, onela_stream stream);

/* Copy the installed prompt state into a caller DEVICE buffer on `stream`:
 * [R][H][d_v][d_k] in cfg.s0_dtype.
 * Errors: ONELA_ERR_ARG, ONELA_ERR_STATE (no prompt state yet), ONELA_ERR_CUDA. */
ONELA_API int onela_read_prompt_state(onela_handle *h, void *S0, onela_stream stream);

/* One decode step t = (number of previous steps since the last rewind) + 1.
 *   W_prev      beams of the previous step; must be 1 at t = 1 (the prompt
 *               root) and the previous call's W afterwards.
 *   W           beams of this step, 1 <= W <= W_max.
 *   q, k        [R][W][H][d_k] in qkv_dtype.
 *   v           [R][W][H][d_v] in qkv_dtype.
 *   g           [R][W][H] fp32, the log of the decay gate: alpha = exp(g).
 *   beta        [R][W][H] fp32, the delta-rule write strength.
 *   parent_idx  [R][W] int32, beam b's parent among the previous step's
 *               beams, in [0, W_prev).  One array serves all heads.  With
 *               ONELA_FLAG_PDL the library reads it, k and gate again during
 *               the later steps of the decode (see the flag).
 *   o           [R][W][H][d_v] fp32, written: o_t = S_t q_t.
 * With the tensor-core kernel, q, k, v and o must start on 16-byte
 * boundaries (ONELA_ERR_ARG otherwise).
 * Also appends the records (alpha_t, delta_t, k_t) of every (beam, head) at
 * depth t and the ancestry rows of depth t; earlier records are never moved.
 * A parent index outside [0, W_prev) is clamped to 0 on the device, recorded
 * in the device error word and reported as ONELA_ERR_PARENT by the next call
 * on the handle (or by onela_status); the outputs of that step are then
 * meaningless.  Step t > T_max is refused (ONELA_ERR_CAPACITY) unless the
 * handle has folded since the last rewind; then the device checks that
 * t - 1 - D_r <= T_max - 1 for every request and otherwise reports
 * ONELA_ERR_CAPACITY the same way (the step's outputs are meaningless).
 * Errors: ONELA_ERR_ARG, ONELA_ERR_STATE, ONELA_ERR_CAPACITY,
 * ONELA_ERR_PARENT, ONELA_ERR_TIMEOUT, ONELA_ERR_UNSUPPORTED, ONELA_ERR_CUDA. */
ONELA_API int onela_decode_step(onela_handle *h, int32_t W_prev, int32_t W,
                      const void *q, const void *k, const void *v,
                      const float *g, const float *beta,
                      const int32_t *parent_idx, float *o,
                      onela_stream stream);

/* Several consecutive decode steps in one call, with every step's inputs
 * given at once: steps t = T + 1 .. T + n, T = steps done before the call.
 * Computes exactly what n calls of onela_decode_step compute (the same
 * kernel, launch by launch), with step i's W_prev the previous step's W (1 at
 * t = 1).
 *   n           1 <= n; the step count.
 *   W           HOST array of n beam counts, 1 <= W[i] <= W_max.
 *   q, k, v, g, beta, parent_idx, o
 *               HOST arrays of n DEVICE pointers: step i's tensors, laid out
 *               as for onela_decode_step with W = W[i].  They are borrowed for
 *               the stream-ordered duration of the call: none may change or
 *               be freed before the call's last step has completed.
 * Because all of a call's inputs exist before its first step runs, the
 * tensor-core kernel launches each step after the first as a programmatic
 * dependent of the step before it (the work that needs no earlier delta runs
 * while the previous step finishes, as with ONELA_FLAG_PDL, but without its
 * contract across calls): only a step whose early record writes would replace
 * a depth stored before the call (possible past T_max steps, with folds) is an
 * ordinary launch.  The first step of a call is always an ordinary launch.
 * Capacity: T + n <= T_max unless the handle has folded since the last
 * rewind.  q, k, v and o must start on 16-byte boundaries on a tensor-core
 * handle.  Every check that can be made on the host is made before the first
 * launch, so a host-side error leaves no work enqueued.
 * Errors: ONELA_ERR_ARG, ONELA_ERR_STATE, ONELA_ERR_CAPACITY,
 * ONELA_ERR_PARENT, ONELA_ERR_TIMEOUT, ONELA_ERR_UNSUPPORTED, ONELA_ERR_CUDA. */
ONELA_API int onela_decode_steps(onela_handle *h, int32_t n, const int32_t *W,
                                 const void *const *q, const void *const *k, const void *const *v,
                                 const float *const *g, const float *const *beta,
                                 const int32_t *const *parent_idx, float *const *o,
                                 onela_stream stream);

/* Bound of every wait inside the tensor-core step kernel on another of its
 * warp roles (the S0 products, the ancestor chains): limit_ns in [1e3, 1e10]
 * nanoseconds, default 2e9.  A wait that runs out sets bit 1 of the error
 * word (ONELA_ERR_TIMEOUT); the kernel then finishes without the missing
 * data (its outputs are void) instead of waiting longer.  stall != 0 is a
 * testing aid: in later tensor-core steps the wait for the ancestor chains
 * then expects one arrival that never comes, so that it runs out at the bound
 * (nothing faults or hangs); stall = 0 restores normal operation.
 * Errors: ONELA_ERR_ARG. */
ONELA_API int onela_set_wait_policy(onela_handle *h, uint64_t limit_ns, int32_t stall);

/* Number of segments the chunked tensor-core prefill cuts a prompt into
 * (1 .. 16; 0, the default, chooses one CTA per segment chain on every SM, at
 * least 4 chunks per segment).  A segment of n chunks costs one chain of n
 * sequential chunk updates; segments after the first also run the chain of
 * their transition matrix, and the combine costs one d x d x d product per
 * later segment.  Fewer segments than asked are used when the prompt has
 * fewer chunks.  Errors: ONELA_ERR_ARG. */
ONELA_API int onela_set_prefill_segments(onela_handle *h, int32_t segments);

/* Beam selection on the device: the next beam set out of the children of
 * the current one (the evolving beam tree of the abstract), so that the
 * parent indices of the next decode step never leave the GPU.  For request r
 * the candidate (b, c), b < W_prev, c < C, scores
 *     s = beam_score[r][b] + logp[r][b][c]      (one fp32 addition)
 * and the W candidates with the largest s are kept, best first; equal scores
 * (+0 and -0 are equal) go to the smaller flat index b*C + c; NaN ranks below
 * every number.  Outputs, DEVICE [R][W]:
 *   parent_idx  int32, b of the candidate (the next step's parent_idx),
 *   token       int32, c of the candidate,
 *   score       fp32, s (the next step's beam_score).
 *   beam_score  DEVICE fp32 [R][W_prev]; logp DEVICE fp32 [R][W_prev][C].
 *   scratch     DEVICE buffer of at least onela_select_scratch_bytes(R,
 *               W_prev, C, W) bytes, owned by the caller, borrowed for the
 *               stream-ordered duration of the call.
 * Sizes: R <= 65535, 1 <= W <= 2048, W <= W_prev * C < 2^32.  No host
 * synchronisation; capturable in a CUDA graph.
 * Errors: ONELA_ERR_ARG (null pointer, bad size), ONELA_ERR_SCRATCH (scratch
 * too small), ONELA_ERR_CUDA. */
ONELA_API size_t onela_select_scratch_bytes(int32_t R, int32_t W_prev, int32_t C, int32_t W);
ONELA_API int onela_select_beams(int32_t R, int32_t W_prev, int32_t C, int32_t W,
                                 const float *beam_score, const float *logp,
                                 int32_t *parent_idx, int32_t *token, float *score,
                                 void *scratch, size_t scratch_bytes, int32_t device,
                                 onela_stream stream);

/* Rewind to step 0 keeping S0 (records and any fold are logically dropped,
 * nothing is freed) and clear the error word.  Waits for `stream` first, so that no
 * step still in flight can set the word after it is cleared; not meant for
 * the inside of a captured region.
 * Errors: ONELA_ERR_ARG, ONELA_ERR_CUDA. */
ONELA_API int onela_reset(onela_handle *h, onela_stream stream);

/* Fold the shared ancestor prefix of every request into its root state, so
 * that later steps replay only the records below it.  An extension of the
 * method: the evolve.pub review's Summary and Weaknesses name the replay
 * cost that grows with decode depth (every ancestor's record is replayed at
 * every step).  For each request r, with t = steps done and W_t the beams of
 * step t: D_r = the deepest depth <= max_depth at which all W_t beams have
 * the same ancestor (D_r = t when W_t = 1; never below the depth already
 * folded).  The root state becomes that ancestor's full state,
 *     S <- alpha_d S + delta_d k_d^T   for the newly folded depths d,
 * (the GDN recurrence of the review's section 3.2, equation 2) computed in
 * fp32 from the records and stored in cfg.s0_dtype, and later steps replay
 * depths D_r + 1 .. t' - 1 only.  The outputs stay those of the unfolded
 * decode up to that one rounding of the folded state.  Records, ancestry
 * rows and the prompt state itself are unchanged; onela_reset,
 * onela_set_prompt_state and onela_prefill return to the prompt state.
 * Folding lets a decode go past T_max steps: the store keeps the last T_max
 * depths, and only the unfolded ones are read.
 *   max_depth  >= 0; values above the steps done act as the steps done;
 *              0 (or no step done yet) leaves everything as it is.
 * Runs on the device only (no host synchronisation; capturable in a CUDA
 * graph: the prompt state is never overwritten, so a captured decode that
 * folds replays from the prompt each time).  Tensor-core handles with
 * d_k = d_v <= 128 and T_max <= 16 fold in one launch that overlaps the
 * steps around it: it starts once the step before it is complete, and a
 * step launched while it runs replays from the root state before the fold
 * (which the fold leaves alone) where those depths still fit the record
 * store, else it waits for the fold; the outputs are the same either way up
 * to rounding.  Other handles fold in ordinary launches, and the next step
 * is an ordinary launch too.  Memory: a second state buffer and, tensor-core
 * kernel, two operand images of it, allocated by onela_create.
 * Errors: ONELA_ERR_ARG, ONELA_ERR_STATE (no prompt state), ONELA_ERR_PARENT
 * (a bad parent index was seen: the ancestry is meaningless), ONELA_ERR_TIMEOUT,
 * ONELA_ERR_CAPACITY, ONELA_ERR_CUDA. */
ONELA_API int onela_fold(onela_handle *h, int32_t max_depth, onela_stream stream);

/* Copy the root state the decode replays from (the prompt state, or the
 * folded state after onela_fold) into a caller DEVICE buffer on `stream`:
 * [R][H][d_v][d_k] in cfg.s0_dtype.
 * Errors: ONELA_ERR_ARG, ONELA_ERR_STATE, ONELA_ERR_CUDA. */
ONELA_API int onela_read_root_state(onela_handle *h, void *S, onela_stream stream);

/* Copy the folded depth D_r of every request into a caller DEVICE buffer of
 * R int32 on `stream` (all 0 when nothing is folded).
 * Errors: ONELA_ERR_ARG, ONELA_ERR_CUDA. */
ONELA_API int onela_read_fold_depth(onela_handle *h, int32_t *depth, onela_stream stream);

/* Wait for the handle's device (cudaDeviceSynchronize on it) and report the
 * error word in *device_err (0: none; bit 0: a bad parent index; bit 1: a
 * bounded wait ran out in a tensor-core kernel, whose outputs are then void;
 * bit 2: a step's unfolded depths did not fit the store; several bits may be
 * set).  Returns ONELA_ERR_PARENT when bit 0 is set, else ONELA_ERR_TIMEOUT
 * when bit 1 is, else ONELA_ERR_CAPACITY when bit 2 is, else ONELA_OK.  The
 * decode calls and onela_fold return the same code, without waiting, for
 * what earlier calls left in the word.
 * Errors: ONELA_ERR_ARG, ONELA_ERR_CUDA. */
ONELA_API int onela_status(onela_handle *h, int32_t *device_err);

/* Free everything the handle owns (synchronises its device first).
 * Errors: ONELA_ERR_ARG. */
ONELA_API int onela_destroy(onela_handle *h);

/* Copy the records of depth t (steps done - T_max < t <= steps done: the
 * depths the store still holds) into caller DEVICE
 * buffers on `stream`: alpha fp32 [R][H][W_t], delta fp32 [R][H][W_t][d_v],
 * k [R][H][W_t][d_k] in qkv_dtype.  Any of the three may be NULL.
 * Errors: ONELA_ERR_ARG, ONELA_ERR_CUDA. */
ONELA_API int onela_read_records(onela_handle *h, int32_t t, float *alpha, float *delta,
                       void *k, onela_stream stream);

/* Copy the ancestry rows of depth t (1 <= t <= steps done, t <= T_max,
 * and t still held: steps done - T_max < t) into a caller
 * DEVICE buffer on `stream`: int32 [R][W_t][t-1], entry [r][b][j] = index of
 * the beam at depth j+1 on the path from the root to beam b of step t.
 * Errors: ONELA_ERR_ARG, ONELA_ERR_CUDA. */
ONELA_API int onela_read_ancestry(onela_handle *h, int32_t t, int32_t *anc,
                        onela_stream stream);

/* Query: number of decode steps done since the last rewind, and the kernel
 * the handle runs (ONELA_KERNEL_SIMT or ONELA_KERNEL_TC). */
ONELA_API int onela_steps_done(const onela_handle *h);
ONELA_API int onela_kernel_kind(const onela_handle *h);
/* Query: kernel launches the last successful decode or prefill call enqueued
 * (onela_decode_step: 1; onela_decode_steps: n; onela_prefill: 4 on the
 * chunked tensor-core path, 2 on the token-by-token path of a tensor-core
 * handle (the recurrence, then the S0 operand image), 1 otherwise; 0 before
 * any call). */
ONELA_API int onela_last_call_launches(const onela_handle *h);

/* Decode step without any device allocation.
 *
 * The paper has no counterpart to this entry point; it exists for callers
 * that cannot allocate device memory: code running while a CUDA stream is
 * being captured (cudaMalloc is refused there) and plug-ins whose host engine
 * owns all device memory and passes them nothing but their input and output
 * tensors.  It computes exactly what onela_decode_step computes (same SIMT
 * kernel), but keeps the record store, the ancestry index and the error word
 * in one fixed array of 32 MiB that is part of the library (a file-scope
 * __device__ array), instead of in memory owned by a handle.
 *
 *   cfg        shapes and dtypes (R, H, d_k, d_v, W_max, T_max, s0_dtype,
 *              qkv_dtype, device); kernel, s0_split and flags are ignored.  W_max and
 *              T_max fix the array's layout and must stay the same for all
 *              steps of one decode.
 *   t          this step's depth, 1..T_max; call t = 1, 2, ... in order.
 *              A call with t = 1 starts a new decode and clears the error
 *              word.
 *   W_prev, W  beams of the previous step (1 at t = 1) and of this one.
 *              W_prev must be the previous call's W: the array keeps no
 *              host-side record of it, so this is not verified, and a larger
 *              W_prev would let parent indices reach rows an earlier decode
 *              left in the array (silently wrong outputs).
 *   S0         [R][H][d_v][d_k] in s0_dtype, read directly at every step.
 *   q, k, v, g, beta, parent_idx, o   as for onela_decode_step.
 *   status     DEVICE pointer to one int32, written on `stream` with the
 *              error word after the step: 0, or bit 0 set when some parent
 *              index of this decode was outside [0, W_prev) (the index was
 *              clamped to 0 and the outputs are meaningless).
 * Memory: the array lives on every device where the library's module holding
 * it is loaded, from the first call on that device until the process exits.
 * Set-up: the first call on a device, with that device current, looks up the
 * array's device address once; make that first call before any stream
 * capture begins.  No call allocates or frees device memory.
 * Sharing: every call, from any thread or stream, uses the same array and
 * sees what the previous call left there, so decodes whose calls overlap on
 * the GPU race with one another and give wrong results; run one decode at a
 * time per device.
 * Errors: ONELA_ERR_ARG (null pointer, invalid shape, t or W out of range),
 * ONELA_ERR_SCRATCH (T_max * R * H * W_max records plus the ancestry rows do
 * not fit in 32 MiB), ONELA_ERR_CUDA. */
ONELA_API int onela_decode_step_noalloc(const onela_config *cfg, int32_t t, int32_t W_prev, int32_t W,
                                        const void *S0, const void *q, const void *k, const void *v,
                                        const float *g, const float *beta, const int32_t *parent_idx,
                                        float *o, int32_t *status, onela_stream stream);

/* Static description of a return code (never NULL). */
ONELA_API const char *onela_error_string(int code);

#ifdef __cplusplus
}
#endif

#endif /* ONELA_H */
