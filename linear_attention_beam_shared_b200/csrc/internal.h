// Internal declarations shared by the runtime and the decode kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace onela {

constexpr int kHistSteps = 33;     // steps of history the tensor-core kernel can see (its window is <= 32)
constexpr int kHistMaxInts = 4096;  // parents of earlier steps the tensor-core kernel
                                    // keeps in shared memory (more: read from global memory)

// Everything one decode step needs.  Record store and ancestry index are the
// handle's; all other pointers are the caller's tensors for this step.
struct StepParams {
  int R, H, dk, dv;
  int W, W_prev;  // beams of this step and of the previous one
  int t;          // 1-based depth of the beams this step creates
  int W_max, T_max;
  const void *q, *k, *v;  // [R][W][H][d] in the qkv type
  const float *g, *beta;  // [R][W][H]
  const int32_t *parents; // [R][W]
  int32_t *par_store;     // [T_max slots][R][W_max]: each step's parents (tensor-core kernel)
  // History of the decode for the tensor-core kernel: entry i describes step
  // j = hbase + i (hbase <= j < t, at most kHistSteps steps back): keys,
  // gates and parents.  Bit i of hist_inputs set: the callers' own arrays of
  // step j (still valid: under ONELA_FLAG_PDL, or a step of the same
  // onela_decode_steps call) -- hk[i] [R][W_j][H][d_k], hg[i] [R][W_j][H]
  // (the gate before exp), hpar[i] [R][W_j].  Bit clear: the record store
  // (rec_k, rec_alpha) and the par_store row of step j.  Parents of request r
  // start at hpar[i] + r * hpar_rs[i]; hW[i] = W_j.  The kernel copies the
  // parents of steps hcopy .. t - 1 to shared memory.
  uint64_t hist_inputs;
  int hbase, hcopy;
  const void *hk[kHistSteps];
  const float *hg[kHistSteps];
  const int32_t *hpar[kHistSteps];
  int hpar_rs[kHistSteps];
  int hW[kHistSteps];
  int hoff[kHistSteps];  // where step j's parents start in the kernel's shared copy (entries)
  int hist_cap;  // entries of shared memory for the parents of steps hcopy..t-1 (0: read them from global memory)
  float *o;               // [R][W][H][dv]
  const void *S0;         // [R][H][dv][dk] in the S0 type
  const void *S0img;      // tensor-core operand image of S0 (see step_tc.cu)
  int s0_planes;          // bf16 terms in S0img (1 for bf16 S0)
  // The record store keeps the last T_max depths: depth s sits in slot
  // (s - 1) mod T_max (rec_slot).  A step replays depths d0 + 1 .. t - 1,
  // which must fit: t - 1 - d0 <= T_max - 1 (else kErrWindow).
  float *rec_alpha;       // [T_max slots][R][H][W_max]
  float *rec_delta;       // [T_max slots][R][H][W_max][dv]
  void *rec_k;            // [T_max slots][R][H][W_max][dk] in the qkv type
  // Ancestry rows [T_max slots][R][W_max][T_max]: the row of a beam of depth
  // s holds its ancestor at depth j + 1 in entry j mod T_max, for the last
  // T_max - 1 depths before s.
  int32_t *anc;
  // Folded prefix (onela_fold), per request: depths 1..d0[r] are folded into
  // S0 (then the folded state), their ancestors are the same for every beam
  // of the request, anc_fold[r][j mod T_max] at depth j + 1 ([R][T_max], the
  // last T_max depths), and only depths d0[r] + 1 .. t - 1 are replayed.
  // d0 null: nothing folded.
  const int32_t *d0;
  const int32_t *anc_fold;
  int32_t *err;           // host-mapped error word (device view)
  // Bound of every wait of the tensor-core kernel on another warp role
  // (nanoseconds); stall = 1 (tests only) makes the wait for the ancestry
  // warp run out at that bound.
  unsigned long long wait_limit_ns;
  int stall;
  // After a one-launch tensor-core fold (and until the next fold or
  // rewind), for the tensor-core kernel: each CTA of that fold adds 1 to
  // fold_done[r] (release at GPU scope) once its part of request r's folded
  // state is written, so fold_done[r] >= fold_target means the fold is
  // complete.  A CTA that sees it complete (acquire) replays from d0 and
  // S0img.  Else, where the folded depth before that fold, d0_old[r] (0 if
  // d0_old is null), still fits the record store (t - 1 - d0_old <= T_max -
  // 1), it replays from it and its image S0img_old, which the fold does not
  // write; else it waits for the kernel before it (whose completion implies
  // the fold's) and replays from d0 and S0img.  fold_pending 0: d0 and S0img.
  // The counts restart with every decode: step 1 zeroes fold_reset[r]
  // (the same counters; null where the handle has none), and fold_target
  // counts the CTAs of the folds since then.
  int fold_pending;
  const int *fold_done;
  int fold_target;
  int *fold_reset;
  const int32_t *d0_old;
  const void *S0img_old;
  // TMA descriptors of k, q and v (tensor-core kernel; encoded per call):
  // 4-D {d, H, W, R} bf16, box {64, 1, 32, 1}, 128-byte swizzle.
  alignas(64) CUtensorMap tm_k;
  alignas(64) CUtensorMap tm_q;
  alignas(64) CUtensorMap tm_v;

};

// Slot of depth s (1-based) in the record store, the parents store and the
// ancestry rows.
__host__ __device__ __forceinline__ int rec_slot(const StepParams &p, int s) { return (s - 1) % p.T_max; }
// Row index of the record of beam b, head h, request r in a slot.
__host__ __device__ __forceinline__ int64_t rec_row_slot(const StepParams &p, int slot, int r, int h, int b) {
  return ((int64_t)(slot * p.R + r) * p.H + h) * p.W_max + b;
}
// Row index of the record of beam b, head h, request r at depth s (1-based).
__host__ __device__ __forceinline__ int64_t rec_row(const StepParams &p, int s, int r, int h, int b) {
  return rec_row_slot(p, rec_slot(p, s), r, h, b);
}
// First entry of the ancestry row of beam b, request r, at depth s (1-based).
__host__ __device__ __forceinline__ int64_t anc_row(const StepParams &p, int s, int r, int b) {
  return ((int64_t)(rec_slot(p, s) * p.R + r) * p.W_max + b) * p.T_max;
}

// Device error word.  Each condition owns one byte of the word, which a
// kernel sets to 1 with a plain byte store, so that two conditions seen in one
// launch never overwrite each other (the word may be host-mapped memory, where
// a read-modify-write from the device is not atomic).  The host turns the raw
// word into the documented bits with err_bits.
constexpr int kErrByteParent = 0;   // a parent index outside [0, W_prev)
constexpr int kErrByteTimeout = 1;  // a bounded wait ran out: that launch's outputs are void
constexpr int kErrByteWindow = 2;   // a step's unfolded depths did not fit the record store
constexpr int32_t kErrParent = 1, kErrTimeout = 2, kErrWindow = 4;  // documented bits
__device__ __forceinline__ void set_err(int32_t *err, int byte) {
  reinterpret_cast<volatile uint8_t *>(err)[byte] = 1;
}
inline int32_t err_bits(int32_t raw) {
  const uint32_t u = (uint32_t)raw;
  return ((u & 0xffu) ? kErrParent : 0) | (((u >> 8) & 0xffu) ? kErrTimeout : 0) |
         (((u >> 16) & 0xffu) ? kErrWindow : 0);
}

// Raises the dynamic shared-memory limit of kernel `func` on the current
// device to at least `smem` bytes.  The attribute is set once per (kernel,
// device, larger size): it is not a stream operation, so it must not be
// repeated inside a captured region.  Safe to call from several host threads.
cudaError_t ensure_smem_limit(const void *func, size_t smem);

// Kernel launchers (step_simt.cu, step_tc.cu).  Return a cudaError_t.
cudaError_t launch_step_simt(const StepParams &p, int qkv_bf16, int s0_bf16, cudaStream_t s);
cudaError_t launch_step_tc(const StepParams &p, int pdl, cudaStream_t s);
// Folds, per request, the deepest ancestor at depth <= max_depth that every
// beam of step p.t shares into the folded state S_fold: reads the previous
// folded depth from d0_in (unless first), writes the new one to d0_out and
// the newly shared ancestors to anc_fold; S_fold becomes the ancestor's full
// state, from S_fold (or p.S0 when first) by S <- alpha S + delta k^T over
// the newly folded depths, fp32 arithmetic, stored in the state's type.
// When first, every request's S_fold is written.  General shapes: two
// ordinary launches.
cudaError_t launch_fold(const StepParams &p, int Wt, int max_depth, int first, const int32_t *d0_in, int32_t *d0_out,
                        int32_t *anc_fold, void *S_fold, int qkv_bf16, int s0_bf16, cudaStream_t s);
// The same for tensor-core handles (bf16 keys, d_k = d_v in {64, 128},
// T_max <= kFoldTcMaxT) in one launch that also writes S_fold's operand image (with
// p.s0_planes terms); programmatic launch when pdl (the kernel waits before
// it reads the ancestry rows and records; it reads S_fold and d0_in before,
// so the previous kernel must not be a fold).
constexpr int kFoldTcMaxT = 16;  // deepest record store of the one-launch tensor-core fold
// Each CTA adds 1 to done[r] (release) when its part of request r is
// written; fold_tc_ctas(p) CTAs per request.
cudaError_t launch_fold_tc(const StepParams &p, int Wt, int max_depth, int first, const int32_t *d0_in,
                           int32_t *d0_out, int32_t *anc_fold, void *S_fold, void *img, int s0_bf16, int pdl,
                           int *done, cudaStream_t s);
int fold_tc_ctas(const StepParams &p);
cudaError_t launch_s0_image(const void *S0, void *img, int R, int H, int dk, int dv,
                            int s0_bf16, int planes, cudaStream_t s);
size_t s0_image_bytes(int R, int H, int dk, int dv, int planes);
// The GDN recurrence from the zero state over L prompt tokens for every
// (request, head): k [R][L][H][dk], v [R][L][H][dv] (bf16 if qkv_bf16, else
// fp32), g and beta [R][L][H] fp32 -> S0 [R][H][dv][dk] (bf16 if s0_bf16).
cudaError_t launch_prefill(const void *k, const void *v, const float *g, const float *beta, void *S0, int R, int L,
                           int H, int dk, int dv, int qkv_bf16, int s0_bf16, cudaStream_t s);
bool tc_supports(int dk, int dv, int qkv_bf16, int T_max, int W_max, int planes);
// The same recurrence in 64-token chunks on the tensor cores (prefill_tc.cu)
// for bf16 k and v with d_k = d_v = d in {64, 128}, k and v 16-byte aligned:
// the prompt is cut into nseg segments whose chains run side by side (one CTA
// per segment for the values, one more per later segment for its transition
// matrix) and are then combined.  ws holds prefill_tc_ws_bytes(R, L, H, d,
// nseg) bytes, 16-byte aligned; a wait that runs out sets the timeout byte of
// err.  Three launches.
constexpr int kMaxPrefillSegments = 16;
bool prefill_tc_supports(int dk, int dv, int qkv_bf16);
int prefill_tc_segments(int R, int L, int H, int want);  // want <= 0: chosen for the SM count
size_t prefill_tc_prep_bytes(int R, int L, int H);
size_t prefill_tc_ws_bytes(int R, int L, int H, int d, int nseg);
cudaError_t launch_prefill_tc(const void *k, const void *v, const float *g, const float *beta, void *S0, int R, int L,
                              int H, int d, int s0_bf16, int nseg, void *ws, unsigned long long wait_ns, int32_t *err,
                              cudaStream_t s);

// Beam selection (select.cu): the W best of W_prev x C candidates per request.
size_t select_scratch_bytes(int R, int W_prev, int C, int W);
cudaError_t launch_select(const float *beam_score, const float *logp, int R, int W_prev, int C, int W,
                          int32_t *parent, int32_t *token, float *score, void *scratch, cudaStream_t s);

}  // namespace onela
