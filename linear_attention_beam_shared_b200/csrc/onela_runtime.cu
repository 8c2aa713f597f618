// Host runtime of the decode library: handle, validation, record store,
// ancestry index, error word, and the C ABI declared in include/onela.h.
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>

#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <map>
#include <mutex>
#include <new>
#include <utility>
#include <vector>

#include "../../include/onela.h"
#include "internal.h"

struct onela_handle {
  onela_config cfg;
  int kernel;        // ONELA_KERNEL_SIMT or ONELA_KERNEL_TC
  int planes;        // bf16 terms of the S0 operand image (tensor-core kernel)
  int steps_done;    // decode steps since the last rewind
  int has_prompt;
  std::vector<int> Ws;  // beams of each step done
  void *S0;
  void *S0img;
  // Folded prefix (onela_fold): the root state the decode replays from once
  // folded, its operand image (tensor-core kernel), and on the device the
  // folded depths d0 [2][R] (double-buffered: a fold reads one and writes
  // the other) and anc_fold [R][T_max].  The prompt state and its image stay
  // as they are, so a rewind needs no device work.
  void *S0f;
  void *S0fimg[2];  // its operand images: [fold_cur] the current one, the other the one before
  int32_t *fold_buf;
  int folded;      // S0f and fold_buf are in use since the last rewind
  int fold_cur;    // which d0 buffer holds the current depths
  int after_fold;  // the last call was a fold
  int fold_prev;   // a fold came before the last one since the rewind (its depth and image are the old ones)
  // The last fold was the one-launch tensor-core fold, whose CTAs count
  // themselves done in fold_buf's done counters ([R], zeroed by step 1 of
  // each decode); fold_target: the count each request's counter reaches once
  // the last fold is complete.
  int fold_pending;
  int fold_target;
  int32_t *par_store;         // each step's parents, written by the kernel
  // Every earlier call's k, gate and parent_idx (caller memory; read again
  // only under ONELA_FLAG_PDL).
  std::vector<const void *> hist_k;
  std::vector<const float *> hist_g;
  std::vector<const int32_t *> hist_par;
  float *rec_alpha;
  float *rec_delta;
  void *rec_k;
  int32_t *anc;
  int32_t *err_host;  // host-mapped error word
  int32_t *err_dev;   // its device view
  // Bound of every wait inside the tensor-core step kernel, and the testing
  // aid of onela_set_wait_policy.
  unsigned long long wait_limit_ns;
  int stall;
  int last_launches;  // kernel launches of the last decode or prefill call
  // Chunked tensor-core prefill: its workspace (grown on demand) and the
  // number of prompt segments asked for (0: chosen from the SM count).
  void *pf_ws;
  size_t pf_ws_bytes;
  int pf_segments;
};

namespace {

size_t esize(int dtype) { return dtype == ONELA_BF16 ? 2 : 4; }

bool valid_dtype(int d) { return d == ONELA_F32 || d == ONELA_BF16; }

// An NVTX range on the host for the duration of a call, when the handle
// asks for them (ONELA_FLAG_NVTX).
struct NvtxRange {
  bool on;
  NvtxRange(const onela_config &c, const char *what, int t) : on((c.flags & ONELA_FLAG_NVTX) != 0) {
    if (!on) return;
    char name[48];
    std::snprintf(name, sizeof(name), t > 0 ? "onela %s %d" : "onela %s", what, t);
    nvtxRangePushA(name);
  }
  ~NvtxRange() {
    if (on) nvtxRangePop();
  }
};

// Switch to the handle's device for the duration of a call.
struct DeviceGuard {
  int prev = -1;
  bool ok = false;
  explicit DeviceGuard(int dev) {
    if (cudaGetDevice(&prev) != cudaSuccess) return;
    ok = (prev == dev) || (cudaSetDevice(dev) == cudaSuccess);
  }
  ~DeviceGuard() {
    if (ok && prev >= 0) cudaSetDevice(prev);
  }
};

// The prompt state is in place: the decode starts again at step 0.
void rewind_to_prompt(onela_handle *h) {
  h->has_prompt = 1;
  h->steps_done = 0;
  h->folded = 0;
  h->after_fold = 0;
  h->fold_pending = 0;
  h->fold_target = 0;
  h->Ws.clear();
  h->hist_k.clear();
  h->hist_g.clear();
  h->hist_par.clear();
}

void free_all(onela_handle *h) {
  cudaFree(h->S0);
  cudaFree(h->S0img);
  cudaFree(h->S0f);
  cudaFree(h->S0fimg[0]);
  cudaFree(h->S0fimg[1]);
  cudaFree(h->fold_buf);
  cudaFree(h->rec_alpha);
  cudaFree(h->par_store);
  cudaFree(h->rec_delta);
  cudaFree(h->rec_k);
  cudaFree(h->anc);
  cudaFree(h->pf_ws);
  if (h->err_host) cudaFreeHost(h->err_host);
}

// The return code for what the device error word holds (ONELA_OK if nothing).
int word_code(const onela_handle *h) {
  const int32_t bits = onela::err_bits(*reinterpret_cast<volatile int32_t *>(h->err_host));
  if (bits & onela::kErrParent) return ONELA_ERR_PARENT;
  if (bits & onela::kErrTimeout) return ONELA_ERR_TIMEOUT;
  if (bits & onela::kErrWindow) return ONELA_ERR_CAPACITY;
  return ONELA_OK;
}

onela::StepParams base_params(const onela_handle *h) {
  onela::StepParams p;
  std::memset(&p, 0, sizeof(p));
  p.R = h->cfg.R;
  p.H = h->cfg.H;
  p.dk = h->cfg.d_k;
  p.dv = h->cfg.d_v;
  p.W_max = h->cfg.W_max;
  p.T_max = h->cfg.T_max;
  p.S0 = h->folded ? h->S0f : h->S0;
  p.S0img = h->folded ? h->S0fimg[h->fold_cur] : h->S0img;
  p.d0 = h->folded ? h->fold_buf + h->fold_cur * h->cfg.R : nullptr;
  p.anc_fold = h->fold_buf + 2 * h->cfg.R;
  p.s0_planes = h->planes;
  p.rec_alpha = h->rec_alpha;
  p.par_store = h->par_store;
  p.rec_delta = h->rec_delta;
  p.rec_k = h->rec_k;
  p.anc = h->anc;
  p.err = h->err_dev;
  p.wait_limit_ns = h->wait_limit_ns;
  p.stall = h->stall;
  return p;
}

}  // namespace

namespace onela {

cudaError_t ensure_smem_limit(const void *func, size_t smem) {
  static std::mutex mu;
  static std::map<std::pair<const void *, int>, size_t> done;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(mu);
  size_t &have = done[{func, dev}];
  if (smem <= have) return cudaSuccess;
  e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e == cudaSuccess) have = smem;
  return e;
}

}  // namespace onela

extern "C" {

const char *onela_error_string(int code) {
  switch (code) {
    case ONELA_OK: return "ok";
    case ONELA_ERR_ARG: return "invalid argument";
    case ONELA_ERR_STATE: return "no prompt state installed";
    case ONELA_ERR_CAPACITY:
      return "beam count beyond W_max, or unfolded depths beyond the T_max the record store keeps";
    case ONELA_ERR_PARENT: return "parent index outside [0, W_prev) seen on the device";
    case ONELA_ERR_CUDA: return "CUDA call failed";
    case ONELA_ERR_UNSUPPORTED: return "kernel does not support this shape";
    case ONELA_ERR_SCRATCH: return "decode does not fit in the 32 MiB array of onela_decode_step_noalloc";
    case ONELA_ERR_TIMEOUT: return "a bounded wait inside a kernel ran out; the outputs since the last check are void";
    default: return "unknown error";
  }
}

int onela_create(const onela_config *cfg, onela_handle **out) {
  if (!cfg || !out) return ONELA_ERR_ARG;
  *out = nullptr;
  const onela_config c = *cfg;
  if (c.R < 1 || c.H < 1 || c.d_k < 1 || c.d_k > 256 || c.d_v < 1 || c.d_v > 256 || c.W_max < 1 ||
      c.T_max < 1 || c.T_max > 64 || !valid_dtype(c.s0_dtype) || !valid_dtype(c.qkv_dtype) ||
      c.kernel < ONELA_KERNEL_AUTO || c.kernel > ONELA_KERNEL_TC || c.device < 0 ||
      !(c.s0_split == 0 || c.s0_split == 2 || c.s0_split == 3) ||
      (c.flags & ~(ONELA_FLAG_PDL | ONELA_FLAG_NVTX)) != 0)
    return ONELA_ERR_ARG;
  // Sizes must stay addressable with 64-bit offsets and the kernels' int grid.
  const double rows = (double)c.T_max * c.R * c.H * c.W_max;
  if (rows * (4.0 + 4.0 * c.d_v + esize(c.qkv_dtype) * (double)c.d_k) > 1.5e11) return ONELA_ERR_ARG;
  if ((double)c.R * c.W_max * c.H * (c.d_k > c.d_v ? c.d_k : c.d_v) > 2.0e9) return ONELA_ERR_ARG;

  const int qkv_bf16 = c.qkv_dtype == ONELA_BF16;
  const int planes = c.s0_dtype == ONELA_BF16 ? 1 : (c.s0_split == 0 ? 2 : c.s0_split);
  int kernel = c.kernel;
  const bool tc_ok = onela::tc_supports(c.d_k, c.d_v, qkv_bf16, c.T_max, c.W_max, planes);
  if (kernel == ONELA_KERNEL_AUTO) kernel = tc_ok ? ONELA_KERNEL_TC : ONELA_KERNEL_SIMT;
  if (kernel == ONELA_KERNEL_TC && !tc_ok) return ONELA_ERR_UNSUPPORTED;

  int ndev = 0;
  if (cudaGetDeviceCount(&ndev) != cudaSuccess || c.device >= ndev) return ONELA_ERR_CUDA;
  DeviceGuard g(c.device);
  if (!g.ok) return ONELA_ERR_CUDA;

  onela_handle *h = new (std::nothrow) onela_handle();
  if (!h) return ONELA_ERR_CUDA;
  h->cfg = c;
  h->kernel = kernel;
  h->planes = planes;
  h->steps_done = 0;
  h->has_prompt = 0;
  h->wait_limit_ns = 2000000000ull;
  h->stall = 0;
  const size_t nS0 = (size_t)c.R * c.H * c.d_v * c.d_k;
  const size_t nrow = (size_t)c.T_max * c.R * c.H * c.W_max;
  bool ok = cudaMalloc(&h->S0, nS0 * esize(c.s0_dtype)) == cudaSuccess;
  ok = ok && cudaMalloc(&h->S0f, nS0 * esize(c.s0_dtype)) == cudaSuccess;
  // d0 [2][R], anc_fold [R][T_max], the fold done counters [R].
  ok = ok && cudaMalloc((void **)&h->fold_buf, (size_t)c.R * (3 + c.T_max) * sizeof(int32_t)) == cudaSuccess;
  if (ok && kernel == ONELA_KERNEL_TC)
    ok = cudaMalloc(&h->S0img, onela::s0_image_bytes(c.R, c.H, c.d_k, c.d_v, h->planes)) == cudaSuccess &&
         cudaMalloc(&h->S0fimg[0], onela::s0_image_bytes(c.R, c.H, c.d_k, c.d_v, h->planes)) == cudaSuccess &&
         cudaMalloc(&h->S0fimg[1], onela::s0_image_bytes(c.R, c.H, c.d_k, c.d_v, h->planes)) == cudaSuccess;
  ok = ok && cudaMalloc((void **)&h->rec_alpha, nrow * sizeof(float)) == cudaSuccess;
  if (ok && kernel == ONELA_KERNEL_TC)
    ok = cudaMalloc((void **)&h->par_store, (size_t)c.T_max * c.R * c.W_max * sizeof(int32_t)) == cudaSuccess;
  ok = ok && cudaMalloc((void **)&h->rec_delta, nrow * c.d_v * sizeof(float)) == cudaSuccess;
  ok = ok && cudaMalloc(&h->rec_k, nrow * c.d_k * esize(c.qkv_dtype)) == cudaSuccess;
  ok = ok && cudaMalloc((void **)&h->anc, (size_t)c.T_max * c.R * c.W_max * c.T_max * sizeof(int32_t)) == cudaSuccess;
  ok = ok && cudaHostAlloc((void **)&h->err_host, sizeof(int32_t), cudaHostAllocMapped) == cudaSuccess;
  ok = ok && cudaHostGetDevicePointer((void **)&h->err_dev, h->err_host, 0) == cudaSuccess;
  if (ok) {
    *h->err_host = 0;
    // Zeroed so that nothing uninitialised is ever read, even after a bad parent.
    ok = cudaMemset(h->rec_alpha, 0, nrow * sizeof(float)) == cudaSuccess &&
         (!h->S0fimg[0] ||
          (cudaMemset(h->S0fimg[0], 0, onela::s0_image_bytes(c.R, c.H, c.d_k, c.d_v, h->planes)) == cudaSuccess &&
           cudaMemset(h->S0fimg[1], 0, onela::s0_image_bytes(c.R, c.H, c.d_k, c.d_v, h->planes)) == cudaSuccess)) &&
         cudaMemset(h->anc, 0, (size_t)c.T_max * c.R * c.W_max * c.T_max * sizeof(int32_t)) == cudaSuccess &&
         cudaMemset(h->fold_buf, 0, (size_t)c.R * (3 + c.T_max) * sizeof(int32_t)) == cudaSuccess &&
         cudaDeviceSynchronize() == cudaSuccess;
  }
  if (!ok) {
    cudaGetLastError();
    free_all(h);
    delete h;
    return ONELA_ERR_CUDA;
  }
  *out = h;
  return ONELA_OK;
}

int onela_set_prompt_state(onela_handle *h, const void *S0, onela_stream stream) {
  if (!h || !S0) return ONELA_ERR_ARG;
  DeviceGuard g(h->cfg.device);
  if (!g.ok) return ONELA_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const onela_config &c = h->cfg;
  const size_t bytes = (size_t)c.R * c.H * c.d_v * c.d_k * esize(c.s0_dtype);
  if (cudaMemcpyAsync(h->S0, S0, bytes, cudaMemcpyDeviceToDevice, s) != cudaSuccess) return ONELA_ERR_CUDA;
  if (h->kernel == ONELA_KERNEL_TC) {
    if (onela::launch_s0_image(h->S0, h->S0img, c.R, c.H, c.d_k, c.d_v, c.s0_dtype == ONELA_BF16, h->planes, s) !=
        cudaSuccess)
      return ONELA_ERR_CUDA;
  }
  rewind_to_prompt(h);
  return ONELA_OK;
}

int onela_prefill(onela_handle *h, int32_t L, const void *k, const void *v, const float *gate, const float *beta,
                  onela_stream stream) {
  if (!h || !k || !v || !gate || !beta || L < 1) return ONELA_ERR_ARG;
  DeviceGuard g(h->cfg.device);
  if (!g.ok) return ONELA_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const onela_config &c = h->cfg;
  NvtxRange nvtx(c, "prefill", 0);
  const bool aligned = ((reinterpret_cast<uintptr_t>(k) | reinterpret_cast<uintptr_t>(v)) & 15u) == 0;
  int launches = 1;
  if (h->kernel == ONELA_KERNEL_TC && aligned &&
      onela::prefill_tc_supports(c.d_k, c.d_v, c.qkv_dtype == ONELA_BF16)) {
    // Chunked on the tensor cores.
    const int nseg = onela::prefill_tc_segments(c.R, L, c.H, h->pf_segments);
    const size_t need = onela::prefill_tc_ws_bytes(c.R, L, c.H, c.d_k, nseg);
    if (need > h->pf_ws_bytes) {
      // The old workspace may still be in use by work queued earlier.
      if (h->pf_ws && cudaStreamSynchronize(s) != cudaSuccess) return ONELA_ERR_CUDA;
      cudaFree(h->pf_ws);
      h->pf_ws = nullptr;
      h->pf_ws_bytes = 0;
      if (cudaMalloc(&h->pf_ws, need) != cudaSuccess) {
        cudaGetLastError();
        return ONELA_ERR_CUDA;
      }
      h->pf_ws_bytes = need;
    }
    if (onela::launch_prefill_tc(k, v, gate, beta, h->S0, c.R, L, c.H, c.d_k, c.s0_dtype == ONELA_BF16, nseg,
                                 h->pf_ws, h->wait_limit_ns, h->err_dev, s) != cudaSuccess) {
      cudaGetLastError();
      return ONELA_ERR_CUDA;
    }
    launches = 3;
  } else if (onela::launch_prefill(k, v, gate, beta, h->S0, c.R, L, c.H, c.d_k, c.d_v, c.qkv_dtype == ONELA_BF16,
                                   c.s0_dtype == ONELA_BF16, s) != cudaSuccess) {
    cudaGetLastError();
    return ONELA_ERR_CUDA;
  }
  h->last_launches = launches + (h->kernel == ONELA_KERNEL_TC ? 1 : 0);
  if (h->kernel == ONELA_KERNEL_TC) {
    if (onela::launch_s0_image(h->S0, h->S0img, c.R, c.H, c.d_k, c.d_v, c.s0_dtype == ONELA_BF16, h->planes, s) !=
        cudaSuccess)
      return ONELA_ERR_CUDA;
  }
  rewind_to_prompt(h);
  return ONELA_OK;
}

size_t onela_select_scratch_bytes(int32_t R, int32_t W_prev, int32_t C, int32_t W) {
  if (R < 1 || W_prev < 1 || C < 1 || W < 1) return 0;
  return onela::select_scratch_bytes(R, W_prev, C, W);
}

int onela_select_beams(int32_t R, int32_t W_prev, int32_t C, int32_t W, const float *beam_score, const float *logp,
                       int32_t *parent_idx, int32_t *token, float *score, void *scratch, size_t scratch_bytes,
                       int32_t device, onela_stream stream) {
  if (!beam_score || !logp || !parent_idx || !token || !score || !scratch) return ONELA_ERR_ARG;
  const long long N = (long long)W_prev * C;
  if (R < 1 || R > 65535 || W_prev < 1 || C < 1 || W < 1 || W > 2048 || N < W || N > 0xffffffffLL || device < 0)
    return ONELA_ERR_ARG;
  if (scratch_bytes < onela::select_scratch_bytes(R, W_prev, C, W)) return ONELA_ERR_SCRATCH;
  DeviceGuard g(device);
  if (!g.ok) return ONELA_ERR_CUDA;
  if (onela::launch_select(beam_score, logp, R, W_prev, C, W, parent_idx, token, score, scratch,
                           static_cast<cudaStream_t>(stream)) != cudaSuccess) {
    cudaGetLastError();
    return ONELA_ERR_CUDA;
  }
  return ONELA_OK;
}

int onela_read_prompt_state(onela_handle *h, void *S0, onela_stream stream) {
  if (!h || !S0) return ONELA_ERR_ARG;
  if (!h->has_prompt) return ONELA_ERR_STATE;
  DeviceGuard g(h->cfg.device);
  if (!g.ok) return ONELA_ERR_CUDA;
  const onela_config &c = h->cfg;
  const size_t bytes = (size_t)c.R * c.H * c.d_v * c.d_k * esize(c.s0_dtype);
  if (cudaMemcpyAsync(S0, h->S0, bytes, cudaMemcpyDeviceToDevice, static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return ONELA_ERR_CUDA;
  return ONELA_OK;
}

}  // extern "C"

namespace {

// One decode step.  call_t0 > 0: the step belongs to an onela_decode_steps
// call whose first step is depth call_t0, so the callers' arrays of steps
// call_t0 .. t-1 are still valid, and a later step of the call may overlap
// the step before it (programmatic launch).
int decode_one(onela_handle *h, int32_t W_prev, int32_t W, const void *q, const void *k, const void *v,
               const float *gate, const float *beta, const int32_t *parent_idx, float *o, cudaStream_t s,
               int call_t0) {
  if (!h || !q || !k || !v || !gate || !beta || !parent_idx || !o) return ONELA_ERR_ARG;
  const int rc = word_code(h);
  if (rc != ONELA_OK) return rc;
  if (!h->has_prompt) return ONELA_ERR_STATE;
  const onela_config &c = h->cfg;
  if (W < 1) return ONELA_ERR_ARG;
  // Past T_max steps only with a fold: the device checks that each step's
  // unfolded depths fit the store (kErrWindow otherwise).
  if (W > c.W_max || (h->steps_done >= c.T_max && !h->folded) || h->steps_done >= (1 << 30))
    return ONELA_ERR_CAPACITY;
  const int expect_prev = h->steps_done == 0 ? 1 : h->Ws.back();
  if (W_prev != expect_prev) return ONELA_ERR_ARG;
  DeviceGuard g(c.device);
  if (!g.ok) return ONELA_ERR_CUDA;

  NvtxRange nvtx(c, "step", h->steps_done + 1);
  onela::StepParams p = base_params(h);
  p.W = W;
  p.W_prev = W_prev;
  p.t = h->steps_done + 1;
  p.q = q;
  p.k = k;
  p.v = v;
  p.g = gate;
  p.beta = beta;
  p.parents = parent_idx;
  p.o = o;
  cudaError_t e;
  const bool contract = (c.flags & ONELA_FLAG_PDL) != 0;
  // A step overlaps the step before it under ONELA_FLAG_PDL, or inside one
  // onela_decode_steps call when the depth its early writes replace
  // (t - T_max) is none, or of the same call (then no step still running
  // reads it from the store).  The tensor-core step right after a fold
  // overlaps the fold: it replays from the folded state before that fold
  // (which the fold does not write) where that still fits the record store,
  // and waits for the fold elsewhere (StepParams::after_fold).
  const int tr = p.t - c.T_max;
  const bool in_call = call_t0 > 0 && p.t > call_t0 && (tr < 1 || tr >= call_t0);
  const bool after_fold = h->after_fold && h->fold_pending;  // after the one-launch tensor-core fold
  const bool pdl = p.t >= 2 && (after_fold || (!h->after_fold && (contract || in_call)));
  if (p.t == 1 && h->kernel == ONELA_KERNEL_TC) p.fold_reset = h->fold_buf + (2 + c.T_max) * c.R;
  if (h->fold_pending && h->kernel == ONELA_KERNEL_TC) {
    p.fold_pending = 1;
    p.fold_done = h->fold_buf + (2 + c.T_max) * c.R;
    p.fold_target = h->fold_target;
    p.d0_old = h->fold_prev ? h->fold_buf + (1 - h->fold_cur) * c.R : nullptr;
    p.S0img_old = h->fold_prev ? h->S0fimg[1 - h->fold_cur] : h->S0img;
  }
  if (h->kernel == ONELA_KERNEL_TC) {
    // The tensor-core kernel reads tiles of q, k, v and o with 16-byte accesses.
    const uintptr_t any = reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(k) |
                          reinterpret_cast<uintptr_t>(v) | reinterpret_cast<uintptr_t>(o);
    if (any & 15u) return ONELA_ERR_ARG;
    // The table covers steps hbase .. t-1 (the kernel replays at most
    // T_max - 1 <= 31 of them); the parents of steps hcopy .. t-1 go to
    // shared memory.  Keys, gates and parents of a step come from the
    // caller's arrays while they are valid (ONELA_FLAG_PDL, or a step of
    // this call), else from the record store and the stored parents (those
    // steps have completed).
    // (T_max + 1 <= kHistSteps entries: a step replays at most T_max - 1
    // depths, from depth t - T_max + 1 on)
    p.hbase = p.t - c.T_max > 1 ? p.t - c.T_max : 1;
    p.hcopy = p.t - c.T_max + 1 > 2 ? p.t - c.T_max + 1 : 2;
    if (p.hcopy < p.hbase + 1) p.hcopy = p.hbase + 1;
    p.hist_inputs = 0;
    int hist = 0;
    for (int j = p.hbase; j < p.t; ++j) {
      const int i = j - p.hbase;
      p.hW[i] = h->Ws[j - 1];
      if (contract || (call_t0 > 0 && j >= call_t0)) {
        p.hist_inputs |= 1ull << i;
        p.hk[i] = h->hist_k[j - 1];
        p.hg[i] = h->hist_g[j - 1];
        p.hpar[i] = h->hist_par[j - 1];
        p.hpar_rs[i] = h->Ws[j - 1];
      } else {
        p.hpar[i] = h->par_store + (size_t)((j - 1) % c.T_max) * c.R * c.W_max;
        p.hpar_rs[i] = c.W_max;
      }
      if (j >= p.hcopy) {
        p.hoff[i] = hist;
        hist += (h->Ws[j - 1] + 3) & ~3;
      }
    }
    p.hist_cap = hist <= onela::kHistMaxInts ? hist : 0;
  }
  if (h->kernel == ONELA_KERNEL_TC)
    e = onela::launch_step_tc(p, pdl, s);
  else
    e = onela::launch_step_simt(p, c.qkv_dtype == ONELA_BF16, c.s0_dtype == ONELA_BF16, s);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return ONELA_ERR_CUDA;
  }
  h->steps_done += 1;
  h->after_fold = 0;
  h->last_launches = 1;
  h->Ws.push_back(W);
  h->hist_k.push_back(k);
  h->hist_g.push_back(gate);
  h->hist_par.push_back(parent_idx);
  return ONELA_OK;
}

}  // namespace

extern "C" {

int onela_decode_step(onela_handle *h, int32_t W_prev, int32_t W, const void *q, const void *k, const void *v,
                      const float *gate, const float *beta, const int32_t *parent_idx, float *o,
                      onela_stream stream) {
  return decode_one(h, W_prev, W, q, k, v, gate, beta, parent_idx, o, static_cast<cudaStream_t>(stream), 0);
}

int onela_decode_steps(onela_handle *h, int32_t n, const int32_t *W, const void *const *q, const void *const *k,
                       const void *const *v, const float *const *gate, const float *const *beta,
                       const int32_t *const *parent_idx, float *const *o, onela_stream stream) {
  if (!h || n < 1 || !W || !q || !k || !v || !gate || !beta || !parent_idx || !o) return ONELA_ERR_ARG;
  for (int i = 0; i < n; ++i)
    if (!q[i] || !k[i] || !v[i] || !gate[i] || !beta[i] || !parent_idx[i] || !o[i]) return ONELA_ERR_ARG;
  const int rc = word_code(h);
  if (rc != ONELA_OK) return rc;
  if (!h->has_prompt) return ONELA_ERR_STATE;
  const onela_config &c = h->cfg;
  // Everything that can be checked on the host is checked before the first
  // launch, so an error leaves no work enqueued.
  for (int i = 0; i < n; ++i) {
    if (W[i] < 1) return ONELA_ERR_ARG;
    if (W[i] > c.W_max) return ONELA_ERR_CAPACITY;
  }
  if (((long long)h->steps_done + n > c.T_max && !h->folded) || (long long)h->steps_done + n >= (1 << 30))
    return ONELA_ERR_CAPACITY;
  if (h->kernel == ONELA_KERNEL_TC)
    for (int i = 0; i < n; ++i)
      if ((reinterpret_cast<uintptr_t>(q[i]) | reinterpret_cast<uintptr_t>(k[i]) | reinterpret_cast<uintptr_t>(v[i]) |
           reinterpret_cast<uintptr_t>(o[i])) & 15u)
        return ONELA_ERR_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int call_t0 = h->steps_done + 1;
  for (int i = 0; i < n; ++i) {
    const int Wp = h->steps_done == 0 ? 1 : h->Ws.back();
    const int e = decode_one(h, Wp, W[i], q[i], k[i], v[i], gate[i], beta[i], parent_idx[i], o[i], s, call_t0);
    if (e != ONELA_OK) return e;
  }
  h->last_launches = n;
  return ONELA_OK;
}

int onela_set_wait_policy(onela_handle *h, uint64_t limit_ns, int32_t stall) {
  if (!h || limit_ns < 1000 || limit_ns > 10000000000ull) return ONELA_ERR_ARG;
  h->wait_limit_ns = limit_ns;
  h->stall = stall != 0;
  return ONELA_OK;
}

int onela_set_prefill_segments(onela_handle *h, int32_t segments) {
  if (!h || segments < 0 || segments > onela::kMaxPrefillSegments) return ONELA_ERR_ARG;
  h->pf_segments = segments;
  return ONELA_OK;
}

int onela_reset(onela_handle *h, onela_stream stream) {
  if (!h) return ONELA_ERR_ARG;
  DeviceGuard g(h->cfg.device);
  if (!g.ok) return ONELA_ERR_CUDA;
  // Work still in flight could set the error word after it is cleared.
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return ONELA_ERR_CUDA;
  *reinterpret_cast<volatile int32_t *>(h->err_host) = 0;
  h->steps_done = 0;
  h->folded = 0;
  h->after_fold = 0;
  h->fold_pending = 0;
  h->fold_target = 0;
  h->Ws.clear();
  h->hist_k.clear();
  h->hist_g.clear();
  h->hist_par.clear();
  return ONELA_OK;
}

int onela_fold(onela_handle *h, int32_t max_depth, onela_stream stream) {
  if (!h || max_depth < 0) return ONELA_ERR_ARG;
  const int rc = word_code(h);
  if (rc != ONELA_OK) return rc;
  if (!h->has_prompt) return ONELA_ERR_STATE;
  if (h->steps_done == 0 || max_depth == 0) return ONELA_OK;  // nothing to fold
  DeviceGuard g(h->cfg.device);
  if (!g.ok) return ONELA_ERR_CUDA;
  const onela_config &c = h->cfg;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  onela::StepParams p = base_params(h);
  p.t = h->steps_done;
  const int first = h->folded ? 0 : 1;
  const int32_t *d0_in = h->fold_buf + h->fold_cur * c.R;
  int32_t *d0_out = h->fold_buf + (1 - h->fold_cur) * c.R, *anc_fold = h->fold_buf + 2 * c.R;
  const int depth = max_depth < h->steps_done ? max_depth : h->steps_done;
  NvtxRange nvtx(c, "fold after step", h->steps_done);
  cudaError_t e;
  int pending = 0;
  if (h->kernel == ONELA_KERNEL_TC && c.d_k <= 128 && c.T_max <= onela::kFoldTcMaxT) {
    // Overlaps the step before it, which writes nothing it reads before its
    // wait (never another fold: it reads the folded state before its wait).
    // The new image goes to the other image buffer: the next step may still
    // read the current one.
    const int pdl = !h->after_fold;
    e = onela::launch_fold_tc(p, h->Ws.back(), depth, first, d0_in, d0_out, anc_fold, h->S0f,
                              h->S0fimg[1 - h->fold_cur], c.s0_dtype == ONELA_BF16, pdl,
                              h->fold_buf + (2 + c.T_max) * c.R, s);
    h->fold_target += onela::fold_tc_ctas(p);
    pending = 1;
  } else if (h->kernel == ONELA_KERNEL_TC) {
    // d = 256, or a store of more than kFoldTcMaxT depths: the general
    // fold, then the folded state's operand image.
    e = onela::launch_fold(p, h->Ws.back(), depth, first, d0_in, d0_out, anc_fold, h->S0f,
                           c.qkv_dtype == ONELA_BF16, c.s0_dtype == ONELA_BF16, s);
    if (e == cudaSuccess)
      e = onela::launch_s0_image(h->S0f, h->S0fimg[1 - h->fold_cur], c.R, c.H, c.d_k, c.d_v,
                                 c.s0_dtype == ONELA_BF16, h->planes, s);
  } else {
    e = onela::launch_fold(p, h->Ws.back(), depth, first, d0_in, d0_out, anc_fold, h->S0f,
                           c.qkv_dtype == ONELA_BF16, c.s0_dtype == ONELA_BF16, s);
  }
  if (e != cudaSuccess) {
    cudaGetLastError();
    return ONELA_ERR_CUDA;
  }
  h->fold_cur = 1 - h->fold_cur;
  h->fold_prev = h->folded;
  h->folded = 1;
  h->after_fold = 1;
  h->fold_pending = pending;
  return ONELA_OK;
}

int onela_read_root_state(onela_handle *h, void *S, onela_stream stream) {
  if (!h || !S) return ONELA_ERR_ARG;
  if (!h->has_prompt) return ONELA_ERR_STATE;
  DeviceGuard g(h->cfg.device);
  if (!g.ok) return ONELA_ERR_CUDA;
  const onela_config &c = h->cfg;
  const size_t bytes = (size_t)c.R * c.H * c.d_v * c.d_k * esize(c.s0_dtype);
  if (cudaMemcpyAsync(S, h->folded ? h->S0f : h->S0, bytes, cudaMemcpyDeviceToDevice,
                      static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return ONELA_ERR_CUDA;
  return ONELA_OK;
}

int onela_read_fold_depth(onela_handle *h, int32_t *depth, onela_stream stream) {
  if (!h || !depth) return ONELA_ERR_ARG;
  DeviceGuard g(h->cfg.device);
  if (!g.ok) return ONELA_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t bytes = (size_t)h->cfg.R * sizeof(int32_t);
  const cudaError_t e = h->folded ? cudaMemcpyAsync(depth, h->fold_buf + h->fold_cur * h->cfg.R, bytes,
                                                    cudaMemcpyDeviceToDevice, s)
                                  : cudaMemsetAsync(depth, 0, bytes, s);
  return e == cudaSuccess ? ONELA_OK : ONELA_ERR_CUDA;
}

int onela_status(onela_handle *h, int32_t *device_err) {
  if (!h) return ONELA_ERR_ARG;
  DeviceGuard g(h->cfg.device);
  if (!g.ok) return ONELA_ERR_CUDA;
  if (cudaDeviceSynchronize() != cudaSuccess) return ONELA_ERR_CUDA;
  if (device_err) *device_err = onela::err_bits(*reinterpret_cast<volatile int32_t *>(h->err_host));
  return word_code(h);
}

int onela_destroy(onela_handle *h) {
  if (!h) return ONELA_ERR_ARG;
  {
    DeviceGuard g(h->cfg.device);
    cudaDeviceSynchronize();
    free_all(h);
  }
  delete h;
  return ONELA_OK;
}

int onela_read_records(onela_handle *h, int32_t t, float *alpha, float *delta, void *k, onela_stream stream) {
  if (!h || t < 1 || t > h->steps_done || t <= h->steps_done - h->cfg.T_max) return ONELA_ERR_ARG;
  DeviceGuard g(h->cfg.device);
  if (!g.ok) return ONELA_ERR_CUDA;
  const onela_config &c = h->cfg;
  const int Wt = h->Ws[t - 1];
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t ks = esize(c.qkv_dtype);
  // Rows are [R][H][W_max]: copy the first W_t rows of each (r, h) block.
  const size_t nblk = (size_t)c.R * c.H;
  const size_t base = (size_t)((t - 1) % c.T_max) * nblk * c.W_max;
  bool ok = true;
  if (alpha)
    ok = ok && cudaMemcpy2DAsync(alpha, Wt * sizeof(float), h->rec_alpha + base, (size_t)c.W_max * sizeof(float),
                                 Wt * sizeof(float), nblk, cudaMemcpyDeviceToDevice, s) == cudaSuccess;
  if (delta)
    ok = ok && cudaMemcpy2DAsync(delta, (size_t)Wt * c.d_v * sizeof(float), h->rec_delta + base * c.d_v,
                                 (size_t)c.W_max * c.d_v * sizeof(float), (size_t)Wt * c.d_v * sizeof(float), nblk,
                                 cudaMemcpyDeviceToDevice, s) == cudaSuccess;
  if (k)
    ok = ok && cudaMemcpy2DAsync(k, (size_t)Wt * c.d_k * ks, static_cast<char *>(h->rec_k) + base * c.d_k * ks,
                                 (size_t)c.W_max * c.d_k * ks, (size_t)Wt * c.d_k * ks, nblk,
                                 cudaMemcpyDeviceToDevice, s) == cudaSuccess;
  return ok ? ONELA_OK : ONELA_ERR_CUDA;
}

int onela_read_ancestry(onela_handle *h, int32_t t, int32_t *anc, onela_stream stream) {
  // Whole rows exist only while the depths 1..t-1 fit the row (t <= T_max).
  if (!h || !anc || t < 1 || t > h->steps_done || t > h->cfg.T_max || t <= h->steps_done - h->cfg.T_max)
    return ONELA_ERR_ARG;
  if (t == 1) return ONELA_OK;  // the chain of a depth-1 beam is empty
  DeviceGuard g(h->cfg.device);
  if (!g.ok) return ONELA_ERR_CUDA;
  const onela_config &c = h->cfg;
  const int Wt = h->Ws[t - 1];
  // Source rows [R][W_max][T_max] (t <= T_max: entry j is depth j + 1) ->
  // dest [R][W_t][t-1].
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  for (int r = 0; r < c.R; ++r) {
    const int32_t *src = h->anc + ((size_t)(t - 1) * c.R + r) * c.W_max * c.T_max;
    if (cudaMemcpy2DAsync(anc + (size_t)r * Wt * (t - 1), (t - 1) * sizeof(int32_t), src, c.T_max * sizeof(int32_t),
                          (t - 1) * sizeof(int32_t), Wt, cudaMemcpyDeviceToDevice, s) != cudaSuccess)
      return ONELA_ERR_CUDA;
  }
  return ONELA_OK;
}

int onela_steps_done(const onela_handle *h) { return h ? h->steps_done : -1; }

int onela_kernel_kind(const onela_handle *h) { return h ? h->kernel : -1; }

int onela_last_call_launches(const onela_handle *h) { return h ? h->last_launches : -1; }

}  // extern "C"
