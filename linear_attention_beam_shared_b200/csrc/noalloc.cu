// onela_decode_step_noalloc: a decode step that allocates no device memory.
//
// The handle-based entry points keep the record store, the ancestry index and
// the error word in memory that onela_create obtains with cudaMalloc.  Some
// callers cannot do that: code that runs while a CUDA stream is being
// captured (cudaMalloc is not a stream operation and is refused there), and
// plug-ins hosted by an engine that owns every byte of device memory and hands
// its plug-ins only their input and output tensors.  For them this file keeps
// that state in one fixed, file-scope device array instead, and runs the same
// SIMT decode-step kernel on it.
//
// The array's name is only a host-side stand-in for the device symbol, so the
// host never passes it to a kernel; it asks the runtime for the array's device
// address (cudaGetSymbolAddress) once per device and passes that.
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/onela.h"
#include "internal.h"

namespace {

// 32 MiB, enough for a 7-step decode of 256 beams x 16 heads at d = 128.
constexpr size_t kScratchBytes = (size_t)32 << 20;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_scratch[kScratchBytes];

std::mutex g_mutex;
unsigned char *g_scratch_dev[kMaxDevices] = {nullptr};

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

// Device address of g_scratch on the current device, looked up on the first
// call made with that device current.
cudaError_t scratch_address(int dev, unsigned char **out) {
  std::lock_guard<std::mutex> lock(g_mutex);
  if (!g_scratch_dev[dev]) {
    void *ptr = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&ptr, g_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_dev[dev] = static_cast<unsigned char *>(ptr);
  }
  *out = g_scratch_dev[dev];
  return cudaSuccess;
}

}  // namespace

extern "C" int onela_decode_step_noalloc(const onela_config *cfg, int32_t t, int32_t W_prev, int32_t W,
                                         const void *S0, const void *q, const void *k, const void *v,
                                         const float *gate, const float *beta, const int32_t *parent_idx,
                                         float *o, int32_t *status, onela_stream stream) {
  if (!cfg || !S0 || !q || !k || !v || !gate || !beta || !parent_idx || !o || !status) return ONELA_ERR_ARG;
  const onela_config c = *cfg;
  const bool dt_ok = (c.s0_dtype == ONELA_F32 || c.s0_dtype == ONELA_BF16) &&
                     (c.qkv_dtype == ONELA_F32 || c.qkv_dtype == ONELA_BF16);
  if (c.R < 1 || c.H < 1 || c.d_k < 1 || c.d_k > 256 || c.d_v < 1 || c.d_v > 256 || c.W_max < 1 ||
      c.T_max < 1 || c.T_max > 64 || !dt_ok || c.device < 0 || c.device >= kMaxDevices)
    return ONELA_ERR_ARG;
  if (t < 1 || t > c.T_max || W < 1 || W > c.W_max || W_prev < 1 || W_prev > c.W_max || (t == 1 && W_prev != 1))
    return ONELA_ERR_ARG;

  // Scratch layout: error word, ancestry rows, then the records of depths
  // 1..T_max (the same row layout the handle uses).
  const size_t esz = c.qkv_dtype == ONELA_BF16 ? 2 : 4;
  const double rows = (double)c.T_max * c.R * c.H * c.W_max;
  const double need_d = 256.0 + (double)c.T_max * c.R * c.W_max * c.T_max * 4 + rows * 4 + rows * c.d_v * 4 +
                        rows * c.d_k * esz + 4 * 256.0;
  if (need_d > (double)kScratchBytes) return ONELA_ERR_SCRATCH;
  const size_t nrow = (size_t)c.T_max * c.R * c.H * c.W_max;
  const size_t off_anc = 256;
  const size_t off_alpha = off_anc + align256((size_t)c.T_max * c.R * c.W_max * c.T_max * 4);
  const size_t off_delta = off_alpha + align256(nrow * 4);
  const size_t off_k = off_delta + align256(nrow * c.d_v * 4);

  int prev = -1;
  if (cudaGetDevice(&prev) != cudaSuccess) return ONELA_ERR_CUDA;
  if (prev != c.device && cudaSetDevice(c.device) != cudaSuccess) return ONELA_ERR_CUDA;
  int rc = ONELA_OK;
  unsigned char *base = nullptr;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (scratch_address(c.device, &base) != cudaSuccess) {
    rc = ONELA_ERR_CUDA;
  } else {
    int32_t *err = reinterpret_cast<int32_t *>(base);
    onela::StepParams p{};
    p.R = c.R;
    p.H = c.H;
    p.dk = c.d_k;
    p.dv = c.d_v;
    p.W = W;
    p.W_prev = W_prev;
    p.t = t;
    p.W_max = c.W_max;
    p.T_max = c.T_max;
    p.q = q;
    p.k = k;
    p.v = v;
    p.g = gate;
    p.beta = beta;
    p.parents = parent_idx;
    p.o = o;
    p.S0 = S0;
    p.S0img = nullptr;
    p.s0_planes = 1;
    p.anc = reinterpret_cast<int32_t *>(base + off_anc);
    p.rec_alpha = reinterpret_cast<float *>(base + off_alpha);
    p.rec_delta = reinterpret_cast<float *>(base + off_delta);
    p.rec_k = base + off_k;
    p.err = err;
    // The error word must start at zero for a new decode; later steps keep
    // (and report) what earlier steps of the decode set.
    bool ok = t != 1 || cudaMemsetAsync(err, 0, sizeof(int32_t), s) == cudaSuccess;
    ok = ok && onela::launch_step_simt(p, c.qkv_dtype == ONELA_BF16, c.s0_dtype == ONELA_BF16, s) == cudaSuccess;
    ok = ok && cudaMemcpyAsync(status, err, sizeof(int32_t), cudaMemcpyDeviceToDevice, s) == cudaSuccess;
    if (!ok) {
      cudaGetLastError();
      rc = ONELA_ERR_CUDA;
    }
  }
  if (prev != c.device) cudaSetDevice(prev);
  return rc;
}
