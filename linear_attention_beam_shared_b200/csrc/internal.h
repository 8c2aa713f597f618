// Internal declarations shared by the runtime and the decode kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace onela {

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
  // Parents of the previous step (step t-1), [R][prev_stride] with W_prev
  // valid entries per request, and the beam count of step t-2 (W_prev2).
  // Used by the tensor-core kernel for t >= 3; may be null otherwise.
  const int32_t *prev_parents;
  int prev_stride, W_prev2;
  int32_t *par_store;     // [T_max][R][W_max]: each step's parents (tensor-core kernel)
  float *o;               // [R][W][H][dv]
  const void *S0;         // [R][H][dv][dk] in the S0 type
  const void *S0img;      // tensor-core operand image of S0 (see step_tc.cu)
  int s0_planes;          // bf16 terms in S0img (1 for bf16 S0)
  float *rec_alpha;       // [T_max][R][H][W_max]
  float *rec_P;           // [T_max][R][H][W_max]: product of the gates on the
                          // path from the root to the record, inclusive
                          // (tensor-core kernel only; may be null otherwise)
  float *rec_delta;       // [T_max][R][H][W_max][dv]
  void *rec_k;            // [T_max][R][H][W_max][dk] in the qkv type
  int32_t *anc;           // [T_max][R][W_max][T_max]
  int32_t *err;           // host-mapped error word (device view)
  // TMA descriptors of k and q (tensor-core kernel; encoded per call):
  // 4-D {d_k, H, W, R} bf16, box {64, 1, 32, 1}, 128-byte swizzle.
  alignas(64) CUtensorMap tm_k;
  alignas(64) CUtensorMap tm_q;
};

// Row index of the record of beam b, head h, request r at depth s (1-based).
__host__ __device__ __forceinline__ int64_t rec_row(const StepParams &p, int s, int r, int h, int b) {
  return ((int64_t)((s - 1) * p.R + r) * p.H + h) * p.W_max + b;
}
// First entry of the ancestry row of beam b, request r, at depth s (1-based).
__host__ __device__ __forceinline__ int64_t anc_row(const StepParams &p, int s, int r, int b) {
  return ((int64_t)((s - 1) * p.R + r) * p.W_max + b) * p.T_max;
}

// Device error word bits.
constexpr int32_t kErrParent = 1;

// Kernel launchers (step_simt.cu, step_tc.cu).  Return a cudaError_t.
cudaError_t launch_step_simt(const StepParams &p, int qkv_bf16, int s0_bf16, cudaStream_t s);
cudaError_t launch_step_tc(const StepParams &p, int pdl, cudaStream_t s);
cudaError_t launch_s0_image(const void *S0, void *img, int R, int H, int dk, int dv,
                            int s0_bf16, int planes, cudaStream_t s);
size_t s0_image_bytes(int R, int H, int dk, int dv, int planes);
bool tc_supports(int dk, int dv, int qkv_bf16, int T_max, int W_max);

}  // namespace onela
