// Folding a shared ancestor prefix into the root state: an extension of the
// method.  The evolve.pub review's Summary counts a replay cost that grows
// with depth among the limitations, and its Weaknesses list replay depth as
// unanalysed beyond small T: every ancestor's record is replayed at every
// step, so a beam at depth t replays t - 1 records.
//
// Once every beam of a request descends from one beam c at depth D, the
// records of c's chain (depths 1..D) are replayed identically by all of them.
// Folding replaces the root state by c's full state,
//     S_c = alpha_D S_{D-1} + delta_D k_D^T,  S_0 = the prompt state,
// (the recurrence of the review's section 3.2 equations), after which the
// decode kernels replay only depths D+1..t-1.  Nothing else changes: the
// record store, the ancestry rows and the outputs stay those of the
// unfolded decode, up to the rounding of S_c to the state's storage type.
// Since only the unfolded depths are read, a decode that keeps folding can
// run past the T_max depths the record store keeps.
//
// The folded depth of each request is double-buffered (d0_in is read, d0_out
// written), so that every CTA of a launch sees the same previous depth.
//
// Tensor-core handles: one launch, fold_tc_kernel.  Each CTA takes a block
// of state rows of one (request, head): it loads its part of the state the
// fold starts from (before waiting on the previous kernel, under
// programmatic launch), finds the shared depth D itself (every CTA of the
// request reads the same ancestry rows and agrees), stages the newly folded
// records (alpha, its rows of delta, k) in shared memory, runs the
// recurrence and writes the folded state and its bf16 operand image for the
// tensor-core decode kernel.
//
// General handles: two ordinary launches,
//   fold_plan_kernel   one CTA per request: D and the ancestors of the newly
//                      folded depths;
//   fold_state_kernel  one thread per state element: the recurrence.
// Both run the recurrence in fp32 as S <- fma(delta_i, k_j, alpha S).
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "internal.h"
#include "sm100_ptx.h"

namespace onela {
namespace {

constexpr int kPlanThreads = 256;
constexpr int kFoldThreads = 256;
constexpr int kFoldMaxT = kFoldTcMaxT;  // deepest decode of the one-launch fold
constexpr int kImgRows = 128;  // rows of an operand image atom

__device__ __forceinline__ float ldf(const float *p, int64_t i) { return p[i]; }
__device__ __forceinline__ float ldf(const __nv_bfloat16 *p, int64_t i) { return __bfloat162float(p[i]); }
__device__ __forceinline__ void stf(float *p, int64_t i, float x) { p[i] = x; }
__device__ __forceinline__ void stf(__nv_bfloat16 *p, int64_t i, float x) { p[i] = __float2bfloat16_rn(x); }

__global__ void __launch_bounds__(kPlanThreads) fold_plan_kernel(const StepParams p, int Wt, int max_depth, int first,
                                                                 const int32_t *d0_in, int32_t *d0_out,
                                                                 int32_t *anc_fold) {
  __shared__ int s_split;  // smallest row index at which two beams differ
  const int r = blockIdx.x, tid = threadIdx.x, t = p.t, TM = p.T_max;
  const int old = first ? 0 : d0_in[r];
  const int n = t - 1;  // ancestry entries of a step-t beam (depths 1..t-1)
  if (tid == 0) s_split = n;
  __syncthreads();
  const int32_t *row0 = p.anc + anc_row(p, t, r, 0);
  // Depths old + 1 .. n can be newly shared; depth j + 1 sits in entry
  // j mod T_max of the rows.
  const int nw = n - old;
  for (int e = tid; e < (Wt - 1) * nw; e += kPlanThreads) {
    const int b = 1 + e / nw, j = old + e - (b - 1) * nw;
    if (p.anc[anc_row(p, t, r, b) + j % TM] != row0[j % TM]) atomicMin(&s_split, j);
  }
  __syncthreads();
  // Sharing an ancestor at a depth implies sharing its ancestors, so the
  // shared depths are 1..s_split; a step that kept one beam shares it too.
  int D = s_split;
  if (D == n && Wt == 1) D = t;
  if (D > max_depth) D = max_depth;
  if (D < old) D = old;
  for (int j = old + tid; j < D; j += kPlanThreads) anc_fold[(int64_t)r * TM + j % TM] = j < n ? row0[j % TM] : 0;
  if (tid == 0) d0_out[r] = D;
}

template <typename QT, typename ST>
__global__ void __launch_bounds__(kFoldThreads) fold_state_kernel(const StepParams p, int first, ST *S_fold,
                                                                  const int32_t *d0_in, const int32_t *d0_out,
                                                                  const int32_t *anc_fold) {
  const int h = blockIdx.y, r = blockIdx.z;
  const int from = first ? 0 : d0_in[r], D = d0_out[r];
  if (!first && from == D) return;  // unchanged: S_fold already holds it
  const int dk = p.dk, dv = p.dv;
  const int64_t e = (int64_t)blockIdx.x * kFoldThreads + threadIdx.x;
  if (e >= (int64_t)dv * dk) return;
  const int i = (int)(e / dk), j = (int)(e - (int64_t)i * dk);
  const int64_t idx = ((int64_t)r * p.H + h) * dv * dk + e;
  const ST *src = first ? static_cast<const ST *>(p.S0) : S_fold;
  float s = ldf(src, idx);
  const QT *rec_k = static_cast<const QT *>(p.rec_k);
#pragma unroll 1
  for (int d = from + 1; d <= D; ++d) {
    const int64_t row = rec_row(p, d, r, h, anc_fold[(int64_t)r * p.T_max + (d - 1) % p.T_max]);
    const float a = p.rec_alpha[row];
    s = fmaf(p.rec_delta[row * dv + i], ldf(rec_k, row * dk + j), a * s);
  }
  stf(S_fold, idx, s);
}

template <typename QT, typename ST>
cudaError_t launch_state(const StepParams &p, int first, void *S_fold, const int32_t *d0_in, const int32_t *d0_out,
                         const int32_t *anc_fold, cudaStream_t s) {
  const int64_t n = (int64_t)p.dv * p.dk;
  const dim3 grid((unsigned)((n + kFoldThreads - 1) / kFoldThreads), p.H, p.R);
  fold_state_kernel<QT, ST><<<grid, kFoldThreads, 0, s>>>(p, first, static_cast<ST *>(S_fold), d0_in, d0_out,
                                                          anc_fold);
  return cudaGetLastError();
}

// 8 consecutive state elements (16- or 32-byte aligned) to and from fp32.
__device__ __forceinline__ void ld8(const float *p, float (&x)[8]) {
  const float4 a = reinterpret_cast<const float4 *>(p)[0], b = reinterpret_cast<const float4 *>(p)[1];
  x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w; x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
}
__device__ __forceinline__ void ld8(const __nv_bfloat16 *p, float (&x)[8]) {
  const uint4 a = *reinterpret_cast<const uint4 *>(p);
  const __nv_bfloat162 *h2 = reinterpret_cast<const __nv_bfloat162 *>(&a);
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const float2 f = __bfloat1622float2(h2[u]);
    x[2 * u] = f.x;
    x[2 * u + 1] = f.y;
  }
}
// Stores x in the state's type; x becomes the stored value.
__device__ __forceinline__ void st8(float *p, float (&x)[8]) {
  reinterpret_cast<float4 *>(p)[0] = make_float4(x[0], x[1], x[2], x[3]);
  reinterpret_cast<float4 *>(p)[1] = make_float4(x[4], x[5], x[6], x[7]);
}
__device__ __forceinline__ void st8(__nv_bfloat16 *p, float (&x)[8]) {
  __align__(16) __nv_bfloat16 o[8];
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    o[u] = __float2bfloat16_rn(x[u]);
    x[u] = __bfloat162float(o[u]);
  }
  *reinterpret_cast<uint4 *>(p) = *reinterpret_cast<const uint4 *>(o);
}

// One launch: plan, recurrence, folded state and its operand image.  Block:
// kFoldThreads threads, DK / 8 per state row (8 columns each), so RB rows.
// After the wait on the previous kernel, two rounds of loads: the ancestry
// rows (beam 0's and each thread's beams'), then the records of every depth
// that may be folded (the shared depth is known only once the rows are
// compared; records past it are loaded and not used).
template <typename ST, int DK>
__global__ void __launch_bounds__(kFoldThreads) fold_tc_kernel(const StepParams p, int Wt, int max_depth, int first,
                                                               const int32_t *d0_in, int32_t *d0_out,
                                                               int32_t *anc_fold, ST *S_fold, uint4 *img, int *done) {
  constexpr int TPR = DK / 8, RB = kFoldThreads / TPR, NK = DK / 64;
  constexpr int KC = DK / 8, DC = RB / 4, PER = KC + DC + 1;  // 16-byte record pieces per depth
  constexpr int MAXI = (kFoldMaxT * PER + kFoldThreads - 1) / kFoldThreads;
  __shared__ int s_split;
  __shared__ int s_row0[kFoldMaxT];  // beam 0's ancestry row (entry j: depth j + 1 mod T_max)
  __shared__ float s_a[kFoldMaxT];
  __shared__ __align__(16) float s_d[kFoldMaxT][RB];
  __shared__ __align__(16) __nv_bfloat16 s_k[kFoldMaxT][DK];
  const int h = blockIdx.y, r = blockIdx.z, tid = threadIdx.x;
  const int dv = p.dv, t = p.t, n = t - 1, TM = p.T_max;
  const int i0 = blockIdx.x * RB, ir = tid / TPR, c = tid - ir * TPR, i = i0 + ir;
  const bool valid = i < dv;
  const int64_t rh = (int64_t)r * p.H + h;
  const int64_t si = (rh * dv + i) * DK + c * 8;

  // The state the fold starts from: the prompt state (read before the wait
  // on the previous kernel), or the folded state of an earlier fold, which
  // may still be running until the kernel before this one is complete.
  float x[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  if (valid && first) ld8(static_cast<const ST *>(p.S0) + si, x);
  if (tid == 0) s_split = n;
  // The ancestry rows and records of step t come from the previous kernel.
  ptx::pdl_wait();
  // The next step may start: it reads what this kernel writes only once the
  // fold's CTAs have counted themselves done (StepParams::fold_done).
  ptx::pdl_launch_dependents();
  if (valid && !first) ld8(S_fold + si, x);
  const int old = first ? 0 : d0_in[r];
  // Depths that can be folded: old + 1 .. Dmax (depth t only when step t
  // kept a single beam, its own record).
  const int jhi = min(n, max_depth);
  // (at most T_max of them: more only after a step reported kErrWindow)
  const int Dmax = max(old, min(min(max_depth, Wt == 1 ? t : n), old + TM));
  const int32_t *row0 = p.anc + anc_row(p, t, r, 0);
  if (tid < min(n, TM)) s_row0[tid] = row0[tid];
  // Entry w of v and w0: depth old + w + 1 (at most T_max - 1 depths can be
  // newly shared, as the step replayed them).
  int v[kFoldMaxT], w0[kFoldMaxT];
  const int b = 1 + tid;  // Wt <= kFoldThreads + 1 here; more beams: the loop below
  if (b < Wt) {
    const int32_t *row = p.anc + anc_row(p, t, r, b);
#pragma unroll
    for (int w = 0; w < kFoldMaxT; ++w) {
      const int j = old + w;
      v[w] = j < jhi ? row[j % TM] : 0;
      w0[w] = j < jhi ? row0[j % TM] : 0;
    }
  }
  __syncthreads();  // s_row0
  // Round two, issued before the comparisons wait for round one.
  uint4 piece[MAXI];
  const int nitems = (Dmax - old) * PER;
#pragma unroll
  for (int m = 0; m < MAXI; ++m) {
    const int e = tid + m * kFoldThreads;
    piece[m] = make_uint4(0u, 0u, 0u, 0u);
    if (e < nitems) {
      const int dd = e / PER, q = e - dd * PER, d = old + dd + 1;
      const int64_t row = rec_row(p, d, r, h, d - 1 < n ? s_row0[(d - 1) % TM] : 0);
      if (q < KC)
        piece[m] = *reinterpret_cast<const uint4 *>(static_cast<const __nv_bfloat16 *>(p.rec_k) + row * DK + q * 8);
      else if (q < KC + DC)
        piece[m] = *reinterpret_cast<const uint4 *>(p.rec_delta + row * dv + i0 + (q - KC) * 4);
      else
        piece[m].x = __float_as_uint(p.rec_alpha[row]);
    }
  }
  int split = n;
  if (b < Wt) {
#pragma unroll
    for (int w = kFoldMaxT - 1; w >= 0; --w)
      if (old + w < jhi && v[w] != w0[w]) split = old + w;
  }
  for (int bb = b + kFoldThreads; bb < Wt; bb += kFoldThreads) {
    const int32_t *row = p.anc + anc_row(p, t, r, bb);
    for (int j = old; j < jhi; ++j)
      if (row[j % TM] != s_row0[j % TM]) {
        split = min(split, j);
        break;
      }
  }
  if (split < n) atomicMin(&s_split, split);
#pragma unroll
  for (int m = 0; m < MAXI; ++m) {
    const int e = tid + m * kFoldThreads;
    if (e < nitems) {
      const int dd = e / PER, q = e - dd * PER;
      if (q < KC)
        *reinterpret_cast<uint4 *>(&s_k[dd][q * 8]) = piece[m];
      else if (q < KC + DC)
        *reinterpret_cast<uint4 *>(&s_d[dd][(q - KC) * 4]) = piece[m];
      else
        s_a[dd] = __uint_as_float(piece[m].x);
    }
  }
  __syncthreads();
  // Sharing an ancestor at a depth implies sharing its ancestors, so the
  // shared depths are 1..s_split; a step that kept one beam shares it too.
  int D = s_split;
  if (D == n && Wt == 1) D = t;
  if (D > max_depth) D = max_depth;
  if (D > Dmax) D = Dmax;
  if (D < old) D = old;
  if (blockIdx.x == 0 && h == 0) {
    for (int j = old + tid; j < D; j += kFoldThreads) anc_fold[(int64_t)r * TM + j % TM] = j < n ? s_row0[j % TM] : 0;
    if (tid == 0) d0_out[r] = D;
  }
  // Unchanged (D == old) the state is stored back as it is: its image goes
  // to the other image buffer all the same.
  if (valid) {
#pragma unroll 1
    for (int dd = 0; dd < D - old; ++dd) {
      const float a = s_a[dd], dl = s_d[dd][ir];
      const uint4 kq = *reinterpret_cast<const uint4 *>(&s_k[dd][c * 8]);
      const __nv_bfloat162 *k2 = reinterpret_cast<const __nv_bfloat162 *>(&kq);
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const float2 kf = __bfloat1622float2(k2[u]);
        x[2 * u] = fmaf(dl, kf.x, a * x[2 * u]);
        x[2 * u + 1] = fmaf(dl, kf.y, a * x[2 * u + 1]);
      }
    }
    st8(S_fold + si, x);
    // The operand image: plane pl holds the bf16 term pl of the split of the
    // stored value (hi, then the bf16 rounding of what is left, ...).
    const int planes = p.s0_planes, ka = c >> 3, cc = c & 7;
    float rest[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) rest[u] = x[u];
    for (int pl = 0; pl < planes; ++pl) {
      __align__(16) __nv_bfloat16 o[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        o[u] = __float2bfloat16_rn(rest[u]);
        rest[u] = rest[u] - __bfloat162float(o[u]);
      }
      const int64_t off = ((rh * planes + pl) * NK + ka) * (kImgRows * 128) + ptx::swz128(i, cc);
      img[off / 16] = *reinterpret_cast<const uint4 *>(o);
    }
  }
  // This CTA's part of request r is written.
  __syncthreads();
  if (tid == 0) {
    __threadfence();
    ptx::red_release_add_gpu(done + r, 1);
  }
}

template <typename ST, int DK>
cudaError_t launch_tc(const StepParams &p, int Wt, int max_depth, int first, const int32_t *d0_in, int32_t *d0_out,
                      int32_t *anc_fold, void *S_fold, void *img, int pdl, int *done, cudaStream_t s) {
  constexpr int RB = kFoldThreads / (DK / 8);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((p.dv + RB - 1) / RB, p.H, p.R);
  cfg.blockDim = dim3(kFoldThreads, 1, 1);
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, fold_tc_kernel<ST, DK>, p, Wt, max_depth, first, d0_in, d0_out, anc_fold,
                            static_cast<ST *>(S_fold), static_cast<uint4 *>(img), done);
}

bool fold_args_ok(const StepParams &p, int Wt, int max_depth) {
  return p.t >= 1 && Wt >= 1 && Wt <= p.W_max && max_depth >= 0 && max_depth <= p.t && p.R >= 1 && p.R <= 65535 &&
         p.H <= 65535;
}

}  // namespace

cudaError_t launch_fold(const StepParams &p, int Wt, int max_depth, int first, const int32_t *d0_in, int32_t *d0_out,
                        int32_t *anc_fold, void *S_fold, int qkv_bf16, int s0_bf16, cudaStream_t s) {
  if (!fold_args_ok(p, Wt, max_depth)) return cudaErrorInvalidValue;
  fold_plan_kernel<<<p.R, kPlanThreads, 0, s>>>(p, Wt, max_depth, first, d0_in, d0_out, anc_fold);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (qkv_bf16)
    return s0_bf16 ? launch_state<__nv_bfloat16, __nv_bfloat16>(p, first, S_fold, d0_in, d0_out, anc_fold, s)
                   : launch_state<__nv_bfloat16, float>(p, first, S_fold, d0_in, d0_out, anc_fold, s);
  return s0_bf16 ? launch_state<float, __nv_bfloat16>(p, first, S_fold, d0_in, d0_out, anc_fold, s)
                 : launch_state<float, float>(p, first, S_fold, d0_in, d0_out, anc_fold, s);
}

int fold_tc_ctas(const StepParams &p) {
  const int RB = kFoldThreads / (p.dk / 8);
  return (p.dv + RB - 1) / RB * p.H;
}

cudaError_t launch_fold_tc(const StepParams &p, int Wt, int max_depth, int first, const int32_t *d0_in,
                           int32_t *d0_out, int32_t *anc_fold, void *S_fold, void *img, int s0_bf16, int pdl,
                           int *done, cudaStream_t s) {
  if (!fold_args_ok(p, Wt, max_depth) || p.T_max > kFoldMaxT || p.dk != p.dv || p.s0_planes < 1 ||
      p.s0_planes > 3)
    return cudaErrorInvalidValue;
  if (p.dk == 64)
    return s0_bf16 ? launch_tc<__nv_bfloat16, 64>(p, Wt, max_depth, first, d0_in, d0_out, anc_fold, S_fold, img, pdl, done, s)
                   : launch_tc<float, 64>(p, Wt, max_depth, first, d0_in, d0_out, anc_fold, S_fold, img, pdl, done, s);
  if (p.dk == 128)
    return s0_bf16 ? launch_tc<__nv_bfloat16, 128>(p, Wt, max_depth, first, d0_in, d0_out, anc_fold, S_fold, img, pdl, done, s)
                   : launch_tc<float, 128>(p, Wt, max_depth, first, d0_in, d0_out, anc_fold, S_fold, img, pdl, done, s);
  return cudaErrorInvalidValue;
}

}  // namespace onela
