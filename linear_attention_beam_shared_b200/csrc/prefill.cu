// Prefill: the prompt-derived state S0 of every (request, head), built on the
// device (the one state all beams share, OneLA abstract; the recurrence is
// the GDN update of the evolve.pub review's key claims on section 3.2,
// equation 2):
//
//   S_l = alpha_l S_{l-1} + delta_l k_l^T,   delta_l = beta_l (v_l - alpha_l S_{l-1} k_l),
//
// from S_0 = 0 over the L prompt tokens, in fp32.
//
// Row i of S evolves on its own: u_i = S[i,:] . k_l uses only row i, and
// the update of row i needs only delta_i.  So one CTA takes 16 rows of one
// (request, head) (small blocks spread the heads over every SM); each row is
// held in the registers of 8 threads (EPT consecutive elements each), and
// per token the 8 threads form their partial dot product, sum it in 3
// shuffles, and update their elements, with the next token's operands
// already on their way from shared memory.  The tokens'
// k, v, gate and beta stream through shared memory in chunks of kTC tokens
// (cp.async, double-buffered); the gates of a chunk become alpha = exp(g)
// once per token, not once per thread.
#include <cuda_bf16.h>

#include "internal.h"
#include "sm100_ptx.h"

namespace onela {
namespace {

constexpr int kRB = 16;       // rows of S per CTA
constexpr int kTPR = 8;       // threads per row
constexpr int kPThreads = kRB * kTPR;
constexpr int kTC = 32;       // tokens per staged chunk

template <typename T> __device__ __forceinline__ float to_f(T x);
template <> __device__ __forceinline__ float to_f<float>(float x) { return x; }
template <> __device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }

// EPT consecutive elements at p (16-byte aligned) as floats.
template <typename T, int EPT>
__device__ __forceinline__ void load_row_part(float (&kk)[EPT], const T *p) {
  if constexpr (sizeof(T) == 4) {
#pragma unroll
    for (int e = 0; e < EPT; e += 4) {
      const float4 x = *reinterpret_cast<const float4 *>(p + e);
      kk[e] = x.x, kk[e + 1] = x.y, kk[e + 2] = x.z, kk[e + 3] = x.w;
    }
  } else {
#pragma unroll
    for (int e = 0; e < EPT; e += 8) {
      const uint4 x = *reinterpret_cast<const uint4 *>(p + e);
      const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&w[q]));
        kk[e + 2 * q] = f.x, kk[e + 2 * q + 1] = f.y;
      }
    }
  }
}

// Shared memory of one chunk buffer: k [kTC][DKP] and v [kTC][kRB] in the
// input type, g and beta [kTC] fp32, alpha [kTC] fp32.
template <typename T, int DKP>
struct __align__(16) ChunkBuf {
  T k[kTC][DKP];
  T v[kTC][kRB];
  float g[kTC];
  float beta[kTC];
  float alpha[kTC];
};

// Copies chunk [l0, l0 + n) of the prompt of (r, h) into buf: 16-byte pieces
// where the rows allow it, 4-byte pieces otherwise; tokens past n are zeros
// (never used).
template <typename T, int DKP>
__device__ void stage_chunk(ChunkBuf<T, DKP> &buf, const T *k, const T *v, const float *g, const float *beta,
                            int R, int L, int H, int dk, int dv, int r, int h, int row0, int l0, int n, int tid) {
  constexpr int ES = (int)sizeof(T);
  // k rows: dk elements, contiguous in [R][L][H][dk].
  const int kb = dk * ES;  // bytes of a k row
  if ((kb & 15) == 0 && ((reinterpret_cast<uintptr_t>(k) & 15) == 0)) {
    const int pr = kb / 16;
    for (int e = tid; e < n * pr; e += kPThreads) {
      const int tl = e / pr, c = e - tl * pr;
      const T *src = k + ((int64_t)(r * L + l0 + tl) * H + h) * dk;
      ptx::cp_async16(reinterpret_cast<uint8_t *>(&buf.k[tl][0]) + c * 16, reinterpret_cast<const uint8_t *>(src) + c * 16,
                      16u);
    }
  } else {
    for (int e = tid; e < n * dk; e += kPThreads) {
      const int tl = e / dk, c = e - tl * dk;
      buf.k[tl][c] = k[((int64_t)(r * L + l0 + tl) * H + h) * dk + c];
    }
  }
  // v: this CTA's rows of each token (16-byte pieces when the row segments
  // allow it, 4-byte ones for fp32, plain copies otherwise).
  const int nr = min(kRB, dv - row0);
  const bool v16 = ((dv * ES) & 15) == 0 && ((nr * ES) & 15) == 0 && ((row0 * ES) & 15) == 0 &&
                   (reinterpret_cast<uintptr_t>(v) & 15) == 0;
  if (v16) {
    const int pr = nr * ES / 16;
    for (int e = tid; e < n * pr; e += kPThreads) {
      const int tl = e / pr, c = e - tl * pr;
      const T *src = v + ((int64_t)(r * L + l0 + tl) * H + h) * dv + row0;
      ptx::cp_async16(reinterpret_cast<uint8_t *>(&buf.v[tl][0]) + c * 16, reinterpret_cast<const uint8_t *>(src) + c * 16,
                      16u);
    }
  } else {
    for (int e = tid; e < n * nr; e += kPThreads) {
      const int tl = e / nr, c = e - tl * nr;
      const T *src = v + ((int64_t)(r * L + l0 + tl) * H + h) * dv + row0 + c;
      if constexpr (ES == 4)
        ptx::cp_async4(&buf.v[tl][c], src);
      else
        buf.v[tl][c] = *src;
    }
  }
  for (int e = tid; e < n; e += kPThreads) {
    const int64_t si = (int64_t)(r * L + l0 + e) * H + h;
    ptx::cp_async4(&buf.g[e], g + si);
    ptx::cp_async4(&buf.beta[e], beta + si);
  }
}

template <typename T, typename TS, int EPT>
__global__ void __launch_bounds__(kPThreads) prefill_kernel(const T *k, const T *v, const float *g, const float *beta,
                                                            TS *S0, int R, int L, int H, int dk, int dv) {
  constexpr int DKP = EPT * kTPR;  // padded key width
  extern __shared__ __align__(16) uint8_t psmem[];
  ChunkBuf<T, DKP> *bufs = reinterpret_cast<ChunkBuf<T, DKP> *>(psmem);
  const int row0 = blockIdx.x * kRB, h = blockIdx.y, r = blockIdx.z;
  const int tid = threadIdx.x, rr = tid / kTPR, part = tid % kTPR;
  const int row = row0 + rr;
  // Zero the padding of the k rows once in both buffers (never written by the copies).
  for (int e = tid; e < 2 * kTC * DKP; e += kPThreads) {
    const int b = e / (kTC * DKP), x = e - b * (kTC * DKP), c = x % DKP;
    if (c >= dk) bufs[b].k[x / DKP][c] = T(0.f);
  }
  float s[EPT];
#pragma unroll
  for (int e = 0; e < EPT; ++e) s[e] = 0.f;

  const int nchunks = (L + kTC - 1) / kTC;
  stage_chunk<T, DKP>(bufs[0], k, v, g, beta, R, L, H, dk, dv, r, h, row0, 0, min(kTC, L), tid);
  ptx::cp_async_commit();
#pragma unroll 1
  for (int c = 0; c < nchunks; ++c) {
    ChunkBuf<T, DKP> &cur = bufs[c & 1];
    const int n = min(kTC, L - c * kTC);
    if (c + 1 < nchunks)
      stage_chunk<T, DKP>(bufs[(c + 1) & 1], k, v, g, beta, R, L, H, dk, dv, r, h, row0, (c + 1) * kTC,
                          min(kTC, L - (c + 1) * kTC), tid);
    ptx::cp_async_commit();
    ptx::cp_async_wait_group1();
    __syncthreads();
    if (tid < n) cur.alpha[tid] = expf(cur.g[tid]);
    __syncthreads();
    // The next token's operands are loaded while this token's sum is reduced.
    float kk[EPT];
    load_row_part<T, EPT>(kk, &cur.k[0][part * EPT]);
    float a = cur.alpha[0], bt = cur.beta[0], vi = row < dv ? to_f(cur.v[0][rr]) : 0.f;
#pragma unroll 1
    for (int tl = 0; tl < n; ++tl) {
      float p0 = 0.f, p1 = 0.f, p2 = 0.f, p3 = 0.f;
#pragma unroll
      for (int e = 0; e < EPT; e += 4) {
        p0 = fmaf(s[e], kk[e], p0);
        p1 = fmaf(s[e + 1], kk[e + 1], p1);
        p2 = fmaf(s[e + 2], kk[e + 2], p2);
        p3 = fmaf(s[e + 3], kk[e + 3], p3);
      }
      float u = (p0 + p1) + (p2 + p3);
      float kn[EPT];
      const int tn = tl + 1 < n ? tl + 1 : tl;
      load_row_part<T, EPT>(kn, &cur.k[tn][part * EPT]);
      const float an = cur.alpha[tn], bn = cur.beta[tn], vn = row < dv ? to_f(cur.v[tn][rr]) : 0.f;
      u += __shfl_xor_sync(0xffffffffu, u, 1);
      u += __shfl_xor_sync(0xffffffffu, u, 2);
      u += __shfl_xor_sync(0xffffffffu, u, 4);
      const float delta = bt * (vi - a * u);
#pragma unroll
      for (int e = 0; e < EPT; ++e) s[e] = fmaf(a, s[e], delta * kk[e]);
#pragma unroll
      for (int e = 0; e < EPT; ++e) kk[e] = kn[e];
      a = an, bt = bn, vi = vn;
    }
    __syncthreads();  // this buffer is refilled by the copies of the chunk after next
  }
  if (row < dv) {
    TS *out = S0 + ((int64_t)(r * H + h) * dv + row) * dk;
#pragma unroll
    for (int e = 0; e < EPT; ++e) {
      const int col = part * EPT + e;
      if (col < dk) {
        if constexpr (sizeof(TS) == 4)
          out[col] = s[e];
        else
          out[col] = __float2bfloat16_rn(s[e]);
      }
    }
  }
}

template <typename T, typename TS, int EPT>
cudaError_t launch_prefill_t(const void *k, const void *v, const float *g, const float *beta, void *S0, int R, int L,
                             int H, int dk, int dv, cudaStream_t s) {
  constexpr int DKP = EPT * kTPR;
  const size_t smem = 2 * sizeof(ChunkBuf<T, DKP>);
  auto kern = prefill_kernel<T, TS, EPT>;
  cudaError_t e = smem > 48 * 1024 ? ensure_smem_limit((const void *)kern, smem) : cudaSuccess;
  if (e != cudaSuccess) return e;
  dim3 grid((dv + kRB - 1) / kRB, H, R);
  kern<<<grid, kPThreads, smem, s>>>(static_cast<const T *>(k), static_cast<const T *>(v), g, beta,
                                     static_cast<TS *>(S0), R, L, H, dk, dv);
  return cudaGetLastError();
}

template <typename T, typename TS>
cudaError_t launch_prefill_ts(const void *k, const void *v, const float *g, const float *beta, void *S0, int R, int L,
                              int H, int dk, int dv, cudaStream_t s) {
  if (dk <= 64) return launch_prefill_t<T, TS, 8>(k, v, g, beta, S0, R, L, H, dk, dv, s);
  if (dk <= 128) return launch_prefill_t<T, TS, 16>(k, v, g, beta, S0, R, L, H, dk, dv, s);
  return launch_prefill_t<T, TS, 32>(k, v, g, beta, S0, R, L, H, dk, dv, s);
}

}  // namespace

cudaError_t launch_prefill(const void *k, const void *v, const float *g, const float *beta, void *S0, int R, int L,
                           int H, int dk, int dv, int qkv_bf16, int s0_bf16, cudaStream_t s) {
  if (dk < 1 || dk > 256 || dv < 1 || dv > 256 || L < 1) return cudaErrorInvalidValue;
  if (qkv_bf16)
    return s0_bf16 ? launch_prefill_ts<__nv_bfloat16, __nv_bfloat16>(k, v, g, beta, S0, R, L, H, dk, dv, s)
                   : launch_prefill_ts<__nv_bfloat16, float>(k, v, g, beta, S0, R, L, H, dk, dv, s);
  return s0_bf16 ? launch_prefill_ts<float, __nv_bfloat16>(k, v, g, beta, S0, R, L, H, dk, dv, s)
                 : launch_prefill_ts<float, float>(k, v, g, beta, S0, R, L, H, dk, dv, s);
}

}  // namespace onela
