// SIMT decode-step kernel: any d_k, d_v <= 256, fp32 or bf16 q/k/v and S0.
//
// One CTA per (request r, head h, tile of BT beams).  Each step of the
// shared-state GDN beam decode (OneLA, evolve.pub review, key claims on
// section 3.2, equations 2-4) runs in this one launch:
//   1. ancestry update: the beam's ancestor row is its parent's row plus the
//      parent itself, so only indices move and records stay where they
//      were written (abstract); parents are range-checked;
//   2. the shared-state products S0 k_b and S0 q_b (S0 staged through shared
//      memory in column chunks and reused by every beam of the tile);
//   3. projection replay over the ancestor records, with vectors only and
//      no per-beam matrix (review, Summary): gate weights, dot products
//      k_j . x, and the two d_v-wide accumulators;
//   4. the step epilogue: delta = beta (v - alpha u_k), o = alpha u_q +
//      delta (k . q), and the append of the record (alpha, delta, k).
// This kernel serves shapes the tensor-core kernel does not (fp32 q/k/v, odd
// widths) and is the plain reference the faster kernel is checked against.
#include <cuda_bf16.h>

#include "internal.h"

namespace onela {
namespace {

constexpr int kBT = 16;   // beams per CTA
constexpr int kNT = 256;  // threads per CTA
constexpr int kJC = 32;   // S0 columns staged per chunk

__device__ __forceinline__ float ld_f(const float *p, int64_t i) { return p[i]; }
__device__ __forceinline__ float ld_f(const __nv_bfloat16 *p, int64_t i) { return __bfloat162float(p[i]); }

template <typename QT, typename ST>
__global__ void __launch_bounds__(kNT) step_simt_kernel(const StepParams p) {
  extern __shared__ float smem[];
  const int tile = blockIdx.x, h = blockIdx.y, r = blockIdx.z;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int b0 = tile * kBT;
  const int nb = min(kBT, p.W - b0);
  const int dk = p.dk, dv = p.dv, H = p.H, t = p.t, TM = p.T_max;
  const int d0 = p.d0 ? p.d0[r] : 0;  // depths 1..d0 are folded into S0
  const int nanc = t - 1 - d0;  // replayed ancestors: chain index j is depth d0 + j + 1

  float *xk = smem;                        // [BT][dk]
  float *xq = xk + kBT * dk;               // [BT][dk]
  float *s0t = xq + kBT * dk;              // [JC][dv + 1]
  float *s_alpha = s0t + kJC * (dv + 1);   // [BT]
  float *s_beta = s_alpha + kBT;           // [BT]
  float *s_G = s_beta + kBT;               // [BT]
  float *s_kq = s_G + kBT;                 // [BT]
  float *s_w = s_kq + kBT;                 // [BT][T_max]
  float *s_ck = s_w + kBT * TM;            // [BT][T_max]
  float *s_cq = s_ck + kBT * TM;           // [BT][T_max]
  int *s_chain = reinterpret_cast<int *>(s_cq + kBT * TM);  // [BT][T_max]

  const QT *q = static_cast<const QT *>(p.q);
  const QT *k = static_cast<const QT *>(p.k);
  const QT *v = static_cast<const QT *>(p.v);
  const ST *S0 = static_cast<const ST *>(p.S0);
  QT *rec_k = static_cast<QT *>(p.rec_k);

  // 1a. The tile's k and q as fp32; k is also appended to the record store.
  for (int e = tid; e < kBT * dk; e += kNT) {
    const int b = e / dk, j = e - b * dk;
    float fk = 0.f, fq = 0.f;
    if (b < nb) {
      const int64_t gi = ((int64_t)(r * p.W + b0 + b) * H + h) * dk + j;
      fk = ld_f(k, gi);
      fq = ld_f(q, gi);
      rec_k[rec_row(p, t, r, h, b0 + b) * dk + j] = k[gi];
    }
    xk[e] = fk;
    xq[e] = fq;
  }
  // 1b. Ancestry row, gate weights and per-beam scalars (one thread per beam).
  if (tid < kBT) {
    const int b = tid;
    float G = 0.f, alpha = 0.f, beta = 0.f;
    if (b < nb) {
      const int gb = b0 + b;
      int par = p.parents[r * p.W + gb];
      if (par < 0 || par >= p.W_prev) {
        *reinterpret_cast<volatile int32_t *>(p.err) = kErrParent;
        par = 0;
      }
      int *chain = s_chain + b * TM;
      if (t >= 2) {
        // The parent's ancestry row holds absolute depths 1..t-2 (the
        // folded prefix included); the chain keeps the replayed ones.
        const int32_t *prow = p.anc + anc_row(p, t - 1, r, par);
        if (nanc >= 1) {
          chain[nanc - 1] = par;
          for (int j = 0; j < nanc - 1; ++j) chain[j] = prow[d0 + j];
        }
        if (h == 0) {
          int32_t *row = p.anc + anc_row(p, t, r, gb);
          for (int j = 0; j < t - 2; ++j) row[j] = prow[j];
          row[t - 2] = par;
        }
      }
      float run = 1.f;
      for (int j = nanc - 1; j >= 0; --j) {  // record at depth d0 + j + 1
        s_w[b * TM + j] = run;
        run *= p.rec_alpha[rec_row(p, d0 + j + 1, r, h, chain[j])];
      }
      G = run;
      const int64_t si = (int64_t)(r * p.W + gb) * H + h;
      alpha = expf(p.g[si]);
      beta = p.beta[si];
      p.rec_alpha[rec_row(p, t, r, h, gb)] = alpha;
    }
    s_G[b] = G;
    s_alpha[b] = alpha;
    s_beta[b] = beta;
  }
  __syncthreads();

  // 2. Dot products: k_j . k_b and k_j . q_b over each beam's ancestors, and
  //    k_b . q_b; one warp per (beam, ancestor) pair.
  {
    const int per = nanc + 1;
    for (int pi = warp; pi < nb * per; pi += kNT / 32) {
      const int b = pi / per, jj = pi - b * per;
      float dkk = 0.f, dkq = 0.f;
      if (jj < nanc) {
        const QT *kr = rec_k + rec_row(p, d0 + jj + 1, r, h, s_chain[b * TM + jj]) * dk;
        for (int l = lane; l < dk; l += 32) {
          const float kj = ld_f(kr, l);
          dkk += kj * xk[b * dk + l];
          dkq += kj * xq[b * dk + l];
        }
      } else {
        for (int l = lane; l < dk; l += 32) dkq += xk[b * dk + l] * xq[b * dk + l];
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        dkk += __shfl_xor_sync(0xffffffffu, dkk, off);
        dkq += __shfl_xor_sync(0xffffffffu, dkq, off);
      }
      if (lane == 0) {
        if (jj < nanc) {
          const float w = s_w[b * TM + jj];
          s_ck[b * TM + jj] = w * dkk;
          s_cq[b * TM + jj] = w * dkq;
        } else {
          s_kq[b] = dkq;
        }
      }
    }
  }

  // 3. Shared-state products S0 x for every beam of the tile.  Thread owns
  //    row i of S0 and the beams grp, grp + ngroups, ...
  const int ngroups = kNT / dv;
  const int active = ngroups * dv;
  const int i = tid % dv, grp = tid / dv;
  const int mb = (kBT - grp + ngroups - 1) / ngroups;
  float acck[kBT], accq[kBT];
#pragma unroll
  for (int m = 0; m < kBT; ++m) acck[m] = accq[m] = 0.f;
  const ST *S0h = S0 + (int64_t)(r * H + h) * dv * dk;
  for (int j0 = 0; j0 < dk; j0 += kJC) {
    __syncthreads();
    for (int e = tid; e < kJC * dv; e += kNT) {
      const int jj = e % kJC, ii = e / kJC;
      s0t[jj * (dv + 1) + ii] = (j0 + jj < dk) ? ld_f(S0h, (int64_t)ii * dk + j0 + jj) : 0.f;
    }
    __syncthreads();
    if (tid < active) {
      const int jn = min(kJC, dk - j0);
      for (int jj = 0; jj < jn; ++jj) {
        const float s = s0t[jj * (dv + 1) + i];
#pragma unroll
        for (int m = 0; m < kBT; ++m) {
          if (m < mb) {
            const int b = grp + m * ngroups;
            acck[m] = fmaf(s, xk[b * dk + j0 + jj], acck[m]);
            accq[m] = fmaf(s, xq[b * dk + j0 + jj], accq[m]);
          }
        }
      }
    }
  }
  __syncthreads();

  // 4. Replay + epilogue; writes o and the record's delta (coalesced in i).
  if (tid < active) {
#pragma unroll
    for (int m = 0; m < kBT; ++m) {
      if (m >= mb) continue;
      const int b = grp + m * ngroups;
      if (b >= nb) continue;
      const int gb = b0 + b;
      float uk = s_G[b] * acck[m];
      float uq = s_G[b] * accq[m];
      for (int jj = 0; jj < nanc; ++jj) {
        const float d = p.rec_delta[rec_row(p, d0 + jj + 1, r, h, s_chain[b * TM + jj]) * dv + i];
        uk = fmaf(s_ck[b * TM + jj], d, uk);
        uq = fmaf(s_cq[b * TM + jj], d, uq);
      }
      const int64_t vi = ((int64_t)(r * p.W + gb) * H + h) * dv + i;
      const float alpha = s_alpha[b];
      const float delta = s_beta[b] * (ld_f(v, vi) - alpha * uk);
      p.o[vi] = fmaf(alpha, uq, delta * s_kq[b]);
      p.rec_delta[rec_row(p, t, r, h, gb) * dv + i] = delta;
    }
  }
}

template <typename QT, typename ST>
cudaError_t launch_typed(const StepParams &p, cudaStream_t s) {
  const size_t smem = sizeof(float) * (2 * kBT * p.dk + kJC * (p.dv + 1) + 4 * kBT + 3 * kBT * p.T_max) +
                      sizeof(int) * kBT * p.T_max;
  auto kern = step_simt_kernel<QT, ST>;
  // Raise the dynamic shared-memory limit once per device (not a stream
  // operation, so it must not be repeated inside a captured region).
  static size_t configured[64] = {0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (smem > configured[dev]) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    configured[dev] = smem;
  }
  dim3 grid((p.W + kBT - 1) / kBT, p.H, p.R);
  kern<<<grid, kNT, smem, s>>>(p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_step_simt(const StepParams &p, int qkv_bf16, int s0_bf16, cudaStream_t s) {
  if (qkv_bf16 && s0_bf16) return launch_typed<__nv_bfloat16, __nv_bfloat16>(p, s);
  if (qkv_bf16) return launch_typed<__nv_bfloat16, float>(p, s);
  if (s0_bf16) return launch_typed<float, __nv_bfloat16>(p, s);
  return launch_typed<float, float>(p, s);
}

}  // namespace onela
