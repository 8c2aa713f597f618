// SIMT decode-step kernel: any d_k, d_v <= 256, fp32 or bf16 q/k/v and S0.
//
// One CTA per (request r, head h, tile of BT beams).  Each step of the
// shared-state GDN beam decode (OneLA, evolve.pub review, key claims on
// section 3.2, equations 2-4) runs in this one launch:
//   1. ancestry update: the beam's ancestor row is its parent's row plus the
//      parent itself, so only indices move and records stay where they
//      were written (abstract); parents are range-checked;
//   2. the shared-state products S0 k_b and S0 q_b (S0 staged through shared
//      memory in column chunks and reused by every beam of the tile; each
//      thread holds a 4-row x 4-beam x {k, q} block of the products);
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
constexpr int kSC = kJC + 1;  // row stride of the staged chunk (conflict-free rows)
constexpr int kNV = 2 * kBT;  // product vectors per tile: k_b, q_b of every beam
constexpr int kPPR = kJC / 4;  // 4-element pieces per row of a chunk
constexpr int kStage = (256 * kPPR + kNT - 1) / kNT;  // pieces per thread per chunk at d_v <= 256

__device__ __forceinline__ float ld_f(const float *p, int64_t i) { return p[i]; }
__device__ __forceinline__ float ld_f(const __nv_bfloat16 *p, int64_t i) { return __bfloat162float(p[i]); }
// Four consecutive elements starting at a multiple of 4 (16- or 8-byte aligned).
__device__ __forceinline__ float4 ld_f4(const float *p, int64_t i) { return *reinterpret_cast<const float4 *>(p + i); }
__device__ __forceinline__ float4 ld_f4(const __nv_bfloat16 *p, int64_t i) {
  const uint2 u = *reinterpret_cast<const uint2 *>(p + i);
  const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u.x));
  const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u.y));
  return make_float4(a.x, a.y, b.x, b.y);
}

template <typename QT, typename ST>
__global__ void __launch_bounds__(kNT) step_simt_kernel(const StepParams p) {
  extern __shared__ float smem[];
  const int tile = blockIdx.x, h = blockIdx.y, r = blockIdx.z;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int b0 = tile * kBT;
  const int nb = min(kBT, p.W - b0);
  const int dk = p.dk, dv = p.dv, H = p.H, t = p.t, TM = p.T_max;
  // Depths 1..d0 are folded into S0; the beams replay depths d0+1..t-1,
  // which must fit the record store's T_max slots.
  int d0 = p.d0 ? p.d0[r] : 0;
  if (t - 1 - d0 > TM - 1) {
    if (tid == 0) set_err(p.err, kErrByteWindow);
    d0 = t - TM;  // keeps every access inside the store; the results are void
  }
  const int nanc = t - 1 - d0;  // replayed ancestors: chain index j is depth d0 + j + 1

  const int XS = dk + 1;                   // row stride of xk, xq
  float *xk = smem;                        // [BT][XS]
  float *xq = xk + kBT * XS;               // [BT][XS]
  float *xt = xq + kBT * XS;               // [dk][NV]: vector 2 b is k_b, 2 b + 1 is q_b
  float *s0c = xt + kNV * dk;              // [dv][SC]: a chunk of S0's columns
  float *s_alpha = s0c + dv * kSC;         // [BT]
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
    xk[b * XS + j] = fk;
    xq[b * XS + j] = fq;
  }
  // 1b. Ancestry row, gate weights and per-beam scalars (one thread per beam).
  if (tid < kBT) {
    const int b = tid;
    float G = 0.f, alpha = 0.f, beta = 0.f;
    if (b < nb) {
      const int gb = b0 + b;
      int par = p.parents[r * p.W + gb];
      if (par < 0 || par >= p.W_prev) {
        set_err(p.err, kErrByteParent);
        par = 0;
      }
      int *chain = s_chain + b * TM;
      if (t >= 2) {
        // The parent's ancestry row holds the ancestor at depth dd in
        // entry (dd - 1) mod T_max for its last T_max - 1 depths (the folded
        // prefix included); the chain keeps the replayed ones.
        const int32_t *prow = p.anc + anc_row(p, t - 1, r, par);
        if (nanc >= 1) {
          chain[nanc - 1] = par;
          for (int j = 0; j < nanc - 1; ++j) chain[j] = prow[(d0 + j) % TM];
        }
        if (h == 0) {
          int32_t *row = p.anc + anc_row(p, t, r, gb);
          for (int dd = max(1, t - TM + 1); dd < t - 1; ++dd) row[(dd - 1) % TM] = prow[(dd - 1) % TM];
          row[(t - 2) % TM] = par;
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

  // 1c. The tile's vectors transposed for the S0 products: xt[j][2 b + z].
  for (int e = tid; e < kNV * dk; e += kNT) {
    const int j = e / kNV, n = e - j * kNV;
    xt[e] = ((n & 1) ? xq : xk)[(n >> 1) * XS + j];
  }

  // 2. Dot products: k_j . k_b and k_j . q_b over each beam's ancestors, and
  //    k_b . q_b; one warp per (beam, ancestor) pair.
  {
    const int per = nanc + 1;
    for (int pi = warp; pi < nb * per; pi += kNT / 32) {
      const int b = pi / per, jj = pi - b * per;
      float dkk = 0.f, dkq = 0.f;
      if (jj < nanc) {
        const QT *kr = rec_k + rec_row(p, d0 + jj + 1, r, h, s_chain[b * TM + jj]) * dk;
#pragma unroll 4
        for (int l = lane; l < dk; l += 32) {
          const float kj = ld_f(kr, l);
          dkk += kj * xk[b * XS + l];
          dkq += kj * xq[b * XS + l];
        }
      } else {
        for (int l = lane; l < dk; l += 32) dkq += xk[b * XS + l] * xq[b * XS + l];
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

  // 3. Shared-state products S0 x for every beam of the tile.  Thread (rg,
  //    bg) holds rows rg, rg + RG, rg + 2 RG, rg + 3 RG (RG = ceil(dv / 4))
  //    of the products with the k and q of beams 4 bg .. 4 bg + 3.
  const int RG = (dv + 3) >> 2;
  const int rg = tid % RG, bg = tid / RG;
  const bool act = bg < kBT / 4;
  float acc[4][8];
#pragma unroll
  for (int u = 0; u < 4; ++u)
#pragma unroll
    for (int n = 0; n < 8; ++n) acc[u][n] = 0.f;
  const ST *S0h = S0 + (int64_t)(r * H + h) * dv * dk;
  for (int j0 = 0; j0 < dk; j0 += kJC) {
    __syncthreads();
    if ((dk & 3) == 0) {
      // 4-element pieces, every load of the chunk issued before the stores.
      float4 pc[kStage];
#pragma unroll
      for (int m = 0; m < kStage; ++m) {
        const int e = tid + m * kNT, ii = e / kPPR, j = j0 + 4 * (e - ii * kPPR);
        pc[m] = (ii < dv && j < dk) ? ld_f4(S0h, (int64_t)ii * dk + j) : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int m = 0; m < kStage; ++m) {
        const int e = tid + m * kNT, ii = e / kPPR, jq = e - ii * kPPR;
        if (ii < dv) {
          float *dst = s0c + ii * kSC + 4 * jq;
          dst[0] = pc[m].x, dst[1] = pc[m].y, dst[2] = pc[m].z, dst[3] = pc[m].w;
        }
      }
    } else {
      for (int e = tid; e < kJC * dv; e += kNT) {
        const int ii = e / kJC, jj = e - ii * kJC;
        s0c[ii * kSC + jj] = (j0 + jj < dk) ? ld_f(S0h, (int64_t)ii * dk + j0 + jj) : 0.f;
      }
    }
    __syncthreads();
    if (act) {
      const int jn = min(kJC, dk - j0);
#pragma unroll 2
      for (int jj = 0; jj < jn; ++jj) {
        float sv[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) sv[u] = rg + u * RG < dv ? s0c[(rg + u * RG) * kSC + jj] : 0.f;
        const float4 x0 = reinterpret_cast<const float4 *>(xt + (j0 + jj) * kNV)[2 * bg];
        const float4 x1 = reinterpret_cast<const float4 *>(xt + (j0 + jj) * kNV)[2 * bg + 1];
        const float xv[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
#pragma unroll
        for (int u = 0; u < 4; ++u)
#pragma unroll
          for (int n = 0; n < 8; ++n) acc[u][n] = fmaf(sv[u], xv[n], acc[u][n]);
      }
    }
  }

  // 4. Replay + epilogue; writes o and the record's delta (coalesced in the
  //    rows).  Depth by depth, the delta rows of all four beams at once.
  if (act) {
    float uk[4][4], uq[4][4];  // [beam m][row u]
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      const float G = 4 * bg + m < nb ? s_G[4 * bg + m] : 0.f;
#pragma unroll
      for (int u = 0; u < 4; ++u) uk[m][u] = G * acc[u][2 * m], uq[m][u] = G * acc[u][2 * m + 1];
    }
#pragma unroll 1
    for (int jj = 0; jj < nanc; ++jj) {
      float dl[4][4];
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        const int b = 4 * bg + m;
        const int64_t row = b < nb ? rec_row(p, d0 + jj + 1, r, h, s_chain[b * TM + jj]) * dv : 0;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int i = rg + u * RG;
          dl[m][u] = (b < nb && i < dv) ? p.rec_delta[row + i] : 0.f;
        }
      }
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        const int b = 4 * bg + m;
        const float ck = b < nb ? s_ck[b * TM + jj] : 0.f, cq = b < nb ? s_cq[b * TM + jj] : 0.f;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          uk[m][u] = fmaf(ck, dl[m][u], uk[m][u]);
          uq[m][u] = fmaf(cq, dl[m][u], uq[m][u]);
        }
      }
    }
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      const int b = 4 * bg + m;
      if (b >= nb) continue;
      const int gb = b0 + b;
      const float alpha = s_alpha[b], beta = s_beta[b], kq = s_kq[b];
      const int64_t vrow = ((int64_t)(r * p.W + gb) * H + h) * dv;
      const int64_t drow = rec_row(p, t, r, h, gb) * dv;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int i = rg + u * RG;
        if (i >= dv) continue;
        const float delta = beta * (ld_f(v, vrow + i) - alpha * uk[m][u]);
        p.o[vrow + i] = fmaf(alpha, uq[m][u], delta * kq);
        p.rec_delta[drow + i] = delta;
      }
    }
  }
}

template <typename QT, typename ST>
cudaError_t launch_typed(const StepParams &p, cudaStream_t s) {
  const size_t smem = sizeof(float) * (2 * kBT * (p.dk + 1) + kNV * p.dk + p.dv * kSC + 4 * kBT +
                                       3 * kBT * p.T_max) +
                      sizeof(int) * kBT * p.T_max;
  auto kern = step_simt_kernel<QT, ST>;
  // Raise the dynamic shared-memory limit once per device (not a stream
  // operation, so it must not be repeated inside a captured region).
  cudaError_t e = ensure_smem_limit((const void *)kern, smem);
  if (e != cudaSuccess) return e;
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
