// Beam selection on the device: the step after the decode step, which turns
// the candidates' scores into the next step's parent indices (the evolving
// beam tree of the OneLA abstract, whose every step keeps a beam set of width
// W out of the children of the previous one).
//
// Candidate (b, c) of request r (b < W_prev beams, c < C children each) has
// score s = beam_score[r][b] + logp[r][b][c], one fp32 addition.  The W
// candidates with the largest scores are kept, ties going to the smaller
// flat index b C + c, in that order (best first).  Each candidate becomes a
// 64-bit key: the score's bits mapped so that unsigned order is float order
// (NaN lowest, -0 equal to +0), then the complement of the flat index; the
// keys are unique and the wanted order is their descending order.
//
// Stage 1 sorts chunks of kChunk keys in shared memory (bitonic, one CTA per
// chunk and request) and keeps the first K = W of each; merge
// rounds sort groups of kChunk / K such survivor lists the same way, until
// one list per request is left; the last round writes parent, token, score.
#include <cuda_runtime.h>
#include <stdint.h>

#include "internal.h"

namespace onela {
namespace {

constexpr int kChunk = 4096;   // keys sorted per CTA
constexpr int kSThreads = 1024;

__device__ __forceinline__ uint32_t orderable(float f) {
  uint32_t u = __float_as_uint(f);
  if ((u & 0x7fffffffu) > 0x7f800000u) return 0u;  // NaN: below everything
  if (u == 0x80000000u) u = 0u;                     // -0 equals +0
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float from_orderable(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

// Sorts n (a power of two, <= kChunk) keys in s descending.  Every thread of
// the block takes part.
__device__ void bitonic_desc(uint64_t *s, int n) {
  for (int k = 2; k <= n; k <<= 1) {
    for (int j = k >> 1; j > 0; j >>= 1) {
      for (int i = threadIdx.x; i < n / 2; i += blockDim.x) {
        // The i-th pair of this stage: positions a < b = a + j.
        const int a = 2 * i - (i & (j - 1));
        const int b = a + j;
        const uint64_t x = s[a], y = s[b];
        const bool desc = (a & k) == 0;  // this run is sorted descending
        if (desc ? (x < y) : (x > y)) {
          s[a] = y;
          s[b] = x;
        }
      }
      __syncthreads();
    }
  }
}

// Stage 1: keys of the candidates of chunk blockIdx.x of request blockIdx.y,
// sorted; the first K go to out [R][nchunks][K].
__global__ void __launch_bounds__(kSThreads) select_chunks(const float *beam_score, const float *logp, int W_prev,
                                                           int C, int K, uint64_t *out) {
  __shared__ uint64_t s[kChunk];
  const int chunk = blockIdx.x, r = blockIdx.y, nchunks = gridDim.x;
  const int64_t N = (int64_t)W_prev * C;
  const int64_t base = (int64_t)chunk * kChunk;
  const int n = (int)(N - base < kChunk ? N - base : kChunk);
  int np = 1;
  while (np < n) np <<= 1;
  for (int e = threadIdx.x; e < np; e += blockDim.x) {
    uint64_t key = 0;  // padding: below every candidate
    if (e < n) {
      const int64_t flat = base + e;
      const int b = (int)(flat / C);
      const float sc = __fadd_rn(beam_score[(int64_t)r * W_prev + b], logp[(int64_t)r * N + flat]);
      key = ((uint64_t)orderable(sc) << 32) | (uint64_t)(0xffffffffu - (uint32_t)flat);
    }
    s[e] = key;
  }
  __syncthreads();
  bitonic_desc(s, np);
  for (int e = threadIdx.x; e < K; e += blockDim.x)
    out[((int64_t)r * nchunks + chunk) * K + e] = e < n ? s[e] : 0ull;
}

// A merge round: groups of `per` lists of K keys (M lists per request) are
// sorted together and cut to their first K keys: out [R][ngroups][K].  With
// `final` set (one group per request), writes the first W as parent, token,
// score instead.
__global__ void __launch_bounds__(kSThreads) select_merge(const uint64_t *in, int M, int K, int per, int C, int W,
                                                          int final_round, uint64_t *out, int32_t *parent,
                                                          int32_t *token, float *score) {
  __shared__ uint64_t s[kChunk];
  const int grp = blockIdx.x, r = blockIdx.y, ngroups = gridDim.x;
  const int l0 = grp * per;
  const int nl = min(per, M - l0);
  const int n = nl * K;
  int np = 1;
  while (np < n) np <<= 1;
  for (int e = threadIdx.x; e < np; e += blockDim.x)
    s[e] = e < n ? in[((int64_t)r * M + l0) * K + e] : 0ull;
  __syncthreads();
  bitonic_desc(s, np);
  if (final_round) {
    for (int e = threadIdx.x; e < W; e += blockDim.x) {
      const uint64_t key = s[e];
      const uint32_t flat = 0xffffffffu - (uint32_t)(key & 0xffffffffu);
      parent[(int64_t)r * W + e] = (int32_t)(flat / (uint32_t)C);
      token[(int64_t)r * W + e] = (int32_t)(flat % (uint32_t)C);
      score[(int64_t)r * W + e] = from_orderable((uint32_t)(key >> 32));
    }
  } else {
    for (int e = threadIdx.x; e < K; e += blockDim.x) out[((int64_t)r * ngroups + grp) * K + e] = s[e];
  }
}

}  // namespace

// Bytes of device scratch the selection needs: two ping-pong arrays of
// survivor keys.
size_t select_scratch_bytes(int R, int W_prev, int C, int W) {
  const int64_t N = (int64_t)W_prev * C;
  const int K = W;
  const int64_t nchunks = (N + kChunk - 1) / kChunk;
  return (size_t)(2 * (int64_t)R * nchunks * K * 8);
}

cudaError_t launch_select(const float *beam_score, const float *logp, int R, int W_prev, int C, int W,
                          int32_t *parent, int32_t *token, float *score, void *scratch, cudaStream_t s) {
  const int64_t N = (int64_t)W_prev * C;
  if (R < 1 || W_prev < 1 || C < 1 || W < 1 || W > kChunk / 2 || N < W || N > 0xffffffffLL || R > 65535)
    return cudaErrorInvalidValue;
  const int K = W;  // W <= kChunk / 2, so at least two lists fit in one merge sort
  const int64_t nchunks = (N + kChunk - 1) / kChunk;
  if (nchunks > 0x7fffffff) return cudaErrorInvalidValue;
  uint64_t *a = static_cast<uint64_t *>(scratch);
  uint64_t *b = a + (size_t)R * nchunks * K;
  select_chunks<<<dim3((unsigned)nchunks, R), kSThreads, 0, s>>>(beam_score, logp, W_prev, C, K, a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  // Merge rounds: `per` lists of K keys fit in one sort of kChunk keys.
  const int per = kChunk / K;
  int64_t M = nchunks;
  for (;;) {
    const int64_t groups = (M + per - 1) / per;
    const bool fin = groups == 1;
    select_merge<<<dim3((unsigned)groups, R), kSThreads, 0, s>>>(a, (int)M, K, per, C, W, fin ? 1 : 0, b, parent,
                                                                  token, score);
    e = cudaGetLastError();
    if (e != cudaSuccess || fin) return e;
    M = groups;
    uint64_t *t = a;
    a = b;
    b = t;
  }
}

}  // namespace onela
