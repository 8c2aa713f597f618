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
// keys are unique and the wanted set is the W largest keys.
//
// Stage 1 (one CTA per chunk of kChunk candidates and request) finds the
// chunk's K = W largest keys by radix selection: eight passes over the 64-bit
// keys, 8 bits at a time from the top, each building a 256-bin histogram of
// the keys that still match the prefix chosen so far (shared-memory
// atomics) and fixing the next 8 bits of the K-th largest key, stopping early
// once the chosen bin holds exactly the keys still wanted; every key >= the
// threshold is kept.  Merge rounds select the W largest of
// groups of survivor lists the same way, until one list per request is left;
// the last round orders it (each key's rank is the number of larger keys)
// and writes parent, token and score.
#include <cuda_runtime.h>
#include <stdint.h>

#include "internal.h"

namespace onela {
namespace {

constexpr int kChunk = 4096;    // keys per CTA
constexpr int kSThreads = 1024;
constexpr int kPer = kChunk / kSThreads;  // keys per thread

__device__ __forceinline__ uint32_t orderable(float f) {
  uint32_t u = __float_as_uint(f);
  if ((u & 0x7fffffffu) > 0x7f800000u) return 0u;  // NaN: below everything
  if (u == 0x80000000u) u = 0u;                     // -0 equals +0
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float from_orderable(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

struct SelectSmem {
  uint32_t hist[256];
  uint64_t prefix;   // bits of the K-th largest key fixed so far
  int want;          // how many keys still to take at or below the prefix
  int count;         // keys written so far
  int done;          // the chosen bin holds exactly the keys still wanted
};

// The K-th largest of the block's keys (kPer per thread in k[], absent ones
// 0, which is below every real key): every thread returns it.  K >= 1 and at
// most the number of real keys.
__device__ uint64_t kth_largest(const uint64_t (&k)[kPer], int K, SelectSmem &sm) {
  const int tid = threadIdx.x, lane = tid & 31;
  if (tid == 0) {
    sm.prefix = 0;
    sm.want = K;
    sm.done = 0;
  }
#pragma unroll 1
  for (int pass = 0; pass < 8; ++pass) {
    const int shift = 56 - 8 * pass;
    const uint64_t hi_mask = pass == 0 ? 0ull : (~0ull << (shift + 8));
    for (int e = tid; e < 256; e += blockDim.x) sm.hist[e] = 0;
    __syncthreads();
    const uint64_t prefix = sm.prefix;
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
      const bool act = (k[i] & hi_mask) == prefix;
      const uint32_t d = (uint32_t)(k[i] >> shift) & 255u;
      if (act) atomicAdd(&sm.hist[d], 1u);
    }
    __syncthreads();
    if (tid < 32) {
      // Bins from the top: lane l sums bins 255 - 8l .. 248 - 8l.
      uint32_t c[8], s = 0;
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        c[q] = sm.hist[255 - 8 * lane - q];
        s += c[q];
      }
      uint32_t incl = s;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t x = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += x;
      }
      const uint32_t above = incl - s;  // keys in the bins above this lane's
      const uint32_t want = (uint32_t)sm.want;
      if (above < want && want <= incl) {  // exactly one lane
        uint32_t run = above;
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          if (run < want && want <= run + c[q]) {
            sm.prefix = prefix | ((uint64_t)(255 - 8 * lane - q) << shift);
            sm.want = (int)(want - run);
            // Every key of this bin is wanted: the threshold is the bin's
            // lowest possible key (the remaining bits zero).
            if (want == run + c[q]) sm.done = 1;
          }
          run += c[q];
        }
      }
    }
    __syncthreads();
    if (sm.done) break;
  }
  return sm.prefix;
}

// Stage 1: the K largest keys of chunk blockIdx.x of request blockIdx.y go
// to out [R][nchunks][K] (unordered; 0 where the chunk has fewer than K).
__global__ void __launch_bounds__(kSThreads) select_chunks(const float *beam_score, const float *logp, int W_prev,
                                                           int C, int K, uint64_t *out) {
  __shared__ SelectSmem sm;
  const int chunk = blockIdx.x, r = blockIdx.y, nchunks = gridDim.x, tid = threadIdx.x;
  const int64_t N = (int64_t)W_prev * C;
  const int64_t base = (int64_t)chunk * kChunk;
  const int n = (int)(N - base < kChunk ? N - base : kChunk);
  uint64_t k[kPer];
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    const int e = i * kSThreads + tid;
    k[i] = 0;
    if (e < n) {
      const int64_t flat = base + e;
      const int b = (int)(flat / C);
      const float sc = __fadd_rn(beam_score[(int64_t)r * W_prev + b], logp[(int64_t)r * N + flat]);
      k[i] = ((uint64_t)orderable(sc) << 32) | (uint64_t)(0xffffffffu - (uint32_t)flat);
    }
  }
  uint64_t *o = out + ((int64_t)r * nchunks + chunk) * K;
  const int take = n < K ? n : K;
  if (tid == 0) sm.count = 0;
  const uint64_t t = kth_largest(k, take, sm);
#pragma unroll
  for (int i = 0; i < kPer; ++i)
    if (k[i] >= t && k[i] != 0) o[atomicAdd(&sm.count, 1)] = k[i];
  for (int e = take + tid; e < K; e += kSThreads) o[e] = 0;
}

// A merge round over lists of K keys, M lists per request, `per` of them per
// CTA (per K <= kChunk): the K largest of each group go to out [R][groups][K];
// in the final round (one group) the W largest are ordered and written as
// parent, token, score.
__global__ void __launch_bounds__(kSThreads) select_merge(const uint64_t *in, int M, int K, int per, int C, int W,
                                                          int final_round, uint64_t *out, int32_t *parent,
                                                          int32_t *token, float *score) {
  __shared__ SelectSmem sm;
  __shared__ uint64_t sel[kChunk / 2];
  const int grp = blockIdx.x, r = blockIdx.y, groups = gridDim.x, tid = threadIdx.x;
  const int l0 = grp * per;
  const int nl = min(per, M - l0);
  const int n = nl * K;
  const uint64_t *src = in + ((int64_t)r * M + l0) * K;
  uint64_t k[kPer];
  int real = 0;
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    const int e = i * kSThreads + tid;
    k[i] = e < n ? src[e] : 0ull;
    real += k[i] != 0;
  }
  // The number of real keys (lists shorter than K are padded with 0).
  if (tid == 0) sm.count = 0;
  __syncthreads();
  atomicAdd(&sm.count, real);
  __syncthreads();
  const int nreal = sm.count;
  const int take = nreal < K ? nreal : K;
  __syncthreads();
  if (tid == 0) sm.count = 0;
  const uint64_t t = kth_largest(k, take, sm);
  if (!final_round) {
    uint64_t *o = out + ((int64_t)r * groups + grp) * K;
#pragma unroll
    for (int i = 0; i < kPer; ++i)
      if (k[i] >= t && k[i] != 0) o[atomicAdd(&sm.count, 1)] = k[i];
    for (int e = take + tid; e < K; e += kSThreads) o[e] = 0;
    return;
  }
  // Final round: the W (= take) kept keys into shared memory, then each one's
  // rank = the number of larger kept keys gives its output position.
#pragma unroll
  for (int i = 0; i < kPer; ++i)
    if (k[i] >= t && k[i] != 0) sel[atomicAdd(&sm.count, 1)] = k[i];
  __syncthreads();
  for (int e = tid; e < take; e += kSThreads) {
    const uint64_t key = sel[e];
    int rank = 0;
    for (int q = 0; q < take; ++q) rank += sel[q] > key;
    const uint32_t flat = 0xffffffffu - (uint32_t)(key & 0xffffffffu);
    parent[(int64_t)r * W + rank] = (int32_t)(flat / (uint32_t)C);
    token[(int64_t)r * W + rank] = (int32_t)(flat % (uint32_t)C);
    score[(int64_t)r * W + rank] = from_orderable((uint32_t)(key >> 32));
  }
}

}  // namespace

// Bytes of device scratch the selection needs: two ping-pong arrays of
// survivor keys.
size_t select_scratch_bytes(int R, int W_prev, int C, int W) {
  const int64_t N = (int64_t)W_prev * C;
  const int64_t nchunks = (N + kChunk - 1) / kChunk;
  return (size_t)(2 * (int64_t)R * nchunks * W * 8);
}

cudaError_t launch_select(const float *beam_score, const float *logp, int R, int W_prev, int C, int W,
                          int32_t *parent, int32_t *token, float *score, void *scratch, cudaStream_t s) {
  const int64_t N = (int64_t)W_prev * C;
  if (R < 1 || W_prev < 1 || C < 1 || W < 1 || W > kChunk / 2 || N < W || N > 0xffffffffLL || R > 65535)
    return cudaErrorInvalidValue;
  const int K = W;  // W <= kChunk / 2, so at least two lists fit in one merge CTA
  const int64_t nchunks = (N + kChunk - 1) / kChunk;
  if (nchunks > 0x7fffffff) return cudaErrorInvalidValue;
  uint64_t *a = static_cast<uint64_t *>(scratch);
  uint64_t *b = a + (size_t)R * nchunks * K;
  select_chunks<<<dim3((unsigned)nchunks, R), kSThreads, 0, s>>>(beam_score, logp, W_prev, C, K, a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
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
