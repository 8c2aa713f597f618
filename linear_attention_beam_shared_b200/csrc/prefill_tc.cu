// Chunked prefill on the tensor cores (tcgen05, sm_100a) for bf16 k and v
// with d_k = d_v in {64, 128}.
//
// The recurrence is the GDN update of the evolve.pub review's key claims on
// section 3.2 (equation 2), run from the zero state over the L prompt tokens:
//
//   S_l = alpha_l S_{l-1} + delta_l k_l^T,   delta_l = beta_l (v_l - alpha_l S_{l-1} k_l).
//
// It is linear in the tokens' deltas, so a chunk of C = 64 tokens can be
// taken at once (the chunked "WY" form of the delta rule; the result is the
// same up to rounding order).  With the state S before the chunk, tokens
// i = 0 .. C-1 of the chunk, gamma_i = alpha_0 ... alpha_i and
// Y = S K^T (column i: S k_i):
//
//   (I + A) Delta = Z,   A_ij = beta_i (gamma_i / gamma_j) (k_i . k_j) for j < i,
//                        Z_i  = beta_i (v_i - gamma_i S k_i),
//   S' = gamma_{C-1} S + sum_j (gamma_{C-1} / gamma_j) delta_j k_j^T.
//
// T = (I + A)^{-1} depends on the keys and gates only, so one kernel forms it
// for every chunk at once (prefill_prep_kernel).  The chain over the chunks
// is three tensor-core products per chunk, all with the state's d_v rows as
// the MMA's M = 128 rows and fp32 accumulators in TMEM:
//
//   Y^T   = S . K^T            (K = the chunk's keys, exact in bf16)
//   Delta^T = Z^T . T^T        (Z^T formed from Y^T, v and the gates)
//   dS    = (Delta^T diag(gamma_{C-1}/gamma_j)) . K
//   S    <- gamma_{C-1} S + dS (fp32, in registers)
//
// Operands that are not bf16 values (S, Z, Delta, T) enter as sums of three
// bf16 terms (hi + mid + lo, each the rounding of what the earlier terms
// leave), and the products keep every pair of terms whose orders add up to at
// most 2, so each product is good to about 2^-24 of its scale, as fp32 is.
//
// Segments: S after a segment of chunks is an affine map of S before it,
// S_end = S_start A_s + B_s (every row of S evolves on its own, and all rows
// see the same keys and gates).  B_s is the chain run from the zero state
// with the segment's values; A_s is the chain run from the identity (rows =
// d_k) with zero values.  The chains of all segments run at once (one CTA
// each), and prefill_combine_kernel folds them left to right,
// S = ((B_0 A_1 + B_1) A_2 + B_2) ..., in fp32.
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include "internal.h"
#include "sm100_ptx.h"
#include "tc_common.h"

namespace onela {
namespace {

constexpr int kC = 64;                     // tokens per chunk
constexpr int kEpiThreads = 512;           // 16 warps: the state's 128 rows x 4 column quarters
constexpr int kCtlWarp = 16;               // loads and MMA issue
constexpr int kChainThreads = kEpiThreads + 32;
constexpr uint32_t kTPlane = kC * 128u;    // one bf16 term of T: 64 rows x 128 B
constexpr uint32_t kGateBytes = 1024u;     // beta [64], gamma [64], ratio [64] fp32, gamma_{C-1}
constexpr uint32_t kPrepBytes = 3u * kTPlane + kGateBytes;  // per (request, head, chunk)
// TMEM of a chain CTA: Y^T [0, 64), Delta^T [64, 128), dS [128, 128 + d_k),
// and from column kTA the bf16 terms of the MMAs' A operand (the state's, or
// those of Z^T and of the scaled Delta^T), two elements per column.
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTA = 256;

// Two floats as bf16x2, rounded to nearest even; lo in the low half.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// x as three bf16 terms (hi, mid, lo), 8 consecutive elements each, packed
// for one 16-byte store per term: each term is the rounding of what the
// earlier terms leave, and the differences are exact in fp32.
__device__ __forceinline__ void split3(const float (&x)[8], uint4 (&o)[3]) {
  uint32_t w[3][4];
#pragma unroll
  for (int z = 0; z < 4; ++z) {
    float a = x[2 * z], b = x[2 * z + 1];
#pragma unroll
    for (int pl = 0; pl < 3; ++pl) {
      const uint32_t t = pack_bf16x2(a, b);
      w[pl][z] = t;
      if (pl < 2) {
        a -= __uint_as_float(t << 16);
        b -= __uint_as_float(t & 0xffff0000u);
      }
    }
  }
#pragma unroll
  for (int pl = 0; pl < 3; ++pl) o[pl] = make_uint4(w[pl][0], w[pl][1], w[pl][2], w[pl][3]);
}

// Four 8x8 tiles of 16-bit elements from shared memory, transposed: lane L
// gives the address of row L % 8 of tile L / 8; the thread gets, per tile,
// the elements (2 (t % 4), t / 4) and (2 (t % 4) + 1, t / 4).
__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
// The inverse layout to shared memory, not transposed: per tile the thread
// holds elements (t / 4, 2 (t % 4)) and (t / 4, 2 (t % 4) + 1).
__device__ __forceinline__ void stsm_x4(uint32_t addr, const uint32_t (&r)[4]) {
  asm volatile("stmatrix.sync.aligned.m8n8.x4.shared.b16 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(r[0]),
               "r"(r[1]), "r"(r[2]), "r"(r[3])
               : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem desc]^T, bf16 inputs, fp32 accumulate; A is
// M rows (lanes) x K bf16 elements, two per 32-bit column.
__device__ __forceinline__ void mma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// 32 lanes x 32 bit, N consecutive columns from thread i of the warp to TMEM
// lane (lane base of the warp) + i.
template <int N>
__device__ __forceinline__ void tmem_st(uint32_t taddr, const uint32_t (&v)[N]);
template <>
__device__ __forceinline__ void tmem_st<8>(uint32_t taddr, const uint32_t (&v)[8]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"r"(taddr),
               "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7])
               : "memory");
}
template <>
__device__ __forceinline__ void tmem_st<16>(uint32_t taddr, const uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]), "r"(v[9]),
      "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
      : "memory");
}

__device__ __forceinline__ void fence_proxy_async() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ------------------------------------------------------------------ prep
// One CTA per 2 chunks of one (request, head): T = (I + A)^{-1} of every
// chunk as three bf16 terms in the 128-byte-swizzled K-major operand layout
// (row i, column j), and the chunk's gates.  The key Gram matrices come from
// the tensor cores (one 128-token product; the chunks' 64 x 64 diagonal
// blocks are used), exact products of bf16 keys with fp32 accumulation; the
// triangular solve is a forward substitution with one column of T per thread,
// held in registers.  Tokens past the prompt have beta = 0, g = 0 and zero
// keys, so they change nothing.
constexpr int kPrepChunks = 2;                   // one 128-token MMA
constexpr int kPrepThreads = kPrepChunks * kC;  // one column of T per thread
constexpr int kAStride = kC + 4;  // row stride of A in shared memory (floats)

struct PrepParams {
  CUtensorMap tm_k;  // [R][L][H][d] bf16, box {64, 1, 128, 1}
  const float *g, *beta;
  uint8_t *ws;
  int L, H, nchunks;
  unsigned long long wait_limit_ns;
  int32_t *err;
};

template <int DK>
struct PrepLayout {
  static constexpr int NK = DK / 64;
  static constexpr uint32_t kt = 0;  // keys [NK][128 tokens][128 B]; later T [2][64][64] fp32
  static constexpr uint32_t ktb = NK * 16384u, tmb = (uint32_t)kPrepChunks * kC * kC * 4u;
  static constexpr uint32_t am = ktb > tmb ? ktb : tmb;                    // A [2][64][kAStride] fp32
  static constexpr uint32_t gc = am + (uint32_t)kPrepChunks * kC * kAStride * 4u;  // log gamma [128]
  static constexpr uint32_t bt = gc + kPrepChunks * kC * 4u;               // beta [128]
  static constexpr uint32_t ws = bt + kPrepChunks * kC * 4u;               // warp sums [4]
  static constexpr uint32_t bar = ws + 64u;                                // 2 barriers, TMEM address
  static constexpr uint32_t total = bar + 64u;
};

template <int DK>
__global__ void __launch_bounds__(kPrepThreads, 3) prefill_prep_kernel(const __grid_constant__ PrepParams p) {
  using PL = PrepLayout<DK>;
  constexpr int NK = PL::NK;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_u32 = ptx::smem_u32(smem_raw);
  uint8_t *base = smem_raw + ((1024u - (raw_u32 & 1023u)) & 1023u);
  float *Am = reinterpret_cast<float *>(base + PL::am);
  float *Tm = reinterpret_cast<float *>(base + PL::kt);
  float *gc = reinterpret_cast<float *>(base + PL::gc);
  float *bt = reinterpret_cast<float *>(base + PL::bt);
  float *wsum = reinterpret_cast<float *>(base + PL::ws);
  uint64_t *bar_k = reinterpret_cast<uint64_t *>(base + PL::bar);
  uint64_t *bar_mma = bar_k + 1;
  uint32_t *s_tmem = reinterpret_cast<uint32_t *>(bar_k + 2);
  const int cb = blockIdx.x * kPrepChunks, h = blockIdx.y, r = blockIdx.z, H = p.H, L = p.L;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int tok0 = cb * kC;  // first token of the CTA

  if (warp == 0) {
    if (lane == 0) {
      ptx::mbar_init(bar_k, 1);
      ptx::mbar_init(bar_mma, 1);
      ptx::mbar_fence_init();
    }
    __syncwarp();
    ptx::tmem_alloc(s_tmem, 128);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *s_tmem;
  bool ok = true;
  if (tid == 0) {
    ptx::mbar_arrive_expect_tx(bar_k, NK * 16384u);
#pragma unroll
    for (int ka = 0; ka < NK; ++ka) ptx::tma_load_4d(base + PL::kt + ka * 16384, &p.tm_k, ka * 64, h, tok0, r, bar_k);
    ok = ptx::mbar_wait(bar_k, 0, p.wait_limit_ns);
    if (!ok) ptx::mbar_wait(bar_k, 0, p.wait_limit_ns);  // the keys still in flight land first (bounded)
    if (ok) {
      ptx::tc_fence_after();
      constexpr uint32_t id = ptx::idesc_bf16_f32(128, 128);
      const uint32_t k_u32 = ptx::smem_u32(base + PL::kt);
      int acc = 0;
#pragma unroll
      for (int ka = 0; ka < NK; ++ka)
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint64_t d = ptx::desc_k128(k_u32 + ka * 16384 + kk * 32);
          ptx::mma_bf16(tmem, d, d, id, acc);
          acc = 1;
        }
      ptx::mma_commit(bar_mma);
    }
  }
  // Gates: log gamma by a prefix sum within each chunk (two warps per chunk).
  {
    const int l = tok0 + tid;
    const int64_t si = (int64_t)(r * L + l) * H + h;
    const float gv = l < L ? p.g[si] : 0.f;
    bt[tid] = l < L ? p.beta[si] : 0.f;
    float sum = gv;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const float t = __shfl_up_sync(0xffffffffu, sum, o);
      if (lane >= o) sum += t;
    }
    if (lane == 31) wsum[warp] = sum;
    __syncthreads();
    gc[tid] = (warp & 1) ? sum + wsum[warp - 1] : sum;
  }
  // A_ij = beta_i (gamma_i / gamma_j) (k_i . k_j) for j < i; row i by the
  // thread of TMEM lane i.
  const bool got = ptx::mbar_wait(bar_mma, 0, p.wait_limit_ns);
  __syncthreads();  // the log gammas of every chunk are in
  ptx::tc_fence_after();
  {
    const int t = tid, ch = t >> 6, i = t & 63;  // TMEM lane t = token t of the pair
    const float gi = gc[t], bi = bt[t];
    float *arow = Am + (ch * kC + i) * kAStride;
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      float gg[32];
      ptx::tmem_ld32(tmem + ((uint32_t)(warp * 32) << 16) + (t & 64) + q * 32, gg);
      ptx::tmem_ld_wait();
#pragma unroll
      for (int x = 0; x < 32; x += 4) {
        float4 v;
        float *vv = reinterpret_cast<float *>(&v);
#pragma unroll
        for (int z = 0; z < 4; ++z) {
          const int j = q * 32 + x + z;
          vv[z] = j < i ? bi * expf(gi - gc[ch * kC + j]) * gg[x + z] : 0.f;
        }
        *reinterpret_cast<float4 *>(arow + q * 32 + x) = v;
      }
    }
  }
  ptx::tc_fence_before();
  __syncthreads();  // A complete; the keys are consumed
  // Forward substitution: thread (chunk ch, column j) holds column j of T.
  {
    const int ch = tid >> 6, j = tid & 63;
    const float *A = Am + ch * kC * kAStride;
    float tcol[kC];
#pragma unroll
    for (int i = 0; i < kC; ++i) {
      float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;
#pragma unroll
      for (int l = 0; l < i; l += 4) {
        const float4 a4 = *reinterpret_cast<const float4 *>(A + i * kAStride + l);
        s0 = fmaf(a4.x, tcol[l], s0);
        if (l + 1 < i) s1 = fmaf(a4.y, tcol[l + 1], s1);
        if (l + 2 < i) s2 = fmaf(a4.z, tcol[l + 2], s2);
        if (l + 3 < i) s3 = fmaf(a4.w, tcol[l + 3], s3);
      }
      tcol[i] = i == j ? 1.f : -((s0 + s1) + (s2 + s3));
    }
#pragma unroll
    for (int l = 0; l < kC; ++l) Tm[(ch * kC + l) * kC + j] = tcol[l];
  }
  __syncthreads();
  // T as three bf16 terms, row by row; the gates of each chunk.
  for (int e = tid; e < kPrepChunks * kC * 8; e += kPrepThreads) {
    const int ch = e / (kC * 8), i = (e >> 3) & 63, c8 = e & 7;
    if (cb + ch >= p.nchunks) continue;
    const float4 lo = *reinterpret_cast<const float4 *>(Tm + (ch * kC + i) * kC + c8 * 8);
    const float4 hi = *reinterpret_cast<const float4 *>(Tm + (ch * kC + i) * kC + c8 * 8 + 4);
    const float x[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
    uint4 o[3];
    split3(x, o);
    uint8_t *out = p.ws + ((int64_t)(r * H + h) * p.nchunks + cb + ch) * kPrepBytes;
#pragma unroll
    for (int pl = 0; pl < 3; ++pl) *reinterpret_cast<uint4 *>(out + pl * kTPlane + ptx::swz128(i, c8)) = o[pl];
  }
  {
    const int ch = tid >> 6, i = tid & 63;
    if (cb + ch < p.nchunks) {
      float *gt = reinterpret_cast<float *>(p.ws + ((int64_t)(r * H + h) * p.nchunks + cb + ch) * kPrepBytes +
                                            3 * kTPlane);
      const float last = gc[ch * kC + kC - 1];  // padded tokens add g = 0
      gt[i] = bt[tid];
      gt[kC + i] = expf(gc[tid]);
      gt[2 * kC + i] = expf(last - gc[tid]);
      if (i == 0) gt[3 * kC] = expf(last);
    }
  }
  if ((tid == 0 && !ok) || !got) set_err(p.err, kErrByteTimeout);
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, 128);
  }
}

// ----------------------------------------------------------------- chain
struct ChainParams {
  CUtensorMap tm_k;  // [R][L][H][d] bf16, box {64, 1, 64, 1}
  CUtensorMap tm_v;
  const uint8_t *prep;  // [R][H][nchunks][kPrepBytes]
  float *units;         // [R][H][2 nseg - 1][d][d]: B_0, A_1, B_1, A_2, B_2, ...
  int H, nchunks, cps;  // cps: chunks per segment
  unsigned long long wait_limit_ns;
  int32_t *err;
};

template <int DK>
struct ChainLayout {
  static constexpr int NK = DK / 64;
  static constexpr uint32_t kt = 0;                           // K tile [NK][64 tokens][128 B]
  static constexpr uint32_t ktt = kt + NK * 8192u;            // K^T [DK rows][128 B]
  static constexpr uint32_t vtt = ktt + DK * 128u;            // v^T [DK rows][128 B]
  static constexpr uint32_t vt = vtt + DK * 128u;             // v tile [NK][64 tokens][128 B]
  static constexpr uint32_t tp = vt + NK * 8192u;             // T terms [3][64][128 B]
  static constexpr uint32_t gt = tp + 3u * kTPlane;           // gates, two buffers
  static constexpr uint32_t bar = gt + 2u * kGateBytes;       // 4 barriers and the TMEM address
  static constexpr uint32_t total = bar + 64u;
};

template <int DK>
__global__ void __launch_bounds__(kChainThreads, 1) prefill_chain_kernel(const __grid_constant__ ChainParams p) {
  using LY = ChainLayout<DK>;
  constexpr int NK = LY::NK;
  constexpr int HC = DK / 4;  // state columns per thread
  constexpr int TT = kC / 4;  // tokens per thread
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_u32 = ptx::smem_u32(smem_raw);
  uint8_t *base = smem_raw + ((1024u - (raw_u32 & 1023u)) & 1023u);
  uint64_t *bar_kv = reinterpret_cast<uint64_t *>(base + LY::bar);  // k (and v) tile landed
  uint64_t *bar_t = bar_kv + 1;    // T terms and gates landed
  uint64_t *bar_mma = bar_kv + 2;  // an MMA group completed
  uint64_t *bar_epi = bar_kv + 3;  // the epilogue warps finished a stage
  uint32_t *s_tmem = reinterpret_cast<uint32_t *>(bar_kv + 4);

  const int u = blockIdx.x, h = blockIdx.y, r = blockIdx.z, H = p.H;
  const int seg = (u + 1) >> 1;
  const bool amode = (u & 1) != 0;  // the transition A_seg: identity start, zero values
  const int c0 = seg * p.cps, c1 = min(p.nchunks, c0 + p.cps);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint64_t lim = p.wait_limit_ns;

  if (warp == kCtlWarp) {
    if (lane == 0) {
      ptx::mbar_init(bar_kv, 1);
      ptx::mbar_init(bar_t, 1);
      ptx::mbar_init(bar_mma, 1);
      ptx::mbar_init(bar_epi, kEpiThreads / 32);
      ptx::mbar_fence_init();
    }
    __syncwarp();
    ptx::tmem_alloc(s_tmem, kTmemCols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *s_tmem;
  const uint32_t kt_u32 = ptx::smem_u32(base + LY::kt);
  const uint32_t ktt_u32 = ptx::smem_u32(base + LY::ktt), tp_u32 = ptx::smem_u32(base + LY::tp);

  if (warp == kCtlWarp) {
    if (lane == 0) {
      // --------------------------------------------- loads and MMA issue
      const uint8_t *prep = p.prep + (int64_t)(r * H + h) * p.nchunks * kPrepBytes;
      auto load_kv = [&](int c) {
        ptx::mbar_arrive_expect_tx(bar_kv, NK * 8192u * (amode ? 1u : 2u));
#pragma unroll
        for (int ka = 0; ka < NK; ++ka) ptx::tma_load_4d(base + LY::kt + ka * 8192, &p.tm_k, ka * 64, h, c * kC, r, bar_kv);
        if (!amode)
#pragma unroll
          for (int ka = 0; ka < NK; ++ka)
            ptx::tma_load_4d(base + LY::vt + ka * 8192, &p.tm_v, ka * 64, h, c * kC, r, bar_kv);
      };
      auto load_t = [&](int c) {
        const uint8_t *src = prep + (int64_t)c * kPrepBytes;
        ptx::mbar_arrive_expect_tx(bar_t, 3u * kTPlane + kGateBytes);
        ptx::bulk_g2s(base + LY::tp, src, 3u * kTPlane, bar_t);
        ptx::bulk_g2s(base + LY::gt + ((c - c0) & 1) * kGateBytes, src + 3u * kTPlane, kGateBytes, bar_t);
      };
      constexpr uint32_t idN64 = ptx::idesc_bf16_f32(128, 64), idS = ptx::idesc_bf16_f32(128, DK);
      bool ok = true;
      int kv_pending = 0, t_pending = 0;  // parity + 1 of a copy not yet seen landing
      uint32_t epi = 0;
      load_kv(c0);
      kv_pending = 1;
      load_t(c0);
      t_pending = 1;
#pragma unroll 1
      for (int c = c0; c < c1 && ok; ++c) {
        const uint32_t it = (uint32_t)(c - c0);
        ok = ptx::mbar_wait(bar_epi, epi++ & 1, lim);  // the state's terms are in
        ok = ok && ptx::mbar_wait(bar_kv, it & 1, lim);
        if (!ok) break;
        kv_pending = 0;
        ptx::tc_fence_after();
        // Y^T = S . K^T
        {
          int acc = 0;
#pragma unroll
          for (int pl = 0; pl < 3; ++pl)
#pragma unroll
            for (int kk = 0; kk < DK / 16; ++kk) {
              mma_bf16_ts(tmem, tmem + kTA + pl * (DK / 2) + kk * 8,
                          ptx::desc_k128(kt_u32 + (kk >> 2) * 8192 + (kk & 3) * 32), idN64, acc);
              acc = 1;
            }
          ptx::mma_commit(bar_mma);
        }
        ok = ptx::mbar_wait(bar_epi, epi++ & 1, lim);  // Z^T and K^T written; k and v read
        if (!ok) break;
        if (c + 1 < c1) {
          load_kv(c + 1);
          kv_pending = 1 + (int)((it + 1) & 1);
        }
        ok = ptx::mbar_wait(bar_t, it & 1, lim);
        if (!ok) break;
        t_pending = 0;
        ptx::tc_fence_after();
        // Delta^T = Z^T . T^T, the term pairs of order <= 2
        {
          int acc = 0;
#pragma unroll
          for (int pa = 0; pa < 3; ++pa)
#pragma unroll
            for (int pb = 0; pb < 3 - pa; ++pb)
#pragma unroll
              for (int kk = 0; kk < 4; ++kk) {
                mma_bf16_ts(tmem + 64, tmem + kTA + pa * 32 + kk * 8, ptx::desc_k128(tp_u32 + pb * kTPlane + kk * 32),
                            idN64, acc);
                acc = 1;
              }
          ptx::mma_commit(bar_mma);
        }
        ok = ptx::mbar_wait(bar_epi, epi++ & 1, lim);  // scaled Delta^T written; T read
        if (!ok) break;
        if (c + 1 < c1) {
          load_t(c + 1);
          t_pending = 1 + (int)((it + 1) & 1);
        }
        ptx::tc_fence_after();
        // dS = Delta~^T . K
        {
          int acc = 0;
#pragma unroll
          for (int pa = 0; pa < 3; ++pa)
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              mma_bf16_ts(tmem + 128, tmem + kTA + pa * 32 + kk * 8, ptx::desc_k128(ktt_u32 + kk * 32), idS, acc);
              acc = 1;
            }
          ptx::mma_commit(bar_mma);
        }
      }
      if (!ok) {
        set_err(p.err, kErrByteTimeout);
        // Let copies still in flight land before the CTA's memory goes away.
        if (kv_pending) ptx::mbar_wait(bar_kv, (uint32_t)(kv_pending - 1), lim);
        if (t_pending) ptx::mbar_wait(bar_t, (uint32_t)(t_pending - 1), lim);
      }
    }
  } else {
    // ------------------------------------------------- the epilogue warps
    const int wq = warp & 3, part = warp >> 2;
    const int e = wq * 32 + lane;  // state row = TMEM lane
    const uint32_t lb = (uint32_t)(wq * 32) << 16;
    const bool live = e < DK;      // rows past d_v stay zero
    float s[HC];                   // columns part*HC .. of row e
#pragma unroll
    for (int m = 0; m < HC; ++m) s[m] = amode && e == part * HC + m ? 1.f : 0.f;
    // The bf16 terms of the A operand go to TMEM, row e = lane e, two
    // elements per column.
    auto store_state = [&]() {
      uint32_t w[3][HC / 2];
#pragma unroll
      for (int g8 = 0; g8 < HC / 8; ++g8) {
        float x[8];
#pragma unroll
        for (int z = 0; z < 8; ++z) x[z] = s[8 * g8 + z];
        uint4 o[3];
        split3(x, o);
#pragma unroll
        for (int pl = 0; pl < 3; ++pl) {
          w[pl][4 * g8] = o[pl].x;
          w[pl][4 * g8 + 1] = o[pl].y;
          w[pl][4 * g8 + 2] = o[pl].z;
          w[pl][4 * g8 + 3] = o[pl].w;
        }
      }
#pragma unroll
      for (int pl = 0; pl < 3; ++pl) tmem_st<HC / 2>(tmem + lb + kTA + pl * (DK / 2) + part * (HC / 2), w[pl]);
    };
    auto store_tokens = [&](const float (&xt)[TT]) {  // Z^T or Delta~^T: row e, tokens part*TT ..
      uint32_t w[3][TT / 2];
#pragma unroll
      for (int g8 = 0; g8 < TT / 8; ++g8) {
        float x[8];
#pragma unroll
        for (int z = 0; z < 8; ++z) x[z] = xt[8 * g8 + z];
        uint4 o[3];
        split3(x, o);
#pragma unroll
        for (int pl = 0; pl < 3; ++pl) {
          w[pl][4 * g8] = o[pl].x;
          w[pl][4 * g8 + 1] = o[pl].y;
          w[pl][4 * g8 + 2] = o[pl].z;
          w[pl][4 * g8 + 3] = o[pl].w;
        }
      }
#pragma unroll
      for (int pl = 0; pl < 3; ++pl) tmem_st<TT / 2>(tmem + lb + kTA + pl * (kC / 2) + part * (TT / 2), w[pl]);
    };
    auto arrive = [&]() {
      ptx::tmem_st_wait();
      fence_proxy_async();  // K^T, written by these threads, is read by the tensor cores
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(bar_epi);
    };
    store_state();
    arrive();
    bool ok = true;
    uint32_t mph = 0;
    // K^T (and v^T) by 8x8 tiles: a warp moves 4 token tiles of one 8-column
    // block per step (a transposing load, a plain store).
    constexpr int KTS = DK / 64;  // steps per warp: (DK / 8) blocks x 2 token halves / 16 warps
    const uint32_t kt_u32e = ptx::smem_u32(base + LY::kt), ktt_u32e = ptx::smem_u32(base + LY::ktt);
    const uint32_t vt_u32e = ptx::smem_u32(base + LY::vt), vtt_u32e = ptx::smem_u32(base + LY::vtt);
#pragma unroll 1
    for (int c = c0; c < c1; ++c) {
      const uint32_t it = (uint32_t)(c - c0);
      if (ok) ok = ptx::mbar_wait(bar_kv, it & 1, lim);
#pragma unroll
      for (int q = 0; q < KTS; ++q) {
        const int ci = warp * KTS + q, nb = ci >> 1, ih = ci & 1;
        const int tk = lane >> 3, tr = lane & 7;
        uint32_t frag[4];
        ldsm_x4_trans(kt_u32e + (nb >> 3) * 8192 + ptx::swz128(ih * 32 + 8 * tk + tr, nb & 7), frag);
        stsm_x4(ktt_u32e + ptx::swz128(8 * nb + tr, ih * 4 + tk), frag);
        if (!amode) {
          ldsm_x4_trans(vt_u32e + (nb >> 3) * 8192 + ptx::swz128(ih * 32 + 8 * tk + tr, nb & 7), frag);
          stsm_x4(vtt_u32e + ptx::swz128(8 * nb + tr, ih * 4 + tk), frag);
        }
      }
      // v^T rows are read by the other epilogue warps: all 16 meet here (named
      // barrier 1; the load and MMA warp does not take part).  The next
      // chunk's transposes come only after every warp has arrived from its
      // Z^T stage, so nothing is overwritten while it is read.
      if (!amode) ptx::bar_sync(1, kEpiThreads);
      const float *gts = reinterpret_cast<const float *>(base + LY::gt + (it & 1) * kGateBytes);
      const int i0 = part * TT;
      // Z^T = (v - gamma . Y) beta, token-wise
      if (ok) ok = ptx::mbar_wait(bar_mma, mph & 1, lim);
      ++mph;
      if (ok) ok = ptx::mbar_wait(bar_t, it & 1, lim);
      ptx::tc_fence_after();
      float y[TT];
      ptx::tmem_ld16(tmem + lb + i0, y);
      ptx::tmem_ld_wait();
      {
        // v of row e for tokens i0 .. i0 + 15 from v^T (two 16-byte loads),
        // beta and gamma as float4.
        uint4 vv[2] = {make_uint4(0u, 0u, 0u, 0u), make_uint4(0u, 0u, 0u, 0u)};
        if (!amode && live) {
          vv[0] = *reinterpret_cast<const uint4 *>(base + LY::vtt + ptx::swz128(e, i0 >> 3));
          vv[1] = *reinterpret_cast<const uint4 *>(base + LY::vtt + ptx::swz128(e, (i0 >> 3) + 1));
        }
        const uint32_t vw[8] = {vv[0].x, vv[0].y, vv[0].z, vv[0].w, vv[1].x, vv[1].y, vv[1].z, vv[1].w};
#pragma unroll
        for (int x4 = 0; x4 < TT / 4; ++x4) {
          const float4 bq = reinterpret_cast<const float4 *>(gts + i0)[x4];
          const float4 gq = reinterpret_cast<const float4 *>(gts + kC + i0)[x4];
          const float bs[4] = {bq.x, bq.y, bq.z, bq.w}, gs[4] = {gq.x, gq.y, gq.z, gq.w};
#pragma unroll
          for (int z = 0; z < 4; ++z) {
            const int x = 4 * x4 + z;
            const uint32_t w = vw[x >> 1];
            const float v = __uint_as_float((x & 1) ? (w & 0xffff0000u) : (w << 16));
            y[x] = bs[z] * fmaf(-gs[z], y[x], v);
          }
        }
      }
      store_tokens(y);
      arrive();
      // Delta~^T = Delta^T diag(gamma_{C-1} / gamma_j)
      if (ok) ok = ptx::mbar_wait(bar_mma, mph & 1, lim);
      ++mph;
      ptx::tc_fence_after();
      ptx::tmem_ld16(tmem + lb + 64 + i0, y);
      ptx::tmem_ld_wait();
#pragma unroll
      for (int x4 = 0; x4 < TT / 4; ++x4) {
        const float4 rq = reinterpret_cast<const float4 *>(gts + 2 * kC + i0)[x4];
        y[4 * x4] *= rq.x;
        y[4 * x4 + 1] *= rq.y;
        y[4 * x4 + 2] *= rq.z;
        y[4 * x4 + 3] *= rq.w;
      }
      store_tokens(y);
      arrive();
      // S <- gamma_{C-1} S + dS
      if (ok) ok = ptx::mbar_wait(bar_mma, mph & 1, lim);
      ++mph;
      ptx::tc_fence_after();
      const float gC = gts[3 * kC];
#pragma unroll
      for (int q = 0; q < HC / 16; ++q) {
        float d[16];
        ptx::tmem_ld16(tmem + lb + 128 + part * HC + q * 16, d);
        ptx::tmem_ld_wait();
#pragma unroll
        for (int x = 0; x < 16; ++x) s[q * 16 + x] = fmaf(gC, s[q * 16 + x], d[x]);
      }
      if (c + 1 < c1) {
        store_state();
        arrive();
      }
    }
    if (!ok) set_err(p.err, kErrByteTimeout);
    if (live && ok) {
      float4 *dst = reinterpret_cast<float4 *>(p.units + ((((int64_t)(r * H + h) * gridDim.x + u) * DK + e) * DK +
                                                          part * HC));
#pragma unroll
      for (int m = 0; m < HC; m += 4) dst[m / 4] = make_float4(s[m], s[m + 1], s[m + 2], s[m + 3]);
    }
  }
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == kCtlWarp) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, kTmemCols);
  }
}

// --------------------------------------------------------------- combine
// S = ((B_0 A_1 + B_1) A_2 + B_2) ..., fp32.  A CTA takes 16 rows of S with
// 16 warps: warp w the columns [DK/8 (w % 8), DK/8 (w % 8 + 1)) and the
// half w / 8 of the sum over m, a thread 2 rows x 4 columns of them, so that
// per step a warp reads one 16-byte piece of A_s per lane group and one pair
// of X per row group; the two halves of the sum meet in shared memory.  Each
// A_s is staged in shared memory (copies in flight while the previous one is
// in use); B_s is read one step ahead.  Written in the state's type.
constexpr int kCombThreads = 512;
template <int DK>
struct CombineShape {
  static constexpr int RB = 16;            // rows of S per CTA
  static constexpr int CW = DK / 8;        // columns per warp
  static constexpr int NQ = CW / 4;        // 4-column groups per warp (lanes: NQ x row pairs)
  static constexpr int RG = 32 / NQ;       // row pairs per warp
  static_assert(2 * RG >= RB, "rows per warp");
  static constexpr size_t smem = (2u * DK * DK + (size_t)DK * RB + 2u * 256u * 4u) * sizeof(float);
};

template <int DK, typename TS>
__global__ void __launch_bounds__(kCombThreads) prefill_combine_kernel(const float *units, TS *S0, int H, int nseg) {
  using CS = CombineShape<DK>;
  extern __shared__ __align__(16) float cb_smem[];
  float *Abuf = cb_smem;                       // [2][DK][DK]
  float *Xt = cb_smem + 2 * DK * DK;           // X transposed: [DK][RB]
  float4 *part = reinterpret_cast<float4 *>(Xt + DK * CS::RB);  // second half's sums [256][2]
  const int h = blockIdx.y, r = blockIdx.z, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int kh = warp >> 3, w8 = warp & 7, slot = tid & 255;
  const int q = lane % CS::NQ, rg = lane / CS::NQ;
  const bool act = 2 * rg < CS::RB;
  const int col = w8 * CS::CW + 4 * q;                // first of the thread's 4 columns
  const int e0 = blockIdx.x * CS::RB + 2 * rg;        // first of its 2 rows
  const int m0 = kh * (DK / 2);
  const int nu = 2 * nseg - 1;
  const float *U = units + (int64_t)(r * H + h) * nu * DK * DK;
  auto stage = [&](int sg, int buf) {
    const float *A = U + (int64_t)(2 * sg - 1) * DK * DK;
    for (int e = tid; e < DK * DK / 4; e += kCombThreads)
      ptx::cp_async16(Abuf + buf * DK * DK + 4 * e, A + 4 * e, 16u);
    ptx::cp_async_commit();
  };
  auto rows = [&](int u, float4 &a, float4 &b) {
    if (act && kh == 0) {
      a = *reinterpret_cast<const float4 *>(U + ((int64_t)u * DK + e0) * DK + col);
      b = *reinterpret_cast<const float4 *>(U + ((int64_t)u * DK + e0 + 1) * DK + col);
    }
  };
  float4 x0 = make_float4(0.f, 0.f, 0.f, 0.f), x1 = x0, b0 = x0, b1 = x0;
  rows(0, x0, x1);
  if (nseg > 1) {
    stage(1, 0);
    rows(2, b0, b1);
  }
#pragma unroll 1
  for (int sg = 1; sg < nseg; ++sg) {
    const int buf = (sg - 1) & 1;
    if (act && kh == 0) {
      const float v0[4] = {x0.x, x0.y, x0.z, x0.w}, v1[4] = {x1.x, x1.y, x1.z, x1.w};
#pragma unroll
      for (int z = 0; z < 4; ++z)
        *reinterpret_cast<float2 *>(Xt + (col + z) * CS::RB + 2 * rg) = make_float2(v0[z], v1[z]);
    }
    if (sg + 1 < nseg) {
      stage(sg + 1, buf ^ 1);
      ptx::cp_async_wait_group1();
    } else {
      ptx::cp_async_wait_all();
    }
    __syncthreads();
    float4 a0 = kh == 0 ? b0 : make_float4(0.f, 0.f, 0.f, 0.f), a1 = kh == 0 ? b1 : a0;
    if (sg + 1 < nseg) rows(2 * sg + 2, b0, b1);
    const float *As = Abuf + buf * DK * DK;
    if (act) {
#pragma unroll 8
      for (int m = m0; m < m0 + DK / 2; ++m) {
        const float2 u = *reinterpret_cast<const float2 *>(Xt + m * CS::RB + 2 * rg);
        const float4 av = *reinterpret_cast<const float4 *>(As + m * DK + col);
        a0.x = fmaf(u.x, av.x, a0.x);
        a0.y = fmaf(u.x, av.y, a0.y);
        a0.z = fmaf(u.x, av.z, a0.z);
        a0.w = fmaf(u.x, av.w, a0.w);
        a1.x = fmaf(u.y, av.x, a1.x);
        a1.y = fmaf(u.y, av.y, a1.y);
        a1.z = fmaf(u.y, av.z, a1.z);
        a1.w = fmaf(u.y, av.w, a1.w);
      }
      if (kh == 1) {
        part[2 * slot] = a0;
        part[2 * slot + 1] = a1;
      }
    }
    __syncthreads();  // X, this buffer and the second half's sums
    if (act && kh == 0) {
      const float4 p0 = part[2 * slot], p1 = part[2 * slot + 1];
      x0 = make_float4(a0.x + p0.x, a0.y + p0.y, a0.z + p0.z, a0.w + p0.w);
      x1 = make_float4(a1.x + p1.x, a1.y + p1.y, a1.z + p1.z, a1.w + p1.w);
    }
  }
  if (!act || kh != 0) return;
  const float4 xs[2] = {x0, x1};
#pragma unroll
  for (int hh = 0; hh < 2; ++hh) {
    TS *out = S0 + ((int64_t)(r * H + h) * DK + e0 + hh) * DK + col;
    if constexpr (sizeof(TS) == 4) {
      *reinterpret_cast<float4 *>(out) = xs[hh];
    } else {
      *reinterpret_cast<uint2 *>(out) = make_uint2(pack_bf16x2(xs[hh].x, xs[hh].y), pack_bf16x2(xs[hh].z, xs[hh].w));
    }
  }
}

template <int DK>
cudaError_t launch_dk(const void *k, const void *v, const float *g, const float *beta, void *S0, int R, int L, int H,
                      int s0_bf16, int nseg, uint8_t *ws, unsigned long long wait_ns, int32_t *err, cudaStream_t s) {
  const int nchunks = (L + kC - 1) / kC;
  const int cps = (nchunks + nseg - 1) / nseg;
  nseg = (nchunks + cps - 1) / cps;  // every segment holds at least one chunk
  const int nu = 2 * nseg - 1;
  uint8_t *prep = ws;
  float *units = reinterpret_cast<float *>(ws + prefill_tc_prep_bytes(R, L, H));

  {
    PrepParams pp = {};
    if (!encode_rows(&pp.tm_k, k, DK, H, L, R, kPrepChunks * kC)) return cudaErrorInvalidValue;
    pp.g = g;
    pp.beta = beta;
    pp.ws = prep;
    pp.L = L;
    pp.H = H;
    pp.nchunks = nchunks;
    pp.wait_limit_ns = wait_ns;
    pp.err = err;
    const size_t psmem = PrepLayout<DK>::total + 1024;
    cudaError_t e0 = ensure_smem_limit((const void *)prefill_prep_kernel<DK>, psmem);
    if (e0 != cudaSuccess) return e0;
    prefill_prep_kernel<DK><<<dim3((nchunks + kPrepChunks - 1) / kPrepChunks, H, R), kPrepThreads, psmem, s>>>(pp);
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;

  ChainParams p = {};
  if (!encode_rows(&p.tm_k, k, DK, H, L, R, kC) || !encode_rows(&p.tm_v, v, DK, H, L, R, kC))
    return cudaErrorInvalidValue;
  p.prep = prep;
  p.units = units;
  p.H = H;
  p.nchunks = nchunks;
  p.cps = cps;
  p.wait_limit_ns = wait_ns;
  p.err = err;
  const size_t csmem = ChainLayout<DK>::total + 1024;
  if ((e = ensure_smem_limit((const void *)prefill_chain_kernel<DK>, csmem)) != cudaSuccess) return e;
  prefill_chain_kernel<DK><<<dim3(nu, H, R), kChainThreads, csmem, s>>>(p);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;

  using CS = CombineShape<DK>;
  const dim3 cgrid(DK / CS::RB, H, R);
  if (s0_bf16) {
    if ((e = ensure_smem_limit((const void *)prefill_combine_kernel<DK, __nv_bfloat16>, CS::smem)) != cudaSuccess)
      return e;
    prefill_combine_kernel<DK, __nv_bfloat16>
        <<<cgrid, kCombThreads, CS::smem, s>>>(units, static_cast<__nv_bfloat16 *>(S0), H, nseg);
  } else {
    if ((e = ensure_smem_limit((const void *)prefill_combine_kernel<DK, float>, CS::smem)) != cudaSuccess) return e;
    prefill_combine_kernel<DK, float><<<cgrid, kCombThreads, CS::smem, s>>>(units, static_cast<float *>(S0), H, nseg);
  }
  return cudaGetLastError();
}

}  // namespace

bool prefill_tc_supports(int dk, int dv, int qkv_bf16) { return qkv_bf16 && dk == dv && (dk == 64 || dk == 128); }

int prefill_tc_segments(int R, int L, int H, int want) {
  const int nchunks = (L + kC - 1) / kC;
  int nseg = want;
  if (nseg <= 0) {
    // One CTA per segment unit on the 148 SMs, at least 4 chunks per segment.
    const int units = 148 / (R * H > 0 ? R * H : 1);
    nseg = (units + 1) / 2;
    nseg = min(nseg, max(1, nchunks / 4));
  }
  nseg = max(1, min(nseg, min(nchunks, kMaxPrefillSegments)));
  const int cps = (nchunks + nseg - 1) / nseg;
  return (nchunks + cps - 1) / cps;
}

size_t prefill_tc_prep_bytes(int R, int L, int H) {
  const size_t nchunks = (size_t)((L + kC - 1) / kC);
  return ((size_t)R * H * nchunks * kPrepBytes + 1023) & ~(size_t)1023;
}

size_t prefill_tc_ws_bytes(int R, int L, int H, int d, int nseg) {
  return prefill_tc_prep_bytes(R, L, H) + (size_t)R * H * (2 * nseg - 1) * d * d * sizeof(float);
}

cudaError_t launch_prefill_tc(const void *k, const void *v, const float *g, const float *beta, void *S0, int R, int L,
                              int H, int d, int s0_bf16, int nseg, void *ws, unsigned long long wait_ns, int32_t *err,
                              cudaStream_t s) {
  if (L < 1 || R < 1 || H < 1 || nseg < 1 || !ws) return cudaErrorInvalidValue;
  uint8_t *w = static_cast<uint8_t *>(ws);
  if (d == 64) return launch_dk<64>(k, v, g, beta, S0, R, L, H, s0_bf16, nseg, w, wait_ns, err, s);
  if (d == 128) return launch_dk<128>(k, v, g, beta, S0, R, L, H, s0_bf16, nseg, w, wait_ns, err, s);
  return cudaErrorNotSupported;
}

}  // namespace onela
