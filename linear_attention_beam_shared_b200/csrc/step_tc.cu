// Tensor-core decode-step kernel (tcgen05, sm_100a) for bf16 q/k/v and
// d_k = d_v in {64, 128}.
//
// One CTA per (request r, head h, tile of 32 beams); 256 threads.  The step
// of the shared-state GDN beam decode (OneLA, evolve.pub review, key claims
// on section 3.2, equations 2-4) becomes two small dense contractions on the
// tensor cores plus a SIMT epilogue:
//
//   D1 = S0 . X^T    S0 [d_v x d_k] (M = 128, rows beyond d_v are zero) times
//                    the tile's 64 vectors X = [k_0..k_31; q_0..q_31]
//                    (N = 64, K = d_k).  S0 is the shared prompt state: its
//                    operand image is read once per CTA and used by every
//                    beam of the tile (abstract: "reuses the shared state
//                    across beams").
//   D2 = KA . X^T    KA = the tile's own keys (rows 0..31) followed by the
//                    distinct ancestor keys of the tile's beams (rows 32..),
//                    so D2 holds every dot product k_j . x the projection
//                    replay needs plus k_b . q_b.
//
// fp32 S0 is split once (when the prompt state is installed) into two or
// three bf16 terms S0 = hi + mid (+ lo); each term is one more pass of D1
// (bf16 x bf16 products are exact in the fp32 accumulator).
//
// The epilogue (TMEM lane i = row i of S0, i.e. output element i) forms
//   u_x = G (S0 x) + sum_j w_j (k_j . x) delta_j          x in {k_b, q_b}
//   delta_b = beta_b (v_b - alpha_b u_k),  o_b = alpha_b u_q + delta_b (k_b . q_b)
// reading each ancestor delta_j row with coalesced loads, and appends the
// record (alpha_b, delta_b, k_b) (review, Summary: records replayed "in
// vector form without ever materializing a per-beam matrix").
//
// The ancestry update (abstract: "lightweight ancestry index ... without
// moving or copying existing records") runs in warp 0: a beam's row is its
// parent's row plus the parent; parents are range-checked, and distinct
// ancestors are found with a warp-wide match so each ancestor key is staged
// once per CTA.
#include <cuda_bf16.h>

#include "internal.h"
#include "sm100_ptx.h"

namespace onela {
namespace {

constexpr int kThreads = 256;
constexpr int kBT = 32;            // beams per CTA
constexpr int kN = 2 * kBT;        // MMA N: k vectors then q vectors
constexpr int kM = 128;            // MMA M
constexpr int kTmemCols = 128;     // D1: columns [0, 64), D2: [64, 128)
constexpr int kTableStride = kN + 1;
constexpr int kMaxT = 32;          // deepest decode the kernel serves
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s: far beyond any legal wait
constexpr int32_t kErrTimeout = 2;

struct Smem {
  // byte offsets from the 1024-aligned base
  uint32_t s0, x, ka, table, book, total;
};

__host__ __device__ inline Smem smem_layout(int nk, int planes, int TM) {
  Smem s;
  s.s0 = 0;
  s.x = s.s0 + (uint32_t)planes * nk * 16384u;
  s.ka = s.x + (uint32_t)nk * 8192u;
  s.table = s.ka + (uint32_t)nk * 16384u;
  s.book = s.table + (uint32_t)kM * kTableStride * 4u;
  // book: 2 mbarriers + tmem addr (32 B), then per-beam arrays
  const uint32_t per_beam = (uint32_t)kBT * TM * 4u;
  s.total = s.book + 64u + 5u * per_beam + 4u * kBT * 4u + (uint32_t)(kBT * TM + kBT) * 4u + 16u;
  return s;
}

template <int DK>
__global__ void __launch_bounds__(kThreads, 1) step_tc_kernel(const StepParams p) {
  constexpr int NK = DK / 64;  // 128-byte K atoms per row
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_u32 = ptx::smem_u32(smem_raw);
  uint8_t *base = smem_raw + ((1024u - (raw_u32 & 1023u)) & 1023u);

  const int tile = blockIdx.x, h = blockIdx.y, r = blockIdx.z;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int b0 = tile * kBT;
  const int nb = min(kBT, p.W - b0);
  const int dv = p.dv, H = p.H, t = p.t, TM = p.T_max, P = p.s0_planes;
  const int nanc = t - 1;

  const Smem L = smem_layout(NK, P, TM);
  uint8_t *s_s0 = base + L.s0;
  uint8_t *s_x = base + L.x;
  uint8_t *s_ka = base + L.ka;
  float *s_table = reinterpret_cast<float *>(base + L.table);
  uint64_t *bar_load = reinterpret_cast<uint64_t *>(base + L.book);
  uint64_t *bar_mma = bar_load + 1;
  uint32_t *s_tmem = reinterpret_cast<uint32_t *>(bar_load + 2);
  int *s_U = reinterpret_cast<int *>(s_tmem + 1);
  int *s_chain = reinterpret_cast<int *>(base + L.book + 64);  // [BT][TM]
  int *s_slot = s_chain + kBT * TM;                            // [BT][TM]
  float *s_w = reinterpret_cast<float *>(s_slot + kBT * TM);   // [BT][TM]
  float *s_ck = s_w + kBT * TM;                                // [BT][TM]
  float *s_cq = s_ck + kBT * TM;                               // [BT][TM]
  float *s_G = s_cq + kBT * TM;                                // [BT]
  float *s_alpha = s_G + kBT;
  float *s_beta = s_alpha + kBT;
  float *s_kq = s_beta + kBT;
  int *s_list = reinterpret_cast<int *>(s_kq + kBT);  // packed (beam << 6 | depth-1), by slot

  const __nv_bfloat16 *q = static_cast<const __nv_bfloat16 *>(p.q);
  const __nv_bfloat16 *k = static_cast<const __nv_bfloat16 *>(p.k);
  const __nv_bfloat16 *v = static_cast<const __nv_bfloat16 *>(p.v);
  __nv_bfloat16 *rec_k = static_cast<__nv_bfloat16 *>(p.rec_k);

  // ---- setup: barriers, TMEM
  if (tid == 0) {
    ptx::mbar_init(bar_load, 1);
    ptx::mbar_init(bar_mma, 1);
    ptx::mbar_fence_init();
  }
  if (warp == 0) {
    ptx::tmem_alloc(s_tmem, kTmemCols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *s_tmem;

  // ---- S0 operand image (planes x K atoms x 128 rows x 128 B) by bulk copy
  const uint32_t s0_bytes = (uint32_t)P * NK * 16384u;
  if (tid == 0) {
    ptx::mbar_arrive_expect_tx(bar_load, s0_bytes);
    const uint8_t *src = static_cast<const uint8_t *>(p.S0img) + (size_t)(r * H + h) * s0_bytes;
    for (uint32_t off = 0; off < s0_bytes; off += 16384u) ptx::bulk_g2s(s_s0 + off, src + off, 16384u, bar_load);
  }

  // ---- X tile (k rows 0..31, q rows 32..63), record k, own keys into KA
  for (int e = tid; e < kN * NK * 8; e += kThreads) {
    const int n = e / (NK * 8), cc = e - n * (NK * 8);
    const int ka = cc >> 3, c = cc & 7;
    const int bb = n & (kBT - 1);
    const bool is_q = n >= kBT;
    uint4 val = make_uint4(0u, 0u, 0u, 0u);
    if (bb < nb) {
      const int64_t row = (int64_t)(r * p.W + b0 + bb) * H + h;
      const uint4 *src = reinterpret_cast<const uint4 *>((is_q ? q : k) + row * DK) + cc;
      val = __ldg(src);
      if (!is_q) reinterpret_cast<uint4 *>(rec_k + rec_row(p, t, r, h, b0 + bb) * DK)[cc] = val;
    }
    *reinterpret_cast<uint4 *>(s_x + ka * (kN * 128) + ptx::swz128(n, c)) = val;
    if (!is_q) *reinterpret_cast<uint4 *>(s_ka + ka * (kM * 128) + ptx::swz128(bb, c)) = val;
  }

  // ---- ancestry, gates, distinct ancestors (warp 0, one lane per beam)
  if (warp == 0) {
    const int b = lane;
    const bool valid = b < nb;
    float G = 1.f, alpha = 0.f, beta = 0.f;
    int *chain = s_chain + b * TM;
    if (valid) {
      const int gb = b0 + b;
      int par = p.parents[r * p.W + gb];
      if (par < 0 || par >= p.W_prev) {
        *reinterpret_cast<volatile int32_t *>(p.err) = kErrParent;
        par = 0;
      }
      if (nanc >= 1) {
        chain[nanc - 1] = par;
        if (nanc >= 2) {
          const int32_t *prow = p.anc + anc_row(p, t - 1, r, par);
          for (int j = 0; j < nanc - 1; ++j) chain[j] = prow[j];
        }
        if (h == 0) {
          int32_t *row = p.anc + anc_row(p, t, r, gb);
          for (int j = 0; j < nanc; ++j) row[j] = chain[j];
        }
      }
      float run = 1.f;
      for (int j = nanc - 1; j >= 0; --j) {
        s_w[b * TM + j] = run;
        run *= p.rec_alpha[rec_row(p, j + 1, r, h, chain[j])];
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
    // Distinct (depth, beam) ancestors; slots 0..31 are the tile's own keys.
    int U = kBT;
    for (int j = 0; j < nanc; ++j) {
      const int a = valid ? chain[j] : -1;
      const unsigned same = __match_any_sync(0xffffffffu, a);
      const int leader = __ffs(same) - 1;
      const bool lead = valid && leader == lane;
      const unsigned leaders = __ballot_sync(0xffffffffu, lead);
      const int my = U + __popc(leaders & ((1u << lane) - 1u));
      if (lead) s_list[my] = (a << 6) | j;
      const int slot = __shfl_sync(0xffffffffu, my, leader);
      if (valid) s_slot[b * TM + j] = slot;
      U += __popc(leaders);
    }
    if (lane == 0) *s_U = U;
  }
  __syncthreads();
  const int U = *s_U;

  // ---- blocks of up to 128 KA rows: stage ancestor keys, run the MMAs
  const uint32_t idesc = ptx::idesc_bf16_f32(kM, kN);
  const uint32_t x_u32 = ptx::smem_u32(s_x), ka_u32 = ptx::smem_u32(s_ka), s0_u32 = ptx::smem_u32(s_s0);
  bool ok = true;
  const int nblocks = (U + kM - 1) / kM;
  for (int blk = 0; blk < nblocks; ++blk) {
    const int row0 = blk == 0 ? kBT : 0;
    const int nrows = min(kM, U - blk * kM);
    if (blk > 0) __syncthreads();  // previous block's table fully consumed
    for (int e = tid; e < (nrows - row0) * NK * 8; e += kThreads) {
      const int lr = row0 + e / (NK * 8), cc = e % (NK * 8);
      const int packed = s_list[blk * kM + lr];
      const int beam = packed >> 6, depth = (packed & 63) + 1;
      const uint4 val =
          __ldg(reinterpret_cast<const uint4 *>(rec_k + rec_row(p, depth, r, h, beam) * DK) + cc);
      *reinterpret_cast<uint4 *>(s_ka + (cc >> 3) * (kM * 128) + ptx::swz128(lr, cc & 7)) = val;
    }
    ptx::fence_proxy_async_smem();
    __syncthreads();
    if (tid == 0) {
      ptx::tc_fence_after();
      if (blk == 0) {
        ok = ptx::mbar_wait(bar_load, 0, kWaitLimitNs);
        ptx::tc_fence_after();
        int acc = 0;
        for (int pl = 0; pl < P; ++pl)
          for (int ka = 0; ka < NK; ++ka)
            for (int kk = 0; kk < 4; ++kk) {
              const uint64_t a = ptx::desc_k128(s0_u32 + (pl * NK + ka) * 16384 + kk * 32);
              const uint64_t bd = ptx::desc_k128(x_u32 + ka * (kN * 128) + kk * 32);
              ptx::mma_bf16(tmem, a, bd, idesc, acc);
              acc = 1;
            }
      }
      for (int ka = 0; ka < NK; ++ka)
        for (int kk = 0; kk < 4; ++kk) {
          const uint64_t a = ptx::desc_k128(ka_u32 + ka * (kM * 128) + kk * 32);
          const uint64_t bd = ptx::desc_k128(x_u32 + ka * (kN * 128) + kk * 32);
          ptx::mma_bf16(tmem + kN, a, bd, idesc, (ka | kk) != 0);
        }
      ptx::mma_commit(bar_mma);
    }
    // Everyone waits for this block's MMAs.
    if (!ptx::mbar_wait(bar_mma, blk & 1, kWaitLimitNs)) ok = false;
    ptx::tc_fence_after();
    // D2 rows -> table (warps 0..3: TMEM lanes 0..127 = KA rows).
    if (warp < 4) {
      const int lr = warp * 32 + lane;
#pragma unroll
      for (int c0 = 0; c0 < kN; c0 += 16) {
        float vals[16];
        ptx::tmem_ld16(tmem + ((uint32_t)(warp * 32) << 16) + kN + c0, vals);
        ptx::tmem_ld_wait();
        if (lr < nrows) {
#pragma unroll
          for (int c = 0; c < 16; ++c) s_table[lr * kTableStride + c0 + c] = vals[c];
        }
      }
    }
    ptx::tc_fence_before();
    __syncthreads();
    // Coefficients of the slots that fall in this block.
    if (warp == 0 && lane < nb) {
      const int b = lane;
      if (blk == 0) s_kq[b] = s_table[b * kTableStride + kBT + b];
      for (int j = 0; j < nanc; ++j) {
        const int s = s_slot[b * TM + j] - blk * kM;
        if (s >= 0 && s < kM) {
          const float w = s_w[b * TM + j];
          s_ck[b * TM + j] = w * s_table[s * kTableStride + b];
          s_cq[b * TM + j] = w * s_table[s * kTableStride + kBT + b];
        }
      }
    }
  }
  if (!ok && tid == 0) *reinterpret_cast<volatile int32_t *>(p.err) = kErrTimeout;
  __syncthreads();

  // ---- epilogue: warp w serves TMEM lanes 32*(w%4).. and beams 16*(w/4)..
  {
    const int i = (warp & 3) * 32 + lane;  // output element (row of S0)
    const int half = warp >> 2;
    float uk[16], uq[16];
    ptx::tc_fence_after();
    ptx::tmem_ld16(tmem + ((uint32_t)((warp & 3) * 32) << 16) + half * 16, uk);
    ptx::tmem_ld16(tmem + ((uint32_t)((warp & 3) * 32) << 16) + kBT + half * 16, uq);
    ptx::tmem_ld_wait();
    if (i < dv && ok) {
#pragma unroll
      for (int m = 0; m < 16; ++m) {
        const int b = half * 16 + m;
        if (b >= nb) continue;
        const int gb = b0 + b;
        float xk = s_G[b] * uk[m];
        float xq = s_G[b] * uq[m];
        for (int j = 0; j < nanc; ++j) {
          const int a = s_chain[b * TM + j];
          const float d = __ldg(p.rec_delta + rec_row(p, j + 1, r, h, a) * dv + i);
          xk = fmaf(s_ck[b * TM + j], d, xk);
          xq = fmaf(s_cq[b * TM + j], d, xq);
        }
        const int64_t vi = ((int64_t)(r * p.W + gb) * H + h) * dv + i;
        const float alpha = s_alpha[b];
        const float delta = s_beta[b] * (__bfloat162float(v[vi]) - alpha * xk);
        p.o[vi] = fmaf(alpha, xq, delta * s_kq[b]);
        p.rec_delta[rec_row(p, t, r, h, gb) * dv + i] = delta;
      }
    }
  }

  // ---- teardown
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 0) ptx::tmem_dealloc(tmem, kTmemCols);
}

__global__ void s0_image_kernel(const void *S0, uint4 *img, int R, int H, int dk, int dv, int s0_bf16,
                                int planes) {
  // One thread per (r, h, plane, K atom, row < 128, 16-byte chunk).
  const int nk = dk / 64;
  const int64_t total = (int64_t)R * H * planes * nk * kM * 8;
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < total;
       e += (int64_t)gridDim.x * blockDim.x) {
    int64_t x = e;
    const int c = (int)(x % 8); x /= 8;
    const int row = (int)(x % kM); x /= kM;
    const int ka = (int)(x % nk); x /= nk;
    const int pl = (int)(x % planes); x /= planes;
    const int64_t rh = x;
    __align__(16) __nv_bfloat16 out[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      float s = 0.f;
      if (row < dv) {
        const int64_t si = (rh * dv + row) * dk + ka * 64 + c * 8 + u;
        s = s0_bf16 ? __bfloat162float(static_cast<const __nv_bfloat16 *>(S0)[si])
                    : static_cast<const float *>(S0)[si];
      }
      // Term pl of the split s = hi + mid + lo (each the bf16 rounding of
      // what the earlier terms leave; the differences are exact in fp32).
      float rest = s;
      __nv_bfloat16 term = __float2bfloat16_rn(rest);
      for (int k2 = 0; k2 < pl; ++k2) {
        rest = rest - __bfloat162float(term);
        term = __float2bfloat16_rn(rest);
      }
      out[u] = term;
    }
    const int64_t off = ((rh * planes + pl) * nk + ka) * (kM * 128) + ptx::swz128(row, c);
    img[off / 16] = *reinterpret_cast<const uint4 *>(out);
  }
}

}  // namespace

bool tc_supports(int dk, int dv, int qkv_bf16, int T_max) {
  return qkv_bf16 && dk == dv && (dk == 64 || dk == 128) && T_max <= kMaxT;
}

size_t s0_image_bytes(int R, int H, int dk, int dv, int planes) {
  (void)dv;
  return (size_t)R * H * planes * (dk / 64) * 16384u;
}

cudaError_t launch_s0_image(const void *S0, void *img, int R, int H, int dk, int dv, int s0_bf16, int planes,
                            cudaStream_t s) {
  const int64_t total = (int64_t)R * H * planes * (dk / 64) * kM * 8;
  const int threads = 256;
  const int blocks = (int)((total + threads - 1) / threads < 148 * 16 ? (total + threads - 1) / threads : 148 * 16);
  s0_image_kernel<<<blocks, threads, 0, s>>>(S0, static_cast<uint4 *>(img), R, H, dk, dv, s0_bf16, planes);
  return cudaGetLastError();
}

template <int DK>
static cudaError_t launch_dk(const StepParams &p, cudaStream_t s) {
  const Smem L = smem_layout(DK / 64, p.s0_planes, p.T_max);
  const size_t smem = L.total + 1024;
  static size_t configured[64] = {0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (smem > configured[dev]) {
    e = cudaFuncSetAttribute(step_tc_kernel<DK>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    configured[dev] = smem;
  }
  dim3 grid((p.W + kBT - 1) / kBT, p.H, p.R);
  step_tc_kernel<DK><<<grid, kThreads, smem, s>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_step_tc(const StepParams &p, int s0_bf16, cudaStream_t s) {
  (void)s0_bf16;
  if (p.T_max > kMaxT || p.s0_planes < 1 || p.s0_planes > 3) return cudaErrorNotSupported;
  if (p.dk == 64 && p.dv == 64) return launch_dk<64>(p, s);
  if (p.dk == 128 && p.dv == 128) return launch_dk<128>(p, s);
  return cudaErrorNotSupported;
}

}  // namespace onela
