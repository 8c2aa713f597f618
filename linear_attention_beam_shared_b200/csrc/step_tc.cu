// Tensor-core decode-step kernel (tcgen05, sm_100a) for bf16 q/k/v and
// d_k = d_v in {64, 128}.
//
// One CTA per (request r, head h, tile of 32 beams); 256 threads; two CTAs
// fit on an SM, so a step launched as a programmatic dependent runs its
// input phase beside the previous step.  The step of the shared-state GDN
// beam decode (OneLA, evolve.pub review, key claims on section 3.2,
// equations 2-4) runs as dense products on the tensor cores, fp32
// accumulators in TMEM:
//
//   D1  = S0 . X^T      S0 k_b and S0 q_b for the tile's 64 vectors
//                       X = [k_0..k_31; q_0..q_31].  The S0 operand image is
//                       read once per CTA and used by every beam of the tile
//                       (abstract: "reuses the shared state across beams");
//                       fp32 S0 is split once, when the prompt state is
//                       installed, into two or three bf16 terms.
//   Dkq = X . K^T       gives k_b . q_b.
//   D2  = X . KA^T      k_a . x for every vector x and every distinct
//                       ancestor a of the tile (KA: their keys).
//   D1 += Delta'^T . C  the projection replay (review, Summary: records
//                       replayed "in vector form without ever materializing a
//                       per-beam matrix").  With P(a) the product of the
//                       gates on the path from the root to record a (kept in
//                       the record store), the weight of record a in the
//                       replay of a beam whose parent is p is P(p) / P(a), so
//                         S_{t-1} x = P(p) [ S0 x + sum_a (delta_a / P(a)) (k_a . x) ]
//                       over the beam's ancestors a.  Delta' holds
//                       delta_a / P(a); C[x][a] is k_a . x where a is an
//                       ancestor of x's beam and 0 elsewhere.  Delta' and C
//                       are split into fp16 hi + lo terms; the passes hi.hi,
//                       hi.lo and lo.hi keep fp32-level accuracy.
//
// The epilogue (TMEM lane i = output element i) forms u_x = P(p) D1_x,
// delta_b = beta_b (v_b - alpha_b u_k), o_b = alpha_b u_q + delta_b (k_b . q_b),
// and appends the record (alpha_b, delta_b, k_b) with P(b) = P(p) alpha_b.
//
// The ancestry (abstract: "lightweight ancestry index ... without moving or
// copying existing records"): beam b with parent p, grandparent g = the
// parent of p at step t-1, has the ancestor row [row of g at depth t-2, g, p].
// The kernel signals its dependents only after its own griddepcontrol.wait,
// so when step t starts, step t-2 has completed: before its wait, step t
// reads only inputs (S0 image, q, k, v, g, beta, parents of steps t and t-1)
// and what steps up to t-2 wrote (ancestor rows of depth t-2).  There it
// stages X, runs D1 and Dkq, forms every beam's ancestor row and finds the
// tile's distinct ancestors with warp-wide matches (parents first, then one
// warp per depth).  After the wait one round of loads stages all the distinct
// ancestors' records (keys, deltas, P) once per CTA.  Every global write
// happens after the wait, so a step never overwrites records that the step
// before it may still be reading.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cudaTypedefs.h>

#include "internal.h"
#include "sm100_ptx.h"

namespace onela {
namespace {

constexpr int kThreads = 256;       // 8 warps
constexpr int kBT = 32;             // beams per CTA
constexpr int kN = 2 * kBT;         // vectors: k rows 0..31, q rows 32..63
constexpr int kM = 128;             // MMA M
constexpr int kBlk = 64;            // distinct ancestors per staging block
constexpr int kTmemCols = 256;      // D1 [0,64), D2 [64,128), Dkq [128,160)
constexpr int kMaxT = 16;           // deepest decode the kernel serves
constexpr int kMaxW = 1024;         // widest beam set the kernel serves
constexpr int kSliceMax = 4096;     // ancestor-row slice copied to shared memory when
                                    // W_max * T_max fits (ints); otherwise rows are gathered
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s: far beyond any legal wait
constexpr int32_t kErrTimeout = 2;

struct Layout {
  uint32_t x;                        // X [NK][128 rows][128 B]: k, q, k, q
  uint32_t a;                        // S0 image, then the block operands
  uint32_t ka, dhi, dlo, chi, clo;   // block operands inside region a
  uint32_t book;                     // barriers and bookkeeping
  uint32_t total;
};

__host__ __device__ inline bool use_slice(int W_max, int TM) { return W_max * TM <= kSliceMax; }

__host__ __device__ inline Layout layout(int nk, int planes, int TM, int W_max) {
  Layout L;
  L.x = 0;
  L.a = (uint32_t)nk * 16384u;
  L.ka = L.a;                                // [NK][64 rows][128 B]
  L.dhi = L.ka + (uint32_t)nk * 8192u;       // [2 M-atoms][8 groups][8 rows][128 B]
  L.dlo = L.dhi + 16384u;
  L.chi = L.dlo + 16384u;                    // [64 rows][128 B]
  L.clo = L.chi + 8192u;
  const uint32_t post_end = L.clo + 8192u;
  const uint32_t pre_end = L.a + (uint32_t)planes * nk * 16384u;
  L.book = post_end > pre_end ? post_end : pre_end;
  // 64 B barriers/counters; 5 per-beam scalars; chain, slot [32][TM];
  // list [32 * TM]; per-depth counts [TM]; the previous step's parents
  // [W_max]; the ancestor-row slice of depth t-2 [W_max][TM] if it fits.
  L.total = L.book + 64u + 5u * kBT * 4u + 3u * kBT * TM * 4u + (uint32_t)(TM + 4) * 4u + (uint32_t)W_max * 4u +
            (use_slice(W_max, TM) ? (uint32_t)W_max * TM * 4u : 0u) + 16u;
  return L;
}

__device__ __forceinline__ void split_f16(float x, __half &hi, __half &lo) {
  hi = __float2half_rn(x);
  lo = __float2half_rn(x - __half2float(hi));
}

template <int DK>
__global__ void __launch_bounds__(kThreads, 2) step_tc_kernel(const __grid_constant__ StepParams p) {
  constexpr int NK = DK / 64;  // 128-byte K atoms per key row
  constexpr int DV = DK;
  constexpr int C4 = DV / 4;   // float4 chunks per delta row
  constexpr int XA = 2 * kN * 128;  // bytes of one K atom of X (128 rows)
  constexpr int NF = kBlk * C4 / kThreads;  // delta float4 chunks per thread per block
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_u32 = ptx::smem_u32(smem_raw);
  uint8_t *base = smem_raw + ((1024u - (raw_u32 & 1023u)) & 1023u);

  const int tile = blockIdx.x, h = blockIdx.y, r = blockIdx.z;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int b0 = tile * kBT;
  const int nb = min(kBT, p.W - b0);
  const int H = p.H, t = p.t, TM = p.T_max, P = p.s0_planes;
  const int nanc = t - 1;
  const int jp = nanc - 1;  // depth index of the parents (depth t-1)
  const bool slice = use_slice(p.W_max, TM);

  const Layout L = layout(NK, P, TM, p.W_max);
  uint8_t *s_x = base + L.x;
  uint64_t *bar_s0 = reinterpret_cast<uint64_t *>(base + L.book);
  uint64_t *bar1 = bar_s0 + 1, *bar2 = bar_s0 + 2, *bar3 = bar_s0 + 3;
  uint32_t *s_tmem = reinterpret_cast<uint32_t *>(bar_s0 + 4);
  int *s_U1 = reinterpret_cast<int *>(s_tmem + 1);
  int *s_par = reinterpret_cast<int *>(base + L.book + 64);
  float *s_alpha = reinterpret_cast<float *>(s_par + kBT);
  float *s_beta = s_alpha + kBT;
  float *s_Gp = s_beta + kBT;  // P(parent): the beam's gate product so far
  float *s_kq = s_Gp + kBT;
  int *s_chain = reinterpret_cast<int *>(s_kq + kBT);  // [32][TM] ancestor beam by depth
  int *s_slot = s_chain + kBT * TM;                     // [32][TM] ancestor slot by depth
  int *s_list = s_slot + kBT * TM;                      // slot -> (beam << 5 | depth-1)
  int *s_cnt = s_list + kBT * TM;                       // distinct ancestors per depth [TM + 4]
  int *s_pp = s_cnt + TM + 4;                           // parents of step t-1 [W_max]
  int *s_slice = s_pp + p.W_max;                        // ancestor rows of depth t-2 [W_max][TM]

  const __nv_bfloat16 *v = static_cast<const __nv_bfloat16 *>(p.v);
  __nv_bfloat16 *rec_k = static_cast<__nv_bfloat16 *>(p.rec_k);
  const int64_t row0 = (int64_t)(r * p.W + b0) * H + h;  // (r, b0, h) row of [R][W][H][d]

  // ------------------------------------------------------------ setup
  if (tid == 0) {
    ptx::mbar_init(bar_s0, 1);
    ptx::mbar_init(bar1, 1);
    ptx::mbar_init(bar2, 1);
    ptx::mbar_init(bar3, 1);
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

  // ------------------------------------------- before the wait
  // Every load of this phase is issued up front: one round trip.
  const uint32_t s0_bytes = (uint32_t)P * NK * 16384u;
  if (tid == kThreads - 32) {
    // S0 image (bulk copy) and X by TMA: rows 0..31 k_b, 32..63 q_b, then
    // the same 64 rows again (so that all four TMEM lane quarters of D2 hold
    // vectors).  Beams past W read as zeros.
    ptx::mbar_arrive_expect_tx(bar_s0, s0_bytes + 2u * kN * 128u * NK);
    const uint8_t *src = static_cast<const uint8_t *>(p.S0img) + (size_t)(r * H + h) * s0_bytes;
    for (uint32_t off = 0; off < s0_bytes; off += 16384u)
      ptx::bulk_g2s(base + L.a + off, src + off, 16384u, bar_s0);
#pragma unroll
    for (int copy = 0; copy < 2; ++copy)
#pragma unroll
      for (int ka = 0; ka < NK; ++ka) {
        uint8_t *dst = s_x + ka * XA + copy * (kN * 128);
        ptx::tma_load_4d(dst, &p.tm_k, ka * 64, h, b0, r, bar_s0);
        ptx::tma_load_4d(dst + kBT * 128, &p.tm_q, ka * 64, h, b0, r, bar_s0);
      }
  }
  // The previous step's parents (an input of step t-1) and the ancestor rows
  // of depth t-2 (written by step t-2, which has completed).
  if (nanc >= 2)
    for (int e = tid; e < p.W_prev; e += kThreads) ptx::cp_async4(s_pp + e, p.prev_parents + r * p.prev_stride + e);
  if (nanc >= 3 && slice) {
    const int w2 = nanc - 2;  // entries per row
    const int32_t *src = p.anc + anc_row(p, nanc - 1, r, 0);
    for (int e = tid; e < p.W_prev2 * w2; e += kThreads) {
      const int row = e / w2, j = e - row * w2;
      ptx::cp_async4(s_slice + e, src + (int64_t)row * TM + j);
    }
  }
  ptx::cp_async_commit();
  int par = -1;
  float g_alpha = 0.f, g_beta = 0.f;
  if (warp == 1 && lane < nb) {
    par = nanc >= 1 ? p.parents[r * p.W + b0 + lane] : 0;
    const int64_t si = row0 + (int64_t)lane * H;
    g_alpha = p.g[si];
    g_beta = p.beta[si];
  }
  // Epilogue mapping: warp w serves TMEM lanes 32*(w%4).. (output elements)
  // and beams 16*(w/4)..+15; v is loaded now, used at the end.
  const int ei = (warp & 3) * 32 + lane;
  const int half = warp >> 2;
  __nv_bfloat16 vreg[16];
#pragma unroll
  for (int m = 0; m < 16; ++m) {
    const int b = half * 16 + m;
    vreg[m] = (b < nb && ei < DV) ? v[(row0 + (int64_t)b * H) * DV + ei] : __float2bfloat16(0.f);
  }
  ptx::cp_async_wait_all();
  ptx::fence_proxy_async_smem();
  __syncthreads();

  bool ok = true;
  const uint32_t x_u32 = ptx::smem_u32(s_x), a_u32 = ptx::smem_u32(base + L.a);
  const uint32_t ka_u32 = ptx::smem_u32(base + L.ka);
  const uint32_t dhi_u32 = ptx::smem_u32(base + L.dhi), dlo_u32 = ptx::smem_u32(base + L.dlo);
  const uint32_t chi_u32 = ptx::smem_u32(base + L.chi), clo_u32 = ptx::smem_u32(base + L.clo);
  if (tid == 0) {
    ok = ptx::mbar_wait(bar_s0, 0, kWaitLimitNs);
    ptx::tc_fence_after();
    constexpr uint32_t idesc1 = ptx::idesc_bf16_f32(kM, kN);
    int acc = 0;
    for (int pl = 0; pl < P; ++pl)
#pragma unroll
      for (int ka = 0; ka < NK; ++ka)
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint64_t ad = ptx::desc_k128(a_u32 + (pl * NK + ka) * 16384 + kk * 32);
          const uint64_t bd = ptx::desc_k128(x_u32 + ka * XA + kk * 32);
          ptx::mma_bf16(tmem, ad, bd, idesc1, acc);
          acc = 1;
        }
    // Dkq = X . K^T: row 32 + b, column b is k_b . q_b.
    constexpr uint32_t idesc_kq = ptx::idesc_bf16_f32(kM, kBT);
#pragma unroll
    for (int ka = 0; ka < NK; ++ka)
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        const uint64_t ad = ptx::desc_k128(x_u32 + ka * XA + kk * 32);
        ptx::mma_bf16(tmem + 128, ad, ad, idesc_kq, (ka | kk) != 0);
      }
    ptx::mma_commit(bar1);
  }
  if (warp == 1) {
    // Each beam's ancestor row: [row of g at depth t-2, g, p].
    const int b = lane;
    if (b < nb) {
      if (par < 0 || par >= p.W_prev) {
        *reinterpret_cast<volatile int32_t *>(p.err) = kErrParent;
        par = 0;
      }
    }
    s_par[b] = b < nb ? par : 0;
    s_alpha[b] = b < nb ? expf(g_alpha) : 0.f;
    s_beta[b] = g_beta;
    if (nanc >= 1) {
      // Distinct parents take slots 0..U1-1.
      const unsigned same = __match_any_sync(0xffffffffu, par);
      const int leader = __ffs(same) - 1;
      const bool lead = b < nb && leader == lane;
      const unsigned leaders = __ballot_sync(0xffffffffu, lead);
      const int my = __popc(leaders & ((1u << lane) - 1u));
      if (lead) s_list[my] = (par << 5) | jp;
      const int slot = __shfl_sync(0xffffffffu, my, leader);
      if (lane == 0) *s_U1 = __popc(leaders);
      if (b < nb) {
        s_slot[b * TM + jp] = slot;
        s_chain[b * TM + jp] = par;
        if (nanc >= 2) {
          int gp = s_pp[par];
          if (gp < 0 || gp >= p.W_prev2) gp = 0;  // already reported by step t-1
          s_chain[b * TM + nanc - 2] = gp;
          if (nanc >= 3) {
            if (slice) {
              for (int j = 0; j < nanc - 2; ++j) s_chain[b * TM + j] = s_slice[gp * (nanc - 2) + j];
            } else {
              const int32_t *grow = p.anc + anc_row(p, nanc - 1, r, gp);
              int tmp[kMaxT - 2];
#pragma unroll
              for (int j = 0; j < kMaxT - 2; ++j)
                if (j < nanc - 2) tmp[j] = grow[j];
#pragma unroll
              for (int j = 0; j < kMaxT - 2; ++j)
                if (j < nanc - 2) s_chain[b * TM + j] = tmp[j];
            }
          }
        }
      }
    } else if (lane == 0) {
      *s_U1 = 0;
    }
  }
  __syncthreads();
  // Deeper ancestors (depths 1..t-2): one warp per depth (warps 1..7; warp 0
  // issues the MMAs) finds the distinct ones; their slots follow the
  // parents', depth by depth.
  for (int j = warp - 1; warp > 0 && j < nanc - 1; j += kThreads / 32 - 1) {
    const int a = lane < nb ? s_chain[lane * TM + j] : -1;
    const unsigned same = __match_any_sync(0xffffffffu, a);
    const int leader = __ffs(same) - 1;
    const bool lead = lane < nb && leader == lane;
    const unsigned leaders = __ballot_sync(0xffffffffu, lead);
    const int my = __popc(leaders & ((1u << lane) - 1u));
    const int rank = __shfl_sync(0xffffffffu, my, leader);
    if (lane < nb) s_slot[lane * TM + j] = rank;
    if (lane == 0) s_cnt[j] = __popc(leaders);
  }
  __syncthreads();
  const int U1 = *s_U1;
  int U = U1;
  for (int j = 0; j < nanc - 1; ++j) U += s_cnt[j];
  for (int j = warp - 1; warp > 0 && j < nanc - 1; j += kThreads / 32 - 1) {
    int base_j = U1;
    for (int j2 = 0; j2 < j; ++j2) base_j += s_cnt[j2];
    if (lane < nb) {
      const int slot = base_j + s_slot[lane * TM + j];
      s_slot[lane * TM + j] = slot;
      s_list[slot] = (s_chain[lane * TM + j] << 5) | j;
    }
  }
  __syncthreads();  // slots and the slot list complete

  // ------------------------------- after the wait: step t-1's records
  ptx::pdl_wait();
  ptx::pdl_launch_dependents();
  // Region A holds the S0 image until D1 is complete.
  if (!ptx::mbar_wait(bar1, 0, kWaitLimitNs)) ok = false;

  // Stage slots [lo, hi) of block blk: keys (cp.async) into KA; deltas / P(a)
  // as fp16 hi + lo into the MN-major Delta' operand.  All loads in flight
  // at once.
  auto stage = [&](int blk, int lo, int hi) {
    for (int e = tid; e < (hi - lo) * NK * 8; e += kThreads) {
      const int s = lo + e / (NK * 8), cc = e % (NK * 8);
      const int packed = s_list[s];
      const int lr = s - blk * kBlk;
      ptx::cp_async16(base + L.ka + (cc >> 3) * (kBlk * 128) + ptx::swz128(lr, cc & 7),
                      rec_k + rec_row(p, (packed & 31) + 1, r, h, packed >> 5) * DK + cc * 8, 16u);
    }
    ptx::cp_async_commit();
    float4 val[NF];
    float pa[NF];
#pragma unroll
    for (int u = 0; u < NF; ++u) {
      const int e = tid + u * kThreads;
      val[u] = make_float4(0.f, 0.f, 0.f, 0.f);
      pa[u] = 1.f;
      if (e < (hi - lo) * C4) {
        const int packed = s_list[lo + e / C4];
        const int64_t rr = rec_row(p, (packed & 31) + 1, r, h, packed >> 5);
        val[u] = __ldcg(reinterpret_cast<const float4 *>(p.rec_delta + rr * DV) + e % C4);
        pa[u] = __ldcg(p.rec_P + rr);
      }
    }
#pragma unroll
    for (int u = 0; u < NF; ++u) {
      const int e = tid + u * kThreads;
      if (e < (hi - lo) * C4) {
        const int lr = lo + e / C4 - blk * kBlk;
        const int i0 = (e % C4) * 4;
        const uint32_t off = (uint32_t)(i0 >> 6) * 8192u + (uint32_t)(lr >> 3) * 1024u +
                             (uint32_t)(lr & 7) * 128u + (uint32_t)((((i0 & 63) >> 3) ^ (lr & 7)) << 4) +
                             (uint32_t)(i0 & 7) * 2u;
        const float inv = 1.f / pa[u];
        const float f[4] = {val[u].x * inv, val[u].y * inv, val[u].z * inv, val[u].w * inv};
        __align__(8) __half hi4[4], lo4[4];
#pragma unroll
        for (int z = 0; z < 4; ++z) split_f16(f[z], hi4[z], lo4[z]);
        *reinterpret_cast<uint2 *>(base + L.dhi + off) = *reinterpret_cast<const uint2 *>(hi4);
        *reinterpret_cast<uint2 *>(base + L.dlo + off) = *reinterpret_cast<const uint2 *>(lo4);
      }
    }
  };
  // P(parent): loaded now, consumed after the staging loads are issued.
  float Gp = 1.f;
  if (warp == 2 && lane < nb && nanc >= 1) Gp = __ldcg(p.rec_P + rec_row(p, nanc, r, h, s_par[lane]));
  if (U > 0) stage(0, 0, min(U, kBlk));
  // This step's outputs that need no arithmetic: records of depth t (alpha,
  // P, k), the ancestor row and the parents of depth t.
  if (warp == 2 && lane < nb) {
    const int b = lane, gb = b0 + lane;
    s_Gp[b] = Gp;
    p.rec_alpha[rec_row(p, t, r, h, gb)] = s_alpha[b];
    p.rec_P[rec_row(p, t, r, h, gb)] = Gp * s_alpha[b];
    if (h == 0) {
      int32_t *row = p.anc + anc_row(p, t, r, gb);
      for (int j = 0; j < nanc; ++j) row[j] = s_chain[b * TM + j];
      p.par_store[((int64_t)(t - 1) * p.R + r) * p.W_max + gb] = s_par[b];
    }
  }
  if (!ptx::mbar_wait(bar_s0, 0, kWaitLimitNs)) ok = false;  // X visible to this thread
  for (int e = tid; e < kBT * NK * 8; e += kThreads) {
    const int n = e / (NK * 8), cc = e - n * (NK * 8);
    if (n < nb)
      reinterpret_cast<uint4 *>(rec_k + rec_row(p, t, r, h, b0 + n) * DK)[cc] =
          *reinterpret_cast<const uint4 *>(s_x + (cc >> 3) * XA + ptx::swz128(n, cc & 7));
  }
  if (warp == 1) {
    // k_b . q_b from Dkq (TMEM lanes 32..63 belong to warp 1).
    ptx::tc_fence_after();
    float d[32];
    ptx::tmem_ld32(tmem + (32u << 16) + 128, d);
    ptx::tmem_ld_wait();
    float kq = 0.f;
#pragma unroll
    for (int z = 0; z < 32; ++z)
      if (z == lane) kq = d[z];
    s_kq[lane] = kq;
  }
  const int nblk = (U + kBlk - 1) / kBlk;

  for (int blk = 0; blk < nblk; ++blk) {
    const int lo = blk * kBlk, hi = min(U, lo + kBlk);
    const int nrows = hi - lo;
    const int kpad = (nrows + 15) & ~15;  // slots the MMAs read (multiple of 16)
    if (blk > 0) {
      if (!ptx::mbar_wait(bar3, (blk - 1) & 1, kWaitLimitNs)) ok = false;
      stage(blk, lo, hi);
    }
    // Slots past the block's last ancestor but inside the MMA K range hold
    // zero deltas.
    for (int e = tid; e < (kpad - nrows) * 2 * 8; e += kThreads) {
      const int lr = nrows + e / 16, rem = e % 16, ma = rem >> 3, c = rem & 7;
      const uint32_t off = (uint32_t)ma * 8192u + (uint32_t)(lr >> 3) * 1024u + ptx::swz128(lr & 7, c);
      *reinterpret_cast<uint4 *>(base + L.dhi + off) = make_uint4(0u, 0u, 0u, 0u);
      *reinterpret_cast<uint4 *>(base + L.dlo + off) = make_uint4(0u, 0u, 0u, 0u);
    }
    ptx::cp_async_wait_all();
    ptx::fence_proxy_async_smem();
    __syncthreads();
    if (tid == 0) {
      ptx::tc_fence_after();
      const uint32_t idesc2 = ptx::idesc_bf16_f32(kM, kpad);
#pragma unroll
      for (int ka = 0; ka < NK; ++ka)
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint64_t ad = ptx::desc_k128(x_u32 + ka * XA + kk * 32);
          const uint64_t bd = ptx::desc_k128(ka_u32 + ka * (kBlk * 128) + kk * 32);
          ptx::mma_bf16(tmem + 64, ad, bd, idesc2, (ka | kk) != 0);
        }
      ptx::mma_commit(bar2);
    }
    // C build: D2 row n (TMEM lane n) is vector n % 64; warp w takes the
    // lane quarter w % 4 and the 16-slot column group (w % 4) / 2 + 2 (w / 4).
    // C[vec][a] = D2[vec][a] where a is an ancestor of vec's beam, else 0,
    // stored as fp16 hi + lo, K-major (row vec, K = slot).
    if (!ptx::mbar_wait(bar2, blk & 1, kWaitLimitNs)) ok = false;
    ptx::tc_fence_after();
    {
      const int qq = warp & 3;
      const int g = (qq >> 1) + 2 * (warp >> 2);
      if (g * 16 < kpad) {
        const int vec = (qq * 32 + lane) & (kN - 1);
        const int b = vec & (kBT - 1);
        float d[16];
        ptx::tmem_ld16(tmem + ((uint32_t)(qq * 32) << 16) + 64 + g * 16, d);
        ptx::tmem_ld_wait();
        uint32_t mask = 0u;
        if (b < nb)
          for (int j = 0; j < nanc; ++j) {
            const int sl = s_slot[b * TM + j] - lo - g * 16;
            if (sl >= 0 && sl < 16) mask |= 1u << sl;
          }
        __align__(16) __half h16[16], l16[16];
#pragma unroll
        for (int z = 0; z < 16; ++z) split_f16(((mask >> z) & 1u) ? d[z] : 0.f, h16[z], l16[z]);
#pragma unroll
        for (int c2 = 0; c2 < 2; ++c2) {
          const uint32_t off = ptx::swz128(vec, g * 2 + c2);
          *reinterpret_cast<uint4 *>(base + L.chi + off) = reinterpret_cast<const uint4 *>(h16)[c2];
          *reinterpret_cast<uint4 *>(base + L.clo + off) = reinterpret_cast<const uint4 *>(l16)[c2];
        }
      }
    }
    ptx::fence_proxy_async_smem();
    ptx::tc_fence_before();
    __syncthreads();
    if (tid == 0) {
      ptx::tc_fence_after();
      constexpr uint32_t idesc3 = ptx::idesc_f16_amn_f32(kM, kN);
      const uint32_t dA[3] = {dhi_u32, dhi_u32, dlo_u32};
      const uint32_t cB[3] = {chi_u32, clo_u32, chi_u32};
#pragma unroll
      for (int term = 0; term < 3; ++term)
        for (int ks = 0; ks < kpad / 16; ++ks) {
          const uint64_t ad = ptx::desc_mn128(dA[term] + ks * 2048, 8192u, 1024u);
          const uint64_t bd = ptx::desc_k128(cB[term] + ks * 32);
          ptx::mma_bf16(tmem, ad, bd, idesc3, 1u);
        }
      ptx::mma_commit(bar3);
    }
  }

  // --------------------------------------------------------- epilogue
  if (nblk > 0 && !ptx::mbar_wait(bar3, (nblk - 1) & 1, kWaitLimitNs)) ok = false;
  if (!ok) *reinterpret_cast<volatile int32_t *>(p.err) = kErrTimeout;
  __syncthreads();  // s_Gp and s_kq visible
  ptx::tc_fence_after();
  {
    const uint32_t lb = (uint32_t)((warp & 3) * 32) << 16;
    float uk[16], uq[16];
    ptx::tmem_ld16(tmem + lb + half * 16, uk);
    ptx::tmem_ld16(tmem + lb + kBT + half * 16, uq);
    ptx::tmem_ld_wait();
    if (ei < DV && ok) {
      const float4 *G4 = reinterpret_cast<const float4 *>(s_Gp + half * 16);
      const float4 *A4 = reinterpret_cast<const float4 *>(s_alpha + half * 16);
      const float4 *B4 = reinterpret_cast<const float4 *>(s_beta + half * 16);
      const float4 *K4 = reinterpret_cast<const float4 *>(s_kq + half * 16);
      const int64_t ostride = (int64_t)H * DV;
      float *op = p.o + (row0 + (int64_t)(half * 16) * H) * DV + ei;
      float *dp = p.rec_delta + (rec_row(p, t, r, h, b0) + half * 16) * DV + ei;
#pragma unroll
      for (int m4 = 0; m4 < 4; ++m4) {
        const float4 G = G4[m4], A = A4[m4], B = B4[m4], KQ = K4[m4];
        const float Gv[4] = {G.x, G.y, G.z, G.w}, Av[4] = {A.x, A.y, A.z, A.w};
        const float Bv[4] = {B.x, B.y, B.z, B.w}, Kv[4] = {KQ.x, KQ.y, KQ.z, KQ.w};
#pragma unroll
        for (int z = 0; z < 4; ++z) {
          const int m = m4 * 4 + z;
          if (half * 16 + m < nb) {
            const float ag = Av[z] * Gv[z];  // alpha P(p)
            const float delta = Bv[z] * fmaf(-ag, uk[m], __bfloat162float(vreg[m]));
            op[m * ostride] = fmaf(ag, uq[m], delta * Kv[z]);
            dp[m * DV] = delta;
          }
        }
      }
    }
  }

  // --------------------------------------------------------- teardown
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

// cuTensorMapEncodeTiled, fetched once from the driver.
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void *ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  }
  return fn;
}

// 4-D map over a [R][W][H][d] bf16 tensor: {d, H, W, R}, box {64, 1, 32, 1},
// 128-byte swizzle (the K-major operand layout), zeros outside the tensor.
bool encode_rows(CUtensorMap *m, const void *base, int d, int H, int W, int R) {
  PFN_cuTensorMapEncodeTiled_v12000 fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)H, (cuuint64_t)W, (cuuint64_t)R};
  const cuuint64_t strides[3] = {(cuuint64_t)d * 2, (cuuint64_t)H * d * 2, (cuuint64_t)W * H * d * 2};
  const cuuint32_t box[4] = {64, 1, (cuuint32_t)kBT, 1};
  const cuuint32_t es[4] = {1, 1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int DK>
cudaError_t launch_dk(const StepParams &p_in, bool pdl, cudaStream_t s) {
  StepParams p = p_in;
  if (!encode_rows(&p.tm_k, p.k, DK, p.H, p.W, p.R) || !encode_rows(&p.tm_q, p.q, DK, p.H, p.W, p.R))
    return cudaErrorInvalidValue;
  const Layout L = layout(DK / 64, p.s0_planes, p.T_max, p.W_max);
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
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((p.W + kBT - 1) / kBT, p.H, p.R);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, step_tc_kernel<DK>, p);
}

}  // namespace

bool tc_supports(int dk, int dv, int qkv_bf16, int T_max, int W_max) {
  return qkv_bf16 && dk == dv && (dk == 64 || dk == 128) && T_max <= kMaxT && W_max <= kMaxW;
}

size_t s0_image_bytes(int R, int H, int dk, int dv, int planes) {
  (void)dv;
  return (size_t)R * H * planes * (dk / 64) * 16384u;
}

cudaError_t launch_s0_image(const void *S0, void *img, int R, int H, int dk, int dv, int s0_bf16, int planes,
                            cudaStream_t s) {
  const int64_t total = (int64_t)R * H * planes * (dk / 64) * kM * 8;
  const int threads = 256;
  const int64_t want = (total + threads - 1) / threads;
  const int blocks = (int)(want < 148 * 16 ? want : 148 * 16);
  s0_image_kernel<<<blocks, threads, 0, s>>>(S0, static_cast<uint4 *>(img), R, H, dk, dv, s0_bf16, planes);
  return cudaGetLastError();
}

cudaError_t launch_step_tc(const StepParams &p, int pdl, cudaStream_t s) {
  if (p.T_max > kMaxT || p.W_max > kMaxW || p.s0_planes < 1 || p.s0_planes > 3 || !p.rec_P)
    return cudaErrorNotSupported;
  if (p.dk == 64 && p.dv == 64) return launch_dk<64>(p, pdl != 0, s);
  if (p.dk == 128 && p.dv == 128) return launch_dk<128>(p, pdl != 0, s);
  return cudaErrorNotSupported;
}

}  // namespace onela
