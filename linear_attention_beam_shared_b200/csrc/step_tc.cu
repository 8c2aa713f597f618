// Tensor-core decode-step kernel (tcgen05, sm_100a) for bf16 q/k/v and
// d_k = d_v in {64, 128}.
//
// One CTA per (request r, head h, tile of 32 beams); 256 threads; two CTAs
// fit on an SM.  The step of the shared-state GDN beam decode (OneLA,
// evolve.pub review, key claims on section 3.2, equations 2-4).  For beam b
// with ancestors a_1 .. a_{t-1} (a_{t-1} = p, its parent) and P(a) the
// product of the gates on the path from the root to record a:
//
//   S_{t-1} x = P(p) S0 x + sum_j delta_{a_j} w_j (k_{a_j} . x),
//   w_j = alpha_{a_{j+1}} ... alpha_{a_{t-1}}   (w = 1 for the parent),
//
// for x = k_b and x = q_b: the records are replayed with vectors only, no
// per-beam matrix is formed (review, Summary).  Then
// delta_b = beta_b (v_b - alpha_b S_{t-1} k_b) and
// o_b = alpha_b S_{t-1} q_b + delta_b (k_b . q_b), and the record
// (alpha_b, delta_b, k_b) is appended.
//
//   D1 = S0 . X^T   tensor cores, fp32 accumulators in TMEM, for the tile's
//                   64 vectors X = [k_0..k_31; q_0..q_31].  The S0 operand
//                   image is read once per CTA and serves every beam of the
//                   tile (the abstract's shared-state reuse across beams);
//                   fp32 S0 is split once, when the prompt state is
//                   installed, into two or three bf16 terms.
//   k_a . x         fp32 FMAs: the distinct ancestors' key rows are gathered
//                   into shared memory (4 rows per TMA instruction) and
//                   every beam's 8 threads form k_a . k_b, k_a . q_b and
//                   k_b . q_b, reducing by shuffles.
//   replay          fp32 FMAs, one thread per (beam, eighth of the elements).
//
// Only the deltas are outputs of earlier steps; ancestors (from the parents
// of every step), their keys and their gates are inputs.  So each kernel
// lets its dependent launch start at once, and before its
// griddepcontrol.wait it reads inputs only: the callers' arrays of the
// earlier steps under ONELA_FLAG_PDL, the record store otherwise (then the
// earlier steps have completed).  Warp roles (hand-offs on mbarriers with
// bounded waits): warp 0 issues the loads and D1; warp 1 builds each beam's
// ancestor chain (parent indices only; records never move, abstract), the
// tile's distinct ancestors and the depth-t entries that need no delta
// (alpha, the ancestry row); warp 2 gathers the gates along each chain into
// the replay weights; warp 3 writes the key records; warps 4-7 stage the
// ancestors' key rows and move D1 to shared memory.  Then all threads form
// the key products.  After the wait the ancestors' delta rows arrive in one
// round of 4-row gathers, every thread replays and writes o and delta.  No
// kernel reads a depth-t entry before step t has completed, so the early
// writes race with nothing.
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
constexpr int kDRows = 128;         // ancestor deltas per staging round after the wait (32 groups of 4)
constexpr int kTmemCols = 64;       // D1
constexpr int kKeyRows = 128;       // ancestor key rows per staging round
constexpr uint32_t kTabBytes = 2u * 8u * kHistSteps + 3u * 4u * kHistSteps;  // per-step table
constexpr int kMaxT = 16;           // deepest decode the kernel serves
constexpr int kMaxW = 1024;         // widest beam set the kernel serves
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s: far beyond any legal wait
constexpr int32_t kErrTimeout = 2;

struct Layout {
  uint32_t x;     // X [NK][64 rows][128 B]: k rows, then q rows
  uint32_t v;     // v [NK][32 rows][128 B]
  uint32_t a;     // region A: the S0 image; then KA and D1^T; then the deltas
  uint32_t ka;    // keys of a D2 block [NK][128 rows][128 B]
  uint32_t d1;    // D1^T [64 vectors][d_v] fp32
  uint32_t dst;   // ancestor deltas [kDRows][d_v] fp32
  uint32_t book;  // barriers and bookkeeping
  uint32_t total;
};

__host__ __device__ inline Layout layout(int nk, int planes, int TM, int W_max, int hist_cap) {
  Layout L;
  L.x = 0;
  L.v = (uint32_t)nk * 8192u;
  L.a = (uint32_t)nk * 12288u;
  L.ka = L.a;
  L.d1 = L.a + (uint32_t)nk * 16384u;
  L.dst = L.a;
  const uint32_t s0 = (uint32_t)planes * nk * 16384u, ops = (uint32_t)nk * 32768u;
  L.book = L.a + (s0 > ops ? s0 : ops);
  // 128 B of barriers and counters; 4 per-beam scalars; per (beam, depth)
  // the replay coefficients (float4), the chain, slot, slot-list ints and
  // weights (the slot list 4 TM longer); a beam-index scratch [W_max]; the
  // parents of steps 2..t-1; the per-step table (2 pointers and 3 ints per
  // step).
  L.total = L.book + 128u + 4u * kBT * 4u + (uint32_t)kBT * TM * 16u + (4u * kBT + 4u) * TM * 4u +
            (uint32_t)((W_max + 3) & ~3) * 4u + (uint32_t)((hist_cap + 3) & ~3) * 4u + kTabBytes + 16u;
  return L;
}

// Copies n ints from global src to shared dst with cp.async, by the 32 lanes
// of one warp: 16-byte pieces when both ends allow it, single ints otherwise.
__device__ __forceinline__ void copy_ints_warp(int *dst, const int32_t *src, int n, int lane) {
  int done = 0;
  if (((ptx::smem_u32(dst) | (uint32_t)reinterpret_cast<uintptr_t>(src)) & 15u) == 0) {
    done = n & ~3;
    for (int e = lane * 4; e < done; e += 128) ptx::cp_async16(dst + e, src + e, 16u);
  }
  for (int e = done + lane; e < n; e += 32) ptx::cp_async4(dst + e, src + e);
}

// Four consecutive bf16 elements at p (8-byte aligned) as floats.
__device__ __forceinline__ float4 bf16x4(const uint8_t *p) {
  const uint2 u = *reinterpret_cast<const uint2 *>(p);
  const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u.x));
  const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u.y));
  return make_float4(a.x, a.y, b.x, b.y);
}

template <int DK>
__global__ void __launch_bounds__(kThreads, 2) step_tc_kernel(const __grid_constant__ StepParams p) {
  constexpr int NK = DK / 64;        // 128-byte K atoms per key row
  constexpr int DV = DK;
  constexpr uint32_t XA = kN * 128;  // bytes of one K atom of X (64 rows)
  constexpr uint32_t VA = kBT * 128; // bytes of one K atom of v (32 rows)
  constexpr int NU = DV / 32;        // 4-element groups per thread, beam-major phase
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_u32 = ptx::smem_u32(smem_raw);
  uint8_t *base = smem_raw + ((1024u - (raw_u32 & 1023u)) & 1023u);

  const int tile = blockIdx.x, h = blockIdx.y, r = blockIdx.z;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int b0 = tile * kBT;
  const int nb = min(kBT, p.W - b0);
  const int H = p.H, t = p.t, TM = p.T_max, P = p.s0_planes;
  const int nanc = t - 1;   // ancestors per beam (depths 1..t-1)
  const int jp = nanc - 1;  // depth index of the parents (depth t-1)
  const bool hin = p.hist_inputs != 0;

  const Layout L = layout(NK, P, TM, p.W_max, p.hist_cap);
  uint8_t *s_x = base + L.x;
  const uint8_t *s_v = base + L.v;
  float *s_d1 = reinterpret_cast<float *>(base + L.d1);
  const float *s_dst = reinterpret_cast<const float *>(base + L.dst);
  uint64_t *bars = reinterpret_cast<uint64_t *>(base + L.book);
  uint64_t *bar_s0 = bars + 0;     // S0 image, X and v landed
  uint64_t *bar1 = bars + 1;       // D1 complete
  uint64_t *bar_d = bars + 3;      // ancestor deltas landed
  uint64_t *bar_chain = bars + 4;  // warp 1: every beam's chain in s_chain
  uint64_t *bar_slots = bars + 5;  // warp 1: slots, slot list and U
  uint64_t *bar_w = bars + 6;      // warp 2: replay weights and P(p)
  uint64_t *bar_keys = bars + 7;   // key rows of the current round landed
  uint32_t *s_tmem = reinterpret_cast<uint32_t *>(base + L.book + 64);
  int *s_U = reinterpret_cast<int *>(s_tmem + 1);
  int *s_par = reinterpret_cast<int *>(base + L.book + 128);
  float *s_alpha = reinterpret_cast<float *>(s_par + kBT);
  float *s_beta = s_alpha + kBT;
  float *s_Gp = s_beta + kBT;  // P(parent)
  // [32][TM]: (w k_a . k_b, w k_a . q_b, slot of a) for the ancestor a of
  // beam b at each depth.
  float4 *s_c = reinterpret_cast<float4 *>(s_Gp + kBT);
  int *s_chain = reinterpret_cast<int *>(s_c + kBT * TM);  // [32][TM] ancestor beam by depth
  int *s_slot = s_chain + kBT * TM;                         // [32][TM] ancestor slot by depth
  // slot -> (beam << 5 | depth-1); every depth's slots start on a multiple
  // of 4 (padding slots repeat the depth's first ancestor), [(32 + 4) TM].
  int *s_list = s_slot + kBT * TM;
  float *s_w = reinterpret_cast<float *>(s_list + (kBT + 4) * TM);  // [32][TM] replay weight by depth
  int *s_seen = reinterpret_cast<int *>(s_w + kBT * TM);           // beam index -> a lane (scratch)
  int *s_hist = s_seen + ((p.W_max + 3) & ~3);                 // parents of steps 2..t-1
  // Per-step table (index = step j), filled by warp 1 before the first
  // barrier with one load per lane: loops then read shared memory instead
  // of indexing the parameters at run time.
  const int32_t **s_tpar = reinterpret_cast<const int32_t **>(s_hist + ((p.hist_cap + 3) & ~3));
  const float **s_tg = reinterpret_cast<const float **>(s_tpar + kHistSteps);
  int *s_toff = reinterpret_cast<int *>(s_tg + kHistSteps);
  int *s_tW = s_toff + kHistSteps;
  int *s_trs = s_tW + kHistSteps;
  uint8_t *s_keys = base + L.ka;                               // key rows [kKeyRows][d_k] bf16
  static_assert(kKeyRows * DK * 2 <= NK * 16384, "the key rows must fit in their area");

  __nv_bfloat16 *rec_k = static_cast<__nv_bfloat16 *>(p.rec_k);
  const int64_t row0 = (int64_t)(r * p.W + b0) * H + h;  // (r, b0, h) row of [R][W][H][d]

  // --------------------------------------- setup; every load issued at once
  const uint32_t s0_bytes = (uint32_t)P * NK * 16384u;
  if (tid == 0) {
    ptx::mbar_init(bar_s0, 1);
    ptx::mbar_init(bar1, 1);
    ptx::mbar_init(bar_d, 32);
    ptx::mbar_init(bar_chain, 32);
    ptx::mbar_init(bar_slots, 32);
    ptx::mbar_init(bar_w, 32);
    ptx::mbar_init(bar_keys, 32);
    ptx::mbar_fence_init();
    // S0 image (bulk copy); k, q, v tiles by TMA, beams past W read as zeros.
    ptx::mbar_arrive_expect_tx(bar_s0, s0_bytes + NK * (XA + VA));
    const uint8_t *src = static_cast<const uint8_t *>(p.S0img) + (size_t)(r * H + h) * s0_bytes;
    for (uint32_t off = 0; off < s0_bytes; off += 16384u)
      ptx::bulk_g2s(base + L.a + off, src + off, 16384u, bar_s0);
#pragma unroll
    for (int ka = 0; ka < NK; ++ka) {
      ptx::tma_load_4d(s_x + ka * XA, &p.tm_k, ka * 64, h, b0, r, bar_s0);
      ptx::tma_load_4d(s_x + ka * XA + kBT * 128, &p.tm_q, ka * 64, h, b0, r, bar_s0);
      ptx::tma_load_4d(base + L.v + ka * VA, &p.tm_v, ka * 64, h, b0, r, bar_s0);
    }
  }
  if (warp == 3) {
    ptx::tmem_alloc(s_tmem, kTmemCols);
    ptx::tmem_relinquish();
  }
  // Before its wait this kernel reads inputs only, so the next step may start.
  ptx::pdl_launch_dependents();
  int par = 0;
  float g_alpha = 0.f, g_beta = 0.f;
  if (warp == 1) {
    // This tile's parents, gates and betas; the per-step table (lane j loads
    // step j: one load per lane, then loops read shared memory instead of
    // indexing the parameters at run time).
    if (lane < nb) {
      par = nanc >= 1 ? p.parents[r * p.W + b0 + lane] : 0;
      const int64_t si = row0 + (int64_t)lane * H;
      g_alpha = p.g[si];
      g_beta = p.beta[si];
    }
    if (lane < kHistSteps) {
      s_tpar[lane] = p.hpar[lane];
      s_tg[lane] = p.hg[lane];
      s_toff[lane] = p.hoff[lane];
      s_tW[lane] = p.hW[lane];
      s_trs[lane] = p.hpar_rs[lane];
    }
  }
  // The parents of steps 2..t-1 for this request, back to back, each array
  // starting on a 16-byte boundary: warp w >= 1 copies steps w + 1, w + 8.
  // Every thread waits for its own copies before the barrier below.
  if (p.hist_cap > 0 && warp >= 1)
#pragma unroll 1
    for (int j = warp + 1; j < t; j += kThreads / 32 - 1)
      copy_ints_warp(s_hist + p.hoff[j], p.hpar[j] + (int64_t)r * p.hpar_rs[j], p.hW[j], lane);
  ptx::cp_async_commit();
  ptx::cp_async_wait_all();
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *s_tmem;

  bool ok = true;
  const uint32_t x_u32 = ptx::smem_u32(s_x), a_u32 = ptx::smem_u32(base + L.a);
  // Key rows of slots [lo, lo + n) (n a multiple of 4) into s_keys, by 32
  // callers i = 0..31: caller i gathers the 4 rows of slots lo + 4i .. + 3
  // (one depth: the slots of a depth start on a multiple of 4) from that
  // depth's row table.  Every caller arrives on bar_keys once.
  auto stage_keys = [&](int lo, int n, int i) {
    if (4 * i < n) {
      const int s0 = lo + 4 * i;
      const int j = s_list[s0] & 31;
      const int Wj = s_tW[j + 1];
      int row[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int a = s_list[s0 + q] >> 5;
        row[q] = hin ? (r * Wj + a) * H + h : (int)rec_row(p, j + 1, r, h, a);
      }
      ptx::fence_proxy_async_smem();
      ptx::mbar_arrive_expect_tx(bar_keys, 4 * DK * 2);
      ptx::tma_gather4(s_keys + 4 * i * DK * 2, &p.tm_krows[j + 1], 0, row[0], row[1], row[2], row[3], bar_keys);
    } else {
      ptx::mbar_arrive(bar_keys);
    }
  };
  const int wq = warp & 3;                        // TMEM lane quarter of this warp
  const uint32_t lb = (uint32_t)(wq * 32) << 16;  // its lane base

  // ------------------------------------------------ warp roles before the wait
  if (warp == 0) {
    // The MMA issuer: D1 = S0 . X^T.
    if (lane == 0) {
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
      ptx::mma_commit(bar1);
    }
  } else if (warp == 1) {
    // The ancestry: beam b's ancestors a[j] at depth j + 1 (a[t-2] = its
    // parent; a[j] is the parent, at step j + 2, of a[j + 1]), the entries of
    // depth t that need no delta, and the distinct ancestors of the tile.
    const int b = lane;
    if (b < nb && nanc >= 1 && (par < 0 || par >= p.W_prev)) {
      *reinterpret_cast<volatile int32_t *>(p.err) = kErrParent;
      par = 0;
    }
    const float alpha_b = b < nb ? expf(g_alpha) : 0.f;
    s_par[b] = par;
    s_alpha[b] = alpha_b;
    s_beta[b] = g_beta;
    if (b < nb && nanc >= 1) {
      int a = par;
      s_chain[b * TM + jp] = a;
#pragma unroll 1
      for (int j = jp - 1; j >= 0; --j) {
        int pa = p.hist_cap > 0 ? s_hist[s_toff[j + 2] + a] : s_tpar[j + 2][(int64_t)r * s_trs[j + 2] + a];
        if (pa < 0 || pa >= s_tW[j + 1]) pa = 0;  // reported by step j + 2
        a = pa;
        s_chain[b * TM + j] = a;
      }
    }
    ptx::mbar_arrive(bar_chain);
    if (b < nb) {
      const int gb = b0 + b;
      p.rec_alpha[rec_row(p, t, r, h, gb)] = alpha_b;
      if (h == 0) {
        int32_t *row = p.anc + anc_row(p, t, r, gb);
#pragma unroll 1
        for (int j = 0; j < nanc; ++j) row[j] = s_chain[b * TM + j];
        p.par_store[((int64_t)(t - 1) * p.R + r) * p.W_max + gb] = par;
      }
    }
    // Distinct ancestors depth by depth: every lane writes its lane number
    // at its ancestor's index, and the lane whose number survives leads that
    // ancestor.  Slots in order of depth, then of the leading lane; each
    // depth's first slot is a multiple of 4.
    int U = 0;
#pragma unroll 1
    for (int j = 0; j < nanc; ++j) {
      const int a = b < nb ? s_chain[b * TM + j] : 0;
      if (b < nb) s_seen[a] = lane;
      __syncwarp();
      const int leader = b < nb ? s_seen[a] : 0;
      __syncwarp();
      const bool lead = b < nb && leader == lane;
      const unsigned leaders = __ballot_sync(0xffffffffu, lead);
      const int slot = U + __popc(leaders & ((1u << leader) - 1u));
      if (lead) s_list[slot] = (a << 5) | j;
      if (b < nb) {
        s_slot[b * TM + j] = slot;
        s_c[b * TM + j] = make_float4(0.f, 0.f, __int_as_float(slot), 0.f);
      }
      __syncwarp();
      // Pad the depth to a whole group of 4 with its first ancestor.
      const int cnt = __popc(leaders), cnt4 = (cnt + 3) & ~3;
      if (lane >= cnt && lane < cnt4) s_list[U + lane] = s_list[U];
      U += cnt4;
    }
    if (lane == 0) *s_U = U;
    ptx::mbar_arrive(bar_slots);
  } else if (warp == 2) {
    // The gates along each beam's chain give the replay weights (products of
    // the later gates) and P(p).  They land in s_w first (one round trip);
    // each entry is then overwritten by the weight of its depth.
    const int b = lane;
    if (!ptx::mbar_wait(bar_chain, 0, kWaitLimitNs)) ok = false;
    if (b < nb) {
#pragma unroll 1
      for (int j = 0; j <= jp; ++j) {
        const int a = s_chain[b * TM + j];
        ptx::cp_async4(s_w + b * TM + j, hin ? s_tg[j + 1] + ((int64_t)r * s_tW[j + 1] + a) * H + h
                                             : p.rec_alpha + rec_row(p, j + 1, r, h, a));
      }
    }
    ptx::cp_async_commit();
    ptx::cp_async_wait_all();
    float w = 1.f;
    if (b < nb) {
#pragma unroll 1
      for (int j = jp; j >= 0; --j) {
        const float gj = s_w[b * TM + j];
        s_w[b * TM + j] = w;
        w *= hin ? expf(gj) : gj;
      }
    }
    s_Gp[b] = w;  // P(p): all the gates on the path
    ptx::mbar_arrive(bar_w);
  } else if (warp == 3) {
    // The key records of depth t, from X.
    if (!ptx::mbar_wait(bar_s0, 0, kWaitLimitNs)) ok = false;
    for (int e = lane; e < kBT * NK * 8; e += 32) {
      const int n = e / (NK * 8), cc = e - n * (NK * 8);
      if (n < nb)
        reinterpret_cast<uint4 *>(rec_k + rec_row(p, t, r, h, b0 + n) * DK)[cc] =
            *reinterpret_cast<const uint4 *>(s_x + (cc >> 3) * XA + ptx::swz128(n, cc & 7));
    }
  } else {
    // Warps 4-7: the key rows of the tile's first kKeyRows distinct
    // ancestors into shared memory (one bulk copy per row), and D1^T.
    const int ei = wq * 32 + lane;  // TMEM lane: output element of D1
    if (!ptx::mbar_wait(bar1, 0, kWaitLimitNs)) ok = false;  // region A is free
    ptx::tc_fence_after();
    if (!ptx::mbar_wait(bar_slots, 0, kWaitLimitNs)) ok = false;
    if (lane < 8) stage_keys(0, min(*s_U, kKeyRows), wq * 8 + lane);  // 8 groups per warp
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      float d[32];
      ptx::tmem_ld32(tmem + lb + half * 32, d);
      ptx::tmem_ld_wait();
      if (wq * 32 < DV)
#pragma unroll
        for (int n = 0; n < 32; ++n) s_d1[(half * 32 + n) * DV + ei] = d[n];
    }
  }
  ptx::tc_fence_before();
  __syncthreads();  // every role done: D1^T, slots, weights
  if (warp == 3) ptx::tmem_dealloc(tmem, kTmemCols);

  // Beam-major phase: thread (bb, l) owns elements 32 u + 4 l + z (z < 4) of
  // beam bb.  u = P(p) D1 + (replayed terms, after the wait); v from its tile.
  const int bb = tid >> 3, l = tid & 7;
  const bool bval = bb < nb;
  if (!ptx::mbar_wait(bar_s0, 0, kWaitLimitNs)) ok = false;  // X and v visible to this thread
  // This thread's elements of k_b and q_b, and k_b . q_b.
  float4 kb[NU], qb[NU];
  float kq = 0.f;
#pragma unroll
  for (int u = 0; u < NU; ++u) {
    const uint32_t off = (uint32_t)(u >> 1) * XA + (uint32_t)(l & 1) * 8u;
    const int c = 4 * (u & 1) + (l >> 1);
    kb[u] = bf16x4(s_x + off + ptx::swz128(bb, c));
    qb[u] = bf16x4(s_x + off + ptx::swz128(kBT + bb, c));
    kq = fmaf(kb[u].x, qb[u].x, kq);
    kq = fmaf(kb[u].y, qb[u].y, kq);
    kq = fmaf(kb[u].z, qb[u].z, kq);
    kq = fmaf(kb[u].w, qb[u].w, kq);
  }
  kq += __shfl_xor_sync(0xffffffffu, kq, 4);
  kq += __shfl_xor_sync(0xffffffffu, kq, 2);
  kq += __shfl_xor_sync(0xffffffffu, kq, 1);
  // k_a . k_b and k_a . q_b for the beam's ancestor a at every depth, from
  // the staged key rows (rounds of kKeyRows slots), weighted.
  const int U = *s_U;
  for (int lo = 0, rnd = 0; lo < U; lo += kKeyRows, ++rnd) {
    const int nrows = min(U - lo, kKeyRows);
    if (rnd > 0) {
      __syncthreads();  // the previous round's rows are consumed
      if (warp == 0) stage_keys(lo, nrows, lane);
    }
    if (!ptx::mbar_wait(bar_keys, rnd & 1, kWaitLimitNs)) ok = false;
    // Two depths per pass: independent loads and shuffle chains interleave.
#pragma unroll 1
    for (int j0 = 0; j0 < nanc; j0 += 2) {
      float dk[2], dq[2];
      int slot[2];
      bool in[2];
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int j = j0 + e;
        slot[e] = bval && j < nanc ? s_slot[bb * TM + j] : -1;
        const unsigned sl = (unsigned)(slot[e] - lo);
        in[e] = sl < (unsigned)nrows;
        const uint8_t *row = s_keys + (in[e] ? sl : 0u) * (DK * 2) + l * 8;
        dk[e] = 0.f, dq[e] = 0.f;
#pragma unroll
        for (int u = 0; u < NU; ++u) {
          const float4 kf = bf16x4(row + u * 64);
          dk[e] = fmaf(kf.x, kb[u].x, dk[e]);
          dk[e] = fmaf(kf.y, kb[u].y, dk[e]);
          dk[e] = fmaf(kf.z, kb[u].z, dk[e]);
          dk[e] = fmaf(kf.w, kb[u].w, dk[e]);
          dq[e] = fmaf(kf.x, qb[u].x, dq[e]);
          dq[e] = fmaf(kf.y, qb[u].y, dq[e]);
          dq[e] = fmaf(kf.z, qb[u].z, dq[e]);
          dq[e] = fmaf(kf.w, qb[u].w, dq[e]);
        }
      }
#pragma unroll
      for (int o = 4; o > 0; o >>= 1)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          dk[e] += __shfl_xor_sync(0xffffffffu, dk[e], o);
          dq[e] += __shfl_xor_sync(0xffffffffu, dq[e], o);
        }
#pragma unroll
      for (int e = 0; e < 2; ++e)
        if (in[e] && l == 0) {
          const float w = s_w[bb * TM + j0 + e];
          s_c[bb * TM + j0 + e] = make_float4(dk[e] * w, dq[e] * w, __int_as_float(slot[e]), 0.f);
        }
    }
  }
  // u = P(p) D1 + (replayed terms, after the wait); v from its tile.
  float acc_k[4 * NU], acc_q[4 * NU];
  float4 vf[NU];
  const float Gp = s_Gp[bb], alpha = s_alpha[bb], beta = s_beta[bb];
#pragma unroll
  for (int u = 0; u < NU; ++u) {
    const float4 dk = reinterpret_cast<const float4 *>(s_d1 + bb * DV)[8 * u + l];
    const float4 dq = reinterpret_cast<const float4 *>(s_d1 + (kBT + bb) * DV)[8 * u + l];
    acc_k[4 * u + 0] = Gp * dk.x, acc_k[4 * u + 1] = Gp * dk.y, acc_k[4 * u + 2] = Gp * dk.z, acc_k[4 * u + 3] = Gp * dk.w;
    acc_q[4 * u + 0] = Gp * dq.x, acc_q[4 * u + 1] = Gp * dq.y, acc_q[4 * u + 2] = Gp * dq.z, acc_q[4 * u + 3] = Gp * dq.w;
    vf[u] = bf16x4(s_v + (u >> 1) * VA + ptx::swz128(bb, 4 * (u & 1) + (l >> 1)) + (l & 1) * 8);
  }
  __syncthreads();  // D1^T and the key rows consumed before the deltas overwrite region A

  // ------------------------------- after the wait: the ancestors' deltas
  ptx::pdl_wait();
  for (int lo = 0, rnd = 0; lo < U; lo += kDRows, ++rnd) {
    const int hi = min(U, lo + kDRows);
    const int nrows = hi - lo;
    if (rnd > 0) __syncthreads();  // the previous round's deltas are consumed
    if (warp == 0) {
      // Lane i gathers the delta rows of slots lo + 4i .. + 3.
      if (4 * lane < nrows) {
        int row[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int packed = s_list[lo + 4 * lane + q];
          row[q] = (int)rec_row(p, (packed & 31) + 1, r, h, packed >> 5);
        }
        ptx::fence_proxy_async_smem();
        ptx::mbar_arrive_expect_tx(bar_d, 4 * DV * 4);
        ptx::tma_gather4(base + L.dst + 4 * lane * DV * 4, &p.tm_delta, 0, row[0], row[1], row[2], row[3], bar_d);
      } else {
        ptx::mbar_arrive(bar_d);
      }
    }
    if (!ptx::mbar_wait(bar_d, rnd & 1, kWaitLimitNs)) ok = false;
    if (bb < nb) {
      // Two depths per pass: their loads are independent.
#pragma unroll 1
      for (int j0 = 0; j0 < nanc; j0 += 2) {
        float4 c[2];
        bool in[2];
        const float4 *row[2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          c[e] = j0 + e < nanc ? s_c[bb * TM + j0 + e] : make_float4(0.f, 0.f, __int_as_float(-1), 0.f);
          const unsigned sl = (unsigned)(__float_as_int(c[e].z) - lo);
          in[e] = sl < (unsigned)nrows;
          row[e] = reinterpret_cast<const float4 *>(s_dst + (in[e] ? sl : 0u) * DV) + l;
          if (!in[e]) c[e].x = c[e].y = 0.f;
        }
#pragma unroll
        for (int u = 0; u < NU; ++u) {
          const float4 d0 = row[0][8 * u], d1 = row[1][8 * u];
          acc_k[4 * u + 0] = fmaf(d1.x, c[1].x, fmaf(d0.x, c[0].x, acc_k[4 * u + 0]));
          acc_k[4 * u + 1] = fmaf(d1.y, c[1].x, fmaf(d0.y, c[0].x, acc_k[4 * u + 1]));
          acc_k[4 * u + 2] = fmaf(d1.z, c[1].x, fmaf(d0.z, c[0].x, acc_k[4 * u + 2]));
          acc_k[4 * u + 3] = fmaf(d1.w, c[1].x, fmaf(d0.w, c[0].x, acc_k[4 * u + 3]));
          acc_q[4 * u + 0] = fmaf(d1.x, c[1].y, fmaf(d0.x, c[0].y, acc_q[4 * u + 0]));
          acc_q[4 * u + 1] = fmaf(d1.y, c[1].y, fmaf(d0.y, c[0].y, acc_q[4 * u + 1]));
          acc_q[4 * u + 2] = fmaf(d1.z, c[1].y, fmaf(d0.z, c[0].y, acc_q[4 * u + 2]));
          acc_q[4 * u + 3] = fmaf(d1.w, c[1].y, fmaf(d0.w, c[0].y, acc_q[4 * u + 3]));
        }
      }
    }
  }

  // --------------------------------------------------------- epilogue
  if (!ok) *reinterpret_cast<volatile int32_t *>(p.err) = kErrTimeout;
  if (bb < nb && ok) {
    float4 *op = reinterpret_cast<float4 *>(p.o + (row0 + (int64_t)bb * H) * DV) + l;
    float4 *dp = reinterpret_cast<float4 *>(p.rec_delta + rec_row(p, t, r, h, b0 + bb) * DV) + l;
#pragma unroll
    for (int u = 0; u < NU; ++u) {
      float4 d, o;
      d.x = beta * fmaf(-alpha, acc_k[4 * u + 0], vf[u].x);
      d.y = beta * fmaf(-alpha, acc_k[4 * u + 1], vf[u].y);
      d.z = beta * fmaf(-alpha, acc_k[4 * u + 2], vf[u].z);
      d.w = beta * fmaf(-alpha, acc_k[4 * u + 3], vf[u].w);
      o.x = fmaf(alpha, acc_q[4 * u + 0], d.x * kq);
      o.y = fmaf(alpha, acc_q[4 * u + 1], d.y * kq);
      o.z = fmaf(alpha, acc_q[4 * u + 2], d.z * kq);
      o.w = fmaf(alpha, acc_q[4 * u + 3], d.w * kq);
      op[8 * u] = o;
      dp[8 * u] = d;
    }
  }
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
  if (!encode_rows(&p.tm_k, p.k, DK, p.H, p.W, p.R) || !encode_rows(&p.tm_q, p.q, DK, p.H, p.W, p.R) ||
      !encode_rows(&p.tm_v, p.v, DK, p.H, p.W, p.R))
    return cudaErrorInvalidValue;
  const Layout L = layout(DK / 64, p.s0_planes, p.T_max, p.W_max, p.hist_cap);
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

bool encode_row_table(CUtensorMap *m, const void *base, int bf16, int width, long long rows) {
  PFN_cuTensorMapEncodeTiled_v12000 fn = encode_fn();
  if (!fn || rows < 1 || rows > 0x7fffffffLL) return false;
  const int es = bf16 ? 2 : 4;
  const cuuint64_t dims[2] = {(cuuint64_t)width, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)width * es};
  const cuuint32_t box[2] = {(cuuint32_t)width, 1};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void *>(base),
            dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

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
  if (p.T_max > kMaxT || p.W_max > kMaxW || p.s0_planes < 1 || p.s0_planes > 3 || p.hist_cap > kHistMaxInts)
    return cudaErrorNotSupported;
  if (p.dk == 64 && p.dv == 64) return launch_dk<64>(p, pdl != 0, s);
  if (p.dk == 128 && p.dv == 128) return launch_dk<128>(p, pdl != 0, s);
  return cudaErrorNotSupported;
}

}  // namespace onela
