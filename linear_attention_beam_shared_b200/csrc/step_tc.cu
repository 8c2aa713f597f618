// Tensor-core decode-step kernel (tcgen05, sm_100a) for bf16 q/k/v and
// d_k = d_v in {64, 128, 256}.
//
// One CTA per (request r, head h, tile of 32 beams) -- at d = 256 two, one
// per half of the rows of S, each streaming its half of the S0 image through
// a ring of shared-memory slots; 320 threads (8 beam warps, an ancestry warp
// and an MMA warp); two CTAs fit on an SM.  The step
// of the shared-state GDN beam decode (OneLA, evolve.pub review, key claims
// on section 3.2, equations 2-4).  For beam b with ancestors a_1 .. a_{t-1}
// (a_{t-1} = p, its parent) and P(a) the product of the gates on the path
// from the root to record a:
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
//   k_a . x         fp32 FMAs: every beam's 8 threads load their pieces of
//                   each ancestor's key row from global memory and reduce
//                   k_a . k_b, k_a . q_b by shuffles.
//   replay          fp32 FMAs, one thread per (beam, eighth of the elements),
//                   over the distinct ancestors' delta rows staged in shared
//                   memory.
//
// Only the deltas are outputs of earlier steps; ancestors (from the parents
// of every step), their keys and their gates are inputs.  So each kernel
// lets its dependent launch start at once, and before its
// griddepcontrol.wait it reads inputs only: the callers' arrays of the
// earlier steps where they are still valid (under ONELA_FLAG_PDL, or steps of
// the same onela_decode_steps call), the record store otherwise (a step that
// overlaps its predecessor never reads from the store a depth that a step
// still running may replace).  Before the wait: the ancestry warp builds
// each beam's ancestor chain (parent indices only; records never move,
// abstract), then the tile's distinct ancestors and the replay weights; the
// MMA warp issues D1 as soon as the image is in; the beam warps form the key
// products as soon as the chains exist, then move D1 to shared memory and
// write the entries of depth t that need no delta.  After the wait the
// ancestors' delta rows arrive in one round of 16-byte copies, every beam
// thread replays and writes o and delta.  No kernel reads a depth-t entry
// before step t has completed, so the early writes race with nothing.
//
// With a folded prefix (onela_fold) S0 is the folded state and the chain
// starts at depth d0 + 1.  The record store is a ring over the last T_max
// depths, so depth t's early writes replace the entries of depth t - T_max:
// the steps that may still run then read only deltas from the store (keys,
// gates and parents come from the callers' arrays under programmatic
// launch), and deltas are written after the wait.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cudaTypedefs.h>

#include "internal.h"
#include "sm100_ptx.h"
#include "tc_common.h"

namespace onela {
namespace {

constexpr int kThreads = 320;       // 8 beam warps, the ancestry warp and the MMA warp
constexpr int kAncWarp = 8;         // the ancestry warp
constexpr int kMmaWarp = 9;         // the MMA warp
constexpr int kBT = 32;             // beams per CTA
constexpr int kN = 2 * kBT;         // vectors: k rows 0..31, q rows 32..63
constexpr int kM = 128;             // MMA M
constexpr int kDRows = 128;         // ancestor deltas per staging round after the wait
constexpr int kRing = 3;            // 16 KB slots of the image ring (d_k = 256)
constexpr int kTmemCols = 64;       // D1
// The per-step table: 3 pointers and 3 ints for each of nhist = T_max + 1
// steps (at most kHistSteps).
__host__ __device__ inline uint32_t tab_bytes(int nhist) { return (3u * 8u + 3u * 4u) * (uint32_t)nhist; }
constexpr int kMaxT = 32;           // deepest decode the kernel serves
constexpr int kMaxW = 4096;         // widest beam set the kernel serves (its beam-index scratch: 4 B per beam)
constexpr int kSMs = 148;           // SMs of a B200

struct Layout {
  uint32_t x;     // X [NK][64 rows][128 B]: k rows, then q rows
  uint32_t v;     // v [NV][32 rows][128 B]: this CTA's d_v columns
  uint32_t a;     // region A: the S0 image (or its ring); then D1^T
  uint32_t d1;    // D1^T [64 vectors][this CTA's d_v rows] fp32
  uint32_t dst;   // ancestor deltas [rows][this CTA's d_v rows] fp32
  uint32_t book;  // barriers and bookkeeping
  uint32_t total;
};

// nk: 64-element K atoms of a key row; nv: 64-row atoms of this CTA's d_v rows.
// ring (d_k = 256): the image passes through kRing slots of region A, and
// the deltas are staged over X and region A, both consumed by then; else the
// whole image sits in region A, which then holds D1^T and the deltas.
__host__ __device__ inline Layout layout(int nk, int nv, int planes, int TM, int W_max, int hist_cap,
                                         bool ring = false) {
  Layout L;
  if (ring) {
    L.v = 0;
    L.x = (uint32_t)nv * 4096u;
    L.a = L.x + (uint32_t)nk * 8192u;
    L.d1 = L.a;
    L.dst = L.x;
    L.book = L.a + (uint32_t)kRing * 16384u;
  } else {
    L.x = 0;
    L.v = (uint32_t)nk * 8192u;
    L.a = L.v + (uint32_t)nv * 4096u;
    L.d1 = L.a + (uint32_t)nv * 16384u;
    L.dst = L.a;
    const uint32_t s0 = (uint32_t)planes * nk * 16384u, ops = (uint32_t)nv * 32768u;
    L.book = L.a + (s0 > ops ? s0 : ops);
  }
  // 128 B of barriers and counters; 4 per-beam scalars; per (beam, depth)
  // the replay coefficients (float4), the chain, slot-list ints and gates
  // (the slot list 4 TM longer); a beam-index scratch [W_max]; the parents
  // of the last steps before t; the per-step table (3 pointers and 3 ints per
  // step).
  L.total = L.book + 128u + 4u * kBT * 4u + (uint32_t)kBT * TM * 16u + (3u * kBT + 4u) * TM * 4u +
            (uint32_t)((W_max + 3) & ~3) * 4u + (uint32_t)((hist_cap + 3) & ~3) * 2u + tab_bytes(TM + 1) + 16u;
  return L;
}

// DK: d_k; DV: the d_v rows of S (and columns of v, o, delta) one CTA
// handles -- all of them for d <= 128, one half of them for d = 256 (the two
// halves of a beam tile are two CTAs; both form the full key products).
// MINB: CTAs per SM the registers must allow (3 only at d = 64).
template <int DK, int DV, int MINB>
__global__ void __launch_bounds__(kThreads, MINB) step_tc_kernel(const __grid_constant__ StepParams p) {
  constexpr bool RING = DK > 128;    // the image streamed through kRing slots (two CTAs per SM)
  constexpr int NK = DK / 64;        // 128-byte K atoms per key row
  constexpr int NV = DV / 64;        // 64-column atoms of this CTA's part of v
  constexpr uint32_t XA = kN * 128;  // bytes of one K atom of X (64 rows)
  constexpr uint32_t VA = kBT * 128; // bytes of one atom of v (32 rows)
  constexpr int NU = DV / 32;        // 4-element groups per thread of a value row, beam-major phase
  constexpr int NUK = DK / 32;       // the same for a key row
  // Ancestor delta rows per staging round after the wait.
  constexpr int DR = RING ? (NK * 8192 + kRing * 16384) / (DV * 4) : kDRows;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_u32 = ptx::smem_u32(smem_raw);
  uint8_t *base = smem_raw + ((1024u - (raw_u32 & 1023u)) & 1023u);

  const int nmt = p.dv / DV;         // CTAs per beam tile (row halves of S)
  const int tile = blockIdx.x, h = blockIdx.y, r = blockIdx.z / nmt, mt = blockIdx.z - r * nmt;
  const int e_off = mt * DV;         // first d_v row of this CTA
  const int DVT = p.dv;              // full d_v: the row stride of o and the delta records
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int b0 = tile * kBT;
  const int nb = min(kBT, p.W - b0);
  const int H = p.H, t = p.t, TM = p.T_max, P = p.s0_planes;
  const int tslot = (t - 1) % TM;  // slot of depth t
  const int hb = p.hbase;       // step of the history table's entry 0
  const uint64_t hmask = p.hist_inputs;  // bit i: history entry i from the callers' arrays

  const Layout L = layout(NK, NV, P, TM, p.W_max, p.hist_cap, RING);
  uint8_t *s_x = base + L.x;
  const uint8_t *s_v = base + L.v;
  float *s_d1 = reinterpret_cast<float *>(base + L.d1);
  const float *s_dst = reinterpret_cast<const float *>(base + L.dst);
  uint64_t *bars = reinterpret_cast<uint64_t *>(base + L.book);
  uint64_t *bar_s0 = bars + 0;     // X and v (and the S0 image unless RING) landed
  uint64_t *bar1 = bars + 1;       // D1 complete
  uint64_t *bar_chain = bars + 2;  // ancestry warp: every beam's chain in s_chain
  uint64_t *bar_full = bars + 10;  // RING: slot holds its image chunk (bytes 80..103)
  uint64_t *bar_empty = bars + 13; // RING: the products reading the slot are done (bytes 104..127)
  uint32_t *s_tmem = reinterpret_cast<uint32_t *>(base + L.book + 64);
  int *s_U = reinterpret_cast<int *>(s_tmem + 1);
  int *s_mode = s_U + 1;  // the CTA's root: [0] its folded depth, [1] how it was chosen
  int *s_par = reinterpret_cast<int *>(base + L.book + 128);
  float *s_alpha = reinterpret_cast<float *>(s_par + kBT);
  float *s_beta = s_alpha + kBT;
  float *s_Gp = s_beta + kBT;  // P(parent)
  // [32][TM]: (k_a . k_b, k_a . q_b, slot of a, replay weight of a) for the
  // ancestor a of beam b at each depth.  The beam warps write the first two
  // words, the ancestry warp the last two.
  float4 *s_c = reinterpret_cast<float4 *>(s_Gp + kBT);
  int *s_chain = reinterpret_cast<int *>(s_c + kBT * TM);  // [32][TM] ancestor beam by depth
  int *s_list = s_chain + kBT * TM;  // slot -> (beam << 5 | depth-1), [(32 + 4) TM]
  float *s_w = reinterpret_cast<float *>(s_list + (kBT + 4) * TM);  // [32][TM] gates along the chains
  int *s_seen = reinterpret_cast<int *>(s_w + kBT * TM);           // beam index -> a lane (scratch)
  uint16_t *s_hist = reinterpret_cast<uint16_t *>(s_seen + ((p.W_max + 3) & ~3));  // parents of steps hcopy..t-1
  // Per-step table (index = step j), filled by the ancestry warp before the
  // first barrier with one load per lane: loops then read shared memory
  // instead of indexing the parameters at run time.
  const int32_t **s_tpar = reinterpret_cast<const int32_t **>(s_hist + ((p.hist_cap + 3) & ~3));
  const int NH = TM + 1;  // table entries: steps t - T_max .. t - 1 (hbase = t - T_max at most)
  const float **s_tg = reinterpret_cast<const float **>(s_tpar + NH);
  const __nv_bfloat16 **s_tk = reinterpret_cast<const __nv_bfloat16 **>(s_tg + NH);
  int *s_toff = reinterpret_cast<int *>(s_tk + NH);
  int *s_tW = s_toff + NH;
  int *s_trs = s_tW + NH;

  __nv_bfloat16 *rec_k = static_cast<__nv_bfloat16 *>(p.rec_k);
  const int64_t row0 = (int64_t)(r * p.W + b0) * H + h;  // (r, b0, h) row of [R][W][H][d]

  // --------------------------------------- setup; every load issued at once
  const uint32_t s0_bytes = (uint32_t)P * NK * 16384u;
  if (tid == 0) {
    ptx::mbar_init(bar_s0, 1);
    ptx::mbar_init(bar1, 1);
    ptx::mbar_init(bar_chain, 32 + (p.stall ? 1 : 0));  // stall (tests): an arrival that never comes
    if (RING)
      for (int i = 0; i < kRing; ++i) {
        ptx::mbar_init(bar_full + i, 1);
        ptx::mbar_init(bar_empty + i, 1);
      }
    ptx::mbar_fence_init();
    // The root this step replays from: the current folded state, or, while
    // the last fold is not complete, the one before it (where its depths fit
    // the record store; else this step waits for the kernel before it, whose
    // completion implies the fold's).  Decided once for the CTA.
    int mode = 0, d0s = 0;  // 0: current, 1: the one before the last fold, 2: current after the wait
    if (p.fold_pending && ptx::ld_acquire_gpu(p.fold_done + r) < p.fold_target) {
      d0s = p.d0_old ? p.d0_old[r] : 0;
      mode = t - 1 - d0s <= TM - 1 ? 1 : 2;
      if (mode == 2) ptx::pdl_wait();
    }
    if (mode != 1 && p.d0) d0s = p.d0[r];
    s_mode[0] = d0s;
    s_mode[1] = mode;
    // A new decode: its folds count from zero (no fold of an earlier decode
    // runs any more: step 1 is an ordinary launch).
    if (t == 1 && p.fold_reset && tile == 0 && h == 0 && mt == 0) p.fold_reset[r] = 0;
    // S0 image (bulk copy; RING: its first chunks, one per slot); k, q, v
    // tiles by TMA, beams past W read as zeros.
    ptx::mbar_arrive_expect_tx(bar_s0, (RING ? 0u : s0_bytes) + NK * XA + NV * VA);
    const uint8_t *src =
        static_cast<const uint8_t *>(mode == 1 ? p.S0img_old : p.S0img) + ((size_t)(r * H + h) * nmt + mt) * s0_bytes;
    if (RING) {
      for (int c = 0; c < kRing && c < P * NK; ++c) {
        ptx::mbar_arrive_expect_tx(bar_full + c, 16384u);
        ptx::bulk_g2s(base + L.a + c * 16384u, src + c * 16384u, 16384u, bar_full + c);
      }
    } else {
      for (uint32_t off = 0; off < s0_bytes; off += 16384u)
        ptx::bulk_g2s(base + L.a + off, src + off, 16384u, bar_s0);
    }
#pragma unroll
    for (int ka = 0; ka < NK; ++ka) {
      ptx::tma_load_4d(s_x + ka * XA, &p.tm_k, ka * 64, h, b0, r, bar_s0);
      ptx::tma_load_4d(s_x + ka * XA + kBT * 128, &p.tm_q, ka * 64, h, b0, r, bar_s0);
    }
#pragma unroll
    for (int ka = 0; ka < NV; ++ka) ptx::tma_load_4d(base + L.v + ka * VA, &p.tm_v, e_off + ka * 64, h, b0, r, bar_s0);
  }
  if (warp == kMmaWarp) {
    ptx::tmem_alloc(s_tmem, kTmemCols);
    ptx::tmem_relinquish();
  }
  // Before its wait this kernel reads inputs only, so the next step may start.
  ptx::pdl_launch_dependents();

  int par = 0;
  float g_alpha = 0.f, g_beta = 0.f;
  if (warp == kAncWarp) {
    // This tile's parents, gates and betas, and the per-step table.
    if (lane < nb) {
      par = t >= 2 ? p.parents[r * p.W + b0 + lane] : 0;
      const int64_t si = row0 + (int64_t)lane * H;
      g_alpha = p.g[si];
      g_beta = p.beta[si];
    }
    for (int e = lane; e < NH; e += 32) {
      s_tpar[e] = p.hpar[e];
      s_tg[e] = p.hg[e];
      s_tk[e] = static_cast<const __nv_bfloat16 *>(p.hk[e]);
      s_toff[e] = p.hoff[e];
      s_tW[e] = p.hW[e];
      s_trs[e] = p.hpar_rs[e];
    }
  }
  // The parents of steps hcopy..t-1 for this request as 16-bit indices,
  // back to back, each array starting on an 8-byte boundary: beam warp w >= 1
  // copies steps hcopy + w - 1, hcopy + w + 6, ...
  if (p.hist_cap > 0 && warp >= 1 && warp < kAncWarp)
#pragma unroll 2
    for (int j = p.hcopy + warp - 1; j < t; j += kAncWarp - 1)
      copy_parents16_warp(s_hist + p.hoff[j - hb], p.hpar[j - hb] + (int64_t)r * p.hpar_rs[j - hb], p.hW[j - hb],
                          lane);
  ptx::cp_async_commit();
  ptx::cp_async_wait_all();
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *s_tmem;
  if (s_mode[1] == 2) ptx::pdl_wait();
  // Depths 1..d0 are folded into the root; the beams replay depths
  // d0+1..t-1, which must fit the record store's T_max slots.
  int d0 = s_mode[0];
  if (t - 1 - d0 > TM - 1) {
    if (tid == 0) set_err(p.err, kErrByteWindow);
    d0 = t - TM;  // keeps every access inside the store; the results are void
  }
  const int nanc = t - 1 - d0;  // ancestors per beam; chain index j is depth d0+j+1
  const int jp = nanc - 1;      // chain index of the parents (depth t-1)
  const int soff = d0 % TM;     // slot of depth d0 + 1

  bool ok = true;
  const uint32_t x_u32 = ptx::smem_u32(s_x), a_u32 = ptx::smem_u32(base + L.a);
  const int wq = warp & 3;                        // TMEM lane quarter of this warp
  const uint32_t lb = (uint32_t)(wq * 32) << 16;  // its lane base

  // Beam-major phase (warps 0-7): thread (bb, l) owns elements
  // 32 (u ^ sx) + 4 l + z (z < 4) of beam bb, where sx = bb & 1: odd beams
  // take the 32-element groups in swapped pairs, so the four beams of a warp
  // reading rows at the same step cover all 32 banks.
  const int bb = tid >> 3, l = tid & 7, sx = bb & 1;
  const bool bval = bb < nb;  // false in the ancestry warp (bb >= 32)
  // This thread's elements of k_b and q_b, bf16: in registers, or (RING,
  // where the registers hold more key pieces in flight) read from X again.
  uint2 kb2[RING ? 1 : NUK], qb2[RING ? 1 : NUK];
  auto xpiece = [&](int u, int row) -> uint2 {
    const int uu = u ^ sx;
    const uint32_t off = (uint32_t)(uu >> 1) * XA + (uint32_t)(l & 1) * 8u;
    return *reinterpret_cast<const uint2 *>(s_x + off + ptx::swz128(row, 4 * (uu & 1) + (l >> 1)));
  };
  float kq = 0.f;

  if (warp == kAncWarp) {
    // ------------------------------------------------ the ancestry warp
    // Beam b's replayed ancestors a[j] at depth d0 + j + 1 (a[nanc-1] = its
    // parent; a[j] is the parent, at step d0 + j + 2, of a[j + 1]), the
    // tile's distinct ancestors and the replay weights.
    const int b = lane;
    if (b < nb && t >= 2 && (par < 0 || par >= p.W_prev)) {
      set_err(p.err, kErrByteParent);
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
        const int st = d0 + j + 2;  // the step whose parent array leads from depth st-1 to st
        const int si = st - hb;
        int pa = p.hist_cap > 0 ? s_hist[s_toff[si] + a] : s_tpar[si][(int64_t)r * s_trs[si] + a];
        if (pa < 0 || pa >= s_tW[si - 1]) pa = 0;  // reported by step st
        a = pa;
        s_chain[b * TM + j] = a;
      }
    }
    ptx::mbar_arrive(bar_chain);
    // The gates along the chain land in s_w (one round trip, overlapping
    // the distinct-ancestor pass); they become the replay weights.
    if (b < nb) {
#pragma unroll 1
      for (int j = 0; j <= jp; ++j) {
        const int a = s_chain[b * TM + j];
        const int di = d0 + j + 1 - hb;  // history entry of the record's depth
        const int sl = soff + j < TM ? soff + j : soff + j - TM;
        ptx::cp_async4(s_w + b * TM + j, (hmask >> di) & 1ull ? s_tg[di] + ((int64_t)r * s_tW[di] + a) * H + h
                                                           : p.rec_alpha + rec_row_slot(p, sl, r, h, a));
      }
    }
    ptx::cp_async_commit();
    // Distinct ancestors depth by depth: every lane writes its lane number
    // at its ancestor's index, and the lane whose number survives leads that
    // ancestor.  Slots in order of depth, then of the leading lane.
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
      if (b < nb) reinterpret_cast<float *>(s_c + b * TM + j)[2] = __int_as_float(slot);
      U += __popc(leaders);
    }
    if (lane == 0) *s_U = U;
    // Replay weights (products of the later gates) and P(p) (all of them).
    ptx::cp_async_wait_all();
    float w = 1.f;
    if (b < nb) {
#pragma unroll 1
      for (int j = jp; j >= 0; --j) {
        const float gj = s_w[b * TM + j];
        reinterpret_cast<float *>(s_c + b * TM + j)[3] = w;
        w *= (hmask >> (d0 + j + 1 - hb)) & 1ull ? expf(gj) : gj;
      }
    }
    s_Gp[b] = w;
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------ the MMA warp
    // D1 = S0 . X^T on the tensor cores, issued by lane 0 once the image is
    // here.
    if (lane == 0 && RING) {
      // The image chunk by chunk (plane-major, then K atom) through the
      // ring: a slot is refilled with the chunk kRing further on once the
      // products reading it are done.  A wait that runs out stops the issue.
      ok = ptx::mbar_wait(bar_s0, 0, p.wait_limit_ns);
      ptx::tc_fence_after();
      constexpr uint32_t idesc1 = ptx::idesc_bf16_f32(kM, kN);
      const uint8_t *src = static_cast<const uint8_t *>(s_mode[1] == 1 ? p.S0img_old : p.S0img) +
                           ((size_t)(r * H + h) * nmt + mt) * s0_bytes;
      const int nch = P * NK;
      int issued = nch < kRing ? nch : kRing, landed = 0;  // chunks issued / waited for
      int acc = 0;
      for (int c = 0; c < nch && ok; ++c) {
        const int sl = c % kRing;
        const uint32_t ph = (uint32_t)(c / kRing) & 1u;
        if (!ptx::mbar_wait(bar_full + sl, ph, p.wait_limit_ns)) {
          ok = false;
          break;
        }
        landed = c + 1;
        ptx::tc_fence_after();
        const int ka = c % NK;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint64_t ad = ptx::desc_k128(a_u32 + sl * 16384 + kk * 32);
          const uint64_t bd = ptx::desc_k128(x_u32 + ka * XA + kk * 32);
          ptx::mma_bf16(tmem, ad, bd, idesc1, acc);
          acc = 1;
        }
        if (c + kRing < nch) {
          ptx::mma_commit(bar_empty + sl);
          if (!ptx::mbar_wait(bar_empty + sl, ph, p.wait_limit_ns)) {
            ok = false;
            break;
          }
          ptx::mbar_arrive_expect_tx(bar_full + sl, 16384u);
          ptx::bulk_g2s(base + L.a + sl * 16384u, src + (size_t)(c + kRing) * 16384u, 16384u, bar_full + sl);
          ++issued;
        }
      }
      // After a wait that ran out, the chunks still in flight land before
      // the CTA goes on (each wait bounded again).
      for (int c = landed; !ok && c < issued; ++c)
        ptx::mbar_wait(bar_full + c % kRing, (uint32_t)(c / kRing) & 1u, p.wait_limit_ns);
      ptx::mma_commit(bar1);
    } else if (lane == 0) {
      ok = ptx::mbar_wait(bar_s0, 0, p.wait_limit_ns);
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
  } else {
    // ------------------------------------------------ the beam warps
    if (!ptx::mbar_wait(bar_s0, 0, p.wait_limit_ns)) {  // X and v visible to this thread
      ok = false;
      // The copies still in flight land before the CTA can exit (bounded again).
      if (tid == 0) ptx::mbar_wait(bar_s0, 0, p.wait_limit_ns);
    }
    // This thread's elements of k_b and q_b, and k_b . q_b.
#pragma unroll
    for (int u = 0; u < NUK; ++u) {
      const uint2 kx = xpiece(u, bb), qx = xpiece(u, kBT + bb);
      if constexpr (!RING) kb2[u] = kx, qb2[u] = qx;
      const float4 kf = bf16x4(kx), qf = bf16x4(qx);
      kq = fmaf(kf.x, qf.x, kq);
      kq = fmaf(kf.y, qf.y, kq);
      kq = fmaf(kf.z, qf.z, kq);
      kq = fmaf(kf.w, qf.w, kq);
    }
    kq += __shfl_xor_sync(0xffffffffu, kq, 4);
    kq += __shfl_xor_sync(0xffffffffu, kq, 2);
    kq += __shfl_xor_sync(0xffffffffu, kq, 1);
    // k_a . k_b and k_a . q_b for the beam's ancestor a at every depth: the
    // thread's pieces of each ancestor's key row come straight from global
    // memory (step j's own k input, or the key records), two depths per
    // pass, the next pass's loads in flight during this pass's arithmetic.
    if (!ptx::mbar_wait(bar_chain, 0, p.wait_limit_ns)) ok = false;
    auto issue = [&](uint2 (&buf)[2][NUK], int j0) {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int j = j0 + e;
        if (bval && j < nanc) {
          const int a = s_chain[bb * TM + j];
          const int di = d0 + j + 1 - hb;
          const int sl = soff + j < TM ? soff + j : soff + j - TM;
          const __nv_bfloat16 *row = (hmask >> di) & 1ull ? s_tk[di] + ((int64_t)(r * s_tW[di] + a) * H + h) * DK
                                         : rec_k + rec_row_slot(p, sl, r, h, a) * DK;
          const uint8_t *rb = reinterpret_cast<const uint8_t *>(row) + l * 8;
#pragma unroll
          for (int u = 0; u < NUK; ++u) buf[e][u] = __ldg(reinterpret_cast<const uint2 *>(rb + (u ^ sx) * 64));
        } else {
#pragma unroll
          for (int u = 0; u < NUK; ++u) buf[e][u] = make_uint2(0u, 0u);
        }
      }
    };
    auto dots = [&](const uint2 (&buf)[2][NUK], int j0) {
      float dk[2], dq[2];
#pragma unroll
      for (int e = 0; e < 2; ++e) dk[e] = 0.f, dq[e] = 0.f;
#pragma unroll
      for (int u = 0; u < NUK; ++u) {
        float4 kbu, qbu;
        if constexpr (RING)
          kbu = bf16x4(xpiece(u, bb)), qbu = bf16x4(xpiece(u, kBT + bb));
        else
          kbu = bf16x4(kb2[u]), qbu = bf16x4(qb2[u]);
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const float4 kf = bf16x4(buf[e][u]);
          dk[e] = fmaf(kf.x, kbu.x, dk[e]);
          dk[e] = fmaf(kf.y, kbu.y, dk[e]);
          dk[e] = fmaf(kf.z, kbu.z, dk[e]);
          dk[e] = fmaf(kf.w, kbu.w, dk[e]);
          dq[e] = fmaf(kf.x, qbu.x, dq[e]);
          dq[e] = fmaf(kf.y, qbu.y, dq[e]);
          dq[e] = fmaf(kf.z, qbu.z, dq[e]);
          dq[e] = fmaf(kf.w, qbu.w, dq[e]);
        }
      }
      // Sum the four values over the beam's 8 threads in 4 shuffles: each
      // level hands half of the values still held to the partner and keeps
      // the other half, so thread l ends with value 2 (l >> 2) + ((l >> 1) & 1)
      // (dk of depth j0, dq of j0, dk of j0 + 1, dq of j0 + 1).
      const bool b2 = (l >> 2) & 1, b1 = (l >> 1) & 1;
      const float s0v = __shfl_xor_sync(0xffffffffu, b2 ? dk[0] : dk[1], 4);
      const float s1v = __shfl_xor_sync(0xffffffffu, b2 ? dq[0] : dq[1], 4);
      const float w0 = (b2 ? dk[1] : dk[0]) + s0v, w1 = (b2 ? dq[1] : dq[0]) + s1v;
      float x = (b1 ? w1 : w0) + __shfl_xor_sync(0xffffffffu, b1 ? w0 : w1, 2);
      x += __shfl_xor_sync(0xffffffffu, x, 1);
      const int j = j0 + (int)b2;
      if ((l & 1) == 0 && bval && j < nanc) reinterpret_cast<float *>(s_c + bb * TM + j)[b1] = x;
    };
    uint2 kA[2][NUK], kB[2][NUK];
    if (nanc > 0) issue(kA, 0);
#pragma unroll 1
    for (int j0 = 0; j0 < nanc; j0 += 4) {
      if (j0 + 2 < nanc) issue(kB, j0 + 2);
      dots(kA, j0);
      if (j0 + 2 >= nanc) break;
      if (j0 + 4 < nanc) issue(kA, j0 + 4);
      dots(kB, j0 + 2);
    }
    if (warp >= 4) {
      // D1^T into shared memory (region A: the image is consumed).
      const int ei = wq * 32 + lane;  // TMEM lane: output element of D1
      if (!ptx::mbar_wait(bar1, 0, p.wait_limit_ns)) ok = false;
      ptx::tc_fence_after();
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        float d[32];
        ptx::tmem_ld32(tmem + lb + half * 32, d);
        ptx::tmem_ld_wait();
        if (wq * 32 < DV)
#pragma unroll
          for (int n = 0; n < 32; ++n) s_d1[(half * 32 + n) * DV + ei] = d[n];
      }
    } else if (mt == 0) {
      // The key records of depth t, from X (once per beam tile).
      for (int e = tid; e < kBT * NK * 8; e += 128) {
        const int n = e / (NK * 8), cc = e - n * (NK * 8);
        if (n < nb)
          reinterpret_cast<uint4 *>(rec_k + rec_row_slot(p, tslot, r, h, b0 + n) * DK)[cc] =
              *reinterpret_cast<const uint4 *>(s_x + (cc >> 3) * XA + ptx::swz128(n, cc & 7));
      }
    }
    // alpha, the ancestry row and the parent of the beam (once per beam tile).
    if (bval && l == 0 && mt == 0) {
      const int gb = b0 + bb;
      p.rec_alpha[rec_row_slot(p, tslot, r, h, gb)] = s_alpha[bb];
      if (h == 0) {
        // Entry (depth - 1) mod T_max for the last T_max - 1 depths before t:
        // the folded ones from the shared ancestors, the others from the chain.
        int32_t *row = p.anc + ((int64_t)(tslot * p.R + r) * p.W_max + gb) * TM;
        // dlo - 1 = t - T_max past the first T_max steps, whose entry
        // follows the slot of depth t; stepped with a wrap.
        const int dlo = max(1, t - TM + 1);
        int e = t > TM ? (tslot + 1 < TM ? tslot + 1 : 0) : 0;
#pragma unroll 1
        for (int dd = dlo; dd < t; ++dd) {
          row[e] = dd <= d0 ? p.anc_fold[r * TM + e] : s_chain[bb * TM + dd - 1 - d0];
          e = e + 1 < TM ? e + 1 : 0;
        }
        p.par_store[((int64_t)tslot * p.R + r) * p.W_max + gb] = s_par[bb];
      }
    }
  }
  ptx::tc_fence_before();
  __syncthreads();  // every role done: D1^T, key products, slots, weights
  if (warp == kMmaWarp) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, kTmemCols);
  }

  // u = P(p) D1 + (replayed terms, after the wait); v from its tile.
  const int U = *s_U;
  float acc_k[4 * NU], acc_q[4 * NU];
  float4 vf[NU];
  const float Gp = warp < kAncWarp ? s_Gp[bb] : 0.f;  // beam warps only from here on
  const float alpha = warp < kAncWarp ? s_alpha[bb] : 0.f, beta = warp < kAncWarp ? s_beta[bb] : 0.f;
  if (warp < kAncWarp) {
#pragma unroll
    for (int u = 0; u < NU; ++u) {
      const int uu = u ^ sx;
      const float4 dk = reinterpret_cast<const float4 *>(s_d1 + bb * DV)[8 * uu + l];
      const float4 dq = reinterpret_cast<const float4 *>(s_d1 + (kBT + bb) * DV)[8 * uu + l];
      acc_k[4 * u + 0] = Gp * dk.x, acc_k[4 * u + 1] = Gp * dk.y, acc_k[4 * u + 2] = Gp * dk.z, acc_k[4 * u + 3] = Gp * dk.w;
      acc_q[4 * u + 0] = Gp * dq.x, acc_q[4 * u + 1] = Gp * dq.y, acc_q[4 * u + 2] = Gp * dq.z, acc_q[4 * u + 3] = Gp * dq.w;
      vf[u] = bf16x4(s_v + (uu >> 1) * VA + ptx::swz128(bb, 4 * (uu & 1) + (l >> 1)) + (l & 1) * 8);
    }
  }
  __syncthreads();  // D1^T consumed before the deltas overwrite region A

  // ------------------------------- after the wait: the ancestors' deltas
  ptx::pdl_wait();
  constexpr int PD = DV / 4;  // 16-byte pieces of a delta row
  for (int lo = 0; lo < U; lo += DR) {
    const int hi = min(U, lo + DR);
    const int nrows = hi - lo;
    if (lo > 0) __syncthreads();  // the previous round's deltas are consumed
    // The rows of slots lo .. hi - 1 in 16-byte pieces (a warp copies whole
    // rows), then every thread waits for its own pieces and the block syncs.
#pragma unroll 1
    for (int e = tid; e < nrows * PD; e += kThreads) {
      const int rr = e / PD, c = e - rr * PD;
      const int packed = s_list[lo + rr];
      const int j = packed & 31, sl = soff + j < TM ? soff + j : soff + j - TM;
      ptx::cp_async16(base + L.dst + (uint32_t)(rr * DV + c * 4) * 4u,
                      p.rec_delta + rec_row_slot(p, sl, r, h, packed >> 5) * DVT + e_off + c * 4, 16u);
    }
    ptx::cp_async_commit();
    ptx::cp_async_wait_all();
    __syncthreads();
    if (bval) {
      // Two depths per pass: their loads are independent.
#pragma unroll 1
      for (int j0 = 0; j0 < nanc; j0 += 2) {
        float ck[2], cq[2];
        const float4 *row[2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const float4 c = j0 + e < nanc ? s_c[bb * TM + j0 + e] : make_float4(0.f, 0.f, __int_as_float(-1), 0.f);
          const unsigned sl = (unsigned)(__float_as_int(c.z) - lo);
          const bool in = sl < (unsigned)nrows;
          row[e] = reinterpret_cast<const float4 *>(s_dst + (in ? sl : 0u) * DV) + l;
          ck[e] = in ? c.x * c.w : 0.f;
          cq[e] = in ? c.y * c.w : 0.f;
        }
#pragma unroll
        for (int u = 0; u < NU; ++u) {
          const float4 e0 = row[0][8 * (u ^ sx)], e1 = row[1][8 * (u ^ sx)];
          acc_k[4 * u + 0] = fmaf(e1.x, ck[1], fmaf(e0.x, ck[0], acc_k[4 * u + 0]));
          acc_k[4 * u + 1] = fmaf(e1.y, ck[1], fmaf(e0.y, ck[0], acc_k[4 * u + 1]));
          acc_k[4 * u + 2] = fmaf(e1.z, ck[1], fmaf(e0.z, ck[0], acc_k[4 * u + 2]));
          acc_k[4 * u + 3] = fmaf(e1.w, ck[1], fmaf(e0.w, ck[0], acc_k[4 * u + 3]));
          acc_q[4 * u + 0] = fmaf(e1.x, cq[1], fmaf(e0.x, cq[0], acc_q[4 * u + 0]));
          acc_q[4 * u + 1] = fmaf(e1.y, cq[1], fmaf(e0.y, cq[0], acc_q[4 * u + 1]));
          acc_q[4 * u + 2] = fmaf(e1.z, cq[1], fmaf(e0.z, cq[0], acc_q[4 * u + 2]));
          acc_q[4 * u + 3] = fmaf(e1.w, cq[1], fmaf(e0.w, cq[0], acc_q[4 * u + 3]));
        }
      }
    }
  }

  // --------------------------------------------------------- epilogue
  if (!ok) set_err(p.err, kErrByteTimeout);
  if (bval && ok) {
    float4 *op = reinterpret_cast<float4 *>(p.o + (row0 + (int64_t)bb * H) * DVT + e_off) + l;
    float4 *dp = reinterpret_cast<float4 *>(p.rec_delta + rec_row_slot(p, tslot, r, h, b0 + bb) * DVT + e_off) + l;
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
      op[8 * (u ^ sx)] = o;
      dp[8 * (u ^ sx)] = d;
    }
  }
}

__global__ void s0_image_kernel(const void *S0, uint4 *img, int R, int H, int dk, int dv, int s0_bf16,
                                int planes) {
  // Layout [r][h][M tile of 128 rows][plane][K atom][128 rows][128 B]; one
  // thread per 16-byte chunk.  Rows past d_v are zero.
  const int nk = dk / 64, nmt = (dv + kM - 1) / kM;
  const int64_t total = (int64_t)R * H * nmt * planes * nk * kM * 8;
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < total;
       e += (int64_t)gridDim.x * blockDim.x) {
    int64_t x = e;
    const int c = (int)(x % 8); x /= 8;
    const int row = (int)(x % kM); x /= kM;
    const int ka = (int)(x % nk); x /= nk;
    const int pl = (int)(x % planes); x /= planes;
    const int mt = (int)(x % nmt); x /= nmt;
    const int64_t rh = x;
    const int srow = mt * kM + row;
    __align__(16) __nv_bfloat16 out[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      float s = 0.f;
      if (srow < dv) {
        const int64_t si = (rh * dv + srow) * dk + ka * 64 + c * 8 + u;
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
    const int64_t off = (((rh * nmt + mt) * planes + pl) * nk + ka) * (kM * 128) + ptx::swz128(row, c);
    img[off / 16] = *reinterpret_cast<const uint4 *>(out);
  }
}

// cuTensorMapEncodeTiled, fetched once from the driver (thread-safe static
// initialisation).
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static const PFN_cuTensorMapEncodeTiled_v12000 fn = []() -> PFN_cuTensorMapEncodeTiled_v12000 {
    void *ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    return nullptr;
  }();
  return fn;
}

}  // namespace

bool encode_rows(CUtensorMap *m, const void *base, int d, int H, int W, int R, int box_rows) {
  PFN_cuTensorMapEncodeTiled_v12000 fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)H, (cuuint64_t)W, (cuuint64_t)R};
  const cuuint64_t strides[3] = {(cuuint64_t)d * 2, (cuuint64_t)H * d * 2, (cuuint64_t)W * H * d * 2};
  const cuuint32_t box[4] = {64, 1, (cuuint32_t)box_rows, 1};
  const cuuint32_t es[4] = {1, 1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

namespace {

template <int DK, int DV, int MINB = 2>
cudaError_t launch_dk(const StepParams &p_in, bool pdl, cudaStream_t s) {
  StepParams p = p_in;
  if (!encode_rows(&p.tm_k, p.k, DK, p.H, p.W, p.R) || !encode_rows(&p.tm_q, p.q, DK, p.H, p.W, p.R) ||
      !encode_rows(&p.tm_v, p.v, DK, p.H, p.W, p.R))
    return cudaErrorInvalidValue;

  const Layout L = layout(DK / 64, DV / 64, p.s0_planes, p.T_max, p.W_max, p.hist_cap, DK > 128);
  const dim3 grid((p.W + kBT - 1) / kBT, p.H, p.R * (p.dv / DV));
  const size_t smem = L.total + 1024;
  cudaError_t e = ensure_smem_limit((const void *)step_tc_kernel<DK, DV, MINB>, smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, step_tc_kernel<DK, DV, MINB>, p);
}

}  // namespace

bool tc_supports(int dk, int dv, int qkv_bf16, int T_max, int W_max, int planes) {
  // d = 256: one CTA per half of the rows of S, its image streamed through
  // a ring of shared-memory slots (any number of terms).
  return qkv_bf16 && dk == dv && (dk == 64 || dk == 128 || dk == 256) && planes >= 1 && planes <= 3 &&
         T_max <= kMaxT && W_max <= kMaxW;
}

size_t s0_image_bytes(int R, int H, int dk, int dv, int planes) {
  return (size_t)R * H * ((dv + kM - 1) / kM) * planes * (dk / 64) * 16384u;
}

cudaError_t launch_s0_image(const void *S0, void *img, int R, int H, int dk, int dv, int s0_bf16, int planes,
                            cudaStream_t s) {
  const int64_t total = (int64_t)R * H * ((dv + kM - 1) / kM) * planes * (dk / 64) * kM * 8;
  const int threads = 256;
  const int64_t want = (total + threads - 1) / threads;
  const int blocks = (int)(want < 148 * 16 ? want : 148 * 16);
  s0_image_kernel<<<blocks, threads, 0, s>>>(S0, static_cast<uint4 *>(img), R, H, dk, dv, s0_bf16, planes);
  return cudaGetLastError();
}

cudaError_t launch_step_tc(const StepParams &p, int pdl, cudaStream_t s) {
  if (p.T_max > kMaxT || p.W_max > kMaxW || p.s0_planes < 1 || p.s0_planes > 3 || p.hist_cap > kHistMaxInts)
    return cudaErrorNotSupported;
  if (p.dk == 64 && p.dv == 64) {
    // At d = 64 the kernel also builds with 64 registers, three CTAs per SM:
    // faster once a step has more CTAs than two per SM hold, slower below
    // (the 80-register build keeps more loads in flight).
    if ((long)((p.W + kBT - 1) / kBT) * p.H * p.R > 2L * kSMs) return launch_dk<64, 64, 3>(p, pdl != 0, s);
    return launch_dk<64, 64, 2>(p, pdl != 0, s);
  }
  if (p.dk == 128 && p.dv == 128) return launch_dk<128, 128>(p, pdl != 0, s);
  if (p.dk == 256 && p.dv == 256) return launch_dk<256, 128>(p, pdl != 0, s);
  return cudaErrorNotSupported;
}

}  // namespace onela
