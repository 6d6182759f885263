// Per-row top-k selection and sparse attention on one thread-block cluster.
//
// Top-k ("Why Is DeepSeek V4.1 Flash So Fast?", sections 3-4: keep the
// Top-K compressed positions by indexer score; ties to the lower index and
// ascending output are this library's readings) and attention (section 3:
// the selected positions plus the 128-token window; "Inference-Efficient
// LLMs", sections 3 and 6: per-layer bf16 window, FP4 global entries; one
// joint softmax, an entry is both key and value and serves every head).
//
// One cluster of CL CTAs owns one query row; CTA c owns a contiguous slice
// of the row's entries.  Histogram slices, counts and softmax partials move
// between the CTAs by st.async into the receiver's shared memory, each
// delivery counted in bytes on the receiver's own mbarrier: a CTA waits only
// for the data it needs, and only the prologue (every CTA running, its
// barriers initialised) and the step between head passes use a cluster-wide
// barrier.
//
// Top-k: exact radix selection on an order-preserving 32-bit key of the
// score, digits of 11, 11 and 10 bits.  The scan kernel has histogrammed
// digit 1 of every visible score.  Each CTA stages that histogram and its
// score slice in shared memory with bulk copies, then
//   1. finds the digit-1 threshold t1 (largest digit whose suffix count
//      reaches k) and lists the elements of its slice with digit 1 >= t1,
//      in index order (each thread masks a contiguous run, one block
//      prefix, then each thread writes its run's candidates), histogramming
//      digit 2 of the elements exactly at t1;
//   2. reduces the cluster's digit-2 histograms (CTA c sums bin slice c of
//      every rank and delivers the sums to every rank; every CTA then finds
//      t2 locally) -> t2;
//   3. only when the boundary bucket (t1, t2) holds more elements than still
//      needed: the same for digit 3 -> t3;
//   4. classifies the candidates as above the threshold key or equal to
//      it.  Equal keys are equal scores; they are taken in index order
//      (lower index first) up to the count still needed.  Prefix sums over
//      ranks and threads give every thread its offset in the output row, so
//      the indices come out ascending.  When every equal key is taken (the
//      usual case: the cluster holds exactly as many as are still needed),
//      a CTA's selection does not depend on the other ranks: it attends at
//      once, and the warps that do not attend exchange the counts and write
//      the output indices meanwhile.
//
// Attention: each CTA attends over an even share of the window rows and over
// the entries it selected itself (with given indices, an even share of the
// index slots), cut into 16-key chunks that kAttnWarps warps take in turn,
// each with its own online softmax in base 2 (the per-warp blocks of
// attn_rows.cuh: gather by cp.async with invalid keys zero-filled, E2M1 ->
// exact bf16, mma.sync m16n8k16 with 16 heads as M):
//   logits  S[h, n] = sum_g s[n, g] * sum_{i in g} q[h, i] * e2m1[n, i]
//           one product per 16-element scale group g; E2M1 values and the
//           bf16 query are exact in bf16, so every product is exact and the
//           group scale is applied in fp32 afterwards;
//   values  O[h, d] += sum_n (P[h, n] * s[n, g(d)]) * e2m1[n, d]
//           with the fp32 weight P*s split into a bf16 pair hi + lo (two
//           products), so the weight keeps ~16 bits.
// Window rows use the same path with scale 1 (bf16 keys and values); they do
// not depend on the selection, so one warp of its own attends over the CTA's
// share of them (its first chunk's copies issued in the prologue, while the
// scan that produces the scores may still run) alongside the entry warps,
// and its state joins the merge.  The warps' states are merged in shared memory (their buffers alias the dead
// top-k working set), and each CTA pushes its partial (max, sum, acc) of
// head h into the shared memory of the CTA that owns h (h mod CL); once its
// partials are in, each owner merges them locally by log-sum-exp.  Which CTA
// handles which key does not change the result, so no entry is moved
// between CTAs.
#pragma once
#include <cooperative_groups.h>

#include "attn_rows.cuh"
#include "common.cuh"
#include "pack.cuh"

namespace csa2 {

namespace cg = cooperative_groups;

constexpr int kRowThreads = 512;
constexpr int kRowWarps = kRowThreads / 32;
constexpr int kStageScores = 16384;  // scores staged in shared memory per round
constexpr int kCandCap = 2048;       // candidates kept in shared memory (more spill to global)
constexpr int kSelCap = 4096;        // selected indices kept in shared memory
constexpr int kHeads = 16;           // heads per pass (the MMA's M)
constexpr int kAttnWarps = 10;       // warps that run attention chunks of the selected entries
constexpr int kWinWarp = kRowWarps - 1;  // the warp that attends over the CTA's window rows

struct RowParams {
  // top-k
  const float *scores;      // [rows_local, score_stride] (this launch's rows)
  int64_t score_stride;
  const uint32_t *hist1;    // [rows_local, kHistStride] (digit-1 histogram first)
  uint2 *cand;              // [rows_local, N] candidate overflow regions
  int64_t N;
  int32_t T;
  int64_t n_prior;
  int32_t ratio;
  int64_t row0;             // first global row of this launch
  int32_t topk;
  int32_t *idx;             // [rows_global, topk]: written (top-k) / read (attention only)
  // attention
  const uint16_t *q;        // [rows_global, H, D] bf16
  const uint8_t *codes;     // [B, N, D/2]
  const float *scales;      // [B, N, D/16]
  const uint16_t *win_k;    // [B, W-1+T, D] bf16
  const uint16_t *win_v;
  int32_t H, W;
  float q_scale;            // sm_scale * log2(e)
  float *out;               // [rows_global, H, D]
  float *lse;               // [rows_global, H] or null
  int do_topk, do_attn;
  // hand-off to an attention kernel launched after this one (top-k only,
  // the kernel's HO instances):
  // CTA c of row r_local writes its selected indices (ascending) to
  // lists[(r_local * CL + c) * list_stride ...] and then n + 1 into the
  // ready flag hist1[r_local * kHistStride + kBins1 + c]; null: no hand-off
  int32_t *lists;
  int64_t list_stride;
};

// Publish this CTA's selection (sel[0..n), ascending) to the attention
// kernel that follows: the indices, then (one thread, after a fence at GPU
// scope) the ready flag n + 1.
template <int CL, class S>
__device__ void publish_selection(S &sm, const RowParams &p, int64_t r_local, int c,
                                  uint32_t n) {
  int32_t *dst = p.lists + (r_local * CL + c) * p.list_stride;
  for (uint32_t i = threadIdx.x; i < n; i += kRowThreads) dst[i] = sm.sel[i];
  __syncthreads();
  if (threadIdx.x == 0) {
    uint32_t *flag = const_cast<uint32_t *>(p.hist1) + r_local * kHistStride + kBins1 + c;
    __threadfence();
    asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(flag), "r"(n + 1u) : "memory");
  }
}

template <int D>
struct RowSmem {
  union {
    struct {  // top-k working set
      float sc[kStageScores];                                    // staged score slice
      uint2 cand[kCandCap];    // candidates (key, index - slice start); more spill to global
    } tk;
    ar::WarpArea<D> aw[kAttnWarps];  // attention: per-warp chunk buffers, then partial states
  } u;
  alignas(16) uint32_t h1[kBins1];    // staged digit-1 histogram
  alignas(16) uint32_t h2[kBins2];    // own digit-2 (then digit-3) histogram
  alignas(16) uint32_t hin[kBins2];   // bin slice this CTA owns, one row per source rank (pushed)
  alignas(16) uint32_t full[kBins2];  // cluster-wide histogram (reduced slices pushed by owners)
  alignas(8) uint32_t cnt_all[32][2];      // every rank's (above, tie) counts (pushed)
  int32_t sel[kSelCap];         // this CTA's selected indices, ascending
  uint16_t qb[kHeads][D + 8];   // query of the head pass, bf16
  // pushed partials of the heads this CTA merges: (m, l, -, -, acc[D])
  alignas(16) float inbox[kHeads][D + 4];
  // per head: the factor of each source (attention warps, then the window
  // state), then the max
  float mf[kHeads][kAttnWarps + 2];
  float fac[kHeads];            // final merge: factor of each inbox slot
  float mrg_m[kHeads], mrg_l[kHeads];  // final merge: max and sum of each merged head
  uint32_t scratch[40];
  uint32_t thr[8];
  uint32_t cnt[4];  // [1] above-threshold, [2] equal-to-threshold, [3] reduced-slice total
  uint32_t sel_base, sel_count, out_base, tie_base;
  uint64_t bar;
  // exchange barriers, one per delivery (bytes counted by st.async):
  // digit-2 slices, digit-2 sums, digit-3 slices, digit-3 sums, counts, partials
  uint64_t xbar[6];
  // the window warp's chunk area, then its partial state
  ar::WarpArea<D> win;
};

__device__ __forceinline__ int64_t row_visible(int64_t N, int64_t n_prior, int32_t ratio,
                                               int64_t t) {
  if (n_prior < 0) return N;
  const int64_t v = n_prior + (t + 1) / ratio;
  return v < N ? v : N;
}

// Candidate class against the threshold key (t1, t2, t3): 2 above, 1 equal, 0 below.
__device__ __forceinline__ uint32_t cand_class(uint32_t k, uint32_t t1, uint32_t t2, uint32_t t3,
                                               bool need3) {
  const uint32_t a = key_d1(k), b = key_d2(k), c = key_d3(k);
  if (a > t1 || (a == t1 && b > t2)) return 2u;
  if (a == t1 && b == t2) {
    if (!need3 || c > t3) return 2u;
    if (c == t3) return 1u;
  }
  return 0u;
}

// Cluster-wide histogram of NB bins (each CTA's own counts in sm.h2) ->
// the largest bin t whose cluster-wide suffix count reaches `need`, the
// count strictly above it and the count of bin t, in out[0..2].  Push-based,
// in 16-byte pieces of 4 bins delivered by st.async: every CTA stores bin
// slice j of its histogram into CTA j's `hin` (counted on bar_in); CTA j,
// once its NB * 4 bytes are in, reduces its slice (thread u sums 4 bins over
// the CL sources) and stores the sums into the `full` of every CTA (counted
// on bar_full); each CTA finds the threshold once its own `full` is
// complete.  No cluster-wide barrier: a CTA reduces only after every CTA has
// delivered to it, i.e. after every CTA is done with the previous use of
// `full`; callers make sure the same holds for `hin`.
template <int D, int CL, int NB>
__device__ void cluster_threshold(RowSmem<D> &sm, cg::cluster_group &cluster, uint32_t need,
                                  uint32_t *out, uint64_t *bar_in, uint64_t *bar_full,
                                  bool &abort) {
  constexpr int BPC = NB / CL;  // bins owned by each CTA
  constexpr int G4 = BPC / 4;   // 4-bin pieces owned by each CTA
  static_assert(BPC % 4 == 0, "16-byte pieces");
  const int tid = threadIdx.x;
  const int c = (int)cluster.block_rank();
  if (tid == 0) {
    mbar_arrive_expect_tx(bar_in, NB * 4);
    mbar_arrive_expect_tx(bar_full, NB * 4);
  }
  for (int q = tid; q < NB / 4; q += kRowThreads) {
    const int i = 4 * q, owner = i / BPC;
    const uint4 v = *reinterpret_cast<const uint4 *>(&sm.h2[i]);
    st_async_v4(&sm.hin[c * BPC + (i - owner * BPC)], v, bar_in, (uint32_t)owner);
  }
  if (!mbar_wait_cluster_bounded(bar_in, 0)) abort = true;
  for (int u = tid; u < G4 * CL; u += kRowThreads) {
    const int g = u % G4, j = u / G4;
    uint4 s = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
    for (int src = 0; src < CL; ++src) {
      const uint4 v = *reinterpret_cast<const uint4 *>(&sm.hin[src * BPC + 4 * g]);
      s.x += v.x;
      s.y += v.y;
      s.z += v.z;
      s.w += v.w;
    }
    st_async_v4(&sm.full[c * BPC + 4 * g], s, bar_full, (uint32_t)j);
  }
  if (!mbar_wait_cluster_bounded(bar_full, 0)) abort = true;
  radix_threshold<kRowThreads, NB>(sm.full, need, sm.scratch, out);
  if (tid == 0) out[2] = sm.full[out[0]];
  __syncthreads();
}


// Returns true when the CTA's selection is complete in `sel` but its
// indices are not yet written to the output row: every tie at the threshold
// key is taken and the selection fits `sel`, so the CTA's selection does not
// depend on the other ranks' counts and attention may start at once; the
// counts exchange and the index write are then left to the warps that do not
// attend (write_row_indices).
template <int D, int CL, bool HO>
__device__ bool row_topk(RowSmem<D> &sm, const RowParams &p, cg::cluster_group &cluster,
                         int64_t r_local, int64_t r, int64_t K, bool bulk, int64_t s0, int64_t s1,
                         bool &abort, uint32_t &phase) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int c = (int)cluster.block_rank();
  const uint32_t lt = lanemask_lt_u32();
  int32_t *orow = p.idx + r * (int64_t)p.topk;
  const float *srow = p.scores + r_local * p.score_stride;
  uint2 *spill = p.cand + r_local * p.N + s0;  // candidates beyond kCandCap, by list position

  // The digit-1 histogram and the first score round were issued in the
  // prologue.  A wait that gives up is recorded in the status word; the CTA
  // still runs every phase (all indices stay bounded) so barriers match.
  if (!mbar_wait_bounded(&sm.bar, phase & 1u)) abort = true;
  ++phase;
  __syncthreads();
  radix_threshold<kRowThreads, kBins1>(sm.h1, (uint32_t)K, sm.scratch, sm.thr);
  const uint32_t t1 = sm.thr[0], r1 = (uint32_t)K - sm.thr[1];

  // 1. candidate list in index order: thread t owns the contiguous run
  //    [32t, 32t + 32) of each staged round; a mask of its elements with
  //    digit 1 >= t1 (16-byte reads, rotated per thread: conflict-free),
  //    one block prefix over the counts, then each thread writes its
  //    candidates and histograms digit 2 of those exactly at t1.
  static_assert(kStageScores == 32 * kRowThreads, "one 32-bit mask per thread and round");
  // digit 1 >= t1  <=>  key >= t1 << 21  <=>  score >= f1, the smallest
  // score with that key (keys are monotone in the score; no -0 or NaN);
  // for t1 <= 3 every key above the NaN patterns qualifies: f1 = -inf
  const uint32_t k1 = t1 << 21;
  const float f1 = (t1 <= 3u) ? -__int_as_float(0x7f800000)
                              : __uint_as_float((k1 & 0x80000000u) ? (k1 & 0x7fffffffu) : ~k1);
  uint32_t count = 0;
  for (int64_t rb = s0; rb < s1; rb += kStageScores) {
    const int n = (int)min64(kStageScores, s1 - rb);
    if (rb != s0 || !bulk) {
      __syncthreads();  // previous round consumed
      if (bulk) {
        if (tid == 0) {
          const uint32_t bytes = (uint32_t)(((n + 3) & ~3) * 4);
          mbar_arrive_expect_tx(&sm.bar, bytes);
          bulk_g2s(sm.u.tk.sc, srow + rb, bytes, &sm.bar);
        }
        if (!mbar_wait_bounded(&sm.bar, phase & 1u)) abort = true;
        ++phase;
      } else {
        for (int i = tid; i < n; i += kRowThreads) sm.u.tk.sc[i] = srow[rb + i];
      }
      __syncthreads();
    }
    const int base = 32 * tid;
    uint32_t bits = 0u;
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const int qq = (q + tid) & 7;
      const int i = base + 4 * qq;
      const float4 v = *reinterpret_cast<const float4 *>(&sm.u.tk.sc[i]);
      bits |= ((uint32_t)(v.x >= f1) | ((uint32_t)(v.y >= f1) << 1) |
               ((uint32_t)(v.z >= f1) << 2) | ((uint32_t)(v.w >= f1) << 3))
              << (4 * qq);
    }
    if (n < kStageScores) bits &= (base >= n) ? 0u : (base + 32 <= n ? ~0u : (1u << (n - base)) - 1u);
    uint32_t total;
    uint32_t pos = count + block_excl_scan<kRowThreads>((uint32_t)__popc(bits), sm.scratch, total);
    while (bits) {
      const int i = base + __ffs(bits) - 1;
      bits &= bits - 1u;
      const uint32_t key = score_key(sm.u.tk.sc[i]);
      const uint2 e = make_uint2(key, (uint32_t)(rb - s0 + i));
      if (pos < (uint32_t)kCandCap)
        sm.u.tk.cand[pos] = e;
      else
        spill[pos] = e;
      if (key_d1(key) == t1) atomicAdd(&sm.h2[key_d2(key)], 1u);
      ++pos;
    }
    count += total;
  }
  __syncthreads();
  auto cand_at = [&](uint32_t i) -> uint2 {
    return (i < (uint32_t)kCandCap) ? sm.u.tk.cand[i] : spill[i];
  };

  // 2. digit-2 threshold from the cluster's histograms
  cluster_threshold<D, CL, kBins2>(sm, cluster, r1, sm.thr + 2, &sm.xbar[0], &sm.xbar[1], abort);
  const uint32_t t2 = sm.thr[2], r2 = r1 - sm.thr[3];
  const bool need3 = sm.thr[4] > r2;

  // 3. digit-3 threshold, only when the boundary bucket must be split
  uint32_t t3 = 0, r3 = 0xffffffffu;
  if (need3) {
    for (int i = tid; i < kBins3; i += kRowThreads) sm.h2[i] = 0u;
    __syncthreads();
    for (uint32_t i = tid; i < count; i += kRowThreads) {
      const uint32_t k = cand_at(i).x;
      if (key_d1(k) == t1 && key_d2(k) == t2) atomicAdd(&sm.h2[key_d3(k)], 1u);
    }
    __syncthreads();
    cluster_threshold<D, CL, kBins3>(sm, cluster, r2, sm.thr + 2, &sm.xbar[2], &sm.xbar[3], abort);
    t3 = sm.thr[2];
    r3 = r2 - sm.thr[3];
  }

  // 4. classify: thread t takes the contiguous candidates [t*per, t*per +
  //    per).  Block prefixes of the (above, tie) counts give each thread
  //    the counts before it; the CTA totals go to every rank.  Ties
  //    are taken in index order while the cluster-wide tie rank stays below
  //    r3, so the ties taken before a thread are min(ties before it, r3 -
  //    this CTA's tie base): no second prefix is needed.
  const uint32_t per = (count + kRowThreads - 1) / kRowThreads;
  const uint32_t i0 = min(count, per * (uint32_t)tid), i1 = min(count, i0 + per);
  uint32_t n_above = 0, n_tie = 0;
  for (uint32_t i = i0; i < i1; ++i) {
    const uint32_t cls = cand_class(cand_at(i).x, t1, t2, t3, need3);
    n_above += (cls == 2u);
    n_tie += (cls == 1u);
  }
  uint32_t tot_above, tot_tie, above_before, tie_before;
  if (count < 65536u) {  // both counts in one prefix (16 bits each)
    uint32_t tot;
    const uint32_t pre = block_excl_scan<kRowThreads>(n_above | (n_tie << 16), sm.scratch, tot);
    above_before = pre & 0xffffu;
    tie_before = pre >> 16;
    tot_above = tot & 0xffffu;
    tot_tie = tot >> 16;
  } else {
    above_before = block_excl_scan<kRowThreads>(n_above, sm.scratch, tot_above);
    tie_before = block_excl_scan<kRowThreads>(n_tie, sm.scratch, tot_tie);
  }
  // this CTA's counts to every rank
  if (tid == 0) mbar_arrive_expect_tx(&sm.xbar[4], CL * 8);
  if (tid < CL) st_async_v2(&sm.cnt_all[c][0], tot_above, tot_tie, &sm.xbar[4], (uint32_t)tid);
  // Every tie taken (no digit-3 split, or the cluster holds exactly as many
  // keys equal to the threshold key as are still needed): the selection is
  // the above-threshold and tied candidates, in index order.
  const bool ties_all = !need3 || sm.thr[4] <= r3;
  const bool early = ties_all && tot_above + tot_tie <= (uint32_t)kSelCap;
  if ((HO || p.do_attn) && early) {
    uint32_t at = above_before + tie_before;
    for (uint32_t i = i0; i < i1; ++i) {
      const uint2 e = cand_at(i);
      if (cand_class(e.x, t1, t2, t3, need3) != 0u) sm.sel[at++] = (int32_t)(s0 + e.y);
    }
    if (tid == 0) {
      sm.sel_base = 0;
      sm.sel_count = tot_above + tot_tie;
    }
    __syncthreads();
    if constexpr (!HO) {
      return true;
    } else {
      // hand-off: the selection goes to the attention kernel now, the
      // ordered output row once every rank's counts are in
      publish_selection<CL>(sm, p, r_local, c, tot_above + tot_tie);
    }
  }
  // wait for every rank's counts
  if (!mbar_wait_cluster_bounded(&sm.xbar[4], 0)) abort = true;
  if (warp == 0) {
    const uint32_t above = (lane < CL) ? sm.cnt_all[lane][0] : 0u;
    const uint32_t ties = (lane < CL) ? sm.cnt_all[lane][1] : 0u;
    const uint32_t tb = warp_incl_scan(ties) - ties;
    const uint32_t take = (tb >= r3) ? 0u : min(ties, r3 - tb);
    const uint32_t sel = above + take;
    const uint32_t ob = warp_incl_scan(sel) - sel;
    if (lane == c) {
      sm.out_base = ob;
      sm.tie_base = tb;
      sm.sel_count = sel;
    }
  }
  __syncthreads();
  // write this thread's selected candidates in index order
  {
    const uint32_t ob = sm.out_base, tb = sm.tie_base;
    const uint32_t room = tb >= r3 ? 0u : r3 - tb;  // ties this CTA may still take
    uint32_t tie_rank = tie_before;                 // CTA-local rank of the next tie
    uint32_t at = ob + above_before + min(tie_before, room);
    for (uint32_t i = i0; i < i1; ++i) {
      const uint2 e = cand_at(i);
      const uint32_t cls = cand_class(e.x, t1, t2, t3, need3);
      bool take = cls == 2u;
      if (cls == 1u) take = tie_rank++ < room;
      if (take) {
        const int32_t n = (int32_t)(s0 + e.y);
        if (at < (uint32_t)p.topk) orow[at] = n;
        if (at - ob < (uint32_t)kSelCap) sm.sel[at - ob] = n;
        ++at;
      }
    }
  }
  if (c == CL - 1)
    for (int64_t i = K + tid; i < p.topk; i += kRowThreads) orow[i] = -1;
  if (tid == 0) sm.sel_base = sm.out_base;
  __syncthreads();
  if constexpr (HO) {  // hand-off of a selection that needed every rank's counts
    if (!early) publish_selection<CL>(sm, p, r_local, c, min(sm.sel_count, (uint32_t)kSelCap));
  }
  return false;
}

// The output indices of a selection left pending by row_topk, written by the
// warps [kAttnWarps, kWinWarp) while the others attend: wait for every
// rank's counts, the rank's output offset from a warp scan over the ranks,
// then the CTA's `sel` (all of it: every tie is taken) at that offset; the
// last rank pads [K, topk) with -1.
template <int D, int CL>
__device__ void write_row_indices(RowSmem<D> &sm, const RowParams &p, int64_t r, int c,
                                  int64_t K) {
  constexpr int kSide = (kWinWarp - kAttnWarps) * 32;
  const int st = threadIdx.x - kAttnWarps * 32, lane = threadIdx.x & 31;
  mbar_wait_cluster_bounded(&sm.xbar[4], 0);  // a wait that gives up is in the status word
  if (st < 32) {
    const uint32_t sel = (lane < CL) ? sm.cnt_all[lane][0] + sm.cnt_all[lane][1] : 0u;
    const uint32_t ob = warp_incl_scan(sel) - sel;
    if (lane == c) sm.out_base = ob;
  }
  asm volatile("bar.sync 1, %0;" ::"n"(kSide) : "memory");
  int32_t *orow = p.idx + r * (int64_t)p.topk;
  const uint32_t ob = sm.out_base, n = sm.sel_count;
  for (uint32_t i = st; i < n; i += kSide)
    if (ob + i < (uint32_t)p.topk) orow[ob + i] = sm.sel[i];
  if (c == CL - 1)
    for (int64_t i = K + st; i < p.topk; i += kSide) orow[i] = -1;
}

// This CTA's window rows [w_lo, w_lo + nwin) of row r (rows t .. t + W - 1 of
// its sequence's window slice).
template <int CL>
__device__ __forceinline__ void window_share(const RowParams &p, int64_t r, int c, int64_t &wrow0,
                                             int &nwin) {
  const int64_t b = r / p.T, t = r % p.T;
  const int w_lo = (p.W * c) / CL;
  nwin = (p.W * (c + 1)) / CL - w_lo;
  wrow0 = b * ((int64_t)p.W - 1 + p.T) + t + w_lo;
}

// Issue (without waiting) the copies of window rows [row0, row0 + nrows)
// (nrows <= 16) into the window area, missing rows zero-filled; one cp.async
// group of the calling warp.
template <int D>
__device__ __forceinline__ void issue_window_rows(ar::WarpArea<D> &wa, const uint16_t *win_k,
                                                  const uint16_t *win_v, int64_t row0, int nrows) {
  constexpr int RP = D / 8;  // 16-byte pieces per row
  const int lane = threadIdx.x & 31;
  for (int i = lane; i < ar::kChunk * RP; i += 32) {
    const int j = i / RP, u = i % RP;
    const bool ok = j < nrows;
    const int64_t row = ok ? row0 + j : row0;
    ar::cp16(&wa.s.kt[j][8 * u], win_k + row * D + 8 * u, ok ? 16u : 0u);
    ar::cp16(&wa.s.vt[j][8 * u], win_v + row * D + 8 * u, ok ? 16u : 0u);
  }
  ar::cp_commit();
}

// ---------------------------------------------------------------------------
// Attention on tensor cores (mma.sync m16n8k16, bf16 x bf16 -> fp32).
// ---------------------------------------------------------------------------
template <int D>
__device__ void load_q(RowSmem<D> &sm, const RowParams &p, int64_t r, int h0, int nh) {
  // 16-byte pieces: 16 heads x D/8 pieces
  constexpr int PPH = D / 8;
  for (int i = threadIdx.x; i < kHeads * PPH; i += kRowThreads) {
    const int h = i / PPH, u = i % PPH;
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (h < nh) v = *reinterpret_cast<const uint4 *>(p.q + (r * p.H + h0 + h) * (int64_t)D + 8 * u);
    *reinterpret_cast<uint4 *>(&sm.qb[h][8 * u]) = v;
  }
}

// Attention of one head pass: this CTA's entries (its own selection `sel`,
// else the given index slots [lo, hi)), cut into 16-key chunks that
// kAttnWarps warps take in turn, each with its own running state, while the
// last warp attends over the CTA's window rows (kWinWarp, its own area) and,
// with idx_pending, the warps between write the selection's output indices.
// The CTA's merged partial of head h then goes to the owner CTA h % CL,
// which merges the CL partials.
template <int D, int CL>
__device__ void row_attend(RowSmem<D> &sm, const RowParams &p, cg::cluster_group &cluster,
                           int64_t r, int c, int h0, int nh, bool from_sel, int64_t lo,
                           int64_t hi, int64_t sel_base, bool win_issued, bool idx_pending,
                           int64_t K) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t b = r / p.T;
  const bool has_win = (p.W * (c + 1)) / CL > (p.W * c) / CL;
  const int64_t nsel = hi - lo;
  const int64_t nch = p.N > 0 ? (nsel + ar::kChunk - 1) / ar::kChunk : 0;
  const int32_t *irow = p.idx + r * (int64_t)p.topk;
  const uint8_t *cseq = p.codes + b * p.N * (D / 2);
  const float *sseq = p.scales + b * p.N * (D / 16);
  __syncthreads();  // top-k buffers dead, query in place
  const bool win_warp = warp == kWinWarp;
  if (warp < kAttnWarps || (win_warp && has_win)) {
    // The entry warps and the window warp run one loop with one copy of the
    // chunk body (window or entry chunk chosen at run time), so an SM
    // fetches that code once.
    ar::WarpArea<D> &wa = win_warp ? sm.win : sm.u.aw[warp];
    ar::WarpState<D> st;
    ar::state_init(st);
    int64_t wrow0 = 0;
    int nwin = 0;
    if (win_warp) window_share<CL>(p, r, c, wrow0, nwin);
    auto entry_of = [&](int64_t ch) -> int32_t {  // this lane's key of entry chunk ch
      const int64_t k = ch * ar::kChunk + (lane & 15);
      if (k >= nsel) return -1;
      if (from_sel) {
        if (k < kSelCap) return sm.sel[k];
        return (sel_base + k < p.topk) ? irow[sel_base + k] : -1;
      }
      return (lo + k < p.topk) ? irow[lo + k] : -1;
    };
    int64_t ech = win_warp ? nch : warp;  // the window warp takes no entry chunk
    uint32_t mask_cur = 0u;
    if (ech < nch) mask_cur = ar::gather_entries<D>(wa, 0, entry_of(ech), p.N, cseq, sseq);
    int wj = 0;  // the window warp's next row
    int ei = 0;  // entry chunks done
#pragma unroll 1
    for (;;) {
      const bool is_win = wj < nwin;
      uint32_t mask;
      int sb = 0;
      if (is_win) {
        const int n = min(ar::kChunk, nwin - wj);
        if (wj == 0 && win_issued) {  // the first chunk's copies were issued early
          ar::cp_wait<0>();
          __syncwarp();
          mask = (1u << n) - 1u;
        } else {
          mask = ar::load_window_rows<D>(wa, p.win_k, p.win_v, wrow0 + wj, n);
        }
        wj += ar::kChunk;
      } else {
        if (ech >= nch) break;
        // entry chunk ech in buffer sb, the next one gathered meanwhile
        sb = ei & 1;
        uint32_t mask_next = 0u;
        const bool more = ech + kAttnWarps < nch;
        if (more)
          mask_next = ar::gather_entries<D>(wa, sb ^ 1, entry_of(ech + kAttnWarps), p.N, cseq, sseq);
        if (more)
          ar::cp_wait<1>();
        else
          ar::cp_wait<0>();
        __syncwarp();
        ar::convert_entries<D>(wa, sb);
        __syncwarp();
        mask = mask_cur;
        mask_cur = mask_next;
        ech += kAttnWarps;
        ++ei;
      }
      ar::attend_chunk16<D>(wa, sm.qb, st, mask, is_win, wa.s.scales[sb], p.q_scale);
      __syncwarp();
    }
    ar::store_state<D>(wa, st);
  } else if (!win_warp && idx_pending) {
    write_row_indices<D, CL>(sm, p, r, c, K);
  }
  __syncthreads();
  // per head: the max over the sources (the attention warps, then the
  // window warp) and each source's factor
  const int ns = kAttnWarps + (has_win ? 1 : 0);
  auto src_area = [&](int v) -> const ar::WarpArea<D> & {
    return v < kAttnWarps ? sm.u.aw[v] : sm.win;
  };
  for (int i = tid; i < nh * ns; i += kRowThreads) {
    const int h = i / ns, w = i % ns;
    float M = -INFINITY;
    for (int v = 0; v < ns; ++v) M = fmaxf(M, src_area(v).merge.m[h]);
    sm.mf[h][w] = M == -INFINITY ? 0.0f : exp2f(src_area(w).merge.m[h] - M);
    if (w == 0) sm.mf[h][kAttnWarps + 1] = M;
  }
  __syncthreads();
  // this CTA's partial of each head (max, sum, acc) -> inbox slot
  // (h / CL) * CL + c of the owner CTA h % CL, in 16-byte pieces: (m, l)
  // first, then the accumulator, delivered by st.async and counted on the
  // owner's partials barrier (the owner expects CL pieces per head it merges)
  constexpr int U = D / 4 + 1;
  if (tid == 0) {
    const int owned = nh > c ? (nh - 1 - c) / CL + 1 : 0;
    mbar_arrive_expect_tx(&sm.xbar[5], (uint32_t)(owned * CL * (D + 4) * 4));
  }
  for (int i = tid; i < nh * U; i += kRowThreads) {
    const int h = i / U, q = i % U;
    float4 v = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    if (q == 0) {
      for (int w = 0; w < ns; ++w) v.y = fmaf(src_area(w).merge.l[h], sm.mf[h][w], v.y);
      v.x = sm.mf[h][kAttnWarps + 1];
    } else {
      for (int w = 0; w < ns; ++w) {
        const float4 o = *reinterpret_cast<const float4 *>(&src_area(w).merge.o[h][4 * (q - 1)]);
        const float f = sm.mf[h][w];
        v.x = fmaf(o.x, f, v.x);
        v.y = fmaf(o.y, f, v.y);
        v.z = fmaf(o.z, f, v.z);
        v.w = fmaf(o.w, f, v.w);
      }
    }
    st_async_v4(&sm.inbox[(h / CL) * CL + c][4 * q],
                make_uint4(__float_as_uint(v.x), __float_as_uint(v.y), __float_as_uint(v.z),
                           __float_as_uint(v.w)),
                &sm.xbar[5], (uint32_t)(h % CL));
  }
  // the partials of the heads this CTA merges (CL sources each); a wait
  // that gives up is recorded in the status word
  mbar_wait_cluster_bounded(&sm.xbar[5], (uint32_t)(h0 / kHeads) & 1u);
  // merge of head h = c + k*CL (k < kHeads / CL) from its CL partials in
  // slots [k*CL, k*CL + CL): warp k finds the max, the factors and the sum,
  // then one thread per (head, dim) sums the weighted partials
  constexpr int KH = kHeads / CL;
  if (warp < KH) {
    const int h = c + warp * CL;
    const float *slot = &sm.inbox[warp * CL][0];
    const float m = (lane < CL) ? slot[lane * (D + 4)] : -INFINITY;
    const float l = (lane < CL) ? slot[lane * (D + 4) + 1] : 0.0f;
    const float M = warp_max(l > 0.0f ? m : -INFINITY);
    const float f = (M != -INFINITY && l > 0.0f) ? exp2f(m - M) : 0.0f;
    const float L = warp_sum(l * f);
    if (lane < CL) sm.fac[warp * CL + lane] = f;
    if (lane == 0) {
      sm.mrg_m[warp] = M;
      sm.mrg_l[warp] = L;
      if (p.lse && h < nh)
        p.lse[r * p.H + h0 + h] =
            M == -INFINITY ? -INFINITY : (M + log2f(L)) * 0.69314718055994530942f;
    }
  }
  __syncthreads();
  for (int i = tid; i < KH * D; i += kRowThreads) {
    const int k = i / D, e = i % D, h = c + k * CL;
    if (h >= nh) continue;
    float *op = p.out + (r * p.H + h0 + h) * (int64_t)D;
    if (sm.mrg_m[k] == -INFINITY) {
      op[e] = 0.0f;
      continue;
    }
    float a = 0.0f;
#pragma unroll
    for (int j = 0; j < CL; ++j) {
      const float fj = sm.fac[k * CL + j];
      if (fj != 0.0f) a = fmaf(sm.inbox[k * CL + j][4 + e], fj, a);
    }
    op[e] = a * (1.0f / sm.mrg_l[k]);
  }
}

// HO: the top-k hands each CTA's selection to an attention kernel launched
// after this one (p.lists, no attention here); its code is compiled only
// into those instances.
template <int D, int CL, bool HO>
__global__ void __launch_bounds__(kRowThreads, 1) row_cluster_kernel(const RowParams p) {
  extern __shared__ __align__(128) unsigned char row_smem_raw[];
  RowSmem<D> &sm = *reinterpret_cast<RowSmem<D> *>(row_smem_raw);
  cg::cluster_group cluster = cg::this_cluster();
  // with a hand-off, the attention kernel launched after this one with
  // programmatic dependent launch may start now; it waits for each list's
  // ready flag itself
  if constexpr (HO) pdl_allow_dependents();
  const int tid = threadIdx.x;
  const int c = (int)cluster.block_rank();
  const int64_t r_local = blockIdx.x / CL, r = p.row0 + r_local;
  const int64_t t = r % p.T;
  const int64_t V = row_visible(p.N, p.n_prior, p.ratio, t);
  const int64_t K = V < p.topk ? V : p.topk;
  const bool bulk =
      (p.score_stride % 4 == 0) && ((reinterpret_cast<uintptr_t>(p.scores) & 15) == 0);
  const int64_t s0 = (c == 0) ? 0 : (((V * c) / CL) & ~int64_t(15));
  const int64_t s1 = (c == CL - 1) ? V : (((V * (c + 1)) / CL) & ~int64_t(15));
  const bool topk_here = p.do_topk && K > 0;

  // Every CTA of the cluster must be running, with its barriers initialised,
  // before any of them writes into another's shared memory: arrive once the
  // barriers are set up, wait before the first such write.
  if (tid == 0) {
    mbar_init(&sm.bar, 1);
    for (int k = 0; k < 6; ++k) mbar_init(&sm.xbar[k], 1);
    fence_barrier_init();
  }
  __syncthreads();
  asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
  // Prologue, independent of the scan that produced the scores: the query.
  // With programmatic dependent launch this overlaps the scan's tail.
  for (int i = tid; i < kBins2; i += kRowThreads) sm.h2[i] = 0u;
  if (p.do_attn) load_q<D>(sm, p, r, 0, min(kHeads, p.H));
  // The window rows do not depend on the selection: the window warp issues
  // the copies of its first chunk now and waits for them when it attends.
  bool win_issued = false;
  if (p.do_attn && p.H > 0 && (tid >> 5) == kWinWarp) {
    int64_t wrow0;
    int nwin;
    window_share<CL>(p, r, c, wrow0, nwin);
    if (nwin > 0) {
      issue_window_rows<D>(sm.win, p.win_k, p.win_v, wrow0, min(ar::kChunk, nwin));
      win_issued = true;
    }
  }
  asm volatile("barrier.cluster.wait.aligned;" ::: "memory");
  pdl_wait_primary();  // the scores and histograms are complete from here on
  if (topk_here && tid == 0) {
    const int n0 = (int)min64(kStageScores, s1 - s0);
    uint32_t bytes = kBins1 * 4;
    if (bulk && n0 > 0) bytes += (uint32_t)(((n0 + 3) & ~3) * 4);
    mbar_arrive_expect_tx(&sm.bar, bytes);
    bulk_g2s(sm.h1, p.hist1 + r_local * kHistStride, kBins1 * 4, &sm.bar);
    if (bulk && n0 > 0)
      bulk_g2s(sm.u.tk.sc, p.scores + r_local * p.score_stride + s0,
               (uint32_t)(((n0 + 3) & ~3) * 4), &sm.bar);
  }

  bool abort = false, idx_pending = false;
  uint32_t phases = 0;
  if (p.do_topk) {
    if (topk_here) {
      idx_pending =
          row_topk<D, CL, HO>(sm, p, cluster, r_local, r, K, bulk, s0, s1, abort, phases);
    } else {
      if (c == 0) {
        int32_t *orow = p.idx + r * (int64_t)p.topk;
        for (int i = tid; i < p.topk; i += kRowThreads) orow[i] = -1;
      }
      if (tid == 0) {
        sm.sel_base = 0;
        sm.sel_count = 0;
      }
      if constexpr (HO) publish_selection<CL>(sm, p, r_local, c, 0u);
    }
    // Attention reads this CTA's own selection from shared memory, so no
    // cluster barrier is needed between top-k and attention.
  }
  if (p.do_attn) {
    int64_t lo, hi;
    if (p.do_topk) {
      lo = 0;
      hi = sm.sel_count;
    } else {
      lo = ((int64_t)p.topk * c) / CL;
      hi = ((int64_t)p.topk * (c + 1)) / CL;
    }
    const int64_t sel_base = p.do_topk ? (int64_t)sm.sel_base : 0;
    for (int h0 = 0; h0 < p.H; h0 += kHeads) {
      const int nh = min(kHeads, p.H - h0);
      if (h0 > 0) {
        cluster.sync();  // the previous merge read this CTA's inbox
        __syncthreads();
        load_q<D>(sm, p, r, h0, nh);
      }
      row_attend<D, CL>(sm, p, cluster, r, c, h0, nh, p.do_topk != 0, lo, hi, sel_base,
                        win_issued && h0 == 0, idx_pending && h0 == 0, K);
    }
  }
  if (abort && tid == 0 && phases > 0)  // let a late bulk copy land before exit
    mbar_wait_bounded(&sm.bar, (phases - 1) & 1u);
}

}  // namespace csa2
