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
// of the row's entries.  Cluster barriers order the phases; histograms,
// counts and softmax partials move through distributed shared memory.
//
// Top-k: exact radix selection on an order-preserving 32-bit key of the
// score, digits of 11, 11 and 10 bits.  The scan kernel has histogrammed
// digit 1 of every visible score.  Each CTA stages that histogram and its
// score slice in shared memory with bulk copies, then
//   1. finds the digit-1 threshold t1 (largest digit whose suffix count
//      reaches k) and lists the elements of its slice with digit 1 >= t1,
//      in index order (each warp walks a contiguous segment: a count pass,
//      one prefix over warps, a write pass), histogramming digit 2 of the
//      elements exactly at t1;
//   2. reduces the cluster's digit-2 histograms (CTA c sums bin slice c of
//      every rank; every CTA then locates the threshold slice from the
//      slice totals and reads only that slice) -> t2;
//   3. only when the boundary bucket (t1, t2) holds more elements than still
//      needed: the same for digit 3 -> t3;
//   4. classifies the candidates as above the threshold key or equal to
//      it.  Equal keys are equal scores; they are taken in index order
//      (lower index first) up to the count still needed.  Prefix sums over
//      ranks and warps give every warp its offset in the output row, so the
//      indices come out ascending.
//
// Attention: each CTA attends over an even share of the window rows (done
// first, while the top-k inputs are still arriving) and over the entries it
// selected itself (their raw FP4 rows gathered in batches of async copies),
// in chunks of 64 keys with an online softmax in base 2.  A chunk is two
// small tensor-core products (mma.sync m16n8k16, bf16 in, fp32 out; 16
// heads is exactly the M = 16 of that shape):
//   logits  S[h, n] = sum_g s[n, g] * sum_{i in g} q[h, i] * e2m1[n, i]
//           one product per 16-element scale group g; E2M1 values and the
//           bf16 query are exact in bf16, so every product is exact and the
//           group scale is applied in fp32 afterwards;
//   values  O[h, d] += sum_n (P[h, n] * s[n, g(d)]) * e2m1[n, d]
//           with the fp32 weight P*s split into a bf16 pair hi + lo (two
//           products), so the weight keeps ~16 bits.
// Window rows use the same path with scale 1 (bf16 keys and values).  Each
// CTA pushes its partial (max, sum, acc) of head h into the shared memory of
// the CTA that owns h (h mod CL); after one cluster barrier the owners merge
// locally by log-sum-exp.  Which CTA handles which key does not change the
// result, so no entry is moved between CTAs.  With given indices (attention
// only), CTA c takes an even share of the selected slots.
#pragma once
#include <cooperative_groups.h>

#include "common.cuh"
#include "pack.cuh"

namespace csa2 {

namespace cg = cooperative_groups;

constexpr int kRowThreads = 512;
constexpr int kRowWarps = kRowThreads / 32;
constexpr int kStageScores = 16384;  // scores staged in shared memory per round
constexpr int kCandCap = 4096;       // candidates kept in shared memory
constexpr int kSelCap = 4096;        // selected indices kept in shared memory
constexpr int kRawCap = 512;         // entries gathered per batch
constexpr int kChunkKeys = 64;
constexpr int kHeads = 16;           // heads per pass (the MMA's M)

struct RowParams {
  // top-k
  const float *scores;      // [rows_local, score_stride] (this launch's rows)
  int64_t score_stride;
  const uint32_t *hist1;    // [rows_local, kBins1]
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
};

template <int D>
struct RowSmem {
  static constexpr int G = D / 16;  // scale groups per entry
  union {
    float sc[kStageScores];  // staged score slice (top-k)
    struct {                 // raw gathered entries (attention)
      uint8_t codes[kRawCap][D / 2];
      float scales[kRawCap][D / 16];
    } raw;
  } st;
  uint32_t h1[kBins1];          // staged digit-1 histogram
  uint32_t h2[kBins2];          // own digit-2 (then digit-3) histogram
  uint32_t hin[kBins2];         // bin slice this CTA owns, one row per source rank (pushed)
  uint32_t full[kBins2];        // cluster-wide histogram (reduced slices pushed by owners)
  uint32_t cnt_all[32][2];      // every rank's (above, tie) counts (pushed)
  uint2 cand[kCandCap];         // candidates (key, index - slice start), index order
  int32_t sel[kSelCap];         // this CTA's selected indices, ascending
  int32_t raw_idx[kRawCap];     // entries of the gathered batch
  uint32_t wa[kRowWarps], wb[kRowWarps], wc[kRowWarps], wd[kRowWarps];
  uint32_t masks[kRowWarps][kStageScores / kRowWarps / 32];  // per-warp ballots of a round
  // attention
  uint16_t kb[kChunkKeys][D + 8];   // keys, row-major bf16 (+8: conflict-free B loads)
  uint16_t vt[D][kChunkKeys + 8];   // values, transposed bf16
  float ks[kChunkKeys][G];          // per-key group scales (1 for window rows)
  float s[kHeads][kChunkKeys + 4];  // logits, then probabilities
  float corr[kHeads];
  uint16_t qb[kHeads][D + 8];       // query, bf16
  float inbox[kHeads][D + 2];       // pushed partials (m, l, acc) of the heads this CTA merges
  int valid[kChunkKeys];
  uint32_t scratch[40];
  uint32_t thr[8];
  uint32_t cnt[4];  // [1] above-threshold, [2] equal-to-threshold, [3] reduced-slice total
  uint32_t sel_base, sel_count, out_base, tie_base;
  uint64_t bar;
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
// count strictly above it and the count of bin t, in out[0..2].  Push-based:
// every CTA stores bin slice j of its histogram into CTA j's `hin`; after a
// barrier CTA j reduces its slice and stores it into every CTA's `full`;
// after a second barrier each CTA finds the threshold locally.  Callers make
// sure no CTA still reads its `hin` or `full` from an earlier use.
template <int D, int CL, int NB>
__device__ void cluster_threshold(RowSmem<D> &sm, cg::cluster_group &cluster, uint32_t need,
                                  uint32_t *out) {
  constexpr int BPC = NB / CL;  // bins owned by each CTA
  const int tid = threadIdx.x;
  const int c = (int)cluster.block_rank();
  for (int i = tid; i < NB; i += kRowThreads) {
    const int owner = i / BPC;
    cluster.map_shared_rank(&sm.hin[0], owner)[c * BPC + (i - owner * BPC)] = sm.h2[i];
  }
  cluster.sync();
  for (int b = tid; b < BPC; b += kRowThreads) {
    uint32_t s = 0;
#pragma unroll
    for (int j = 0; j < CL; ++j) s += sm.hin[j * BPC + b];
#pragma unroll
    for (int j = 0; j < CL; ++j) cluster.map_shared_rank(&sm.full[0], j)[c * BPC + b] = s;
  }
  cluster.sync();
  radix_threshold<kRowThreads, NB>(sm.full, need, sm.scratch, out);
  if (tid == 0) out[2] = sm.full[out[0]];
  __syncthreads();
}

// Exclusive prefix of one value per warp (sm.* arrays of kRowWarps), done by
// warp 0; returns nothing, writes the prefix into `dst` and the total into
// dst_total.  Caller synchronises before and after.
__device__ __forceinline__ void warp0_prefix16(const uint32_t *src, uint32_t *dst,
                                               uint32_t *dst_total) {
  const int lane = threadIdx.x & 31;
  const uint32_t v = (lane < kRowWarps) ? src[lane] : 0u;
  const uint32_t incl = warp_incl_scan(v);
  if (lane < kRowWarps) dst[lane] = incl - v;
  if (lane == 31) *dst_total = incl;
}

template <int D, int CL>
__device__ void row_topk(RowSmem<D> &sm, const RowParams &p, cg::cluster_group &cluster,
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

  // 1. candidate list in index order: warp w owns segment [seg0, seg1) of
  //    each staged round; a counting pass, one prefix over warps, a ballot
  //    pass that writes the candidates.
  uint32_t count = 0;
  for (int64_t rb = s0; rb < s1; rb += kStageScores) {
    const int n = (int)min64(kStageScores, s1 - rb);
    if (rb != s0 || !bulk) {
      __syncthreads();  // previous round consumed
      if (bulk) {
        if (tid == 0) {
          const uint32_t bytes = (uint32_t)(((n + 3) & ~3) * 4);
          mbar_arrive_expect_tx(&sm.bar, bytes);
          bulk_g2s(sm.st.sc, srow + rb, bytes, &sm.bar);
        }
        if (!mbar_wait_bounded(&sm.bar, phase & 1u)) abort = true;
        ++phase;
      } else {
        for (int i = tid; i < n; i += kRowThreads) sm.st.sc[i] = srow[rb + i];
      }
      __syncthreads();
    }
    // one ballot per 32 elements of the warp's segment, kept in shared memory
    const int seg0 = (n * warp) / kRowWarps, seg1 = (n * (warp + 1)) / kRowWarps;
    constexpr int STEPS = kStageScores / kRowWarps / 32;
    uint32_t mine = 0;
#pragma unroll 8
    for (int j = 0; j < STEPS; ++j) {
      const int i = seg0 + 32 * j + lane;
      const bool in = (i < seg1) && key_d1(score_key(sm.st.sc[i])) >= t1;
      const uint32_t bal = __ballot_sync(0xffffffffu, in);
      if (lane == (j & 31)) sm.masks[warp][j] = bal;
      mine += __popc(bal);
    }
    if (lane == 0) sm.wa[warp] = mine;
    __syncthreads();
    if (warp == 0) warp0_prefix16(sm.wa, sm.wb, &sm.scratch[0]);
    __syncthreads();
    // write pass: only the steps that hold candidates
    uint32_t pos = count + sm.wb[warp];
    for (int j = 0; j < STEPS; ++j) {
      const uint32_t bal = sm.masks[warp][j];
      if (bal == 0u) continue;  // warp-uniform
      if ((bal >> lane) & 1u) {
        const int i = seg0 + 32 * j + lane;
        const uint32_t key = score_key(sm.st.sc[i]);
        const uint32_t at = pos + __popc(bal & lt);
        const uint2 e = make_uint2(key, (uint32_t)(rb - s0 + i));
        if (at < (uint32_t)kCandCap)
          sm.cand[at] = e;
        else
          spill[at] = e;
      }
      pos += __popc(bal);
    }
    count += sm.scratch[0];
  }
  __syncthreads();
  auto cand_at = [&](uint32_t i) -> uint2 {
    return (i < (uint32_t)kCandCap) ? sm.cand[i] : spill[i];
  };
  // digit-2 histogram of the candidates exactly at t1 (few atomics)
  for (uint32_t i = tid; i < count; i += kRowThreads) {
    const uint32_t k = cand_at(i).x;
    if (key_d1(k) == t1) atomicAdd(&sm.h2[key_d2(k)], 1u);
  }
  __syncthreads();

  // 2. digit-2 threshold from the cluster's histograms
  cluster_threshold<D, CL, kBins2>(sm, cluster, r1, sm.thr + 2);
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
    cluster_threshold<D, CL, kBins3>(sm, cluster, r2, sm.thr + 2);
    t3 = sm.thr[2];
    r3 = r2 - sm.thr[3];
  }

  // 4. classify: warp w takes candidates [count*w/16, count*(w+1)/16)
  const uint32_t c0 = (uint32_t)(((uint64_t)count * warp) / kRowWarps);
  const uint32_t c1 = (uint32_t)(((uint64_t)count * (warp + 1)) / kRowWarps);
  uint32_t n_above = 0, n_tie = 0;
  for (uint32_t i = c0 + lane; i < c1; i += 32) {
    const uint32_t cls = cand_class(cand_at(i).x, t1, t2, t3, need3);
    n_above += (cls == 2u);
    n_tie += (cls == 1u);
  }
  n_above = __reduce_add_sync(0xffffffffu, n_above);
  n_tie = __reduce_add_sync(0xffffffffu, n_tie);
  if (lane == 0) {
    sm.wa[warp] = n_above;
    sm.wb[warp] = n_tie;
  }
  __syncthreads();
  if (warp == 0) {
    uint32_t tot_tie;
    warp0_prefix16(sm.wb, sm.wd, &tot_tie);  // tie prefix per warp
    const uint32_t v = (lane < kRowWarps) ? sm.wa[lane] : 0u;
    const uint32_t tot_above = __reduce_add_sync(0xffffffffu, v);
    tot_tie = __shfl_sync(0xffffffffu, tot_tie, 31);
    // push this CTA's counts to every rank
    if (lane < CL) {
      uint32_t *dst = cluster.map_shared_rank(&sm.cnt_all[0][0], lane);
      dst[2 * c] = tot_above;
      dst[2 * c + 1] = tot_tie;
    }
  }
  cluster.sync();  // every rank's (above, tie) counts are in cnt_all
  if (warp == 0) {
    const uint32_t above = (lane < CL) ? sm.cnt_all[lane][0] : 0u;
    const uint32_t ties = (lane < CL) ? sm.cnt_all[lane][1] : 0u;
    const uint32_t tb = warp_incl_scan(ties) - ties;
    const uint32_t take = (tb >= r3) ? 0u : min(ties, r3 - tb);
    const uint32_t sel = above + take;
    const uint32_t ob = warp_incl_scan(sel) - sel;
    const uint32_t ob_c = __shfl_sync(0xffffffffu, ob, c);
    const uint32_t tb_c = __shfl_sync(0xffffffffu, tb, c);
    // per-warp offsets inside this CTA: warp w selects its above-class
    // candidates plus its ties whose CTA-wide rank stays below r3 - tb_c
    uint32_t wsel = 0;
    if (lane < kRowWarps) {
      const uint32_t tie_before = tb_c + sm.wd[lane];
      const uint32_t wt = sm.wb[lane];
      const uint32_t wtake = (tie_before >= r3) ? 0u : min(wt, r3 - tie_before);
      wsel = sm.wa[lane] + wtake;
    }
    const uint32_t wo = warp_incl_scan(wsel) - wsel;
    if (lane < kRowWarps) sm.wc[lane] = ob_c + wo;  // output position of that warp's first
    if (lane == 0) {
      sm.out_base = ob_c;
      sm.tie_base = tb_c;
    }
    const uint32_t total_sel = __shfl_sync(0xffffffffu, wo + wsel, kRowWarps - 1);
    if (lane == 0) sm.sel_count = total_sel;
  }
  __syncthreads();
  // write: warp w walks its candidates in order again
  {
    uint32_t pos = sm.wc[warp];                     // output row position
    uint32_t tie_rank = sm.tie_base + sm.wd[warp];  // CTA-wide tie rank of the next tie
    const uint32_t ob = sm.out_base;
    for (uint32_t i0 = c0; i0 < c1; i0 += 32) {
      const uint32_t i = i0 + lane;
      uint2 e = make_uint2(0u, 0u);
      uint32_t cls = 0u;
      if (i < c1) {
        e = cand_at(i);
        cls = cand_class(e.x, t1, t2, t3, need3);
      }
      const uint32_t tbal = __ballot_sync(0xffffffffu, cls == 1u);
      const bool take = (cls == 2u) || (cls == 1u && tie_rank + __popc(tbal & lt) < r3);
      const uint32_t sb = __ballot_sync(0xffffffffu, take);
      if (take) {
        const uint32_t at = pos + __popc(sb & lt);
        const int32_t n = (int32_t)(s0 + e.y);
        if (at < (uint32_t)p.topk) orow[at] = n;
        if (at - ob < (uint32_t)kSelCap) sm.sel[at - ob] = n;
      }
      pos += __popc(sb);
      tie_rank += __popc(tbal);
    }
  }
  if (c == CL - 1)
    for (int64_t i = K + tid; i < p.topk; i += kRowThreads) orow[i] = -1;
  if (tid == 0) sm.sel_base = sm.out_base;
  __syncthreads();
}

// ---------------------------------------------------------------------------
// Attention on tensor cores (mma.sync m16n8k16, bf16 x bf16 -> fp32).
// ---------------------------------------------------------------------------
__device__ __forceinline__ void mma_bf16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t lds32(const uint16_t *p) {
  return *reinterpret_cast<const uint32_t *>(p);
}

// fp32 pair -> (hi, lo) packed bf16 pairs with x ~= hi + lo.
__device__ __forceinline__ void split_bf16x2(float x0, float x1, uint32_t &hi, uint32_t &lo) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(x0, x1);
  const float2 hf = __bfloat1622float2(h);
  const __nv_bfloat162 l = __floats2bfloat162_rn(x0 - hf.x, x1 - hf.y);
  hi = *reinterpret_cast<const uint32_t *>(&h);
  lo = *reinterpret_cast<const uint32_t *>(&l);
}

// 8 E2M1 codes (one 32-bit word, element 2i in the low nibble of byte i) ->
// 8 exact bf16 values (as 4 packed pairs, lower element in the low half).
__device__ __forceinline__ void e2m1x8_to_bf16(uint32_t word, uint32_t (&o)[4]) {
  uint32_t h[4];
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "mov.b32 {b0, b1, b2, b3}, %4;\n\t"
      "cvt.rn.f16x2.e2m1x2 %0, b0;\n\t"
      "cvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
      "cvt.rn.f16x2.e2m1x2 %2, b2;\n\t"
      "cvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
      : "=r"(h[0]), "=r"(h[1]), "=r"(h[2]), "=r"(h[3])
      : "r"(word));
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&h[i]));
    const __nv_bfloat162 b = __floats2bfloat162_rn(f.x, f.y);  // exact: <= 3 significant bits
    o[i] = *reinterpret_cast<const uint32_t *>(&b);
  }
}

__device__ __forceinline__ void cp_async16(void *smem_dst, const void *gmem_src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(smem_dst)),
               "l"(gmem_src)
               : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
}

// Write one key of a chunk into shared memory: kv (keys) and vv (values) are
// EP/2 packed bf16 pairs for elements [part*EP, part*EP + EP) of key j.
template <int D>
__device__ __forceinline__ void store_key_part(RowSmem<D> &sm, int j, int part,
                                               const uint32_t *kv, const uint32_t *vv) {
  constexpr int EP = D / 8;
#pragma unroll
  for (int u = 0; u < EP / 8; ++u)
    *reinterpret_cast<uint4 *>(&sm.kb[j][part * EP + 8 * u]) =
        make_uint4(kv[4 * u], kv[4 * u + 1], kv[4 * u + 2], kv[4 * u + 3]);
#pragma unroll
  for (int i = 0; i < EP / 2; ++i) {
    sm.vt[part * EP + 2 * i][j] = (uint16_t)(vv[i] & 0xffffu);
    sm.vt[part * EP + 2 * i + 1][j] = (uint16_t)(vv[i] >> 16);
  }
}

// Window rows [row0, row0 + nkeys) -> chunk buffers (bf16 as stored, scale 1).
template <int D>
__device__ void load_window_chunk(RowSmem<D> &sm, const RowParams &p, int64_t row0, int nkeys) {
  constexpr int EP = D / 8;  // 512 threads = 64 keys x 8 parts
  const int tid = threadIdx.x, j = tid % kChunkKeys, part = tid / kChunkKeys;
  uint32_t kv[EP / 2], vv[EP / 2];
  const bool ok = j < nkeys;
  if (ok) {
    const uint4 *kp = reinterpret_cast<const uint4 *>(p.win_k + (row0 + j) * D + part * EP);
    const uint4 *vp = reinterpret_cast<const uint4 *>(p.win_v + (row0 + j) * D + part * EP);
#pragma unroll
    for (int u = 0; u < EP / 8; ++u) {
      const uint4 k4 = kp[u], v4 = vp[u];
      kv[4 * u] = k4.x, kv[4 * u + 1] = k4.y, kv[4 * u + 2] = k4.z, kv[4 * u + 3] = k4.w;
      vv[4 * u] = v4.x, vv[4 * u + 1] = v4.y, vv[4 * u + 2] = v4.z, vv[4 * u + 3] = v4.w;
    }
  } else {
#pragma unroll
    for (int i = 0; i < EP / 2; ++i) kv[i] = vv[i] = 0u;
  }
  if (EP == 16 || (part & 1) == 0) sm.ks[j][(part * EP) / 16] = 1.0f;
  if (part == 0) sm.valid[j] = ok;
  store_key_part<D>(sm, j, part, kv, vv);
}

// Gathered entries [b0, b0 + nkeys) of the raw batch -> chunk buffers
// (E2M1 values as exact bf16, group scales kept apart).
template <int D>
__device__ void load_entry_chunk(RowSmem<D> &sm, const RowParams &p, int b0, int nkeys) {
  constexpr int EP = D / 8;
  const int tid = threadIdx.x, j = tid % kChunkKeys, part = tid / kChunkKeys;
  uint32_t kv[EP / 2];
  const int slot = b0 + j;
  const int32_t n = (j < nkeys) ? sm.raw_idx[slot] : -1;
  const bool ok = n >= 0 && (int64_t)n < p.N;
  float s = 0.0f;
  if (ok) {
    s = sm.st.raw.scales[slot][(part * EP) / 16];
    if constexpr (EP == 16) {
      const uint2 cw = *reinterpret_cast<const uint2 *>(&sm.st.raw.codes[slot][part * 8]);
      uint32_t o0[4], o1[4];
      e2m1x8_to_bf16(cw.x, o0);
      e2m1x8_to_bf16(cw.y, o1);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        kv[i] = o0[i];
        kv[4 + i] = o1[i];
      }
    } else {
      const uint32_t cw = *reinterpret_cast<const uint32_t *>(&sm.st.raw.codes[slot][part * 4]);
      uint32_t o0[4];
      e2m1x8_to_bf16(cw, o0);
#pragma unroll
      for (int i = 0; i < 4; ++i) kv[i] = o0[i];
    }
  } else {
#pragma unroll
    for (int i = 0; i < EP / 2; ++i) kv[i] = 0u;
  }
  if (EP == 16 || (part & 1) == 0) sm.ks[j][(part * EP) / 16] = s;
  if (part == 0) sm.valid[j] = ok;
  store_key_part<D>(sm, j, part, kv, kv);
}

// One head pass's running softmax state (per thread: output fragment of the
// PV warps, max/sum of the head owned by this warp).
struct AttnState {
  float o[4];
  float m, l;
};

// Logits, online softmax and PV update of the chunk now in the buffers.
template <int D>
__device__ void attend_chunk(RowSmem<D> &sm, const RowParams &p, AttnState &st, int nh) {
  constexpr int G = D / 16;
  constexpr int PV_WARPS = D / 8;  // warp w owns output dims [8w, 8w + 8)
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int gid = lane >> 2, tig = lane & 3;
  (void)tid;
  // logits: warp w < 8 owns keys [8w, 8w + 8)
  if (warp < kChunkKeys / 8) {
    float sacc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
    const int key0 = 8 * warp + 2 * tig;  // this thread's two key columns
#pragma unroll
    for (int g = 0; g < G; ++g) {
      float d4[4] = {0.0f, 0.0f, 0.0f, 0.0f};
      const uint32_t a0 = lds32(&sm.qb[gid][16 * g + 2 * tig]);
      const uint32_t a1 = lds32(&sm.qb[gid + 8][16 * g + 2 * tig]);
      const uint32_t a2 = lds32(&sm.qb[gid][16 * g + 8 + 2 * tig]);
      const uint32_t a3 = lds32(&sm.qb[gid + 8][16 * g + 8 + 2 * tig]);
      const uint32_t b0 = lds32(&sm.kb[8 * warp + gid][16 * g + 2 * tig]);
      const uint32_t b1 = lds32(&sm.kb[8 * warp + gid][16 * g + 8 + 2 * tig]);
      mma_bf16(d4, a0, a1, a2, a3, b0, b1);
      const float s0 = sm.ks[key0][g], s1 = sm.ks[key0 + 1][g];
      sacc[0] = fmaf(d4[0], s0, sacc[0]);
      sacc[1] = fmaf(d4[1], s1, sacc[1]);
      sacc[2] = fmaf(d4[2], s0, sacc[2]);
      sacc[3] = fmaf(d4[3], s1, sacc[3]);
    }
    const bool v0 = sm.valid[key0], v1 = sm.valid[key0 + 1];
    sm.s[gid][key0] = v0 ? sacc[0] * p.q_scale : -INFINITY;
    sm.s[gid][key0 + 1] = v1 ? sacc[1] * p.q_scale : -INFINITY;
    sm.s[gid + 8][key0] = v0 ? sacc[2] * p.q_scale : -INFINITY;
    sm.s[gid + 8][key0 + 1] = v1 ? sacc[3] * p.q_scale : -INFINITY;
  }
  __syncthreads();
  // online softmax: warp h owns head h (padding heads get zero weights)
  {
    const int h = warp;
    const float z0 = sm.s[h][lane], z1 = sm.s[h][lane + 32];
    const float new_m = fmaxf(st.m, warp_max(fmaxf(z0, z1)));
    float p0 = 0.0f, p1 = 0.0f, corr = 1.0f;
    if (h < nh && new_m != -INFINITY) {
      p0 = exp2f(z0 - new_m);
      p1 = exp2f(z1 - new_m);
      corr = exp2f(st.m - new_m);  // 0 when the running max is -inf
      st.l = st.l * corr + warp_sum(p0 + p1);
      st.m = new_m;
    }
    sm.s[h][lane] = p0;
    sm.s[h][lane + 32] = p1;
    if (lane == 0) sm.corr[h] = corr;
  }
  __syncthreads();
  // values: warp w < D/8 owns output dims [8w, 8w + 8) in scale group w/2
  if (warp < PV_WARPS) {
    const int g = warp >> 1;
    const float c0 = sm.corr[gid], c1 = sm.corr[gid + 8];
    st.o[0] *= c0;
    st.o[1] *= c0;
    st.o[2] *= c1;
    st.o[3] *= c1;
#pragma unroll
    for (int kk = 0; kk < kChunkKeys / 16; ++kk) {
      const int k0 = 16 * kk + 2 * tig, k1 = k0 + 8;
      const float sa = sm.ks[k0][g], sb = sm.ks[k0 + 1][g];
      const float sc = sm.ks[k1][g], sd = sm.ks[k1 + 1][g];
      uint32_t ah[4], al[4];
      split_bf16x2(sm.s[gid][k0] * sa, sm.s[gid][k0 + 1] * sb, ah[0], al[0]);
      split_bf16x2(sm.s[gid + 8][k0] * sa, sm.s[gid + 8][k0 + 1] * sb, ah[1], al[1]);
      split_bf16x2(sm.s[gid][k1] * sc, sm.s[gid][k1 + 1] * sd, ah[2], al[2]);
      split_bf16x2(sm.s[gid + 8][k1] * sc, sm.s[gid + 8][k1 + 1] * sd, ah[3], al[3]);
      const uint32_t b0 = lds32(&sm.vt[8 * warp + gid][k0]);
      const uint32_t b1 = lds32(&sm.vt[8 * warp + gid][k1]);
      mma_bf16(st.o, ah[0], ah[1], ah[2], ah[3], b0, b1);
      mma_bf16(st.o, al[0], al[1], al[2], al[3], b0, b1);
    }
  }
}

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

// Window rows of this CTA for one head pass.
template <int D, int CL>
__device__ void attend_window(RowSmem<D> &sm, const RowParams &p, AttnState &st, int64_t r,
                              int c, int nh) {
  const int64_t b = r / p.T, t = r % p.T;
  const int w_lo = (p.W * c) / CL, w_hi = (p.W * (c + 1)) / CL;
  const int64_t row0 = b * ((int64_t)p.W - 1 + p.T) + t + w_lo;
  for (int k0 = 0; k0 < w_hi - w_lo; k0 += kChunkKeys) {
    __syncthreads();  // chunk buffers free (and q written)
    load_window_chunk<D>(sm, p, row0 + k0, min(kChunkKeys, w_hi - w_lo - k0));
    __syncthreads();
    attend_chunk<D>(sm, p, st, nh);
  }
}

// Selected entries [lo, hi) of this CTA's list for one head pass: gathered
// in batches of kRawCap with async copies, then attended chunk by chunk.
// `from_sel`: indices come from sm.sel (own selection, beyond kSelCap from
// the output row) or, when false, straight from the given index row.
template <int D>
__device__ void attend_selected(RowSmem<D> &sm, const RowParams &p, AttnState &st, int64_t r,
                                int64_t lo, int64_t hi, bool from_sel, int64_t sel_base,
                                int nh) {
  const int tid = threadIdx.x;
  const int64_t b = r / p.T;
  const int32_t *irow = p.idx + r * (int64_t)p.topk;
  constexpr int CCH = D / 32;                  // 16-byte code chunks per entry
  constexpr int SCH = (D / 16 * 4 + 15) / 16;  // 16-byte scale chunks per entry
  for (int64_t bb = lo; bb < hi; bb += kRawCap) {
    const int nb = (int)min64(kRawCap, hi - bb);
    __syncthreads();  // raw buffers free
    for (int i = tid; i < nb; i += kRowThreads) {
      const int64_t k = bb + i;  // position in this CTA's list / the index row
      int32_t n;
      if (from_sel)
        n = (k - lo < kSelCap) ? sm.sel[k - lo] : irow[sel_base + k - lo];
      else
        n = irow[k];
      const bool ok = n >= 0 && (int64_t)n < p.N;
      if (n >= 0 && !ok) raise_status(kStatusBadIndex);
      sm.raw_idx[i] = ok ? n : -1;
      if (ok) {
        const int64_t row = b * p.N + n;
        const uint8_t *cp = p.codes + row * (D / 2);
        const float *sp = p.scales + row * (D / 16);
#pragma unroll
        for (int u = 0; u < CCH; ++u) cp_async16(&sm.st.raw.codes[i][16 * u], cp + 16 * u);
#pragma unroll
        for (int u = 0; u < SCH; ++u) cp_async16(&sm.st.raw.scales[i][4 * u], sp + 4 * u);
      }
    }
    cp_async_wait_all();
    __syncthreads();
    for (int k0 = 0; k0 < nb; k0 += kChunkKeys) {
      if (k0 > 0) __syncthreads();  // previous chunk consumed
      load_entry_chunk<D>(sm, p, k0, min(kChunkKeys, nb - k0));
      __syncthreads();
      attend_chunk<D>(sm, p, st, nh);
    }
  }
}

// Push this CTA's partial of heads h0..h0+nh-1 to the owners, barrier, merge
// the heads this CTA owns.
template <int D, int CL>
__device__ void merge_heads(RowSmem<D> &sm, const RowParams &p, cg::cluster_group &cluster,
                            const AttnState &st, int64_t r, int h0, int nh) {
  constexpr int PV_WARPS = D / 8;
  constexpr int DL = D / 32;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int gid = lane >> 2, tig = lane & 3;
  const int c = (int)cluster.block_rank();
  // head h's partial goes to CTA h % CL, inbox slot (h / CL) * CL + c
  if (warp < PV_WARPS) {
    const int d0 = 8 * warp + 2 * tig;
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      const int h = gid + 8 * half;
      float *dst = cluster.map_shared_rank(&sm.inbox[0][0], h % CL) + ((h / CL) * CL + c) * (D + 2);
      dst[2 + d0] = st.o[2 * half];
      dst[2 + d0 + 1] = st.o[2 * half + 1];
    }
  }
  if (lane == 0) {  // warp h holds the max and sum of head h
    const int h = warp;
    float *dst = cluster.map_shared_rank(&sm.inbox[0][0], h % CL) + ((h / CL) * CL + c) * (D + 2);
    dst[0] = st.m;
    dst[1] = st.l;
  }
  cluster.sync();
  // merge: warp k merges head h = c + k*CL from CL partials in the inbox
  const int h = c + warp * CL;
  if (warp < kHeads / CL && h < nh) {
    const float *slot = &sm.inbox[warp * CL][0];
    const float m = (lane < CL) ? slot[lane * (D + 2)] : -INFINITY;
    const float l = (lane < CL) ? slot[lane * (D + 2) + 1] : 0.0f;
    const float M = warp_max(l > 0.0f ? m : -INFINITY);
    float *op = p.out + (r * p.H + h0 + h) * (int64_t)D;
    if (M == -INFINITY) {
#pragma unroll
      for (int i = 0; i < DL; ++i) op[lane + 32 * i] = 0.0f;
      if (p.lse && lane == 0) p.lse[r * p.H + h0 + h] = -INFINITY;
    } else {
      const float f = (l > 0.0f) ? exp2f(m - M) : 0.0f;
      const float L = warp_sum(l * f);
      float a[DL];
#pragma unroll
      for (int i = 0; i < DL; ++i) a[i] = 0.0f;
#pragma unroll
      for (int j = 0; j < CL; ++j) {
        const float fj = __shfl_sync(0xffffffffu, f, j);
        if (fj != 0.0f) {
#pragma unroll
          for (int i = 0; i < DL; ++i) a[i] = fmaf(slot[j * (D + 2) + 2 + lane + 32 * i], fj, a[i]);
        }
      }
      const float inv = 1.0f / L;
#pragma unroll
      for (int i = 0; i < DL; ++i) op[lane + 32 * i] = a[i] * inv;
      if (p.lse && lane == 0) p.lse[r * p.H + h0 + h] = (M + log2f(L)) * 0.69314718055994530942f;
    }
  }
}

// grid.x = rows * CL, cluster (CL, 1, 1).
template <int D, int CL>
__global__ void __launch_bounds__(kRowThreads, 1) row_cluster_kernel(const RowParams p) {
  extern __shared__ __align__(128) unsigned char row_smem_raw[];
  RowSmem<D> &sm = *reinterpret_cast<RowSmem<D> *>(row_smem_raw);
  cg::cluster_group cluster = cg::this_cluster();
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

  if (tid == 0) {
    mbar_init(&sm.bar, 1);
    fence_barrier_init();
  }
  __syncthreads();
  // Prologue, independent of the scan that produced the scores: the query and
  // the window part of attention.  With programmatic dependent launch this
  // overlaps the scan's tail.
  for (int i = tid; i < kBins2; i += kRowThreads) sm.h2[i] = 0u;
  AttnState st{{0.0f, 0.0f, 0.0f, 0.0f}, -INFINITY, 0.0f};
  if (p.do_attn) {
    load_q<D>(sm, p, r, 0, min(kHeads, p.H));
    attend_window<D, CL>(sm, p, st, r, c, min(kHeads, p.H));
  }
  pdl_wait_primary();  // the scores and histograms are complete from here on
  if (topk_here && tid == 0) {
    const int n0 = (int)min64(kStageScores, s1 - s0);
    uint32_t bytes = kBins1 * 4;
    if (bulk && n0 > 0) bytes += (uint32_t)(((n0 + 3) & ~3) * 4);
    mbar_arrive_expect_tx(&sm.bar, bytes);
    bulk_g2s(sm.h1, p.hist1 + r_local * kBins1, kBins1 * 4, &sm.bar);
    if (bulk && n0 > 0)
      bulk_g2s(sm.st.sc, p.scores + r_local * p.score_stride + s0,
               (uint32_t)(((n0 + 3) & ~3) * 4), &sm.bar);
  }

  bool abort = false;
  uint32_t phases = 0;
  if (p.do_topk) {
    if (topk_here) {
      row_topk<D, CL>(sm, p, cluster, r_local, r, K, bulk, s0, s1, abort, phases);
    } else {
      if (c == 0) {
        int32_t *orow = p.idx + r * (int64_t)p.topk;
        for (int i = tid; i < p.topk; i += kRowThreads) orow[i] = -1;
      }
      if (tid == 0) {
        sm.sel_base = 0;
        sm.sel_count = 0;
      }
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
        st = AttnState{{0.0f, 0.0f, 0.0f, 0.0f}, -INFINITY, 0.0f};
        attend_window<D, CL>(sm, p, st, r, c, nh);
      }
      if (p.do_topk) {
        attend_selected<D>(sm, p, st, r, lo, hi, true, sel_base, nh);
      } else {
        attend_selected<D>(sm, p, st, r, lo, hi, false, 0, nh);
      }
      __syncthreads();
      merge_heads<D, CL>(sm, p, cluster, st, r, h0, nh);
    }
  }
  if (abort && tid == 0 && phases > 0)  // let a late bulk copy land before exit
    mbar_wait_bounded(&sm.bar, (phases - 1) & 1u);
}

}  // namespace csa2
