// Exact top-k of index scores, ties to the lower index, output ascending.
//
// "Why Is DeepSeek V4.1 Flash So Fast?", sections 3-4: keep the Top-K
// compressed positions by indexer score.  Tie rule (lower index first) and
// the ascending output order are this library's readings.
//
// Radix selection over an order-preserving 32-bit key of the score, split
// into digits of 11, 11 and 10 bits:
//  * the scan kernel histograms digit 1 of every visible score (hist1);
//  * select (many CTAs per row): finds the digit-1 threshold t1 (the
//    largest digit whose suffix count reaches k), keeps every element with
//    digit 1 >= t1 as a candidate -- written in index order into the CTA's
//    own region -- and histograms digit 2 of the elements exactly at t1;
//  * finalize (one CTA per row): finds t2 from hist2 and, only when the
//    boundary bucket (t1, t2) holds more elements than still needed, a
//    digit-3 threshold t3 over that bucket; elements whose whole key equals
//    the threshold key are then taken in index order, which is the
//    lower-index tie rule.  A stable block-wide compaction over the
//    candidate regions in order writes the indices ascending.
// Every decision is made on integer keys, so the result is exact and does
// not depend on scheduling.
#pragma once
#include "common.cuh"

namespace csa2 {

constexpr int kSelThreads = 256, kSelItems = 8, kSelSpan = kSelThreads * kSelItems;
constexpr int kFinThreads = 512, kFinItems = 8, kFinSpan = kFinThreads * kFinItems;
constexpr int kMaxRegions = 1024;

__device__ __forceinline__ int64_t visible_rows(int64_t N, int64_t n_prior, int32_t ratio,
                                                int64_t t) {
  if (n_prior < 0) return N;
  int64_t v = n_prior + (t + 1) / ratio;
  return v < N ? v : N;
}

__device__ __forceinline__ uint32_t lanemask_lt() {
  uint32_t m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

// grid = (G2 regions, rows).
__global__ void __launch_bounds__(kSelThreads)
    topk_select_kernel(const float *__restrict__ scores, int64_t N, int32_t T, int64_t n_prior,
                       int32_t ratio, int64_t row0, int32_t topk,
                       const uint32_t *__restrict__ hist1, uint32_t *__restrict__ hist2,
                       uint2 *__restrict__ cand, uint32_t *__restrict__ cand_cnt) {
  __shared__ uint32_t sh_h2[kBins2];
  __shared__ uint32_t scratch[40];
  __shared__ uint32_t thr[2];
  __shared__ uint32_t warp_cnt[kSelThreads / 32];

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t r_local = blockIdx.y, r = row0 + r_local, t = r % T;
  const int G2 = gridDim.x, g = blockIdx.x;
  const int64_t V = visible_rows(N, n_prior, ratio, t);
  const int64_t K = V < topk ? V : topk;
  if (K == 0) {
    if (tid == 0) cand_cnt[r_local * G2 + g] = 0u;
    return;
  }
  for (int i = tid; i < kBins2; i += kSelThreads) sh_h2[i] = 0u;
  radix_threshold<kSelThreads, kBins1>(hist1 + r_local * kBins1, (uint32_t)K, scratch, thr);
  const uint32_t t1 = thr[0];

  const int64_t s0 = (V * g) / G2, s1 = (V * (g + 1)) / G2;
  const float *srow = scores + r_local * N;
  uint2 *out = cand + r_local * N + s0;
  uint32_t count = 0;
  for (int64_t base = s0; base < s1; base += kSelSpan) {
    uint32_t key[kSelItems];
#pragma unroll
    for (int j = 0; j < kSelItems; ++j) {
      const int64_t n = base + j * kSelThreads + tid;
      key[j] = (n < s1) ? score_key(srow[n]) : 0u;
    }
#pragma unroll
    for (int j = 0; j < kSelItems; ++j) {
      const int64_t n = base + j * kSelThreads + tid;
      const bool in = (n < s1) && key_d1(key[j]) >= t1;
      if (in && key_d1(key[j]) == t1) atomicAdd(&sh_h2[key_d2(key[j])], 1u);
      const uint32_t bal = __ballot_sync(0xffffffffu, in);
      if (lane == 0) warp_cnt[warp] = __popc(bal);
      __syncthreads();
      uint32_t off = 0, tot = 0;
#pragma unroll
      for (int w2 = 0; w2 < kSelThreads / 32; ++w2) {
        const uint32_t c = warp_cnt[w2];
        off += (w2 < warp) ? c : 0u;
        tot += c;
      }
      if (in) out[count + off + __popc(bal & lanemask_lt())] = make_uint2(key[j], (uint32_t)n);
      count += tot;
      __syncthreads();
    }
  }
  __syncthreads();
  uint32_t *h2row = hist2 + r_local * kBins2;
  for (int i = tid; i < kBins2; i += kSelThreads) {
    const uint32_t v = sh_h2[i];
    if (v) atomicAdd(h2row + i, v);
  }
  if (tid == 0) cand_cnt[r_local * G2 + g] = count;
}

// Locate candidate number i (0-based over all regions of the row, in
// order): region g with off[g] <= i < off[g+1].
__device__ __forceinline__ int find_region(const uint32_t *off, int G2, uint32_t i) {
  int lo = 0, hi = G2 - 1;  // largest g with off[g] <= i
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (off[mid] <= i)
      lo = mid;
    else
      hi = mid - 1;
  }
  return lo;
}

// grid = (rows).
__global__ void __launch_bounds__(kFinThreads)
    topk_finalize_kernel(int64_t N, int32_t T, int64_t n_prior, int32_t ratio, int64_t row0,
                         int32_t topk, const uint32_t *__restrict__ hist1,
                         const uint32_t *__restrict__ hist2, const uint2 *__restrict__ cand,
                         const uint32_t *__restrict__ cand_cnt, int G2,
                         int32_t *__restrict__ idx_out) {
  __shared__ uint32_t sh_off[kMaxRegions + 1];
  __shared__ uint32_t sh_h3[kBins3];
  __shared__ uint32_t scratch[40];
  __shared__ uint32_t thr1[2], thr2[2], thr3[2];

  const int tid = threadIdx.x;
  const int64_t r_local = blockIdx.x, r = row0 + r_local, t = r % T;
  const int64_t V = visible_rows(N, n_prior, ratio, t);
  const int64_t K = V < topk ? V : topk;
  int32_t *orow = idx_out + r * (int64_t)topk;
  if (K == 0) {
    for (int i = tid; i < topk; i += kFinThreads) orow[i] = -1;
    return;
  }

  // Region start offsets (exclusive prefix of the per-region counts).
  {
    constexpr int PER = (kMaxRegions + kFinThreads - 1) / kFinThreads;
    uint32_t c[PER], s = 0;
#pragma unroll
    for (int j = 0; j < PER; ++j) {
      const int gi = tid * PER + j;
      c[j] = (gi < G2) ? cand_cnt[r_local * G2 + gi] : 0u;
      s += c[j];
    }
    uint32_t total;
    uint32_t e = block_excl_scan<kFinThreads>(s, scratch, total);
#pragma unroll
    for (int j = 0; j < PER; ++j) {
      const int gi = tid * PER + j;
      if (gi < G2) sh_off[gi] = e;
      e += c[j];
    }
    if (tid == 0) sh_off[G2] = total;
  }
  __syncthreads();
  const uint32_t C = sh_off[G2];

  radix_threshold<kFinThreads, kBins1>(hist1 + r_local * kBins1, (uint32_t)K, scratch, thr1);
  const uint32_t t1 = thr1[0], r1 = (uint32_t)K - thr1[1];
  radix_threshold<kFinThreads, kBins2>(hist2 + r_local * kBins2, r1, scratch, thr2);
  const uint32_t t2 = thr2[0], r2 = r1 - thr2[1];
  const uint32_t nE = hist2[r_local * kBins2 + t2];
  const bool need3 = nE > r2;

  const uint2 *crow = cand + r_local * N;
  // Fetch candidates [i0, i0 + kFinItems) (blocked per thread) into registers.
  auto fetch = [&](uint32_t i0, uint2 *e, bool *ok) {
    if (i0 >= C) {
#pragma unroll
      for (int j = 0; j < kFinItems; ++j) ok[j] = false;
      return;
    }
    int gi = find_region(sh_off, G2, i0);
    uint32_t pos = i0 - sh_off[gi];
#pragma unroll
    for (int j = 0; j < kFinItems; ++j) {
      const uint32_t i = i0 + j;
      ok[j] = i < C;
      if (ok[j]) {
        while (sh_off[gi + 1] <= i) {  // step over finished / empty regions
          ++gi;
          pos = 0;
        }
        const int64_t s0 = (V * gi) / G2;
        e[j] = crow[s0 + pos];
        ++pos;
      }
    }
  };

  uint32_t t3 = 0, r3 = 0xffffffffu;
  if (need3) {
    for (int i = tid; i < kBins3; i += kFinThreads) sh_h3[i] = 0u;
    __syncthreads();
    for (uint32_t base = 0; base < C; base += kFinSpan) {
      uint2 e[kFinItems];
      bool ok[kFinItems];
      fetch(base + tid * kFinItems, e, ok);
#pragma unroll
      for (int j = 0; j < kFinItems; ++j)
        if (ok[j] && key_d1(e[j].x) == t1 && key_d2(e[j].x) == t2)
          atomicAdd(&sh_h3[key_d3(e[j].x)], 1u);
    }
    __syncthreads();
    radix_threshold<kFinThreads, kBins3>(sh_h3, r2, scratch, thr3);
    t3 = thr3[0];
    r3 = r2 - thr3[1];
  }

  // Stable compaction of the selected candidates, in index order.
  uint32_t written = 0, ties_before = 0;
  for (uint32_t base = 0; base < C; base += kFinSpan) {
    uint2 e[kFinItems];
    bool ok[kFinItems];
    fetch(base + tid * kFinItems, e, ok);
    // class: 2 = strictly above the threshold key, 1 = equal to it, 0 = below
    uint32_t cls[kFinItems];
    uint32_t nties = 0;
#pragma unroll
    for (int j = 0; j < kFinItems; ++j) {
      cls[j] = 0;
      if (!ok[j]) continue;
      const uint32_t k = e[j].x, a = key_d1(k), b2 = key_d2(k), c3 = key_d3(k);
      if (a > t1 || (a == t1 && b2 > t2))
        cls[j] = 2;
      else if (a == t1 && b2 == t2) {
        if (!need3 || c3 > t3)
          cls[j] = 2;
        else if (c3 == t3)
          cls[j] = 1;
      }
      nties += (cls[j] == 1);
    }
    uint32_t tie_total;
    uint32_t tie_rank = ties_before + block_excl_scan<kFinThreads>(nties, scratch, tie_total);
    bool sel[kFinItems];
    uint32_t nsel = 0;
#pragma unroll
    for (int j = 0; j < kFinItems; ++j) {
      sel[j] = (cls[j] == 2) || (cls[j] == 1 && tie_rank < r3);
      if (cls[j] == 1) ++tie_rank;
      nsel += sel[j];
    }
    uint32_t sel_total;
    uint32_t pos = written + block_excl_scan<kFinThreads>(nsel, scratch, sel_total);
#pragma unroll
    for (int j = 0; j < kFinItems; ++j)
      if (sel[j]) {
        if (pos < (uint32_t)topk) orow[pos] = (int32_t)e[j].y;
        ++pos;
      }
    written += sel_total;
    ties_before += tie_total;
  }
  for (int64_t i = (int64_t)written + tid; i < topk; i += kFinThreads) orow[i] = -1;
}

}  // namespace csa2
