// Sparse attention of decode rows on one thread-block cluster per row
// ("Why Is DeepSeek V4.1 Flash So Fast?", section 3: the query attends to
// its Top-K compressed entries and to the 128-token sliding window;
// "Inference-Efficient LLMs", sections 3 and 6: bf16 window, FP4 entries,
// one joint softmax).
//
// CL CTAs of 8 warps per query row: CTA c attends over index slots
// [k c / CL, k (c+1) / CL) of the row and over its share of the window rows,
// in 16-key chunks (the per-warp blocks of attn_rows.cuh: cp.async gathers,
// E2M1 -> exact bf16, mma.sync m16n8k16 with 16 heads as M, base-2 online
// softmax).  Warp 0 takes the window chunks, then every warp a takes entry
// chunks a, a + 8, ...; one loop with one chunk body serves both, so the
// window chunks leave that code fetched for the entry chunks.
//
// Launched after the selection with programmatic dependent launch, the
// kernel loads the query and attends over the window -- neither depends on
// the selection -- while the selection still runs on other SMs, and waits
// for the selection's results only before its first entry chunk.
//
// Merge: per head the max over the warps' states and each state's factor;
// the CTA's partial (max, sum, acc) of head h goes by one bulk copy into
// inbox slot (h / CL) * CL + c of the CTA that owns h (h mod CL), counted in
// bytes on the owner's barrier; each owner merges its heads' CL partials by
// log-sum-exp, writes out and lse, and acknowledges to every CTA of the
// cluster; a CTA leaves only once every CTA has acknowledged, i.e. once its
// copies have read all they read from its shared memory.
#pragma once
#include <cooperative_groups.h>

#include "attn_rows.cuh"
#include "common.cuh"

namespace csa2 {
namespace ac {

namespace cg = cooperative_groups;

constexpr int kWarps = 8;
constexpr int kThreads = 32 * kWarps;
constexpr int kHeads = 16;  // heads per pass (the MMAs' M)

template <int D, int CL>
struct Smem {
  ar::WarpArea<D> aw[kWarps];   // per-warp entry chunk buffers, then states
  ar::WarpArea<D> win;          // window chunk buffers
  uint16_t qb[kHeads][D + 8];   // query of the head pass, bf16
  alignas(16) float stage[kHeads][D + 4];  // this CTA's partial of each head, to send
  alignas(16) float inbox[kHeads][D + 4];  // received partials of the heads it merges
  float mf[kHeads][kWarps + 1];  // per head: each warp's factor, then the max
  float fac[kHeads];             // final merge: factor of each inbox slot
  float mrg_m[kHeads], mrg_l[kHeads];
  uint64_t bar_part;  // partials (bulk copies, bytes announced by this CTA)
  uint64_t bar_ack;   // CL arrivals: every CTA has received its partials
};

template <int D, int CL>
__device__ void load_q(Smem<D, CL> &sm, const ar::Params &p, int64_t r, int h0, int nh) {
  constexpr int PPH = D / 8;  // 16-byte pieces per head
  for (int i = threadIdx.x; i < kHeads * PPH; i += kThreads) {
    const int h = i / PPH, u = i % PPH;
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (h < nh) v = *reinterpret_cast<const uint4 *>(p.q + (r * p.H + h0 + h) * (int64_t)D + 8 * u);
    *reinterpret_cast<uint4 *>(&sm.qb[h][8 * u]) = v;
  }
}

// One warp's part of a head pass, into its state area (see the file
// comment); with `wait` the warp waits for the kernel it depends on before
// reading the index row.
template <int D, int CL>
__device__ void attend_warp(Smem<D, CL> &sm, const ar::Params &p, int64_t r, int c, bool wait) {
  const int lane = threadIdx.x & 31, a = threadIdx.x >> 5;
  const int64_t b = r / p.T, t = r % p.T;
  const int32_t *irow = p.idx + r * (int64_t)p.topk;
  const uint8_t *cseq = p.codes + b * p.N * (D / 2);
  const float *sseq = p.scales + b * p.N * (D / 16);
  const int64_t lo = ((int64_t)p.topk * c) / CL, hi = ((int64_t)p.topk * (c + 1)) / CL;
  const int w_lo = (p.W * c) / CL;
  const int nwin = (a == 0) ? (p.W * (c + 1)) / CL - w_lo : 0;  // window rows of warp 0
  const int64_t wrow0 = b * ((int64_t)p.W - 1 + p.T) + t + w_lo;
  const int64_t nch = p.N > 0 ? (hi - lo + ar::kChunk - 1) / ar::kChunk : 0;
  ar::WarpArea<D> &wa = sm.aw[a];
  ar::WarpState<D> st;
  ar::state_init(st);
  auto entry_of = [&](int64_t ch) -> int32_t {  // this lane's key of entry chunk ch
    const int64_t k = lo + ch * ar::kChunk + (lane & 15);
    return k < hi ? irow[k] : -1;
  };
  bool ready = false;  // first entry chunk issued
  int64_t ech = a;     // this warp's current entry chunk
  int wr = 0;          // next window row
  int sb = 0;          // staging buffer of the current entry chunk
  uint32_t mask_next = 0u;
#pragma unroll 1
  for (;;) {
    const bool is_win = wr < nwin;
    uint32_t mask;
    if (is_win) {
      mask = ar::load_window_rows<D>(sm.win, p.win_k, p.win_v, wrow0 + wr,
                                     min(ar::kChunk, nwin - wr));
    } else {
      if (!ready) {
        if (wait) pdl_wait_primary();  // the index row is complete from here on
        if (ech < nch) mask_next = ar::gather_entries<D>(wa, 0, entry_of(ech), p.N, cseq, sseq);
        ready = true;
      }
      if (ech >= nch) break;
      // chunk ech sits in buffer sb; the next one goes into sb ^ 1
      mask = mask_next;
      const bool more = ech + kWarps < nch;
      if (more)
        mask_next = ar::gather_entries<D>(wa, sb ^ 1, entry_of(ech + kWarps), p.N, cseq, sseq);
      if (more)
        ar::cp_wait<1>();
      else
        ar::cp_wait<0>();
      __syncwarp();
      ar::convert_entries<D>(wa, sb);
      __syncwarp();
    }
    ar::WarpArea<D> &ca = is_win ? sm.win : wa;
    ar::attend_chunk16<D>(ca, sm.qb, st, mask, is_win, ca.s.scales[is_win ? 0 : sb], p.q_scale);
    __syncwarp();
    if (is_win) {
      wr += ar::kChunk;
    } else {
      ech += kWarps;
      sb ^= 1;
    }
  }
  ar::store_state<D>(wa, st);
}

// The merge of a head pass (see the file comment).
template <int D, int CL>
__device__ void merge(Smem<D, CL> &sm, const ar::Params &p, int64_t r, int c, int h0, int nh,
                      uint32_t pass) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  for (int i = tid; i < nh * kWarps; i += kThreads) {
    const int h = i / kWarps, w = i % kWarps;
    float M = -INFINITY;
#pragma unroll
    for (int v = 0; v < kWarps; ++v) M = fmaxf(M, sm.aw[v].merge.m[h]);
    sm.mf[h][w] = M == -INFINITY ? 0.0f : exp2f(sm.aw[w].merge.m[h] - M);
    if (w == 0) sm.mf[h][kWarps] = M;
  }
  __syncthreads();
  constexpr int U = D / 4 + 1;  // 16-byte pieces of a partial: (m, l, 0, 0), then acc
  if (tid == 0) {
    const int owned = nh > c ? (nh - 1 - c) / CL + 1 : 0;
    mbar_arrive_expect_tx(&sm.bar_part, (uint32_t)(owned * CL * (D + 4) * 4));
  }
  for (int i = tid; i < nh * U; i += kThreads) {
    const int h = i / U, q = i % U;
    float4 v = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    if (q == 0) {
#pragma unroll
      for (int w = 0; w < kWarps; ++w) v.y = fmaf(sm.aw[w].merge.l[h], sm.mf[h][w], v.y);
      v.x = sm.mf[h][kWarps];
    } else {
#pragma unroll
      for (int w = 0; w < kWarps; ++w) {
        const float4 o = *reinterpret_cast<const float4 *>(&sm.aw[w].merge.o[h][4 * (q - 1)]);
        const float f = sm.mf[h][w];
        v.x = fmaf(o.x, f, v.x);
        v.y = fmaf(o.y, f, v.y);
        v.z = fmaf(o.z, f, v.z);
        v.w = fmaf(o.w, f, v.w);
      }
    }
    *reinterpret_cast<float4 *>(&sm.stage[h][4 * q]) = v;
  }
  fence_proxy_async_smem();
  __syncthreads();
  if (warp == 0 && lane < nh)
    bulk_s2s_cluster(&sm.inbox[(lane / CL) * CL + c][0], &sm.stage[lane][0],
                     (uint32_t)((D + 4) * 4), &sm.bar_part, (uint32_t)(lane % CL));
  // the partials of the heads this CTA merges; a wait that gives up is
  // recorded in the status word
  mbar_wait_cluster_bounded(&sm.bar_part, pass & 1u);
  if (warp == 0 && lane < CL) mbar_remote_arrive(&sm.bar_ack, (uint32_t)lane);
  // head h = c + k*CL (k < kHeads / CL) from its CL partials in slots
  // [k*CL, k*CL + CL): warp k finds the max, the factors and the sum, then
  // one thread per (head, dim) sums the weighted partials
  constexpr int KH = kHeads / CL;
  static_assert(KH <= kWarps, "one warp per merged head");
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
  for (int i = tid; i < KH * D; i += kThreads) {
    const int k = i / D, e = i % D, h = c + k * CL;
    if (h >= nh) continue;
    float *op = p.out + (r * p.H + h0 + h) * (int64_t)D;
    if (sm.mrg_m[k] == -INFINITY) {
      op[e] = 0.0f;
      continue;
    }
    float acc = 0.0f;
#pragma unroll
    for (int j = 0; j < CL; ++j) {
      const float fj = sm.fac[k * CL + j];
      if (fj != 0.0f) acc = fmaf(sm.inbox[k * CL + j][4 + e], fj, acc);
    }
    op[e] = acc * (1.0f / sm.mrg_l[k]);
  }
  // this CTA's copies of the pass have landed once every CTA has acknowledged
  mbar_wait_cluster_bounded(&sm.bar_ack, pass & 1u);
}

template <int D, int CL>
__global__ void __launch_bounds__(kThreads, 1)
    attn_cluster_kernel(const ar::Params p, int wait_primary) {
  extern __shared__ __align__(128) unsigned char ac_smem_raw[];
  Smem<D, CL> &sm = *reinterpret_cast<Smem<D, CL> *>(ac_smem_raw);
  cg::cluster_group cluster = cg::this_cluster();
  const int tid = threadIdx.x;
  const int c = (int)cluster.block_rank();
  const int64_t r = p.row0 + blockIdx.x / CL;
  if (tid == 0) {
    mbar_init(&sm.bar_part, 1);
    mbar_init(&sm.bar_ack, CL);
    fence_barrier_init();
  }
  __syncthreads();
  // every CTA running with its barriers initialised before any copy into it
  asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
  load_q<D, CL>(sm, p, r, 0, min(kHeads, p.H));
  __syncthreads();
  asm volatile("barrier.cluster.wait.aligned;" ::: "memory");
  for (int h0 = 0; h0 < p.H; h0 += kHeads) {
    const int nh = min(kHeads, p.H - h0);
    if (h0 > 0) {
      cluster.sync();  // the previous merge read this CTA's inbox
      load_q<D, CL>(sm, p, r, h0, nh);
      __syncthreads();
    }
    attend_warp<D, CL>(sm, p, r, c, wait_primary != 0 && h0 == 0);
    __syncthreads();  // every warp's state is stored
    merge<D, CL>(sm, p, r, c, h0, nh, (uint32_t)(h0 / kHeads));
  }
}

}  // namespace ac
}  // namespace csa2
