// Sparse attention of decode rows handed over by the per-row selection
// ("Why Is DeepSeek V4.1 Flash So Fast?", section 3: the query attends to
// its Top-K compressed entries and to the 128-token sliding window;
// "Inference-Efficient LLMs", sections 3 and 6: bf16 window, FP4 entries,
// one joint softmax).
//
// The selection kernel's CTA g of row r publishes the indices it selected
// (ascending) and then a ready flag (n + 1); this kernel's CTA (r, g), 8
// warps, attends over exactly that list, so it can start on it as soon as
// that one CTA has selected -- no cluster, no wait for the whole selection.
// Launched right after the selection with programmatic dependent launch, it
// first loads the query and attends over its share of the window rows
// (neither depends on the selection) while the selection still runs.
//
// Chunks of 16 keys, one online softmax in base 2 per warp (the per-warp
// blocks of attn_rows.cuh: cp.async gathers, E2M1 -> exact bf16, mma.sync
// m16n8k16 with 16 heads as M): warp 0 takes the window chunks, then every
// warp w takes list chunks w, w + 8, ...; one loop with one chunk body
// serves both.  The warps' states merge into the CTA's partial (max, sum,
// acc) per head, written to global memory; the row's last CTA to finish
// (an atomic counter) merges the G partials of every head by log-sum-exp
// and writes out and lse.
#pragma once

#include "attn_rows.cuh"
#include "common.cuh"

namespace csa2 {
namespace ah {

constexpr int kWarps = 8;
constexpr int kThreads = 32 * kWarps;
constexpr int kHeads = 16;  // heads per pass (the MMAs' M)
constexpr int kMaxG = 16;   // lists (selecting CTAs) per row, at most

struct Params {
  ar::Params a;              // q, codes, scales, win_k, win_v, N, T, H, W, q_scale, out, lse, row0
  const int32_t *lists;      // [rows_local][G][list_stride]
  int64_t list_stride;
  uint32_t *flags;           // per row (stride flag_stride): G ready flags, then the done counter
  int64_t flag_stride;
  float *part;               // [rows_local][G][H][D + 4]: (m, l, -, -, acc[D]) per head
  int32_t G;
};

template <int D>
struct Smem {
  ar::WarpArea<D> aw[kWarps];   // per-warp list chunk buffers, then states
  ar::WarpArea<D> win;          // window chunk buffers
  uint16_t qb[kHeads][D + 8];   // query of the head pass, bf16
  float mf[kHeads][kWarps + 1]; // per head: each warp's factor, then the max
  float gf[kHeads][kMaxG];      // final merge: factor of each list's partial
  float gl[kHeads];             // final merge: 1 / sum
  uint32_t last;
};

template <int D>
__device__ void load_q(Smem<D> &sm, const ar::Params &p, int64_t r, int h0, int nh) {
  constexpr int PPH = D / 8;  // 16-byte pieces per head
  for (int i = threadIdx.x; i < kHeads * PPH; i += kThreads) {
    const int h = i / PPH, u = i % PPH;
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (h < nh) v = *reinterpret_cast<const uint4 *>(p.q + (r * p.H + h0 + h) * (int64_t)D + 8 * u);
    *reinterpret_cast<uint4 *>(&sm.qb[h][8 * u]) = v;
  }
}

// The list length once the selection has published it (every lane polls
// with acquire at GPU scope, then reads the list).  Gives up after ~2^31
// cycles: recorded in the status word, and the list taken as empty.
__device__ __forceinline__ uint32_t wait_list(const uint32_t *flag, int64_t cap) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(flag) : "memory");
  if (v == 0u) {
    const long long start = clock64();
    do {
      asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(flag) : "memory");
      if (v == 0u && clock64() - start > (1ll << 31)) {
        raise_status(kStatusWaitTimeout);
        return 0u;
      }
    } while (v == 0u);
  }
  return (uint32_t)min64((int64_t)v - 1, cap);
}

// One warp's part of a head pass into its state area; `first`: the first
// pass, whose list is not yet known.
template <int D>
__device__ void attend_warp(Smem<D> &sm, const Params &hp, int64_t rl, int g, bool first,
                            uint32_t &n_list) {
  const ar::Params &p = hp.a;
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int64_t r = p.row0 + rl;
  const int64_t b = r / p.T, t = r % p.T;
  const int32_t *list = hp.lists + (rl * hp.G + g) * hp.list_stride;
  const uint8_t *cseq = p.codes + b * p.N * (D / 2);
  const float *sseq = p.scales + b * p.N * (D / 16);
  const int w_lo = (p.W * g) / hp.G;
  const int nwin = (w == 0) ? (p.W * (g + 1)) / hp.G - w_lo : 0;  // window rows of warp 0
  const int64_t wrow0 = b * ((int64_t)p.W - 1 + p.T) + t + w_lo;
  ar::WarpArea<D> &wa = sm.aw[w];
  ar::WarpState<D> st;
  ar::state_init(st);
  int64_t nch = 0;
  auto entry_of = [&](int64_t ch) -> int32_t {  // this lane's key of list chunk ch
    const int64_t k = ch * ar::kChunk + (lane & 15);
    return k < (int64_t)n_list ? __ldcg(list + k) : -1;  // written by the selection kernel
  };
  bool ready = false;  // list known, first chunk issued
  int64_t ech = w;     // this warp's current list chunk
  int wr = 0;          // next window row
  int sb = 0;          // staging buffer of the current list chunk
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
        if (first)
          n_list = wait_list(hp.flags + rl * hp.flag_stride + g, hp.list_stride);
        nch = p.N > 0 ? ((int64_t)n_list + ar::kChunk - 1) / ar::kChunk : 0;
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

// This CTA's partial of heads h0 .. h0 + nh - 1 from the warps' states,
// into part[rl][g][h0 + h]: (max, sum, 0, 0, acc[D]).
template <int D>
__device__ void write_partial(Smem<D> &sm, const Params &hp, int64_t rl, int g, int h0, int nh) {
  const int tid = threadIdx.x;
  for (int i = tid; i < nh * kWarps; i += kThreads) {
    const int h = i / kWarps, w = i % kWarps;
    float M = -INFINITY;
#pragma unroll
    for (int v = 0; v < kWarps; ++v) M = fmaxf(M, sm.aw[v].merge.m[h]);
    sm.mf[h][w] = M == -INFINITY ? 0.0f : exp2f(sm.aw[w].merge.m[h] - M);
    if (w == 0) sm.mf[h][kWarps] = M;
  }
  __syncthreads();
  constexpr int U = D / 4 + 1;  // 16-byte pieces of a partial
  float *dst = hp.part + (rl * hp.G + g) * (int64_t)hp.a.H * (D + 4);
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
    *reinterpret_cast<float4 *>(dst + (int64_t)(h0 + h) * (D + 4) + 4 * q) = v;
  }
}

// The row's final merge, by its last CTA: for every head the G partials by
// log-sum-exp (a partial with sum 0 saw nothing and has factor 0).
template <int D>
__device__ void merge_row(Smem<D> &sm, const Params &hp, int64_t rl) {
  const ar::Params &p = hp.a;
  const int tid = threadIdx.x;
  const int64_t r = p.row0 + rl;
  const float *base = hp.part + rl * hp.G * (int64_t)p.H * (D + 4);
  for (int h0 = 0; h0 < p.H; h0 += kHeads) {
    const int nh = min(kHeads, p.H - h0);
    for (int h = tid >> 5; h < nh; h += kWarps) {  // warp: the factors and sum of a head
      const int lane = tid & 31;
      const float *ph = base + (int64_t)lane * p.H * (D + 4) + (int64_t)(h0 + h) * (D + 4);
      const float m = lane < hp.G ? __ldcg(ph) : -INFINITY;
      const float l = lane < hp.G ? __ldcg(ph + 1) : 0.0f;
      const float M = warp_max(l > 0.0f ? m : -INFINITY);
      const float f = (M != -INFINITY && l > 0.0f) ? exp2f(m - M) : 0.0f;
      const float L = warp_sum(l * f);
      if (lane < kMaxG) sm.gf[h][lane] = lane < hp.G ? f : 0.0f;
      if (lane == 0) {
        sm.gl[h] = M == -INFINITY ? 0.0f : 1.0f / L;
        if (p.lse)
          p.lse[r * p.H + h0 + h] =
              M == -INFINITY ? -INFINITY : (M + log2f(L)) * 0.69314718055994530942f;
      }
    }
    __syncthreads();
    // one thread per (head, 4 dims): the G partials' accumulators loaded
    // together (independent 16-byte loads, all in flight), then summed
    for (int i = tid; i < nh * (D / 4); i += kThreads) {
      const int h = i / (D / 4), q = i % (D / 4);
      const float *src = base + (int64_t)(h0 + h) * (D + 4) + 4 + 4 * q;
      float4 v[kMaxG];
#pragma unroll
      for (int j = 0; j < kMaxG; ++j)
        v[j] = j < hp.G ? __ldcg(reinterpret_cast<const float4 *>(src + (int64_t)j * p.H * (D + 4)))
                        : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
      float4 acc = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
#pragma unroll
      for (int j = 0; j < kMaxG; ++j) {
        const float fj = sm.gf[h][j];  // 0 beyond G and for a partial that saw nothing
        acc.x = fmaf(v[j].x, fj, acc.x);
        acc.y = fmaf(v[j].y, fj, acc.y);
        acc.z = fmaf(v[j].z, fj, acc.z);
        acc.w = fmaf(v[j].w, fj, acc.w);
      }
      const float inv = sm.gl[h];
      float *o = p.out + (r * p.H + h0 + h) * (int64_t)D + 4 * q;
      o[0] = acc.x * inv;
      o[1] = acc.y * inv;
      o[2] = acc.z * inv;
      o[3] = acc.w * inv;
    }
    __syncthreads();
  }
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1) attn_handoff_kernel(const Params hp) {
  extern __shared__ __align__(128) unsigned char ah_smem_raw[];
  Smem<D> &sm = *reinterpret_cast<Smem<D> *>(ah_smem_raw);
  const ar::Params &p = hp.a;
  const int tid = threadIdx.x;
  const int64_t rl = blockIdx.x / hp.G;
  const int g = (int)(blockIdx.x % hp.G);
  const int64_t r = p.row0 + rl;
  uint32_t n_list = 0u;
  for (int h0 = 0; h0 < p.H; h0 += kHeads) {
    const int nh = min(kHeads, p.H - h0);
    load_q<D>(sm, p, r, h0, nh);
    __syncthreads();
    attend_warp<D>(sm, hp, rl, g, h0 == 0, n_list);
    __syncthreads();  // every warp's state is stored
    write_partial<D>(sm, hp, rl, g, h0, nh);
    __syncthreads();  // states read (the next pass reuses the areas)
  }
  // the last CTA of the row to get here merges the row
  if (tid == 0) {
    __threadfence();  // this CTA's partials before its count
    uint32_t *done = hp.flags + rl * hp.flag_stride + hp.G;
    const uint32_t old = atomicAdd(done, 1u);
    sm.last = (old == (uint32_t)hp.G - 1u) ? 1u : 0u;
    if (sm.last) __threadfence();  // every CTA's partials after the count
  }
  __syncthreads();
  if (sm.last) merge_row<D>(sm, hp, rl);
}

}  // namespace ah
}  // namespace csa2
