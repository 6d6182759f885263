// Fused decode layer: index scan, exact Top-K and sparse attention of a
// batch of decode query rows (one query token per sequence) in one
// cooperative launch, one CTA per SM.
//
// What it computes is the layer step of index_scan.cuh + row_cluster.cuh
// ("Why Is DeepSeek V4.1 Flash So Fast?", sections 3-4: index every
// compressed position, keep the Top-K, attend over them and the 128-token
// window; "Inference-Efficient LLMs", section 6: FP4 entries with per-group
// scales), with the same score, selection and attention rules.  What
// differs is where the work runs and how the CTAs meet:
//
//   scan     The rows' keys, laid end to end (row r, entry n -> r*N + n), are
//            cut into one equal slice per CTA.  Each CTA streams its slice
//            through a ring of shared-memory tiles (1-D bulk copies on
//            mbarriers), keeps every score of the slice in shared memory
//            (the scores never go to HBM) and histograms digit 1 of each
//            score's order-preserving key.  At the end of each row segment
//            it adds its histogram into the row's global histogram and
//            arrives on the row's first counter.
//   round 1  Once every CTA holding part of row r has arrived, each of them
//            finds the digit-1 threshold bin t1 from the row's histogram and
//            writes the elements of its slice with digit 1 >= t1 (every
//            entry that can be selected), in index order, to its own region
//            of the row's candidate array, with the count; then it arrives
//            on the row's second counter.
//   round 2  P attention CTAs per row wait for every candidate list of the
//            row, load them (index order across slices), and each finds the
//            exact threshold key (digits 2 and 3 within the bin t1, ties to
//            the lower index) and every selected entry's output position.
//            CTA j writes output positions [K*j/P, K*(j+1)/P) and attends
//            over those entries and its share of the window rows (the
//            per-warp blocks of attn_rows.cuh), writes its partial softmax
//            state per head, and arrives on the row's third counter; the
//            CTA that arrives last merges the P partials by log-sum-exp.
//
// Every CTA must be resident at once (CTAs wait for one another), which
// the cooperative launch guarantees; every wait is bounded and records a
// timeout in the device status word, after which the CTA carries on with
// every index still bounded.  The row histograms and counters start at
// zero (the host clears them before the launch).  Data written by other
// CTAs during the launch is read through L2 only (ld.global.cg).
#pragma once
#include "attn_rows.cuh"
#include "common.cuh"
#include "pack.cuh"

namespace csa2 {
namespace fd {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kAttnWarps = 10;     // warps that run attention chunks
constexpr int kHeads = 16;         // heads of a query row (the MMAs' M)
constexpr int kMaxStages = 8;
constexpr int kMaxG = 512;         // CTAs of a launch (one per SM)
constexpr int kSelCap = 4096;      // output positions one CTA handles
constexpr int kMaxP = 16;          // attention CTAs per row at most
constexpr int kHistStride = kBins1 + 4;
constexpr int kArrive = 4;         // counters per row: scanned, listed, attended

struct Params {
  // indexer
  const int8_t *q_idx;   // [rows_global, H_I, d_I]
  const float *w;        // [rows_global, H_I]
  const int8_t *k_idx;   // [B, N, d_I] int8 keys; with FP4 keys the codes [B, N, d_I/2]
  const uint8_t *k_exps; // FP4 keys only: [B, N, d_I/32] biased block exponents
                         // (row r of this launch reads sequence row0 + r)
  int64_t N;
  int32_t R;             // rows of this launch
  int64_t row0;
  int32_t topk;
  int32_t *idx;          // [rows_global, topk]
  int64_t per_cta;       // keys per CTA slice (a multiple of 16)
  int32_t g_row;         // CTAs per row: CTA c scans slice c % g_row of row c / g_row
  // workspace
  uint32_t *hist1;       // [R, kHistStride]  (zero at launch)
  uint32_t *arrive;      // [R, kArrive]      (zero at launch)
  uint32_t *cnt;         // [R, G] candidates per slice
  uint2 *cand;           // [R, N] (key, entry) lists, slice c's at its first entry
  float *part;           // [R, p_att, kHeads, D + 4] partial states (m, l, -, -, acc)
  // optional: block maxima of the rows' scores for a candidate pool
  // (hierarchical indexer): bkey[rg, j] = the largest score key of positions
  // [j*pool_block, (j+1)*pool_block) of global row rg (zero at launch)
  uint32_t *bkey;        // [rows_global, n_pool_blocks] or null
  int32_t pool_block;
  int64_t n_pool_blocks;
  // shared-memory layout (bytes)
  uint32_t off_sc, off_hist, off_qs, cap;  // ring at 0; phase-3 buffers alias it
  int32_t stages;
  int32_t p_att;         // attention CTAs per row
  // attention
  int32_t do_attn;
  const uint16_t *q;     // bf16 [rows_global, H, D]
  const uint8_t *codes;  // [B, N, D/2]
  const float *scales;   // [B, N, D/16]
  const uint16_t *win_k; // bf16 [B, W, D]
  const uint16_t *win_v;
  int32_t H, W;
  float q_scale;         // sm_scale * log2(e)
  float *out;            // [rows_global, H, D]
  float *lse;            // [rows_global, H] or null
};

// ---------------------------------------------------------------------------
// Cross-CTA helpers.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t ld_acquire_gpu(const uint32_t *p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Spin (one thread) until *ctr >= target, for at most ~2^31 cycles; a
// timeout is recorded in the status word.
__device__ __forceinline__ bool wait_count(const uint32_t *ctr, uint32_t target,
                                           long long limit = (1ll << 31)) {
  if (ld_acquire_gpu(ctr) >= target) return true;
  const long long start = clock64();
  while (ld_acquire_gpu(ctr) < target) {
    if (clock64() - start > limit) {
      raise_status(kStatusWaitTimeout);
      return false;
    }
  }
  return true;
}

// Every thread's prior global writes, then one arrival (thread 0).
// Contains __syncthreads().  Returns the counter's old value on thread 0.
__device__ __forceinline__ uint32_t arrive_all(uint32_t *ctr) {
  __threadfence();
  __syncthreads();
  uint32_t old = 0;
  if (threadIdx.x == 0) old = atomicAdd(ctr, 1u);
  return old;
}

// Slice s of a row: entries [min(s*per, N), min((s+1)*per, N)).
__host__ __device__ __forceinline__ int64_t slice_begin(int64_t s, int64_t per, int64_t N) {
  const int64_t f = s * per;
  return f < N ? f : N;
}

// CTAs whose slice holds part of row r: [first, last] (the row's first
// ceil(N / per) CTAs; the rest of its g_row CTAs have empty slices).
__device__ __forceinline__ void row_ctas(int64_t r, int64_t N, int64_t per, int g_row, int &first,
                                         int &last) {
  const int64_t ns = (N + per - 1) / per;
  first = (int)(r * g_row);
  last = first + (int)(ns < g_row ? ns : g_row) - 1;
}

// Candidate class against the threshold key (t1, t2, t3): 2 above, 1 equal, 0 below.
__device__ __forceinline__ uint32_t key_class(uint32_t k, uint32_t t1, uint32_t t2, uint32_t t3,
                                              bool need3) {
  const uint32_t a = key_d1(k), b = key_d2(k), c = key_d3(k);
  if (a > t1 || (a == t1 && b > t2)) return 2u;
  if (a == t1 && b == t2) {
    if (!need3 || c > t3) return 2u;
    if (c == t3) return 1u;
  }
  return 0u;
}

// Key formats: int8 index keys, or FP4 index keys (E2M1 codes with one
// power-of-two scale per 32 elements, pack.cuh).
constexpr int kKeysInt8 = 0, kKeysFp4 = 1;

// A row's global histogram into shared memory: every thread issues its
// loads before storing any (one L2 round trip, not one per bin).
__device__ __forceinline__ void load_hist(uint32_t *dst, const uint32_t *src) {
  constexpr int PER = kBins1 / kThreads;
  uint32_t v[PER];
#pragma unroll
  for (int u = 0; u < PER; ++u) v[u] = __ldcg(src + threadIdx.x + u * kThreads);
#pragma unroll
  for (int u = 0; u < PER; ++u) dst[threadIdx.x + u * kThreads] = v[u];
}

template <int DI, int HI, int KF>
struct Shape {
  // int8: NCH 16-byte chunks of d_I keys bytes; FP4: NCH blocks of 32
  // elements, one 16-byte chunk of codes each
  static constexpr int NCH = KF == kKeysInt8 ? DI / 16 : DI / 32;
  static constexpr int CB = KF == kKeysInt8 ? DI : DI / 2;  // key bytes per key in the tile
  static constexpr int EB = KF == kKeysInt8 ? 0 : DI / 32;  // exponent bytes per key
  static constexpr int TK = CB <= 64 ? kThreads : 16384 / CB;  // keys per tile
  static constexpr int TILE_BYTES = TK * (CB + EB);
  static constexpr int QW = KF == kKeysInt8 ? 1 : 2;         // query int4 per chunk
  static constexpr bool QREG = HI * NCH * QW <= 16;
  static_assert(DI % 16 == 0 && NCH >= 1 && NCH <= 8, "d_I in {16,32,64,128}");
  static_assert(KF == kKeysInt8 || (DI % 32 == 0 && HI * NCH * QW <= 16), "FP4 keys shape");
};

// Rotation of the chunk order of thread t: the 8 threads of a 128-byte
// shared-memory phase read 8 different 16-byte bank groups.
template <int NCH>
__device__ __forceinline__ int chunk_rot(int t) {
  return (NCH == 1) ? 0 : (t / (8 / NCH)) % NCH;
}

template <int D>
struct StaticSmem {
  uint64_t full_bar[kMaxStages];
  uint32_t scratch[40];
  uint32_t thr[8];
  uint32_t pref[kMaxG + 1];
  int32_t sel[kSelCap];
  alignas(16) uint16_t qb[kHeads][D + 8];
  float mf[kHeads][kAttnWarps + 1];
  float fac[32][kHeads];
  float mrg_m[kHeads], mrg_l[kHeads];
  uint32_t last;
};

// ---------------------------------------------------------------------------
// The kernel.
// ---------------------------------------------------------------------------
template <int DI, int HI, int D, int KF>
__global__ void __launch_bounds__(kThreads, 1) decode_fused_kernel(const Params p) {
  using S = Shape<DI, HI, KF>;
  constexpr int NCH = S::NCH, TK = S::TK, QW = S::QW;
  extern __shared__ __align__(128) unsigned char dsm[];
  __shared__ StaticSmem<D> ss;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int c = blockIdx.x, G = gridDim.x;
  const int64_t N = p.N;
  // this CTA's slice: entries [n0, n1) of row c / g_row, as flattened
  // positions f = row * N + n (a slice never crosses a row)
  const int my_row = c / p.g_row;
  const int64_t my_n0 = slice_begin(c % p.g_row, p.per_cta, N);
  const int64_t my_n1 = slice_begin(c % p.g_row + 1, p.per_cta, N);
  const int64_t f0 = (int64_t)my_row * N + my_n0, f1 = (int64_t)my_row * N + my_n1;
  const int r_lo = f0 < f1 ? my_row : 0;
  const int r_hi = f0 < f1 ? my_row : -1;  // rows [r_lo, r_hi] hold this slice
  const int64_t K = N < p.topk ? N : p.topk;            // entries selected per row

  float *sc = reinterpret_cast<float *>(dsm + p.off_sc);       // this slice's scores
  uint32_t *hist = reinterpret_cast<uint32_t *>(dsm + p.off_hist);
  int8_t *qs = reinterpret_cast<int8_t *>(dsm + p.off_qs);     // index query (when not in registers)

  // ---------------------------------------------------------------- scan --
  // Tile k of the slice: row and entry range (tiles never cross a row).
  int ntiles = 0;
  for (int r = r_lo; r <= r_hi; ++r) {
    const int64_t s0 = (f0 > r * N ? f0 : r * N) - r * N;
    const int64_t s1 = (f1 < (r + 1) * N ? f1 : (r + 1) * N) - r * N;
    ntiles += (int)((s1 - s0 + TK - 1) / TK);
  }
  auto tile_of = [&](int k, int &row, int64_t &n0, int &nk) {
    row = r_lo;
    n0 = 0;
    nk = 0;
    for (int r = r_lo; r <= r_hi; ++r) {
      const int64_t s0 = (f0 > r * N ? f0 : r * N) - r * N;
      const int64_t s1 = (f1 < (r + 1) * N ? f1 : (r + 1) * N) - r * N;
      const int nt = (int)((s1 - s0 + TK - 1) / TK);
      if (k < nt) {
        row = r;
        n0 = s0 + (int64_t)k * TK;
        nk = (int)min64(TK, s1 - n0);
        return;
      }
      k -= nt;
    }
  };
  auto issue = [&](int k) {  // thread 0: bulk copy of tile k into its stage
    int row, nk;
    int64_t n0;
    tile_of(k, row, n0, nk);
    const int s = k % p.stages;
    const int64_t key0 = (p.row0 + row) * N + n0;
    unsigned char *stage = dsm + (size_t)s * S::TILE_BYTES;
    if constexpr (KF == kKeysInt8) {
      const uint32_t bytes = (uint32_t)nk * DI;
      mbar_arrive_expect_tx(&ss.full_bar[s], bytes);
      bulk_g2s(stage, p.k_idx + key0 * DI, bytes, &ss.full_bar[s]);
    } else {  // codes, then the block exponents behind them
      const uint32_t cb = (uint32_t)nk * S::CB, eb = (uint32_t)nk * S::EB;
      mbar_arrive_expect_tx(&ss.full_bar[s], cb + eb);
      bulk_g2s(stage, p.k_idx + key0 * S::CB, cb, &ss.full_bar[s]);
      bulk_g2s(stage + TK * S::CB, p.k_exps + key0 * S::EB, eb, &ss.full_bar[s]);
    }
  };

  for (int i = tid; i < kBins1; i += kThreads) hist[i] = 0u;
  if (tid == 0) {
    for (int s = 0; s < p.stages; ++s) mbar_init(&ss.full_bar[s], 1);
    fence_barrier_init();
  }
  __syncthreads();
  if (tid == 0)
    for (int k = 0; k < p.stages && k < ntiles; ++k) issue(k);

  const int x = chunk_rot<NCH>(tid);
  int4 qreg[S::QREG ? HI * NCH * QW : 1];
  float wh[HI];
  int cur = -1;  // row whose query is loaded
  int abort_it = -1;
  auto flush_row = [&](int r) {  // histogram of the finished row segment -> global, arrive
    __syncthreads();  // every thread's counts of the row's last tile are in
    uint32_t *g = p.hist1 + (int64_t)r * kHistStride;
    for (int i = tid; i < kBins1; i += kThreads) {
      const uint32_t v = hist[i];
      if (v) {
        atomicAdd(g + i, v);
        hist[i] = 0u;
      }
    }
    arrive_all(p.arrive + (int64_t)r * kArrive + 0);
  };
  for (int it = 0; it < ntiles; ++it) {
    const int s = it % p.stages;
    const bool ok = mbar_wait_bounded(&ss.full_bar[s], (uint32_t)(it / p.stages) & 1u);
    if (__syncthreads_or(!ok)) {
      abort_it = it;
      break;
    }
    if (tid == 0 && it >= 1 && it - 1 + p.stages < ntiles) {
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      issue(it - 1 + p.stages);
    }
    int row, nk;
    int64_t n0;
    tile_of(it, row, n0, nk);
    if (row != cur) {
      if (cur >= 0) flush_row(cur);
      cur = row;
      const int64_t rg = p.row0 + row;
      // this row's index query, pre-permuted by the thread's chunk rotation
      const int4 *qrow = reinterpret_cast<const int4 *>(p.q_idx + rg * HI * DI);
      if constexpr (S::QREG) {
#pragma unroll
        for (int h = 0; h < HI; ++h)
#pragma unroll
          for (int cc = 0; cc < NCH; ++cc)
#pragma unroll
            for (int u = 0; u < QW; ++u)
              qreg[(h * NCH + cc) * QW + u] = qrow[(h * NCH + (cc ^ x)) * QW + u];
      } else {
        __syncthreads();
        for (int i = tid; i < HI * NCH * QW; i += kThreads)
          reinterpret_cast<int4 *>(qs)[i] = qrow[i];
        __syncthreads();
      }
#pragma unroll
      for (int h = 0; h < HI; ++h) wh[h] = p.w[rg * HI + h];
    }
    const unsigned char *tile = dsm + (size_t)s * S::TILE_BYTES;
    const int64_t lbase = (int64_t)row * N + n0 - f0;  // local index of the tile's first key
    if constexpr (KF == kKeysFp4) {
      if (tid < nk) {
        const float score = fp4_key_score<NCH, HI, S::QREG>(
            tile + tid * S::CB, tile + TK * S::CB + tid * S::EB, qreg,
            reinterpret_cast<const int4 *>(qs), wh, x);
        sc[lbase + tid] = score;
        atomicAdd(&hist[key_d1(score_key(score))], 1u);
      }
    } else if (tid < nk) {
      const unsigned char *krow = tile + tid * DI;
      int dot[HI];
#pragma unroll
      for (int h = 0; h < HI; ++h) dot[h] = 0;
#pragma unroll
      for (int cc = 0; cc < NCH; ++cc) {
        const int4 kv = *reinterpret_cast<const int4 *>(krow + ((cc ^ x) << 4));
#pragma unroll
        for (int h = 0; h < HI; ++h) {
          int4 qv;
          if constexpr (S::QREG)
            qv = qreg[h * NCH + cc];
          else
            qv = reinterpret_cast<const int4 *>(qs)[h * NCH + (cc ^ x)];
          dot[h] = __dp4a(kv.x, qv.x, dot[h]);
          dot[h] = __dp4a(kv.y, qv.y, dot[h]);
          dot[h] = __dp4a(kv.z, qv.z, dot[h]);
          dot[h] = __dp4a(kv.w, qv.w, dot[h]);
        }
      }
      float acc = 0.0f;
#pragma unroll
      for (int h = 0; h < HI; ++h) acc = __fadd_rn(acc, __fmul_rn(wh[h], __int2float_rn(dot[h])));
      const float score = __fadd_rn(acc, 0.0f);
      sc[lbase + tid] = score;
      atomicAdd(&hist[key_d1(score_key(score))], 1u);
    }
  }
  if (abort_it >= 0) {  // let the copies in flight land before their buffers are reused
    if (tid == 0) {
      const int upto = min(ntiles, max(abort_it - 1, 0) + p.stages);
      for (int k = 0; k < p.stages && k < upto; ++k) {
        const int last = k + ((upto - 1 - k) / p.stages) * p.stages;
        mbar_wait_bounded(&ss.full_bar[k], (uint32_t)(last / p.stages) & 1u);
      }
    }
    __syncthreads();
    // the rows this CTA has not flushed still get their arrival, so that no
    // other CTA waits for it (results are wrong; the status word says so)
  }
  if (cur >= 0) flush_row(cur);
  for (int r = (cur >= 0 ? cur + 1 : r_lo); r <= r_hi; ++r) arrive_all(p.arrive + (int64_t)r * kArrive);

  // ----------------------------------------------------------- round 1 --
  // Per row segment: the digit-1 threshold, then this slice's candidates.
  for (int r = r_lo; r <= r_hi; ++r) {
    int cf, cl;
    row_ctas(r, N, p.per_cta, p.g_row, cf, cl);
    if (tid == 0) wait_count(p.arrive + (int64_t)r * kArrive + 0, (uint32_t)(cl - cf + 1));
    __syncthreads();
    load_hist(hist, p.hist1 + (int64_t)r * kHistStride);
    __syncthreads();
    radix_threshold<kThreads, kBins1>(hist, (uint32_t)K, ss.scratch, ss.thr);
    const uint32_t t1 = ss.thr[0];
    const uint32_t k1 = t1 << 21;
    // digit 1 >= t1  <=>  score >= f1 (keys are monotone in the score)
    const float fth = (t1 <= 3u) ? -__int_as_float(0x7f800000)
                                 : __uint_as_float((k1 & 0x80000000u) ? (k1 & 0x7fffffffu) : ~k1);
    const int64_t s0 = (f0 > r * N ? f0 : r * N) - r * N;
    const int64_t s1 = (f1 < (r + 1) * N ? f1 : (r + 1) * N) - r * N;
    const float *srow = sc + (r * N + s0 - f0);
    uint2 *dst = p.cand + (int64_t)r * N + s0;
    const int64_t len = s1 - s0;
    uint32_t count = 0;
    for (int64_t rb = 0; rb < len; rb += 32 * kThreads) {
      const int n = (int)min64(32 * kThreads, len - rb);
      const int base = 32 * tid;
      uint32_t bits = 0u;
#pragma unroll 8
      for (int q = 0; q < 32; ++q) {
        const int qq = (q + tid) & 31;  // rotated: conflict-free
        const int i = base + qq;
        if (i < n && srow[rb + i] >= fth) bits |= 1u << qq;
      }
      uint32_t total;
      uint32_t pos = count + block_excl_scan<kThreads>((uint32_t)__popc(bits), ss.scratch, total);
      while (bits) {
        const int i = base + __ffs(bits) - 1;
        bits &= bits - 1u;
        dst[pos++] = make_uint2(score_key(srow[rb + i]), (uint32_t)(s0 + rb + i));
      }
      count += total;
    }
    if (tid == 0) p.cnt[(int64_t)r * G + c] = count;
    if (p.bkey) {  // block maxima of this segment (a block may span two slices)
      const int64_t blk = p.pool_block;
      uint32_t *brow = p.bkey + (p.row0 + r) * p.n_pool_blocks;
      for (int64_t jb = s0 / blk + tid; jb * blk < s1; jb += kThreads) {
        const int64_t a = jb * blk > s0 ? jb * blk : s0;
        const int64_t e = (jb + 1) * blk < s1 ? (jb + 1) * blk : s1;
        float m = srow[a - s0];
        for (int64_t n = a + 1; n < e; ++n) m = fmaxf(m, srow[n - s0]);
        atomicMax(brow + jb, score_key(m));
      }
    }
    arrive_all(p.arrive + (int64_t)r * kArrive + 1);
  }

  // ----------------------------------------------------------- round 2 --
  const int ra = my_row;
  const int j = c % p.g_row;  // attention CTA j of row ra when j < P
  const int P = p.p_att;
  if (j >= P || ra >= p.R) return;
  const int64_t rg = p.row0 + ra;
  int cf, cl;
  row_ctas(ra, N, p.per_cta, p.g_row, cf, cl);
  const int nseg = cl - cf + 1;
  uint2 *clist = reinterpret_cast<uint2 *>(dsm);                    // candidate list
  uint32_t *h2 = reinterpret_cast<uint32_t *>(dsm + (size_t)p.cap * 8);  // digit-2/3 histogram
  if (tid == 0) wait_count(p.arrive + (int64_t)ra * kArrive + 1, (uint32_t)nseg);
  __syncthreads();
  // digit-1 threshold of the row again (from the complete histogram)
  load_hist(h2, p.hist1 + (int64_t)ra * kHistStride);
  // slice counts -> list offsets (one slice per thread; nseg <= kMaxG)
  const uint32_t my_cnt = tid < nseg ? __ldcg(p.cnt + (int64_t)ra * G + cf + tid) : 0u;
  uint32_t Ctot;
  {
    // clamp: a slice never lists more entries than it holds
    uint32_t v = my_cnt;
    if (tid < nseg) {
      const int64_t a = slice_begin(tid, p.per_cta, N), b = slice_begin(tid + 1, p.per_cta, N);
      if ((int64_t)v > b - a) v = (uint32_t)(b - a);
    }
    const uint32_t e = block_excl_scan<kThreads>(v, ss.scratch, Ctot);
    if (tid < nseg) ss.pref[tid] = e;
    if (tid == 0) ss.pref[nseg] = Ctot;
  }
  __syncthreads();
  radix_threshold<kThreads, kBins1>(h2, (uint32_t)K, ss.scratch, ss.thr);
  const uint32_t t1 = ss.thr[0];
  const uint32_t r1 = (uint32_t)K - ss.thr[1];
  const bool in_smem = Ctot <= p.cap;
  // list entry i: slice s with pref[s] <= i < pref[s+1]
  auto seg_of = [&](uint32_t i) -> int {
    int lo = 0, hi = nseg - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (ss.pref[mid] <= i) lo = mid; else hi = mid - 1;
    }
    return lo;
  };
  auto from_global = [&](uint32_t i) -> uint2 {
    const int s = seg_of(i);
    const int64_t a = slice_begin(s, p.per_cta, N);
    return __ldcg(p.cand + (int64_t)ra * N + a + (i - ss.pref[s]));
  };
  if (in_smem) {  // 8 loads in flight per thread and round
    for (uint32_t i0 = tid; i0 < Ctot; i0 += 8 * kThreads) {
      uint2 v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const uint32_t i = min(i0 + u * kThreads, Ctot - 1);
        v[u] = from_global(i);
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const uint32_t i = i0 + u * kThreads;
        if (i < Ctot) clist[i] = v[u];
      }
    }
  }
  auto entry = [&](uint32_t i) -> uint2 { return in_smem ? clist[i] : from_global(i); };
  // digit 2 within bin t1
  __syncthreads();
  for (int i = tid; i < kBins2; i += kThreads) h2[i] = 0u;
  __syncthreads();
  for (uint32_t i = tid; i < Ctot; i += kThreads) {
    const uint32_t k = entry(i).x;
    if (key_d1(k) == t1) atomicAdd(&h2[key_d2(k)], 1u);
  }
  __syncthreads();
  radix_threshold<kThreads, kBins2>(h2, r1, ss.scratch, ss.thr + 2);
  const uint32_t t2 = ss.thr[2], r2 = r1 - ss.thr[3];
  const bool need3 = h2[t2] > r2;
  uint32_t t3 = 0, r3 = 0xffffffffu;
  if (need3) {  // uniform: every thread read the same histogram
    __syncthreads();
    for (int i = tid; i < kBins3; i += kThreads) h2[i] = 0u;
    __syncthreads();
    for (uint32_t i = tid; i < Ctot; i += kThreads) {
      const uint32_t k = entry(i).x;
      if (key_d1(k) == t1 && key_d2(k) == t2) atomicAdd(&h2[key_d3(k)], 1u);
    }
    __syncthreads();
    radix_threshold<kThreads, kBins3>(h2, r2, ss.scratch, ss.thr + 4);
    t3 = ss.thr[4];
    r3 = r2 - ss.thr[5];
  }
  // classify: thread t takes the contiguous list part [t*per, t*per + per);
  // one packed prefix of the (above, tie) counts gives each thread its
  // output offset; ties are taken in index order while their rank < r3
  const uint32_t per = (Ctot + kThreads - 1) / kThreads;
  const uint32_t i0 = min(Ctot, per * (uint32_t)tid), i1 = min(Ctot, i0 + per);
  uint32_t n_above = 0, n_tie = 0;
  for (uint32_t i = i0; i < i1; ++i) {
    const uint32_t cls = key_class(entry(i).x, t1, t2, t3, need3);
    n_above += (cls == 2u);
    n_tie += (cls == 1u);
  }
  uint32_t above_before, tie_before;
  if (Ctot < 65536u) {
    uint32_t tot;
    const uint32_t pre = block_excl_scan<kThreads>(n_above | (n_tie << 16), ss.scratch, tot);
    above_before = pre & 0xffffu;
    tie_before = pre >> 16;
  } else {
    uint32_t tot;
    above_before = block_excl_scan<kThreads>(n_above, ss.scratch, tot);
    tie_before = block_excl_scan<kThreads>(n_tie, ss.scratch, tot);
  }
  const uint32_t lo = (uint32_t)((K * j) / P), hi = (uint32_t)((K * (j + 1)) / P);
  int32_t *orow = p.idx + rg * (int64_t)p.topk;
  {
    uint32_t tie_rank = tie_before;
    uint32_t at = above_before + min(tie_before, r3);
    for (uint32_t i = i0; i < i1 && at < hi; ++i) {
      const uint2 e = entry(i);
      const uint32_t cls = key_class(e.x, t1, t2, t3, need3);
      bool take = cls == 2u;
      if (cls == 1u) take = tie_rank++ < r3;
      if (take) {
        if (at >= lo && at < hi) {
          orow[at] = (int32_t)e.y;
          if (at - lo < (uint32_t)kSelCap) ss.sel[at - lo] = (int32_t)e.y;
        }
        ++at;
      }
    }
  }
  if (j == P - 1)
    for (int64_t i = K + tid; i < p.topk; i += kThreads) orow[i] = -1;
  if (!p.do_attn) return;
  __syncthreads();  // sel complete; the list and histogram are dead

  // ------------------------------------------------------- attention --
  const int nh = min(kHeads, p.H);
  {
    constexpr int PPH = D / 8;
    for (int i = tid; i < kHeads * PPH; i += kThreads) {
      const int h = i / PPH, u = i % PPH;
      uint4 v = make_uint4(0u, 0u, 0u, 0u);
      if (h < nh) v = *reinterpret_cast<const uint4 *>(p.q + (rg * p.H + h) * (int64_t)D + 8 * u);
      *reinterpret_cast<uint4 *>(&ss.qb[h][8 * u]) = v;
    }
  }
  ar::WarpArea<D> *aw = reinterpret_cast<ar::WarpArea<D> *>(dsm);
  const int w_lo = (p.W * j) / P, w_hi = (p.W * (j + 1)) / P;
  const int nwin = w_hi - w_lo;
  const int64_t nsel = (int64_t)(hi - lo) < kSelCap ? (int64_t)(hi - lo) : kSelCap;
  const int64_t cw = (nwin + ar::kChunk - 1) / ar::kChunk;
  const int64_t ce = (nsel + ar::kChunk - 1) / ar::kChunk;
  const uint8_t *cseq = p.codes + rg * N * (D / 2);
  const float *sseq = p.scales + rg * N * (D / 16);
  const int64_t wrow0 = rg * (int64_t)p.W + w_lo;
  __syncthreads();
  if (warp < kAttnWarps) {
    ar::WarpArea<D> &wa = aw[warp];
    ar::WarpState<D> st;
    ar::state_init(st);
    const int64_t nch = cw + ce;
    auto entry_of = [&](int64_t ch) -> int32_t {
      const int64_t k = (ch - cw) * ar::kChunk + (lane & 15);
      return k < nsel ? ss.sel[k] : -1;
    };
    int64_t ech = warp;
    while (ech < cw) ech += kAttnWarps;
    uint32_t mask_cur = 0u;
    if (ech < nch) mask_cur = ar::gather_entries<D>(wa, 0, entry_of(ech), N, cseq, sseq);
    for (int64_t ch = warp; ch < cw; ch += kAttnWarps) {
      const int j0 = (int)ch * ar::kChunk;
      const uint32_t mask = ar::load_window_rows<D>(wa, p.win_k, p.win_v, wrow0 + j0,
                                                    min(ar::kChunk, nwin - j0));
      ar::attend_chunk16<D>(wa, ss.qb, st, mask, true, nullptr, p.q_scale);
      __syncwarp();
    }
    for (int it = 0; ech < nch; ++it, ech += kAttnWarps) {
      const int sb = it & 1;
      uint32_t mask_next = 0u;
      const bool more = ech + kAttnWarps < nch;
      if (more) mask_next = ar::gather_entries<D>(wa, sb ^ 1, entry_of(ech + kAttnWarps), N, cseq, sseq);
      if (more)
        ar::cp_wait<1>();
      else
        ar::cp_wait<0>();
      __syncwarp();
      ar::convert_entries<D>(wa, sb);
      __syncwarp();
      ar::attend_chunk16<D>(wa, ss.qb, st, mask_cur, false, wa.s.scales[sb], p.q_scale);
      __syncwarp();
      mask_cur = mask_next;
    }
    ar::store_state<D>(wa, st);
  }
  __syncthreads();
  // this CTA's partial per head: max over the warps, each warp's factor
  for (int i = tid; i < kHeads * kAttnWarps; i += kThreads) {
    const int h = i / kAttnWarps, w = i % kAttnWarps;
    float M = -INFINITY;
#pragma unroll
    for (int v = 0; v < kAttnWarps; ++v) M = fmaxf(M, aw[v].merge.m[h]);
    ss.mf[h][w] = M == -INFINITY ? 0.0f : exp2f(aw[w].merge.m[h] - M);
    if (w == 0) ss.mf[h][kAttnWarps] = M;
  }
  __syncthreads();
  constexpr int U = D / 4 + 1;  // 16-byte pieces per head: (m, l, -, -), acc
  float *mypart = p.part + (((int64_t)ra * P + j) * kHeads) * (D + 4);
  for (int i = tid; i < kHeads * U; i += kThreads) {
    const int h = i / U, q = i % U;
    float4 v = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    if (q == 0) {
#pragma unroll
      for (int w = 0; w < kAttnWarps; ++w) v.y = fmaf(aw[w].merge.l[h], ss.mf[h][w], v.y);
      v.x = ss.mf[h][kAttnWarps];
    } else {
#pragma unroll
      for (int w = 0; w < kAttnWarps; ++w) {
        const float4 o = *reinterpret_cast<const float4 *>(&aw[w].merge.o[h][4 * (q - 1)]);
        const float f = ss.mf[h][w];
        v.x = fmaf(o.x, f, v.x);
        v.y = fmaf(o.y, f, v.y);
        v.z = fmaf(o.z, f, v.z);
        v.w = fmaf(o.w, f, v.w);
      }
    }
    __stcg(reinterpret_cast<float4 *>(mypart + h * (D + 4) + 4 * q), v);
  }
  const uint32_t old = arrive_all(p.arrive + (int64_t)ra * kArrive + 2);
  if (tid == 0) ss.last = (old == (uint32_t)(P - 1)) ? 1u : 0u;
  __syncthreads();
  if (!ss.last) return;
  __threadfence();

  // ---------------------------------------------- merge (last CTA) --
  const float *rpart = p.part + ((int64_t)ra * P * kHeads) * (D + 4);
  if (warp < kHeads) {  // warp h: max over the P partials, their factors and the sum
    const int h = warp;
    float m = -INFINITY, l = 0.0f;
    if (lane < P) {
      const float2 ml = __ldcg(reinterpret_cast<const float2 *>(rpart + ((int64_t)lane * kHeads + h) * (D + 4)));
      m = ml.x;
      l = ml.y;
    }
    const float M = warp_max(l > 0.0f ? m : -INFINITY);
    const float f = (M != -INFINITY && l > 0.0f) ? exp2f(m - M) : 0.0f;
    const float L = warp_sum(l * f);
    if (lane < kMaxP) ss.fac[lane][h] = lane < P ? f : 0.0f;
    if (lane == 0) {
      ss.mrg_m[h] = M;
      ss.mrg_l[h] = L;
      if (p.lse && h < nh)
        p.lse[rg * p.H + h] = M == -INFINITY ? -INFINITY : (M + log2f(L)) * 0.69314718055994530942f;
    }
  }
  __syncthreads();
  // thread -> 4 consecutive dims of one head; the kMaxP partial loads are
  // issued together (slots past P read partial P-1 with factor 0)
  for (int i = tid; i < nh * (D / 4); i += kThreads) {
    const int h = i / (D / 4), e = 4 * (i % (D / 4));
    float4 v[kMaxP];
#pragma unroll
    for (int q = 0; q < kMaxP; ++q)
      v[q] = __ldcg(reinterpret_cast<const float4 *>(
          rpart + ((int64_t)min(q, P - 1) * kHeads + h) * (D + 4) + 4 + e));
    float4 a = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
#pragma unroll
    for (int q = 0; q < kMaxP; ++q) {
      if (q >= P) break;
      const float fq = ss.fac[q][h];
      a.x = fmaf(v[q].x, fq, a.x);
      a.y = fmaf(v[q].y, fq, a.y);
      a.z = fmaf(v[q].z, fq, a.z);
      a.w = fmaf(v[q].w, fq, a.w);
    }
    const bool none = ss.mrg_m[h] == -INFINITY;
    const float il = none ? 0.0f : 1.0f / ss.mrg_l[h];
    *reinterpret_cast<float4 *>(p.out + (rg * p.H + h) * (int64_t)D + e) =
        make_float4(a.x * il, a.y * il, a.z * il, a.w * il);
  }
}

}  // namespace fd
}  // namespace csa2

namespace csa2 {
namespace fd {

// Self-test of the bounded waits: an mbarrier phase that never completes
// (two arrivals expected, one made) and a global counter that nothing
// raises, each waited on with a short limit.  Both waits must give up,
// record kStatusWaitTimeout in the status word and return; the kernel then
// ends normally.  One thread.
__device__ uint32_t g_never_raised;  // zero-initialised, never written

__global__ void wait_timeout_selftest_kernel(long long limit) {
  __shared__ uint64_t bar;
  if (threadIdx.x != 0) return;
  mbar_init(&bar, 2);
  fence_barrier_init();
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(&bar)) : "memory");
  mbar_wait_bounded(&bar, 0, limit);
  wait_count(&g_never_raised, 1u, limit);
}

}  // namespace fd
}  // namespace csa2
