// Indexer scan: score every visible entry of a query row.
//
// "Why Is DeepSeek V4.1 Flash So Fast?", section 4 ("The indexer"): index
// heads run a cheap relevance search over all compressed positions.  Score
// of entry n for query row r (this library's reading):
//   dot_h = sum_i q_idx[r, h, i] * k_idx[b, n, i]        exact int32 (dp4a)
//   score = ((0 + w_0 * dot_0) + w_1 * dot_1) + ... + 0   fp32, each op rounded
//
// Data movement.  The scan is HBM-bound (d_I bytes per entry, a few hundred
// integer ops), so it streams keys, it does not reshape them into a GEMM.
// Each CTA owns a contiguous slice of one row's entries and pulls it through
// a STAGES-deep ring of shared-memory tiles with 1-D bulk copies
// (cp.async.bulk, completion counted on an mbarrier); one elected thread
// issues the copies, so loads cost no per-thread address arithmetic.  Each
// thread scores whole keys from shared memory.  A key is d_I/16 chunks of 16
// bytes; thread t reads chunk c ^ x(t) at step c, with x(t) chosen so the 8
// threads of a 128-byte shared-memory phase hit 8 different 16-byte bank
// groups, and holds its index-query chunks pre-permuted the same way, so the
// dot product needs no data-dependent register indexing.  The score's top
// radix digit goes to a shared-memory histogram, merged into the row's
// global histogram at the end for the top-k selection.
#pragma once
#include "common.cuh"
#include "pack.cuh"

namespace csa2 {

constexpr int kScanThreads = 256;
// Words per row of the digit-1 histogram region: the 2,048 bins, then (for
// a selection handed to a following attention kernel) one ready flag per
// selecting CTA and a done counter of the row's attention CTAs, all cleared
// with the bins before each scan.
constexpr int kHandoffFlags = 16;  // selecting CTAs per row, at most
constexpr int kHistStride = kBins1 + 32;

// Index key formats: int8, or FP4 (E2M1 codes with one power-of-two scale
// per 32 elements: d_I/2 code bytes + d_I/32 exponent bytes per key, see
// pack.cuh).
constexpr int kScanKeysInt8 = 0, kScanKeysFp4 = 1;

template <int DI, int HI, int KF = kScanKeysInt8>
struct ScanShape {
  static constexpr bool FP4 = KF == kScanKeysFp4;
  static constexpr int NCH = FP4 ? DI / 32 : DI / 16;     // 16-byte chunks (FP4: blocks) per key
  static constexpr int CB = FP4 ? DI / 2 : DI;            // key bytes in the tile
  static constexpr int EB = FP4 ? DI / 32 : 0;            // exponent bytes per key
  static constexpr int KPT = FP4 ? 512 / DI : ((DI >= 64) ? 1 : 64 / DI);  // keys per thread per tile
  static constexpr int TILE_KEYS = kScanThreads * KPT;
  static constexpr int TILE_BYTES = TILE_KEYS * (CB + EB); // 16 KiB int8 (32 KiB for d_I = 128); 17-18 KiB FP4
  static constexpr int STAGES = (TILE_BYTES > 20000) ? 3 : 4;
  static constexpr int QW = FP4 ? 2 : 1;                  // query int4 per chunk
  static constexpr bool QREG = HI * NCH * QW <= 16;       // index query fits in registers
  static constexpr size_t SMEM = size_t(STAGES) * TILE_BYTES;
  static_assert(DI % 16 == 0 && NCH >= 1 && NCH <= 8, "d_I in {16,32,64,128}");
  static_assert(!FP4 || (DI % 32 == 0 && QREG), "FP4 keys: d_I % 32 == 0, query in registers");
};

// Rotation of the chunk order of thread t (see the header comment).
template <int NCH>
__device__ __forceinline__ int chunk_xor(int t) {
  return (NCH == 1) ? 0 : (t / (8 / NCH)) % NCH;
}

// Block maxima taken by the scan itself (a Full layer's candidate pool, see
// pool.cuh): per row, the largest score of every `block` consecutive
// positions (block a power of two <= 16, so a block's keys sit on
// consecutive lanes of one warp and never cross a slice or a tile) into
// bscores [rows, bstride], and their digit-1 histogram into bhist [rows,
// kHistStride] (zeroed).
struct ScanBlockMax {
  float *bscores;
  int64_t bstride;
  uint32_t *bhist;
  int32_t block;
};

// grid = (G slices, rows).  hist1: [rows][kHistStride], zeroed.  With FP4
// keys, k_idx holds the codes [B, N, d_I/2] and k_exps the exponents [B, N,
// d_I/32] (N % 16 == 0, so every copy starts on a 16-byte boundary).  BM:
// also the block maxima of `bm` (int8 keys).
template <int DI, int HI, int KF = kScanKeysInt8, bool BM = false>
__global__ void __launch_bounds__(kScanThreads, 2)
    index_scan_kernel(const int8_t *__restrict__ q_idx, const float *__restrict__ w,
                      const int8_t *__restrict__ k_idx, const uint8_t *__restrict__ k_exps,
                      int32_t T, int64_t N, int64_t n_prior, int32_t ratio, int64_t row0,
                      float *__restrict__ scores, int64_t score_stride,
                      uint32_t *__restrict__ hist1, int write_masked, const ScanBlockMax bm) {
  using S = ScanShape<DI, HI, KF>;
  constexpr int NCH = S::NCH, STAGES = S::STAGES, TK = S::TILE_KEYS, QW = S::QW;
  static_assert(!BM || KF == kScanKeysInt8, "block maxima with int8 keys");
  const int bshift = BM ? __ffs(bm.block) - 1 : 0;
  extern __shared__ __align__(128) unsigned char smem_tiles[];
  __shared__ uint64_t full_bar[STAGES];
  __shared__ uint32_t sh_hist[kBins1];
  __shared__ uint32_t sh_bhist[BM ? kBins1 : 1];
  __shared__ __align__(16) int4 sh_q[S::QREG ? 1 : HI * NCH * QW];

  const int tid = threadIdx.x;
  const int64_t r_local = blockIdx.y, r = row0 + r_local;
  const int64_t b = r / T, t = r % T;
  const int G = gridDim.x, g = blockIdx.x;

  int64_t V = N;
  if (n_prior >= 0) {
    V = n_prior + (t + 1) / ratio;
    if (V > N) V = N;
  }
  // Slice [n0, n1) of [0, V); inner boundaries on multiples of 16 keys.
  const int64_t n0 = ((V * g) / G) & ~int64_t(15);
  const int64_t n1 = (g == G - 1) ? V : (((V * (g + 1)) / G) & ~int64_t(15));
  const int ntiles = (int)((n1 - n0 + TK - 1) / TK);
  // tile t: keys [n0 + t*TK, ...) -> its stage (codes, then FP4 exponents)
  auto issue = [&](int t, int stage) {
    const int64_t keys = min64(TK, n1 - n0 - (int64_t)t * TK);
    const int64_t key0 = b * N + n0 + (int64_t)t * TK;
    unsigned char *dst = smem_tiles + stage * S::TILE_BYTES;
    const uint32_t cb = (uint32_t)(keys * S::CB), eb = (uint32_t)(keys * S::EB);
    mbar_arrive_expect_tx(&full_bar[stage], cb + eb);
    bulk_g2s(dst, k_idx + key0 * S::CB, cb, &full_bar[stage]);
    if constexpr (S::FP4) bulk_g2s(dst + TK * S::CB, k_exps + key0 * S::EB, eb, &full_bar[stage]);
  };

  // The per-row selection kernel that follows may be scheduled now; it waits
  // for this grid's results before reading them.
  pdl_allow_dependents();
  for (int i = tid; i < kBins1; i += kScanThreads) sh_hist[i] = 0u;
  if constexpr (BM)
    for (int i = tid; i < kBins1; i += kScanThreads) sh_bhist[i] = 0u;
  if (tid == 0) {
    for (int s = 0; s < STAGES; ++s) mbar_init(&full_bar[s], 1);
    fence_barrier_init();
  }
  __syncthreads();
  if (tid == 0)
    for (int s = 0; s < STAGES && s < ntiles; ++s) issue(s, s);

  // This thread's index-query chunks, pre-permuted by its chunk rotation.
  const int x = chunk_xor<NCH>(tid);
  int4 qreg[S::QREG ? HI * NCH * QW : 1];
  const int4 *qrow = reinterpret_cast<const int4 *>(q_idx + r * HI * DI);
  if constexpr (S::QREG) {
#pragma unroll
    for (int h = 0; h < HI; ++h)
#pragma unroll
      for (int c = 0; c < NCH; ++c)
#pragma unroll
        for (int u = 0; u < QW; ++u) qreg[(h * NCH + c) * QW + u] = qrow[(h * NCH + (c ^ x)) * QW + u];
  } else {
    for (int i = tid; i < HI * NCH * QW; i += kScanThreads) sh_q[i] = qrow[i];
  }
  float wh[HI];
#pragma unroll
  for (int h = 0; h < HI; ++h) wh[h] = w[r * HI + h];
  if constexpr (!S::QREG) __syncthreads();

  float *srow = scores + r_local * score_stride;
  int abort_it = -1;
  for (int it = 0; it < ntiles; ++it) {
    const int s = it % STAGES;
    const bool ok = mbar_wait_bounded(&full_bar[s], (uint32_t)(it / STAGES) & 1u);
    // One barrier per tile: uniform abort decision, and every thread is done
    // with tile it-1, so its stage can be refilled with tile it-1+STAGES.
    if (__syncthreads_or(!ok)) {
      abort_it = it;
      break;
    }
    if (tid == 0 && it >= 1 && it - 1 + STAGES < ntiles) {
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      issue(it - 1 + STAGES, (it - 1) % STAGES);
    }
    const unsigned char *tile = smem_tiles + s * S::TILE_BYTES;
    const int64_t tbase = n0 + (int64_t)it * TK;
    const int tkeys = (int)min64(TK, n1 - tbase);
#pragma unroll
    for (int j = 0; j < S::KPT; ++j) {
      const int kl = tid + j * kScanThreads;
      const bool valid = kl < tkeys;
      float score = 0.0f;
      if constexpr (S::FP4) {
        if (valid) {
          score = fp4_key_score<NCH, HI, S::QREG>(tile + kl * S::CB,
                                                  tile + TK * S::CB + kl * S::EB, qreg, sh_q, wh, x);
          srow[tbase + kl] = score;
        }
      } else if (valid) {
        const unsigned char *krow = tile + kl * DI;
        int dot[HI];
#pragma unroll
        for (int h = 0; h < HI; ++h) dot[h] = 0;
#pragma unroll
        for (int c = 0; c < NCH; ++c) {
          const int4 kv = *reinterpret_cast<const int4 *>(krow + ((c ^ x) << 4));
#pragma unroll
          for (int h = 0; h < HI; ++h) {
            int4 qv;
            if constexpr (S::QREG)
              qv = qreg[h * NCH + c];
            else
              qv = sh_q[h * NCH + (c ^ x)];
            dot[h] = __dp4a(kv.x, qv.x, dot[h]);
            dot[h] = __dp4a(kv.y, qv.y, dot[h]);
            dot[h] = __dp4a(kv.z, qv.z, dot[h]);
            dot[h] = __dp4a(kv.w, qv.w, dot[h]);
          }
        }
        float acc = 0.0f;
#pragma unroll
        for (int h = 0; h < HI; ++h) acc = __fadd_rn(acc, __fmul_rn(wh[h], __int2float_rn(dot[h])));
        score = __fadd_rn(acc, 0.0f);
        srow[tbase + kl] = score;
      }
      // plain shared-memory reduction (a warp-aggregating match costs more
      // on its narrow issue pipe than the bin conflicts it saves)
      if (valid) atomicAdd(&sh_hist[key_d1(score_key(score))], 1u);
      if constexpr (BM) {  // the block's largest score, by its first lane
        float m = valid ? score : -__int_as_float(0x7f800000);
#pragma unroll
        for (int o = 1; o < 16; o <<= 1)
          if (o < bm.block) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        if (valid && (kl & (bm.block - 1)) == 0) {
          bm.bscores[r_local * bm.bstride + ((tbase + kl) >> bshift)] = m;
          atomicAdd(&sh_bhist[key_d1(score_key(m))], 1u);
        }
      }
    }
  }
  if (abort_it >= 0) {
    // Drain the copies this CTA issued (tiles [0, upto)) before exiting.
    if (tid == 0) {
      const int upto = min(ntiles, max(abort_it - 1, 0) + STAGES);
      for (int k = 0; k < STAGES && k < upto; ++k) {
        const int last = k + ((upto - 1 - k) / STAGES) * STAGES;  // last tile issued into stage k
        mbar_wait_bounded(&full_bar[k], (uint32_t)(last / STAGES) & 1u);
      }
    }
    __syncthreads();
    return;
  }

  // Entries the row may not see (prefill): -inf when scores are requested.
  if (write_masked && V < N) {
    const int64_t m0 = V + ((N - V) * g) / G, m1 = V + ((N - V) * (g + 1)) / G;
    for (int64_t n = m0 + tid; n < m1; n += kScanThreads) srow[n] = -__int_as_float(0x7f800000);
  }

  __syncthreads();
  uint32_t *grow = hist1 + r_local * kHistStride;
  for (int i = tid; i < kBins1; i += kScanThreads) {
    const uint32_t v = sh_hist[i];
    if (v) atomicAdd(grow + i, v);
  }
  if constexpr (BM) {
    uint32_t *brow = bm.bhist + r_local * kHistStride;
    for (int i = tid; i < kBins1; i += kScanThreads) {
      const uint32_t v = sh_bhist[i];
      if (v) atomicAdd(brow + i, v);
    }
  }
}

}  // namespace csa2

namespace csa2 {

// ---------------------------------------------------------------------------
// Several queries of one sequence (multi-token decode, e.g. a few draft
// tokens verified together): the CTAs of a sequence stream its keys once and
// score every query row of the sequence against each key, so the key bytes
// per token fall by the number of rows.  Two warps per query row: warp 2t+i
// scores half of every key tile against row t, with the row's index query in
// registers (pre-permuted by the lane's chunk rotation, as above), so shared
// memory serves only key chunks.  Same score, histogram and slice rules as
// index_scan_kernel; row t sees n < V_t.
// grid = (G slices, sequences of the pass); block = 64 * TQ threads; rows of
// sequence b are b*T .. b*T + T - 1 (T <= TQ); hist1 rows per query row.
// ---------------------------------------------------------------------------
template <int DI, int HI, int TQ>
struct ScanGroupShape {
  static_assert(DI <= 64, "16 KiB key tiles");
  static constexpr int THREADS = 64 * TQ;
  static constexpr int NCH = DI / 16;
  static constexpr int TILE_KEYS = 16384 / DI;            // 16 KiB tiles
  static constexpr int TILE_BYTES = 16384;
  static constexpr int KPL = TILE_KEYS / 64;              // keys per lane and tile
  static constexpr int STAGES = 4;
  static constexpr bool QREG = HI * NCH <= 16;            // index query fits in registers
  static constexpr size_t HIST_BYTES = size_t(TQ) * kBins1 * 4;
  static constexpr size_t SMEM = size_t(STAGES) * TILE_BYTES + HIST_BYTES;
};

template <int DI, int HI, int TQ>
__global__ void __launch_bounds__(64 * TQ, TQ <= 4 ? 2 : 1)
    index_scan_group_kernel(const int8_t *__restrict__ q_idx, const float *__restrict__ w,
                            const int8_t *__restrict__ k_idx, int32_t T, int64_t N,
                            int64_t n_prior, int32_t ratio, int64_t row0,
                            float *__restrict__ scores, int64_t score_stride,
                            uint32_t *__restrict__ hist1, int write_masked) {
  using S = ScanGroupShape<DI, HI, TQ>;
  constexpr int NCH = S::NCH, STAGES = S::STAGES, TK = S::TILE_KEYS, THREADS = S::THREADS;
  extern __shared__ __align__(128) unsigned char smem_tiles[];
  uint32_t *sh_hist = reinterpret_cast<uint32_t *>(smem_tiles + STAGES * S::TILE_BYTES);
  __shared__ uint64_t full_bar[STAGES];
  __shared__ __align__(16) int4 sh_q[S::QREG ? 1 : TQ][S::QREG ? 1 : HI * NCH];

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int t = warp >> 1;          // this warp's query row within the sequence
  const int half = warp & 1;        // and its half of every key tile
  const bool row_live = t < T;
  const int64_t gl = blockIdx.y;    // sequence within the pass
  const int64_t rl0 = gl * T;       // its first row within the pass
  const int64_t b = (row0 + rl0) / T;
  const int G = gridDim.x, g = blockIdx.x;

  int64_t V = N;   // the group's largest visible count (visibility grows with t)
  int64_t Vt = N;  // this warp's row
  if (n_prior >= 0) {
    V = n_prior + (int64_t)T / ratio;
    if (V > N) V = N;
    Vt = n_prior + (int64_t)(t + 1) / ratio;
    if (Vt > N) Vt = N;
  }
  const int64_t n0 = ((V * g) / G) & ~int64_t(15);
  const int64_t n1 = (g == G - 1) ? V : (((V * (g + 1)) / G) & ~int64_t(15));
  const int ntiles = (int)((n1 - n0 + TK - 1) / TK);
  const int8_t *src = k_idx + (b * N + n0) * DI;

  pdl_allow_dependents();
  for (int i = tid; i < TQ * kBins1; i += THREADS) sh_hist[i] = 0u;
  if (tid == 0) {
    for (int s = 0; s < STAGES; ++s) mbar_init(&full_bar[s], 1);
    fence_barrier_init();
  }
  // this row's index query (registers, pre-permuted; or shared memory) and weights
  const int x = chunk_xor<NCH>(lane);
  const int64_t r = b * T + (row_live ? t : 0);
  int4 qreg[S::QREG ? HI * NCH : 1];
  const int4 *qrow = reinterpret_cast<const int4 *>(q_idx + r * HI * DI);
  if constexpr (S::QREG) {
#pragma unroll
    for (int h = 0; h < HI; ++h)
#pragma unroll
      for (int c = 0; c < NCH; ++c) qreg[h * NCH + c] = qrow[h * NCH + (c ^ x)];
  } else {
    for (int i = tid; i < TQ * HI * NCH; i += THREADS) {
      const int tt = i / (HI * NCH), j = i % (HI * NCH);
      sh_q[tt][j] = (tt < T) ? reinterpret_cast<const int4 *>(q_idx + (b * T + tt) * HI * DI)[j]
                             : make_int4(0, 0, 0, 0);
    }
  }
  float wh[HI];
#pragma unroll
  for (int h = 0; h < HI; ++h) wh[h] = w[r * HI + h];
  __syncthreads();
  if (tid == 0) {
    for (int s = 0; s < STAGES && s < ntiles; ++s) {
      const int64_t keys = min64(TK, n1 - n0 - (int64_t)s * TK);
      const uint32_t bytes = (uint32_t)(keys * DI);
      mbar_arrive_expect_tx(&full_bar[s], bytes);
      bulk_g2s(smem_tiles + s * S::TILE_BYTES, src + (int64_t)s * TK * DI, bytes, &full_bar[s]);
    }
  }

  float *srow = scores + (rl0 + (row_live ? t : 0)) * score_stride;
  uint32_t *hrow = sh_hist + (row_live ? t : 0) * kBins1;
  int abort_it = -1;
  for (int it = 0; it < ntiles; ++it) {
    const int s = it % STAGES;
    const bool ok = mbar_wait_bounded(&full_bar[s], (uint32_t)(it / STAGES) & 1u);
    if (__syncthreads_or(!ok)) {
      abort_it = it;
      break;
    }
    if (tid == 0 && it >= 1 && it - 1 + STAGES < ntiles) {
      const int nt = it - 1 + STAGES, ps = (it - 1) % STAGES;
      const int64_t keys = min64(TK, n1 - n0 - (int64_t)nt * TK);
      const uint32_t bytes = (uint32_t)(keys * DI);
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      mbar_arrive_expect_tx(&full_bar[ps], bytes);
      bulk_g2s(smem_tiles + ps * S::TILE_BYTES, src + (int64_t)nt * TK * DI, bytes,
               &full_bar[ps]);
    }
    if (!row_live) continue;  // warp-uniform; the warp still takes every barrier
    const unsigned char *tile = smem_tiles + s * S::TILE_BYTES;
    const int64_t tbase = n0 + (int64_t)it * TK;
    const int tkeys = (int)min64(TK, n1 - tbase);
#pragma unroll
    for (int j = 0; j < S::KPL; ++j) {
      const int kl = half * (TK / 2) + j * 32 + lane;
      const int64_t n = tbase + kl;
      const bool vis = kl < tkeys && n < Vt;
      float score = 0.0f;
      if (vis) {
        const unsigned char *krow = tile + kl * DI;
        int dot[HI];
#pragma unroll
        for (int h = 0; h < HI; ++h) dot[h] = 0;
#pragma unroll
        for (int c = 0; c < NCH; ++c) {
          const int4 kv = *reinterpret_cast<const int4 *>(krow + ((c ^ x) << 4));
#pragma unroll
          for (int h = 0; h < HI; ++h) {
            int4 qv;
            if constexpr (S::QREG)
              qv = qreg[h * NCH + c];
            else
              qv = sh_q[t][h * NCH + (c ^ x)];
            dot[h] = __dp4a(kv.x, qv.x, dot[h]);
            dot[h] = __dp4a(kv.y, qv.y, dot[h]);
            dot[h] = __dp4a(kv.z, qv.z, dot[h]);
            dot[h] = __dp4a(kv.w, qv.w, dot[h]);
          }
        }
        float acc = 0.0f;
#pragma unroll
        for (int h = 0; h < HI; ++h) acc = __fadd_rn(acc, __fmul_rn(wh[h], __int2float_rn(dot[h])));
        score = __fadd_rn(acc, 0.0f);
        srow[n] = score;
        // plain shared-memory reduction: with a few rows per key the
        // warp-aggregation of the single-row scan (match) would bound the
        // kernel on its narrow issue pipe
        atomicAdd(&hrow[key_d1(score_key(score))], 1u);
      }
    }
  }
  if (abort_it >= 0) {
    if (tid == 0) {
      const int upto = min(ntiles, max(abort_it - 1, 0) + STAGES);
      for (int k = 0; k < STAGES && k < upto; ++k) {
        const int last = k + ((upto - 1 - k) / STAGES) * STAGES;
        mbar_wait_bounded(&full_bar[k], (uint32_t)(last / STAGES) & 1u);
      }
    }
    __syncthreads();
    return;
  }
  // entries a row may not see: -inf when scores are requested
  if (write_masked && row_live && Vt < N) {
    const int64_t m0 = Vt + ((N - Vt) * g) / G, m1 = Vt + ((N - Vt) * (g + 1)) / G;
    for (int64_t n = m0 + half * 32 + lane; n < m1; n += 64) srow[n] = -__int_as_float(0x7f800000);
  }
  __syncthreads();
  for (int tt = 0; tt < T && tt < TQ; ++tt) {
    uint32_t *grow = hist1 + (rl0 + tt) * kHistStride;
    for (int i = tid; i < kBins1; i += THREADS) {
      const uint32_t v = sh_hist[tt * kBins1 + i];
      if (v) atomicAdd(grow + i, v);
    }
  }
}

}  // namespace csa2

namespace csa2 {

// ---------------------------------------------------------------------------
// Multi-token scan on tensor cores (4 index heads, d_I in {32, 64}).
//
// With T query tokens per sequence the index dots of one key against all
// 4T query heads are a small exact integer contraction, so each warp takes
// 16 keys of the tile at a time as the rows of an int8 mma.sync m16n8k32
// (A = 16 keys x 32 bytes, ldmatrix from the staged tile; B = 8 query heads,
// i.e. 2 tokens, held in registers; int32 accumulators, exact) instead of
// the dp4a chains of index_scan_group_kernel.  In the accumulator a lane
// holds heads 2(tig&1), +1 of token 2u + tig/2 for keys gid and gid + 8; one
// exchange with lane ^ 1 gives each lane all 4 heads of one key (the even
// lane key gid, the odd lane key gid + 8), whose score it forms in the same
// fixed fp32 order as the other scans.  Keys stream through the same bulk-
// copy ring; slices, visibility, histograms and scores as
// index_scan_group_kernel.
// grid = (G slices, sequences of the pass); 256 threads; dynamic shared
// memory STAGES * 16 KiB + T * kBins1 * 4 (the per-token histograms).
// ---------------------------------------------------------------------------
template <int DI, int TQ>
struct ScanMmaShape {
  static_assert(DI == 32 || DI == 64, "d_I in {32, 64}");
  static constexpr int HI = 4;
  static constexpr int KS = DI / 32;             // k-steps of 32 bytes
  static constexpr int NT = (TQ * HI + 7) / 8;   // n-tiles of 8 query heads (2 tokens)
  static constexpr int THREADS = 256;
  static constexpr int TILE_BYTES = 16384;
  static constexpr int TILE_KEYS = TILE_BYTES / DI;
  static constexpr int SUB = TILE_KEYS / 16;     // 16-key row blocks per tile
  static constexpr int STAGES = 4;
  static size_t smem(int T) { return size_t(STAGES) * TILE_BYTES + size_t(T) * kBins1 * 4; }
};

__device__ __forceinline__ void mma_s8_16832(int (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                             uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

template <int DI, int TQ>
__global__ void __launch_bounds__(256, 2)
    index_scan_mma_kernel(const int8_t *__restrict__ q_idx, const float *__restrict__ w,
                          const int8_t *__restrict__ k_idx, int32_t T, int64_t N,
                          int64_t n_prior, int32_t ratio, int64_t row0,
                          float *__restrict__ scores, int64_t score_stride,
                          uint32_t *__restrict__ hist1, int write_masked) {
  using S = ScanMmaShape<DI, TQ>;
  constexpr int STAGES = S::STAGES, TK = S::TILE_KEYS, NT = S::NT, KS = S::KS;
  extern __shared__ __align__(128) unsigned char smem_tiles[];
  uint32_t *sh_hist = reinterpret_cast<uint32_t *>(smem_tiles + STAGES * S::TILE_BYTES);
  __shared__ uint64_t full_bar[STAGES];

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int gid = lane >> 2, tig = lane & 3;
  const bool odd = tig & 1;
  const int64_t gl = blockIdx.y;    // sequence within the pass
  const int64_t rl0 = gl * T;       // its first row within the pass
  const int64_t b = (row0 + rl0) / T;
  const int G = gridDim.x, g = blockIdx.x;

  int64_t V = N;  // the group's largest visible count (visibility grows with t)
  if (n_prior >= 0) {
    V = n_prior + (int64_t)T / ratio;
    if (V > N) V = N;
  }
  const int64_t n0 = ((V * g) / G) & ~int64_t(15);
  const int64_t n1 = (g == G - 1) ? V : (((V * (g + 1)) / G) & ~int64_t(15));
  const int ntiles = (int)((n1 - n0 + TK - 1) / TK);
  const int8_t *src = k_idx + (b * N + n0) * DI;

  pdl_allow_dependents();
  for (int i = tid; i < T * kBins1; i += S::THREADS) sh_hist[i] = 0u;
  if (tid == 0) {
    for (int s = 0; s < STAGES; ++s) mbar_init(&full_bar[s], 1);
    fence_barrier_init();
  }
  // B fragments: query head j = 8u + gid (token j / 4, head j % 4), bytes
  // [32k + 4 tig, +4) and [32k + 16 + 4 tig, +4); zero past the last token
  uint32_t bq[NT][KS][2];
#pragma unroll
  for (int u = 0; u < NT; ++u) {
    const int j = 8 * u + gid, tq = j >> 2;
    const int8_t *qr = q_idx + ((b * T + (tq < T ? tq : 0)) * 4 + (j & 3)) * (int64_t)DI;
#pragma unroll
    for (int k = 0; k < KS; ++k) {
      bq[u][k][0] = tq < T ? *reinterpret_cast<const uint32_t *>(qr + 32 * k + 4 * tig) : 0u;
      bq[u][k][1] = tq < T ? *reinterpret_cast<const uint32_t *>(qr + 32 * k + 16 + 4 * tig) : 0u;
    }
  }
  // this lane's token in n-tile u: its weights, visible count (0 past the
  // last token), score row and histogram
  float wt[NT][4];
  int64_t vq[NT];
  float *srow[NT];
  uint32_t *hrow[NT];
#pragma unroll
  for (int u = 0; u < NT; ++u) {
    const int tq = 2 * u + (tig >> 1);
    const int tc = tq < T ? tq : 0;
#pragma unroll
    for (int h = 0; h < 4; ++h) wt[u][h] = tq < T ? w[(b * T + tq) * 4 + h] : 0.0f;
    int64_t v = tq < T ? N : 0;
    if (n_prior >= 0 && tq < T) {
      v = n_prior + (int64_t)(tq + 1) / ratio;
      if (v > N) v = N;
    }
    vq[u] = v;
    srow[u] = scores + (rl0 + tc) * score_stride;
    hrow[u] = sh_hist + tc * kBins1;
  }
  __syncthreads();
  if (tid == 0) {
    for (int s = 0; s < STAGES && s < ntiles; ++s) {
      const int64_t keys = min64(TK, n1 - n0 - (int64_t)s * TK);
      const uint32_t bytes = (uint32_t)(keys * DI);
      mbar_arrive_expect_tx(&full_bar[s], bytes);
      bulk_g2s(smem_tiles + s * S::TILE_BYTES, src + (int64_t)s * TK * DI, bytes, &full_bar[s]);
    }
  }

  int abort_it = -1;
  for (int it = 0; it < ntiles; ++it) {
    const int s = it % STAGES;
    const bool ok = mbar_wait_bounded(&full_bar[s], (uint32_t)(it / STAGES) & 1u);
    if (__syncthreads_or(!ok)) {
      abort_it = it;
      break;
    }
    if (tid == 0 && it >= 1 && it - 1 + STAGES < ntiles) {
      const int nt = it - 1 + STAGES, ps = (it - 1) % STAGES;
      const int64_t keys = min64(TK, n1 - n0 - (int64_t)nt * TK);
      const uint32_t bytes = (uint32_t)(keys * DI);
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      mbar_arrive_expect_tx(&full_bar[ps], bytes);
      bulk_g2s(smem_tiles + ps * S::TILE_BYTES, src + (int64_t)nt * TK * DI, bytes,
               &full_bar[ps]);
    }
    const unsigned char *tile = smem_tiles + s * S::TILE_BYTES;
    const int64_t tbase = n0 + (int64_t)it * TK;
    const int tkeys = (int)min64(TK, n1 - tbase);
    // per n-tile: this lane's keys of the tile that its token sees
    int lim[NT];
    float *sp[NT];
#pragma unroll
    for (int u = 0; u < NT; ++u) {
      const int64_t rem = vq[u] - tbase;
      lim[u] = (int)min64(tkeys, rem > 0 ? rem : 0);
      sp[u] = srow[u] + tbase;
    }
#pragma unroll
    for (int i = 0; i < S::SUB / (S::THREADS / 32); ++i) {
      const int kb = (warp + i * (S::THREADS / 32)) * 16;  // first key of these 16 in the tile
      if (kb >= tkeys) break;                              // warp-uniform
      // A fragments (keys kb..kb+15 x 32 bytes per k-step): matrix m = lane / 8
      // of ldmatrix.x4 holds rows (m & 1) * 8 + 0..7, bytes (m >> 1) * 16 + 0..15
      uint32_t a[KS][4];
      const unsigned char *arow = tile + (kb + (lane & 7) + ((lane >> 3) & 1) * 8) * DI + (lane >> 4) * 16;
#pragma unroll
      for (int k = 0; k < KS; ++k)
        asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                     : "=r"(a[k][0]), "=r"(a[k][1]), "=r"(a[k][2]), "=r"(a[k][3])
                     : "r"(smem_u32(arow + 32 * k)));
      const int kk = kb + gid + (odd ? 8 : 0);  // this lane's key in the tile
#pragma unroll
      for (int u = 0; u < NT; ++u) {
        int c[4] = {0, 0, 0, 0};
#pragma unroll
        for (int k = 0; k < KS; ++k) mma_s8_16832(c, a[k], bq[u][k][0], bq[u][k][1]);
        // even lane: key gid, its heads 0,1 + the partner's heads 2,3 of key
        // gid; odd lane: key gid + 8, the partner's heads 0,1 + its 2,3
        const int x0 = __shfl_xor_sync(0xffffffffu, odd ? c[0] : c[2], 1);
        const int x1 = __shfl_xor_sync(0xffffffffu, odd ? c[1] : c[3], 1);
        const int d0 = odd ? x0 : c[0], d1 = odd ? x1 : c[1];
        const int d2 = odd ? c[2] : x0, d3 = odd ? c[3] : x1;
        if (kk < lim[u]) {
          float acc = 0.0f;
          acc = __fadd_rn(acc, __fmul_rn(wt[u][0], __int2float_rn(d0)));
          acc = __fadd_rn(acc, __fmul_rn(wt[u][1], __int2float_rn(d1)));
          acc = __fadd_rn(acc, __fmul_rn(wt[u][2], __int2float_rn(d2)));
          acc = __fadd_rn(acc, __fmul_rn(wt[u][3], __int2float_rn(d3)));
          const float score = __fadd_rn(acc, 0.0f);
          sp[u][kk] = score;
          atomicAdd(&hrow[u][key_d1(score_key(score))], 1u);
        }
      }
    }
  }
  if (abort_it >= 0) {
    if (tid == 0) {
      const int upto = min(ntiles, max(abort_it - 1, 0) + STAGES);
      for (int k = 0; k < STAGES && k < upto; ++k) {
        const int last = k + ((upto - 1 - k) / STAGES) * STAGES;
        mbar_wait_bounded(&full_bar[k], (uint32_t)(last / STAGES) & 1u);
      }
    }
    __syncthreads();
    return;
  }
  // entries a row may not see: -inf when scores are requested
  if (write_masked && n_prior >= 0) {
    for (int tt = 0; tt < T; ++tt) {
      int64_t Vt = n_prior + (int64_t)(tt + 1) / ratio;
      if (Vt > N) Vt = N;
      const int64_t m0 = Vt + ((N - Vt) * g) / G, m1 = Vt + ((N - Vt) * (g + 1)) / G;
      float *srow = scores + (rl0 + tt) * score_stride;
      for (int64_t m = m0 + tid; m < m1; m += S::THREADS) srow[m] = -__int_as_float(0x7f800000);
    }
  }
  __syncthreads();
  for (int tt = 0; tt < T; ++tt) {
    uint32_t *grow = hist1 + (rl0 + tt) * kHistStride;
    for (int i = tid; i < kBins1; i += S::THREADS) {
      const uint32_t v = sh_hist[tt * kBins1 + i];
      if (v) atomicAdd(grow + i, v);
    }
  }
}

}  // namespace csa2
