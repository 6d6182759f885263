// Indexer scan (decode and small-T queries): score every visible entry.
//
// "Why Is DeepSeek V4.1 Flash So Fast?", section 4 ("The indexer"): index
// heads run a cheap relevance search over all compressed positions.  Score
// of entry n for query row r (this library's reading):
//   dot_h = sum_i q_idx[r, h, i] * k_idx[b, n, i]        exact int32 (dp4a)
//   score = ((0 + w_0 * dot_0) + w_1 * dot_1) + ... + 0   fp32, each op rounded
//
// Layout and data movement.  Keys are int8 [B, N, d_I]; a key is d_I/16
// 16-byte chunks.  Each warp load instruction reads 512 contiguous bytes
// (lane l: bytes 16l .. 16l+15), so the lanes of one key hold its chunks.
// A warp issues NCH loads (NCH = d_I/16) per 32-key group, each lane forms
// per-head partial dot products of its chunk, and a butterfly
// reduce-scatter across the NCH lanes of a key leaves lane l holding the
// complete per-head dots of exactly one key.  That lane then forms the fp32
// score, writes it, and adds the key's top radix digit to a shared-memory
// histogram (merged into the row's global histogram at the end), which the
// top-k selection uses to find its threshold without another pass.
#pragma once
#include "common.cuh"

namespace csa2 {

constexpr int kScanThreads = 256;

template <int DI, int HI>
struct ScanShape {
  static constexpr int NCH = DI / 16;     // 16-byte chunks (= lanes) per key
  static constexpr int KPL = 32 / NCH;    // keys covered by one warp load
  // 32-key groups a warp processes per iteration: at least 8 loads of
  // 16 bytes per lane in flight (4 KB per warp).
  static constexpr int GROUPS = (NCH >= 8) ? 1 : 8 / NCH;
  static constexpr int KEYS_PER_ITER = 32 * GROUPS;
  static_assert(DI % 16 == 0 && NCH >= 1 && NCH <= 8, "d_I in {16,32,64,128}");
  static_assert(HI * NCH <= 32, "register budget of the per-lane partials");
};

__device__ __forceinline__ int dp4a(int a, int b, int c) { return __dp4a(a, b, c); }

// grid = (G slices, rows); rows = B * T query rows.
template <int DI, int HI>
__global__ void __launch_bounds__(kScanThreads, 3)
    index_scan_kernel(const int8_t *__restrict__ q_idx, const float *__restrict__ w,
                      const int8_t *__restrict__ k_idx, int32_t T, int64_t N, int64_t n_prior,
                      int32_t ratio, int64_t row0, float *__restrict__ scores,
                      uint32_t *__restrict__ hist1, int write_masked) {
  using S = ScanShape<DI, HI>;
  constexpr int NCH = S::NCH, KPL = S::KPL, GROUPS = S::GROUPS;
  __shared__ uint32_t sh_hist[kBins1];

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t r_local = blockIdx.y;       // row within this launch
  const int64_t r = row0 + r_local;         // global query row b*T + t
  const int64_t b = r / T, t = r % T;
  const int G = gridDim.x, g = blockIdx.x;

  int64_t V = N;
  if (n_prior >= 0) {
    V = n_prior + (t + 1) / ratio;
    if (V > N) V = N;
  }

  for (int i = tid; i < kBins1; i += kScanThreads) sh_hist[i] = 0u;

  // Slice [n0, n1) of [0, V), boundaries on 32-key multiples.
  int64_t n0 = ((V * g) / G) & ~int64_t(31);
  int64_t n1 = (g == G - 1) ? V : (((V * (g + 1)) / G) & ~int64_t(31));

  // This lane's chunk of every head's index query, and the head weights.
  const int c = lane % NCH;
  int4 qv[HI];
  float wh[HI];
#pragma unroll
  for (int h = 0; h < HI; ++h) {
    qv[h] = *reinterpret_cast<const int4 *>(q_idx + (r * HI + h) * DI + c * 16);
    wh[h] = w[r * HI + h];
  }
  __syncthreads();

  const int8_t *keys = k_idx + b * N * DI;
  float *srow = scores + r_local * N;
  const int NW = kScanThreads / 32;

  for (int64_t base = n0 + (int64_t)warp * S::KEYS_PER_ITER; base < n1;
       base += (int64_t)NW * S::KEYS_PER_ITER) {
    // ---- loads: GROUPS x NCH loads of 16 bytes per lane ----
    int4 kv[GROUPS][NCH];
#pragma unroll
    for (int gr = 0; gr < GROUPS; ++gr)
#pragma unroll
      for (int u = 0; u < NCH; ++u) {
        const int64_t key = base + gr * 32 + u * KPL + lane / NCH;
        if (key < n1)
          kv[gr][u] = ld_stream_v4(keys + key * DI + c * 16);
        else
          kv[gr][u] = make_int4(0, 0, 0, 0);
      }
#pragma unroll
    for (int gr = 0; gr < GROUPS; ++gr) {
      // ---- per-lane partial dots of its chunk ----
      int p[NCH][HI];
#pragma unroll
      for (int u = 0; u < NCH; ++u)
#pragma unroll
        for (int h = 0; h < HI; ++h) {
          int a = dp4a(kv[gr][u].x, qv[h].x, 0);
          a = dp4a(kv[gr][u].y, qv[h].y, a);
          a = dp4a(kv[gr][u].z, qv[h].z, a);
          p[u][h] = dp4a(kv[gr][u].w, qv[h].w, a);
        }
      // ---- reduce-scatter over the NCH lanes of each key ----
#pragma unroll
      for (int m = NCH / 2; m >= 1; m >>= 1) {
        const bool upper = (c & m) != 0;
#pragma unroll
        for (int i = 0; i < m; ++i)
#pragma unroll
          for (int h = 0; h < HI; ++h) {
            const int send = upper ? p[i][h] : p[i + m][h];
            const int keep = upper ? p[i + m][h] : p[i][h];
            p[i][h] = keep + __shfl_xor_sync(0xffffffffu, send, m);
          }
      }
      // lane now holds the dots of key (c * KPL + lane / NCH) of this group
      const int64_t key = base + gr * 32 + c * KPL + lane / NCH;
      const bool valid = key < n1;
      float acc = 0.0f;
#pragma unroll
      for (int h = 0; h < HI; ++h) acc = __fadd_rn(acc, __fmul_rn(wh[h], __int2float_rn(p[0][h])));
      const float score = __fadd_rn(acc, 0.0f);
      const uint32_t bin = key_d1(score_key(score));
      if (valid) srow[key] = score;
      const uint32_t active = __ballot_sync(0xffffffffu, valid);
      if (valid) {
        const uint32_t peers = __match_any_sync(active, bin);
        if (lane == __ffs(peers) - 1) atomicAdd(&sh_hist[bin], __popc(peers));
      }
    }
  }

  // Entries the row may not see (prefill): -inf when scores are requested.
  if (write_masked && V < N) {
    const int64_t m0 = V + ((N - V) * g) / G, m1 = V + ((N - V) * (g + 1)) / G;
    for (int64_t n = m0 + tid; n < m1; n += kScanThreads) srow[n] = -__int_as_float(0x7f800000);
  }

  __syncthreads();
  uint32_t *grow = hist1 + r_local * kBins1;
  for (int i = tid; i < kBins1; i += kScanThreads) {
    const uint32_t v = sh_hist[i];
    if (v) atomicAdd(grow + i, v);
  }
}

}  // namespace csa2
