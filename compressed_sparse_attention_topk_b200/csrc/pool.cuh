// Hierarchical sparse indexing: the candidate pool of a Full layer and the
// top-k of a Reindex layer within it.
//
// "Inference-Efficient LLMs: How Sparse Compute and Compressed Memory Work",
// section 5 ("Hierarchical Sparse Indexing"): an earlier Full layer searches
// the whole context and keeps a candidate pool (the example: 2,048 blocks of
// eight positions, 16,384 candidates); later Reindex layers search only that
// pool.  This library's reading: block j covers positions [j*block,
// (j+1)*block) of the store (the last block only its visible positions); a
// block's score is the largest index score among its positions; the best
// n_blocks blocks are kept, ties to the lower block; the pool lists their
// positions in ascending order.  A Reindex row scores only the pool's
// positions (the same index score as the full scan) and keeps their top-k,
// ties to the lower position.
//
// Both selections run on the per-row cluster kernel's exact radix top-k
// (row_cluster.cuh) over a score row that these kernels prepare: the block
// maxima of a Full row's scores, or the scores of a row's pool positions.
// These kernels stream a few MB at most per call and are plain one-element-
// per-thread passes; each also builds the digit-1 histogram the top-k needs
// (shared-memory counts merged into the row's global histogram).
#pragma once
#include "common.cuh"
#include "index_scan.cuh"

namespace csa2 {

constexpr int kPoolThreads = 256;

// Merge a CTA's shared histogram into the row's global one.
__device__ __forceinline__ void flush_hist(const uint32_t *sh, uint32_t *grow) {
  for (int i = threadIdx.x; i < kBins1; i += blockDim.x) {
    const uint32_t v = sh[i];
    if (v) atomicAdd(grow + i, v);
  }
}

// grid = (ceil(nb / 256), rows).  scores: [rows, sstride] (the row's visible
// scores, N of them); bscores: [rows, bstride] block maxima; bhist: [rows,
// kHistStride], zeroed.
__global__ void __launch_bounds__(kPoolThreads) block_max_kernel(
    const float *__restrict__ scores, int64_t sstride, int64_t N, int32_t block,
    float *__restrict__ bscores, int64_t bstride, uint32_t *__restrict__ bhist) {
  __shared__ uint32_t sh[kBins1];
  for (int i = threadIdx.x; i < kBins1; i += kPoolThreads) sh[i] = 0u;
  __syncthreads();
  const int64_t r = blockIdx.y;
  const int64_t nb = (N + block - 1) / block;
  const int64_t j = (int64_t)blockIdx.x * kPoolThreads + threadIdx.x;
  if (j < nb) {
    const float *s = scores + r * sstride;
    const int64_t n0 = j * block, n1 = min64(n0 + block, N);
    float m = s[n0];
    for (int64_t n = n0 + 1; n < n1; ++n) m = fmaxf(m, s[n]);
    bscores[r * bstride + j] = m;
    atomicAdd(&sh[key_d1(score_key(m))], 1u);
  }
  __syncthreads();
  flush_hist(sh, bhist + r * kHistStride);
}

// grid = (ceil(n_blocks * block / 256), rows).  bidx: [rows, n_blocks] kept
// blocks ascending (-1 padded); pool: [rows, n_blocks * block].
__global__ void __launch_bounds__(kPoolThreads) expand_pool_kernel(
    const int32_t *__restrict__ bidx, int32_t n_blocks, int32_t block, int64_t N,
    int32_t *__restrict__ pool) {
  const int64_t r = blockIdx.y;
  const int64_t P = (int64_t)n_blocks * block;
  const int64_t i = (int64_t)blockIdx.x * kPoolThreads + threadIdx.x;
  if (i >= P) return;
  const int32_t b = bidx[r * n_blocks + i / block];
  const int64_t pos = (int64_t)b * block + i % block;
  pool[r * P + i] = (b >= 0 && pos < N) ? (int32_t)pos : -1;
}

// grid = (ceil(P / 256), rows).  Index score of each pool position of row r
// (decode: one query per sequence), -inf for entries that are not positions
// of the store (-1 padding; an entry >= N is also recorded as a bad index).
// q_idx [rows, H_I, d_I], w [rows, H_I], k_idx [rows, N, d_I], pool [rows, P].
__global__ void __launch_bounds__(kPoolThreads) pool_scan_kernel(
    const int8_t *__restrict__ q_idx, const float *__restrict__ w,
    const int8_t *__restrict__ k_idx, int32_t H_I, int32_t d_I, int64_t N,
    const int32_t *__restrict__ pool, int32_t P, float *__restrict__ pscores, int64_t pstride,
    uint32_t *__restrict__ phist) {
  __shared__ uint32_t sh[kBins1];
  __shared__ __align__(16) int8_t sq[8 * 128];
  __shared__ float sw[8];
  const int64_t r = blockIdx.y;
  for (int i = threadIdx.x; i < kBins1; i += kPoolThreads) sh[i] = 0u;
  for (int i = threadIdx.x; i < H_I * d_I; i += kPoolThreads) sq[i] = q_idx[r * H_I * d_I + i];
  if (threadIdx.x < H_I) sw[threadIdx.x] = w[r * H_I + threadIdx.x];
  __syncthreads();
  const int64_t i = (int64_t)blockIdx.x * kPoolThreads + threadIdx.x;
  if (i < P) {
    const int32_t p = pool[r * P + i];
    float score = -__int_as_float(0x7f800000);
    if (p >= N) raise_status(kStatusBadIndex);
    if (p >= 0 && p < N) {
      const int4 *key = reinterpret_cast<const int4 *>(k_idx + (r * N + p) * d_I);
      const int4 *qv = reinterpret_cast<const int4 *>(sq);
      const int nch = d_I / 16;
      float acc = 0.0f;
      for (int h = 0; h < H_I; ++h) {
        int dot = 0;
        for (int c = 0; c < nch; ++c) {
          const int4 k = key[c], q = qv[h * nch + c];
          dot = __dp4a(k.x, q.x, dot);
          dot = __dp4a(k.y, q.y, dot);
          dot = __dp4a(k.z, q.z, dot);
          dot = __dp4a(k.w, q.w, dot);
        }
        acc = __fadd_rn(acc, __fmul_rn(sw[h], __int2float_rn(dot)));
      }
      score = __fadd_rn(acc, 0.0f);
    }
    pscores[r * pstride + i] = score;
    atomicAdd(&sh[key_d1(score_key(score))], 1u);
  }
  __syncthreads();
  flush_hist(sh, phist + r * kHistStride);
}

// grid = (ceil(topk / 256), rows).  sel: [rows, topk] selected pool slots
// (ascending, -1 padded) -> idx_out: their positions (-1 for a slot that
// holds no position of the store).
__global__ void __launch_bounds__(kPoolThreads) map_pool_kernel(
    const int32_t *__restrict__ sel, int32_t topk, const int32_t *__restrict__ pool, int32_t P,
    int64_t N, int32_t *__restrict__ idx_out) {
  const int64_t r = blockIdx.y;
  const int64_t j = (int64_t)blockIdx.x * kPoolThreads + threadIdx.x;
  if (j >= topk) return;
  const int32_t s = sel[r * topk + j];
  int32_t pos = -1;
  if (s >= 0 && s < P) {
    const int32_t p = pool[r * P + s];
    pos = (p >= 0 && p < N) ? p : -1;
  }
  idx_out[r * topk + j] = pos;
}

// grid = (ceil(nb / 256), rows).  Block maxima kept as score keys (by the
// fused decode kernel) -> block scores and their digit-1 histogram, the
// input of the row kernel's top-k.  bkey [rows, nb]; bscores [rows,
// bstride]; bhist [rows, kHistStride], zeroed.
__global__ void __launch_bounds__(kPoolThreads) block_keys_to_scores_kernel(
    const uint32_t *__restrict__ bkey, int64_t nb, float *__restrict__ bscores, int64_t bstride,
    uint32_t *__restrict__ bhist) {
  __shared__ uint32_t sh[kBins1];
  for (int i = threadIdx.x; i < kBins1; i += kPoolThreads) sh[i] = 0u;
  __syncthreads();
  const int64_t r = blockIdx.y;
  const int64_t j = (int64_t)blockIdx.x * kPoolThreads + threadIdx.x;
  if (j < nb) {
    const uint32_t k = bkey[r * nb + j];
    const float m = __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
    bscores[r * bstride + j] = m;
    atomicAdd(&sh[key_d1(k)], 1u);
  }
  __syncthreads();
  flush_hist(sh, bhist + r * kHistStride);
}

}  // namespace csa2
