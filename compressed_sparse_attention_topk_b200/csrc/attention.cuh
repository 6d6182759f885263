// Sparse attention over the selected FP4 entries plus the bf16 local window.
//
// "Why Is DeepSeek V4.1 Flash So Fast?", section 3: attention reads the
// recent context through a 128-token sliding window and a small set of
// indexer-selected compressed positions; "Inference-Efficient LLMs",
// sections 3 and 6: local keys/values are the layer's own and stay at
// higher precision than the FP4 global entries.  Readings: one joint
// softmax over selected entries and window rows; a global entry is both key
// and value and serves every head (MQA); index -1 is padding.
//
// Work split.  A query row's key list (topk selected slots, then W window
// rows) is cut into chunks of 64 keys; a CTA takes a run of consecutive
// chunks for up to 16 heads, keeps a running (max, sum, acc) per head with
// an online softmax, and writes one partial.  Decode spreads the chunks of
// a row over many CTAs (split-K) so a few sequences fill the GPU; a second
// kernel merges the partials by log-sum-exp.  Logits are kept in base 2
// (the query is pre-scaled by sm_scale * log2 e).
#pragma once
#include "common.cuh"
#include "pack.cuh"

namespace csa2 {

constexpr int kAttnThreads = 256;
constexpr int kAttnKeys = 64;    // keys per chunk
constexpr int kAttnHeads = 16;   // heads per CTA

template <int D>
struct AttnSmem {
  float q[kAttnHeads][D];
  float k[kAttnKeys][D + 1];     // +1: conflict-free column reads
  float v[kAttnKeys][D + 1];     // window values (selected entries reuse k)
  float p[kAttnHeads][kAttnKeys];
  int valid[kAttnKeys];
};

__device__ __forceinline__ float bf16_bits_to_f32(uint16_t b) {
  return __uint_as_float(((uint32_t)b) << 16);
}

// grid = (splits, rows, head groups).  part: [rows, H, splits, D + 2].
template <int D>
__global__ void __launch_bounds__(kAttnThreads, 2)
    sparse_attn_partial_kernel(const uint16_t *__restrict__ q, const uint8_t *__restrict__ codes,
                               const float *__restrict__ scales, const int32_t *__restrict__ idx,
                               const uint16_t *__restrict__ win_k,
                               const uint16_t *__restrict__ win_v, int32_t T, int32_t H,
                               int64_t N, int32_t topk, int32_t W, float q_scale,
                               int32_t chunks_per_split, float *__restrict__ part) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  AttnSmem<D> &sm = *reinterpret_cast<AttnSmem<D> *>(smem_raw);
  constexpr int DL = D / 32;  // dims per lane in the PV step

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int split = blockIdx.x, splits = gridDim.x;
  const int64_t r = blockIdx.y, b = r / T, t = r % T;
  const int h0 = blockIdx.z * kAttnHeads;
  const int nh = min(kAttnHeads, H - h0);
  const int n_sel = (topk + kAttnKeys - 1) / kAttnKeys;
  const int n_win = (W + kAttnKeys - 1) / kAttnKeys;
  const int n_chunks = n_sel + n_win;
  const int c_begin = split * chunks_per_split;
  const int c_end = min(n_chunks, c_begin + chunks_per_split);

  for (int i = tid; i < nh * D; i += kAttnThreads) {
    const int h = i / D, d = i % D;
    sm.q[h][d] = bf16_bits_to_f32(q[((r * H) + h0 + h) * (int64_t)D + d]) * q_scale;
  }

  // Running softmax state of heads (warp, warp + 8), dims lane + 32 * i.
  float run_m[2], run_l[2], acc[2][DL];
#pragma unroll
  for (int s = 0; s < 2; ++s) {
    run_m[s] = -INFINITY;
    run_l[s] = 0.0f;
#pragma unroll
    for (int i = 0; i < DL; ++i) acc[s][i] = 0.0f;
  }

  const int64_t win_rows = (int64_t)W - 1 + T;
  for (int chunk = c_begin; chunk < c_end; ++chunk) {
    __syncthreads();  // previous chunk fully consumed (and q written)
    const bool is_win = chunk >= n_sel;
    {
      const int j = tid % kAttnKeys, qtr = tid / kAttnKeys;  // 4 quarters of D
      constexpr int EQ = D / 4;                              // elements per quarter
      if (!is_win) {
        const int slot = chunk * kAttnKeys + j;
        const int32_t n = (slot < topk) ? idx[r * (int64_t)topk + slot] : -1;
        const bool ok = n >= 0 && (int64_t)n < N;
        if (n >= 0 && (int64_t)n >= N && qtr == 0) raise_status(kStatusBadIndex);
        if (qtr == 0) sm.valid[j] = ok;
        float vals[EQ];
        if (ok) {
          const int64_t row = b * N + n;
          const uint8_t *cp = codes + row * (D / 2) + qtr * (EQ / 2);
          const float *sp = scales + row * (D / 16) + qtr * (EQ / 16);
          if constexpr (EQ == 32) {
            const uint4 cw = *reinterpret_cast<const uint4 *>(cp);
            const float2 s2 = *reinterpret_cast<const float2 *>(sp);
            e2m1x8_to_f32(cw.x, s2.x, vals + 0);
            e2m1x8_to_f32(cw.y, s2.x, vals + 8);
            e2m1x8_to_f32(cw.z, s2.y, vals + 16);
            e2m1x8_to_f32(cw.w, s2.y, vals + 24);
          } else {
            const uint2 cw = *reinterpret_cast<const uint2 *>(cp);
            const float s1 = *sp;
            e2m1x8_to_f32(cw.x, s1, vals + 0);
            e2m1x8_to_f32(cw.y, s1, vals + 8);
          }
        } else {
#pragma unroll
          for (int e = 0; e < EQ; ++e) vals[e] = 0.0f;
        }
#pragma unroll
        for (int e = 0; e < EQ; ++e) sm.k[j][qtr * EQ + e] = vals[e];
      } else {
        const int wj = (chunk - n_sel) * kAttnKeys + j;
        const bool ok = wj < W;
        if (qtr == 0) sm.valid[j] = ok;
        if (ok) {
          const int64_t row = b * win_rows + t + wj;
          const uint4 *kp = reinterpret_cast<const uint4 *>(win_k + row * D + qtr * EQ);
          const uint4 *vp = reinterpret_cast<const uint4 *>(win_v + row * D + qtr * EQ);
#pragma unroll
          for (int u = 0; u < EQ / 8; ++u) {
            const uint4 kk = kp[u], vv = vp[u];
            const uint32_t kw[4] = {kk.x, kk.y, kk.z, kk.w}, vw[4] = {vv.x, vv.y, vv.z, vv.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              sm.k[j][qtr * EQ + 8 * u + 2 * e] = __uint_as_float(kw[e] << 16);
              sm.k[j][qtr * EQ + 8 * u + 2 * e + 1] = __uint_as_float(kw[e] & 0xffff0000u);
              sm.v[j][qtr * EQ + 8 * u + 2 * e] = __uint_as_float(vw[e] << 16);
              sm.v[j][qtr * EQ + 8 * u + 2 * e + 1] = __uint_as_float(vw[e] & 0xffff0000u);
            }
          }
        } else {
#pragma unroll
          for (int e = 0; e < EQ; ++e) {
            sm.k[j][qtr * EQ + e] = 0.0f;
            sm.v[j][qtr * EQ + e] = 0.0f;
          }
        }
      }
    }
    __syncthreads();

#pragma unroll
    for (int s = 0; s < 2; ++s) {
      const int hh = warp + 8 * s;
      if (hh >= nh) continue;  // warp-uniform
      // logits of keys lane and lane + 32
      float z0 = 0.0f, z1 = 0.0f;
#pragma unroll 8
      for (int d = 0; d < D; ++d) {
        const float qd = sm.q[hh][d];
        z0 = fmaf(qd, sm.k[lane][d], z0);
        z1 = fmaf(qd, sm.k[lane + 32][d], z1);
      }
      if (!sm.valid[lane]) z0 = -INFINITY;
      if (!sm.valid[lane + 32]) z1 = -INFINITY;
      const float cm = warp_max(fmaxf(z0, z1));
      const float new_m = fmaxf(run_m[s], cm);
      if (new_m == -INFINITY) continue;  // nothing valid yet (warp-uniform)
      const float p0 = exp2f(z0 - new_m), p1 = exp2f(z1 - new_m);
      const float corr = exp2f(run_m[s] - new_m);  // 0 when run_m = -inf
      run_l[s] = run_l[s] * corr + warp_sum(p0 + p1);
      run_m[s] = new_m;
      sm.p[hh][lane] = p0;
      sm.p[hh][lane + 32] = p1;
      __syncwarp();
      const float(*vsrc)[D + 1] = sm.k;
#pragma unroll
      for (int i = 0; i < DL; ++i) acc[s][i] *= corr;
      if (is_win) {
#pragma unroll 4
        for (int j = 0; j < kAttnKeys; ++j) {
          const float pj = sm.p[hh][j];
#pragma unroll
          for (int i = 0; i < DL; ++i) acc[s][i] = fmaf(pj, sm.v[j][lane + 32 * i], acc[s][i]);
        }
      } else {
#pragma unroll 4
        for (int j = 0; j < kAttnKeys; ++j) {
          const float pj = sm.p[hh][j];
#pragma unroll
          for (int i = 0; i < DL; ++i) acc[s][i] = fmaf(pj, vsrc[j][lane + 32 * i], acc[s][i]);
        }
      }
      __syncwarp();
    }
  }

#pragma unroll
  for (int s = 0; s < 2; ++s) {
    const int hh = warp + 8 * s;
    if (hh >= nh) continue;
    float *pp = part + (((r * H) + h0 + hh) * (int64_t)splits + split) * (D + 2);
    if (lane == 0) {
      pp[0] = run_m[s];
      pp[1] = run_l[s];
    }
#pragma unroll
    for (int i = 0; i < DL; ++i) pp[2 + lane + 32 * i] = acc[s][i];
  }
}

// One warp per (row, head): merge the split partials.
template <int D>
__global__ void __launch_bounds__(256)
    sparse_attn_combine_kernel(const float *__restrict__ part, int32_t splits, int64_t rows_x_heads,
                               float *__restrict__ out, float *__restrict__ lse) {
  constexpr int DL = D / 32;
  const int lane = threadIdx.x & 31;
  const int64_t gw = blockIdx.x * (int64_t)(blockDim.x / 32) + (threadIdx.x >> 5);
  if (gw >= rows_x_heads) return;
  const float *p = part + gw * splits * (D + 2);
  float M = -INFINITY;
  for (int c = 0; c < splits; ++c) {
    const float m = p[c * (D + 2)], l = p[c * (D + 2) + 1];
    if (l > 0.0f) M = fmaxf(M, m);
  }
  float *o = out + gw * D;
  if (M == -INFINITY) {
#pragma unroll
    for (int i = 0; i < DL; ++i) o[lane + 32 * i] = 0.0f;
    if (lse && lane == 0) lse[gw] = -INFINITY;
    return;
  }
  float L = 0.0f, acc[DL];
#pragma unroll
  for (int i = 0; i < DL; ++i) acc[i] = 0.0f;
  for (int c = 0; c < splits; ++c) {
    const float *pc = p + c * (D + 2);
    const float l = pc[1];
    if (!(l > 0.0f)) continue;
    const float f = exp2f(pc[0] - M);
    L += l * f;
#pragma unroll
    for (int i = 0; i < DL; ++i) acc[i] = fmaf(pc[2 + lane + 32 * i], f, acc[i]);
  }
  const float inv = 1.0f / L;
#pragma unroll
  for (int i = 0; i < DL; ++i) o[lane + 32 * i] = acc[i] * inv;
  if (lse && lane == 0) lse[gw] = (M + log2f(L)) * 0.69314718055994530942f;
}

}  // namespace csa2
