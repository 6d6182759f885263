// Sparse attention for many query rows at once (chunked prefill, large
// batches): one CTA per (query row, 16-head pass), throughput-oriented.
//
// Per row and head h ("Why Is DeepSeek V4.1 Flash So Fast?", section 3: the
// query attends to its Top-K compressed entries and to the sliding window):
// logits over the selected entries (dequantised FP4, used as key and value)
// and the W window rows (bf16 K_win / V_win), scale 1/sqrt(D), one joint
// softmax, output sum_j p_j v_j / sum_j p_j and lse = log sum_j exp(z_j).
//
// Work split: the row's keys are cut into 16-key chunks (selected entries
// first, then window rows); warp w of 8 takes chunks w, w+8, ... with its own
// online-softmax state (flash-decoding inside the CTA), so the main loop has
// no CTA-wide barrier.  Entry chunks are gathered with cp.async one chunk
// ahead into a per-warp staging area (invalid or padding keys zero-filled),
// converted once to exact bf16 E2M1 values, and read back as mma.sync
// m16n8k16 fragments with ldmatrix (QK^T: M = 16 heads, N = keys, K = one
// 16-element scale group per step, group scale applied in fp32; PV: A = P x
// group scale split into bf16 hi + lo, B = E2M1 values).  The 8 partial
// states are merged by log-sum-exp at the end.
#pragma once
#include "common.cuh"

namespace csa2 {
namespace ar {

constexpr int kWarps = 8;
constexpr int kThreads = 32 * kWarps;
constexpr int kChunk = 16;  // keys per chunk (the PV MMA's K)
constexpr int kHeads = 16;  // heads per pass (the MMAs' M)

struct Params {
  const uint16_t *q;        // bf16 [B, T, H, D]
  const uint8_t *codes;     // [B, N, D/2]
  const float *scales;      // [B, N, D/16]
  const int32_t *idx;       // [B, T, topk]
  const uint16_t *win_k;    // bf16 [B, W-1+T, D]
  const uint16_t *win_v;
  int64_t N;
  int32_t T, H, W, topk;
  float q_scale;            // sm_scale * log2(e): logits in base 2
  float *out;               // [B, T, H, D]
  float *lse;               // [B, T, H] (nullable)
  int64_t row0;             // first row (b*T + t) of this launch
};

template <int D>
struct alignas(16) WarpArea {
  static constexpr int CB = D / 2;                  // code bytes per entry
  static constexpr int SB = D / 4;                  // scale bytes per entry
  static constexpr int PIECES = (CB + SB) / 16;     // 16-byte pieces per entry
  union {
    struct {
      uint8_t codes[2][kChunk][CB];                 // staging, double-buffered
      float scales[2][kChunk][D / 16];
      uint16_t kt[kChunk][D + 8];                   // keys of the chunk (bf16)
      uint16_t vt[kChunk][D + 8];                   // window values (bf16)
    } s;
    struct {
      alignas(16) float o[kHeads][D];               // partial output for the merge
      float m[kHeads], l[kHeads];
    } merge;
  };
};

template <int D>
struct Smem {
  uint16_t q[kHeads][D + 8];
  WarpArea<D> w[kWarps];
};

__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], const void *p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(smem_u32(p)));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t (&r)[4], const void *p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(smem_u32(p)));
}
__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
// 16-byte async copy; src_bytes = 0 zero-fills the destination.
__device__ __forceinline__ void cp16(void *dst, const void *src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src),
               "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
// fp32 pair -> packed bf16 pairs hi, lo with x ~= hi + lo.
__device__ __forceinline__ void split2(float x0, float x1, uint32_t &hi, uint32_t &lo) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(x0, x1);
  const float2 hf = __bfloat1622float2(h);
  const __nv_bfloat162 l = __floats2bfloat162_rn(x0 - hf.x, x1 - hf.y);
  hi = *reinterpret_cast<const uint32_t *>(&h);
  lo = *reinterpret_cast<const uint32_t *>(&l);
}
// Eight E2M1 codes (one word, element 2i in the low nibble of byte i) ->
// four exact bf16 pairs (lower element in the low half).
__device__ __forceinline__ uint4 e2m1x8_bf16(uint32_t word) {
  uint32_t h[4];
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "mov.b32 {b0, b1, b2, b3}, %4;\n\t"
      "cvt.rn.f16x2.e2m1x2 %0, b0;\n\t"
      "cvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
      "cvt.rn.f16x2.e2m1x2 %2, b2;\n\t"
      "cvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
      : "=r"(h[0]), "=r"(h[1]), "=r"(h[2]), "=r"(h[3])
      : "r"(word));
  uint32_t o[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&h[i]));
    const __nv_bfloat162 b = __floats2bfloat162_rn(f.x, f.y);  // exact: <= 3 significant bits
    o[i] = *reinterpret_cast<const uint32_t *>(&b);
  }
  return make_uint4(o[0], o[1], o[2], o[3]);
}

// ---------------------------------------------------------------------------
// Per-warp building blocks (also used by the per-row cluster kernel).
// A warp owns one WarpArea and one running state for 16 heads; a chunk is
// 16 keys.  Fragment layout of the state: o[i] holds heads gid and gid + 8,
// output dims 8i + 2 tig, +1 (mma.sync m16n8k16 C layout); m/l are the base-2
// running max and the lane's partial sum of each of its two heads.
// ---------------------------------------------------------------------------
template <int D>
struct WarpState {
  float o[D / 8][4];
  float m0, m1, l0, l1;
};

template <int D>
__device__ __forceinline__ void state_init(WarpState<D> &st) {
#pragma unroll
  for (int i = 0; i < D / 8; ++i) st.o[i][0] = st.o[i][1] = st.o[i][2] = st.o[i][3] = 0.0f;
  st.m0 = st.m1 = -INFINITY;
  st.l0 = st.l1 = 0.0f;
}

// Issue the async gather of 16 entries into staging buffer sb.  Lane j and
// lane j + 16 hold the entry index n of key j (n < 0: none; n >= N is
// recorded as a bad index and skipped).  Missing keys are zero-filled.
// Returns the mask of real keys; commits one cp.async group.
template <int D>
__device__ __forceinline__ uint32_t gather_entries(WarpArea<D> &wa, int sb, int32_t n, int64_t N,
                                                   const uint8_t *cseq, const float *sseq) {
  using WA = WarpArea<D>;
  const int lane = threadIdx.x & 31;
  if (n >= N) {
    raise_status(kStatusBadIndex);
    n = -1;
  }
  const uint32_t mask = __ballot_sync(0xffffffffu, n >= 0) & 0xffffu;
#pragma unroll
  for (int i = 0; i < (kChunk * WA::PIECES + 31) / 32; ++i) {
    // every lane takes part in the shuffle (a lane past the last piece asks
    // for key 0 and copies nothing)
    const int piece = lane + 32 * i;
    const bool live = piece < kChunk * WA::PIECES;
    const bool is_code = piece < kChunk * (WA::CB / 16);
    const int sp = piece - kChunk * (WA::CB / 16);
    const int key = !live ? 0 : (is_code ? piece / (WA::CB / 16) : sp / (WA::SB / 16));
    const int off = !live ? 0 : (is_code ? piece % (WA::CB / 16) : sp % (WA::SB / 16));
    const int32_t nk = __shfl_sync(0xffffffffu, n, key);
    if (live) {
      const bool ok = nk >= 0;
      const int64_t nn = ok ? nk : 0;
      if (is_code)
        cp16(&wa.s.codes[sb][key][16 * off], cseq + nn * (D / 2) + 16 * off, ok ? 16u : 0u);
      else
        cp16(reinterpret_cast<uint8_t *>(&wa.s.scales[sb][key][0]) + 16 * off,
             reinterpret_cast<const uint8_t *>(sseq + nn * (D / 16)) + 16 * off, ok ? 16u : 0u);
    }
  }
  cp_commit();
  return mask;
}

// Staged E2M1 codes of buffer sb -> exact bf16 values in kt.  Lane = (key
// lane/2, half of the dims).
template <int D>
__device__ __forceinline__ void convert_entries(WarpArea<D> &wa, int sb) {
  const int lane = threadIdx.x & 31;
  const int j = lane >> 1, hf = lane & 1;
  constexpr int HB = D / 4;  // code bytes per half row
  const uint8_t *src = &wa.s.codes[sb][j][hf * HB];
  uint16_t *dst = &wa.s.kt[j][hf * (D / 2)];
#pragma unroll
  for (int u = 0; u < HB / 4; u += 2) {  // two words = 16 elements per step
    const uint2 w2 = *reinterpret_cast<const uint2 *>(src + 4 * u);
    *reinterpret_cast<uint4 *>(dst + 8 * u) = e2m1x8_bf16(w2.x);
    *reinterpret_cast<uint4 *>(dst + 8 * u + 8) = e2m1x8_bf16(w2.y);
  }
}

// Window rows [row0, row0 + nrows) (nrows <= 16) -> kt / vt, bf16 as
// stored, missing rows zero-filled; waits for every copy of this warp.
template <int D>
__device__ __forceinline__ uint32_t load_window_rows(WarpArea<D> &wa, const uint16_t *win_k,
                                                     const uint16_t *win_v, int64_t row0,
                                                     int nrows) {
  constexpr int RP = D / 8;  // 16-byte pieces per row
  const int lane = threadIdx.x & 31;
  for (int i = lane; i < kChunk * RP; i += 32) {
    const int j = i / RP, u = i % RP;
    const bool ok = j < nrows;
    const int64_t row = ok ? row0 + j : row0;
    cp16(&wa.s.kt[j][8 * u], win_k + row * D + 8 * u, ok ? 16u : 0u);
    cp16(&wa.s.vt[j][8 * u], win_v + row * D + 8 * u, ok ? 16u : 0u);
  }
  cp_commit();
  cp_wait<0>();
  __syncwarp();
  return (1u << nrows) - 1u;
}

// QK^T, online-softmax update and PV for the chunk in kt (values: vt for
// window rows, else kt with per-key group scales sc[key][g]).
template <int D>
__device__ __forceinline__ void attend_chunk16(WarpArea<D> &wa, const uint16_t (*q)[D + 8],
                                               WarpState<D> &st, uint32_t mask, bool window,
                                               const float (*sc)[D / 16], float q_scale) {
  constexpr int G = D / 16;
  constexpr int NT = D / 8;
  const int lane = threadIdx.x & 31;
  const int tig = lane & 3;
  // logits
  float s[2][4];
#pragma unroll
  for (int nt = 0; nt < 2; ++nt) s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.0f;
#pragma unroll
  for (int g = 0; g < G; ++g) {
    uint32_t a[4], kb[4];
    ldsm_x4(a, &q[(lane & 7) + ((lane >> 3) & 1) * 8][16 * g + (lane >> 4) * 8]);
    ldsm_x4(kb, &wa.s.kt[((lane >> 4) << 3) + (lane & 7)][16 * g + ((lane >> 3) & 1) * 8]);
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      float d4[4] = {0.0f, 0.0f, 0.0f, 0.0f};
      mma16816(d4, a, kb[2 * nt], kb[2 * nt + 1]);
      const int k0 = 8 * nt + 2 * tig;
      const float s0 = window ? 1.0f : sc[k0][g], s1 = window ? 1.0f : sc[k0 + 1][g];
      s[nt][0] = fmaf(d4[0], s0, s[nt][0]);
      s[nt][1] = fmaf(d4[1], s1, s[nt][1]);
      s[nt][2] = fmaf(d4[2], s0, s[nt][2]);
      s[nt][3] = fmaf(d4[3], s1, s[nt][3]);
    }
  }
  // online softmax (base 2); the lanes of a quad share heads gid and gid + 8
  float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
  for (int nt = 0; nt < 2; ++nt) {
    const int k0 = 8 * nt + 2 * tig;
    const bool v0 = (mask >> k0) & 1u, v1 = (mask >> (k0 + 1)) & 1u;
    s[nt][0] = v0 ? s[nt][0] * q_scale : -INFINITY;
    s[nt][1] = v1 ? s[nt][1] * q_scale : -INFINITY;
    s[nt][2] = v0 ? s[nt][2] * q_scale : -INFINITY;
    s[nt][3] = v1 ? s[nt][3] * q_scale : -INFINITY;
    mx0 = fmaxf(mx0, fmaxf(s[nt][0], s[nt][1]));
    mx1 = fmaxf(mx1, fmaxf(s[nt][2], s[nt][3]));
  }
  mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
  mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
  mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
  mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
  const float n0 = fmaxf(st.m0, mx0), n1 = fmaxf(st.m1, mx1);
  const float c0 = n0 == -INFINITY ? 1.0f : exp2f(st.m0 - n0);
  const float c1 = n1 == -INFINITY ? 1.0f : exp2f(st.m1 - n1);
  float pr[2][4];
#pragma unroll
  for (int nt = 0; nt < 2; ++nt) {
    pr[nt][0] = n0 == -INFINITY ? 0.0f : exp2f(s[nt][0] - n0);
    pr[nt][1] = n0 == -INFINITY ? 0.0f : exp2f(s[nt][1] - n0);
    pr[nt][2] = n1 == -INFINITY ? 0.0f : exp2f(s[nt][2] - n1);
    pr[nt][3] = n1 == -INFINITY ? 0.0f : exp2f(s[nt][3] - n1);
  }
  st.l0 = st.l0 * c0 + (pr[0][0] + pr[0][1] + pr[1][0] + pr[1][1]);
  st.l1 = st.l1 * c1 + (pr[0][2] + pr[0][3] + pr[1][2] + pr[1][3]);
  st.m0 = n0;
  st.m1 = n1;
#pragma unroll
  for (int i = 0; i < NT; ++i) {
    st.o[i][0] *= c0;
    st.o[i][1] *= c0;
    st.o[i][2] *= c1;
    st.o[i][3] *= c1;
  }
  // PV per scale group: A = P x scale (hi + lo), B = values of 16 dims
  const uint16_t(*vsrc)[D + 8] = window ? wa.s.vt : wa.s.kt;
#pragma unroll
  for (int g = 0; g < G; ++g) {
    float sa = 1.0f, sb = 1.0f, sc2 = 1.0f, sd = 1.0f;
    if (!window) {
      sa = sc[2 * tig][g];
      sb = sc[2 * tig + 1][g];
      sc2 = sc[8 + 2 * tig][g];
      sd = sc[9 + 2 * tig][g];
    }
    uint32_t ah[4], al[4];
    split2(pr[0][0] * sa, pr[0][1] * sb, ah[0], al[0]);
    split2(pr[0][2] * sa, pr[0][3] * sb, ah[1], al[1]);
    split2(pr[1][0] * sc2, pr[1][1] * sd, ah[2], al[2]);
    split2(pr[1][2] * sc2, pr[1][3] * sd, ah[3], al[3]);
    uint32_t vb[4];
    ldsm_x4_t(vb, &vsrc[((lane >> 3) & 1) * 8 + (lane & 7)][16 * g + (lane >> 4) * 8]);
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      mma16816(st.o[2 * g + nt], ah, vb[2 * nt], vb[2 * nt + 1]);
      mma16816(st.o[2 * g + nt], al, vb[2 * nt], vb[2 * nt + 1]);
    }
  }
}

// Final per-head sums over the quad, then the state into the warp's merge
// area (the warp must be done with its staging buffers).
template <int D>
__device__ __forceinline__ void store_state(WarpArea<D> &wa, WarpState<D> &st) {
  const int lane = threadIdx.x & 31;
  const int gid = lane >> 2, tig = lane & 3;
  st.l0 += __shfl_xor_sync(0xffffffffu, st.l0, 1);
  st.l0 += __shfl_xor_sync(0xffffffffu, st.l0, 2);
  st.l1 += __shfl_xor_sync(0xffffffffu, st.l1, 1);
  st.l1 += __shfl_xor_sync(0xffffffffu, st.l1, 2);
  __syncwarp();
#pragma unroll
  for (int i = 0; i < D / 8; ++i) {
    const int d0 = 8 * i + 2 * tig;
    wa.merge.o[gid][d0] = st.o[i][0];
    wa.merge.o[gid][d0 + 1] = st.o[i][1];
    wa.merge.o[gid + 8][d0] = st.o[i][2];
    wa.merge.o[gid + 8][d0 + 1] = st.o[i][3];
  }
  if (tig == 0) {
    wa.merge.m[gid] = st.m0;
    wa.merge.m[gid + 8] = st.m1;
    wa.merge.l[gid] = st.l0;
    wa.merge.l[gid + 8] = st.l1;
  }
}

template <int D>
__global__ void __launch_bounds__(kThreads, 2) attn_rows_kernel(const Params p) {
  extern __shared__ __align__(16) unsigned char ar_smem_raw[];
  Smem<D> &sm = *reinterpret_cast<Smem<D> *>(ar_smem_raw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t r = p.row0 + blockIdx.x;  // query row b*T + t
  const int64_t b = r / p.T, t = r % p.T;
  const int h0 = blockIdx.y * kHeads;
  const int nh = min(kHeads, p.H - h0);
  WarpArea<D> &wa = sm.w[warp];

  // queries of the pass (padding heads zero)
  constexpr int QP = D / 8;  // 16-byte pieces per head
  for (int i = tid; i < kHeads * QP; i += kThreads) {
    const int h = i / QP, u = i % QP;
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (h < nh) v = *reinterpret_cast<const uint4 *>(p.q + ((r * p.H + h0 + h) * (int64_t)D + 8 * u));
    *reinterpret_cast<uint4 *>(&sm.q[h][8 * u]) = v;
  }
  __syncthreads();

  const int ne = p.N > 0 ? (p.topk + kChunk - 1) / kChunk : 0;  // entry chunks
  const int nw = (p.W + kChunk - 1) / kChunk;                    // window chunks
  const int32_t *irow = p.idx + r * p.topk;
  const uint8_t *cseq = p.codes + b * p.N * (D / 2);
  const float *sseq = p.scales + b * p.N * (D / 16);
  WarpState<D> st;
  state_init(st);
  auto entry_of = [&](int c) -> int32_t {  // this lane's key of entry chunk c
    const int k = c * kChunk + (lane & 15);
    return k < p.topk ? irow[k] : -1;
  };

  // window chunks (bf16 rows straight into kt / vt)
  const int64_t wrow0 = b * (int64_t)(p.W - 1 + p.T) + t;  // rows t .. t + W - 1
  for (int c = (warp - ne % kWarps + kWarps) % kWarps; c < nw; c += kWarps) {
    const uint32_t mask = load_window_rows<D>(wa, p.win_k, p.win_v, wrow0 + c * kChunk,
                                              min(kChunk, p.W - c * kChunk));
    attend_chunk16<D>(wa, sm.q, st, mask, true, nullptr, p.q_scale);
    __syncwarp();
  }

  // entry chunks, gathered one chunk ahead
  int c = warp;
  uint32_t mask_cur = 0u;
  if (c < ne) mask_cur = gather_entries<D>(wa, 0, entry_of(c), p.N, cseq, sseq);
  for (int it = 0; c < ne; ++it, c += kWarps) {
    const int sb = it & 1;
    uint32_t mask_next = 0u;
    const bool more = c + kWarps < ne;
    if (more) mask_next = gather_entries<D>(wa, sb ^ 1, entry_of(c + kWarps), p.N, cseq, sseq);
    if (more)
      cp_wait<1>();
    else
      cp_wait<0>();
    __syncwarp();
    convert_entries<D>(wa, sb);
    __syncwarp();
    attend_chunk16<D>(wa, sm.q, st, mask_cur, false, wa.s.scales[sb], p.q_scale);
    __syncwarp();  // kt and this staging buffer free again
    mask_cur = mask_next;
  }

  // merge the warps' states
  __syncthreads();  // every warp is done with its staging area
  store_state<D>(wa, st);
  __syncthreads();
  for (int i = tid; i < nh * D; i += kThreads) {
    const int h = i / D, d = i % D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) M = fmaxf(M, sm.w[w].merge.m[h]);
    float L = 0.0f, acc = 0.0f;
    if (M != -INFINITY) {
#pragma unroll
      for (int w = 0; w < kWarps; ++w) {
        const float f = exp2f(sm.w[w].merge.m[h] - M);  // 0 for a warp that saw nothing
        L = fmaf(sm.w[w].merge.l[h], f, L);
        acc = fmaf(sm.w[w].merge.o[h][d], f, acc);
      }
    }
    const int64_t oh = r * p.H + h0 + h;
    p.out[oh * D + d] = M == -INFINITY ? 0.0f : acc / L;
    if (d == 0 && p.lse)
      p.lse[oh] = M == -INFINITY ? -INFINITY : (M + log2f(L)) * 0.69314718055994531f;
  }
}

}  // namespace ar
}  // namespace csa2
