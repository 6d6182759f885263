// FP4 (E2M1) entry store: pack and unpack kernels.
//
// FP4 storage of the main cache entries with per-group scaling:
// "Inference-Efficient LLMs", section 6; "DeepSeek-V4.1-Flash" (visual
// explainer), section "Fast memory, persistent storage and recomputation".
// Element format E2M1 with one fp32 scale per 16 elements; s = amax / 6;
// codes round to nearest, ties to the even code, saturate at 6; zero
// magnitude is always code 0; element 2i is the low nibble of byte i.
#pragma once
#include "common.cuh"

namespace csa2 {

// Magnitude code of y >= 0 on the E2M1 grid {0, .5, 1, 1.5, 2, 3, 4, 6}.
// Each comparison moves past one midpoint; at a midpoint the strict / non-
// strict choice sends the value to the neighbour with an even code.
__device__ __forceinline__ uint32_t e2m1_mag_code(float y) {
  return (uint32_t)(y > 0.25f) + (uint32_t)(y >= 0.75f) + (uint32_t)(y > 1.25f) +
         (uint32_t)(y >= 1.75f) + (uint32_t)(y > 2.5f) + (uint32_t)(y >= 3.5f) +
         (uint32_t)(y > 5.0f);
}

// The FP4 codes (two words) and scale of one group of 16 fp32 values.
__device__ __forceinline__ void pack_group16(const float (&x)[16], uint2 &code, float &scale) {
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const float a = fabsf(x[i]);
    if (a > amax) amax = a;
  }
  const float s = __fdiv_rn(amax, 6.0f);
  uint32_t lo = 0, hi = 0;
  if (s > 0.0f) {
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const float y = __fdiv_rn(x[i], s);
      uint32_t c = e2m1_mag_code(fabsf(y));
      if (c != 0u && x[i] < 0.0f) c |= 8u;
      if (i < 8)
        lo |= c << (4 * i);
      else
        hi |= c << (4 * (i - 8));
    }
  }
  code = make_uint2(lo, hi);
  scale = s;
}

// One thread per group of 16 elements.
__global__ void __launch_bounds__(256) pack_fp4_kernel(const float *__restrict__ src,
                                                       int64_t groups,
                                                       uint8_t *__restrict__ codes,
                                                       float *__restrict__ scales) {
  for (int64_t g = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; g < groups;
       g += (int64_t)gridDim.x * blockDim.x) {
    const float4 *p = reinterpret_cast<const float4 *>(src + g * 16);
    float x[16];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float4 v = __ldcs(p + i);
      x[4 * i + 0] = v.x;
      x[4 * i + 1] = v.y;
      x[4 * i + 2] = v.z;
      x[4 * i + 3] = v.w;
    }
    uint2 code;
    float s;
    pack_group16(x, code, s);
    reinterpret_cast<uint2 *>(codes)[g] = code;
    scales[g] = s;
  }
}

// Entry append ("DeepSeek-V4.1-Flash", section "Fast memory, persistent
// storage and recomputation": the main cache entries are stored in FP4;
// "Inference-Efficient LLMs", section 6: per-group scaling): one decode
// step writes each sequence's completed entry into row pos[b] of its store
// -- the FP4 codes and scales of src[b] (the rule of pack_fp4_kernel) and
// the int8 index key key[b] -- and nothing for a sequence with pos[b] < 0.
// A position >= N is recorded as a bad index and skipped.  One thread per
// 16-element group of an entry or 16-byte piece of a key.
__global__ void __launch_bounds__(128) append_entry_kernel(
    const float *__restrict__ src, const int8_t *__restrict__ key, const int64_t *__restrict__ pos,
    int32_t B, int32_t D, int32_t d_I, int64_t N, uint8_t *__restrict__ codes,
    float *__restrict__ scales, int8_t *__restrict__ k_idx) {
  const int G = D / 16, KP = d_I / 16;  // groups and key pieces per sequence
  const int64_t total = (int64_t)B * (G + KP);
  for (int64_t u = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; u < total;
       u += (int64_t)gridDim.x * blockDim.x) {
    const int64_t b = u / (G + KP);
    const int q = (int)(u % (G + KP));
    const int64_t n = pos[b];
    if (n < 0) continue;
    if (n >= N) {
      if (q == 0) raise_status(kStatusBadIndex);
      continue;
    }
    const int64_t row = b * N + n;
    if (q < G) {
      const float4 *p = reinterpret_cast<const float4 *>(src + b * D + 16 * q);
      float x[16];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float4 v = p[i];
        x[4 * i + 0] = v.x;
        x[4 * i + 1] = v.y;
        x[4 * i + 2] = v.z;
        x[4 * i + 3] = v.w;
      }
      uint2 code;
      float s;
      pack_group16(x, code, s);
      reinterpret_cast<uint2 *>(codes + row * (D / 2))[q] = code;
      scales[row * G + q] = s;
    } else {
      const int k = q - G;
      reinterpret_cast<int4 *>(k_idx + row * d_I)[k] =
          reinterpret_cast<const int4 *>(key + b * d_I)[k];
    }
  }
}

// ---------------------------------------------------------------------------
// FP4 index keys ("Inference-Efficient LLMs", section 6: FP4 in parts of the
// attention indexing machinery).  This library's reading: E2M1 elements with
// one power-of-two scale per block of 32 elements, kept as an 8-bit biased
// exponent (the OCP Microscaling MXFP4 block format).  Per block: shared
// exponent s = floor(log2(amax)) - 2 (2 = the largest E2M1 exponent),
// clamped to [-127, 127], stored as s + 127; each element's code is the
// E2M1 value nearest to x / 2^s (IEEE divide; ties to the even code,
// saturating at 6; a zero magnitude is code 0); an all-zero block stores
// exponent byte 0 and zero codes.  Element 2i is the low nibble of byte i.
// ---------------------------------------------------------------------------

// floor(log2(a)) of a finite a > 0, from its bits.
__device__ __forceinline__ int floor_log2_pos(float a) {
  const uint32_t u = __float_as_uint(a);
  const int e = (int)((u >> 23) & 0xffu);
  if (e != 0) return e - 127;
  return (31 - __clz((int)(u & 0x7fffffu))) - 149;  // subnormal: mantissa * 2^-149
}

// 2^e as fp32 for -149 <= e <= 127 (exact).
__device__ __forceinline__ float pow2_f32(int e) {
  return e >= -126 ? __uint_as_float((uint32_t)(e + 127) << 23)
                   : __uint_as_float(1u << (e + 149));
}

// One thread per block of 32 elements: codes [blocks, 16] bytes, exps [blocks].
__global__ void __launch_bounds__(256) pack_keys_fp4_kernel(const float *__restrict__ src,
                                                            int64_t blocks,
                                                            uint8_t *__restrict__ codes,
                                                            uint8_t *__restrict__ exps) {
  for (int64_t g = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; g < blocks;
       g += (int64_t)gridDim.x * blockDim.x) {
    const float4 *p = reinterpret_cast<const float4 *>(src + g * 32);
    float x[32];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float4 v = p[i];
      x[4 * i + 0] = v.x;
      x[4 * i + 1] = v.y;
      x[4 * i + 2] = v.z;
      x[4 * i + 3] = v.w;
    }
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(x[i]));
    uint32_t w[4] = {0u, 0u, 0u, 0u};
    uint8_t eb = 0;
    if (amax > 0.0f) {
      int s = floor_log2_pos(amax) - 2;
      s = s < -127 ? -127 : (s > 127 ? 127 : s);
      eb = (uint8_t)(s + 127);
      const float X = pow2_f32(s);
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const float y = __fdiv_rn(x[i], X);
        uint32_t c = e2m1_mag_code(fabsf(y));
        if (c != 0u && x[i] < 0.0f) c |= 8u;
        w[i >> 3] |= c << (4 * (i & 7));
      }
    }
    reinterpret_cast<uint4 *>(codes)[g] = make_uint4(w[0], w[1], w[2], w[3]);
    exps[g] = eb;
  }
}

// Eight E2M1 codes (one word, element order) -> two words of four int8
// values, each twice the E2M1 value (an integer in {0, +-1, +-2, +-3, +-4,
// +-6, +-8, +-12}), element order: byte permutes from a magnitude table and
// its negation, chosen per byte by the code's sign bit (replicated into a
// byte mask by the permute's sign mode).
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}
__device__ __forceinline__ void e2m1x8_to_i8x8(uint32_t w, uint32_t &lo, uint32_t &hi) {
  constexpr uint32_t kPos0 = 0x03020100u, kPos1 = 0x0C080604u;  // 0 1 2 3 | 4 6 8 12
  constexpr uint32_t kNeg0 = 0xFDFEFF00u, kNeg1 = 0xF4F8FAFCu;  // their negations
  const uint32_t a = w << 4;  // even elements' sign bits to their byte's top bit
  const uint32_t sl = w & 0x7777u, sh = (w >> 16) & 0x7777u;
  const uint32_t ml = prmt(a, w, 0xD9C8u), mh = prmt(a, w, 0xFBEAu);  // 0xFF where negative
  lo = (prmt(kPos0, kPos1, sl) & ~ml) | (prmt(kNeg0, kNeg1, sl) & ml);
  hi = (prmt(kPos0, kPos1, sh) & ~mh) | (prmt(kNeg0, kNeg1, sh) & mh);
}

// Index score of one FP4 key (this library's reading, see the header of the
// FP4 index key calls): per head h and key block b the exact integer
// idot = sum over the block of q[h, i] * (2 * E2M1(code_i)), the head's dot
// = fp32 sum over the blocks in ascending order of idot * 2^(exp_b - 128),
// score = ((0 + w_0 * dot_0) + w_1 * dot_1) + ... + 0 (each op rounded).
// kc: the key's NB x 16 code bytes, ke: its NB exponent bytes (shared
// memory).  The thread visits block c ^ x at step c (bank-conflict-free
// rotation); its query is either in registers, pre-permuted the same way
// (qreg[(h * NB + c) * 2 + u] = query int4 u of block c ^ x), or in shared
// memory in natural order (qs).
template <int NB, int HI, bool QREG>
__device__ __forceinline__ float fp4_key_score(const unsigned char *kc, const unsigned char *ke,
                                               const int4 *qreg, const int4 *qs,
                                               const float *wh, int x) {
  uint32_t ew = 0;
#pragma unroll
  for (int b = 0; b < NB; ++b) ew |= (uint32_t)ke[b] << (8 * b);
  float term[HI][NB];
#pragma unroll
  for (int cc = 0; cc < NB; ++cc) {
    const int blk = cc ^ x;
    const int4 kv = *reinterpret_cast<const int4 *>(kc + (blk << 4));
    uint32_t kw[8];
    e2m1x8_to_i8x8((uint32_t)kv.x, kw[0], kw[1]);
    e2m1x8_to_i8x8((uint32_t)kv.y, kw[2], kw[3]);
    e2m1x8_to_i8x8((uint32_t)kv.z, kw[4], kw[5]);
    e2m1x8_to_i8x8((uint32_t)kv.w, kw[6], kw[7]);
    const float scale = pow2_f32((int)((ew >> (8 * blk)) & 0xffu) - 128);
#pragma unroll
    for (int h = 0; h < HI; ++h) {
      int4 q0, q1;
      if constexpr (QREG) {
        q0 = qreg[(h * NB + cc) * 2 + 0];
        q1 = qreg[(h * NB + cc) * 2 + 1];
      } else {
        q0 = qs[(h * NB + blk) * 2 + 0];
        q1 = qs[(h * NB + blk) * 2 + 1];
      }
      int idot = 0;
      idot = __dp4a((int)kw[0], q0.x, idot);
      idot = __dp4a((int)kw[1], q0.y, idot);
      idot = __dp4a((int)kw[2], q0.z, idot);
      idot = __dp4a((int)kw[3], q0.w, idot);
      idot = __dp4a((int)kw[4], q1.x, idot);
      idot = __dp4a((int)kw[5], q1.y, idot);
      idot = __dp4a((int)kw[6], q1.z, idot);
      idot = __dp4a((int)kw[7], q1.w, idot);
      const float t = __fmul_rn(__int2float_rn(idot), scale);
#pragma unroll
      for (int b = 0; b < NB; ++b)
        if (b == blk) term[h][b] = t;
    }
  }
  float acc = 0.0f;
#pragma unroll
  for (int h = 0; h < HI; ++h) {
    float dot = 0.0f;
#pragma unroll
    for (int b = 0; b < NB; ++b) dot = __fadd_rn(dot, term[h][b]);
    acc = __fadd_rn(acc, __fmul_rn(wh[h], dot));
  }
  return __fadd_rn(acc, 0.0f);
}

// Four E2M1 codes pairs (one 32-bit word = 8 codes) -> 8 fp32 values times a
// scale, through the sm_100a hardware converter (e2m1x2 -> f16x2, exact).
__device__ __forceinline__ void e2m1x8_to_f32(uint32_t word, float s, float *out) {
  uint32_t h0, h1, h2, h3;
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "mov.b32 {b0, b1, b2, b3}, %4;\n\t"
      "cvt.rn.f16x2.e2m1x2 %0, b0;\n\t"
      "cvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
      "cvt.rn.f16x2.e2m1x2 %2, b2;\n\t"
      "cvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
      : "=r"(h0), "=r"(h1), "=r"(h2), "=r"(h3)
      : "r"(word));
  const uint32_t h[4] = {h0, h1, h2, h3};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    __half2 v = *reinterpret_cast<const __half2 *>(&h[i]);
    float2 f = __half22float2(v);
    out[2 * i + 0] = __fmul_rn(f.x, s);
    out[2 * i + 1] = __fmul_rn(f.y, s);
  }
}

// One thread per group of 16 elements.
__global__ void __launch_bounds__(256) unpack_fp4_kernel(const uint8_t *__restrict__ codes,
                                                         const float *__restrict__ scales,
                                                         int64_t groups, float *__restrict__ out) {
  for (int64_t g = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; g < groups;
       g += (int64_t)gridDim.x * blockDim.x) {
    const uint2 c = reinterpret_cast<const uint2 *>(codes)[g];
    const float s = scales[g];
    float v[16];
    e2m1x8_to_f32(c.x, s, v);
    e2m1x8_to_f32(c.y, s, v + 8);
    float4 *o = reinterpret_cast<float4 *>(out + g * 16);
#pragma unroll
    for (int i = 0; i < 4; ++i) o[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
  }
}

}  // namespace csa2
