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
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      float a = fabsf(x[i]);
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
    reinterpret_cast<uint2 *>(codes)[g] = make_uint2(lo, hi);
    scales[g] = s;
  }
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
