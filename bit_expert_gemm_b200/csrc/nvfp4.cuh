// NVFP4 helpers shared by the quantiser and the block-scaled GEMM.
#pragma once

#include "common.cuh"

namespace moe {

// Largest decode batch the CUDA-core NVFP4 path takes (decode_fp4.cu).
constexpr int kFp4DecodeMaxT = 16;

// FP32 -> E4M3 (round to nearest even, saturating to +-448).
__device__ __forceinline__ uint32_t f32_to_e4m3(float v) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.0f), "f"(v));
  return r & 0xFFu;
}

// E4M3 -> FP32 (exact: every E4M3 value is an FP16 value).
__device__ __forceinline__ float e4m3_to_f32(uint32_t code) {
  uint32_t packed;
  const uint16_t c16 = uint16_t(code & 0xFFu);
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(packed) : "h"(c16));
  return __half2float(__ushort_as_half(uint16_t(packed & 0xFFFFu)));
}

// Eight FP32 values -> eight E2M1 codes (round to nearest even, saturating
// to +-6), element 2j in the low nibble of byte j.
__device__ __forceinline__ uint32_t f32x8_to_e2m1(const float (&q)[8]) {
  uint32_t r;
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
      "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
      : "=r"(r)
      : "f"(q[0]), "f"(q[1]), "f"(q[2]), "f"(q[3]), "f"(q[4]), "f"(q[5]), "f"(q[6]), "f"(q[7]));
  return r;
}

// Quantises one block of 16 values with global scale s_g (the recipe in
// include/moe.h, every operation an IEEE FP32 round-to-nearest-even):
//   s_b = e4m3(amax / (6 s_g)),  c = e2m1(v / (e4m3(s_b) s_g)),  c = +0 if that is 0.
// Returns the scale code; codes[0..1] receive the 16 packed nibbles.
__device__ __forceinline__ uint32_t nvfp4_quant_block(const float (&v)[16], float s_g, uint32_t (&codes)[2]) {
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(v[i]));
  const float t = __fmul_rn(6.0f, s_g);
  const uint32_t sb = t > 0.0f ? f32_to_e4m3(__fdiv_rn(amax, t)) : 0u;
  const float denom = __fmul_rn(e4m3_to_f32(sb), s_g);
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    float q[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) q[i] = denom > 0.0f ? __fdiv_rn(v[8 * h + i], denom) : 0.0f;
    codes[h] = f32x8_to_e2m1(q);
  }
  return sb;
}

// Global scale from an amax: s_g = amax / (6 * 448).
__device__ __forceinline__ float nvfp4_global_scale(float amax) { return __fdiv_rn(amax, 2688.0f); }

}  // namespace moe
