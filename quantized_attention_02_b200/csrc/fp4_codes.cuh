// fp4_codes.cuh -- E2M1 / E4M3 conversions and the microscaling of one group of 16 values,
// used by the FP4 quantization kernels (the conversions also by the FP4 attention kernel).
//
// Microscaling (SageAttention3 entry: microscaling FP4 attention; the format is the
// one Blackwell's block-scaled FP4 products read): one UE4M3 scale per 16 elements along the
// contraction dimension, e4m3(fl32(max|z| / 6)); codes e2m1(fl32(z * fl32(1 / scale))), a zero
// scale giving zero codes.
#pragma once
#include <cuda_fp16.h>
#include <cstdint>

namespace sage {

// One fp32 value to its E4M3 code (round to nearest even, saturating).
__device__ __forceinline__ uint32_t e4m3_code(float t) {
  uint16_t h;  // cvt packs its first source into the upper byte
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(h) : "f"(0.f), "f"(t));
  return h & 0xFFu;
}

// Value of an E4M3 code (exact in fp32); the code is placed in both bytes so that either half
// of the converted pair holds it.
__device__ __forceinline__ float e4m3_value(uint32_t code) {
  const uint16_t pair = static_cast<uint16_t>(code | (code << 8));
  uint32_t h2;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(pair));
  return __half2float(__ushort_as_half(static_cast<unsigned short>(h2 & 0xFFFFu)));
}

// Eight fp32 values to E2M1 (round to nearest even, saturating), element 0 in the low nibble.
__device__ __forceinline__ uint32_t e2m1x8(const float* y) {
  uint32_t out;
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
      "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
      : "=r"(out)
      : "f"(y[0]), "f"(y[1]), "f"(y[2]), "f"(y[3]), "f"(y[4]), "f"(y[5]), "f"(y[6]), "f"(y[7]));
  return out;
}

// Microscaling of one group of 16 values z: two words of codes and the scale's code.
__device__ __forceinline__ uint32_t microscale16(const float (&z)[16], uint32_t& w0, uint32_t& w1) {
  float gm = 0.f;
#pragma unroll
  for (int k = 0; k < 16; ++k) gm = fmaxf(gm, fabsf(z[k]));
  const uint32_t s8 = e4m3_code(__fdiv_rn(gm, 6.0f));
  const float sd = e4m3_value(s8);
  const float inv = sd > 0.f ? __frcp_rn(sd) : 0.f;
  float y[16];
#pragma unroll
  for (int k = 0; k < 16; ++k) y[k] = __fmul_rn(z[k], inv);
  w0 = e2m1x8(y);
  w1 = e2m1x8(y + 8);
  return s8;
}

}  // namespace sage
