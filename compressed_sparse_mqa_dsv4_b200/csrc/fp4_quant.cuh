// Block-scaled FP4 quantisation of one group of 16 values (e2m1 codes + one E4M3 scale),
// shared by dsv4_quantize_fp4 and the FP4 emission of the decode state ("CSA And HCA:
// Definition, State, And Cost Model", s3.1 and the s8 precision table: the indexer keys are
// cached in 4-bit floating point).
//   scale = RNE_E4M3(amax / 6) (fp32 quotient, IEEE division, saturating at 448);
//   code  = RNE_e2m1(x / scale) (fp32 quotient, saturating at +-6); a zero scale gives codes 0.
// Rounding uses the sm_100a conversion instructions (round-to-nearest-even, saturating).
#pragma once
#include "dsv4_common.cuh"

namespace dsv4 {

// e4m3 byte -> float (exact): exponent field 0 is subnormal (m * 2^-9).
__device__ __forceinline__ float e4m3_to_float(uint32_t b) {
  const uint32_t e = (b >> 3) & 15u, mt = b & 7u;
  float v = e == 0 ? (float)mt * 0x1p-9f : (float)(8u + mt) * exp2f((float)e - 10.f);
  return (b & 0x80u) ? -v : v;
}

__device__ __forceinline__ uint32_t f32_to_e4m3_rn_sat(float x) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.0f), "f"(x));
  return r & 0xFFu;  // second source operand lands in the low byte
}

// two fp32 -> one byte of e2m1 codes: `lo` in bits 0..3, `hi` in bits 4..7
__device__ __forceinline__ uint32_t f32x2_to_e2m1_rn_sat(float lo, float hi) {
  uint32_t r;
  asm("{\n .reg .b8 t;\n cvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n cvt.u32.u8 %0, t;\n}"
      : "=r"(r) : "f"(hi), "f"(lo));
  return r & 0xFFu;
}

// 16 values -> codes (element 2j in the low nibble of byte j: bytes 0-3 in w0, 4-7 in w1) and
// the scale byte
__device__ __forceinline__ void fp4_quantize_group(const float (&v)[16], uint32_t& w0, uint32_t& w1,
                                                   uint32_t& sb) {
  float amax = 0.f;
#pragma unroll
  for (int j = 0; j < 16; ++j) amax = fmaxf(amax, fabsf(v[j]));
  sb = f32_to_e4m3_rn_sat(__fdiv_rn(amax, 6.0f));
  const float s = e4m3_to_float(sb);
  w0 = 0;
  w1 = 0;
  if (s > 0.f) {
#pragma unroll
    for (int j = 0; j < 8; j += 2) {
      w0 |= f32x2_to_e2m1_rn_sat(__fdiv_rn(v[j], s), __fdiv_rn(v[j + 1], s)) << (4 * j);
      w1 |= f32x2_to_e2m1_rn_sat(__fdiv_rn(v[8 + j], s), __fdiv_rn(v[9 + j], s)) << (4 * j);
    }
  }
}

}  // namespace dsv4
