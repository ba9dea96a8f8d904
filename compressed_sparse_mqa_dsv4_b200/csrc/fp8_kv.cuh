// Production main-KV entry of "CSA And HCA: Definition, State, And Cost Model", s8 precision
// table: the non-RoPE channels of an entry in FP8 E4M3 and its last `rope` (RoPE) channels
// in bf16. The pages leave the scale metadata open; this library stores one fp32 scale per
// 64 consecutive FP8 channels: scale = fp32(amax / 448), code = RNE_E4M3(fp32(x / scale))
// saturating at 448 with the IEEE sign, and zero codes for a zero scale.
//
// Device layout of a pool of `rows` entries of c channels (c - rope a multiple of 64):
//   codes  uint8 [rows, c - rope]   (E4M3 fn bytes: sign << 7 | exponent << 3 | mantissa)
//   scales fp32  [rows, (c - rope) / 64]
//   rope   bf16  [rows, rope]
#pragma once

#include "dsv4_common.cuh"

namespace dsv4 {

constexpr int kFp8Group = 64;

// E4M3 (fn) byte of x: round to nearest even, saturating at 448, IEEE sign.
__device__ __forceinline__ uint32_t e4m3_byte(float x) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.0f), "f"(x));
  return r & 0xFFu;                                  // the second source lands in the low byte
}

// Exact value of an E4M3 (fn) byte, from its bit fields: exponent 0 is subnormal (m * 2^-9),
// otherwise (1 + m/8) * 2^(e - 7).
__device__ __forceinline__ float e4m3_value(uint32_t b) {
  const uint32_t e = (b >> 3) & 15u, mt = b & 7u;
  const float mag = e == 0 ? (float)mt * 0x1p-9f : __uint_as_float(((e + 120u) << 23) | (mt << 20));
  return (b & 0x80u) ? -mag : mag;
}

// One 64-channel group held by a warp, two channels per lane (v0 = channel 2*lane,
// v1 = channel 2*lane + 1): the group's scale and this lane's two codes (low byte v0).
__device__ __forceinline__ float fp8_group_quantize(float v0, float v1, uint32_t& code2) {
  float amax = fmaxf(fabsf(v0), fabsf(v1));
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
  const float scale = __fdiv_rn(amax, 448.0f);
  code2 = 0;
  if (scale > 0.f) code2 = e4m3_byte(__fdiv_rn(v0, scale)) | (e4m3_byte(__fdiv_rn(v1, scale)) << 8);
  return scale;
}

// bf16 of an E4M3 value times its group scale, rounded once (to nearest even): the product of
// a 4-bit and a 24-bit significand is exact in double precision.
__device__ __forceinline__ __nv_bfloat16 fp8_dequant_bf16(uint32_t code, float scale) {
  return __double2bfloat16((double)e4m3_value(code) * (double)scale);
}

}  // namespace dsv4
