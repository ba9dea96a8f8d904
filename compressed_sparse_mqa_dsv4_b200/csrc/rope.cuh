// Rotary position embedding of "CSA And HCA: Definition, State, And Cost Model", s5.2: the
// last `rope` channels of a query head, of a compressed entry and of a local entry are
// rotated by their position; the attention output's last `rope` channels are rotated back at
// the query's position. Channel pair i (channels c - rope + 2i, c - rope + 2i + 1) turns by
// the angle p * 10000^(-2i / rope) (adjacent pairs, base 10000: the pages fix which channels
// rotate and the positions, not the pairing or the base).
#pragma once

#include <cuda_runtime.h>

namespace dsv4 {

// cos and sin of pair i's angle at position p. Positions reach 2^20 and more, where a
// single-precision angle would be off by a large fraction of a radian, so the angle is
// formed and reduced to [-pi, pi] in double precision before the single-precision sine and
// cosine of the remainder.
__device__ __forceinline__ void rope_cos_sin(long long p, int i, int rope, float& cs, float& sn) {
  const double two_pi = 6.283185307179586476925286766559;
  const double ang = (double)p * pow(10000.0, -2.0 * (double)i / (double)rope);
  const double r = ang - two_pi * rint(ang / two_pi);
  sincosf((float)r, &sn, &cs);
}

// Rotate the pair (a, b) by the angle whose cos / sin are given; inverse rotates by minus it.
__device__ __forceinline__ void rope_apply(float& a, float& b, float cs, float sn, bool inverse) {
  if (inverse) sn = -sn;
  const float x = a * cs - b * sn;
  const float y = a * sn + b * cs;
  a = x;
  b = y;
}

}  // namespace dsv4
