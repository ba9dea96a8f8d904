// dsv4_norm_rope: RMS normalisation and rotary position embedding of attention rows, in
// place ("CSA And HCA: Definition, State, And Cost Model", s5.2: every query head and the
// shared KV head are RMS-normalised right before core attention, and their last 64
// channels carry RoPE at the row's position; the output is rotated back at the query's).
//
// One warp per row: the sum of squares in fp32 across the row, x / sqrt(mean(x^2) + eps),
// then each rotated channel pair turned by its angle (rope.cuh); one rounding to the
// storage type at the end. HBM-bound: each row is read twice (the second read hits L1)
// and written once.
#include "dsv4_common.cuh"
#include "rope.cuh"

namespace dsv4 {

template <typename T>
__global__ void __launch_bounds__(256) norm_rope_kernel(T* __restrict__ x, const int32_t* __restrict__ pos,
                                                        long long rows, int rows_per_pos, int c,
                                                        int rope, int norm, int inverse, float eps) {
  const int lane = threadIdx.x & 31;
  const long long warps = (long long)gridDim.x * (blockDim.x >> 5);
  for (long long r = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); r < rows;
       r += warps) {
    T* xr = x + r * c;
    const long long p = __ldg(pos + r / rows_per_pos);
    if (p < 0) {
      if (lane == 0) flag_status(DSV4_ERR_DEVICE_BOUNDS);
      continue;
    }
    float scale = 1.f;
    if (norm) {
      float ss = 0.f;
      for (int d = lane; d < c; d += 32) {
        const float v = to_f32(xr[d]);
        ss = fmaf(v, v, ss);
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
      scale = 1.f / sqrtf(ss / (float)c + eps);
      for (int d = lane; d < c - rope; d += 32) xr[d] = from_f32<T>(to_f32(xr[d]) * scale);
    }
    for (int i = lane; i < rope / 2; i += 32) {
      const int d = c - rope + 2 * i;
      float a = to_f32(xr[d]) * scale, b = to_f32(xr[d + 1]) * scale;
      float cs, sn;
      rope_cos_sin(p, i, rope, cs, sn);
      rope_apply(a, b, cs, sn, inverse != 0);
      xr[d] = from_f32<T>(a);
      xr[d + 1] = from_f32<T>(b);
    }
  }
}

}  // namespace dsv4

extern "C" int dsv4_norm_rope(int dtype, void* x, const int32_t* pos, int64_t rows,
                              int rows_per_pos, int c, int rope, int norm, int inverse, float eps,
                              void* stream) {
  using namespace dsv4;
  if (rows < 0 || rows_per_pos < 1 || c < 1 || rope < 0 || rope > c || (rope & 1) ||
      (norm != 0 && norm != 1) || (inverse != 0 && inverse != 1) || !(eps >= 0.f))
    return fail(DSV4_ERR_INVALID_ARG,
                "dsv4_norm_rope: bad sizes rows=%lld rows_per_pos=%d c=%d rope=%d norm=%d inverse=%d",
                (long long)rows, rows_per_pos, c, rope, norm, inverse);
  if (rows == 0) return DSV4_OK;
  if (!x || !pos) return fail(DSV4_ERR_INVALID_ARG, "dsv4_norm_rope: NULL pointer");
  cudaStream_t st = (cudaStream_t)stream;
  long long blocks = (rows + 7) / 8;
  if (blocks > 148 * 32) blocks = 148 * 32;
  if (dtype == DSV4_F32)
    norm_rope_kernel<float><<<(int)blocks, 256, 0, st>>>(static_cast<float*>(x), pos, rows,
                                                         rows_per_pos, c, rope, norm, inverse, eps);
  else if (dtype == DSV4_BF16)
    norm_rope_kernel<__nv_bfloat16><<<(int)blocks, 256, 0, st>>>(
        static_cast<__nv_bfloat16*>(x), pos, rows, rows_per_pos, c, rope, norm, inverse, eps);
  else
    return fail(DSV4_ERR_INVALID_ARG, "dsv4_norm_rope: dtype %d not F32/BF16", dtype);
  return launch_status("dsv4_norm_rope");
}
