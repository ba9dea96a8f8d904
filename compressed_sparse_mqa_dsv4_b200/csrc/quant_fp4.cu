// dsv4_quantize_fp4: bf16 rows -> e2m1 codes + one E4M3 scale per 16 elements.
//
// The FP4 indexer path of "CSA And HCA: Definition, State, And Cost Model" (s3.1: the
// indexer attention is computed in FP4; s8 precision table: indexer Q/K cached, loaded
// and multiplied in 4-bit floating point). Group layout follows the block-scaled
// tensor-core operand format: 16 consecutive elements share one E4M3 scale.
//
// One thread per 16-element group: two 16-byte loads, one 8-byte store of codes and one
// scale byte. Rounding uses the sm_100a conversion instructions (round-to-nearest-even
// with saturation) on fp32 quotients computed with IEEE division.
#include "dsv4_common.cuh"
#include "fp4_quant.cuh"

namespace dsv4 {

__global__ void __launch_bounds__(256) quantize_fp4_kernel(
    const __nv_bfloat16* __restrict__ x, uint8_t* __restrict__ codes,
    uint8_t* __restrict__ scales, long long groups) {
  for (long long g = (long long)blockIdx.x * blockDim.x + threadIdx.x; g < groups;
       g += (long long)gridDim.x * blockDim.x) {
    float v[16];
    float a[8], b[8];
    load16_f32(x + g * 16, a);
    load16_f32(x + g * 16 + 8, b);
#pragma unroll
    for (int j = 0; j < 8; ++j) { v[j] = a[j]; v[8 + j] = b[j]; }
    uint32_t w0, w1, sb;
    fp4_quantize_group(v, w0, w1, sb);
    *reinterpret_cast<uint2*>(codes + g * 8) = make_uint2(w0, w1);
    scales[g] = (uint8_t)sb;
  }
}

}  // namespace dsv4

extern "C" int dsv4_quantize_fp4(const void* x, uint8_t* codes, uint8_t* scales, int64_t rows,
                                 int cols, void* stream) {
  using namespace dsv4;
  if (rows < 0 || cols < 0 || cols % 16 != 0)
    return fail(DSV4_ERR_INVALID_ARG, "dsv4_quantize_fp4: rows=%lld cols=%d (cols %% 16 != 0)",
                (long long)rows, cols);
  const long long groups = (long long)rows * (cols / 16);
  if (groups == 0) return DSV4_OK;
  if (!x || !codes || !scales)
    return fail(DSV4_ERR_INVALID_ARG, "dsv4_quantize_fp4: NULL pointer");
  if (!aligned16(x) || (reinterpret_cast<uintptr_t>(codes) & 7u))
    return fail(DSV4_ERR_INVALID_ARG, "dsv4_quantize_fp4: x must be 16-byte and codes 8-byte aligned");
  long long blocks = (groups + 255) / 256;
  if (blocks > 148LL * 32) blocks = 148LL * 32;
  quantize_fp4_kernel<<<(int)blocks, 256, 0, (cudaStream_t)stream>>>(
      (const __nv_bfloat16*)x, codes, scales, groups);
  return launch_status("dsv4_quantize_fp4");
}
