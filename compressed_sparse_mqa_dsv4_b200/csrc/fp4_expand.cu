// Expansion of block-scaled FP4 indexer operands (e2m1 codes, one E4M3 scale per 16
// elements; "CSA And HCA: Definition, State, And Cost Model", s3.1 and the s8 precision
// table) to bf16 or f16 for the tensor-core score kernel.
//
// Every e2m1 magnitude has at most 2 significant bits and every E4M3 scale at most 4, so a
// code times its scale has at most 6 and is exact in bf16 (8 significant bits) and in f16
// (11; the products lie in [2^-10, 2688], inside f16's normal range): the expanded operands
// hold exactly the dequantised values, and the fp32-accumulated scores are those of the
// block-scaled FP4 product.
#include <cuda_fp16.h>

#include <type_traits>

#include "dsv4_common.cuh"
#include "index_common.cuh"

namespace dsv4 {
namespace {

// One thread per 16 elements (one scale): 8 code bytes in, 32 bytes of bf16 or f16 out.
template <typename T>
__global__ void __launch_bounds__(256) fp4_expand_kernel(const uint8_t* __restrict__ codes,
                                                         const uint8_t* __restrict__ scales,
                                                         long long groups, T* __restrict__ out) {
  const long long gi = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (gi >= groups) return;
  const uint2 cb = reinterpret_cast<const uint2*>(codes)[gi];
  const float sc = e4m3_decode(scales[gi]);
  uint32_t packed[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const uint32_t byte = ((i < 4 ? cb.x : cb.y) >> (8 * (i & 3))) & 255u;
    // element 2i in the low nibble, 2i+1 in the high nibble
    const float lo = e2m1_decode(byte & 15u) * sc, hi = e2m1_decode(byte >> 4) * sc;
    if constexpr (sizeof(T) == 2 && std::is_same<T, __half>::value) {
      __half2 p = __floats2half2_rn(lo, hi);
      packed[i] = *reinterpret_cast<uint32_t*>(&p);
    } else {
      __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);
      packed[i] = *reinterpret_cast<uint32_t*>(&p);
    }
  }
  uint4* o = reinterpret_cast<uint4*>(out + gi * 16);
  o[0] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
  o[1] = make_uint4(packed[4], packed[5], packed[6], packed[7]);
}

}  // namespace

template <typename T>
static int fp4_expand(const uint8_t* codes, const uint8_t* scales, long long rows, int cols, T* out,
                      cudaStream_t st) {
  const long long groups = rows * (cols / 16);
  if (groups <= 0) return DSV4_OK;
  if ((reinterpret_cast<uintptr_t>(codes) & 7u) || (reinterpret_cast<uintptr_t>(out) & 15u))
    return fail(DSV4_ERR_INVALID_ARG, "fp4 expand: misaligned codes or output");
  const long long blocks = (groups + 255) / 256;
  if (blocks > 0x7fffffffll) return fail(DSV4_ERR_UNSUPPORTED, "fp4 expand: %lld groups", groups);
  fp4_expand_kernel<T><<<(unsigned)blocks, 256, 0, st>>>(codes, scales, groups, out);
  return launch_status("fp4 expand");
}

int launch_fp4_expand(const uint8_t* codes, const uint8_t* scales, long long rows, int cols,
                      __nv_bfloat16* out, cudaStream_t st) {
  return fp4_expand(codes, scales, rows, cols, out, st);
}

int launch_fp4_expand_f16(const uint8_t* codes, const uint8_t* scales, long long rows, int cols,
                          __half* out, cudaStream_t st) {
  return fp4_expand(codes, scales, rows, cols, out, st);
}

}  // namespace dsv4
