// FP8 main-KV entries (layout and rounding in fp8_kv.cuh): quantisation of bf16 / fp32 rows,
// the exact-as-bf16 expansion back, and attention of decode queries over an FP8 pool (the
// selected rows are gathered and expanded to bf16 next to the query, then the tensor-core
// attention runs on them).
#include "attn_common.cuh"
#include "fp8_kv.cuh"

namespace dsv4 {

// One warp per row: the FP8 groups two channels per lane, then the RoPE channels as bf16.
template <typename T>
__global__ void __launch_bounds__(256) quantize_main_kv_kernel(
    const T* __restrict__ x, uint8_t* __restrict__ codes, float* __restrict__ scales,
    __nv_bfloat16* __restrict__ rope_out, long long rows, int c, int rope) {
  const int lane = threadIdx.x & 31;
  const int nf = c - rope, ng = nf / kFp8Group;
  const long long warps = (long long)gridDim.x * (blockDim.x >> 5);
  for (long long r = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); r < rows;
       r += warps) {
    const T* xr = x + r * c;
    for (int g = 0; g < ng; ++g) {
      const int ch = g * kFp8Group + 2 * lane;
      uint32_t code2;
      const float s = fp8_group_quantize(to_f32(xr[ch]), to_f32(xr[ch + 1]), code2);
      *reinterpret_cast<uint16_t*>(codes + r * nf + ch) = (uint16_t)code2;
      if (lane == 0) scales[r * ng + g] = s;
    }
    for (int d = lane; d < rope; d += 32) rope_out[r * rope + d] = __float2bfloat16_rn(to_f32(xr[nf + d]));
  }
}

// One warp per row: bf16 row = RNE_bf16(E4M3 value * scale), rounded once, and the RoPE
// channels as stored.
__global__ void __launch_bounds__(256) dequantize_main_kv_kernel(
    const uint8_t* __restrict__ codes, const float* __restrict__ scales,
    const __nv_bfloat16* __restrict__ rope_in, __nv_bfloat16* __restrict__ out, long long rows,
    int c, int rope) {
  const int lane = threadIdx.x & 31;
  const int nf = c - rope, ng = nf / kFp8Group;
  const long long warps = (long long)gridDim.x * (blockDim.x >> 5);
  for (long long r = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); r < rows;
       r += warps) {
    for (int g = 0; g < ng; ++g) {
      const int ch = g * kFp8Group + 2 * lane;
      const float s = scales[r * ng + g];
      const uint32_t c2 = *reinterpret_cast<const uint16_t*>(codes + r * nf + ch);
      __nv_bfloat162 v;
      v.x = fp8_dequant_bf16(c2 & 0xFFu, s);
      v.y = fp8_dequant_bf16(c2 >> 8, s);
      *reinterpret_cast<__nv_bfloat162*>(out + r * c + ch) = v;
    }
    for (int d = lane; d < rope; d += 32) out[r * c + nf + d] = rope_in[r * rope + d];
  }
}

// Decode attention over an FP8 pool, stage 1: one warp per (sequence b, slot j < k). A valid
// selection idx[b, j] < floor((t+1)/m) of a row inside the pool is expanded to bf16 into
// staging row b*k + j and listed as candidate j; an invalid one is listed as -1 (the
// attention kernel skips and reports it). Also writes the staging row offsets b*k.
__global__ void __launch_bounds__(256) gather_main_kv_kernel(
    const uint8_t* __restrict__ codes, const float* __restrict__ scales,
    const __nv_bfloat16* __restrict__ rope_in, long long pool_rows,
    const int64_t* __restrict__ kv_row_off, const int32_t* __restrict__ idx,
    const int32_t* __restrict__ counts, const int32_t* __restrict__ q_pos0, int B, int k, int c,
    int rope, int m, __nv_bfloat16* __restrict__ staged, int32_t* __restrict__ idx2,
    int64_t* __restrict__ off2) {
  const int lane = threadIdx.x & 31;
  const long long item = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (item >= (long long)B * k) return;
  const int b = (int)(item / k), j = (int)(item % k);
  if (j == 0 && lane == 0) off2[b] = (int64_t)b * k;
  int cnt = counts[b];
  cnt = cnt < 0 ? 0 : (cnt > k ? k : cnt);
  if (j >= cnt) {
    if (lane == 0) idx2[item] = -1;
    return;
  }
  const long long Et = ((long long)q_pos0[b] + 1) / m;
  const long long s = idx[item];
  const long long row = kv_row_off[b] + s;
  if (s < 0 || s >= Et || row < 0 || row >= pool_rows) {
    if (lane == 0) idx2[item] = -1;                 // skipped and reported by the attention
    return;
  }
  if (lane == 0) idx2[item] = j;
  const int nf = c - rope, ng = nf / kFp8Group;
  __nv_bfloat16* dst = staged + item * c;
  for (int g = 0; g < ng; ++g) {
    const int ch = g * kFp8Group + 2 * lane;
    const float sc = scales[row * ng + g];
    const uint32_t c2 = *reinterpret_cast<const uint16_t*>(codes + row * nf + ch);
    __nv_bfloat162 v;
    v.x = fp8_dequant_bf16(c2 & 0xFFu, sc);
    v.y = fp8_dequant_bf16(c2 >> 8, sc);
    *reinterpret_cast<__nv_bfloat162*>(dst + ch) = v;
  }
  for (int d = lane; d < rope; d += 32) dst[nf + d] = rope_in[row * rope + d];
}

static long long round256(long long v) { return (v + 255) / 256 * 256; }

}  // namespace dsv4

using namespace dsv4;

static int check_fp8_shape(const char* who, int c, int rope) {
  if (c < 1 || rope < 0 || rope > c || (rope & 1) || (c - rope) % kFp8Group != 0)
    return fail(DSV4_ERR_INVALID_ARG, "%s: c=%d rope=%d (c - rope must be a multiple of %d)", who, c,
                rope, kFp8Group);
  return DSV4_OK;
}

extern "C" int dsv4_quantize_main_kv(int dtype, const void* x, uint8_t* codes, float* scales,
                                     void* rope_out, int64_t rows, int c, int rope, void* stream) {
  int s = check_fp8_shape("dsv4_quantize_main_kv", c, rope);
  if (s != DSV4_OK) return s;
  if (rows < 0) return fail(DSV4_ERR_INVALID_ARG, "dsv4_quantize_main_kv: rows %lld", (long long)rows);
  if (rows == 0) return DSV4_OK;
  if (!x || !codes || !scales || (rope > 0 && !rope_out))
    return fail(DSV4_ERR_INVALID_ARG, "dsv4_quantize_main_kv: NULL pointer");
  if ((reinterpret_cast<uintptr_t>(codes) & 1u) || (reinterpret_cast<uintptr_t>(x) & 3u))
    return fail(DSV4_ERR_INVALID_ARG, "dsv4_quantize_main_kv: codes must be 2-byte, x 4-byte aligned");
  long long blocks = (rows + 7) / 8;
  if (blocks > 148 * 32) blocks = 148 * 32;
  cudaStream_t st = (cudaStream_t)stream;
  if (dtype == DSV4_F32)
    quantize_main_kv_kernel<float><<<(int)blocks, 256, 0, st>>>(
        (const float*)x, codes, scales, (__nv_bfloat16*)rope_out, rows, c, rope);
  else if (dtype == DSV4_BF16)
    quantize_main_kv_kernel<__nv_bfloat16><<<(int)blocks, 256, 0, st>>>(
        (const __nv_bfloat16*)x, codes, scales, (__nv_bfloat16*)rope_out, rows, c, rope);
  else
    return fail(DSV4_ERR_INVALID_ARG, "dsv4_quantize_main_kv: dtype %d not F32/BF16", dtype);
  return launch_status("dsv4_quantize_main_kv");
}

extern "C" int dsv4_dequantize_main_kv(const uint8_t* codes, const float* scales,
                                       const void* rope_in, void* out, int64_t rows, int c,
                                       int rope, void* stream) {
  int s = check_fp8_shape("dsv4_dequantize_main_kv", c, rope);
  if (s != DSV4_OK) return s;
  if (rows < 0) return fail(DSV4_ERR_INVALID_ARG, "dsv4_dequantize_main_kv: rows %lld", (long long)rows);
  if (rows == 0) return DSV4_OK;
  if (!codes || !scales || !out || (rope > 0 && !rope_in))
    return fail(DSV4_ERR_INVALID_ARG, "dsv4_dequantize_main_kv: NULL pointer");
  if ((reinterpret_cast<uintptr_t>(codes) & 1u) || (reinterpret_cast<uintptr_t>(out) & 3u))
    return fail(DSV4_ERR_INVALID_ARG, "dsv4_dequantize_main_kv: codes must be 2-byte, out 4-byte aligned");
  long long blocks = (rows + 7) / 8;
  if (blocks > 148 * 32) blocks = 148 * 32;
  dequantize_main_kv_kernel<<<(int)blocks, 256, 0, (cudaStream_t)stream>>>(
      codes, scales, (const __nv_bfloat16*)rope_in, (__nv_bfloat16*)out, rows, c, rope);
  return launch_status("dsv4_dequantize_main_kv");
}

extern "C" size_t dsv4_hybrid_sparse_attn_fp8_workspace_size(int B, int H, int c, int k) {
  if (B <= 0 || k <= 0 || c <= 0) return 0;
  return (size_t)(round256((long long)B * k * c * 2) + round256((long long)B * k * 4) +
                  round256((long long)B * 8) + dsv4_hybrid_sparse_attn_workspace_size(B, 1, H, c));
}

extern "C" int dsv4_hybrid_sparse_attn_fp8(const void* Q, const uint8_t* pool_codes,
                                           const float* pool_scales, const void* pool_rope,
                                           int64_t pool_rows, const int64_t* kv_row_off,
                                           const int32_t* idx, const int32_t* counts, int k,
                                           const void* local, int R, const int32_t* q_pos0,
                                           int B, int H, int c, int rope, int m, int w,
                                           const float* sink, float scale, void* O, float* lse,
                                           void* workspace, size_t workspace_bytes, void* stream) {
  int s = check_fp8_shape("dsv4_hybrid_sparse_attn_fp8", c, rope);
  if (s != DSV4_OK) return s;
  if (B < 0 || k < 1 || m < 1 || w < 1 || R < 1 || H < 1 || pool_rows < 0)
    return fail(DSV4_ERR_INVALID_ARG, "dsv4_hybrid_sparse_attn_fp8: bad sizes B=%d k=%d m=%d w=%d R=%d H=%d",
                B, k, m, w, R, H);
  if (B == 0) return DSV4_OK;
  if (!Q || !pool_codes || !pool_scales || (rope > 0 && !pool_rope) || !kv_row_off || !idx ||
      !counts || !local || !q_pos0 || !O)
    return fail(DSV4_ERR_INVALID_ARG, "dsv4_hybrid_sparse_attn_fp8: NULL pointer");
  if ((reinterpret_cast<uintptr_t>(pool_codes) & 1u))
    return fail(DSV4_ERR_INVALID_ARG, "dsv4_hybrid_sparse_attn_fp8: pool codes must be 2-byte aligned");
  const size_t need = dsv4_hybrid_sparse_attn_fp8_workspace_size(B, H, c, k);
  if (!workspace || workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return fail(DSV4_ERR_WORKSPACE, "dsv4_hybrid_sparse_attn_fp8: workspace %zu bytes < %zu (256-byte aligned)",
                workspace_bytes, need);
  char* base = static_cast<char*>(workspace);
  __nv_bfloat16* staged = reinterpret_cast<__nv_bfloat16*>(base);
  base += round256((long long)B * k * c * 2);
  int32_t* idx2 = reinterpret_cast<int32_t*>(base);
  base += round256((long long)B * k * 4);
  int64_t* off2 = reinterpret_cast<int64_t*>(base);
  base += round256((long long)B * 8);
  const long long warps = (long long)B * k;
  gather_main_kv_kernel<<<(unsigned)((warps + 7) / 8), 256, 0, (cudaStream_t)stream>>>(
      pool_codes, pool_scales, (const __nv_bfloat16*)pool_rope, pool_rows, kv_row_off, idx, counts,
      q_pos0, B, k, c, rope, m, staged, idx2, off2);
  s = launch_status("dsv4_hybrid_sparse_attn_fp8 (gather)");
  if (s != DSV4_OK) return s;
  // the candidates of sequence b are its staged rows b*k + j: index j, visibility already
  // checked against the query's completed entries
  return dsv4_hybrid_sparse_attn(DSV4_BF16, Q, staged, (int64_t)B * k, off2, idx2, counts, k, local,
                                 R, q_pos0, B, 1, H, c, m, w, sink, scale, O, lse, base,
                                 workspace_bytes - (size_t)(base - static_cast<char*>(workspace)),
                                 stream);
}
