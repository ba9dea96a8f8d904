// Shared declarations of the indexer / top-k kernels.
#pragma once
#include <cuda_fp16.h>

#include "dsv4_common.cuh"

namespace dsv4 {

struct IndexArgs {
  int qdtype;
  const void* qI;
  const uint8_t* qI_scales;
  const float* w;
  const void* KI;
  const uint8_t* KI_scales;
  long long ki_rows;
  const int64_t* kv_row_off;
  const int32_t* q_pos0;
  int B, nq, H_I, c_I, m, k;
  int max_e;           // score row capacity: queries with more entries are clamped + flagged
  int32_t* idx;
  int32_t* counts;
  float* scores;       // score rows of queries [score_q0, score_q0 + rows)
  long long scores_ld;
  int score_q0;        // global query id of score row 0
  // Q rows the tensor-core kernel reads start at query q_map_q0 and number q_map_rows
  // (0: the whole request; the FP4 path reads a per-chunk bf16 expansion)
  int q_map_q0;
  long long q_map_rows;
  // top-k of long rows, one region of cand_row_bytes per score row:
  //  * topk_pipe = 1 (few rows, decode): threshold pipeline; the region holds hist1 of the
  //    top TK_H1_BITS key bits (TK_HDR bytes); hist1_done: the score kernel built hist1;
  //  * nseg > 1 (many rows): per-segment selection then a merge; the region holds nseg * k
  //    candidate scores, then their nseg * k entry indices.
  // k_fp4 = 1: K^I stays FP4 (KI = e2m1 codes [ki_rows, c_I/2], KI_scales = E4M3 [ki_rows,
  // c_I/16]) and is expanded inside the tensor-core score kernel; qI is then f16
  int k_fp4;
  int topk_pipe;
  int nseg;
  char* cand;
  long long cand_row_bytes;
  int hist1_done;
};

// Order-preserving 32-bit key of a score (larger score -> larger key; -0 folded into +0).
__device__ __forceinline__ uint32_t score_key(float s) {
  s = s + 0.0f;                                  // fold -0 into +0
  const uint32_t u = __float_as_uint(s);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// One histogram update per distinct bin among the warp's active lanes.
__device__ __forceinline__ void hist_add(int* hist, uint32_t bin, bool pred) {
  const uint32_t active = __ballot_sync(0xffffffffu, pred);
  if (!pred) return;
  const uint32_t same = __match_any_sync(active, bin);
  if ((threadIdx.x & 31) == __ffs(same) - 1) atomicAdd(&hist[bin], __popc(same));
}

// Completed entries of query (b, i), clamped to the score-row capacity (flagged).
__device__ __forceinline__ int visible_entries(const IndexArgs& a, int b, int i) {
  const long long t = (long long)a.q_pos0[b] + i;
  long long Et = (t + 1) / a.m;
  if (Et < 0) Et = 0;
  if (Et > a.max_e) {
    flag_status(DSV4_ERR_DEVICE_BOUNDS);
    Et = a.max_e;
  }
  return (int)Et;
}

// e4m3 byte -> float (exact)
__device__ __forceinline__ float e4m3_decode(uint32_t b) {
  const uint32_t e = (b >> 3) & 15u, mt = b & 7u;
  float v = e == 0 ? (float)mt * 0x1p-9f : (float)(8u + mt) * exp2f((float)e - 10.f);
  return (b & 0x80u) ? -v : v;
}

__device__ __forceinline__ float e2m1_decode(uint32_t nib) {
  const float mag[8] = {0.f, 0.5f, 1.f, 1.5f, 2.f, 3.f, 4.f, 6.f};
  const float v = mag[nib & 7u];
  return (nib & 8u) ? -v : v;
}

// Element d of row `row` of an indexer operand, decoded to fp32.
template <int QD>
__device__ __forceinline__ float load_elem(const void* p, const uint8_t* scales, long long row,
                                           int d, int cols) {
  if (QD == DSV4_F32) return reinterpret_cast<const float*>(p)[row * cols + d];
  if (QD == DSV4_BF16)
    return __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(p)[row * cols + d]);
  const uint8_t byte = reinterpret_cast<const uint8_t*>(p)[row * (cols / 2) + d / 2];
  const uint32_t nib = (d & 1) ? (byte >> 4) : (byte & 15u);
  return e2m1_decode(nib) * e4m3_decode(scales[row * (cols / 16) + d / 16]);
}

// The threshold top-k's per-row region, zeroed before each score launch: hist1 [TK_H1_BINS]
// at byte 0 (the row's scores binned by the top TK_H1_BITS bits of their order-preserving
// keys). The int at byte TK_WORK_BYTE of a launch's first row hands out the score kernel's
// work units.
constexpr int TK_H1_BITS = 11;
constexpr int TK_H1_BINS = 1 << TK_H1_BITS;
constexpr int TK_HDR = 8448;
constexpr int TK_WORK_BYTE = 8192;

int launch_index_scores_simt(const IndexArgs& a, int q_begin, int q_count, int max_e,
                             cudaStream_t st);
// *used: the tensor-core kernel took the request; *hist1_built: it also built the threshold
// top-k's first histograms.
int launch_index_scores_tc(const IndexArgs& a, int q_begin, int q_count, int max_e,
                           cudaStream_t st, bool* used, bool* hist1_built);
int launch_topk(const IndexArgs& a, int q_begin, int q_count, cudaStream_t st);
// Zeroes the threshold top-k headers of the score rows of queries [q_begin, q_begin +
// q_count) (before the score kernel, which may build the first histogram).
int topk_prepare(const IndexArgs& a, int q_begin, int q_count, cudaStream_t st);
// Top-k scheme for a request of `rows` queries with up to max_entries entries and k winners:
// 0 single CTA per row, 1 segments + merge, 2 threshold pipeline; and the workspace bytes
// per score row it needs (0 for scheme 0).
int topk_scheme(int max_entries, int k, long long rows);
long long topk_row_bytes(int max_entries, int k, long long rows);
int topk_segments(int max_entries);
// FP4 codes [rows, cols/2] + E4M3 scales [rows, cols/16] -> bf16 [rows, cols] (exact).
int launch_fp4_expand(const uint8_t* codes, const uint8_t* scales, long long rows, int cols,
                      __nv_bfloat16* out, cudaStream_t st);
int launch_fp4_expand_f16(const uint8_t* codes, const uint8_t* scales, long long rows, int cols,
                          __half* out, cudaStream_t st);

}  // namespace dsv4
