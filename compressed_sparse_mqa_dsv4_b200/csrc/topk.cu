// Per-query TopK over the indexer scores ("CSA And HCA: Definition, State, And Cost Model",
// s3.1: S_t = TopK_{s in E_t}(I_{t,s}, k)); per-query valid counts as in pypto-lib PR #834
// (cmp_counts).
//
// S_t is a set. The kernel returns the k_eff = min(k, E_t) entries with the largest scores
// (ties at the threshold go to the lower entry index) in ascending entry order, padded with
// -1. One CTA of 256 threads per query:
//   E_t <= k : every entry is selected, no score is read;
//   otherwise: a 4-pass MSB radix select over order-preserving 32-bit keys (8-bit digits,
//   shared-memory histograms, one block suffix scan per pass) finds the k_eff-th largest key
//   T; then each thread counts, over its contiguous range of entries, the keys above T and
//   those equal to T; two block exclusive scans give every thread its output offset and its
//   share of the ties, and the selected indices are written in entry order.
#include "dsv4_common.cuh"
#include "index_common.cuh"

namespace dsv4 {

constexpr int TOPK_THREADS = 256;

__device__ __forceinline__ uint32_t score_key(float s) {
  s = s + 0.0f;                                  // fold -0 into +0
  const uint32_t u = __float_as_uint(s);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Block-wide exclusive prefix sum over the 256 threads; also returns the total.
__device__ __forceinline__ int block_exclusive_scan(int v, int* warp_tot, int& total) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  int incl = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int t = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += t;
  }
  if (lane == 31) warp_tot[wid] = incl;
  __syncthreads();
  int before = 0;
  total = 0;
#pragma unroll
  for (int w = 0; w < TOPK_THREADS / 32; ++w) {
    const int t = warp_tot[w];
    before += w < wid ? t : 0;
    total += t;
  }
  __syncthreads();
  return before + incl - v;
}

__global__ void __launch_bounds__(TOPK_THREADS) topk_kernel(IndexArgs a, int q_begin) {
  __shared__ int hist[256];
  __shared__ int warp_tot[TOPK_THREADS / 32];
  __shared__ int sh_sel, sh_above;
  const int qg = q_begin + blockIdx.x;
  const int b = qg / a.nq, i = qg % a.nq;
  const int Et = visible_entries(a, b, i);
  const int k = a.k;
  const int keff = min(k, Et);
  int32_t* out = a.idx + (long long)qg * k;
  if (threadIdx.x == 0) a.counts[qg] = keff;
  for (int j = keff + threadIdx.x; j < k; j += blockDim.x) out[j] = -1;
  if (keff == 0) return;
  if (Et <= k) {                                  // every visible entry is selected
    for (int j = threadIdx.x; j < Et; j += blockDim.x) out[j] = j;
    return;
  }
  const float* sc = a.scores + (long long)(qg - a.score_q0) * a.scores_ld;

  // ---- radix select of the keff-th largest key
  uint32_t prefix = 0, pmask = 0;
  int remaining = keff;                           // still to take at or below the prefix
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    hist[threadIdx.x] = 0;
    __syncthreads();
    for (int j = threadIdx.x; j < Et; j += blockDim.x) {
      const uint32_t key = score_key(__ldg(sc + j));
      if ((key & pmask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1);
    }
    __syncthreads();
    // suffix sums over digits: thread t owns digit 255 - t, so an exclusive prefix over
    // threads is the count of keys in higher digits
    const int d = 255 - threadIdx.x;
    const int h = hist[d];
    int tot;
    const int above = block_exclusive_scan(h, warp_tot, tot);
    if (above < remaining && remaining <= above + h) {
      sh_sel = d;
      sh_above = above;
    }
    __syncthreads();
    remaining -= sh_above;
    prefix |= (uint32_t)sh_sel << shift;
    pmask |= 255u << shift;
    __syncthreads();
  }
  const uint32_t T = prefix;
  const int need_eq = remaining;                  // keys equal to T to take (lowest index first)

  // ---- order-preserving compaction over contiguous per-thread ranges
  const int per = (Et + TOPK_THREADS - 1) / TOPK_THREADS;
  const int lo = threadIdx.x * per, hi = min(Et, lo + per);
  int n_gt = 0, n_eq = 0;
  for (int j = lo; j < hi; ++j) {
    const uint32_t key = score_key(__ldg(sc + j));
    n_gt += key > T;
    n_eq += key == T;
  }
  int tot;
  const int eq_before = block_exclusive_scan(n_eq, warp_tot, tot);
  const int take_eq = max(0, min(n_eq, need_eq - eq_before));
  const int pos0 = block_exclusive_scan(n_gt + take_eq, warp_tot, tot);
  int pos = pos0, eq_seen = 0;
  for (int j = lo; j < hi; ++j) {
    const uint32_t key = score_key(__ldg(sc + j));
    if (key > T || (key == T && eq_seen++ < take_eq)) {
      if (pos < keff) out[pos] = j;
      ++pos;
    }
  }
}

int launch_topk(const IndexArgs& a, int q_begin, int q_count, cudaStream_t st) {
  if (q_count <= 0) return DSV4_OK;
  topk_kernel<<<q_count, TOPK_THREADS, 0, st>>>(a, q_begin);
  return launch_status("top-k select");
}

}  // namespace dsv4
