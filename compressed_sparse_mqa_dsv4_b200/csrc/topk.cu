// Per-query TopK over the indexer scores ("CSA And HCA: Definition, State, And Cost
// Model", s3.1: S_t = TopK_{s in E_t}(I_{t,s}, k)); per-query valid counts as in
// pypto-lib PR #834 (cmp_counts).
//
// One CTA (1024 threads) per query. Scores are mapped to order-preserving 32-bit keys.
// Short rows (E_t <= 1024) are sorted whole. Longer rows first find the k-th largest
// key by a 4-pass MSB radix select (8-bit digits, shared-memory histograms), then gather
// every key above it plus the lowest-index keys equal to it (an ordered block scan), and
// sort only those. The final order is a bitonic sort of 64-bit composites
// (key << 32 | ~index): score descending, then index ascending -- deterministic for any
// ties.
#include "dsv4_common.cuh"
#include "index_common.cuh"

namespace dsv4 {

constexpr int TOPK_THREADS = 1024;
constexpr int TOPK_MAX = 4096;   // largest k (and largest directly sorted row)

__device__ __forceinline__ uint32_t score_key(float s) {
  s = s + 0.0f;                                  // fold -0 into +0
  const uint32_t u = __float_as_uint(s);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ unsigned long long compose(uint32_t key, int s) {
  return ((unsigned long long)key << 32) | (unsigned long long)(0xFFFFFFFFu - (uint32_t)s);
}
__device__ __forceinline__ int index_of(unsigned long long c) {
  return (int)(0xFFFFFFFFu - (uint32_t)(c & 0xFFFFFFFFull));
}

// Descending bitonic sort of keys[0, N), N a power of two.
__device__ void bitonic_desc(unsigned long long* keys, int N) {
  for (int size = 2; size <= N; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int j = threadIdx.x; j < N / 2; j += blockDim.x) {
        const int lo = 2 * j - (j & (stride - 1));
        const int hi = lo + stride;
        const bool desc = (lo & size) == 0;
        const unsigned long long x = keys[lo], y = keys[hi];
        if (desc ? (x < y) : (x > y)) { keys[lo] = y; keys[hi] = x; }
      }
      __syncthreads();
    }
  }
}

__global__ void __launch_bounds__(TOPK_THREADS) topk_kernel(IndexArgs a, int q_begin) {
  __shared__ unsigned long long keys[TOPK_MAX];
  __shared__ int hist[256];
  __shared__ int warp_cnt[TOPK_THREADS / 32];
  __shared__ int sh_sel, sh_above, sh_cnt_g, sh_eq_base;
  const int qg = q_begin + blockIdx.x;
  const int b = qg / a.nq, i = qg % a.nq;
  const int Et = visible_entries(a, b, i);
  const int k = a.k;
  const int keff = min(k, Et);
  int32_t* out = a.idx + (long long)qg * k;
  if (threadIdx.x == 0) a.counts[qg] = keff;
  for (int j = keff + threadIdx.x; j < k; j += blockDim.x) out[j] = -1;
  if (keff == 0) return;
  const float* sc = a.scores + (long long)(qg - a.score_q0) * a.scores_ld;

  if (Et <= 1024) {                                  // sort the whole row
    int N = 1;
    while (N < Et) N <<= 1;
    for (int j = threadIdx.x; j < N; j += blockDim.x)
      keys[j] = j < Et ? compose(score_key(sc[j]), j) : 0ull;
    __syncthreads();
    bitonic_desc(keys, N);
    for (int j = threadIdx.x; j < keff; j += blockDim.x) out[j] = index_of(keys[j]);
    return;
  }

  // ---- radix select of the keff-th largest key
  uint32_t prefix = 0, pmask = 0;
  int remaining = keff;                 // how many still to take at/below the prefix
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    for (int d = threadIdx.x; d < 256; d += blockDim.x) hist[d] = 0;
    __syncthreads();
    for (int j = threadIdx.x; j < Et; j += blockDim.x) {
      const uint32_t key = score_key(sc[j]);
      if ((key & pmask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1);
    }
    __syncthreads();
    if (threadIdx.x < 32) {
      const int lane = threadIdx.x;
      int own = 0;
#pragma unroll
      for (int d = 0; d < 8; ++d) own += hist[8 * lane + d];
      int suf = own;                     // inclusive suffix sum over lanes >= lane
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int v = __shfl_down_sync(0xffffffffu, suf, off);
        if (lane + off < 32) suf += v;
      }
      const int above = suf - own;       // keys in bins of higher lanes
      if (above < remaining && remaining <= suf) {
        int acc = above;
        for (int d = 8 * lane + 7; d >= 8 * lane; --d) {
          if (acc + hist[d] >= remaining) { sh_sel = d; sh_above = acc; break; }
          acc += hist[d];
        }
      }
    }
    __syncthreads();
    remaining -= sh_above;
    prefix |= (uint32_t)sh_sel << shift;
    pmask |= 255u << shift;
    __syncthreads();
  }
  const uint32_t T = prefix;
  const int need_eq = remaining;         // keys equal to T to take (lowest indices first)
  const int n_gt = keff - need_eq;       // keys strictly above T (all taken)
  if (threadIdx.x == 0) { sh_cnt_g = 0; sh_eq_base = 0; }
  __syncthreads();
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  for (int base = 0; base < Et; base += blockDim.x) {
    const int j = base + threadIdx.x;
    const uint32_t key = j < Et ? score_key(sc[j]) : 0u;
    const bool gt = j < Et && key > T;
    const bool eq = j < Et && key == T;
    if (gt) {
      const int pos = atomicAdd(&sh_cnt_g, 1);
      if (pos < n_gt) keys[pos] = compose(key, j);
    }
    const unsigned bal = __ballot_sync(0xffffffffu, eq);
    if (lane == 0) warp_cnt[wid] = __popc(bal);
    __syncthreads();
    int before = sh_eq_base;
    for (int w2 = 0; w2 < wid; ++w2) before += warp_cnt[w2];
    const int rank = before + __popc(bal & ((1u << lane) - 1u));
    if (eq && rank < need_eq) keys[n_gt + rank] = compose(key, j);
    __syncthreads();
    if (threadIdx.x == 0) {
      int tot = 0;
      for (int w2 = 0; w2 < TOPK_THREADS / 32; ++w2) tot += warp_cnt[w2];
      sh_eq_base += tot;
    }
    __syncthreads();
  }
  int N = 1;
  while (N < keff) N <<= 1;
  for (int j = keff + threadIdx.x; j < N; j += blockDim.x) keys[j] = 0ull;
  __syncthreads();
  bitonic_desc(keys, N);
  for (int j = threadIdx.x; j < keff; j += blockDim.x) out[j] = index_of(keys[j]);
}

int launch_topk(const IndexArgs& a, int q_begin, int q_count, cudaStream_t st) {
  if (q_count <= 0) return DSV4_OK;
  topk_kernel<<<q_count, TOPK_THREADS, 0, st>>>(a, q_begin);
  return launch_status("top-k select");
}

}  // namespace dsv4
