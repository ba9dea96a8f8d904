// Per-query TopK over the indexer scores ("CSA And HCA: Definition, State, And Cost Model",
// s3.1: S_t = TopK_{s in E_t}(I_{t,s}, k)); per-query valid counts as in pypto-lib PR #834
// (cmp_counts).
//
// S_t is a set. The kernel returns the k_eff = min(k, E_t) entries with the largest scores
// (ties at the threshold go to the lower entry index) in ascending entry order, padded with
// -1. Selection inside one CTA (select_topk):
//   a 4-pass MSB radix select over order-preserving 32-bit keys (8-bit digits, shared-memory
//   histograms with warp-aggregated updates -- scores crowd into a few top-byte bins -- and
//   one block suffix scan per pass) finds the k_eff-th largest key T; then each warp counts,
//   over its contiguous range of entries, the keys above T and those equal to T; two block
//   exclusive scans give every warp its output offset and its share of the ties, and the
//   selected positions are emitted in ascending order.
// Rows up to TOPK_SEG entries: one CTA per query (E_t <= k selects everything without
// reading a score). Longer rows (decode over long contexts): stage 1 selects, per segment
// of TOPK_SEG entries, that segment's top k under the same order (score descending, then
// entry ascending) -- every entry of the query's top k is in its segment's top k, since the
// entries ranked above it within the segment are a subset of those ranked above it overall;
// stage 2 selects the query's top k among the concatenated segment candidates, which are
// already in ascending entry order.
#include "dsv4_common.cuh"
#include "index_common.cuh"

namespace dsv4 {

constexpr int TOPK_SEG = 16384;                  // longer rows take the two-stage path

__device__ __forceinline__ uint32_t score_key(float s) {
  s = s + 0.0f;                                  // fold -0 into +0
  const uint32_t u = __float_as_uint(s);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Block-wide exclusive prefix sum over the NT threads; also returns the total.
template <int NT>
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
  for (int w = 0; w < NT / 32; ++w) {
    const int t = warp_tot[w];
    before += w < wid ? t : 0;
    total += t;
  }
  __syncthreads();
  return before + incl - v;
}

// One histogram update per distinct bin among the warp's active lanes.
__device__ __forceinline__ void hist_add(int* hist, uint32_t bin, bool pred) {
  const uint32_t active = __ballot_sync(0xffffffffu, pred);
  if (!pred) return;
  const uint32_t same = __match_any_sync(active, bin);
  if ((threadIdx.x & 31) == __ffs(same) - 1) atomicAdd(&hist[bin], __popc(same));
}

struct TopkShared {
  int hist[256];
  int warp_tot[32];
  int sel, above;
};

// Selects the keff (< n) largest of sc[0, n) under (score descending, position ascending) and
// calls emit(p, j) for the p-th selected position j, p ascending with j. All NT threads call.
// kShort: rows of at most a few thousand entries -- scalar loads and plain shared atomics
// for the histograms and per-thread contiguous ranges for the compaction cost less there.
template <int NT, bool kShort, typename Emit>
__device__ __forceinline__ void select_topk(const float* sc, int n, int keff, TopkShared& sh,
                                            Emit emit) {
  int* hist = sh.hist;
  int* warp_tot = sh.warp_tot;
  const int Et = n;
  // ---- radix select of the keff-th largest key
  const bool vec = (reinterpret_cast<uintptr_t>(sc) & 15) == 0;
  uint32_t prefix = 0, pmask = 0;
  int remaining = keff;                           // still to take at or below the prefix
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    if (threadIdx.x < 256) hist[threadIdx.x] = 0;
    __syncthreads();
    // whole warps iterate together (match/ballot need converged lanes); four keys per lane
    // per step from one 16-byte load when the row is aligned
    if (kShort) {
      for (int j = threadIdx.x; j < Et; j += NT) {
        const uint32_t key = score_key(__ldg(sc + j));
        if ((key & pmask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1);
      }
    }
    // (UNR independent loads in flight per thread: the scan is latency bound otherwise)
    constexpr int UNR = 4;
    for (int j0 = 4 * (threadIdx.x & ~31); !kShort && j0 < Et; j0 += 4 * NT * UNR) {
      float4 f[UNR];
#pragma unroll
      for (int r = 0; r < UNR; ++r) {
        const int j = j0 + 4 * NT * r + 4 * (threadIdx.x & 31);
        f[r] = make_float4(0.f, 0.f, 0.f, 0.f);
        if (vec && j + 3 < Et) {
          f[r] = __ldg(reinterpret_cast<const float4*>(sc + j));
        } else {
          if (j < Et) f[r].x = __ldg(sc + j);
          if (j + 1 < Et) f[r].y = __ldg(sc + j + 1);
          if (j + 2 < Et) f[r].z = __ldg(sc + j + 2);
          if (j + 3 < Et) f[r].w = __ldg(sc + j + 3);
        }
      }
#pragma unroll
      for (int r = 0; r < UNR; ++r) {
        const int j = j0 + 4 * NT * r + 4 * (threadIdx.x & 31);
        const float fv[4] = {f[r].x, f[r].y, f[r].z, f[r].w};
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const uint32_t key = score_key(fv[u]);
          hist_add(hist, (key >> shift) & 255u, j + u < Et && (key & pmask) == prefix);
        }
      }
    }
    __syncthreads();
    // suffix sums over digits: thread t < 256 owns digit 255 - t, so an exclusive prefix over
    // threads is the count of keys in higher digits
    const int d = 255 - (int)threadIdx.x;
    const int h = d >= 0 ? hist[d] : 0;
    int tot;
    const int above = block_exclusive_scan<NT>(h, warp_tot, tot);
    if (d >= 0 && above < remaining && remaining <= above + h) {
      sh.sel = d;
      sh.above = above;
    }
    __syncthreads();
    remaining -= sh.above;
    prefix |= (uint32_t)sh.sel << shift;
    pmask |= 255u << shift;
    __syncthreads();
  }
  const uint32_t T = prefix;
  const int need_eq = remaining;                  // keys equal to T to take (lowest index first)

  if (kShort) {
    // ---- order-preserving compaction over contiguous per-thread ranges
    const int per = (Et + NT - 1) / NT;
    const int lo = threadIdx.x * per, hi = min(Et, lo + per);
    int n_gt = 0, n_eq = 0;
    for (int j = lo; j < hi; ++j) {
      const uint32_t key = score_key(__ldg(sc + j));
      n_gt += key > T;
      n_eq += key == T;
    }
    int tot;
    const int eq_before = block_exclusive_scan<NT>(n_eq, warp_tot, tot);
    const int take_eq = max(0, min(n_eq, need_eq - eq_before));
    int pos = block_exclusive_scan<NT>(n_gt + take_eq, warp_tot, tot), eq_seen = 0;
    for (int j = lo; j < hi; ++j) {
      const uint32_t key = score_key(__ldg(sc + j));
      if (key > T || (key == T && eq_seen++ < take_eq)) {
        if (pos < keff) emit(pos, j);
        ++pos;
      }
    }
    return;
  }
  // ---- order-preserving compaction: each warp owns a contiguous range of entries, read
  // 32 at a time (coalesced); ballots give in-warp ranks, block scans give warp offsets.
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const uint32_t lt = (1u << lane) - 1u;
  const int per_w = ((Et + NT / 32 - 1) / (NT / 32) + 31) & ~31;
  const int lo = wid * per_w, hi = min(Et, lo + per_w);
  int n_gt = 0, n_eq = 0;
  for (int j0 = lo; j0 < hi; j0 += 128) {
    float v[4];
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const int j = j0 + 32 * r + lane;
      v[r] = j < hi ? __ldg(sc + j) : 0.f;
    }
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const int j = j0 + 32 * r + lane;
      const uint32_t key = score_key(v[r]);
      n_gt += __popc(__ballot_sync(0xffffffffu, j < hi && key > T));
      n_eq += __popc(__ballot_sync(0xffffffffu, j < hi && key == T));
    }
  }
  // warp totals are uniform across the warp: lane 0 contributes them to the block scans
  int tot;
  const int eq_before = block_exclusive_scan<NT>(lane == 0 ? n_eq : 0, warp_tot, tot);
  const int eq_b = __shfl_sync(0xffffffffu, eq_before, 0);
  const int take_eq = max(0, min(n_eq, need_eq - eq_b));
  const int pos_b = block_exclusive_scan<NT>(lane == 0 ? n_gt + take_eq : 0, warp_tot, tot);
  int pos = __shfl_sync(0xffffffffu, pos_b, 0), eq_seen = 0;
  for (int j0 = lo; j0 < hi; j0 += 128) {
    float v[4];
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const int j = j0 + 32 * r + lane;
      v[r] = j < hi ? __ldg(sc + j) : 0.f;
    }
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const int j = j0 + 32 * r + lane;
      const uint32_t key = score_key(v[r]);
      const bool gt = j < hi && key > T, eq = j < hi && key == T;
      const uint32_t eqb = __ballot_sync(0xffffffffu, eq);
      const bool sel = gt || (eq && eq_seen + __popc(eqb & lt) < take_eq);
      const uint32_t selb = __ballot_sync(0xffffffffu, sel);
      const int p = pos + __popc(selb & lt);
      if (sel && p < keff) emit(p, j);
      pos += __popc(selb);
      eq_seen += __popc(eqb);
    }
  }
}

// Single stage: one CTA per query.
template <int NT>
__global__ void __launch_bounds__(NT) topk_kernel(IndexArgs a, int q_begin) {
  __shared__ TopkShared sh;
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
  select_topk<NT, NT == 256>(sc, Et, keff, sh, [&](int p, int j) { out[p] = j; });
}

// Stage 1 of the long-row path: grid (segment, query). Writes the segment's top
// min(k, segment length) entries (global entry index and score) in ascending entry order to
// its k candidate slots and pads the rest with score -inf / index -1.
template <int NT>
__global__ void __launch_bounds__(NT) topk_seg_kernel(IndexArgs a, int q_begin) {
  __shared__ TopkShared sh;
  const int qg = q_begin + blockIdx.y, seg = blockIdx.x;
  const int b = qg / a.nq, i = qg % a.nq;
  const int Et = visible_entries(a, b, i);
  const int k = a.k;
  const long long row = qg - a.score_q0;
  float* cs = a.cand_score + (row * a.nseg + seg) * k;
  int32_t* ci = a.cand_idx + (row * a.nseg + seg) * k;
  const int lo = seg * TOPK_SEG;
  const int len = max(0, min(Et, lo + TOPK_SEG) - lo);
  const int kseg = min(k, len);
  const float* sc = a.scores + row * a.scores_ld + lo;
  for (int j = kseg + threadIdx.x; j < k; j += blockDim.x) {
    cs[j] = -INFINITY;
    ci[j] = -1;
  }
  if (kseg == len) {                              // the whole segment is a candidate set
    for (int j = threadIdx.x; j < len; j += blockDim.x) {
      cs[j] = sc[j];
      ci[j] = lo + j;
    }
    return;
  }
  select_topk<NT, false>(sc, len, kseg, sh, [&](int p, int j) {
    cs[p] = sc[j];
    ci[p] = lo + j;
  });
}

// Stage 2 of the long-row path: one CTA per query over its nseg * k candidates.
template <int NT>
__global__ void __launch_bounds__(NT) topk_merge_kernel(IndexArgs a, int q_begin) {
  __shared__ TopkShared sh;
  const int qg = q_begin + blockIdx.x;
  const int b = qg / a.nq, i = qg % a.nq;
  const int Et = visible_entries(a, b, i);
  const int k = a.k;
  const int keff = min(k, Et);
  int32_t* out = a.idx + (long long)qg * k;
  if (threadIdx.x == 0) a.counts[qg] = keff;
  for (int j = keff + threadIdx.x; j < k; j += blockDim.x) out[j] = -1;
  if (keff == 0) return;
  if (Et <= k) {
    for (int j = threadIdx.x; j < Et; j += blockDim.x) out[j] = j;
    return;
  }
  const long long row = qg - a.score_q0;
  const float* cs = a.cand_score + row * a.nseg * k;
  const int32_t* ci = a.cand_idx + row * a.nseg * k;
  select_topk<NT, false>(cs, a.nseg * k, keff, sh, [&](int p, int j) { out[p] = ci[j]; });
}

int launch_topk(const IndexArgs& a, int q_begin, int q_count, cudaStream_t st) {
  if (q_count <= 0) return DSV4_OK;
  if (a.nseg > 1) {
    topk_seg_kernel<256><<<dim3(a.nseg, q_count), 256, 0, st>>>(a, q_begin);
    if ((long long)a.nseg * a.k >= 4096)
      topk_merge_kernel<1024><<<q_count, 1024, 0, st>>>(a, q_begin);
    else
      topk_merge_kernel<256><<<q_count, 256, 0, st>>>(a, q_begin);
  } else if (a.max_e > TOPK_SEG) {                // long rows without candidate scratch
    topk_kernel<1024><<<q_count, 1024, 0, st>>>(a, q_begin);
  } else {
    topk_kernel<256><<<q_count, 256, 0, st>>>(a, q_begin);
  }
  return launch_status("top-k select");
}

int topk_segments(int max_entries) {
  return max_entries > TOPK_SEG ? (max_entries + TOPK_SEG - 1) / TOPK_SEG : 1;
}

}  // namespace dsv4
