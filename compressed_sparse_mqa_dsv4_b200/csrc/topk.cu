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
// reading a score). Longer rows (decode over long contexts) take a threshold pipeline whose
// passes stream the row across many CTAs (see "threshold pipeline" below).
#include "dsv4_common.cuh"
#include "index_common.cuh"

namespace dsv4 {

constexpr int TOPK_SEG = 16384;                  // longer rows take the threshold pipeline


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

// Rows of at most R * NT entries: each thread holds its contiguous run of R keys in
// registers for all four radix passes and the ordered compaction (the loop over global
// loads re-read every key once per pass, one dependent load at a time).
template <int NT, int R, typename Emit>
__device__ __forceinline__ void select_topk_regs(const float* sc, int n, int keff, TopkShared& sh,
                                                 Emit emit) {
  int* hist = sh.hist;
  const int per = (n + NT - 1) / NT;              // <= R
  const int lo = threadIdx.x * per, hi = min(n, lo + per);
  uint32_t key[R];
#pragma unroll
  for (int r = 0; r < R; ++r) key[r] = (r < hi - lo) ? score_key(__ldg(sc + lo + r)) : 0u;
  const int cnt = max(0, hi - lo);
  uint32_t prefix = 0, pmask = 0;
  int remaining = keff;
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    if (threadIdx.x < 256) hist[threadIdx.x] = 0;
    __syncthreads();
#pragma unroll
    for (int r = 0; r < R; ++r)
      if (r < cnt && (key[r] & pmask) == prefix) atomicAdd(&hist[(key[r] >> shift) & 255u], 1);
    __syncthreads();
    const int d = 255 - (int)threadIdx.x;
    const int h = d >= 0 ? hist[d] : 0;
    int tot;
    const int above = block_exclusive_scan<NT>(h, sh.warp_tot, tot);
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
  int n_gt = 0, n_eq = 0;
#pragma unroll
  for (int r = 0; r < R; ++r) {
    n_gt += r < cnt && key[r] > T;
    n_eq += r < cnt && key[r] == T;
  }
  int tot;
  const int eq_before = block_exclusive_scan<NT>(n_eq, sh.warp_tot, tot);
  const int take_eq = max(0, min(n_eq, remaining - eq_before));
  int pos = block_exclusive_scan<NT>(n_gt + take_eq, sh.warp_tot, tot), eq_seen = 0;
#pragma unroll
  for (int r = 0; r < R; ++r) {
    if (r < cnt && (key[r] > T || (key[r] == T && eq_seen++ < take_eq))) {
      if (pos < keff) emit(pos, lo + r);
      ++pos;
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
  auto emit = [&](int p, int j) { out[p] = j; };
  if (NT == 256 && Et <= 8 * NT)
    select_topk_regs<NT, 8>(sc, Et, keff, sh, emit);
  else
    select_topk<NT, NT == 256>(sc, Et, keff, sh, emit);
}

// ---------------------------------------------------------------- segments + merge
// Requests with many long rows: stage 1 selects, per segment of TOPK_SEG entries, that
// segment's top k under the same order (score descending, then entry ascending) -- every
// entry of the query's top k is in its segment's top k, since the entries ranked above it
// within the segment are a subset of those ranked above it overall; stage 2 selects the
// query's top k among the concatenated segment candidates, already in ascending entry order.
// Candidates of a row: nseg * k scores, then nseg * k entry indices, in its region.

// Stage 1: grid (segment, query). Writes the segment's top min(k, segment length) entries
// (score and global entry index) in ascending entry order to its k candidate slots and pads
// the rest with score -inf / index -1.
template <int NT>
__global__ void __launch_bounds__(NT) topk_seg_kernel(IndexArgs a, int q_begin) {
  __shared__ TopkShared sh;
  const int qg = q_begin + blockIdx.y, seg = blockIdx.x;
  const int b = qg / a.nq, i = qg % a.nq;
  const int Et = visible_entries(a, b, i);
  const int k = a.k;
  const long long row = qg - a.score_q0;
  char* region = a.cand + row * a.cand_row_bytes;
  float* cs = reinterpret_cast<float*>(region) + (long long)seg * k;
  int32_t* ci = reinterpret_cast<int32_t*>(region + (long long)a.nseg * k * 4) + (long long)seg * k;
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

// Stage 2: one CTA per query over its nseg * k candidates.
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
  const char* region = a.cand + row * a.cand_row_bytes;
  const float* cs = reinterpret_cast<const float*>(region);
  const int32_t* ci = reinterpret_cast<const int32_t*>(region + (long long)a.nseg * k * 4);
  select_topk<NT, false>(cs, a.nseg * k, keff, sh, [&](int p, int j) { out[p] = ci[j]; });
}

// ---------------------------------------------------------------- threshold pipeline
// Requests with few rows longer than TOPK_SEG entries (decode over long contexts). Each pass
// is spread over
// CTAs of TK_PASS entries and streams the row once:
//   hist1  per-row histogram of key bits 31..24;
//   hist2  the bin B1 holding the k_eff-th largest key -> histogram of bits 23..16 of the
//          keys in B1;
//   filter the bin B2 holding the k_eff-th largest key among those -> keys whose top 16 bits
//          exceed (B1, B2) are selected; keys equal to it in their top 16 bits are boundary
//          candidates, kept as (low 16 key bits, ~entry) so that a larger value means a larger
//          score or, for equal scores, a lower entry;
//   final  per row: the k_eff - (selected) largest boundary candidates by a radix select over
//          those 48-bit values (all distinct), then the selected entries in ascending order.
// A row whose boundary candidates exceed TK_CAND is selected by the single-CTA select over
// the whole row instead (many scores sharing their top 16 bits).
constexpr int TK_PASS = 8192;                    // entries per CTA of a pass
constexpr int TK_CAND = 8192;                    // boundary candidates kept per row
constexpr int TK_MAXK = 4096;                    // larger k: single-CTA select

struct TkRow {
  int* hist1;                                    // [256]
  int* hist2;                                    // [256]
  int* counters;                                 // n_sel, n_cand
  int32_t* sel;                                  // [k]
  unsigned long long* cand;                      // [TK_CAND]
};

__device__ __forceinline__ TkRow tk_row(const IndexArgs& a, long long row) {
  char* base = a.cand + row * a.cand_row_bytes;
  TkRow r;
  r.hist1 = reinterpret_cast<int*>(base);
  r.hist2 = reinterpret_cast<int*>(base + 1024);
  r.counters = reinterpret_cast<int*>(base + 2048);
  r.sel = reinterpret_cast<int32_t*>(base + TK_HDR);
  r.cand = reinterpret_cast<unsigned long long*>(base + TK_HDR + (((long long)a.k * 4 + 255) & ~255ll));
  return r;
}

// The bin (by thread: thread t owns bin 255 - t) where the count from the top first reaches
// `need`; returns the bin and the count strictly above it through shared memory.
template <int NT>
__device__ __forceinline__ void tk_find_bin(const int* hist_g, int need, TopkShared& sh) {
  if (threadIdx.x == 0) {                         // (not found: an inconsistent row, which the
    sh.sel = -1;                                  // final stage sends to the whole-row select)
    sh.above = 0;
  }
  const int d = 255 - (int)threadIdx.x;
  const int h = d >= 0 ? __ldcg(hist_g + d) : 0;
  int tot;
  const int above = block_exclusive_scan<NT>(h, sh.warp_tot, tot);
  if (d >= 0 && above < need && need <= above + h) {
    sh.sel = d;
    sh.above = above;
  }
  __syncthreads();
}

// One pass over entries [lo, hi) of a score row: 32 keys per thread, loaded as float4s
// (8 in flight per thread). f(j, key, valid) is called by whole warps.
template <int NT, typename F>
__device__ __forceinline__ void tk_scan(const float* sc, int lo, int hi, F f) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  for (int j0 = lo + 128 * wid; j0 < hi; j0 += 128 * (NT / 32) * 8) {
    float4 v[8];
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      const int j = j0 + 128 * (NT / 32) * r + 4 * lane;
      v[r] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (j + 3 < hi) {
        v[r] = __ldcg(reinterpret_cast<const float4*>(sc + j));
      } else {
        if (j < hi) v[r].x = __ldcg(sc + j);
        if (j + 1 < hi) v[r].y = __ldcg(sc + j + 1);
        if (j + 2 < hi) v[r].z = __ldcg(sc + j + 2);
      }
    }
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      const int j = j0 + 128 * (NT / 32) * r + 4 * lane;
      const float fv[4] = {v[r].x, v[r].y, v[r].z, v[r].w};
#pragma unroll
      for (int u = 0; u < 4; ++u) f(j + u, score_key(fv[u]), j + u < hi);
    }
  }
}

// Warp-aggregated append of one value per flagged lane to list[*counter ...]; returns the
// position of this lane's value (or -1).
__device__ __forceinline__ int tk_append(int* counter, bool pred) {
  const uint32_t m = __ballot_sync(0xffffffffu, pred);
  if (m == 0) return -1;
  const int lane = threadIdx.x & 31;
  int base = 0;
  if (lane == __ffs(m) - 1) base = atomicAdd(counter, __popc(m));
  base = __shfl_sync(0xffffffffu, base, __ffs(m) - 1);
  return pred ? base + __popc(m & ((1u << lane) - 1u)) : -1;
}

struct TkCta {
  int qg, Et, keff, lo, hi;
  long long row;
  bool active;
};

__device__ __forceinline__ TkCta tk_cta(const IndexArgs& a, int q_begin) {
  TkCta c;
  c.qg = q_begin + blockIdx.y;
  const int b = c.qg / a.nq, i = c.qg % a.nq;
  c.Et = visible_entries(a, b, i);
  c.keff = min(a.k, c.Et);
  c.row = c.qg - a.score_q0;
  c.lo = blockIdx.x * TK_PASS;
  c.hi = min(c.Et, c.lo + TK_PASS);
  c.active = c.Et > a.k && c.lo < c.hi;          // shorter rows: the final kernel selects all
  return c;
}

template <int NT>
__global__ void __launch_bounds__(NT) topk_hist1_kernel(IndexArgs a, int q_begin) {
  __shared__ TopkShared sh;
  const TkCta c = tk_cta(a, q_begin);
  if (!c.active) return;
  const TkRow r = tk_row(a, c.row);
  if (threadIdx.x < 256) sh.hist[threadIdx.x] = 0;
  __syncthreads();
  tk_scan<NT>(a.scores + c.row * a.scores_ld, c.lo, c.hi,
              [&](int, uint32_t key, bool valid) { hist_add(sh.hist, key >> 24, valid); });
  __syncthreads();
  if (threadIdx.x < 256 && sh.hist[threadIdx.x]) atomicAdd(r.hist1 + threadIdx.x, sh.hist[threadIdx.x]);
}

template <int NT>
__global__ void __launch_bounds__(NT) topk_hist2_kernel(IndexArgs a, int q_begin) {
  __shared__ TopkShared sh;
  const TkCta c = tk_cta(a, q_begin);
  if (!c.active) return;
  const TkRow r = tk_row(a, c.row);
  tk_find_bin<NT>(r.hist1, c.keff, sh);
  const uint32_t b1 = (uint32_t)sh.sel;
  if (threadIdx.x < 256) sh.hist[threadIdx.x] = 0;
  __syncthreads();
  // few keys fall in bin B1 and they spread over the second byte: plain shared atomics
  tk_scan<NT>(a.scores + c.row * a.scores_ld, c.lo, c.hi, [&](int, uint32_t key, bool valid) {
    if (valid && (key >> 24) == b1) atomicAdd(&sh.hist[(key >> 16) & 255u], 1);
  });
  __syncthreads();
  if (threadIdx.x < 256 && sh.hist[threadIdx.x]) atomicAdd(r.hist2 + threadIdx.x, sh.hist[threadIdx.x]);
}

template <int NT>
__global__ void __launch_bounds__(NT) topk_filter_kernel(IndexArgs a, int q_begin) {
  __shared__ TopkShared sh;
  const TkCta c = tk_cta(a, q_begin);
  if (!c.active) return;
  const TkRow r = tk_row(a, c.row);
  tk_find_bin<NT>(r.hist1, c.keff, sh);
  const uint32_t b1 = (uint32_t)sh.sel;
  const int above1 = sh.above;
  __syncthreads();
  tk_find_bin<NT>(r.hist2, c.keff - above1, sh);
  const uint32_t t16 = (b1 << 8) | (uint32_t)sh.sel;
  tk_scan<NT>(a.scores + c.row * a.scores_ld, c.lo, c.hi, [&](int j, uint32_t key, bool valid) {
    const uint32_t top = key >> 16;
    const int ps = tk_append(r.counters, valid && top > t16);
    if (ps >= 0 && ps < a.k) r.sel[ps] = j;
    const int pc = tk_append(r.counters + 1, valid && top == t16);
    if (pc >= 0 && pc < TK_CAND)
      r.cand[pc] = ((unsigned long long)(key & 0xFFFFu) << 32) | (unsigned long long)(0xFFFFFFFFu - (uint32_t)j);
  });
}

// Final stage: one CTA per row. Dynamic shared memory: TK_CAND candidates + TK_MAXK outputs.
template <int NT>
__global__ void __launch_bounds__(NT) topk_final_kernel(IndexArgs a, int q_begin) {
  __shared__ TopkShared sh;
  __shared__ int n_out;
  extern __shared__ unsigned long long tk_smem[];
  unsigned long long* cv = tk_smem;                         // [TK_CAND]
  int* outl = reinterpret_cast<int*>(tk_smem + TK_CAND);    // [TK_MAXK]
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
  const long long row = qg - a.score_q0;
  const TkRow r = tk_row(a, row);
  const int n_sel = __ldcg(r.counters), n_cand = __ldcg(r.counters + 1);
  const int need = keff - n_sel;
  if (n_cand > TK_CAND || need < 0 || need > n_cand) {
    // too many scores share the threshold's top 16 bits: select over the whole row
    const float* sc = a.scores + row * a.scores_ld;
    select_topk<NT, false>(sc, Et, keff, sh, [&](int p, int j) { out[p] = j; });
    return;
  }
  for (int e = threadIdx.x; e < n_cand; e += NT) cv[e] = __ldcg(r.cand + e);
  for (int e = threadIdx.x; e < n_sel; e += NT) outl[e] = __ldcg(r.sel + e);
  if (threadIdx.x == 0) n_out = n_sel;
  __syncthreads();
  if (need > 0) {
    // radix select of the need-th largest 48-bit candidate value, 8 bits per pass
    unsigned long long prefix = 0, pmask = 0;
    int remaining = need;
    for (int pass = 0; pass < 6; ++pass) {
      const int shift = 40 - 8 * pass;
      if (threadIdx.x < 256) sh.hist[threadIdx.x] = 0;
      __syncthreads();
      for (int e = threadIdx.x; e < n_cand; e += NT) {
        const unsigned long long v = cv[e];
        if ((v & pmask) == prefix) atomicAdd(&sh.hist[(v >> shift) & 255u], 1);
      }
      __syncthreads();
      const int d = 255 - (int)threadIdx.x;
      const int h = d >= 0 ? sh.hist[d] : 0;
      int tot;
      const int above = block_exclusive_scan<NT>(h, sh.warp_tot, tot);
      if (d >= 0 && above < remaining && remaining <= above + h) {
        sh.sel = d;
        sh.above = above;
      }
      __syncthreads();
      remaining -= sh.above;
      prefix |= (unsigned long long)sh.sel << shift;
      pmask |= 255ull << shift;
      __syncthreads();
    }
    // candidate values are distinct: exactly `need` of them are >= the threshold
    for (int e = threadIdx.x; e < n_cand; e += NT) {
      const unsigned long long v = cv[e];
      if (v >= prefix) {
        const int p = atomicAdd(&n_out, 1);
        if (p < TK_MAXK) outl[p] = (int)(0xFFFFFFFFu - (uint32_t)(v & 0xFFFFFFFFull));
      }
    }
    __syncthreads();
  }
  // ascending entry order: bitonic sort of the keff selected entries (padded to a power of 2)
  int n2 = 1;
  while (n2 < keff) n2 <<= 1;
  for (int e = keff + threadIdx.x; e < n2; e += NT) outl[e] = 0x7FFFFFFF;
  __syncthreads();
  for (int size = 2; size <= n2; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int e = threadIdx.x; e < n2 / 2; e += NT) {
        const int lo = 2 * e - (e & (stride - 1));
        const int hi = lo + stride;
        const bool up = (lo & size) == 0;
        const int x = outl[lo], y = outl[hi];
        if ((x > y) == up) {
          outl[lo] = y;
          outl[hi] = x;
        }
      }
      __syncthreads();
    }
  }
  for (int e = threadIdx.x; e < keff; e += NT) out[e] = outl[e];
}

int launch_topk(const IndexArgs& a, int q_begin, int q_count, cudaStream_t st) {
  if (q_count <= 0) return DSV4_OK;
  if (a.topk_pipe) {
    constexpr int kFinalSmem = TK_CAND * 8 + TK_MAXK * 4;
    static bool attr_set = false;
    if (!attr_set) {
      const cudaError_t e = cudaFuncSetAttribute(topk_final_kernel<1024>,
                                                 cudaFuncAttributeMaxDynamicSharedMemorySize, kFinalSmem);
      if (e != cudaSuccess) return fail(DSV4_ERR_CUDA, "top-k: %s", cudaGetErrorString(e));
      attr_set = true;
    }
    // (headers zeroed by topk_prepare; the score kernel may have built hist1 already)
    const dim3 grid((a.max_e + TK_PASS - 1) / TK_PASS, q_count);
    if (!a.hist1_done) topk_hist1_kernel<256><<<grid, 256, 0, st>>>(a, q_begin);
    topk_hist2_kernel<256><<<grid, 256, 0, st>>>(a, q_begin);
    topk_filter_kernel<256><<<grid, 256, 0, st>>>(a, q_begin);
    topk_final_kernel<1024><<<q_count, 1024, kFinalSmem, st>>>(a, q_begin);
  } else if (a.nseg > 1) {
    topk_seg_kernel<256><<<dim3(a.nseg, q_count), 256, 0, st>>>(a, q_begin);
    if ((long long)a.nseg * a.k >= 4096)
      topk_merge_kernel<1024><<<q_count, 1024, 0, st>>>(a, q_begin);
    else
      topk_merge_kernel<256><<<q_count, 256, 0, st>>>(a, q_begin);
  } else if (a.max_e > TOPK_SEG) {                // long rows without the pipeline's scratch
    topk_kernel<1024><<<q_count, 1024, 0, st>>>(a, q_begin);
  } else {
    topk_kernel<256><<<q_count, 256, 0, st>>>(a, q_begin);
  }
  return launch_status("top-k select");
}

int topk_prepare(const IndexArgs& a, int q_begin, int q_count, cudaStream_t st) {
  if (!a.topk_pipe || q_count <= 0) return DSV4_OK;
  const long long row0 = q_begin - a.score_q0;
  const cudaError_t e = cudaMemset2DAsync(a.cand + row0 * a.cand_row_bytes, (size_t)a.cand_row_bytes, 0,
                                          (size_t)TK_HDR, (size_t)q_count, st);
  return e == cudaSuccess ? DSV4_OK : fail(DSV4_ERR_CUDA, "top-k: %s", cudaGetErrorString(e));
}

int topk_segments(int max_entries) {
  return max_entries > TOPK_SEG ? (max_entries + TOPK_SEG - 1) / TOPK_SEG : 1;
}

// The pipeline pays its per-row final select and its extra passes only when few rows share
// the GPU (a decode batch); many rows keep every SM busy with per-segment selects.
constexpr long long TK_PIPE_ROWS = 1024;

int topk_scheme(int max_entries, int k, long long rows) {
  if (max_entries <= TOPK_SEG || k <= 0) return 0;
  return (rows <= TK_PIPE_ROWS && k <= TK_MAXK) ? 2 : 1;
}

long long topk_row_bytes(int max_entries, int k, long long rows) {
  switch (topk_scheme(max_entries, k, rows)) {
    case 2: return TK_HDR + (((long long)k * 4 + 255) & ~255ll) + (long long)TK_CAND * 8;
    case 1: return (long long)topk_segments(max_entries) * k * 8;
    default: return 0;
  }
}

}  // namespace dsv4
