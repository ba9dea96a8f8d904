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
  int sel, above, cnt;
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
// registers for the radix passes and the ordered compaction (the loop over global loads
// re-read every key once per pass, one dependent load at a time). A pass takes two barriers:
// after the histogram updates, warp 0 alone scans the 256 digit counts (8 per lane) while the
// other warps clear the second histogram for the next pass. The passes stop once the
// selected bin is taken whole (its count is what is still needed): every key at or above the
// digits fixed so far is selected and no tie needs breaking.
template <int NT, int R, typename Emit>
__device__ __forceinline__ void select_topk_regs(const float* sc, int n, int keff, TopkShared& sh,
                                                 Emit emit) {
  static_assert(NT >= 64 && NT % 32 == 0, "one scanning warp and at least one clearing warp");
  __shared__ __align__(16) int hist2[2][256];
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int per = (n + NT - 1) / NT;              // <= R
  const int lo = threadIdx.x * per, hi = min(n, lo + per);
  uint32_t key[R];
#pragma unroll
  for (int r = 0; r < R; ++r) key[r] = (r < hi - lo) ? score_key(__ldg(sc + lo + r)) : 0u;
  const int cnt = max(0, hi - lo);
  for (int t = threadIdx.x; t < 256; t += NT) hist2[0][t] = 0;
  __syncthreads();
  uint32_t prefix = 0, pmask = 0;
  int remaining = keff;
  bool whole = false;
  int cur = 0;
  for (int hi_bit = 31; hi_bit >= 0;) {
    const int width = min(8, hi_bit + 1);
    const int shift = hi_bit + 1 - width;
    const uint32_t dmask = (1u << width) - 1u;
    int* hist = hist2[cur];
#pragma unroll
    for (int r = 0; r < R; ++r)
      if (r < cnt && (key[r] & pmask) == prefix) atomicAdd(&hist[(key[r] >> shift) & dmask], 1);
    __syncthreads();
    if (wid == 0) {
      // lane l owns digits 255 - 8l - i, i = 0..7 (descending): lane-local sums, then a warp
      // exclusive scan gives the count of keys in higher digits
      const int4 h1 = *reinterpret_cast<const int4*>(&hist[248 - 8 * lane]);
      const int4 h0 = *reinterpret_cast<const int4*>(&hist[252 - 8 * lane]);
      const int v[8] = {h0.w, h0.z, h0.y, h0.x, h1.w, h1.z, h1.y, h1.x};
      int tot = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) tot += v[i];
      int incl = tot;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += t;
      }
      int above = incl - tot;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        if (above < remaining && remaining <= above + v[i]) {
          sh.sel = 255 - 8 * lane - i;
          sh.above = above;
          sh.cnt = v[i];
        }
        above += v[i];
      }
    } else {
      for (int t = threadIdx.x - 32; t < 256; t += NT - 32) hist2[cur ^ 1][t] = 0;
    }
    __syncthreads();
    remaining -= sh.above;
    prefix |= (uint32_t)sh.sel << shift;
    pmask |= dmask << shift;
    hi_bit -= width;
    if (sh.cnt == remaining) {
      whole = true;
      break;
    }
    cur ^= 1;
  }
  // selected: keys above T, and (unless the last bin was taken whole) the first `remaining`
  // keys equal to T in entry order
  const uint32_t T = prefix;
  int n_gt = 0, n_eq = 0;
#pragma unroll
  for (int r = 0; r < R; ++r) {
    n_gt += r < cnt && (whole ? key[r] >= T : key[r] > T);
    n_eq += r < cnt && !whole && key[r] == T;
  }
  int tot, take_eq = 0;
  if (!whole) {
    const int eq_before = block_exclusive_scan<NT>(n_eq, sh.warp_tot, tot);
    take_eq = max(0, min(n_eq, remaining - eq_before));
  }
  int pos = block_exclusive_scan<NT>(n_gt + take_eq, sh.warp_tot, tot), eq_seen = 0;
#pragma unroll
  for (int r = 0; r < R; ++r) {
    if (r < cnt && (whole ? key[r] >= T : (key[r] > T || (key[r] == T && eq_seen++ < take_eq)))) {
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
// Requests with few rows longer than TOPK_SEG entries (decode over long contexts). Order-
// preserving keys are binned by their top TK_H1_BITS bits (sign, exponent, two mantissa
// bits: quarter-octave bins):
//   hist1  per-row histogram of those 11 bits, built by the score kernel (else by a pass over
//          CTAs of TK_PASS entries); the bin B1 holding the k_eff-th largest key and its
//          population follow from it;
//   filter CTAs of TK_FPASS entries of the rows whose bin B1 holds at most TK_CAND keys: keys
//          above B1 are selected, keys in B1 are boundary candidates, kept as (low 21 key
//          bits, ~entry) so that a larger value means a larger score or, for equal scores, a
//          lower entry. Each CTA gathers them in shared memory and reserves room in the row's
//          lists with one global atomic per list;
//   final  one CTA per row: the k_eff - (selected) largest candidates by a radix select over
//          those values (all distinct; 11-bit digits, stopping once a digit's bin is taken
//          whole), then the selected entries in ascending order (a bitmap over the row). A row
//          whose bin B1 is crowded takes a second level here -- a histogram of key bits 20..13
//          of the keys in B1 and the filter against B1:B2, both in this CTA -- and a row whose
//          boundary candidates still exceed TK_CAND (many equal scores) the whole-row select.
// Keys are compared as the scores themselves: a bin's lowest key maps back to a float bound.
constexpr int TK_PASS = 8192;                    // entries per CTA of the hist1 pass
constexpr int TK_FPASS = 16384;                  // entries per CTA of the filter
constexpr int TK_CAND = 8192;                    // boundary candidates kept per row
constexpr int TK_MAXK = 4096;                    // larger k: single-CTA select
constexpr int TK_LSEL = 1024;                    // shared-memory lists of a filter CTA
constexpr int TK_LCAND = 1024;
constexpr int TK_H1_SHIFT = 32 - TK_H1_BITS;     // first level: key bits 31..21
constexpr int TK_H2_SHIFT = TK_H1_SHIFT - 8;     // second level: key bits 20..13
constexpr int TK_BITMAP_MAX = 1 << 19;           // rows up to this many entries: bitmap order
constexpr int TK_FINAL_NT = 512;
constexpr int TK_FINAL_SMEM = TK_CAND * 8 + TK_MAXK * 4 + TK_BITMAP_MAX / 8;
constexpr int TK_CNT_BYTE = TK_WORK_BYTE + 64;   // n_sel, n_cand of the row's lists
static_assert(4 * TK_H1_BINS <= TK_WORK_BYTE && TK_CNT_BYTE + 8 <= TK_HDR, "top-k row header");

struct TkRow {
  int* hist1;                                    // [TK_H1_BINS]
  int* counters;                                 // n_sel, n_cand
  int32_t* sel;                                  // [k]
  unsigned long long* cand;                      // [TK_CAND]
};

__device__ __forceinline__ TkRow tk_row(const IndexArgs& a, long long row) {
  char* base = a.cand + row * a.cand_row_bytes;
  TkRow r;
  r.hist1 = reinterpret_cast<int*>(base);
  r.counters = reinterpret_cast<int*>(base + TK_CNT_BYTE);
  r.sel = reinterpret_cast<int32_t*>(base + TK_HDR);
  r.cand = reinterpret_cast<unsigned long long*>(base + TK_HDR + (((long long)a.k * 4 + 255) & ~255ll));
  return r;
}

// The bin where the count from the top first reaches `need`, over `bins` <= P * NT bins read
// through ld(bin); thread t owns bins bins-1-P*t .. bins-P*(t+1). Returns through shared
// memory the bin (-1 if none: an inconsistent row, which goes to the whole-row select), the
// count strictly above it and its own count.
template <int NT, int P, typename Ld>
__device__ __forceinline__ void tk_find_bin(Ld ld, int bins, int need, TopkShared& sh) {
  if (threadIdx.x == 0) {
    sh.sel = -1;
    sh.above = 0;
    sh.cnt = 0;
  }
  int h[P], sum = 0;
#pragma unroll
  for (int r = 0; r < P; ++r) {
    const int d = bins - 1 - P * (int)threadIdx.x - r;
    h[r] = d >= 0 ? ld(d) : 0;
    sum += h[r];
  }
  int tot;
  int above = block_exclusive_scan<NT>(sum, sh.warp_tot, tot);
#pragma unroll
  for (int r = 0; r < P; ++r) {
    const int d = bins - 1 - P * (int)threadIdx.x - r;
    if (d >= 0 && above < need && need <= above + h[r]) {
      sh.sel = d;
      sh.above = above;
      sh.cnt = h[r];
    }
    above += h[r];
  }
  __syncthreads();
}

// One pass over entries [lo, hi) of a score row: 32 keys per thread, loaded as 8 float4s in
// flight. The loads are unconditional: lo is a multiple of 4 and the row's stride a multiple
// of 4 that covers its entries, so an index clamped to the row's last float4 (ld4) stays in
// the row (what lies past hi is passed as invalid). f(j, key, valid) is called by whole warps.
template <int NT, typename F>
__device__ __forceinline__ void tk_scan(const float* sc, int ld4, int lo, int hi, F f) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  for (int j0 = lo + 128 * wid; j0 < hi; j0 += 128 * (NT / 32) * 8) {
    float4 v[8];
#pragma unroll
    for (int r = 0; r < 8; ++r)
      v[r] = __ldcg(reinterpret_cast<const float4*>(sc + min(j0 + 128 * (NT / 32) * r + 4 * lane, ld4)));
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      const int j = j0 + 128 * (NT / 32) * r + 4 * lane;
      const float fv[4] = {v[r].x, v[r].y, v[r].z, v[r].w};
#pragma unroll
      for (int u = 0; u < 4; ++u) f(j + u, score_key(fv[u]), j + u < hi);
    }
  }
}

// Float bounds of bin `thr` of the keys' top 32 - shift bits: key >> shift > thr <=> score >= hi
// (never for the top bin), key >> shift >= thr <=> score >= lo. (A bin of NaN keys gives NaN
// bounds that nothing passes; the final stage then finds the lists inconsistent.)
struct TkBounds {
  float lo, hi;
  bool has_hi;
  uint32_t low;                                  // the key bits below the bin
};

__device__ __forceinline__ float tk_key_float(uint32_t key) {
  return __uint_as_float((key & 0x80000000u) ? (key & 0x7FFFFFFFu) : ~key);
}

__device__ __forceinline__ TkBounds tk_bounds(uint32_t thr, int shift) {
  TkBounds b;
  b.lo = tk_key_float(thr << shift);
  const uint32_t next = (thr + 1u) << shift;     // 0: thr is the top bin
  b.has_hi = next != 0u;
  b.hi = b.has_hi ? tk_key_float(next) : 0.f;
  b.low = (1u << shift) - 1u;
  return b;
}

// Filters entries [lo, hi) of a row against the bounds: selected entries go to sel_list,
// boundary candidates to cand_list; n[0], n[1] (shared) count them all. Every thread tests
// its 32 keys on its own; a warp reserves room for its entries with one shared atomic per
// list. Entries beyond sel_cap / cand_cap go to spill(is_selected, value).
template <int NT, typename Spill>
__device__ __forceinline__ void tk_filter_range(const float* sc, int ld4, int lo, int hi,
                                                const TkBounds& b, int* n, int* sel_list,
                                                int sel_cap, unsigned long long* cand_list,
                                                int cand_cap, Spill spill) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  for (int j0 = lo + 128 * wid; j0 < hi; j0 += 128 * (NT / 32) * 8) {
    float4 v[8];
#pragma unroll
    for (int q = 0; q < 8; ++q)
      v[q] = __ldcg(reinterpret_cast<const float4*>(sc + min(j0 + 128 * (NT / 32) * q + 4 * lane, ld4)));
    uint32_t msel = 0, mcand = 0;
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const int jb = j0 + 128 * (NT / 32) * q + 4 * lane;
      const float fv[4] = {v[q].x, v[q].y, v[q].z, v[q].w};
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const bool in = jb + u < hi;
        const bool s = in && b.has_hi && fv[u] >= b.hi;
        const bool c = in && !s && fv[u] >= b.lo;
        msel |= s ? 1u << (4 * q + u) : 0u;
        mcand |= c ? 1u << (4 * q + u) : 0u;
      }
    }
    const int ns = __popc(msel), nc = __popc(mcand);
    if (!__any_sync(0xffffffffu, (ns | nc) != 0)) continue;
    int ps = ns, pc = nc;                          // inclusive warp scans
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int x = __shfl_up_sync(0xffffffffu, ps, o), y = __shfl_up_sync(0xffffffffu, pc, o);
      if (lane >= o) {
        ps += x;
        pc += y;
      }
    }
    int bs = 0, bc = 0;
    if (lane == 31) {
      bs = ps ? atomicAdd(&n[0], ps) : 0;
      bc = pc ? atomicAdd(&n[1], pc) : 0;
    }
    bs = __shfl_sync(0xffffffffu, bs, 31) + ps - ns;
    bc = __shfl_sync(0xffffffffu, bc, 31) + pc - nc;
    if ((msel | mcand) == 0) continue;
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const int jb = j0 + 128 * (NT / 32) * q + 4 * lane;
      const float fv[4] = {v[q].x, v[q].y, v[q].z, v[q].w};
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int bit = 4 * q + u;
        if ((msel >> bit) & 1u) {
          if (bs < sel_cap) sel_list[bs] = jb + u;
          else spill(true, (unsigned long long)(jb + u));
          ++bs;
        } else if ((mcand >> bit) & 1u) {
          const unsigned long long cv = ((unsigned long long)(score_key(fv[u]) & b.low) << 32) |
                                        (unsigned long long)(0xFFFFFFFFu - (uint32_t)(jb + u));
          if (bc < cand_cap) cand_list[bc] = cv;
          else spill(false, cv);
          ++bc;
        }
      }
    }
  }
}

struct TkCta {
  int qg, Et, keff, lo, hi;
  long long row;
  bool active;
};

__device__ __forceinline__ TkCta tk_cta(const IndexArgs& a, int q_begin, int pass) {
  TkCta c;
  c.qg = q_begin + blockIdx.y;
  const int b = c.qg / a.nq, i = c.qg % a.nq;
  c.Et = visible_entries(a, b, i);
  c.keff = min(a.k, c.Et);
  c.row = c.qg - a.score_q0;
  c.lo = blockIdx.x * pass;
  c.hi = min(c.Et, c.lo + pass);
  c.active = c.Et > a.k && c.lo < c.hi;          // shorter rows: the final kernel selects all
  return c;
}

template <int NT>
__global__ void __launch_bounds__(NT) topk_hist1_kernel(IndexArgs a, int q_begin) {
  __shared__ int h1[TK_H1_BINS];
  const TkCta c = tk_cta(a, q_begin, TK_PASS);
  if (!c.active) return;
  const TkRow r = tk_row(a, c.row);
  for (int e = threadIdx.x; e < TK_H1_BINS; e += NT) h1[e] = 0;
  __syncthreads();
  tk_scan<NT>(a.scores + c.row * a.scores_ld, (int)a.scores_ld - 4, c.lo, c.hi,
              [&](int, uint32_t key, bool valid) { hist_add(h1, key >> TK_H1_SHIFT, valid); });
  __syncthreads();
  for (int e = threadIdx.x; e < TK_H1_BINS; e += NT)
    if (h1[e]) atomicAdd(r.hist1 + e, h1[e]);
}

template <int NT>
__global__ void __launch_bounds__(NT, 2) topk_filter_kernel(IndexArgs a, int q_begin) {
  __shared__ TopkShared sh;
  __shared__ int l_n[2], l_base[2];
  __shared__ int l_sel[TK_LSEL];
  __shared__ unsigned long long l_cand[TK_LCAND];
  const TkCta c = tk_cta(a, q_begin, TK_FPASS);
  if (!c.active) return;
  const TkRow r = tk_row(a, c.row);
  if (threadIdx.x < 2) l_n[threadIdx.x] = 0;     // (ordered by the barriers below)
  tk_find_bin<NT, TK_H1_BINS / NT>([&](int d) { return __ldcg(r.hist1 + d); }, TK_H1_BINS, c.keff, sh);
  const int b1 = sh.sel, c1 = sh.cnt;
  if (b1 < 0 || c1 > TK_CAND) return;            // the final kernel takes such rows whole
  const TkBounds bd = tk_bounds((uint32_t)b1, TK_H1_SHIFT);
  tk_filter_range<NT>(a.scores + c.row * a.scores_ld, (int)a.scores_ld - 4, c.lo, c.hi, bd, l_n,
                      l_sel, TK_LSEL, l_cand, TK_LCAND, [&](bool is_sel, unsigned long long v) {
                        const int pg = atomicAdd(r.counters + (is_sel ? 0 : 1), 1);
                        if (is_sel && pg < a.k) r.sel[pg] = (int32_t)v;
                        if (!is_sel && pg < TK_CAND) r.cand[pg] = v;
                      });
  __syncthreads();
  const int ns = min(l_n[0], TK_LSEL), nc = min(l_n[1], TK_LCAND);
  if (threadIdx.x == 0) l_base[0] = ns ? atomicAdd(r.counters, ns) : 0;
  if (threadIdx.x == 32) l_base[1] = nc ? atomicAdd(r.counters + 1, nc) : 0;
  __syncthreads();
  for (int e = threadIdx.x; e < ns; e += NT)
    if (l_base[0] + e < a.k) r.sel[l_base[0] + e] = l_sel[e];
  for (int e = threadIdx.x; e < nc; e += NT)
    if (l_base[1] + e < TK_CAND) r.cand[l_base[1] + e] = l_cand[e];
}

// Final stage: one CTA per row. Dynamic shared memory: TK_CAND candidates, TK_MAXK outputs,
// the bitmap of a row of up to TK_BITMAP_MAX entries.
template <int NT>
__global__ void __launch_bounds__(NT) topk_final_kernel(IndexArgs a, int q_begin) {
  __shared__ TopkShared sh;
  __shared__ int n_list[2], n_out;
  __shared__ int rh[TK_H1_BINS];                 // radix digit histogram (<= 11 bits)
  extern __shared__ unsigned long long tk_smem[];
  unsigned long long* cv = tk_smem;                         // [TK_CAND]
  int* outl = reinterpret_cast<int*>(tk_smem + TK_CAND);    // [TK_MAXK]
  uint32_t* bm = reinterpret_cast<uint32_t*>(outl + TK_MAXK);  // [TK_BITMAP_MAX / 32]
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
  const float* sc = a.scores + row * a.scores_ld;
  const int ld4 = (int)a.scores_ld - 4;
  auto whole_row = [&]() { select_topk<NT, false>(sc, Et, keff, sh, [&](int p, int j) { out[p] = j; }); };

  tk_find_bin<NT, TK_H1_BINS / NT>([&](int d) { return __ldcg(r.hist1 + d); }, TK_H1_BINS, keff, sh);
  const int b1 = sh.sel, c1 = sh.cnt;
  int above = sh.above;
  if (threadIdx.x < 2) n_list[threadIdx.x] = 0;
  __syncthreads();
  if (b1 < 0) {                                   // inconsistent histogram (not expected)
    whole_row();
    return;
  }
  int n_sel, n_cand, shift;
  if (c1 <= TK_CAND) {                            // the filter kernel gathered the row's lists
    shift = TK_H1_SHIFT;
    n_sel = __ldcg(r.counters);
    n_cand = __ldcg(r.counters + 1);
    if (n_sel == above && n_cand <= TK_CAND) {
      for (int e = threadIdx.x; e < n_cand; e += NT) cv[e] = __ldcg(r.cand + e);
      for (int e = threadIdx.x; e < n_sel; e += NT) outl[e] = __ldcg(r.sel + e);
    }
  } else {
    // crowded bin B1: the second level (key bits 20..13 of the keys in B1) and the filter
    // against B1:B2, both over the whole row in this CTA
    if (threadIdx.x < 256) sh.hist[threadIdx.x] = 0;
    __syncthreads();
    const uint32_t ub1 = (uint32_t)b1;
    tk_scan<NT>(sc, ld4, 0, Et, [&](int, uint32_t key, bool valid) {
      if (valid && (key >> TK_H1_SHIFT) == ub1) atomicAdd(&sh.hist[(key >> TK_H2_SHIFT) & 255u], 1);
    });
    __syncthreads();
    tk_find_bin<NT, 1>([&](int d) { return sh.hist[d]; }, 256, keff - above, sh);
    const int b2 = sh.sel;
    above += sh.above;
    __syncthreads();
    if (b2 < 0) {
      whole_row();
      return;
    }
    shift = TK_H2_SHIFT;
    const TkBounds bd = tk_bounds((ub1 << 8) | (uint32_t)b2, TK_H2_SHIFT);
    tk_filter_range<NT>(sc, ld4, 0, Et, bd, n_list, outl, TK_MAXK, cv, TK_CAND,
                        [](bool, unsigned long long) {});
    __syncthreads();
    n_sel = n_list[0];
    n_cand = n_list[1];
  }
  const int need = keff - n_sel;
  if (n_sel != above || n_cand > TK_CAND || need < 0 || need > n_cand) {
    // too many scores share the threshold's bits: select over the whole row
    whole_row();
    return;
  }
  if (threadIdx.x == 0) n_out = n_sel;
  __syncthreads();
  if (need > 0) {
    // radix select of the need-th largest candidate value over its 32 + shift bits, digits of
    // up to 11 bits from the top; stops once the chosen digit's bin is taken whole
    unsigned long long prefix = 0, pmask = 0;
    int remaining = need, hi = 32 + shift;
    bool bad = false;
    while (hi > 0) {
      const int nb = hi < 11 ? hi : 11, shift = hi - nb, bins = 1 << nb;
      for (int e = threadIdx.x; e < bins; e += NT) rh[e] = 0;
      __syncthreads();
      for (int e = threadIdx.x; e < n_cand; e += NT) {
        const unsigned long long v = cv[e];
        if ((v & pmask) == prefix) atomicAdd(&rh[(v >> shift) & (unsigned)(bins - 1)], 1);
      }
      __syncthreads();
      tk_find_bin<NT, (TK_H1_BINS + NT - 1) / NT>([&](int d) { return rh[d]; }, bins, remaining, sh);
      const int sel = sh.sel, above = sh.above, cnt = sh.cnt;
      __syncthreads();
      if (sel < 0) {
        bad = true;
        break;
      }
      remaining -= above;
      prefix |= (unsigned long long)sel << shift;
      pmask |= (unsigned long long)(bins - 1) << shift;
      hi = shift;
      if (cnt == remaining) break;                 // the whole bin is selected
    }
    if (bad || (hi == 0 && remaining != 1)) {      // inconsistent candidates (not expected)
      whole_row();
      return;
    }
    // exactly `need` candidates lie at or above the prefix in their masked bits
    for (int e = threadIdx.x; e < n_cand; e += NT) {
      const unsigned long long v = cv[e];
      if ((v & pmask) >= prefix) {
        const int p = atomicAdd(&n_out, 1);
        if (p < TK_MAXK) outl[p] = (int)(0xFFFFFFFFu - (uint32_t)(v & 0xFFFFFFFFull));
      }
    }
    __syncthreads();
  }
  if (Et <= TK_BITMAP_MAX) {
    // ascending entry order: mark the selected entries in a bitmap of the row, then every
    // thread emits the set bits of its words at its block-scan offset
    const int nw = (Et + 31) >> 5, per = (nw + NT - 1) / NT;
    for (int e = threadIdx.x; e < nw; e += NT) bm[e] = 0;
    __syncthreads();
    for (int e = threadIdx.x; e < keff; e += NT) {
      const int j = outl[e];
      if (j >= 0 && j < Et) atomicOr(&bm[j >> 5], 1u << (j & 31));
    }
    __syncthreads();
    const int w0 = threadIdx.x * per;
    int cnt = 0;
    for (int q = 0; q < per; ++q)
      if (w0 + q < nw) cnt += __popc(bm[w0 + q]);
    int tot;
    int pos = block_exclusive_scan<NT>(cnt, sh.warp_tot, tot);
    for (int q = 0; q < per; ++q) {
      if (w0 + q >= nw) break;
      uint32_t x = bm[w0 + q];
      while (x) {
        const int bit = __ffs(x) - 1;
        if (pos < keff) out[pos] = 32 * (w0 + q) + bit;
        ++pos;
        x &= x - 1u;
      }
    }
    return;
  }
  // longer rows: bitonic sort of the keff selected entries (padded to a power of 2)
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
    static bool attr_set = false;
    if (!attr_set) {
      const cudaError_t e = cudaFuncSetAttribute(topk_final_kernel<TK_FINAL_NT>,
                                                 cudaFuncAttributeMaxDynamicSharedMemorySize, TK_FINAL_SMEM);
      if (e != cudaSuccess) return fail(DSV4_ERR_CUDA, "top-k: %s", cudaGetErrorString(e));
      attr_set = true;
    }
    // (headers zeroed by topk_prepare; the score kernel may have built hist1 already)
    if (!a.hist1_done)
      topk_hist1_kernel<256><<<dim3((a.max_e + TK_PASS - 1) / TK_PASS, q_count), 256, 0, st>>>(a, q_begin);
    topk_filter_kernel<256><<<dim3((a.max_e + TK_FPASS - 1) / TK_FPASS, q_count), 256, 0, st>>>(a, q_begin);
    topk_final_kernel<TK_FINAL_NT><<<q_count, TK_FINAL_NT, TK_FINAL_SMEM, st>>>(a, q_begin);
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
