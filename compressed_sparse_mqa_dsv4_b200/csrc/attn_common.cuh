// Shared declarations of the hybrid sparse attention kernels.
#pragma once
#include "dsv4_common.cuh"
#include "rope.cuh"

namespace dsv4 {

struct AttnArgs {
  const void* Q;
  const void* pool;
  long long pool_rows;
  const int64_t* kv_row_off;
  const int32_t* idx;      // NULL: dense read of all completed entries
  const int32_t* counts;
  int k;
  const void* local;
  int R;
  const int32_t* q_pos0;
  int B, nq, H, c, m, w;
  const float* sink;
  float scale;
  void* O;
  float* lse;
  // > 0: rotate the output's last rope_out channels back by the query's position (inverse
  // RoPE of "CSA And HCA: Definition, State, And Cost Model", s5.2) before it is stored
  int rope_out;
  // split candidate lists (tensor-core path): nsplit partials per (query, head group) in
  // part_o [items * nsplit][64 heads][c] fp32 and part_ml [items * nsplit][64] (m, L)
  int nsplit;
  float* part_o;
  float2* part_ml;
};

// Candidate j of query (b, t): compressed part first, then the local window
// ("CSA And HCA: Definition, State, And Cost Model", s5.1: one concatenated list).
// Returns a row pointer offset (in elements) into pool or local, and which one, or -1
// for an invalid candidate (out-of-range index: flagged by the caller).
struct CandidateSet {
  long long pool_base;     // first pool row of this sequence
  long long local_base;    // first local row of this sequence (b * R)
  const int32_t* sel;      // selected entries (NULL = dense)
  int n_comp;              // compressed candidates
  int n_local;             // local candidates
  long long win0;          // first local position
  int Et;                  // completed entries (validity bound of selected indices)
};

__device__ __forceinline__ CandidateSet make_candidates(const AttnArgs& a, int b, int i) {
  CandidateSet cs;
  const long long t = (long long)a.q_pos0[b] + i;
  cs.pool_base = a.kv_row_off[b];
  cs.local_base = (long long)b * a.R;
  cs.Et = (int)((t + 1) / a.m);
  if (a.idx) {
    cs.sel = a.idx + ((long long)b * a.nq + i) * a.k;
    int cnt = a.counts[(long long)b * a.nq + i];
    cs.n_comp = cnt < 0 ? 0 : (cnt > a.k ? a.k : cnt);
  } else {
    cs.sel = nullptr;
    cs.n_comp = cs.Et;
  }
  cs.win0 = t - a.w + 1 < 0 ? 0 : t - a.w + 1;
  cs.n_local = (int)(t - cs.win0 + 1);
  if (cs.n_local > a.R) {            // the ring cannot hold this window: slots would alias
    flag_status(DSV4_ERR_DEVICE_BOUNDS);
    cs.win0 = t - a.R + 1;
    cs.n_local = a.R;
  }
  return cs;
}

// Row index of candidate j: >= 0 pool row (is_local = false) or local row; -1 invalid.
__device__ __forceinline__ long long candidate_row(const AttnArgs& a, const CandidateSet& cs, int j,
                                                   bool& is_local) {
  if (j < cs.n_comp) {
    is_local = false;
    const long long s = cs.sel ? (long long)cs.sel[j] : (long long)j;
    if (s < 0 || s >= cs.Et) return -1;
    const long long row = cs.pool_base + s;
    if (row < 0 || row >= a.pool_rows) return -1;
    return row;
  }
  is_local = true;
  const long long pos = cs.win0 + (j - cs.n_comp);
  return cs.local_base + pos % a.R;
}

int launch_attn_simt(const AttnArgs& a, int dtype, cudaStream_t st);
int launch_attn_tc(const AttnArgs& a, cudaStream_t st, bool* used);
// Split partials: at most this many splits per (query, head group); bytes per split of one
// (query, 64-head group) item.
constexpr int ATTN_MAX_SPLIT = 8;
long long attn_split_bytes_per_item(int c);

}  // namespace dsv4
