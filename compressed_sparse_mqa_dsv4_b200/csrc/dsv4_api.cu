// C ABI of the dsv4 library: status handling, argument validation and dispatch of the
// indexer / attention entry points (compress and FP4 quantisation live beside their
// kernels). Declarations and the contract of every entry point are in include/dsv4.h.
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <string>

#include "attn_common.cuh"
#include "index_common.cuh"

namespace dsv4 {

__device__ int g_status = 0;

static thread_local std::string t_last_error;

int fail(int status, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  t_last_error = buf;
  return status;
}

int launch_status(const char* what) {
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(DSV4_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
  return DSV4_OK;
}

static long long round_up(long long a, long long b) { return (a + b - 1) / b * b; }

// DSV4_VERBOSE=1: report on stderr which kernel path each entry point takes.
static void trace_path(const char* what) {
  static const bool verbose = [] {
    const char* e = std::getenv("DSV4_VERBOSE");
    return e && e[0] == '1';
  }();
  if (verbose) std::fprintf(stderr, "[dsv4] %s\n", what);
}

}  // namespace dsv4

using namespace dsv4;

extern "C" int dsv4_abi_version(void) { return 1; }

extern "C" const char* dsv4_status_string(int s) {
  switch (s) {
    case DSV4_OK: return "ok";
    case DSV4_ERR_INVALID_ARG: return "invalid argument";
    case DSV4_ERR_UNSUPPORTED: return "unsupported";
    case DSV4_ERR_CUDA: return "CUDA error";
    case DSV4_ERR_DEVICE_TIMEOUT: return "device-side wait timed out";
    case DSV4_ERR_DEVICE_BOUNDS: return "device-side index out of range (skipped)";
    case DSV4_ERR_WORKSPACE: return "workspace too small";
    default: return "unknown status";
  }
}

extern "C" const char* dsv4_last_error_message(void) { return t_last_error.c_str(); }

extern "C" int dsv4_check_errors(void* stream) {
  cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
  if (e != cudaSuccess) return fail(DSV4_ERR_CUDA, "dsv4_check_errors: %s", cudaGetErrorString(e));
  int word = 0;
  e = cudaMemcpyFromSymbol(&word, g_status, sizeof(int));
  if (e != cudaSuccess) return fail(DSV4_ERR_CUDA, "dsv4_check_errors: %s", cudaGetErrorString(e));
  if (word != 0) {
    const int zero = 0;
    e = cudaMemcpyToSymbol(g_status, &zero, sizeof(int));
    if (e != cudaSuccess) return fail(DSV4_ERR_CUDA, "dsv4_check_errors: %s", cudaGetErrorString(e));
    return fail(word, "device status word: %s", dsv4_status_string(word));
  }
  return DSV4_OK;
}

// ----------------------------------------------------------------------------- indexer

static long long scores_ld_for(int max_entries) { return round_up(max_entries > 0 ? max_entries : 1, 4); }

static const long long kScoreChunkBytes = 256ll << 20;

// Workspace bytes per query row: its fp32 scores and, for long rows, the region of the
// threshold top-k.
static long long candidate_bytes_per_row(int max_entries, int k, long long rows) {
  return topk_row_bytes(max_entries, k, rows);
}

// Workspace layout for a chunk of `rows` queries:
//   [bf16 expansion of K^I (FP4 tensor-core path)]
//   [scores: rows x ld fp32 (absent when the caller supplies score rows)]
//   [threshold top-k regions of long rows (histograms, counters, selected, candidates)]
//   [bf16 expansion of the chunk's q^I rows (FP4 tensor-core path)]
struct IxLayout {
  long long scores, cand, qx, total;
};
static IxLayout ix_layout(long long rows, long long ld, long long cand_per_row, long long kx_bytes,
                          long long qx_per_row, bool with_scores) {
  IxLayout L;
  long long off = round_up(kx_bytes, 256);
  L.scores = off;
  off += with_scores ? round_up(rows * ld * 4, 256) : 0;
  L.cand = off;
  off += round_up(rows * cand_per_row, 256);
  L.qx = off;
  off += round_up(rows * qx_per_row, 256);
  L.total = off;
  return L;
}

static bool fp4_tensor_path(int qdtype, int H_I, int c_I) {
  const char* force = std::getenv("DSV4_FORCE_SIMT");
  return qdtype == DSV4_FP4 && H_I == 64 && c_I == 128 && !(force && force[0] == '1');
}

extern "C" size_t dsv4_index_topk_workspace_size_ex(int qdtype, int B, int nq, int H_I, int c_I,
                                                    int max_entries, int k, int64_t ki_rows) {
  if (B <= 0 || nq <= 0 || max_entries <= 0) return 0;
  const bool fp4 = fp4_tensor_path(qdtype, H_I, c_I);
  const long long ld = scores_ld_for(max_entries);
  const long long cand = candidate_bytes_per_row(max_entries, k > 0 ? k : 0, (long long)B * nq);
  const long long qx = fp4 ? (long long)H_I * c_I * 2 : 0;
  const long long kx = fp4 ? (ki_rows > 0 ? ki_rows : 0) * c_I * 2 : 0;
  const long long total = (long long)B * nq;
  long long rows = kScoreChunkBytes / (ld * 4 + cand + qx);
  if (rows < 1) rows = 1;
  if (rows > total) rows = total;
  return (size_t)ix_layout(rows, ld, cand, kx, qx, true).total;
}

extern "C" size_t dsv4_index_topk_workspace_size(int B, int nq, int max_entries, int k) {
  return dsv4_index_topk_workspace_size_ex(DSV4_BF16, B, nq, 64, 128, max_entries, k, 0);
}

extern "C" int dsv4_index_topk(int qdtype, const void* qI, const uint8_t* qI_scales,
                               const float* w, const void* KI, const uint8_t* KI_scales,
                               int64_t ki_rows, const int64_t* kv_row_off,
                               const int32_t* q_pos0, int B, int nq, int H_I, int c_I, int m,
                               int k, int max_entries, int32_t* idx, int32_t* counts,
                               float* scores_out, int64_t scores_ld, void* workspace,
                               size_t workspace_bytes, void* stream) {
  if (qdtype != DSV4_F32 && qdtype != DSV4_BF16 && qdtype != DSV4_FP4)
    return fail(DSV4_ERR_INVALID_ARG, "dsv4_index_topk: qdtype %d", qdtype);
  if (B < 0 || nq < 0 || H_I < 1 || c_I < 16 || c_I % 16 != 0 || m < 1 || k < 0 || k > 4096 ||
      max_entries < 0 || ki_rows < 0)
    return fail(DSV4_ERR_INVALID_ARG,
                "dsv4_index_topk: bad sizes B=%d nq=%d H_I=%d c_I=%d m=%d k=%d max_entries=%d",
                B, nq, H_I, c_I, m, k, max_entries);
  if (qdtype == DSV4_FP4 && (c_I % 64 != 0 || !qI_scales || !KI_scales))
    return fail(DSV4_ERR_INVALID_ARG, "dsv4_index_topk: FP4 needs c_I %% 64 == 0 and scale arrays");
  if ((long long)B * nq == 0 || k == 0) {
    if ((long long)B * nq > 0 && counts) {
      cudaError_t e = cudaMemsetAsync(counts, 0, sizeof(int32_t) * (size_t)B * nq, (cudaStream_t)stream);
      if (e != cudaSuccess) return fail(DSV4_ERR_CUDA, "dsv4_index_topk: %s", cudaGetErrorString(e));
    }
    return DSV4_OK;
  }
  if (!qI || !w || !KI || !kv_row_off || !q_pos0 || !idx || !counts)
    return fail(DSV4_ERR_INVALID_ARG, "dsv4_index_topk: NULL pointer");
  IndexArgs a;
  a.qdtype = qdtype; a.qI = qI; a.qI_scales = qI_scales; a.w = w; a.KI = KI;
  a.KI_scales = KI_scales; a.ki_rows = ki_rows; a.kv_row_off = kv_row_off; a.q_pos0 = q_pos0;
  a.B = B; a.nq = nq; a.H_I = H_I; a.c_I = c_I; a.m = m; a.k = k; a.max_e = max_entries;
  a.idx = idx;
  a.counts = counts;
  a.topk_pipe = 0;
  a.nseg = 1;
  a.cand = nullptr;
  a.cand_row_bytes = 0;
  a.hist1_done = 0;
  a.k_fp4 = 0;
  a.q_map_q0 = 0;
  a.q_map_rows = 0;
  cudaStream_t st = (cudaStream_t)stream;
  const int total = B * nq;
  const bool ws_ok = workspace && !(reinterpret_cast<uintptr_t>(workspace) & 255u);
  if (!scores_out && !ws_ok)
    return fail(DSV4_ERR_WORKSPACE, "dsv4_index_topk: workspace missing or not 256-byte aligned");
  if (scores_out && scores_ld < max_entries)
    return fail(DSV4_ERR_INVALID_ARG, "dsv4_index_topk: scores_ld %lld < max_entries %d",
                (long long)scores_ld, max_entries);
  // FP4 operands take the tensor-core kernel through an exact bf16 expansion in the workspace
  // (K^I once, q^I per chunk) when the workspace has room for it; else the CUDA-core kernel.
  const long long ld = scores_ld_for(max_entries);
  const long long cand = candidate_bytes_per_row(max_entries, k, (long long)B * nq);
  const long long wsb = ws_ok ? (long long)workspace_bytes : 0;
  bool fp4x = ws_ok && fp4_tensor_path(qdtype, H_I, c_I) && ki_rows > 0 &&
              !(reinterpret_cast<uintptr_t>(KI) & 7u) && !(reinterpret_cast<uintptr_t>(qI) & 7u);
  // one query per sequence (decode) with 16-byte aligned key codes and scales: the score
  // kernel expands K^I itself as it streams it, and only q^I goes through the workspace (f16)
  const bool f4k = fp4x && nq == 1 && ki_rows >= 130 && aligned16(KI) && aligned16(KI_scales);
  const long long kx = fp4x && !f4k ? ki_rows * c_I * 2 : 0;
  const long long qx = fp4x ? (long long)H_I * c_I * 2 : 0;
  long long rows;
  if (scores_out) {
    rows = total;                                  // one chunk; single-stage top-k
    if (fp4x && ix_layout(rows, ld, 0, kx, qx, false).total > wsb) fp4x = false;
  } else {
    // largest chunk that fits, preferring the threshold top-k, then the FP4 expansion
    auto fit = [&](long long c_row, long long kx_b, long long qx_row) {
      const long long per = ld * 4 + c_row + qx_row;
      long long r = (wsb - round_up(kx_b, 256)) / per;
      if (r > total) r = total;
      while (r > 1 && ix_layout(r, ld, c_row, kx_b, qx_row, true).total > wsb) --r;
      return (r >= 1 && ix_layout(r, ld, c_row, kx_b, qx_row, true).total <= wsb) ? r : 0ll;
    };
    long long c_use = cand;
    rows = fit(c_use, kx, qx);
    if (rows < 1 && cand > 0) { c_use = 0; rows = fit(c_use, kx, qx); }
    if (rows < 1 && fp4x) { fp4x = false; c_use = cand; rows = fit(c_use, 0, 0); }
    if (rows < 1 && cand > 0) { c_use = 0; rows = fit(c_use, 0, 0); }
    if (rows < 1)
      return fail(DSV4_ERR_WORKSPACE, "dsv4_index_topk: workspace %zu bytes < one score row (%lld)",
                  workspace_bytes, ld * 4);
    const IxLayout L = ix_layout(rows, ld, c_use, fp4x ? kx : 0, fp4x ? qx : 0, true);
    char* base = static_cast<char*>(workspace);
    a.scores = reinterpret_cast<float*>(base + L.scores);
    a.scores_ld = ld;
    if (c_use > 0) {
      if (topk_scheme(max_entries, k, total) == 2) a.topk_pipe = 1;
      else a.nseg = topk_segments(max_entries);
      a.cand = base + L.cand;
      a.cand_row_bytes = c_use;
    }
  }
  if (scores_out) {
    a.scores = scores_out;
    a.scores_ld = scores_ld > 0 ? scores_ld : 1;
  }
  IndexArgs ax = a;                                // the bf16 view of FP4 operands
  if (fp4x) {
    const IxLayout L = ix_layout(rows, ld, scores_out ? 0 : (a.cand ? cand : 0), kx, qx,
                                 !scores_out);
    char* base = static_cast<char*>(workspace);
    ax.qdtype = DSV4_BF16;                         // a 16-bit query tile (f16 with FP4 keys)
    ax.qI = base + L.qx;
    ax.qI_scales = nullptr;
    if (f4k) {
      ax.k_fp4 = 1;                                // KI / KI_scales stay the FP4 pool
    } else {
      __nv_bfloat16* kbuf = reinterpret_cast<__nv_bfloat16*>(base);
      int s = launch_fp4_expand(static_cast<const uint8_t*>(KI), KI_scales, ki_rows, c_I, kbuf, st);
      if (s != DSV4_OK) return s;
      ax.KI = kbuf;
      ax.KI_scales = nullptr;
    }
  }
  const int chunk = (int)rows;
  for (int q0 = 0; q0 < total; q0 += chunk) {
    const int qn = total - q0 < chunk ? total - q0 : chunk;
    a.score_q0 = scores_out ? 0 : q0;
    ax.score_q0 = a.score_q0;
    bool used = false, hist1_built = false;
    int s = topk_prepare(a, q0, qn, st);
    if (s != DSV4_OK) return s;
    if (fp4x) {
      const long long qrow0 = (long long)q0 * H_I;
      const uint8_t* qc = static_cast<const uint8_t*>(qI) + qrow0 * (c_I / 2);
      const uint8_t* qs = qI_scales + qrow0 * (c_I / 16);
      void* qdst = const_cast<void*>(ax.qI);
      s = f4k ? launch_fp4_expand_f16(qc, qs, (long long)qn * H_I, c_I, static_cast<__half*>(qdst), st)
              : launch_fp4_expand(qc, qs, (long long)qn * H_I, c_I, static_cast<__nv_bfloat16*>(qdst), st);
      if (s != DSV4_OK) return s;
      ax.q_map_q0 = q0;
      ax.q_map_rows = (long long)qn * H_I;
      s = launch_index_scores_tc(ax, q0, qn, max_entries, st, &used, &hist1_built);
    } else {
      s = launch_index_scores_tc(a, q0, qn, max_entries, st, &used, &hist1_built);
    }
    if (s != DSV4_OK) return s;
    if (q0 == 0)
      trace_path(used ? (f4k ? "index scores: tcgen05 (FP4 keys expanded in the kernel, f16)"
                             : fp4x ? "index scores: tcgen05 (FP4 expanded to bf16)" : "index scores: tcgen05")
                      : "index scores: CUDA cores");
    if (!used) {
      s = launch_index_scores_simt(a, q0, qn, max_entries, st);
      if (s != DSV4_OK) return s;
    }
    a.hist1_done = used && hist1_built ? 1 : 0;
    s = launch_topk(a, q0, qn, st);
    if (s != DSV4_OK) return s;
  }
  return DSV4_OK;
}

// ----------------------------------------------------------------------------- attention

// Split partials pay off only when (query, 64-head group) items are fewer than the SMs.
static int attn_sm_count() {
  static int sms = 0;
  if (sms == 0) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0)
      sms = 148;
  }
  return sms;
}

extern "C" size_t dsv4_hybrid_sparse_attn_workspace_size(int B, int nq, int H, int c) {
  if (B <= 0 || nq <= 0 || H < 64 || H % 64 != 0 || c <= 0) return 0;
  const long long items = (long long)B * nq * (H / 64);
  if (items >= attn_sm_count()) return 0;
  return (size_t)round_up(items * ATTN_MAX_SPLIT * attn_split_bytes_per_item(c), 256);
}

static int hybrid_sparse_attn(int dtype, const void* Q, const void* pool, int64_t pool_rows,
                              const int64_t* kv_row_off, const int32_t* idx, const int32_t* counts,
                              int k, const void* local, int R, const int32_t* q_pos0, int B,
                              int nq, int H, int c, int m, int w, const float* sink, float scale,
                              void* O, float* lse, void* workspace, size_t workspace_bytes,
                              int rope_out, void* stream) {
  if (dtype != DSV4_F32 && dtype != DSV4_BF16)
    return fail(DSV4_ERR_INVALID_ARG, "dsv4_hybrid_sparse_attn: dtype %d", dtype);
  if (rope_out < 0 || rope_out > c || (rope_out & 1))
    return fail(DSV4_ERR_INVALID_ARG, "dsv4_hybrid_sparse_attn_rope: rope_dims %d (c=%d)", rope_out, c);
  if (B < 0 || nq < 0 || H < 1 || c < 1 || m < 1 || w < 1 || R < 1 || pool_rows < 0 ||
      (idx && k < 0))
    return fail(DSV4_ERR_INVALID_ARG,
                "dsv4_hybrid_sparse_attn: bad sizes B=%d nq=%d H=%d c=%d m=%d w=%d R=%d k=%d", B,
                nq, H, c, m, w, R, k);
  if ((dtype == DSV4_BF16 && c % 8 != 0) || (dtype == DSV4_F32 && c % 4 != 0))
    return fail(DSV4_ERR_INVALID_ARG, "dsv4_hybrid_sparse_attn: c=%d not a multiple of the 16-byte vector", c);
  if ((long long)B * nq == 0) return DSV4_OK;
  if (!Q || !local || !kv_row_off || !q_pos0 || !O || (idx && !counts) || (!pool && pool_rows > 0))
    return fail(DSV4_ERR_INVALID_ARG, "dsv4_hybrid_sparse_attn: NULL pointer");
  AttnArgs a;
  a.Q = Q; a.pool = pool; a.pool_rows = pool_rows; a.kv_row_off = kv_row_off; a.idx = idx;
  a.counts = counts; a.k = idx ? k : 0; a.local = local; a.R = R; a.q_pos0 = q_pos0; a.B = B;
  a.nq = nq; a.H = H; a.c = c; a.m = m; a.w = w; a.sink = sink; a.scale = scale; a.O = O;
  a.lse = lse;
  a.rope_out = rope_out;
  a.nsplit = 1;
  a.part_o = nullptr;
  a.part_ml = nullptr;
  if (workspace && workspace_bytes > 0 && H % 64 == 0) {
    if (reinterpret_cast<uintptr_t>(workspace) & 255u)
      return fail(DSV4_ERR_WORKSPACE, "dsv4_hybrid_sparse_attn: workspace not 256-byte aligned");
    const long long items = (long long)B * nq * (H / 64);
    long long cap = (long long)workspace_bytes / (items * attn_split_bytes_per_item(c));
    if (cap > ATTN_MAX_SPLIT) cap = ATTN_MAX_SPLIT;
    if (cap > 1) {
      a.nsplit = (int)cap;                           // capacity; the launcher picks the count
      a.part_o = reinterpret_cast<float*>(workspace);
    }
  }
  cudaStream_t st = (cudaStream_t)stream;
  if (dtype == DSV4_BF16) {
    bool used = false;
    int s = launch_attn_tc(a, st, &used);
    if (s != DSV4_OK || used) {
      trace_path("hybrid attention: tcgen05, single CTA");
      return s;
    }
  }
  trace_path("hybrid attention: CUDA cores");
  return launch_attn_simt(a, dtype, st);
}

extern "C" int dsv4_hybrid_sparse_attn(int dtype, const void* Q, const void* pool,
                                       int64_t pool_rows, const int64_t* kv_row_off,
                                       const int32_t* idx, const int32_t* counts, int k,
                                       const void* local, int R, const int32_t* q_pos0, int B,
                                       int nq, int H, int c, int m, int w, const float* sink,
                                       float scale, void* O, float* lse, void* workspace,
                                       size_t workspace_bytes, void* stream) {
  return hybrid_sparse_attn(dtype, Q, pool, pool_rows, kv_row_off, idx, counts, k, local, R,
                            q_pos0, B, nq, H, c, m, w, sink, scale, O, lse, workspace,
                            workspace_bytes, 0, stream);
}

extern "C" int dsv4_hybrid_sparse_attn_rope(int dtype, const void* Q, const void* pool,
                                            int64_t pool_rows, const int64_t* kv_row_off,
                                            const int32_t* idx, const int32_t* counts, int k,
                                            const void* local, int R, const int32_t* q_pos0,
                                            int B, int nq, int H, int c, int m, int w,
                                            const float* sink, float scale, void* O, float* lse,
                                            void* workspace, size_t workspace_bytes,
                                            int rope_dims, void* stream) {
  return hybrid_sparse_attn(dtype, Q, pool, pool_rows, kv_row_off, idx, counts, k, local, R,
                            q_pos0, B, nq, H, c, m, w, sink, scale, O, lse, workspace,
                            workspace_bytes, rope_dims, stream);
}
