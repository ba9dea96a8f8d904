// Lightning-indexer scores on the 5th-generation tensor cores (bf16 operands).
//
// I_{t,s} = sum_h w_{t,h} ReLU(q^I_{t,h} . K^I_s), s < floor((t+1)/m)
// ("CSA And HCA: Definition, State, And Cost Model", s3.1).
//
// Transposed tile, like the attention kernel: the MMA M dimension is 128 compressed
// entries and N is (up to 4 queries) x 64 indexer heads, so each TMEM lane holds one
// entry's dot products with every head of every query in the tile, and the weighted
// ReLU head sum is a per-thread reduction in registers:
//     D[128 entries x 64*nqt] = K^I_blk[128 x c_I] . qI_tile[64*nqt x c_I]^T
// One CTA per (tile of <= 4 queries of one sequence, chunk of 4096-16384 entries), 10 warps:
//   warps 0-7  epilogue: warp w reads TMEM lane quadrant w%4 for queries 2(w/4), 2(w/4)+1
//   warp 8     producer: the query tile once, then 128-entry key blocks by 2D TMA into a
//              4-stage ring
//   warp 9     MMA issuer and TMEM owner; D is double-buffered (2 x 256 columns)
// Scores of entries a query cannot see are not written. All waits are bounded.
#include <cstdlib>

#include "index_common.cuh"
#include "tc_common.cuh"

namespace dsv4 {
namespace {

constexpr int IX_CI = 128;             // indexer dim handled by this kernel
constexpr int IX_HI = 64;              // indexer heads per query
constexpr int IX_QT = 4;               // queries per tile
constexpr int IX_BLK = 128;            // entries per MMA tile
constexpr int IX_STAGES = 4;
constexpr int IX_CHUNK = 4096;         // smallest entry chunk per CTA (grid.y splits rows)
constexpr int IX_THREADS = 320;
constexpr uint32_t IX_TM_COLS = 512;

// QT queries per tile, NST key stages in flight. One-query tiles (decode) need a quarter of
// the Q buffer and spend the room on a deeper key ring. HIST: the tile also histograms its
// scores for the threshold top-k (kept out of the layout otherwise: a few KiB more shared
// memory cost the prefill shape ~10 % through a smaller L1).
template <int QT, int NST, bool HIST>
struct IndexSmem {
  uint8_t q[2][QT * IX_HI * 128];           // K-major SW128: [QT*64 rows][64 ch] per K half
  uint8_t k[NST][2][IX_BLK * 128];          // [128 entries][64 ch] per K half
  float w[QT][IX_HI];
  int hist[HIST ? QT : 1][HIST ? 256 : 1];  // key bits 31..24 of the tile's scores
  uint64_t q_full;
  uint64_t k_full[NST], k_empty[NST];
  uint64_t d_full[2], d_empty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};
#ifdef DSV4_TRACE
__device__ unsigned long long g_ix_trace[32][8];
#define IX_TRACE(ev, b_)                                                                       \
  do {                                                                                         \
    if (blockIdx.x == 0 && blockIdx.y == 1 && (b_) >= 32 && (b_) < 64) {                         \
      unsigned long long t_;                                                                   \
      asm volatile("mov.u64 %0, %%clock64;" : "=l"(t_)::"memory");                             \
      g_ix_trace[(b_) - 32][ev] = t_;                                                          \
    }                                                                                          \
  } while (0)
#else
#define IX_TRACE(ev, b_) \
  do {                   \
  } while (0)
#endif

template <int QT, int NST, bool HIST>
constexpr size_t ix_smem() { return sizeof(IndexSmem<QT, NST, HIST>) + 1024; }
static_assert(ix_smem<4, IX_STAGES, true>() <= 232448 && ix_smem<1, 6, true>() <= 232448,
              "shared memory of the index score kernel");

template <int QT, int NST, bool HIST>
__global__ void __launch_bounds__(IX_THREADS, 1)
    index_tc_kernel(const IndexArgs a, const __grid_constant__ CUtensorMap map_q,
                    const __grid_constant__ CUtensorMap map_k, int q_begin, int q_count,
                    int tile0, int tiles_per_seq, int chunk, uint32_t spin) {
  extern __shared__ uint8_t smem_raw[];
  IndexSmem<QT, NST, HIST>& s = *reinterpret_cast<IndexSmem<QT, NST, HIST>*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int tile = tile0 + blockIdx.x;
  const int b = tile / tiles_per_seq;
  const int i0 = (tile % tiles_per_seq) * QT;
  // queries of this tile inside [q_begin, q_begin + q_count)
  int qlo = b * a.nq + i0, qhi = b * a.nq + min(i0 + QT, a.nq);
  qlo = max(qlo, q_begin);
  qhi = min(qhi, q_begin + q_count);
  const int nqt = qhi - qlo;                       // queries in the tile (may be 0)
  int e_tile = 0;                                  // entries seen by the tile's last query
  if (nqt > 0) e_tile = visible_entries(a, b, qhi - 1 - b * a.nq);
  const int e0 = blockIdx.y * chunk;
  const int e1 = min(e_tile, e0 + chunk);
  const long long base = nqt > 0 ? a.kv_row_off[b] : 0;
  const bool bounds_ok = base >= 0 && base + e_tile <= a.ki_rows;
  if (nqt <= 0 || e1 <= e0 || !bounds_ok) {
    if (nqt > 0 && !bounds_ok && tid == 0 && blockIdx.y == 0) flag_status(DSV4_ERR_DEVICE_BOUNDS);
    return;                                        // uniform exit before any barrier
  }
  const int nblk = (e1 - e0 + IX_BLK - 1) / IX_BLK;
  volatile int* abort = &s.abort;

  if (tid == 0) {
    tc::mbar_init(&s.q_full, 1);
    for (int i = 0; i < NST; ++i) {
      tc::mbar_init(&s.k_full[i], 1);
      tc::mbar_init(&s.k_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      tc::mbar_init(&s.d_full[i], 1);
      tc::mbar_init(&s.d_empty[i], 256);
    }
    tc::mbar_init(&s.drain, 1);
    s.abort = 0;
    tc::fence_barrier_init();
  }
  if constexpr (HIST)
    for (int e = tid; e < QT * 256; e += blockDim.x) s.hist[e >> 8][e & 255] = 0;
  for (int e = tid; e < QT * IX_HI; e += blockDim.x) {
    const int u = e / IX_HI, h = e % IX_HI;
    s.w[u][h] = u < nqt ? a.w[(long long)(qlo + u) * a.H_I + h] : 0.f;
  }
  if (warp == 9) {
    tc::tmem_alloc(&s.tmem_base, IX_TM_COLS);
    tc::tmem_relinquish();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = s.tmem_base;

  if (warp == 8) {
    // ------------------------------------------------------------------ producer
    if (lane == 0) {
      int issued[NST];
#pragma unroll
      for (int st = 0; st < NST; ++st) issued[st] = 0;
      tc::prefetch_tensormap(&map_q);
      tc::prefetch_tensormap(&map_k);
      tc::mbar_arrive_expect_tx(&s.q_full, 2 * QT * IX_HI * 128);
      const int qrow = (qlo - a.q_map_q0) * IX_HI;
      tc::tma_load_2d(s.q[0], &map_q, &s.q_full, 0, qrow);
      tc::tma_load_2d(s.q[1], &map_q, &s.q_full, 64, qrow);
      for (int blk = 0; blk < nblk; ++blk) {
        const int st = blk % NST, use = blk / NST;
        if (use > 0 && !tc::mbar_wait(&s.k_empty[st], (uint32_t)((use - 1) & 1), spin, abort)) break;
        tc::mbar_arrive_expect_tx(&s.k_full[st], 2 * IX_BLK * 128);
        const int row = (int)(base + e0 + blk * IX_BLK);
        tc::tma_load_2d(s.k[st][0], &map_k, &s.k_full[st], 0, row);
        tc::tma_load_2d(s.k[st][1], &map_k, &s.k_full[st], 64, row);
        IX_TRACE(0, blk);
        issued[st] = use + 1;
      }
      if (*abort) {
        volatile int never = 0;
        for (int st = 0; st < NST; ++st)
          if (issued[st] > 0) tc::mbar_wait(&s.k_full[st], (uint32_t)((issued[st] - 1) & 1), spin, &never);
        tc::mbar_wait(&s.q_full, 0, spin, &never);
      }
    }
    __syncwarp();
  } else if (warp == 9) {
    // ------------------------------------------------------------------ MMA issuer
    // The warp stays converged: every lane waits (acquire per lane), the warp takes one
    // decision, and elect.sync lets one lane issue. A single-lane branch issued the MMAs and
    // passed completed barriers several times more slowly, which capped the key stream.
    {
      const uint32_t idesc = tc::idesc_bf16_f32(128, IX_HI * nqt, 0, 0);
      const uint64_t d_k0 = tc::sdesc_sw128(tc::smem_u32(s.k[0][0]), 16, 1024);
      const uint64_t d_q0 = tc::sdesc_sw128(tc::smem_u32(s.q[0]), 16, 1024);
      auto wwait = [&](uint64_t* bar, uint32_t parity) {
        return __all_sync(0xffffffffu, tc::mbar_wait(bar, parity, spin, abort)) != 0;
      };
      bool ok = wwait(&s.q_full, 0);
      for (int blk = 0; blk < nblk && ok; ++blk) {
        const int st = blk % NST, buf = blk & 1;
        ok = wwait(&s.k_full[st], (uint32_t)((blk / NST) & 1));
        IX_TRACE(1, blk);
        if (ok && blk >= 2) ok = wwait(&s.d_empty[buf], (uint32_t)(((blk >> 1) - 1) & 1));
        IX_TRACE(2, blk);
        if (!ok) break;
        tc::tc_fence_after();
        // descriptor start addresses (16-byte units): key stage st, K half kk/4, K step kk%4
#pragma unroll
        for (int kk = 0; kk < IX_CI / 16; ++kk)
          tc::mma_bf16_ss_warp(tmem + buf * 256,
                               d_k0 + (uint64_t)(st * (2 * IX_BLK * 128 / 16) + (kk >> 2) * (IX_BLK * 128 / 16) + (kk & 3) * 2),
                               d_q0 + (uint64_t)((kk >> 2) * (QT * IX_HI * 128 / 16) + (kk & 3) * 2), idesc,
                               kk > 0 ? 1u : 0u);
        tc::mma_commit_warp(&s.k_empty[st]);
        tc::mma_commit_warp(&s.d_full[buf]);
        IX_TRACE(3, blk);
      }
      if (!ok) {
        // let every issued MMA finish before TMEM is released
        tc::mma_commit_warp(&s.drain);
        volatile int never = 0;
        tc::mbar_wait(&s.drain, 0, spin, &never);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------------ epilogue warps
    const int quad = warp & 3;                    // TMEM lane quadrant
    const int qp = warp >> 2;                     // query pair: queries 2qp, 2qp+1
    const uint32_t lane_base = (uint32_t)(32 * quad) << 16;
    int Et[2];
    long long srow[2];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int qu = 2 * qp + u;
      Et[u] = qu < nqt ? visible_entries(a, b, qlo + qu - b * a.nq) : 0;
      srow[u] = (long long)(qlo + qu - a.score_q0) * a.scores_ld;
    }
    for (int blk = 0; blk < nblk; ++blk) {
      const int buf = blk & 1;
      if (!tc::mbar_wait(&s.d_full[buf], (uint32_t)((blk >> 1) & 1), spin, abort)) break;
      if (tid == 0) IX_TRACE(4, blk);
      tc::tc_fence_after();
      float d0[32], d1[32], d2[32], d3[32];
      const uint32_t col = tmem + lane_base + buf * 256 + qp * 128;
      const bool two = 2 * qp < nqt;              // this warp has work in the tile
      if (two) {
        tc::tmem_ld32(col, d0);
        tc::tmem_ld32(col + 32, d1);
        if constexpr (QT > 1) {                   // one-query tiles have no second query
          tc::tmem_ld32(col + 64, d2);
          tc::tmem_ld32(col + 96, d3);
        }
        tc::tmem_wait_ld();
      }
      tc::tc_fence_before();
      tc::mbar_arrive(&s.d_empty[buf]);
      if (tid == 0) IX_TRACE(5, blk);
      if (!two) continue;
      const int sidx = e0 + blk * IX_BLK + 32 * quad + lane;
      float sc0 = 0.f, sc1 = 0.f;
      const float* w0 = s.w[QT > 1 ? 2 * qp : 0];
      const float* w1 = s.w[QT > 1 ? 2 * qp + 1 : 0];
#pragma unroll
      for (int h = 0; h < 32; ++h) sc0 = fmaf(w0[h], fmaxf(d0[h], 0.f), sc0);
#pragma unroll
      for (int h = 0; h < 32; ++h) sc0 = fmaf(w0[32 + h], fmaxf(d1[h], 0.f), sc0);
      if constexpr (QT > 1) {
#pragma unroll
        for (int h = 0; h < 32; ++h) sc1 = fmaf(w1[h], fmaxf(d2[h], 0.f), sc1);
#pragma unroll
        for (int h = 0; h < 32; ++h) sc1 = fmaf(w1[32 + h], fmaxf(d3[h], 0.f), sc1);
      }
      if (sidx < Et[0]) a.scores[srow[0] + sidx] = sc0;
      if constexpr (HIST) {                      // first histogram of the threshold top-k
        hist_add(s.hist[QT > 1 ? 2 * qp : 0], score_key(sc0) >> 24, sidx < Et[0]);
        if (QT > 1) hist_add(s.hist[QT > 1 ? 2 * qp + 1 : 0], score_key(sc1) >> 24, 2 * qp + 1 < nqt && sidx < Et[1]);
      }
      if (tid == 0) IX_TRACE(6, blk);
      if (QT > 1 && 2 * qp + 1 < nqt && sidx < Et[1]) a.scores[srow[1] + sidx] = sc1;
    }
  }
  tc::tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, IX_TM_COLS);
  }
  if constexpr (HIST) {
    // add the tile's histograms to the rows' first histograms (int hist1[256] at the start
    // of each row's top-k region)
    for (int e = tid; e < nqt * 256; e += blockDim.x) {
      const int u = e >> 8, v = s.hist[u][e & 255];
      if (v) atomicAdd(reinterpret_cast<int*>(a.cand + (long long)(qlo + u - a.score_q0) * a.cand_row_bytes) + (e & 255), v);
    }
  }
}

}  // namespace

int launch_index_scores_tc(const IndexArgs& a, int q_begin, int q_count, int max_e,
                           cudaStream_t st, bool* used) {
  *used = false;
  const char* force = std::getenv("DSV4_FORCE_SIMT");
  if (force && force[0] == '1') return DSV4_OK;
  if (a.qdtype != DSV4_BF16 || a.c_I != IX_CI || a.H_I != IX_HI) return DSV4_OK;
  if (!aligned16(a.qI) || !aligned16(a.KI)) return DSV4_OK;
  if (q_count <= 0 || max_e <= 0) {
    *used = true;
    return DSV4_OK;
  }
  const long long q_rows = a.q_map_rows > 0 ? a.q_map_rows : (long long)a.B * a.nq * IX_HI;
  if (q_rows >= (1ll << 31) || a.ki_rows >= (1ll << 31) || a.ki_rows <= 0) return DSV4_OK;
  // one query per sequence (decode): one-query tiles with a 6-stage key ring
  const int qt = a.nq == 1 ? 1 : IX_QT;
  CUtensorMap mq, mk;
  int s = encode_tensor_map_2d(&mq, a.qI, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, IX_CI, q_rows, 64,
                               qt * IX_HI, CU_TENSOR_MAP_SWIZZLE_128B);
  if (s != DSV4_OK) return s;
  s = encode_tensor_map_2d(&mk, a.KI, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, IX_CI, a.ki_rows, 64,
                           IX_BLK, CU_TENSOR_MAP_SWIZZLE_128B);
  if (s != DSV4_OK) return s;
  const int tps = (a.nq + qt - 1) / qt;
  auto tile_of = [&](int qg) { return (qg / a.nq) * tps + (qg % a.nq) / qt; };
  const int t0 = tile_of(q_begin), t1 = tile_of(q_begin + q_count - 1);
  // Long rows with few query tiles (decode): larger entry chunks per CTA amortise its setup
  // (Q tile, TMEM, pipeline fill) while keeping at least 4 CTAs per SM of work.
  int chunk = IX_CHUNK;
  const long long tiles = t1 - t0 + 1;
  while (chunk < 4 * IX_CHUNK && tiles * ((max_e + 2 * chunk - 1) / (2 * chunk)) >= 4 * 148) chunk *= 2;
  dim3 grid((unsigned)tiles, (max_e + chunk - 1) / chunk);
  if (grid.y > 65535) return DSV4_OK;
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(index_tc_kernel<IX_QT, IX_STAGES, false>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)ix_smem<IX_QT, IX_STAGES, false>());
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(index_tc_kernel<IX_QT, IX_STAGES, true>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, (int)ix_smem<IX_QT, IX_STAGES, true>());
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(index_tc_kernel<1, 6, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)ix_smem<1, 6, false>());
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(index_tc_kernel<1, 6, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)ix_smem<1, 6, true>());
    if (e != cudaSuccess) return fail(DSV4_ERR_CUDA, "index_tc: %s", cudaGetErrorString(e));
    attr_set = true;
  }
  const int sp = spin_limit();
  if (qt == 1) {
    if (a.topk_pipe)
      index_tc_kernel<1, 6, true><<<grid, IX_THREADS, ix_smem<1, 6, true>(), st>>>(a, mq, mk, q_begin, q_count,
                                                                                 t0, tps, chunk, sp);
    else
      index_tc_kernel<1, 6, false><<<grid, IX_THREADS, ix_smem<1, 6, false>(), st>>>(a, mq, mk, q_begin, q_count,
                                                                                   t0, tps, chunk, sp);
  } else {
    if (a.topk_pipe)
      index_tc_kernel<IX_QT, IX_STAGES, true><<<grid, IX_THREADS, ix_smem<IX_QT, IX_STAGES, true>(), st>>>(
          a, mq, mk, q_begin, q_count, t0, tps, chunk, sp);
    else
      index_tc_kernel<IX_QT, IX_STAGES, false><<<grid, IX_THREADS, ix_smem<IX_QT, IX_STAGES, false>(), st>>>(
          a, mq, mk, q_begin, q_count, t0, tps, chunk, sp);
  }
  *used = true;
  return launch_status("index scores (tensor cores)");
}

}  // namespace dsv4

#ifdef DSV4_TRACE
extern "C" int dsv4_trace_read_ix(unsigned long long* host, size_t n) {
  return cudaMemcpyFromSymbol(host, dsv4::g_ix_trace, n * sizeof(unsigned long long)) == cudaSuccess ? 0 : 3;
}
#endif
