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
// CTAs walk work units (tile of <= 4 queries of one sequence, chunk of 2048-16384 entries):
// persistent, one per SM, for multi-query tiles; for one-query tiles (decode) either one CTA
// per unit or -- with the threshold top-k's zeroed row headers at hand -- persistent CTAs
// that draw units from a global counter (dynamic scheduling over rows of very different
// lengths without a CTA start per unit). 10 warps:
//   warps 0-7  epilogue: warp w reads TMEM lane quadrant w%4 for queries 2(w/4), 2(w/4)+1
//              (one-query tiles: heads 32(w/4)..+31 of the one query)
//   warp 8     producer: per unit the query tile, then 128-entry key blocks by 2D TMA into a
//              4-stage ring (6 stages for one-query tiles) that runs on across units
//   warp 9     MMA issuer and TMEM owner; D is double-buffered (2 x 256 columns)
// FP4 keys (one-query tiles): the producer's TMA brings each block's e2m1 codes and E4M3
// scales into a staging ring; warps 8-15 expand them to f16 (exact: a code times its scale has
// at most 6 significant bits) into the key ring the MMAs read, and the query tile is f16; the
// producer and MMA warps are 16 and 17. The key stream from HBM shrinks from 256 to 72 bytes
// per entry.
// Scores of entries a query cannot see are not written. All waits are bounded.
#include <cstddef>
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
// FP4 keys: warps 8-15 expand the keys, the producer and MMA warps move to 16 and 17
constexpr int IX_THREADS_F4 = 576;
template <bool F4>
constexpr int ix_threads() { return F4 ? IX_THREADS_F4 : IX_THREADS; }
constexpr uint32_t IX_TM_COLS = 512;

// QT queries per tile, NST key stages in flight. One-query tiles (decode) need a quarter of
// the Q buffer and spend the room on a deeper key ring. HIST (one-query tiles): the tile
// also histograms its scores for the threshold top-k, by the top TK_H1_BITS bits of their
// keys (kept out of the layout otherwise: a few KiB more shared memory cost the prefill
// shape ~10 % through a smaller L1).
// DYN: units come from a global counter through a shared-memory FIFO; pre[] holds the dense
// unit list's per-tile offsets.
constexpr int IX_DYN_TILES = 1024;     // tiles of one launch the dynamic scheduler indexes
constexpr int IX_DYN_CHUNK = 2048;     // entries per dynamically scheduled unit
constexpr int IX_UQ = 4;               // unit FIFO depth
constexpr int IX_NSG = 6;              // FP4 keys: staging stages (codes + scales of a block)
constexpr int IX_SG_PAIRS = IX_BLK / 2 + 1;  // scale row pairs a block's staging holds
// a TMA tile's shared-memory destination must be 128-byte aligned: scale stages 1152 apart
constexpr int IX_SG_STRIDE = (IX_SG_PAIRS * 16 + 127) / 128 * 128;

// sum_h w[h] ReLU(d[h]) over 32 heads: four interleaved partial sums (heads h = j mod 4),
// combined as (p0 + p1) + (p2 + p3). w: 16-byte aligned shared memory.
__device__ __forceinline__ float ix_half_sum(const float (&d)[32], const float* w) {
  const float4* wq = reinterpret_cast<const float4*>(w);
  float p0 = 0.f, p1 = 0.f, p2 = 0.f, p3 = 0.f;
#pragma unroll
  for (int h = 0; h < 8; ++h) {
    const float4 wv = wq[h];
    p0 = fmaf(wv.x, fmaxf(d[4 * h], 0.f), p0);
    p1 = fmaf(wv.y, fmaxf(d[4 * h + 1], 0.f), p1);
    p2 = fmaf(wv.z, fmaxf(d[4 * h + 2], 0.f), p2);
    p3 = fmaf(wv.w, fmaxf(d[4 * h + 3], 0.f), p3);
  }
  return (p0 + p1) + (p2 + p3);
}

template <int QT, int NST, bool HIST, bool DYN, bool F4>
struct IndexSmem {
  uint8_t q[2][QT * IX_HI * 128];           // K-major SW128: [QT*64 rows][64 ch] per K half
  uint8_t k[NST][2][IX_BLK * 128];          // [128 entries][64 ch] per K half
  // F4: a block's e2m1 codes [4 chunks][128 rows][16 B] and the E4M3 scales of the 65 row
  // pairs from the pair holding its first row; sg_last: the pool's last row's scales when the
  // row count is odd (that row has no pair partner, so the scale tensor map stops before it)
  uint8_t sg_codes[F4 ? IX_NSG : 1][F4 ? IX_BLK * 64 : 16];
  uint8_t sg_scales[F4 ? IX_NSG : 1][F4 ? IX_SG_STRIDE : 16];
  uint64_t sg_last[F4 ? IX_NSG : 1];
  uint64_t sg_full[F4 ? IX_NSG : 1], sg_empty[F4 ? IX_NSG : 1];
  alignas(16) float w[QT][IX_HI];
  float part[QT == 1 ? 2 : 1][QT == 1 ? IX_BLK : 1];  // one query: second head half's sums
  int hist[HIST ? QT : 1][HIST ? TK_H1_BINS : 1];  // top key bits of the tile's scores
  int pre[DYN ? IX_DYN_TILES : 1];          // first dense unit of each tile
  int wsum[8];
  int n_dense;                              // units in the dense list
  int uid[IX_UQ];                           // unit FIFO (-1: no more units)
  uint64_t u_full[IX_UQ], u_empty[IX_UQ];
  uint64_t q_full, q_empty;
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

template <int QT, int NST, bool HIST, bool DYN, bool F4>
constexpr size_t ix_smem() {
  static_assert(!HIST || QT == 1, "multi-query tiles leave the first histogram to a pass");
  static_assert(!F4 || QT == 1, "FP4 keys: one-query tiles (warps 8-15 expand the keys)");
  return sizeof(IndexSmem<QT, NST, HIST, DYN, F4>) + 1024;
}
using IxSmemF4 = IndexSmem<1, 4, true, true, true>;
static_assert(offsetof(IxSmemF4, sg_codes) % 128 == 0 && offsetof(IxSmemF4, sg_scales) % 128 == 0 &&
                  IX_SG_STRIDE % 128 == 0,
              "TMA destinations of the FP4 staging ring");
static_assert(ix_smem<4, IX_STAGES, false, false, false>() <= 232448 &&
                  ix_smem<1, 6, true, true, false>() <= 232448 && ix_smem<1, 4, true, true, true>() <= 232448,
              "shared memory of the index score kernel");

// F4: a block's 128 rows expanded to f16 by warps 8-15. Row r of the block: 64 code bytes
// (element 2b in the low nibble of byte b) and 8 E4M3 scales (one per 16 elements); it becomes
// 16 pieces of 8 f16 in the K-major 128-byte-swizzled key tile (pieces 0-7 in the first K
// half, 8-15 in the second).
// 4 code bytes (8 e2m1 elements) -> 4 f16x2 words, byte i -> word i (low nibble in the low half)
__device__ __forceinline__ void e2m1x8_to_f16x8(uint32_t w, uint32_t& o0, uint32_t& o1, uint32_t& o2,
                                                uint32_t& o3) {
  asm("{\n .reg .b8 b0, b1, b2, b3;\n mov.b32 {b0, b1, b2, b3}, %4;\n"
      " cvt.rn.f16x2.e2m1x2 %0, b0;\n cvt.rn.f16x2.e2m1x2 %1, b1;\n"
      " cvt.rn.f16x2.e2m1x2 %2, b2;\n cvt.rn.f16x2.e2m1x2 %3, b3;\n}"
      : "=r"(o0), "=r"(o1), "=r"(o2), "=r"(o3)
      : "r"(w));
}
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t two) {
  uint32_t r;
  asm("{\n .reg .b16 h0, h1;\n mov.b32 {h0, h1}, %1;\n cvt.rn.f16x2.e4m3x2 %0, h0;\n}"
      : "=r"(r)
      : "r"(two));
  return r;
}
__device__ __forceinline__ uint32_t hmul2_u32(uint32_t a, uint32_t b) {
  __half2 x = *reinterpret_cast<__half2*>(&a), y = *reinterpret_cast<__half2*>(&b);
  __half2 z = __hmul2(x, y);
  return *reinterpret_cast<uint32_t*>(&z);
}
// One (row r, 32-channel chunk) item: 16 code bytes and their 2 scales (E4M3, low byte first)
// become 4 pieces of 8 f16 at pieces p0 .. p0+3 of row r of one K half of the key tile.
__device__ __forceinline__ void f4_expand_chunk(const uint8_t* codes, uint32_t scales2, uint8_t* tile,
                                                int r, int p0) {
  const uint4 cw = *reinterpret_cast<const uint4*>(codes);
  const uint32_t two = e4m3x2_to_f16x2(scales2);
  const uint32_t s0 = (two & 0xFFFFu) * 0x10001u, s1 = (two >> 16) * 0x10001u;
  const uint32_t wv[4] = {cw.x, cw.y, cw.z, cw.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {                  // piece p0 + i: elements 8i .. 8i+7 of the chunk
    const uint32_t sc = i < 2 ? s0 : s1;
    uint4 o;
    e2m1x8_to_f16x8(wv[i], o.x, o.y, o.z, o.w);
    o.x = hmul2_u32(o.x, sc);
    o.y = hmul2_u32(o.y, sc);
    o.z = hmul2_u32(o.z, sc);
    o.w = hmul2_u32(o.w, sc);
    *reinterpret_cast<uint4*>(tile + r * 128 + (((p0 + i) ^ (r & 7)) << 4)) = o;
  }
}

// Named-barrier OR-reduction over `threads` threads (all take the same decision).
__device__ __forceinline__ bool ix_red_or(uint32_t id, uint32_t threads, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n .reg .pred p, q;\n setp.ne.u32 p, %1, 0;\n"
      " barrier.red.or.pred q, %2, %3, p;\n selp.u32 %0, 1, 0, q;\n}"
      : "=r"(r)
      : "r"((uint32_t)pred), "r"(id), "r"(threads)
      : "memory");
  return r != 0;
}

// A work unit: a tile of <= QT queries of one sequence and a chunk of its entries. Every
// role derives the same units in the same order and skips the empty ones.
struct IxUnit {
  int b, qlo, nqt, e0, e1, e_tile;
  long long base;
  bool valid;
};

// Chunk c of tile `tile`; `flag`: report a key-row range outside the key buffer.
template <int QT>
__device__ __forceinline__ IxUnit ix_tile_unit(const IndexArgs& a, int tile, int c, int q_begin,
                                               int q_count, int tiles_per_seq, int chunk, bool flag) {
  IxUnit r;
  r.b = tile / tiles_per_seq;
  const int i0 = (tile % tiles_per_seq) * QT;
  r.qlo = max(r.b * a.nq + i0, q_begin);
  const int qhi = min(r.b * a.nq + min(i0 + QT, a.nq), q_begin + q_count);
  r.nqt = qhi - r.qlo;
  const int e_tile = r.nqt > 0 ? visible_entries(a, r.b, qhi - 1 - r.b * a.nq) : 0;
  r.e_tile = e_tile;
  r.e0 = c * chunk;
  r.e1 = min(e_tile, r.e0 + chunk);
  r.base = r.nqt > 0 ? a.kv_row_off[r.b] : 0;
  const bool bounds_ok = r.base >= 0 && r.base + e_tile <= a.ki_rows;
  r.valid = r.nqt > 0 && r.e1 > r.e0 && bounds_ok;
  if (r.nqt > 0 && !bounds_ok && flag) flag_status(DSV4_ERR_DEVICE_BOUNDS);
  return r;
}

// Static schedule: units are numbered chunk-major (all tiles' first chunks, then their second
// chunks, ...), so the valid units of rows of different lengths form a dense prefix that the
// CTAs' round robin spreads evenly.
template <int QT>
__device__ __forceinline__ IxUnit ix_unit(const IndexArgs& a, int u, int q_begin, int q_count,
                                          int tile0, int tiles_per_seq, int chunk, int ntiles) {
  const int c = u / ntiles;
  return ix_tile_unit<QT>(a, tile0 + u % ntiles, c, q_begin, q_count, tiles_per_seq, chunk,
                          c == 0 && threadIdx.x == 0);
}

// Dynamic schedule: unit d of the dense tile-major list of valid units (tile i owns units
// pre[i] .. pre[i+1] - 1, one per chunk).
template <int QT, int NST, bool HIST, bool DYN, bool F4>
__device__ __forceinline__ IxUnit ix_dense_unit(const IndexArgs& a, const IndexSmem<QT, NST, HIST, DYN, F4>& s,
                                                int d, int q_begin, int q_count, int tile0,
                                                int tiles_per_seq, int chunk, int ntiles) {
  int lo = 0, hi = ntiles - 1;                 // the last tile i with pre[i] <= d
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (s.pre[mid] <= d) lo = mid;
    else hi = mid - 1;
  }
  return ix_tile_unit<QT>(a, tile0 + lo, d - s.pre[lo], q_begin, q_count, tiles_per_seq, chunk, false);
}

// Persistent: each CTA walks the work units blockIdx.x, blockIdx.x + gridDim.x, ... (DYN:
// the units the producer draws from *work, passed on through a FIFO); the key ring, the TMEM
// double buffer and their barrier phases run on across units (global block counter), the Q
// buffer is reloaded per unit once the MMAs of the previous unit are done.
template <int QT, int NST, bool HIST, bool DYN, bool F4>
__global__ void __launch_bounds__(ix_threads<F4>(), 1)
    index_tc_kernel(const IndexArgs a, const __grid_constant__ CUtensorMap map_q,
                    const __grid_constant__ CUtensorMap map_k, const __grid_constant__ CUtensorMap map_ks,
                    int q_begin, int q_count, int tile0, int tiles_per_seq, int chunk, int ntiles,
                    int units, int* work, uint32_t spin) {
  constexpr int EPI = 256;                             // epilogue threads (warps 0-7)
  constexpr int PROD_WARP = F4 ? 16 : 8, MMA_WARP = PROD_WARP + 1;
  constexpr int XW = 256;                              // F4: expanding threads (warps 8-15)
  extern __shared__ uint8_t smem_raw[];
  IndexSmem<QT, NST, HIST, DYN, F4>& s = *reinterpret_cast<IndexSmem<QT, NST, HIST, DYN, F4>*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  volatile int* abort = &s.abort;

  if (tid == 0) {
    tc::mbar_init(&s.q_full, 1);
    tc::mbar_init(&s.q_empty, 1);
    for (int i = 0; i < NST; ++i) {
      tc::mbar_init(&s.k_full[i], F4 ? 256 : 1);    // F4: the expanding threads
      tc::mbar_init(&s.k_empty[i], 1);
    }
    if constexpr (F4)
      for (int i = 0; i < IX_NSG; ++i) {
        tc::mbar_init(&s.sg_full[i], 1);
        tc::mbar_init(&s.sg_empty[i], 256);
      }
    for (int i = 0; i < 2; ++i) {
      tc::mbar_init(&s.d_full[i], 1);
      tc::mbar_init(&s.d_empty[i], EPI);
    }
    tc::mbar_init(&s.drain, 1);
    for (int i = 0; i < IX_UQ; ++i) {
      tc::mbar_init(&s.u_full[i], 1);
      tc::mbar_init(&s.u_empty[i], F4 ? 3 : 2);    // the MMA warp, the epilogue (F4: expanders)
    }
    s.abort = 0;
    tc::fence_barrier_init();
  }
  if constexpr (HIST)
    for (int e = tid; e < QT * TK_H1_BINS; e += blockDim.x) s.hist[e / TK_H1_BINS][e % TK_H1_BINS] = 0;
  if constexpr (DYN) {
    // The dense unit list: every epilogue thread counts the chunks of four consecutive tiles,
    // then a block scan turns the counts into each tile's first unit.
    if (warp < 8) {
      int cnt[4], sum = 0;
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const int i = 4 * tid + r;
        cnt[r] = 0;
        if (i < ntiles) {
          const IxUnit w0 = ix_tile_unit<QT>(a, tile0 + i, 0, q_begin, q_count, tiles_per_seq,
                                             chunk, blockIdx.x == 0);
          if (w0.valid) cnt[r] = (w0.e_tile + chunk - 1) / chunk;
        }
        sum += cnt[r];
      }
      int inc = sum;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += v;
      }
      if (lane == 31) s.wsum[warp] = inc;
      tc::named_barrier(1, 256);
      int run = inc - sum;
      for (int w2 = 0; w2 < warp; ++w2) run += s.wsum[w2];
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        if (4 * tid + r < ntiles) s.pre[4 * tid + r] = run;
        run += cnt[r];
      }
      if (tid == 255) s.n_dense = run;
    }
  }
  if (warp == MMA_WARP) {
    tc::tmem_alloc(&s.tmem_base, IX_TM_COLS);
    tc::tmem_relinquish();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = s.tmem_base;

  uint32_t prod_gb = 0;                                // key blocks the producer issued
  int prod_k = 0;                                      // units whose Q it loaded
  if (warp == PROD_WARP) {
    // ------------------------------------------------------------------ producer
    if (lane == 0) {
      tc::prefetch_tensormap(&map_q);
      tc::prefetch_tensormap(&map_k);
      if constexpr (F4) tc::prefetch_tensormap(&map_ks);
      uint32_t& gb = prod_gb;                          // key blocks issued so far
      int& k = prod_k;                                 // units loaded so far
      bool ok = true;
      int d = 0;                                       // DYN: this unit's ticket
      if constexpr (DYN) d = atomicAdd(work, 1);
      for (int it = 0, u = blockIdx.x; ok; ++it, u += gridDim.x) {
        IxUnit w;
        if constexpr (DYN) {
          // publish the unit (or the end) to the MMA warp and the epilogue; the next ticket is
          // drawn now and arrives while this unit's blocks stream
          const bool more = d < s.n_dense;
          const int nd = more ? atomicAdd(work, 1) : 0;
          const int slot = it % IX_UQ;
          if (it >= IX_UQ && !tc::mbar_wait(&s.u_empty[slot], (uint32_t)((it / IX_UQ - 1) & 1), spin, abort))
            break;
          s.uid[slot] = more ? d : -1;
          tc::mbar_arrive(&s.u_full[slot]);
          if (!more) break;
          w = ix_dense_unit(a, s, d, q_begin, q_count, tile0, tiles_per_seq, chunk, ntiles);
          d = nd;
        } else {
          if (u >= units) break;
          w = ix_unit<QT>(a, u, q_begin, q_count, tile0, tiles_per_seq, chunk, ntiles);
          if (!w.valid) continue;
        }
        // The unit's Q goes into the single Q buffer once the MMAs of the previous unit have
        // completed (q_empty). Meanwhile the unit's first key blocks already enter the ring:
        // up to NST of them reuse stages the previous units released, so the ring stays full
        // across the unit boundary; a later block's stage is released only by this unit's
        // MMAs, which need its Q, so Q is loaded (waiting if need be) before that.
        bool q_loaded = false;
        auto load_q = [&]() {
          tc::mbar_arrive_expect_tx(&s.q_full, 2 * QT * IX_HI * 128);
          const int qrow = (w.qlo - a.q_map_q0) * IX_HI;
          tc::tma_load_2d(s.q[0], &map_q, &s.q_full, 0, qrow);
          tc::tma_load_2d(s.q[1], &map_q, &s.q_full, 64, qrow);
          q_loaded = true;
        };
        auto q_free = [&](bool block) {
          if (k == 0) return true;
          const uint32_t par = (uint32_t)((k - 1) & 1);
          return block ? tc::mbar_wait(&s.q_empty, par, spin, abort) : tc::mbar_test_wait(&s.q_empty, par);
        };
        const uint32_t gb0 = gb;
        const int nblk = (w.e1 - w.e0 + IX_BLK - 1) / IX_BLK;
        constexpr int RING = F4 ? IX_NSG : NST;         // the ring this warp fills
        for (int blk = 0; blk < nblk; ++blk, ++gb) {
          const int st = gb % RING, use = gb / RING;
          if (!q_loaded && gb >= gb0 + RING) {
            if (!q_free(true)) {
              ok = false;
              break;
            }
            load_q();
          }
          uint64_t* empty = F4 ? &s.sg_empty[st] : &s.k_empty[st];
          if (use > 0 && !tc::mbar_wait(empty, (uint32_t)((use - 1) & 1), spin, abort)) {
            ok = false;
            break;
          }
          if (!q_loaded && q_free(false)) load_q();
          const int row = (int)(w.base + w.e0 + blk * IX_BLK);
          if constexpr (F4) {
            // codes of rows [row, row + 128) and scales of the row pairs from row / 2 (rows
            // past the pool read as zeros); an odd pool's last row is loaded on its own
            if ((a.ki_rows & 1) && row <= a.ki_rows - 1 && a.ki_rows - 1 < row + IX_BLK)
              s.sg_last[st] = *reinterpret_cast<const uint64_t*>(a.KI_scales + (a.ki_rows - 1) * 8);
            tc::mbar_arrive_expect_tx(&s.sg_full[st], IX_BLK * 64 + IX_SG_PAIRS * 16);
            tc::tma_load_3d(s.sg_codes[st], &map_k, &s.sg_full[st], 0, row, 0);
            tc::tma_load_2d(s.sg_scales[st], &map_ks, &s.sg_full[st], 0, row >> 1);
          } else {
            tc::mbar_arrive_expect_tx(&s.k_full[st], 2 * IX_BLK * 128);
            tc::tma_load_2d(s.k[st][0], &map_k, &s.k_full[st], 0, row);
            tc::tma_load_2d(s.k[st][1], &map_k, &s.k_full[st], 64, row);
          }
          IX_TRACE(0, (int)gb);
        }
        if (ok && !q_loaded) {
          if (!q_free(true)) break;
          load_q();
        }
        if (q_loaded) ++k;
      }
    }
    __syncwarp();
  } else if (warp == MMA_WARP) {
    // ------------------------------------------------------------------ MMA issuer
    // The warp stays converged: every lane waits (acquire per lane), the warp takes one
    // decision, and elect.sync lets one lane issue. A single-lane branch issued the MMAs and
    // passed completed barriers several times more slowly, which capped the key stream.
    {
      const uint64_t d_k0 = tc::sdesc_sw128(tc::smem_u32(s.k[0][0]), 16, 1024);
      const uint64_t d_q0 = tc::sdesc_sw128(tc::smem_u32(s.q[0]), 16, 1024);
      auto wwait = [&](uint64_t* bar, uint32_t parity) {
        return __all_sync(0xffffffffu, tc::mbar_wait(bar, parity, spin, abort)) != 0;
      };
      uint32_t gb = 0;
      int k = 0;
      bool ok = true;
      for (int it = 0, u = blockIdx.x; ok; ++it, u += gridDim.x) {
        IxUnit w;
        if constexpr (DYN) {
          const int slot = it % IX_UQ;
          ok = wwait(&s.u_full[slot], (uint32_t)((it / IX_UQ) & 1));
          if (!ok) break;
          const int d = s.uid[slot];
          __syncwarp();
          if (lane == 0) tc::mbar_arrive(&s.u_empty[slot]);
          if (d < 0) break;
          w = ix_dense_unit(a, s, d, q_begin, q_count, tile0, tiles_per_seq, chunk, ntiles);
        } else {
          if (u >= units) break;
          w = ix_unit<QT>(a, u, q_begin, q_count, tile0, tiles_per_seq, chunk, ntiles);
          if (!w.valid) continue;
        }
        ok = wwait(&s.q_full, (uint32_t)(k & 1));
        ++k;
        const uint32_t idesc = F4 ? tc::idesc_f16_f32(128, IX_HI * w.nqt, 0, 0)
                                  : tc::idesc_bf16_f32(128, IX_HI * w.nqt, 0, 0);
        const int nblk = (w.e1 - w.e0 + IX_BLK - 1) / IX_BLK;
        for (int blk = 0; blk < nblk && ok; ++blk, ++gb) {
          const int st = gb % NST, buf = gb & 1;
          ok = wwait(&s.k_full[st], (uint32_t)((gb / NST) & 1));
          IX_TRACE(1, (int)gb);
          if (ok && gb >= 2) ok = wwait(&s.d_empty[buf], (uint32_t)(((gb >> 1) - 1) & 1));
          IX_TRACE(2, (int)gb);
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
          IX_TRACE(3, (int)gb);
        }
        if (ok) tc::mma_commit_warp(&s.q_empty);       // the unit's Q is no longer read
      }
      if (!ok) {
        // let every issued MMA finish before TMEM is released
        tc::mma_commit_warp(&s.drain);
        tc::mbar_drain(&s.drain, 0);
      }
    }
    __syncwarp();
  } else if (F4 && warp >= 8) {
    // ------------------------------------------------------------------ FP4 key expansion
    // 256 threads expand the 512 (row, 32-channel chunk) items of every block, two each; each
    // quarter warp takes one chunk of 8 consecutive rows: its staging reads are 128 contiguous
    // bytes (the staging is chunk-major) and its tile stores land in 8 distinct swizzle slots
    const int xt = tid - 256, xw = xt >> 5, xl = xt & 31;
    uint32_t gb = 0;
    bool ok = true;
    for (int it = 0, u = blockIdx.x; ok; ++it, u += gridDim.x) {
      IxUnit w;
      if constexpr (DYN) {
        const int slot = it % IX_UQ;
        int d = 0;
        if (ok) ok = tc::mbar_wait(&s.u_full[slot], (uint32_t)((it / IX_UQ) & 1), spin, abort);
        if (ok) d = s.uid[slot];
        if (ix_red_or(4, XW, !ok)) break;          // all of them read the slot (or gave up)
        if (xt == 0) tc::mbar_arrive(&s.u_empty[slot]);
        if (d < 0) break;
        w = ix_dense_unit(a, s, d, q_begin, q_count, tile0, tiles_per_seq, chunk, ntiles);
      } else {
        if (u >= units) break;
        w = ix_unit<QT>(a, u, q_begin, q_count, tile0, tiles_per_seq, chunk, ntiles);
        if (!w.valid) continue;
      }
      const int nblk = (w.e1 - w.e0 + IX_BLK - 1) / IX_BLK;
      for (int blk = 0; blk < nblk && ok; ++blk, ++gb) {
        const int sg = gb % IX_NSG, st = gb % NST;
        ok = tc::mbar_wait(&s.sg_full[sg], (uint32_t)((gb / IX_NSG) & 1), spin, abort);
        if (ok && gb >= (uint32_t)NST) ok = tc::mbar_wait(&s.k_empty[st], (uint32_t)((gb / NST - 1) & 1), spin, abort);
        if (!ok) break;
        const long long row0 = w.base + w.e0 + (long long)blk * IX_BLK;
#pragma unroll
        for (int k2 = 0; k2 < 2; ++k2) {
          const int r = 16 * xw + 8 * k2 + (xl & 7), c = xl >> 3;
          uint32_t sc2 = *reinterpret_cast<const uint16_t*>(s.sg_scales[sg] + ((row0 & 1) + r) * 8 + 2 * c);
          if ((a.ki_rows & 1) && row0 + r == a.ki_rows - 1) sc2 = (uint32_t)(s.sg_last[sg] >> (16 * c)) & 0xFFFFu;
          f4_expand_chunk(s.sg_codes[sg] + c * (IX_BLK * 16) + r * 16, sc2, s.k[st][c >> 1], r, 4 * (c & 1));
        }
        tc::fence_proxy_async_smem();              // generic stores -> tensor-core reads
        tc::mbar_arrive(&s.sg_empty[sg]);
        tc::mbar_arrive(&s.k_full[st]);
      }
    }
  } else {
    // ------------------------------------------------------------------ epilogue warps
    const int quad = warp & 3;                    // TMEM lane quadrant
    const int qp = warp >> 2;                     // query pair: queries 2qp, 2qp+1
    const uint32_t lane_base = (uint32_t)(32 * quad) << 16;
    uint32_t gb = 0;
    bool ok = true;
    for (int it = 0, u = blockIdx.x;; ++it, u += gridDim.x) {
      IxUnit w;
      if constexpr (DYN) {
        const int slot = it % IX_UQ;
        int d = 0;
        if (ok) ok = tc::mbar_wait(&s.u_full[slot], (uint32_t)((it / IX_UQ) & 1), spin, abort);
        if (ok) d = s.uid[slot];
        // every epilogue thread has finished the previous unit and read this slot; after a
        // failed wait all of them leave here together (named barriers below need all of them)
        if (ix_red_or(1, EPI, !ok)) break;
        if (tid == 0) tc::mbar_arrive(&s.u_empty[slot]);
        if (d < 0) break;
        w = ix_dense_unit(a, s, d, q_begin, q_count, tile0, tiles_per_seq, chunk, ntiles);
      } else {
        if (u >= units) break;
        w = ix_unit<QT>(a, u, q_begin, q_count, tile0, tiles_per_seq, chunk, ntiles);
        if (!w.valid) continue;
        // every epilogue thread has finished the previous unit; after a failed wait all of
        // them leave here together (named barriers below need all of them)
        if (ix_red_or(1, EPI, !ok)) break;
      }
      // the unit's head weights
      for (int e = tid; e < QT * IX_HI; e += EPI) {
        const int q = e / IX_HI, h = e % IX_HI;
        s.w[q][h] = q < w.nqt ? a.w[(long long)(w.qlo + q) * a.H_I + h] : 0.f;
      }
      tc::named_barrier(1, EPI);
      int Et[2];
      long long srow[2];
#pragma unroll
      for (int v = 0; v < 2; ++v) {
        const int qu = 2 * qp + v;
        Et[v] = qu < w.nqt ? visible_entries(a, w.b, w.qlo + qu - w.b * a.nq) : 0;
        srow[v] = (long long)(w.qlo + qu - a.score_q0) * a.scores_ld;
      }
      const int nblk = (w.e1 - w.e0 + IX_BLK - 1) / IX_BLK;
      for (int blk = 0; blk < nblk; ++blk, ++gb) {
        const int buf = gb & 1;
        ok = tc::mbar_wait(&s.d_full[buf], (uint32_t)((gb >> 1) & 1), spin, abort);
        if (!ok) break;
        if (tid == 0) IX_TRACE(4, (int)gb);
        tc::tc_fence_after();
        if constexpr (QT == 1) {
          // one query: warps w and w+4 share TMEM lane quadrant w%4 (the block's entries
          // 32(w%4)..+31) and take heads 0-31 and 32-63; the second half's partial sums meet
          // the first half's through shared memory
          const int hh = warp >> 2;
          float d0[32];
          tc::tmem_ld32(tmem + lane_base + buf * 256 + hh * 32, d0);
          tc::tmem_wait_ld_dep(d0);
          tc::tc_fence_before();
          tc::mbar_arrive(&s.d_empty[buf]);
          if (tid == 0) IX_TRACE(5, (int)gb);
          const float part = ix_half_sum(d0, &s.w[0][32 * hh]);
          const int e = 32 * quad + lane;
          if (hh == 1) s.part[buf][e] = part;
          tc::named_barrier(1, 256);
          if (hh == 0) {
            const int sidx = w.e0 + blk * IX_BLK + e;
            const float sc0 = part + s.part[buf][e];
            if (sidx < Et[0]) a.scores[srow[0] + sidx] = sc0;
            if constexpr (HIST)                  // first histogram of the threshold top-k
              hist_add(s.hist[0], score_key(sc0) >> (32 - TK_H1_BITS), sidx < Et[0]);
          }
          if (tid == 0) IX_TRACE(6, (int)gb);
        } else {
          const uint32_t col = tmem + lane_base + buf * 256 + qp * 128;
          const bool two = 2 * qp < w.nqt;        // this warp has work in the tile
          // per 32-head half four interleaved sums (short dependency chains), combined in the
          // one-query tile's order; one query's TMEM columns at a time (register budget)
          float sc0 = 0.f, sc1 = 0.f;
          if (two) {
            float d0[32], d1[32];
            tc::tmem_ld32(col, d0);
            tc::tmem_ld32(col + 32, d1);
            tc::tmem_wait_ld();
            sc0 = ix_half_sum(d0, &s.w[2 * qp][0]) + ix_half_sum(d1, &s.w[2 * qp][32]);
            tc::tmem_ld32(col + 64, d0);
            tc::tmem_ld32(col + 96, d1);
            tc::tmem_wait_ld();
            sc1 = ix_half_sum(d0, &s.w[2 * qp + 1][0]) + ix_half_sum(d1, &s.w[2 * qp + 1][32]);
          }
          tc::tc_fence_before();
          tc::mbar_arrive(&s.d_empty[buf]);
          if (tid == 0) IX_TRACE(5, (int)gb);
          if (!two) continue;
          const int sidx = w.e0 + blk * IX_BLK + 32 * quad + lane;
          if (sidx < Et[0]) a.scores[srow[0] + sidx] = sc0;
          if (tid == 0) IX_TRACE(6, (int)gb);
          if (2 * qp + 1 < w.nqt && sidx < Et[1]) a.scores[srow[1] + sidx] = sc1;
        }
      }
      if constexpr (HIST) {
        // add the unit's histogram to its row's first histogram (int hist1[TK_H1_BINS] at
        // the start of the row's top-k region) and clear it for the next unit
        tc::named_barrier(1, EPI);
        int* h1 = reinterpret_cast<int*>(a.cand + (long long)(w.qlo - a.score_q0) * a.cand_row_bytes);
        for (int e = tid; e < TK_H1_BINS; e += EPI) {
          const int v = s.hist[0][e];
          if (v) {
            atomicAdd(h1 + e, v);
            s.hist[0][e] = 0;
          }
        }
      }
    }
  }
  tc::tc_fence_before();
  __syncthreads();
  if (warp == MMA_WARP) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, IX_TM_COLS);
  }
  if (tid == PROD_WARP * 32 && *abort) {
    // After an abort (final now: every thread has passed the barrier) the producer's last
    // key blocks and Q may still be landing: let them land before the CTA's shared memory
    // is released. Without an abort the MMAs consumed them all.
    constexpr uint32_t RING = F4 ? IX_NSG : NST;
    for (uint32_t g = prod_gb > RING ? prod_gb - RING : 0; g < prod_gb; ++g)
      tc::mbar_drain(F4 ? &s.sg_full[g % RING] : &s.k_full[g % RING], (g / RING) & 1);
    if (prod_k > 0) tc::mbar_drain(&s.q_full, (uint32_t)((prod_k - 1) & 1));
  }
}

}  // namespace

int launch_index_scores_tc(const IndexArgs& a, int q_begin, int q_count, int max_e,
                           cudaStream_t st, bool* used, bool* hist1_built) {
  *used = false;
  *hist1_built = false;
  const char* force = std::getenv("DSV4_FORCE_SIMT");
  if (force && force[0] == '1') return DSV4_OK;
  if (a.qdtype != DSV4_BF16 || a.c_I != IX_CI || a.H_I != IX_HI) return DSV4_OK;
  if (!aligned16(a.qI) || !aligned16(a.KI)) return DSV4_OK;
  // FP4 keys: one query per sequence, 16-byte aligned scales, a pool of at least one staging
  // box of scale row pairs
  const bool f4 = a.k_fp4 != 0;
  if (f4 && (a.nq != 1 || !aligned16(a.KI_scales) || a.ki_rows < 2 * IX_SG_PAIRS)) return DSV4_OK;
  if (q_count <= 0 || max_e <= 0) {
    *used = true;
    *hist1_built = true;
    return DSV4_OK;
  }
  const long long q_rows = a.q_map_rows > 0 ? a.q_map_rows : (long long)a.B * a.nq * IX_HI;
  if (q_rows >= (1ll << 31) || a.ki_rows >= (1ll << 31) || a.ki_rows <= 0) return DSV4_OK;
  // one query per sequence (decode): one-query tiles with a 6-stage key ring
  const int qt = a.nq == 1 ? 1 : IX_QT;
  CUtensorMap mq, mk, mks;
  int s = encode_tensor_map_2d(&mq, a.qI, f4 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                               2, IX_CI, q_rows, 64, qt * IX_HI, CU_TENSOR_MAP_SWIZZLE_128B);
  if (s != DSV4_OK) return s;
  if (f4) {
    // codes [ki_rows, 64 B] seen as (16-byte piece, row, chunk) so that a box of 128 rows lands
    // chunk-major -- [4 chunks][128 rows][16 B]: consecutive rows of one chunk are adjacent --
    // and scales as 16-byte row pairs [ki_rows / 2, 16 B] in boxes of 65 pairs (an odd pool's
    // last row is read on its own)
    const uint64_t cdims[3] = {16, (uint64_t)a.ki_rows, 4}, cstr[2] = {64, 16};
    const uint32_t cbox[3] = {16, IX_BLK, 4};
    s = encode_tensor_map_3d(&mk, a.KI, CU_TENSOR_MAP_DATA_TYPE_UINT8, cdims, cstr, cbox);
    if (s != DSV4_OK) return s;
    s = encode_tensor_map_2d(&mks, a.KI_scales, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, 16, a.ki_rows / 2, 16,
                             IX_SG_PAIRS, CU_TENSOR_MAP_SWIZZLE_NONE);
  } else {
    s = encode_tensor_map_2d(&mk, a.KI, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, IX_CI, a.ki_rows, 64,
                             IX_BLK, CU_TENSOR_MAP_SWIZZLE_128B);
    mks = mk;
  }
  if (s != DSV4_OK) return s;
  const int tps = (a.nq + qt - 1) / qt;
  auto tile_of = [&](int qg) { return (qg / a.nq) * tps + (qg % a.nq) / qt; };
  const int t0 = tile_of(q_begin), t1 = tile_of(q_begin + q_count - 1);
  // Work units (tile, chunk of entries); one persistent CTA per SM walks them.
  static int sms = 0;
  if (sms == 0) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0)
      sms = 148;
  }
  // Prefill tiles (several queries): persistent CTAs, one per SM, walk units of IX_CHUNK
  // entries (per-tile CTAs paid their setup and pipeline fill on only a few key blocks).
  // One-query tiles (decode over long rows of very different lengths) with the threshold
  // top-k's row headers: persistent CTAs draw IX_DYN_CHUNK-entry units from a counter in the
  // first row's header (zeroed before this launch) -- finely balanced, no CTA start per unit
  // (2048-entry units: 469 us for the 2.35 GB of keys of 64 rows of 32k-262k entries; 4096:
  // 475 us; 8192: 485 us; one CTA per 16384-entry unit: 530 us, top-k passes included).
  // Otherwise one CTA per unit, so that the hardware hands units to SMs as they free up (a
  // static walk balanced them worse); units grow to 16384 entries while there are at least 4
  // per SM.
  const long long tiles = t1 - t0 + 1;
  const bool dyn = qt == 1 && a.topk_pipe && a.cand && tiles <= IX_DYN_TILES;
  int chunk = dyn ? IX_DYN_CHUNK : IX_CHUNK;
  if (qt == 1 && !dyn)
    while (chunk < 4 * IX_CHUNK && tiles * ((max_e + 2 * chunk - 1) / (2 * chunk)) >= 4 * sms) chunk *= 2;
  const long long nchunk = (max_e + chunk - 1) / chunk;
  const long long units = tiles * nchunk;
  if (units >= (1ll << 31)) return DSV4_OK;
  const unsigned grid = (unsigned)((qt == 1 && !dyn) || units < sms ? units : sms);
  int* work = dyn ? reinterpret_cast<int*>(a.cand + (long long)(q_begin - a.score_q0) * a.cand_row_bytes +
                                           TK_WORK_BYTE)
                  : nullptr;
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaSuccess;
    auto smem_attr = [&](const void* fn, size_t bytes) {
      if (e == cudaSuccess) e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    };
    smem_attr((const void*)index_tc_kernel<IX_QT, IX_STAGES, false, false, false>, ix_smem<IX_QT, IX_STAGES, false, false, false>());
    smem_attr((const void*)index_tc_kernel<1, 6, false, false, false>, ix_smem<1, 6, false, false, false>());
    smem_attr((const void*)index_tc_kernel<1, 6, true, false, false>, ix_smem<1, 6, true, false, false>());
    smem_attr((const void*)index_tc_kernel<1, 6, true, true, false>, ix_smem<1, 6, true, true, false>());
    smem_attr((const void*)index_tc_kernel<1, 4, false, false, true>, ix_smem<1, 4, false, false, true>());
    smem_attr((const void*)index_tc_kernel<1, 4, true, false, true>, ix_smem<1, 4, true, false, true>());
    smem_attr((const void*)index_tc_kernel<1, 4, true, true, true>, ix_smem<1, 4, true, true, true>());
    if (e != cudaSuccess) return fail(DSV4_ERR_CUDA, "index_tc: %s", cudaGetErrorString(e));
    attr_set = true;
  }
  const int sp = spin_limit();
#define IX_LAUNCH(QT_, NST_, HIST_, DYN_, F4_)                                                  \
  index_tc_kernel<QT_, NST_, HIST_, DYN_, F4_><<<grid, ix_threads<F4_>(), ix_smem<QT_, NST_, HIST_, DYN_, F4_>(), st>>>( \
      a, mq, mk, mks, q_begin, q_count, t0, tps, chunk, (int)tiles, (int)units, work, sp)
  if (f4) {
    if (dyn) IX_LAUNCH(1, 4, true, true, true);
    else if (a.topk_pipe) IX_LAUNCH(1, 4, true, false, true);
    else IX_LAUNCH(1, 4, false, false, true);
  } else if (qt == 1) {
    if (dyn) IX_LAUNCH(1, 6, true, true, false);
    else if (a.topk_pipe) IX_LAUNCH(1, 6, true, false, false);
    else IX_LAUNCH(1, 6, false, false, false);
  } else {
    IX_LAUNCH(IX_QT, IX_STAGES, false, false, false);
  }
#undef IX_LAUNCH
  *used = true;
  *hist1_built = qt == 1 && a.topk_pipe;
  return launch_status("index scores (tensor cores)");
}

}  // namespace dsv4

#ifdef DSV4_TRACE
extern "C" int dsv4_trace_read_ix(unsigned long long* host, size_t n) {
  return cudaMemcpyFromSymbol(host, dsv4::g_ix_trace, n * sizeof(unsigned long long)) == cudaSuccess ? 0 : 3;
}
#endif
