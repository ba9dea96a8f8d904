// Hybrid shared-KV MQA on the tensor cores with double-buffered 64-slot KV blocks
// (prefill: one CTA per SM, persistent over (query, 64-head group) items). Selected with
// DSV4_ATTN_DB=1; the 128-slot single-buffer kernel is the default.
//
// "CSA And HCA: Definition, State, And Cost Model": s3.2/s4 every candidate row is both key
// and value for all heads; s5.1 one candidate list (selected or all completed compressed
// entries, then the local window) under one softmax per head; s5.3 the sink logit joins
// the denominator only. Per-query valid counts follow pypto-lib PR #834.
//
// Same transposed contraction as the single-buffered kernel, on blocks of 64 candidate
// slots so that two blocks fit in shared memory next to Q:
//   GEMM1  S^T[64 slots x 64 heads] = KV[slots x c] . Q[heads x c]^T   (M = 64, K = c)
//   GEMM2  O^T[c x 64 heads]      += KV^T[c x slots] . P^T[slots x heads] (M = 128, K = 64)
// The MMA warp issues the K chunks of GEMM1(G) as they land and GEMM2(G-1) as soon as the
// softmax has published P of block G-1, so the tensor core works on block G while the
// softmax warps turn block G-1 into P; GEMM2 tile q of block G releases KV chunks 2q, 2q+1
// of its buffer to the producer warp that fills them for block G+2. S^T and P are
// double-buffered too.
//
// Warps: 0-7 softmax/epilogue (warp w: S^T rows 16(w%4)..+15 in the M=64 TMEM layout, heads
// 32(w/4)..+31, read as 16x256b fragments: each thread holds 2 slots x 8 heads); 8-11
// cp.async row gather, warp 8+q filling chunk pair q (window rows by 2D TMA); 12 watcher
// (waits for the chunk-pair releases on the producers' behalf, passes them on through named
// barriers); 13 MMA issuer and TMEM owner. All waits are bounded.
//
// Measured on B200 (flash CSA prefill, n = 8192, k = 512, w = 128): 1.57 ms against 1.27 ms
// for the 128-slot kernel. The gather alone (no MMA, no softmax) takes 0.9 ms in this
// structure; with the MMAs running, the gathered rows land several times slower, because
// the tensor core's shared-memory operand reads (Q is re-read for every 64-slot block) and
// the cp.async writes share the shared-memory bandwidth.
#include <cstdio>
#include <cstdlib>

#include "attn_common.cuh"
#include "tc_common.cuh"

namespace dsv4 {
namespace {

constexpr int DB_C = 512;
constexpr int DB_H = 64;
constexpr int DB_BLK = 64;
constexpr int DB_CHUNKS = DB_C / 64;
constexpr int DB_SOFT = 256;
constexpr int DB_PROD = 128;
constexpr int DB_THREADS = DB_SOFT + DB_PROD + 64;
constexpr uint32_t DB_TM_S = 0;             // S^T buffers: columns [0, 64) and [64, 128)
constexpr uint32_t DB_TM_O = 128;           // O^T: 4 tiles x 64 columns
constexpr uint32_t DB_TM_COLS = 512;
constexpr float DB_TAU = 8.f;               // log2-domain growth tolerated before rescaling
constexpr float DB_LOG2E = 1.4426950408889634f;
constexpr float DB_LN2 = 0.6931471805599453f;
// named barriers: 1-3 softmax warps, 5 producers, 6-13 chunk-pair gates (buffer b, pair q:
// 6 + 4b + q), 14 item gate
constexpr uint32_t DB_GATE_ITEM = 14;
constexpr uint32_t DB_GATE_PAIR0 = 6;

struct DbSmem {
  uint8_t q[DB_CHUNKS][DB_H * 128];           // K-major SW128 [64 heads][64 ch] per chunk
  uint8_t kv[2][DB_CHUNKS][DB_BLK * 128];     // per buffer: [64 slots][64 ch] per chunk
  uint8_t p[2][DB_BLK * 128];                 // MN-major SW128 P^T [64 slots][64 heads];
                                              // together the O staging boxes of the epilogue
  float red[4][DB_H];
  float mcur[DB_H];
  float moff[DB_H];
  float fac[DB_H];
  float inv[DB_H];
  uint64_t rowaddr[DB_BLK];
  uint64_t q_full, q_empty;
  uint64_t ch_full[2][DB_CHUNKS];
  uint64_t kv_empty[2][4];               // chunk pair q of buffer b released by GEMM2
  uint64_t s_full[2], s_empty[2], p_full[2];
  uint64_t o_done, o_final, drain;
  uint32_t tmem_base;
  int abort;
};
constexpr size_t DB_SMEM = sizeof(DbSmem) + 1024;
static_assert(DB_SMEM <= 232448, "shared memory of the double-buffered attention kernel");

#ifdef DSV4_TRACE
__device__ unsigned long long g_db_trace[4][12][32];
#define DB_TRACE(ev, k_, j_)                                     \
  do {                                                           \
    if (blockIdx.x == 0 && (k_) >= 40 && (k_) < 44 && (j_) < 12) \
      g_db_trace[(k_) - 40][j_][ev] = clock64();                 \
  } while (0)
#else
#define DB_TRACE(ev, k_, j_) \
  do {                       \
  } while (0)
#endif

__device__ __forceinline__ bool db_red_or(uint32_t id, uint32_t threads, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n .reg .pred p, q;\n setp.ne.u32 p, %1, 0;\n"
      " barrier.red.or.pred q, %2, %3, p;\n selp.u32 %0, 1, 0, q;\n}"
      : "=r"(r)
      : "r"((uint32_t)pred), "r"(id), "r"(threads)
      : "memory");
  return r != 0;
}
// Non-blocking test of an mbarrier phase (acquire on success).
__device__ __forceinline__ bool db_test(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}"
      : "=r"(ok)
      : "r"(tc::smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded wait for an mbarrier phase, as tc::mbar_wait, but gentler on the shared-memory
// pipe that the producers' cp.async traffic also uses: each poll may suspend the thread
// until the phase completes (try_wait with a time hint) or, in mode 2, polls sleep.
#ifndef DB_WAIT_MODE
#define DB_WAIT_MODE 1
#endif
__device__ __forceinline__ bool db_try(uint64_t* bar, uint32_t parity) {
#if DB_WAIT_MODE == 1
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n selp.u32 %0, 1, 0, p;\n}"
      : "=r"(ok)
      : "r"(tc::smem_u32(bar)), "r"(parity), "r"(2000u)
      : "memory");
  return ok != 0;
#elif DB_WAIT_MODE == 2
  if (tc::mbar_try_wait(bar, parity)) return true;
  __nanosleep(64);
  return false;
#else
  return tc::mbar_try_wait(bar, parity);
#endif
}
__device__ __forceinline__ bool db_wait(uint64_t* bar, uint32_t parity, uint32_t spin_limit,
                                        volatile int* abort) {
  for (uint32_t i = 0; i < spin_limit; ++i) {
    if (db_try(bar, parity)) return true;
    if ((i & 63u) == 63u) {
      if (*abort) return false;
      if (*reinterpret_cast<volatile int*>(&g_status) == DSV4_ERR_DEVICE_TIMEOUT) {
        *abort = 1;
        return false;
      }
    }
  }
  flag_status(DSV4_ERR_DEVICE_TIMEOUT);
  *abort = 1;
  return false;
}
__device__ __forceinline__ bool db_gate(uint32_t id, bool pred) {
  return db_red_or(id, DB_PROD + 32, pred);
}
// Pair gates: one producer warp and the watcher warp.
__device__ __forceinline__ void db_arrive(uint32_t id) {
  asm volatile("bar.arrive %0, %1;" ::"r"(id), "r"(64) : "memory");
}
__device__ __forceinline__ void db_sync(uint32_t id) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(64) : "memory");
}
__device__ __forceinline__ void db_cp16(uint32_t dst, uint64_t src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void db_cp_arrive(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(tc::smem_u32(bar))
               : "memory");
}
__device__ __forceinline__ uint32_t db_pack(float lo, float hi) {
  __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&p);
}
__device__ __forceinline__ float2 db_unpack(uint32_t u) {
  return __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u));
}
// Four 8x8 b16 matrices, stored row-major: register j of thread t holds elements
// (t/4, 2(t%4)) and (t/4, 2(t%4)+1) of matrix j; threads 8j..8j+7 give its row addresses.
__device__ __forceinline__ void db_stmatrix_x4(uint32_t addr, uint32_t r0, uint32_t r1, uint32_t r2,
                                               uint32_t r3) {
  asm volatile("stmatrix.sync.aligned.m8n8.x4.shared.b16 [%0], {%1, %2, %3, %4};" ::"r"(addr),
               "r"(r0), "r"(r1), "r"(r2), "r"(r3)
               : "memory");
}

// Candidate slot g of a query: whether it holds a candidate and, for the producers, its row
// address (pool or local); slots past a part's count fetch an in-range row and are masked.
struct DbSlot {
  bool valid;
  bool bad_index;
  uint64_t addr;
};

__device__ __forceinline__ DbSlot db_slot(const AttnArgs& a, const CandidateSet& cs, int nc4, int g) {
  DbSlot r;
  r.bad_index = false;
  const uint64_t pool_addr = reinterpret_cast<uint64_t>(a.pool);
  const uint64_t local_addr = reinterpret_cast<uint64_t>(a.local);
  r.addr = local_addr + (uint64_t)cs.local_base * DB_C * 2;
  if (g < nc4) {
    r.valid = g < cs.n_comp;
    if (r.valid) {
      const long long s = cs.sel ? (long long)__ldg(cs.sel + g) : (long long)g;
      const long long row = cs.pool_base + s;
      if (s < 0 || s >= cs.Et || row < 0 || row >= a.pool_rows) {
        r.valid = false;
        r.bad_index = true;
      } else {
        r.addr = pool_addr + (uint64_t)row * DB_C * 2;
      }
    }
  } else {
    const int jl = g - nc4;
    r.valid = jl < cs.n_local;
    if (r.valid) r.addr = local_addr + (uint64_t)(cs.local_base + (cs.win0 + jl) % a.R) * DB_C * 2;
  }
  return r;
}

struct DbItem {
  int qi, hg, nc4, nb;
  CandidateSet cs;
};

__device__ __forceinline__ DbItem db_item(const AttnArgs& a, int item, int head_groups) {
  DbItem it;
  it.qi = item / head_groups;
  it.hg = item % head_groups;
  const int b = it.qi / a.nq, i = it.qi % a.nq;
  it.cs = make_candidates(a, b, i);
  it.nc4 = (it.cs.n_comp + 3) & ~3;
  const int nl4 = (it.cs.n_local + 3) & ~3;
  it.nb = (it.nc4 + nl4 + DB_BLK - 1) / DB_BLK;
  return it;
}

__global__ void __maxnreg__(128)
    attn_db_kernel(const AttnArgs a, const __grid_constant__ CUtensorMap map_q,
                   const __grid_constant__ CUtensorMap map_local,
                   const __grid_constant__ CUtensorMap map_o, int head_groups, int items,
                   float scale_log2, uint32_t spin) {
  extern __shared__ uint8_t smem_raw[];
  DbSmem& s = *reinterpret_cast<DbSmem*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  volatile int* abort = &s.abort;

  if (tid == 0) {
    tc::mbar_init(&s.q_full, 1);
    tc::mbar_init(&s.q_empty, 1);
    for (int b = 0; b < 2; ++b) {
      for (int c = 0; c < DB_CHUNKS; ++c) tc::mbar_init(&s.ch_full[b][c], 32);
      for (int q = 0; q < 4; ++q) tc::mbar_init(&s.kv_empty[b][q], 1);
      tc::mbar_init(&s.s_full[b], 1);
      tc::mbar_init(&s.s_empty[b], DB_SOFT);
      tc::mbar_init(&s.p_full[b], DB_SOFT);
    }
    tc::mbar_init(&s.o_done, 1);
    tc::mbar_init(&s.o_final, 1);
    tc::mbar_init(&s.drain, 1);
    s.abort = 0;
    tc::fence_barrier_init();
  }
  if (tid < DB_H) s.mcur[tid] = -INFINITY;
  if (warp == 13) {
    tc::tmem_alloc(&s.tmem_base, DB_TM_COLS);
    tc::tmem_relinquish();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = s.tmem_base;

  if (warp >= 8 && warp < 12) {
    // ------------------------------------------------------------------ producer (4 warps)
    const int pt = tid - DB_SOFT, pw = pt >> 5;
    uint32_t G = 0;                                    // global block counter of this CTA
    int k = 0;
    bool ok = true;
    if (pt == 0) tc::prefetch_tensormap(&map_q);
    for (int item = blockIdx.x; item < items && ok; item += gridDim.x) {
      const DbItem it = db_item(a, item, head_groups);
      ok = !db_gate(DB_GATE_ITEM, false);              // the Q buffer is free (or abort)
      if (!ok) break;
      if (pt == 0) {
        tc::mbar_arrive_expect_tx(&s.q_full, DB_CHUNKS * DB_H * 128);
        const int qrow = it.qi * a.H + it.hg * DB_H;
        for (int c = 0; c < DB_CHUNKS; ++c) tc::tma_load_2d(s.q[c], &map_q, &s.q_full, 64 * c, qrow);
      }
      for (int j = 0; j < it.nb; ++j, ++G) {
        const int b = G & 1;
        // Window slots of this block whose rows are contiguous (no ring wrap) and start on a
        // 32-slot boundary come in by 2D TMA boxes of 32 rows; the rest by cp.async.
        const int bs = j * DB_BLK;
        int ls = it.nc4 - bs;
        if (ls < 0) ls = 0;
        bool tma_win = false;
        long long first_row = 0;
        if (ls < DB_BLK && (ls & 31) == 0) {
          const long long jl0 = bs + ls - it.nc4;
          if (jl0 < it.cs.n_local) {
            const long long p0 = it.cs.win0 + jl0;
            const long long last = it.cs.win0 + it.cs.n_local - 1;
            tma_win = (p0 % a.R) + (last - p0) < a.R;
            first_row = it.cs.local_base + p0 % a.R;
          }
        }
        const int cp_end = tma_win ? ls : DB_BLK;
        for (int u = pt; u < cp_end; u += DB_PROD) {
          const DbSlot r = db_slot(a, it.cs, it.nc4, bs + u);
          if (r.bad_index) flag_status(DSV4_ERR_DEVICE_BOUNDS);
          s.rowaddr[u] = r.addr;
        }
        tc::named_barrier(5, DB_PROD);
        if (pt == 0) DB_TRACE(0, k, j);
        // Producer warp pw fills chunks 2pw and 2pw+1 (the pair GEMM2 tile pw releases): per
        // chunk 16 copies of 16 bytes per lane, a warp instruction covering 4 rows x 128 bytes,
        // then one completion arrival per lane (these arrivals are costly to issue, so each
        // thread makes two per block rather than one per chunk).
        const int c0 = 2 * pw;
        uint64_t src[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int row = (lane >> 3) + 4 * i;
          src[i] = row < cp_end ? s.rowaddr[row] + (uint64_t)(16 * (lane & 7)) : 0;
        }
        // chunks c0, c0+1 of buffer b are free once GEMM2 tile pw of block G-2 completed: the
        // watcher saw it (so their full-barrier phases of block G-2 are complete too)
        if (G >= 2) db_sync(DB_GATE_PAIR0 + 4 * b + pw);
        if (lane == 0) DB_TRACE(16 + pw, k, j);
        if (tma_win && lane == 0) {
          tc::mbar_expect_tx(&s.ch_full[b][c0], (DB_BLK - ls) * 128);
          tc::mbar_expect_tx(&s.ch_full[b][c0 + 1], (DB_BLK - ls) * 128);
        }
        const uint32_t kv0 = tc::smem_u32(s.kv[b][0]);
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
          const int c = c0 + cc;
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const int row = (lane >> 3) + 4 * i;
            if (row < cp_end)
              db_cp16(kv0 + (uint32_t)(c * DB_BLK * 128 + row * 128 + (((lane & 7) ^ (row & 7)) << 4)),
                      src[i] + (uint64_t)(128 * c));
          }
          if (tma_win && lane == 0) {
            for (int r0 = ls; r0 < DB_BLK; r0 += 32)
              tc::tma_load_2d(s.kv[b][c] + r0 * 128, &map_local, &s.ch_full[b][c], 64 * c,
                              (int32_t)(first_row + (r0 - ls)));
          }
          db_cp_arrive(&s.ch_full[b][c]);
        }
        if (lane == 0) DB_TRACE(20 + pw, k, j);
        if (pt == 0) DB_TRACE(2, k, j);
        tc::named_barrier(5, DB_PROD);                 // rowaddr[] is rewritten next block
      }
      ++k;
    }
    asm volatile("cp.async.wait_all;" ::: "memory");
    if (pt == 0 && *abort) {
      // the consumers gave up: let this thread's own bulk copies land before exiting
      volatile int never = 0;
      if (k > 0) tc::mbar_wait(&s.q_full, (uint32_t)((k - 1) & 1), spin, &never);
      for (uint32_t g = G >= 2 ? G - 2 : 0; g < G; ++g)
        for (int c = 0; c < DB_CHUNKS; ++c)
          tc::mbar_wait(&s.ch_full[g & 1][c], (g >> 1) & 1, spin, &never);
    }
  } else if (warp == 12) {
    // ------------------------------------------------------------------ watcher
    // Waits for the Q buffer and the KV chunk-pair releases on the producers' behalf. Item
    // gate: blocking OR-reduction (one abort decision for both sides). Pair gates: one named
    // barrier per (buffer, chunk pair); the watcher only arrives (it is already waiting for
    // the next release while the producers copy) and the producers sync. The release of pair
    // q of buffer b for block G needs GEMM2 of block G-2, hence GEMM1 of block G-2, hence all
    // of its copies, hence the producers past the previous gate of the same barrier: at most
    // one arrival is ever outstanding per barrier. After a failed wait the watcher syncs (lock
    // step) until the next item gate ends both loops.
    auto wwait = [&](uint64_t* bar, uint32_t parity) {
      return __all_sync(0xffffffffu, db_wait(bar, parity, spin, abort)) != 0;
    };
    uint32_t G = 0;
    int k = 0;
    bool ok = true;
    for (int item = blockIdx.x; item < items && ok; item += gridDim.x) {
      const DbItem it = db_item(a, item, head_groups);
      if (k > 0) ok = wwait(&s.q_empty, (uint32_t)((k - 1) & 1));
      ok = !db_gate(DB_GATE_ITEM, !ok || *abort != 0);
      ++k;
      for (int j = 0; j < it.nb && ok; ++j, ++G) {
        if (G < 2) continue;
        const int b = G & 1;
        for (int q = 0; q < 4; ++q) {
          if (wwait(&s.kv_empty[b][q], ((G >> 1) - 1) & 1)) {
            if (lane == 0) DB_TRACE(q == 0 ? 9 : 24 + q, k - 1, j);
            db_arrive(DB_GATE_PAIR0 + 4 * b + q);
          } else {
            db_sync(DB_GATE_PAIR0 + 4 * b + q);
          }
        }
      }
    }
  } else if (warp == 13) {
    // ------------------------------------------------------------------ MMA issuer (converged)
    // Per block G: the four K chunks of GEMM1(G) as they land and, as soon as the softmax has
    // published P of block G-1, GEMM2(G-1) in between (the warp polls both without blocking).
    // GEMM2 of an item's last block follows its GEMM1 directly. s_full of block G is
    // committed after GEMM2(G-2) was issued, so it also certifies that GEMM2 (KV buffer,
    // P buffer and O^T contribution of block G-2).
    {
      const uint32_t id1 = tc::idesc_bf16_f32(DB_BLK, DB_H, 0, 0);   // A, B K-major
      const uint32_t id2 = tc::idesc_bf16_f32(128, DB_H, 1, 1);      // A, B MN-major
      const uint64_t d_q1 = tc::sdesc_sw128(tc::smem_u32(s.q[0]), 16, 1024);
      uint32_t G = 0;
      int k = 0;
      bool ok = true;
      auto wwait = [&](uint64_t* bar, uint32_t parity) {
        return __all_sync(0xffffffffu, db_wait(bar, parity, spin, abort)) != 0;
      };
      auto ready = [&](uint64_t* bar, uint32_t parity) {
        return __all_sync(0xffffffffu, db_test(bar, parity)) != 0;
      };
      // GEMM2 of block g (P published): O^T (+)= KV^T . P^T, four 128-channel M tiles x four
      // 16-slot K steps; tile q releases KV chunks 2q, 2q+1 of the buffer
      auto issue_gemm2 = [&](uint32_t g, int jj, bool accumulate) {
        const int b = g & 1;
        if (lane == 0) DB_TRACE(5, k - 1, jj);
        tc::tc_fence_after();
        const uint64_t d_kv2 = tc::sdesc_sw128(tc::smem_u32(s.kv[b][0]), DB_BLK * 128, 1024);
        const uint64_t d_p2 = tc::sdesc_sw128(tc::smem_u32(s.p[b]), DB_BLK * 128, 1024);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
#pragma unroll
          for (int ks = 0; ks < DB_BLK / 16; ++ks)
            tc::mma_bf16_ss_warp(tmem + DB_TM_O + 64 * q,
                                 d_kv2 + (uint64_t)(2 * q * (DB_BLK * 128 / 16) + ks * 128),
                                 d_p2 + (uint64_t)(ks * 128), id2,
                                 (ks > 0 || accumulate) ? 1u : 0u);
          tc::mma_commit_warp(&s.kv_empty[b][q]);
        }
        tc::mma_commit_warp(&s.o_done);
      };
      const unsigned long long poll_limit = 16ull * spin;
      for (int item = blockIdx.x; item < items && ok; item += gridDim.x) {
        const DbItem it = db_item(a, item, head_groups);
        ok = wwait(&s.q_full, (uint32_t)(k & 1));
        ++k;
        for (int j = 0; j < it.nb && ok; ++j, ++G) {
          const int b = G & 1;
          if (G >= 2) {
            ok = wwait(&s.s_empty[b], ((G >> 1) - 1) & 1);
            if (!ok) break;
          }
          const uint64_t d_kv1 = tc::sdesc_sw128(tc::smem_u32(s.kv[b][0]), 16, 1024);
          bool pend2 = j > 0;                          // GEMM2 of block G-1 not issued yet
          int c = 0;
          unsigned long long polls = 0;
          while (c < DB_CHUNKS || pend2) {
            if (pend2 && ready(&s.p_full[(G - 1) & 1], ((G - 1) >> 1) & 1)) {
              issue_gemm2(G - 1, j - 1, j > 1);
              pend2 = false;
              continue;
            }
            if (c < DB_CHUNKS && ready(&s.ch_full[b][c], (G >> 1) & 1)) {
              if (lane == 0 && c == 0) DB_TRACE(3, k - 1, j);
              if (lane == 0 && c == 7) DB_TRACE(4, k - 1, j);
              tc::fence_proxy_async_smem();            // cp.async (generic) -> tensor core
              tc::tc_fence_after();
#pragma unroll
              for (int kk = 0; kk < 4; ++kk)
                tc::mma_bf16_ss_warp(tmem + DB_TM_S + 64 * b,
                                     d_kv1 + (uint64_t)(c * (DB_BLK * 128 / 16) + 2 * kk),
                                     d_q1 + (uint64_t)(c * (DB_H * 128 / 16) + 2 * kk), id1,
                                     (c | kk) != 0);
              if (++c == DB_CHUNKS) {
                tc::mma_commit_warp(&s.s_full[b]);
                if (j + 1 == it.nb) tc::mma_commit_warp(&s.q_empty);
              }
              continue;
            }
            ++polls;
#if DB_WAIT_MODE != 0
            __nanosleep(32);
#endif
            bool give_up = polls > poll_limit;
            if ((polls & 63) == 0)
              give_up |= *abort != 0 || *reinterpret_cast<volatile int*>(&g_status) == DSV4_ERR_DEVICE_TIMEOUT;
            if (__any_sync(0xffffffffu, give_up)) {
              if (lane == 0 && polls > poll_limit) flag_status(DSV4_ERR_DEVICE_TIMEOUT);
              *abort = 1;
              ok = false;
              break;
            }
          }
        }
        if (!ok) break;
        // the item's last block
        ok = wwait(&s.p_full[(G - 1) & 1], ((G - 1) >> 1) & 1);
        if (!ok) break;
        issue_gemm2(G - 1, it.nb - 1, it.nb > 1);
        tc::mma_commit_warp(&s.o_final);
      }
      if (!ok) {
        tc::mma_commit_warp(&s.drain);
        volatile int never = 0;
        tc::mbar_wait(&s.drain, 0, spin, &never);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------------ softmax + epilogue
    // Thread (quad, half, lane): slots s0 = 16 quad + lane/4 and s0 + 8 of each block, heads
    // hb + 8 kk + 2 (lane % 4) + {0, 1}, kk = 0..3 (one 16x256b TMEM fragment).
    const int quad = warp & 3, half = warp >> 2;
    const int hb = 32 * half;
    const int tq = lane & 3, tr = lane >> 2;
    const int s0 = 16 * quad + tr;
    const uint32_t lane_base = (uint32_t)(32 * quad) << 16;
    // P^T rows written by this thread's stmatrix address slots (row lane%8 of matrix lane/8):
    // slot 16 quad + lane%8 (+ 8 for the second store), heads hb + 8 (lane/8) .. + 7
    const uint32_t p_off = (uint32_t)((16 * quad + (lane & 7)) * 128 +
                                      (((4 * half + (lane >> 3)) ^ (lane & 7)) << 4));
    uint32_t G = 0;
    int k = 0;
    bool ok = true;
    // the item's description, sink logit and the validity of this thread's two slots in the
    // next block are loaded one step ahead
    int item = blockIdx.x;
    DbItem it = db_item(a, item < items ? item : 0, head_groups);
    float sink_h = (quad == 0 && a.sink) ? __ldg(a.sink + it.hg * DB_H + hb + lane) : 0.f;
    bool v0n = db_slot(a, it.cs, it.nc4, s0).valid;
    bool v1n = db_slot(a, it.cs, it.nc4, s0 + 8).valid;
    for (; item < items && ok; item += gridDim.x) {
      float lsum[8];                                   // sums of the bf16-rounded weights
#pragma unroll
      for (int e = 0; e < 8; ++e) lsum[e] = 0.f;
      for (int j = 0; j < it.nb; ++j, ++G) {
        const int b = G & 1;
        const bool v0 = v0n, v1 = v1n;
        if (j + 1 < it.nb) {
          v0n = db_slot(a, it.cs, it.nc4, (j + 1) * DB_BLK + s0).valid;
          v1n = db_slot(a, it.cs, it.nc4, (j + 1) * DB_BLK + s0 + 8).valid;
        }
        if (tid == 0) DB_TRACE(6, k, j);
        ok = db_wait(&s.s_full[b], (G >> 1) & 1, spin, abort);
        ok = !db_red_or(3, DB_SOFT, !ok);              // all 256 threads take the same branch
        if (!ok) break;
        if (tid == 0) DB_TRACE(7, k, j);
        tc::tc_fence_after();
        float z[16];
        tc::tmem_ld16x256b_x4(tmem + lane_base + DB_TM_S + 64 * b + hb, z);
        tc::tmem_wait_ld_dep16(z);
        tc::tc_fence_before();
        tc::mbar_arrive(&s.s_empty[b]);                // S^T buffer b may be overwritten
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          z[4 * kk] = v0 ? z[4 * kk] * scale_log2 : -INFINITY;
          z[4 * kk + 1] = v0 ? z[4 * kk + 1] * scale_log2 : -INFINITY;
          z[4 * kk + 2] = v1 ? z[4 * kk + 2] * scale_log2 : -INFINITY;
          z[4 * kk + 3] = v1 ? z[4 * kk + 3] * scale_log2 : -INFINITY;
        }
        // s_full of this block certifies GEMM2 of block G-2, the last reader of P buffer b
        const uint32_t paddr = tc::smem_u32(s.p[b]) + p_off;
        bool rescale = false;
        // After an item's first block the weights are taken against the running max m (they
        // are exact whatever m is, m cancels in the normalisation); block maxima are needed
        // only when a score exceeds its running max by more than TAU.
        bool exact = j == 0;
        if (!exact) {
          uint32_t pk[8];
          bool over = false;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const int h = hb + 8 * kk + 2 * tq;
            const float2 m2 = *reinterpret_cast<const float2*>(&s.mcur[h]);
            const float2 o2 = *reinterpret_cast<const float2*>(&s.moff[h]);
            over |= !(z[4 * kk] <= m2.x + DB_TAU) | !(z[4 * kk + 1] <= m2.y + DB_TAU) |
                    !(z[4 * kk + 2] <= m2.x + DB_TAU) | !(z[4 * kk + 3] <= m2.y + DB_TAU);
            pk[kk] = db_pack(exp2f(z[4 * kk] - o2.x), exp2f(z[4 * kk + 1] - o2.y));
            pk[4 + kk] = db_pack(exp2f(z[4 * kk + 2] - o2.x), exp2f(z[4 * kk + 3] - o2.y));
          }
          exact = db_red_or(2, DB_SOFT, over);
          if (!exact) {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              // the denominator sums the same bf16-rounded weights the PV product uses
              const float2 r0 = db_unpack(pk[kk]), r1 = db_unpack(pk[4 + kk]);
              lsum[2 * kk] += r0.x + r1.x;
              lsum[2 * kk + 1] += r0.y + r1.y;
            }
            db_stmatrix_x4(paddr, pk[0], pk[1], pk[2], pk[3]);
            db_stmatrix_x4(paddr + 8 * 128, pk[4], pk[5], pk[6], pk[7]);
          }
        }
        if (exact) {
          // per-head maxima over the warp's 16 slots (lanes of equal lane%4 share heads),
          // then over the four quadrant warps through shared memory
          float bm[8];
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            bm[2 * kk] = fmaxf(z[4 * kk], z[4 * kk + 2]);
            bm[2 * kk + 1] = fmaxf(z[4 * kk + 1], z[4 * kk + 3]);
          }
#pragma unroll
          for (int off = 4; off < 32; off <<= 1)
#pragma unroll
            for (int e = 0; e < 8; ++e) bm[e] = fmaxf(bm[e], __shfl_xor_sync(0xffffffffu, bm[e], off));
          if (tr == 0)
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              *reinterpret_cast<float2*>(&s.red[quad][hb + 8 * kk + 2 * tq]) =
                  make_float2(bm[2 * kk], bm[2 * kk + 1]);
          tc::named_barrier(1, DB_SOFT);
          bool grow = false;
          if (quad == 0) {                             // warps 0 and 4 own heads hb + lane
            const int h = hb + lane;
            const float m = fmaxf(fmaxf(s.red[0][h], s.red[1][h]), fmaxf(s.red[2][h], s.red[3][h]));
            const float mo = s.mcur[h];
            float mn = mo, f = 1.f;
            if (mo == -INFINITY) {
              mn = m;
              f = 0.f;
            } else if (m > mo + DB_TAU) {
              mn = m;
              f = exp2f(mo - mn);
              grow = true;
            }
            s.mcur[h] = mn;
            s.moff[h] = mn == -INFINITY ? 0.f : mn;
            s.fac[h] = f;
          }
          rescale = db_red_or(2, DB_SOFT, grow) && j > 0;
          uint32_t pk[8];
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const int h = hb + 8 * kk + 2 * tq;
            const float2 o2 = *reinterpret_cast<const float2*>(&s.moff[h]);
            const float2 f2 = *reinterpret_cast<const float2*>(&s.fac[h]);
            pk[kk] = db_pack(exp2f(z[4 * kk] - o2.x), exp2f(z[4 * kk + 1] - o2.y));
            pk[4 + kk] = db_pack(exp2f(z[4 * kk + 2] - o2.x), exp2f(z[4 * kk + 3] - o2.y));
            const float2 r0 = db_unpack(pk[kk]), r1 = db_unpack(pk[4 + kk]);
            lsum[2 * kk] = fmaf(lsum[2 * kk], f2.x, r0.x + r1.x);
            lsum[2 * kk + 1] = fmaf(lsum[2 * kk + 1], f2.y, r0.y + r1.y);
          }
          db_stmatrix_x4(paddr, pk[0], pk[1], pk[2], pk[3]);
          db_stmatrix_x4(paddr + 8 * 128, pk[4], pk[5], pk[6], pk[7]);
        }
        if (rescale) {                                 // rare: a head's max grew by > 2^TAU
          // O^T holds blocks up to G-1 once GEMM2 of block G-1 completed
          ok = db_wait(&s.o_done, (G - 1) & 1, spin, abort);
          ok = !db_red_or(3, DB_SOFT, !ok);
          if (!ok) break;
          tc::tc_fence_after();
#pragma unroll 1
          for (int q = 0; q < 4; ++q) {
            asm volatile("" ::: "memory");             // re-read the factors each tile
            float o[32];
            const uint32_t addr = tmem + lane_base + DB_TM_O + 64 * q + hb;
            tc::tmem_ld32(addr, o);
            tc::tmem_wait_ld_dep(o);
#pragma unroll
            for (int u = 0; u < 32; u += 4) {
              const float4 fa = *reinterpret_cast<const float4*>(&s.fac[hb + u]);
              o[u] *= fa.x;
              o[u + 1] *= fa.y;
              o[u + 2] *= fa.z;
              o[u + 3] *= fa.w;
            }
            tc::tmem_st32(addr, o);
          }
          tc::tmem_wait_st();
        }
        tc::fence_proxy_async_smem();
        tc::tc_fence_before();
        tc::mbar_arrive(&s.p_full[b]);
        if (tid == 0) DB_TRACE(8, k, j);
      }
      if (!ok) break;
      // ---------------------------------------------------------------- epilogue
      const int nitem = item + gridDim.x;
      DbItem nx = it;
      float nsink = 0.f;
      if (nitem < items) {
        nx = db_item(a, nitem, head_groups);
        nsink = (quad == 0 && a.sink) ? __ldg(a.sink + nx.hg * DB_H + hb + lane) : 0.f;
        v0n = db_slot(a, nx.cs, nx.nc4, s0).valid;
        v1n = db_slot(a, nx.cs, nx.nc4, s0 + 8).valid;
      }
      // GEMM2 of the item's last block is complete (one o_final phase per item)
      ok = db_wait(&s.o_final, (uint32_t)(k & 1), spin, abort);
      ok = !db_red_or(3, DB_SOFT, !ok);
      if (!ok) break;
      if (tid == 0) DB_TRACE(10, k, 0);
      tc::tc_fence_after();
#pragma unroll
      for (int off = 4; off < 32; off <<= 1)
#pragma unroll
        for (int e = 0; e < 8; ++e) lsum[e] += __shfl_xor_sync(0xffffffffu, lsum[e], off);
      if (tr == 0)
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          *reinterpret_cast<float2*>(&s.red[quad][hb + 8 * kk + 2 * tq]) =
              make_float2(lsum[2 * kk], lsum[2 * kk + 1]);
      tc::named_barrier(1, DB_SOFT);
      const int h0 = it.hg * DB_H;
      if (quad == 0) {
        const int h = hb + lane;
        const float L = (s.red[0][h] + s.red[1][h]) + (s.red[2][h] + s.red[3][h]);
        const float m = s.mcur[h];
        const float s2 = a.sink ? sink_h * DB_LOG2E : -INFINITY;
        const float mf = fmaxf(m, s2);
        const float em = m == -INFINITY ? 0.f : exp2f(m - mf);
        const float den = L * em + (a.sink ? exp2f(s2 - mf) : 0.f);
        float inv = 0.f, lse = -INFINITY;
        if (den > 0.f && mf != -INFINITY) {
          inv = em / den;
          lse = (mf + log2f(den)) * DB_LN2;
        }
        s.inv[h] = inv;
        if (a.lse) a.lse[(long long)it.qi * a.H + h0 + h] = lse;
        s.mcur[h] = -INFINITY;                         // the next item starts fresh
      }
      tc::named_barrier(1, DB_SOFT);
      // O^T tiles of 128 channels: each warp reads its 32 channels x 32 heads as two 16-lane
      // fragments (thread t: channels c0 + t/4 and c0 + 8 + t/4, head pairs 2(t%4) + 8kk),
      // scales and packs them to bf16 and writes them with transposing 8x8 matrix stores, so
      // each stored 16-byte row is 8 consecutive channels of one head. The rows land in the
      // two P buffers (free now) as two [64 heads x 64 channels] 128-byte swizzle boxes, which
      // TMA stores to O.
      const int mrow = lane & 7, mat = lane >> 3;
      float2 inv2[4];
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        inv2[kk] = *reinterpret_cast<const float2*>(&s.inv[hb + 8 * kk + 2 * tq]);
      const uint32_t p0 = tc::smem_u32(s.p[0]) + (uint32_t)((quad >> 1) * (DB_H * 128));
      for (int q = 0; q < 4; ++q) {
        uint32_t pk[2][8];                             // [channel half][matrix slot]
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          float v[16];
          tc::tmem_ld16x256b_x4(tmem + ((uint32_t)(32 * quad + 16 * hh) << 16) + DB_TM_O + 64 * q + hb, v);
          tc::tmem_wait_ld_dep16(v);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            pk[hh][2 * kk] = db_pack(v[4 * kk] * inv2[kk].x, v[4 * kk + 1] * inv2[kk].y);
            pk[hh][2 * kk + 1] = db_pack(v[4 * kk + 2] * inv2[kk].x, v[4 * kk + 3] * inv2[kk].y);
          }
        }
        if (q > 0) {                                   // the previous tile's stores read P
          if (tid == 0) tc::bulk_wait_read();
          tc::named_barrier(1, DB_SOFT);
        }
#pragma unroll
        for (int hh = 0; hh < 2; ++hh)
#pragma unroll
          for (int jx = 0; jx < 2; ++jx) {
            // matrices {A_k, B_k, A_k+1, B_k+1}, k = 2 jx: A = channels c0..c0+7, B = c0+8..
            const int kk = 2 * jx + (mat >> 1);
            const int h = hb + 8 * kk + mrow;          // stored row: one head
            const int unit = 4 * (quad & 1) + 2 * hh + (mat & 1);
            const uint32_t addr = p0 + (uint32_t)(h * 128 + ((unit ^ mrow) << 4));
            tc::stmatrix_x4_trans(addr, pk[hh][4 * jx], pk[hh][4 * jx + 1], pk[hh][4 * jx + 2],
                                  pk[hh][4 * jx + 3]);
          }
        tc::fence_proxy_async_smem();
        tc::named_barrier(1, DB_SOFT);
        if (tid == 0) {
          const int orow = it.qi * a.H + h0;
          tc::tma_store_2d(&map_o, s.p[0], 128 * q, orow);
          tc::tma_store_2d(&map_o, s.p[1], 128 * q + 64, orow);
          tc::bulk_commit();
        }
      }
      // the next item's softmax writes P only after a barrier this thread reaches after here
      if (tid == 0) tc::bulk_wait_read();
      if (tid == 0) DB_TRACE(11, k, 0);
      tc::tc_fence_before();
      ++k;
      it = nx;
      sink_h = nsink;
    }
    if (tid == 0) tc::bulk_wait_all();                 // output stores complete before exit
  }
  tc::tc_fence_before();
  __syncthreads();
  if (warp == 13) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, DB_TM_COLS);
  }
}

}  // namespace

// Double-buffered tensor-core attention for unsplit candidate lists (c = 512, 64-head
// groups). Returns DSV4_OK with *used = false when the shapes or alignments do not fit.
int launch_attn_db(const AttnArgs& a, cudaStream_t st, bool* used) {
  *used = false;
  if (a.c != DB_C || a.H % DB_H != 0) return DSV4_OK;
  if (!aligned16(a.Q) || !aligned16(a.local) || !aligned16(a.O) || (a.pool && !aligned16(a.pool)))
    return DSV4_OK;
  const long long nrows_q = (long long)a.B * a.nq * a.H;
  const long long items = (long long)a.B * a.nq * (a.H / DB_H);
  const long long nrows_local = (long long)a.B * a.R;
  if (nrows_q >= (1ll << 31) || items >= (1ll << 31) || nrows_local >= (1ll << 31)) return DSV4_OK;
  static int sms = 0;
  if (sms == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (sms <= 0) sms = 148;
    const cudaError_t e = cudaFuncSetAttribute(attn_db_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               (int)DB_SMEM);
    if (e != cudaSuccess) return fail(DSV4_ERR_CUDA, "attn_db: %s", cudaGetErrorString(e));
  }
  CUtensorMap mq, mlocal, mo;
  int s = encode_tensor_map_2d(&mq, a.Q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, DB_C, nrows_q, 64,
                               DB_H, CU_TENSOR_MAP_SWIZZLE_128B);
  if (s != DSV4_OK) return s;
  s = encode_tensor_map_2d(&mo, a.O, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, DB_C, nrows_q, 64, DB_H,
                           CU_TENSOR_MAP_SWIZZLE_128B);
  if (s != DSV4_OK) return s;
  s = encode_tensor_map_2d(&mlocal, a.local, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, DB_C, nrows_local,
                           64, 32, CU_TENSOR_MAP_SWIZZLE_128B);
  if (s != DSV4_OK) return s;
  const long long grid = items < sms ? items : sms;
  attn_db_kernel<<<(unsigned)grid, DB_THREADS, DB_SMEM, st>>>(a, mq, mlocal, mo, a.H / DB_H, (int)items,
                                                              a.scale * DB_LOG2E, spin_limit());
  *used = true;
  return launch_status("hybrid attention (tensor cores, double-buffered)");
}

}  // namespace dsv4

#ifdef DSV4_TRACE
extern "C" int dsv4_trace_read_db(unsigned long long* host, size_t n) {
  return cudaMemcpyFromSymbol(host, dsv4::g_db_trace, n * sizeof(unsigned long long)) == cudaSuccess ? 0 : 3;
}
#endif
