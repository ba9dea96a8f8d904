// Hybrid shared-KV MQA on the 5th-generation tensor cores (tcgen05 + TMEM), one CTA per SM,
// persistent, cp.async row gathers.
//
// "CSA And HCA: Definition, State, And Cost Model": s3.2/s4 every candidate row is both key
// and value for all heads; s5.1 one candidate list (selected or all completed compressed
// entries, then the local window) under one softmax per head; s5.3 the sink logit joins
// the denominator only. Per-query valid counts follow pypto-lib PR #834.
//
// Because all heads share each KV row, the contraction for one query is dense with the
// candidates as one MMA dimension. The transposed form puts 128 candidate slots on the MMA
// M dimension (full tensor-core rate) and the 64 heads on N:
//   GEMM1  S^T[128 slots x 64 heads] = KV[slots x c] . Q[heads x c]^T      (K = c = 512)
//   GEMM2  O^T[c x 64 heads]        += KV^T[c x slots] . P^T[slots x heads] (K = 128)
// The same shared-memory KV tile (eight 64-channel chunks in 128-byte swizzle atoms) is the
// K-major A operand of GEMM1 and the MN-major A operand of GEMM2. O^T stays in TMEM for the
// whole item (4 M-tiles x 64 columns); S^T takes 64 more columns.
//
// Work item = (query, group of 64 heads); CTAs loop over items. Warps:
//   0-7   softmax/epilogue: warp w reads TMEM lane quadrant w%4 (slot / channel row) for
//         heads 32(w/4)..+31; per-head block maxima by a transposing butterfly plus a
//         4-quadrant exchange; O^T is rescaled only when a head's max grows by > 2^8;
//         P^T is written as bf16; the epilogue stages O through shared memory for 16-byte
//         stores.
//   8-11  producer (one per sub-partition; each warp instruction moves one 128-byte chunk
//         of 4 rows): resolves the block's 128 row addresses, then gathers them with 16-byte
//         cp.async, chunk by chunk as GEMM2 of the previous block releases each chunk pair;
//         completion is signalled per half block (chunks 0-3, 4-7).
//   12    watcher: waits for GEMM2's chunk releases and the Q buffer on the producers'
//         behalf and passes them on through named-barrier gates (a producer's own mbarrier
//         wait would queue behind its cp.async traffic and stall the gather).
//   13    MMA issuer and TMEM owner; the warp stays converged and elect.sync issues.
// Candidate slots: [0, round4(n_comp)) compressed, then the local window; slots past a
// part's count are masked (p = 0) and fetch an in-range row, so every value is finite.
// All waits are bounded (see tc_common.cuh).
#include <cstdio>
#include <cstdlib>

#include "attn_common.cuh"
#include "tc_common.cuh"

namespace dsv4 {
namespace {

constexpr int AT_C = 512;
constexpr int AT_H = 64;
constexpr int AT_BLK = 128;
constexpr int AT_CHUNKS = AT_C / 64;
constexpr int AT_SOFT = 256;
constexpr int AT_PROD_WARPS = 4;                   // 6 were measured slower
constexpr int AT_PROD = 32 * AT_PROD_WARPS;
constexpr int AT_WATCH_WARP = 8 + AT_PROD_WARPS;   // warps 0-7 softmax, then the producers
constexpr int AT_MMA_WARP = AT_WATCH_WARP + 1;
constexpr int AT_THREADS = AT_SOFT + AT_PROD + 64;
// Named barriers: 1-3 softmax warps, 5 producers, and the producer/watcher gates.
constexpr uint32_t GATE_ITEM = 10;
constexpr uint32_t GATE_PAIR0 = 6;          // 6..9: chunk pairs 0..3
constexpr uint32_t TM_S = 0;
constexpr uint32_t TM_O = 64;
constexpr uint32_t TM_COLS = 512;
constexpr int AT_ORDER_MAX = 256;            // split lists ranked longest first up to this many
constexpr float TAU = 8.f;                  // log2-domain growth tolerated before rescaling
constexpr float LOG2E = 1.4426950408889634f;
constexpr float LN2 = 0.6931471805599453f;

struct AttnSmem {
  uint8_t q[AT_CHUNKS][AT_H * 128];         // K-major SW128: [64 heads][64 ch] per chunk
  uint8_t kv[AT_CHUNKS][AT_BLK * 128];      // [128 slots][64 ch] per chunk
  uint8_t p[AT_BLK * 128];                  // MN-major SW128 P^T [128 slots][64 heads];
                                            // also the O staging tile of the epilogue
  float red[4][AT_H];
  float mcur[AT_H];
  float moff[AT_H];                         // exp2 offset: mcur, or 0 while mcur = -inf
  float fac[AT_H];
  float inv[AT_H];
  float rcos[32], rsin[32];                 // inverse RoPE of O: the item's pair angles
  uint64_t rowaddr[AT_BLK];
  uint64_t q_full, q_empty;
  uint64_t ch_full[AT_CHUNKS], ch_empty[4];  // ch_full[3], ch_full[7]: chunks 0-3, 4-7 landed
  uint64_t s_full, p_full, o_done, drain;
  uint32_t tmem_base;
  int abort;
  int first;                                // split lists: this CTA's work item
  int order_nb[AT_ORDER_MAX];               // split lists: blocks per (query, head group)
};
constexpr size_t AT_SMEM = sizeof(AttnSmem) + 1024;
static_assert(AT_SMEM <= 232448, "shared memory of the attention kernel");

#ifdef DSV4_TRACE
__device__ unsigned long long g_attn1_trace[4][8][32];
#define A1_TRACE(ev, k_, j_)                                 \
  do {                                                       \
    if (blockIdx.x == 0 && (k_) >= 40 && (k_) < 44 && (j_) < 8) \
      g_attn1_trace[(k_) - 40][j_][ev] = clock64();          \
  } while (0)
#else
#define A1_TRACE(ev, k_, j_) \
  do {                       \
  } while (0)
#endif

__device__ __forceinline__ bool bar_red_or(uint32_t id, uint32_t threads, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n .reg .pred p, q;\n setp.ne.u32 p, %1, 0;\n"
      " barrier.red.or.pred q, %2, %3, p;\n selp.u32 %0, 1, 0, q;\n}"
      : "=r"(r)
      : "r"((uint32_t)pred), "r"(id), "r"(threads)
      : "memory");
  return r != 0;
}
// Producer/watcher rendezvous (all producer warps and the watcher warp). gate() blocks both
// sides and returns the OR of their predicates; pair_arrive / pair_sync are the watcher's
// non-blocking and the producers' blocking halves of a one-way release.
__device__ __forceinline__ bool gate(uint32_t id, bool pred) {
  return bar_red_or(id, AT_PROD + 32, pred);
}
__device__ __forceinline__ void pair_arrive(uint32_t id) {
  asm volatile("bar.arrive %0, %1;" ::"r"(id), "r"(AT_PROD + 32) : "memory");
}
__device__ __forceinline__ void pair_sync(uint32_t id) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(AT_PROD + 32) : "memory");
}
__device__ __forceinline__ void cp_async16(uint32_t dst, uint64_t src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void bulk_prefetch_l2(uint64_t src, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}
__device__ __forceinline__ void cp_async_arrive_noinc(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(tc::smem_u32(bar))
               : "memory");
}

// Transposing butterfly over 32 per-lane values: lane L ends with the reduction of value L.
template <bool MAX>
__device__ __forceinline__ float xpose_reduce32(float (&v)[32]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int step = 0; step < 5; ++step) {
    const int half = 16 >> step;
    const int mask = 16 >> step;
    const bool up = (lane & mask) != 0;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      if (i < half) {
        const float send = up ? v[i] : v[i + half];
        const float keep = up ? v[i + half] : v[i];
        const float recv = __shfl_xor_sync(0xffffffffu, send, mask);
        v[i] = MAX ? fmaxf(keep, recv) : keep + recv;
      }
    }
  }
  return v[0];
}

// 2^x by the PTX approximate base-2 exponential, results below 2^-126 flushed to zero (the
// weights are rounded to bf16 next; one that small is zero beside the block's largest)
__device__ __forceinline__ float ex2_ftz(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
// a0 += lo(v), a1 += hi(v) for a bf16 pair v, each widened exactly (sm_100 mixed-precision add)
__device__ __forceinline__ void add_bf16x2_f32(float& a0, float& a1, uint32_t v) {
  asm("{\n .reg .b16 l, h;\n mov.b32 {l, h}, %2;\n"
      " add.rn.f32.bf16 %0, l, %0;\n add.rn.f32.bf16 %1, h, %1;\n}"
      : "+f"(a0), "+f"(a1)
      : "r"(v));
}
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&p);
}

// Slot g of the query's candidate list: part (0 pool, 1 local), global row, validity.
struct SlotRow {
  int part;
  long long row;
  bool valid;
  bool bad_index;
};

__device__ __forceinline__ SlotRow slot_row(const AttnArgs& a, const CandidateSet& cs, int nc4,
                                            int g) {
  SlotRow r;
  r.bad_index = false;
  if (g < nc4) {
    r.part = 0;
    r.valid = g < cs.n_comp;
    r.row = -1;
    if (r.valid) {
      const long long s = cs.sel ? (long long)__ldg(cs.sel + g) : (long long)g;
      const long long row = cs.pool_base + s;
      if (s < 0 || s >= cs.Et || row < 0 || row >= a.pool_rows) {
        r.valid = false;
        r.bad_index = true;
      } else {
        r.row = row;
      }
    }
  } else {
    r.part = 1;
    const int jl = g - nc4;
    r.valid = jl < cs.n_local;
    r.row = r.valid ? cs.local_base + (cs.win0 + jl) % a.R : cs.local_base;
  }
  return r;
}

// Work item = (query, group of 64 heads, split). With nsplit > 1 the candidate blocks of a
// query are divided evenly among its splits (a split may own none) and each split leaves
// an unnormalised partial for the combine kernel.
struct ItemInfo {
  int qi, hg, nc4, nb, jb, je, base;
  CandidateSet cs;
};

template <bool kSplit>
__device__ __forceinline__ ItemInfo item_info(const AttnArgs& a, int item, int head_groups) {
  ItemInfo it;
  const int split = kSplit ? item % a.nsplit : 0;
  it.base = kSplit ? item / a.nsplit : item;
  it.qi = it.base / head_groups;
  it.hg = it.base % head_groups;
  const int b = it.qi / a.nq, i = it.qi % a.nq;
  it.cs = make_candidates(a, b, i);
  it.nc4 = (it.cs.n_comp + 3) & ~3;
  const int nl4 = (it.cs.n_local + 3) & ~3;
  it.nb = (it.nc4 + nl4 + AT_BLK - 1) / AT_BLK;
  it.jb = kSplit ? (int)((long long)split * it.nb / a.nsplit) : 0;
  it.je = kSplit ? (int)((long long)(split + 1) * it.nb / a.nsplit) : it.nb;
  return it;
}

template <bool kSplit>
__global__ void __maxnreg__(128)
    attn_tc_kernel(const AttnArgs a, const __grid_constant__ CUtensorMap map_q, int head_groups,
                   int items, float scale_log2, uint32_t spin) {
  extern __shared__ uint8_t smem_raw[];
  AttnSmem& s = *reinterpret_cast<AttnSmem*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  volatile int* abort = &s.abort;

  if (tid == 0) {
    tc::mbar_init(&s.q_full, 1);
    tc::mbar_init(&s.q_empty, 1);
    for (int k = 0; k < AT_CHUNKS; ++k) tc::mbar_init(&s.ch_full[k], AT_PROD);
    for (int k = 0; k < 4; ++k) tc::mbar_init(&s.ch_empty[k], 1);
    tc::mbar_init(&s.s_full, 1);
    tc::mbar_init(&s.p_full, AT_SOFT);
    tc::mbar_init(&s.o_done, 1);
    tc::mbar_init(&s.drain, 1);
    s.abort = 0;
    tc::fence_barrier_init();
  }
  if (tid < AT_H) s.mcur[tid] = -INFINITY;
  if (warp == AT_MMA_WARP) {
    tc::tmem_alloc(&s.tmem_base, TM_COLS);
    tc::tmem_relinquish();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = s.tmem_base;
  // Split lists run one CTA per work item and the hardware dispatches CTAs in index order,
  // so CTA r*nsplit + sp takes split sp of the list ranked r by length (longest first, ties
  // by position): long lists start in the first wave and short ones fill the tail, as in
  // longest-processing-time-first scheduling.
  int first = blockIdx.x;
  if constexpr (kSplit) {
    const int nbase = items / a.nsplit;
    if (nbase <= AT_ORDER_MAX) {
      for (int t = tid; t < nbase; t += AT_THREADS) s.order_nb[t] = item_info<false>(a, t, head_groups).nb;
      __syncthreads();
      const int r = blockIdx.x / a.nsplit;
      for (int t = tid; t < nbase; t += AT_THREADS) {
        const int v = s.order_nb[t];
        int rank = 0;
        for (int j = 0; j < nbase; ++j) {
          const int u = s.order_nb[j];
          rank += (u > v || (u == v && j < t)) ? 1 : 0;
        }
        if (rank == r) s.first = t * a.nsplit + blockIdx.x % a.nsplit;
      }
      __syncthreads();
      first = s.first;
    }
  }

  // blocks and items the producers loaded (their bulk copies are drained before exit)
  uint32_t prod_G = 0;
  int prod_k = 0;
  if (warp >= 8 && warp < AT_WATCH_WARP) {
    // ------------------------------------------------------------------ producer (4 warps)
    const int pt = tid - AT_SOFT;
    const uint64_t pool_addr = reinterpret_cast<uint64_t>(a.pool);
    const uint64_t local_addr = reinterpret_cast<uint64_t>(a.local);
    uint32_t& G = prod_G;
    int& k = prod_k;
    bool ok = true;
    if (pt == 0) tc::prefetch_tensormap(&map_q);
    for (int item = first; item < items && ok; item += gridDim.x) {
      const ItemInfo it = item_info<kSplit>(a, item, head_groups);
      if (kSplit && it.je <= it.jb) continue;          // a split without blocks: no work
      ok = !gate(GATE_ITEM, false);                    // the Q buffer is free (or abort)
      if (!ok) break;
      if (pt == 0) {
        tc::mbar_arrive_expect_tx(&s.q_full, AT_CHUNKS * AT_H * 128);
        const int qrow = it.qi * a.H + it.hg * AT_H;
        for (int c = 0; c < AT_CHUNKS; ++c) tc::tma_load_2d(s.q[c], &map_q, &s.q_full, 64 * c, qrow);
      }
      for (int j = it.jb; j < it.je && ok; ++j, ++G) {
        // Every slot of the block comes in by cp.async, local-window rows included (2D TMA
        // boxes of 32 contiguous window rows were measured slower here: the TMA issue of
        // small boxes paced the window block's gather at about half the cp.async rate).
        const int bs = j * AT_BLK;
        // the block's row addresses (one index load per slot)
        for (int u = pt; u < AT_BLK; u += AT_PROD) {
          const SlotRow r = slot_row(a, it.cs, it.nc4, bs + u);
          if (r.bad_index) flag_status(DSV4_ERR_DEVICE_BOUNDS);
          const uint64_t ra = (r.part == 0 && r.valid)
                                  ? pool_addr + (uint64_t)r.row * AT_C * 2
                                  : local_addr + (uint64_t)(r.part == 1 ? r.row : it.cs.local_base) * AT_C * 2;
          s.rowaddr[u] = ra;
          if constexpr (kSplit) {
            // Split lists (decode) read their rows from HBM: the next block's rows start
            // toward L2 now, a block ahead of their gather (which waits for GEMM2 to free the
            // buffer), and an item's first block its own rows.
            if (j == it.jb) bulk_prefetch_l2(ra, AT_C * 2);
            if (j + 1 < it.je) {
              const SlotRow r2 = slot_row(a, it.cs, it.nc4, bs + AT_BLK + u);
              if (r2.valid)
                bulk_prefetch_l2((r2.part == 0 ? pool_addr : local_addr) + (uint64_t)r2.row * AT_C * 2,
                                 AT_C * 2);
            }
          }
        }
        tc::named_barrier(5, AT_PROD);
        if (pt == 0) A1_TRACE(0, k, j);
        // this thread's copies of every chunk: rows/pieces e = pt + 96 i (same for each chunk)
        constexpr int NPER = (AT_BLK * 8 + AT_PROD - 1) / AT_PROD;
        constexpr int ncopy = AT_BLK * 8;
        uint64_t src[NPER];
        uint32_t dsto[NPER];
#pragma unroll
        for (int i = 0; i < NPER; ++i) {
          const int e = pt + AT_PROD * i;
          const int row = (e >> 3) & (AT_BLK - 1), piece = e & 7;
          src[i] = e < ncopy ? s.rowaddr[row] + (uint64_t)(16 * piece) : 0;
          dsto[i] = (uint32_t)(row * 128 + ((piece ^ (row & 7)) << 4));
        }
        const uint32_t kv0 = tc::smem_u32(s.kv[0]);
        for (int c = 0; c < AT_CHUNKS; ++c) {
          if ((c & 1) == 0) {
            // GEMM2 of the previous block released chunks c, c+1 (so their full-barrier
            // phases of that block are complete and the TMA bytes go to this block's phase).
            // The watcher warp saw the release; waiting on the mbarrier here instead would
            // queue behind this thread's own cp.async traffic and starve the gather.
            if (G > 0) pair_sync(GATE_PAIR0 + (c >> 1));
            if (pt == 0) A1_TRACE(8 + (c >> 1), k, j);
          }
#pragma unroll
          for (int i = 0; i < NPER; ++i)
            if (pt + AT_PROD * i < ncopy)
              cp_async16(kv0 + (uint32_t)(c * AT_BLK * 128) + dsto[i], src[i] + (uint64_t)(128 * c));
          // One completion arrival per four chunks: each such arrival stalls the issuing
          // thread for a few hundred cycles (measured), so per-chunk arrivals throttled the
          // gather; GEMM1 then consumes the block in two halves.
          if ((c & 3) == 3) cp_async_arrive_noinc(&s.ch_full[c]);
          if (pt == 0 && (c & 1)) A1_TRACE(28 + (c >> 1), k, j);
        }
        if (pt == 0) A1_TRACE(1, k, j);
        tc::named_barrier(5, AT_PROD);                 // rowaddr[] is rewritten next block
      }
      ++k;
    }
    asm volatile("cp.async.wait_all;" ::: "memory");
  } else if (warp == AT_WATCH_WARP) {
    // ------------------------------------------------------------------ watcher
    // Performs the producers' mbarrier waits and passes each result on; both sides take
    // the same sequence of gates (one per item, four per block after the first).
    //  * item gate: a blocking OR-reduction, so both sides take the same abort decision;
    //  * pair gates: the watcher only arrives (it does not block, so it is already waiting
    //    for the next release while the producers copy) and the producers sync. A release
    //    of pair q of block j needs all of block j's copies, so at most one arrival per
    //    gate is outstanding. After an abort the watcher syncs instead (lock step with the
    //    producers) until the next item gate ends both loops.
    auto wwait = [&](uint64_t* bar, uint32_t parity) {
      return __all_sync(0xffffffffu, tc::mbar_wait(bar, parity, spin, abort));
    };
    uint32_t G = 0;
    int k = 0;
    bool ok = true;
    for (int item = first; item < items && ok; item += gridDim.x) {
      const ItemInfo it = item_info<kSplit>(a, item, head_groups);
      if (kSplit && it.je <= it.jb) continue;
      if (k > 0) ok = wwait(&s.q_empty, (uint32_t)((k - 1) & 1));
      ok = !gate(GATE_ITEM, !ok || *abort != 0);
      ++k;
      for (int j = it.jb; j < it.je && ok; ++j, ++G) {
        if (G == 0) continue;
        for (int q = 0; q < 4; ++q) {
          if (wwait(&s.ch_empty[q], (G - 1) & 1))
            pair_arrive(GATE_PAIR0 + q);
          else
            pair_sync(GATE_PAIR0 + q);
        }
      }
    }
  } else if (warp == AT_MMA_WARP) {
    // ------------------------------------------------------------------ MMA issuer (converged)
    {
      const uint32_t id1 = tc::idesc_bf16_f32(128, AT_H, 0, 0);   // A, B K-major
      const uint32_t id2 = tc::idesc_bf16_f32(128, AT_H, 1, 1);   // A, B MN-major
      // Base descriptors; a K step or a chunk only moves the start address, which is the low
      // 14-bit field (address >> 4), so the loops just add small constants.
      const uint64_t d_kv1 = tc::sdesc_sw128(tc::smem_u32(s.kv[0]), 16, 1024);
      const uint64_t d_q1 = tc::sdesc_sw128(tc::smem_u32(s.q[0]), 16, 1024);
      const uint64_t d_kv2 = tc::sdesc_sw128(tc::smem_u32(s.kv[0]), AT_BLK * 128, 1024);
      const uint64_t d_p2 = tc::sdesc_sw128(tc::smem_u32(s.p), AT_BLK * 128, 1024);
      // every lane waits (acquire per lane) and the warp takes one decision
      auto wwait = [&](uint64_t* bar, uint32_t parity) {
        return __all_sync(0xffffffffu, tc::mbar_wait(bar, parity, spin, abort));
      };
      uint32_t G = 0;
      int k = 0;
      bool ok = true;
      for (int item = first; item < items && ok; item += gridDim.x) {
        const ItemInfo it = item_info<kSplit>(a, item, head_groups);
        if (kSplit && it.je <= it.jb) continue;
        ok = wwait(&s.q_full, (uint32_t)(k & 1));
        ++k;
        for (int j = it.jb; j < it.je && ok; ++j, ++G) {
#pragma unroll
          for (int c = 0; c < AT_CHUNKS; ++c) {
            if ((c & 3) == 0) ok = wwait(&s.ch_full[c | 3], G & 1);
            if (!ok) break;
            if (lane == 0 && (c & 1)) A1_TRACE(12 + (c >> 1), k, j);
            tc::fence_proxy_async_smem();          // cp.async (generic) -> tensor core (async)
            tc::tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              tc::mma_bf16_ss_warp(tmem + TM_S, d_kv1 + (uint64_t)(c * (AT_BLK * 128 / 16) + 2 * kk),
                                   d_q1 + (uint64_t)(c * (AT_H * 128 / 16) + 2 * kk), id1,
                                   (c | kk) != 0);
          }
          if (!ok) break;
          tc::mma_commit_warp(&s.s_full);
          if (lane == 0) A1_TRACE(3, k, j);
          if (j + 1 == it.je) tc::mma_commit_warp(&s.q_empty);
          ok = wwait(&s.p_full, G & 1);
          if (!ok) break;
          if (lane == 0) A1_TRACE(4, k, j);
          tc::tc_fence_after();
          const uint32_t acc0 = j > it.jb ? 1u : 0u;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
#pragma unroll
            for (int ks = 0; ks < AT_BLK / 16; ++ks)
              tc::mma_bf16_ss_warp(tmem + TM_O + 64 * q,
                                   d_kv2 + (uint64_t)(2 * q * (AT_BLK * 128 / 16) + ks * 128),
                                   d_p2 + (uint64_t)(ks * 128), id2, ks > 0 ? 1u : acc0);
            tc::mma_commit_warp(&s.ch_empty[q]);
          }
          tc::mma_commit_warp(&s.o_done);
          if (lane == 0) A1_TRACE(5, k, j);
        }
      }
      if (!ok) {
        tc::mma_commit_warp(&s.drain);               // every issued MMA completes before
        tc::mbar_drain(&s.drain, 0);                 // TMEM is released
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------------ softmax + epilogue
    const int quad = warp & 3, half = warp >> 2;
    const int slot = 32 * quad + lane;                 // TMEM lane: slot / channel row
    const int hb = 32 * half;                          // this thread's first head
    const uint32_t lane_base = (uint32_t)(32 * quad) << 16;
    uint32_t G = 0;
    int k = 0;
    bool ok = true;
    // The item's description, its sink logit and the validity of this thread's slot in the
    // next block are loaded one step ahead (global loads queue behind the producers' gather
    // traffic, so their latency is long).
    int item = first;
    ItemInfo it = item_info<kSplit>(a, item < items ? item : 0, head_groups);
    float sink_h = (quad == 0 && a.sink) ? __ldg(a.sink + it.hg * AT_H + hb + lane) : 0.f;
    bool vnext = item < items && it.je > it.jb && slot_row(a, it.cs, it.nc4, it.jb * AT_BLK + slot).valid;
    for (; item < items && ok; item += gridDim.x) {
      if (kSplit && it.je <= it.jb) {                  // a split without blocks: empty partial
        if (quad == 0) a.part_ml[((long long)item * AT_H + hb + lane)] = make_float2(-INFINITY, 0.f);
        const int nitem = item + gridDim.x;
        if (nitem < items) {
          it = item_info<kSplit>(a, nitem, head_groups);
          sink_h = (quad == 0 && a.sink) ? __ldg(a.sink + it.hg * AT_H + hb + lane) : 0.f;
          vnext = it.je > it.jb && slot_row(a, it.cs, it.nc4, it.jb * AT_BLK + slot).valid;
        }
        continue;
      }
      float lsum[32];                                  // sums of the bf16-rounded weights
#pragma unroll
      for (int h = 0; h < 32; ++h) lsum[h] = 0.f;
      for (int j = it.jb; j < it.je; ++j, ++G) {
        const bool valid = vnext;
        if (j + 1 < it.je) vnext = slot_row(a, it.cs, it.nc4, (j + 1) * AT_BLK + slot).valid;
        if (tid == 0) A1_TRACE(6, k, j);
        ok = tc::mbar_wait(&s.s_full, G & 1, spin, abort);
        ok = !bar_red_or(3, AT_SOFT, !ok);             // all 256 threads take the same branch
        if (!ok) break;
        if (tid == 0) A1_TRACE(7, k, j);
        tc::tc_fence_after();
        float z[32];
        tc::tmem_ld32(tmem + lane_base + TM_S + hb, z);
        tc::tmem_wait_ld_dep(z);
        // GEMM1 of this block completing implies GEMM2 of the previous block completed (it
        // waited for the chunks that GEMM2 released), so P and O^T are free to touch.
        uint8_t* prow = s.p + slot * 128;
        bool rescale = false;
        // After an item's first block every head has a finite running max m. Weights taken
        // against m are exact whatever m is (m cancels in the normalisation); they only have
        // to stay bounded, so the block maxima are needed just when some score exceeds its
        // running max by more than TAU -- then the exact path below recomputes this block.
        bool exact = j == it.jb;
        if (!exact) {
          // one FMA per weight: x = z * scale - m (log2 units); an invalid slot takes scale 0
          // (its x is -m, finite or +inf) and its weights are zeroed after the exponential
          uint32_t pk[16];
          bool over = false;
          const float sc = valid ? scale_log2 : 0.f;
#pragma unroll
          for (int h = 0; h < 32; h += 4) {
            const float4 m4 = *reinterpret_cast<const float4*>(&s.mcur[hb + h]);
            const float x0 = fmaf(z[h], sc, -m4.x), x1 = fmaf(z[h + 1], sc, -m4.y);
            const float x2 = fmaf(z[h + 2], sc, -m4.z), x3 = fmaf(z[h + 3], sc, -m4.w);
            over |= !(x0 <= TAU) | !(x1 <= TAU) | !(x2 <= TAU) | !(x3 <= TAU);
            __nv_bfloat162 b0 = __floats2bfloat162_rn(ex2_ftz(x0), ex2_ftz(x1));
            __nv_bfloat162 b1 = __floats2bfloat162_rn(ex2_ftz(x2), ex2_ftz(x3));
            pk[h / 2] = *reinterpret_cast<uint32_t*>(&b0);
            pk[h / 2 + 1] = *reinterpret_cast<uint32_t*>(&b1);
          }
          exact = bar_red_or(2, AT_SOFT, over && valid);
          if (!exact) {
            if (!valid) {
#pragma unroll
              for (int i = 0; i < 16; ++i) pk[i] = 0u;
            }
            // the denominator sums the same bf16-rounded weights the PV product uses
#pragma unroll
            for (int h = 0; h < 32; h += 2) add_bf16x2_f32(lsum[h], lsum[h + 1], pk[h / 2]);
#pragma unroll
            for (int c = 0; c < 4; ++c)
              *reinterpret_cast<uint4*>(prow + (((4 * half + c) ^ (slot & 7)) << 4)) =
                  make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
          }
        }
        if (exact) {
#pragma unroll
          for (int h = 0; h < 32; ++h) z[h] = valid ? z[h] * scale_log2 : -INFINITY;
          // the butterfly consumes z; the scores are read from TMEM again (S^T is not
          // overwritten before this block's P is published) while the block max is combined
          s.red[quad][hb + lane] = xpose_reduce32<true>(z);
          tc::tmem_ld32(tmem + lane_base + TM_S + hb, z);
          tc::named_barrier(1, AT_SOFT);
          bool grow = false;
          if (quad == 0) {                             // warps 0 and 4 own heads hb + lane
            const int h = hb + lane;
            const float bm = fmaxf(fmaxf(s.red[0][h], s.red[1][h]), fmaxf(s.red[2][h], s.red[3][h]));
            const float mo = s.mcur[h];
            float mn = mo, f = 1.f;
            if (mo == -INFINITY) {
              mn = bm;
              f = 0.f;
            } else if (bm > mo + TAU) {
              mn = bm;
              f = exp2f(mo - mn);
              grow = true;
            }
            s.mcur[h] = mn;
            s.moff[h] = mn == -INFINITY ? 0.f : mn;
            s.fac[h] = f;
          }
          rescale = bar_red_or(2, AT_SOFT, grow) && j > it.jb;
          tc::tmem_wait_ld_dep(z);
#pragma unroll
          for (int h = 0; h < 32; ++h) z[h] = valid ? z[h] * scale_log2 : -INFINITY;
          if (tid == 0) A1_TRACE(18, k, j);
#pragma unroll
          for (int c = 0; c < 4; ++c) {                // 8 heads -> one 16-byte P store
            uint32_t pk[4];
#pragma unroll
            for (int v = 0; v < 2; ++v) {
              const int h = 8 * c + 4 * v;
              const float4 mo = *reinterpret_cast<const float4*>(&s.moff[hb + h]);
              const float4 fa = *reinterpret_cast<const float4*>(&s.fac[hb + h]);
              __nv_bfloat162 b0 = __floats2bfloat162_rn(ex2_ftz(z[h] - mo.x), ex2_ftz(z[h + 1] - mo.y));
              __nv_bfloat162 b1 = __floats2bfloat162_rn(ex2_ftz(z[h + 2] - mo.z), ex2_ftz(z[h + 3] - mo.w));
              // the denominator sums the same bf16-rounded weights the PV product uses
              const float2 r0 = __bfloat1622float2(b0), r1 = __bfloat1622float2(b1);
              lsum[h] = fmaf(lsum[h], fa.x, r0.x);
              lsum[h + 1] = fmaf(lsum[h + 1], fa.y, r0.y);
              lsum[h + 2] = fmaf(lsum[h + 2], fa.z, r1.x);
              lsum[h + 3] = fmaf(lsum[h + 3], fa.w, r1.y);
              pk[2 * v] = *reinterpret_cast<uint32_t*>(&b0);
              pk[2 * v + 1] = *reinterpret_cast<uint32_t*>(&b1);
            }
            *reinterpret_cast<uint4*>(prow + (((4 * half + c) ^ (slot & 7)) << 4)) =
                make_uint4(pk[0], pk[1], pk[2], pk[3]);
          }
        }
        if (rescale) {                                 // rare: a head's max grew by > 2^TAU
#pragma unroll 1
          for (int q = 0; q < 4; ++q) {
            asm volatile("" ::: "memory");             // re-read the factors: keeps them out
            float o[32];                               // of registers across iterations
            const uint32_t addr = tmem + lane_base + TM_O + 64 * q + hb;
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
        tc::mbar_arrive(&s.p_full);
        if (tid == 0) A1_TRACE(17, k, j);
      }
      if (!ok) break;
      // ---------------------------------------------------------------- epilogue
      const int nitem = item + gridDim.x;
      ItemInfo nx = it;
      float nsink = 0.f;
      if (nitem < items) {
        nx = item_info<kSplit>(a, nitem, head_groups);
        nsink = (quad == 0 && a.sink) ? __ldg(a.sink + nx.hg * AT_H + hb + lane) : 0.f;
        vnext = nx.je > nx.jb && slot_row(a, nx.cs, nx.nc4, nx.jb * AT_BLK + slot).valid;
      }
      // GEMM2 of the last block is complete (GEMM1 of that block completing already implies
      // GEMM2 of the block before it, so the phase waited here is unambiguous).
      ok = tc::mbar_wait(&s.o_done, (G - 1) & 1, spin, abort);
      ok = !bar_red_or(3, AT_SOFT, !ok);
      if (!ok) break;
      if (tid == 0) A1_TRACE(20, k, 0);
      tc::tc_fence_after();
      s.red[quad][hb + lane] = xpose_reduce32<false>(lsum);
      tc::named_barrier(1, AT_SOFT);
      if (tid == 0) A1_TRACE(21, k, 0);
      const int h0 = it.hg * AT_H;
      if (kSplit) {
        // partial of this split: running max m (log2 units), denominator L relative to m and
        // the unnormalised O^T, all fp32; the combine kernel applies the sink and normalises
        if (quad == 0) {
          const int h = hb + lane;
          const float L = (s.red[0][h] + s.red[1][h]) + (s.red[2][h] + s.red[3][h]);
          a.part_ml[(long long)item * AT_H + h] = make_float2(s.mcur[h], L);
          s.mcur[h] = -INFINITY;
        }
        float* po = a.part_o + ((long long)item * AT_H + hb) * AT_C + 32 * quad + lane;
        for (int q = 0; q < 4; ++q) {
          float o[32];
          tc::tmem_ld32(tmem + lane_base + TM_O + 64 * q + hb, o);
          tc::tmem_wait_ld_dep(o);
#pragma unroll
          for (int u = 0; u < 32; ++u) po[(long long)u * AT_C + 128 * q] = o[u];
        }
        tc::tc_fence_before();
        ++k;
        it = nx;
        sink_h = nsink;
        continue;
      }
      if (quad == 0) {
        const int h = hb + lane;
        const float L = (s.red[0][h] + s.red[1][h]) + (s.red[2][h] + s.red[3][h]);
        const float m = s.mcur[h];
        const float s2 = a.sink ? sink_h * LOG2E : -INFINITY;
        const float mf = fmaxf(m, s2);
        const float em = m == -INFINITY ? 0.f : exp2f(m - mf);
        const float den = L * em + (a.sink ? exp2f(s2 - mf) : 0.f);
        float inv = 0.f, lse = -INFINITY;
        if (den > 0.f && mf != -INFINITY) {
          inv = em / den;
          lse = (mf + log2f(den)) * LN2;
        }
        s.inv[h] = inv;
        if (a.lse) a.lse[(long long)it.qi * a.H + h0 + h] = lse;
        s.mcur[h] = -INFINITY;                         // the next item starts fresh
      }
      if (a.rope_out && tid < 32) {                    // pair tid of the last 64 channels
        const int qb = it.qi / a.nq;
        const long long tpos = (long long)a.q_pos0[qb] + (it.qi - qb * a.nq);
        rope_cos_sin(tpos, tid, 64, s.rcos[tid], s.rsin[tid]);
      }
      tc::named_barrier(1, AT_SOFT);
      if (tid == 0) A1_TRACE(22, k, 0);
      // O^T tiles of 128 channels. Each warp reads its 32 channels x 32 heads as two 16-lane
      // loads in the m8n8 fragment layout (thread t: channels c0 + t/4 and c0 + 8 + t/4, head
      // pairs 2(t%4) + 8k), scales and packs them to bf16 and writes them with transposing
      // 8x8 matrix stores, so each stored 16-byte row is 8 consecutive channels of one head.
      // The rows land in the warp's own part of the P buffer (free now: 32 heads x 64 bytes
      // of a 128-byte swizzled [64 heads x 64 channels] box), which the warp reads back as
      // rows of one head and stores to O with 16-byte stores: no CTA barrier or bulk-copy
      // wait between tiles.
      const int tq = lane & 3, mrow = lane & 7, mat = lane >> 3;
      float2 inv2[4];                                  // 1/denominator of this thread's heads
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) inv2[kk] = *reinterpret_cast<const float2*>(&s.inv[hb + 8 * kk + 2 * tq]);
      const uint32_t p0 = tc::smem_u32(s.p) + (uint32_t)((quad >> 1) * (AT_H * 128));
      // read-back mapping: a phase of 8 lanes covers heads r and r + 4 (unit sets disjoint
      // under the swizzle), 4 lanes per head row of 64 bytes
      const int rb_u = 4 * (quad & 1) + (lane & 3);
      const int rb_r = (lane >> 3) + 4 * ((lane >> 2) & 1);
      __nv_bfloat16* const obase =
          static_cast<__nv_bfloat16*>(a.O) + ((long long)it.qi * a.H + h0 + hb) * AT_C + 32 * quad + 8 * (lane & 3);
      for (int q = 0; q < 4; ++q) {
        uint32_t pk[2][8];                             // [channel half][matrix slot]
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          float v[16];
          tc::tmem_ld16x256b_x4(tmem + ((uint32_t)(32 * quad + 16 * hh) << 16) + TM_O + 64 * q + hb, v);
          tc::tmem_wait_ld_dep16(v);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            v[4 * kk] *= inv2[kk].x;
            v[4 * kk + 1] *= inv2[kk].y;
            v[4 * kk + 2] *= inv2[kk].x;
            v[4 * kk + 3] *= inv2[kk].y;
          }
          if (a.rope_out && q == 3 && quad >= 2) {
            // channels 448..511 (TMEM lanes 64..127 of the last M-tile): the pair partner of
            // lane L is lane L^1, held by thread lane^4 in the same register
            const bool odd = (lane >> 2) & 1;
#pragma unroll
            for (int r = 0; r < 16; ++r) {
              const float other = __shfl_xor_sync(0xffffffffu, v[r], 4);
              const int ch = 32 * quad + 16 * hh + (lane >> 2) + 8 * ((r & 3) >> 1);   // 64..127
              const int pr = (ch - 64) >> 1;
              const float cs = s.rcos[pr], sn = s.rsin[pr];
              // rotation by minus the angle: a' = a cos + b sin, b' = b cos - a sin
              v[r] = odd ? fmaf(v[r], cs, -other * sn) : fmaf(v[r], cs, other * sn);
            }
          }
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            pk[hh][2 * kk] = pack_bf16(v[4 * kk], v[4 * kk + 1]);
            pk[hh][2 * kk + 1] = pack_bf16(v[4 * kk + 2], v[4 * kk + 3]);
          }
        }
        __syncwarp();                                  // the previous tile's read-back done
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
        __syncwarp();
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int r = 8 * i + rb_r;                  // head hb + r
          const int row = hb + r;
          uint4 v;
          asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                       : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                       : "r"(p0 + (uint32_t)(row * 128 + ((rb_u ^ (row & 7)) << 4)))
                       : "memory");
          *reinterpret_cast<uint4*>(obase + (long long)r * AT_C + 128 * q) = v;
        }
        if (tid == 0) A1_TRACE(24 + q, k, 0);
      }
      // the next item's softmax writes P only after a barrier this thread reaches after here
      tc::tc_fence_before();
      if (tid == 0) A1_TRACE(23, k, 0);
      ++k;
      it = nx;
      sink_h = nsink;
    }
  }
  tc::tc_fence_before();
  __syncthreads();
  if (warp == AT_MMA_WARP) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, TM_COLS);
  }
  if (tid == AT_SOFT && *abort) {
    // After an abort (final now: every thread has passed the barrier) the last item's Q and
    // the last block's cp.async arrivals may still be landing: let them land
    // before the CTA's shared memory is released. Without an abort they were all consumed.
    if (prod_k > 0) tc::mbar_drain(&s.q_full, (uint32_t)((prod_k - 1) & 1));
    if (prod_G > 0)
      for (int c = 3; c < AT_CHUNKS; c += 4) tc::mbar_drain(&s.ch_full[c], (prod_G - 1) & 1);
  }
}

// Merges the nsplit partials of every (query, head group): one warp per head (grid: items x
// 8 CTAs of 8 warps), the combined max M over the splits and the sink, weights 2^(m_s - M),
// one normalisation, bf16 output, LSE. Splits without candidates carry m = -inf and are not
// read.
__global__ void __launch_bounds__(256) attn_combine_kernel(const AttnArgs a, int head_groups) {
  const int base = blockIdx.x;
  const int qi = base / head_groups, hg = base % head_groups;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int S = a.nsplit;
  {
    const int hl = 8 * blockIdx.y + warp;              // head within the group
    const int h = hg * AT_H + hl;
    const float2 ml = lane < S ? a.part_ml[((long long)base * S + lane) * AT_H + hl]
                               : make_float2(-INFINITY, 0.f);
    float M = ml.x;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
    const float s2 = a.sink ? __ldg(a.sink + h) * LOG2E : -INFINITY;
    M = fmaxf(M, s2);
    const float e = (ml.x == -INFINITY || M == -INFINITY) ? 0.f : exp2f(ml.x - M);
    float den = e * ml.y;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) den += __shfl_xor_sync(0xffffffffu, den, off);
    if (a.sink && M != -INFINITY) den += exp2f(s2 - M);
    const float inv = den > 0.f ? 1.f / den : 0.f;
    float acc[16];
#pragma unroll
    for (int u = 0; u < 16; ++u) acc[u] = 0.f;
    for (int sp = 0; sp < S; ++sp) {
      const float es = __shfl_sync(0xffffffffu, e, sp);
      if (es == 0.f) continue;
      const float4* src = reinterpret_cast<const float4*>(
          a.part_o + (((long long)base * S + sp) * AT_H + hl) * AT_C + 16 * lane);
#pragma unroll
      for (int v = 0; v < 4; ++v) {
        const float4 x = src[v];
        acc[4 * v] = fmaf(es, x.x, acc[4 * v]);
        acc[4 * v + 1] = fmaf(es, x.y, acc[4 * v + 1]);
        acc[4 * v + 2] = fmaf(es, x.z, acc[4 * v + 2]);
        acc[4 * v + 3] = fmaf(es, x.w, acc[4 * v + 3]);
      }
    }
    if (a.rope_out && lane >= (AT_C - 64) / 16) {      // channels 448..511: inverse RoPE
      const int qb = qi / a.nq;
      const long long tpos = (long long)a.q_pos0[qb] + (qi - qb * a.nq);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        float cs, sn;
        rope_cos_sin(tpos, 8 * (lane - (AT_C - 64) / 16) + j, 64, cs, sn);
        rope_apply(acc[2 * j], acc[2 * j + 1], cs, sn, true);
      }
    }
    uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(a.O) +
                                          ((long long)qi * a.H + h) * AT_C + 16 * lane);
    dst[0] = make_uint4(pack_bf16(acc[0] * inv, acc[1] * inv), pack_bf16(acc[2] * inv, acc[3] * inv),
                        pack_bf16(acc[4] * inv, acc[5] * inv), pack_bf16(acc[6] * inv, acc[7] * inv));
    dst[1] = make_uint4(pack_bf16(acc[8] * inv, acc[9] * inv), pack_bf16(acc[10] * inv, acc[11] * inv),
                        pack_bf16(acc[12] * inv, acc[13] * inv), pack_bf16(acc[14] * inv, acc[15] * inv));
    if (lane == 0 && a.lse)
      a.lse[(long long)qi * a.H + h] = (den > 0.f && M != -INFINITY) ? (M + log2f(den)) * LN2 : -INFINITY;
  }
}

}  // namespace

// Bytes of split partials per (query, head group) and split.
long long attn_split_bytes_per_item(int c) { return (long long)AT_H * ((long long)c * 4 + 8); }

int launch_attn_tc(const AttnArgs& a_in, cudaStream_t st, bool* used) {
  AttnArgs a = a_in;
  *used = false;
  const char* force = std::getenv("DSV4_FORCE_SIMT");
  if (force && force[0] == '1') return DSV4_OK;
  if (a.c != AT_C || a.H % AT_H != 0 || (a.rope_out != 0 && a.rope_out != 64)) return DSV4_OK;
  if (!aligned16(a.Q) || !aligned16(a.local) || (a.pool && !aligned16(a.pool))) return DSV4_OK;
  const long long nrows_q = (long long)a.B * a.nq * a.H;
  const long long items = (long long)a.B * a.nq * (a.H / AT_H);
  if (nrows_q >= (1ll << 31) || items >= (1ll << 31)) return DSV4_OK;
  static int sms = 0;
  if (sms == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (sms <= 0) sms = 148;
    cudaError_t e = cudaFuncSetAttribute(attn_tc_kernel<false>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)AT_SMEM);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(attn_tc_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)AT_SMEM);
    if (e != cudaSuccess) return fail(DSV4_ERR_CUDA, "attn_tc: %s", cudaGetErrorString(e));
  }
  const long long nrows_local = (long long)a.B * a.R;
  if (nrows_local >= (1ll << 31) || !aligned16(a.O)) return DSV4_OK;
  CUtensorMap mq;
  int s = encode_tensor_map_2d(&mq, a.Q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, AT_C, nrows_q, 64,
                               AT_H, CU_TENSOR_MAP_SWIZZLE_128B);
  if (s != DSV4_OK) return s;
  // Few (query, head group) items: split each candidate list so that about one and a half
  // work items per SM exist, as far as the caller's workspace (a.nsplit = its capacity)
  // allows (measured on 64 dense decode lists of 9-65 blocks: 4 splits 138 us, 5 splits
  // 151 us, 8 splits 156 us; each split pays its own Q load, setup and partial write).
  // A selected list has at most round4(k) + round4(w) candidates; a split must keep at least
  // 4 blocks.
  int nsplit = 1;
  if (a.part_o && a.nsplit > 1 && items < sms) {
    nsplit = (int)((3 * sms / 2 + items - 1) / items);
    if (nsplit > a.nsplit) nsplit = a.nsplit;
    if (a.idx) {
      const int nb_max = (((a.k + 3) & ~3) + ((a.w + 3) & ~3) + AT_BLK - 1) / AT_BLK;
      if (nsplit > nb_max / 4) nsplit = nb_max / 4 > 1 ? nb_max / 4 : 1;
    }
  }
  a.nsplit = nsplit;
  if (nsplit > 1)
    a.part_ml = reinterpret_cast<float2*>(a.part_o + items * nsplit * AT_H * (long long)AT_C);

  const long long work = items * nsplit;
  // split lists (decode): one CTA per work item, so that the hardware hands items of very
  // different lengths to SMs as they free up; unsplit lists: persistent, one CTA per SM
  const long long grid = (nsplit > 1 || work < sms) ? work : sms;
  if (nsplit > 1)
    attn_tc_kernel<true><<<(unsigned)grid, AT_THREADS, AT_SMEM, st>>>(
        a, mq, a.H / AT_H, (int)work, a.scale * LOG2E, spin_limit());
  else
    attn_tc_kernel<false><<<(unsigned)grid, AT_THREADS, AT_SMEM, st>>>(
        a, mq, a.H / AT_H, (int)work, a.scale * LOG2E, spin_limit());
  *used = true;
  int s2 = launch_status("hybrid attention (tensor cores)");
  if (s2 != DSV4_OK || nsplit == 1) return s2;
  attn_combine_kernel<<<dim3((unsigned)items, AT_H / 8), 256, 0, st>>>(a, a.H / AT_H);
  return launch_status("hybrid attention split combine");
}

}  // namespace dsv4

#ifdef DSV4_TRACE
extern "C" int dsv4_trace_read_attn1(unsigned long long* host, size_t n) {
  return cudaMemcpyFromSymbol(host, dsv4::g_attn1_trace, n * sizeof(unsigned long long)) == cudaSuccess ? 0 : 3;
}
#endif
