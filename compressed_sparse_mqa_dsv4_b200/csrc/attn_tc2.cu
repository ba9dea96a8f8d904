// Hybrid shared-KV MQA on the 5th-generation tensor cores, channel-split over a 2-CTA
// cluster, persistent, with cp.async row gathers.
//
// "CSA And HCA: Definition, State, And Cost Model": s3.2/s4 every candidate row is both key
// and value for all heads; s5.1 one candidate list (selected or all completed compressed
// entries, then the local window) under one softmax per head; s5.3 the sink logit joins
// the denominator only. Per-query valid counts follow pypto-lib PR #834.
//
// Work item = (query, group of 64 heads). A cluster of two CTAs (two SMs) owns one item at a
// time; CTA r holds channels [256r, 256r+256) of every candidate row and of Q, so each SM
// keeps half of a 128-slot KV block and can double-buffer it:
//   GEMM1  S_r^T[128 slots x 64 heads] = KV_r[slots x 256] . Q_r[heads x 256]^T   (partial)
//   exchange: each CTA sends its partial S (all heads) to the other over DSMEM and adds the
//          other's, so both hold the identical full S and run the identical softmax; each
//          writes the full P^T into its own shared memory (no further exchange)
//   GEMM2  O_r^T[256 channels x 64 heads] += KV_r^T . P^T
// Both GEMMs use M = 128 (full tensor-core rate). The same swizzled KV stage is the K-major
// A operand of GEMM1 and the MN-major A operand of GEMM2. GEMM1 of block j+1 overlaps the
// softmax of block j (two S buffers, two KV stages).
//
// Candidate rows are gathered with 16-byte cp.async by three producer warps (one 512-byte
// half-row per warp instruction): on B200 that moves a gathered block about 3x faster than
// TMA row gathers. Q uses 2D TMA.
//
// Warps: 0-7 softmax/epilogue (warp w reads TMEM lane quadrant w%4 for heads 32(w/4)..+31),
// 8-10 producer, 11 MMA issuer and TMEM owner (12 warps: 3 per SM sub-partition, so up to
// 168 registers per thread). Every wait is bounded; a cluster barrier at
// the end keeps both CTAs alive until neither can touch the other's shared memory.
#include <cstdio>
#include <cstdlib>

#include "attn_common.cuh"
#include "tc_common.cuh"

namespace dsv4 {
namespace {

constexpr int A2_C = 512;               // channels of a row
constexpr int A2_CH = 256;              // channels per CTA
constexpr int A2_H = 64;                // heads per item
constexpr int A2_BLK = 128;             // candidate slots per block
constexpr int A2_KCH = A2_CH / 64;      // 64-channel chunks per CTA
constexpr int A2_SOFT = 256;            // softmax threads (8 warps)
constexpr int A2_PROD = 96;             // producer threads (3 warps)
constexpr int A2_THREADS = A2_SOFT + A2_PROD + 32;
constexpr uint32_t T2_S = 0;            // S buffers at columns 0 and 64
constexpr uint32_t T2_O = 128;          // O^T tiles at 128 + 64 q
constexpr uint32_t T2_COLS = 256;
constexpr float TAU2 = 8.f;             // log2-domain max growth tolerated before rescaling
constexpr float LOG2E2 = 1.4426950408889634f;
constexpr float LN2_2 = 0.6931471805599453f;

struct Smem2 {
  uint8_t q[A2_KCH][A2_H * 128];              // 32 KiB, K-major SW128 [64 heads][64 ch]
  uint8_t kv[2][A2_KCH][A2_BLK * 128];        // 128 KiB, [128 slots][64 ch] per chunk
  uint8_t p[A2_BLK * 128];                    // 16 KiB, P^T [slots][64 heads] MN-major SW128;
                                              // also the O staging tile of the epilogue
  float xs[A2_BLK][A2_H];                     // 32 KiB, the peer's partial S (swizzled rows)
  float red[4][A2_H];
  float mcur[A2_H];
  float fac[A2_H];
  float inv[A2_H];
  uint64_t rowaddr[A2_BLK];                   // global address of each slot's row (producer)
  uint64_t q_full, q_empty;
  uint64_t kv_full[2], kv_empty[2];
  uint64_t s_full[2], xs_full, xs_empty, p_full;
  uint64_t o_blk[2], drain;
  uint32_t tmem_base;
  int abort;
};
constexpr size_t A2_SMEM = sizeof(Smem2) + 1024;
static_assert(A2_SMEM <= 232448, "shared memory of the cluster attention kernel");

#ifdef DSV4_TRACE
// Phase timestamps (clock64) of cluster 0, first 4 items, first 8 blocks: a profiling aid
// compiled only into traced builds.
__device__ unsigned long long g_attn_trace[2][4][8][32];
#define A2_TRACE(ev, k_, j_)                                   \
  do {                                                         \
    if (cluster_id == 0 && (k_) < 4 && (j_) < 8)               \
      g_attn_trace[rank][k_][j_][ev] = clock64();              \
  } while (0)
#else
#define A2_TRACE(ev, k_, j_) \
  do {                       \
  } while (0)
#endif

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\nbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ uint32_t mapa(uint32_t local, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(local), "r"(rank));
  return r;
}
// 16-byte store into the peer CTA's shared memory whose completion is counted (in bytes) on
// the peer's mbarrier; no release fence is needed for the peer to observe it.
__device__ __forceinline__ void st_async_v4(uint32_t addr, float a, float b, float c, float d,
                                            uint32_t remote_bar) {
  asm volatile(
      "st.async.shared::cluster.mbarrier::complete_tx::bytes.v4.f32 [%0], {%1, %2, %3, %4}, [%5];" ::"r"(
          addr),
      "f"(a), "f"(b), "f"(c), "f"(d), "r"(remote_bar)
      : "memory");
}
__device__ __forceinline__ void arrive_remote(uint32_t bar_cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(bar_cluster_addr)
               : "memory");
}
__device__ __forceinline__ bool try_wait_cluster(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}"
      : "=r"(ok)
      : "r"(tc::smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded wait on a local barrier that also receives the peer's release arrivals.
__device__ __forceinline__ bool wait_cluster(uint64_t* bar, uint32_t parity, uint32_t spin,
                                             volatile int* abort) {
  for (uint32_t i = 0; i < spin; ++i) {
    if (try_wait_cluster(bar, parity)) return true;
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
__device__ __forceinline__ bool bar_red_or2(uint32_t id, uint32_t threads, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n .reg .pred p, q;\n setp.ne.u32 p, %1, 0;\n"
      " barrier.red.or.pred q, %2, %3, p;\n selp.u32 %0, 1, 0, q;\n}"
      : "=r"(r)
      : "r"((uint32_t)pred), "r"(id), "r"(threads)
      : "memory");
  return r != 0;
}
__device__ __forceinline__ void cp_async16(uint32_t dst, uint64_t src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
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

struct Slot {
  int part;            // 0 pool, 1 local
  long long row;
  bool valid, bad;
};

__device__ __forceinline__ Slot slot_of(const AttnArgs& a, const CandidateSet& cs, int nc4, int g) {
  Slot r;
  r.bad = false;
  if (g < nc4) {
    r.part = 0;
    r.row = -1;
    r.valid = g < cs.n_comp;
    if (r.valid) {
      const long long s = cs.sel ? (long long)__ldg(cs.sel + g) : (long long)g;
      const long long row = cs.pool_base + s;
      if (s < 0 || s >= cs.Et || row < 0 || row >= a.pool_rows) {
        r.valid = false;
        r.bad = true;
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

struct ItemInfo {
  int qi, hg, nc4, nb;
  CandidateSet cs;
};

__device__ __forceinline__ ItemInfo item_info(const AttnArgs& a, int item, int head_groups) {
  ItemInfo it;
  it.qi = item / head_groups;
  it.hg = item % head_groups;
  const int b = it.qi / a.nq, i = it.qi % a.nq;
  it.cs = make_candidates(a, b, i);
  it.nc4 = (it.cs.n_comp + 3) & ~3;
  const int nl4 = (it.cs.n_local + 3) & ~3;
  it.nb = (it.nc4 + nl4 + A2_BLK - 1) / A2_BLK;
  return it;
}

__global__ void __cluster_dims__(2, 1, 1) __maxnreg__(168)
    attn_tc2_kernel(const AttnArgs a, const __grid_constant__ CUtensorMap map_q, int head_groups,
                    int items, float scale_log2, uint32_t spin) {
  extern __shared__ uint8_t smem_raw[];
  Smem2& s = *reinterpret_cast<Smem2*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                       ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t rank = cluster_rank(), peer = rank ^ 1u;
  const int cluster_id = blockIdx.x >> 1, nclusters = gridDim.x >> 1;
  volatile int* abort = &s.abort;

  if (tid == 0) {
    tc::mbar_init(&s.q_full, 1);
    tc::mbar_init(&s.q_empty, 1);
    for (int i = 0; i < 2; ++i) {
      tc::mbar_init(&s.kv_full[i], A2_PROD);
      tc::mbar_init(&s.kv_empty[i], 1);
      tc::mbar_init(&s.s_full[i], 1);
      tc::mbar_init(&s.o_blk[i], 1);
    }
    tc::mbar_init(&s.xs_full, 1);                   // local expect_tx + the peer's st.async bytes
    tc::mbar_init(&s.xs_empty, 1);                  // one remote arrive per consumed block
    tc::mbar_init(&s.p_full, A2_SOFT);
    tc::mbar_init(&s.drain, 1);
    s.abort = 0;
    tc::fence_barrier_init();
  }
  if (tid < A2_H) s.mcur[tid] = -INFINITY;
  if (warp == 11) {
    tc::tmem_alloc(&s.tmem_base, T2_COLS);
    tc::tmem_relinquish();
  }
  tc::tc_fence_before();
  __syncthreads();
  cluster_sync();                       // the peer's barriers exist before any remote arrive
  tc::tc_fence_after();
  const uint32_t tmem = s.tmem_base;

  if (warp >= 8 && warp < 11) {
    // ------------------------------------------------------------------ producer (4 warps)
    const int pt = tid - A2_SOFT, pw = pt >> 5;
    // this lane's 16 bytes of a 512-byte half-row: chunk (64 channels) and piece (8 channels)
    const int piece = lane & 7, chunk = lane >> 3;
    const uint64_t my_off = (uint64_t)rank * A2_CH * 2 + chunk * 128 + piece * 16;
    const uint64_t pool_addr = reinterpret_cast<uint64_t>(a.pool);
    const uint64_t local_addr = reinterpret_cast<uint64_t>(a.local);
    uint32_t G = 0;
    int k = 0;
    bool ok = true;
    if (pt == 0) tc::prefetch_tensormap(&map_q);
    for (int item = cluster_id; item < items && ok; item += nclusters, ++k) {
      const ItemInfo it = item_info(a, item, head_groups);
      if (pt == 0) {
        if (k > 0) ok = tc::mbar_wait(&s.q_empty, (uint32_t)((k - 1) & 1), spin, abort);
        if (ok) {
          tc::mbar_arrive_expect_tx(&s.q_full, A2_KCH * A2_H * 128);
          const int qrow = it.qi * a.H + it.hg * A2_H;
          for (int c = 0; c < A2_KCH; ++c)
            tc::tma_load_2d(s.q[c], &map_q, &s.q_full, (int)rank * A2_CH + 64 * c, qrow);
        }
      }
      ok = !bar_red_or2(4, A2_PROD, !ok);
      if (!ok) break;
      for (int j = 0; j < it.nb; ++j, ++G) {
        const int st = G & 1;
        // resolve the block's 128 row addresses (one index load per slot)
        for (int u = pt; u < A2_BLK; u += A2_PROD) {
          const Slot sl = slot_of(a, it.cs, it.nc4, j * A2_BLK + u);
          if (sl.bad && rank == 0) flag_status(DSV4_ERR_DEVICE_BOUNDS);
          s.rowaddr[u] =
              (sl.part == 0 && sl.valid)
                  ? pool_addr + (uint64_t)sl.row * A2_C * 2
                  : local_addr + (uint64_t)(sl.part == 1 ? sl.row : it.cs.local_base) * A2_C * 2;
        }
        ok = G >= 2 ? tc::mbar_wait(&s.kv_empty[st], ((G >> 1) - 1) & 1, spin, abort) : true;
        ok = !bar_red_or2(4, A2_PROD, !ok);             // also publishes rowaddr[]
        if (!ok) break;
        if (pt == 0) A2_TRACE(0, k, j);
        uint8_t* dst_base = s.kv[st][chunk];
        // warp pw copies rows pw, pw + 3, ...: one 512-byte half-row per warp instruction
#pragma unroll 4
        for (int row = pw; row < A2_BLK; row += A2_PROD / 32) {
          const uint64_t src = s.rowaddr[row] + my_off;
          cp_async16(tc::smem_u32(dst_base + row * 128 + ((piece ^ (row & 7)) << 4)), src);
        }
        cp_async_arrive_noinc(&s.kv_full[st]);
        if (pt == 0) A2_TRACE(1, k, j);
        tc::named_barrier(5, A2_PROD);                  // rowaddr[] is rewritten next block
      }
    }
    // let every copy of this thread land before the CTA can exit
    asm volatile("cp.async.wait_all;" ::: "memory");
  } else if (warp == 11) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t id1 = tc::idesc_bf16_f32(128, A2_H, 0, 0);
      const uint32_t id2 = tc::idesc_bf16_f32(128, A2_H, 1, 1);
      uint32_t G = 0;
      int k = 0;
      bool ok = true;
      auto gemm1 = [&](uint32_t g) -> bool {
        const int st = g & 1;
        if (!tc::mbar_wait(&s.kv_full[st], (g >> 1) & 1, spin, abort)) return false;
        // rows written by cp.async (generic proxy) are read by the tensor core (async proxy)
        tc::fence_proxy_async_smem();
        tc::tc_fence_after();
#pragma unroll
        for (int c = 0; c < A2_KCH; ++c) {
          const uint32_t kvb = tc::smem_u32(s.kv[st][c]), qb = tc::smem_u32(s.q[c]);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            tc::mma_bf16_ss(tmem + T2_S + 64 * st, tc::sdesc_sw128(kvb + kk * 32, 16, 1024),
                            tc::sdesc_sw128(qb + kk * 32, 16, 1024), id1, (c | kk) != 0);
        }
        tc::mma_commit(&s.s_full[st]);
        return true;
      };
      for (int item = cluster_id; item < items && ok; item += nclusters, ++k) {
        const ItemInfo it = item_info(a, item, head_groups);
        ok = tc::mbar_wait(&s.q_full, (uint32_t)(k & 1), spin, abort);
        if (!ok) break;
        ok = gemm1(G);
        A2_TRACE(3, k, 0);
        if (it.nb == 1 && ok) tc::mma_commit(&s.q_empty);
        for (int j = 0; j < it.nb && ok; ++j, ++G) {
          if (j + 1 < it.nb) {
            ok = gemm1(G + 1);
            A2_TRACE(3, k, j + 1);
            if (!ok) break;
            if (j + 2 == it.nb) tc::mma_commit(&s.q_empty);
          }
          const int st = G & 1;
          ok = tc::mbar_wait(&s.p_full, G & 1, spin, abort);
          if (!ok) break;
          A2_TRACE(4, k, j);
          tc::tc_fence_after();
          const uint32_t pb = tc::smem_u32(s.p);
#pragma unroll
          for (int q = 0; q < 2; ++q) {
            const uint32_t kvb = tc::smem_u32(s.kv[st][2 * q]);
#pragma unroll
            for (int ks = 0; ks < A2_BLK / 16; ++ks)
              tc::mma_bf16_ss(tmem + T2_O + 64 * q,
                              tc::sdesc_sw128(kvb + ks * 2048, A2_BLK * 128, 1024),
                              tc::sdesc_sw128(pb + ks * 2048, A2_BLK * 128, 1024), id2,
                              (j > 0 || ks > 0) ? 1u : 0u);
          }
          tc::mma_commit(&s.kv_empty[st]);
          tc::mma_commit(&s.o_blk[st]);
          A2_TRACE(5, k, j);
        }
      }
      if (!ok) {
        tc::mma_commit(&s.drain);
        volatile int never = 0;
        tc::mbar_wait(&s.drain, 0, spin, &never);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------------ softmax + epilogue
    const int quad = warp & 3, half = warp >> 2;        // lane quadrant, head half
    const int slot = 32 * quad + lane;                  // TMEM lane = slot / channel row
    const int hb = 32 * half;                           // first head of this thread
    const uint32_t lane_base = (uint32_t)(32 * quad) << 16;
    const uint32_t r_xs = mapa(tc::smem_u32(&s.xs[slot][0]), peer);   // my row in the peer
    const uint32_t rb_xs_full = mapa(tc::smem_u32(&s.xs_full), peer);
    const uint32_t rb_xs_empty = mapa(tc::smem_u32(&s.xs_empty), peer);
    uint32_t G = 0;
    int k = 0;
    bool ok = true;
    for (int item = cluster_id; item < items && ok; item += nclusters, ++k) {
      const ItemInfo it = item_info(a, item, head_groups);
      float lsum[32];                                   // sums of the bf16-rounded weights
#pragma unroll
      for (int h = 0; h < 32; ++h) lsum[h] = 0.f;
      for (int j = 0; j < it.nb; ++j, ++G) {
        const int st = G & 1;
        const Slot sl = slot_of(a, it.cs, it.nc4, j * A2_BLK + slot);   // load overlaps the wait
        if (tid == 0) A2_TRACE(6, k, j);
        ok = tc::mbar_wait(&s.s_full[st], (G >> 1) & 1, spin, abort);
        ok = !bar_red_or2(3, A2_SOFT, !ok);
        if (!ok) break;
        if (tid == 0) A2_TRACE(7, k, j);
        tc::tc_fence_after();
        float z[32];
        tc::tmem_ld32(tmem + lane_base + T2_S + 64 * st + hb, z);
        tc::tmem_wait_ld();
        // my partial -> the peer (after it consumed the previous block's partial)
        if (G > 0) {
          ok = wait_cluster(&s.xs_empty, (G - 1) & 1, spin, abort);
          ok = !bar_red_or2(3, A2_SOFT, !ok);
          if (!ok) break;
        }
        // asynchronous remote stores; each one counts its bytes on the peer's xs_full
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const int cc = 8 * half + c;                  // 16-byte chunk within the 256-B row
          st_async_v4(r_xs + 16 * (cc ^ (slot & 7)), z[4 * c], z[4 * c + 1], z[4 * c + 2],
                      z[4 * c + 3], rb_xs_full);
        }
        if (tid == 0) tc::mbar_arrive_expect_tx(&s.xs_full, A2_BLK * A2_H * 4);
        if (tid == 0) A2_TRACE(9, k, j);
        ok = wait_cluster(&s.xs_full, G & 1, spin, abort);
        ok = !bar_red_or2(3, A2_SOFT, !ok);
        if (!ok) break;
        if (tid == 0) A2_TRACE(10, k, j);
        const float* xr = s.xs[slot];
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const int cc = 8 * half + c;
          const float4 x4 = *reinterpret_cast<const float4*>(xr + 4 * (cc ^ (slot & 7)));
          z[4 * c] = sl.valid ? (z[4 * c] + x4.x) * scale_log2 : -INFINITY;
          z[4 * c + 1] = sl.valid ? (z[4 * c + 1] + x4.y) * scale_log2 : -INFINITY;
          z[4 * c + 2] = sl.valid ? (z[4 * c + 2] + x4.z) * scale_log2 : -INFINITY;
          z[4 * c + 3] = sl.valid ? (z[4 * c + 3] + x4.w) * scale_log2 : -INFINITY;
        }
        // block max per head: butterfly within the warp, then the 4 lane quadrants
        {
          float red[32];
#pragma unroll
          for (int h = 0; h < 32; ++h) red[h] = z[h];
          s.red[quad][hb + lane] = xpose_reduce32<true>(red);
        }
        tc::named_barrier(1, A2_SOFT);
        // every thread has read its xs row: the peer may send its next partial
        if (tid == 0) arrive_remote(rb_xs_empty);
        if (tid == 0) A2_TRACE(11, k, j);
        bool grow = false;
        if (quad == 0) {                                // warps 0 and 4 own heads hb + lane
          const int h = hb + lane;
          const float bm = fmaxf(fmaxf(s.red[0][h], s.red[1][h]), fmaxf(s.red[2][h], s.red[3][h]));
          const float mo = s.mcur[h];
          float mn = mo, f = 1.f;
          if (mo == -INFINITY) {
            mn = bm;
            f = 0.f;
          } else if (bm > mo + TAU2) {
            mn = bm;
            f = exp2f(mo - mn);
            grow = true;
          }
          s.mcur[h] = mn;
          s.fac[h] = f;
        }
        const bool rescale = bar_red_or2(2, A2_SOFT, grow) && j > 0;
        if (tid == 0) A2_TRACE(12, k, j);
        // the single P buffer: GEMM2 of the previous block must have read it
        if (j > 0) {
          ok = tc::mbar_wait(&s.o_blk[(G - 1) & 1], ((G - 1) >> 1) & 1, spin, abort);
          ok = !bar_red_or2(3, A2_SOFT, !ok);
          if (!ok) break;
        }
        if (tid == 0) A2_TRACE(14, k, j);
        uint32_t packed[16];
#pragma unroll
        for (int h = 0; h < 32; h += 2) {
          const float m0 = s.mcur[hb + h], m1 = s.mcur[hb + h + 1];
          const float p0 = exp2f(z[h] - (m0 == -INFINITY ? 0.f : m0));
          const float p1 = exp2f(z[h + 1] - (m1 == -INFINITY ? 0.f : m1));
          __nv_bfloat162 pb2 = __floats2bfloat162_rn(p0, p1);
          const float2 pr = __bfloat1622float2(pb2);
          lsum[h] = fmaf(lsum[h], s.fac[hb + h], pr.x);
          lsum[h + 1] = fmaf(lsum[h + 1], s.fac[hb + h + 1], pr.y);
          packed[h / 2] = *reinterpret_cast<uint32_t*>(&pb2);
        }
        uint8_t* prow = s.p + slot * 128;
#pragma unroll
        for (int c = 0; c < 4; ++c)
          *reinterpret_cast<uint4*>(prow + (((4 * half + c) ^ (slot & 7)) << 4)) =
              make_uint4(packed[4 * c], packed[4 * c + 1], packed[4 * c + 2], packed[4 * c + 3]);
        if (rescale) {
          tc::tc_fence_after();
#pragma unroll
          for (int q = 0; q < 2; ++q) {
            float o[32];
            const uint32_t addr = tmem + lane_base + T2_O + 64 * q + hb;
            tc::tmem_ld32(addr, o);
            tc::tmem_wait_ld();
#pragma unroll
            for (int u = 0; u < 32; ++u) o[u] *= s.fac[hb + u];
            tc::tmem_st32(addr, o);
          }
          tc::tmem_wait_st();
        }
        tc::fence_proxy_async_smem();
        tc::tc_fence_before();
        tc::mbar_arrive(&s.p_full);
        if (tid == 0) A2_TRACE(17, k, j);
      }
      if (!ok) break;
      // ---------------------------------------------------------------- epilogue
      // GEMM2 of the item's last block (hence every earlier one) is complete. One barrier per
      // S/KV parity keeps the waited phase unambiguous: GEMM1 of block G completing implies
      // GEMM2 of block G-2 completed (issued before it).
      ok = tc::mbar_wait(&s.o_blk[(G - 1) & 1], ((G - 1) >> 1) & 1, spin, abort);
      ok = !bar_red_or2(3, A2_SOFT, !ok);
      if (!ok) break;
      if (tid == 0) A2_TRACE(20, k, 0);
      tc::tc_fence_after();
      s.red[quad][hb + lane] = xpose_reduce32<false>(lsum);
      tc::named_barrier(1, A2_SOFT);
      const int h0 = it.hg * A2_H;
      if (quad == 0) {
        const int h = hb + lane;
        const float L = (s.red[0][h] + s.red[1][h]) + (s.red[2][h] + s.red[3][h]);
        const float m = s.mcur[h];
        const float s2 = a.sink ? a.sink[h0 + h] * LOG2E2 : -INFINITY;
        const float mf = fmaxf(m, s2);
        const float em = m == -INFINITY ? 0.f : exp2f(m - mf);
        const float den = L * em + (a.sink ? exp2f(s2 - mf) : 0.f);
        float inv = 0.f, lse = -INFINITY;
        if (den > 0.f && mf != -INFINITY) {
          inv = em / den;
          lse = (mf + log2f(den)) * LN2_2;
        }
        s.inv[h] = inv;
        if (a.lse && (int)rank == half) a.lse[(long long)it.qi * a.H + h0 + h] = lse;
        s.mcur[h] = -INFINITY;                          // the next item starts fresh
      }
      tc::named_barrier(1, A2_SOFT);
      // O^T tiles -> bf16 [64 heads][128 channels] staging in the P buffer -> 16-byte stores
      __nv_bfloat16* stage = reinterpret_cast<__nv_bfloat16*>(s.p);
      __nv_bfloat16* O = reinterpret_cast<__nv_bfloat16*>(a.O) + ((long long)it.qi * a.H + h0) * A2_C +
                         (int)rank * A2_CH;
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        float o[32];
        tc::tmem_ld32(tmem + lane_base + T2_O + 64 * q + hb, o);
        tc::tmem_wait_ld();
#pragma unroll
        for (int u = 0; u < 32; ++u)
          stage[(hb + u) * A2_BLK + slot] = __float2bfloat16_rn(o[u] * s.inv[hb + u]);
        tc::named_barrier(1, A2_SOFT);
#pragma unroll
        for (int e = tid; e < A2_H * A2_BLK / 8; e += A2_SOFT) {
          const int h = e >> 4, c8 = e & 15;
          *reinterpret_cast<uint4*>(O + (long long)h * A2_C + 128 * q + 8 * c8) =
              *reinterpret_cast<const uint4*>(stage + h * A2_BLK + 8 * c8);
        }
        tc::named_barrier(1, A2_SOFT);
      }
      tc::tc_fence_before();
      if (tid == 0) A2_TRACE(23, k, 0);
    }
  }
  tc::tc_fence_before();
  __syncthreads();
  cluster_sync();                       // no remote access may target an exited peer
  if (warp == 11) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, T2_COLS);
  }
}

}  // namespace

// Returns DSV4_OK with *used = false when the shape or the device does not fit this kernel.
int launch_attn_tc2(const AttnArgs& a, cudaStream_t st, bool* used) {
  *used = false;
  // the single-CTA kernel is the default; DSV4_ATTN_CLUSTER=1 selects this one
  const char* on = std::getenv("DSV4_ATTN_CLUSTER");
  if (!on || on[0] != '1') return DSV4_OK;
  const char* force = std::getenv("DSV4_FORCE_SIMT");
  if (force && force[0] == '1') return DSV4_OK;
  if (a.c != A2_C || a.H % A2_H != 0) return DSV4_OK;
  if (!aligned16(a.Q) || !aligned16(a.local) || (a.pool && !aligned16(a.pool))) return DSV4_OK;
  const long long nrows_q = (long long)a.B * a.nq * a.H;
  const long long items = (long long)a.B * a.nq * (a.H / A2_H);
  if (nrows_q >= (1ll << 31) || items >= (1ll << 31)) return DSV4_OK;
  static int max_clusters = -1;
  if (max_clusters < 0) {
    cudaError_t e = cudaFuncSetAttribute(attn_tc2_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)A2_SMEM);
    if (e != cudaSuccess) return fail(DSV4_ERR_CUDA, "attn_tc2: %s", cudaGetErrorString(e));
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2, 1, 1);
    cfg.blockDim = dim3(A2_THREADS, 1, 1);
    cfg.dynamicSmemBytes = A2_SMEM;
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeClusterDimension;
    attr.val.clusterDim.x = 2;
    attr.val.clusterDim.y = 1;
    attr.val.clusterDim.z = 1;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    int n = 0;
    e = cudaOccupancyMaxActiveClusters(&n, attn_tc2_kernel, &cfg);
    const char* verbose = std::getenv("DSV4_VERBOSE");
    if (verbose && verbose[0] == '1')
      std::fprintf(stderr, "[dsv4] cluster attention: %d co-resident clusters (%s)\n", n,
                   cudaGetErrorString(e));
    if (e != cudaSuccess) {
      cudaGetLastError();
      n = 0;
    }
    int per_sm = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, attn_tc2_kernel, A2_THREADS, A2_SMEM);
    if (verbose && verbose[0] == '1')
      std::fprintf(stderr, "[dsv4] cluster attention: %d CTAs per SM (%s)\n", per_sm,
                   cudaGetErrorString(e));
    const char* force_n = std::getenv("DSV4_CLUSTERS");
    if (force_n && std::atoi(force_n) > 0) n = std::atoi(force_n);
    max_clusters = n;
  }
  if (max_clusters <= 0) return DSV4_OK;
  CUtensorMap mq;
  int s = encode_tensor_map_2d(&mq, a.Q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, A2_C, nrows_q, 64,
                               A2_H, CU_TENSOR_MAP_SWIZZLE_128B);
  if (s != DSV4_OK) return s;
  const long long nclusters = items < max_clusters ? items : max_clusters;
  attn_tc2_kernel<<<(unsigned)(2 * nclusters), A2_THREADS, A2_SMEM, st>>>(
      a, mq, a.H / A2_H, (int)items, a.scale * LOG2E2, spin_limit());
  *used = true;
  return launch_status("hybrid attention (tensor cores, 2-CTA cluster)");
}

}  // namespace dsv4

#ifdef DSV4_TRACE
extern "C" int dsv4_trace_read_attn(unsigned long long* host, size_t n) {
  return cudaMemcpyFromSymbol(host, dsv4::g_attn_trace, n * sizeof(unsigned long long)) == cudaSuccess ? 0 : 3;
}
#endif
