// Hybrid shared-KV MQA on the 5th-generation tensor cores, channel-split over a 2-CTA
// cluster, persistent.
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
//   exchange over DSMEM: CTA r owns heads [32r, 32r+32); it sends the peer its partial for
//          the peer's heads and adds the peer's partial for its own heads
//   softmax for the 32 owned heads (block max, conditional rescale, exp2), P^T columns of
//          those heads written to both CTAs' shared memory; rescale factors exchanged
//   GEMM2  O_r^T[256 channels x 64 heads] += KV_r^T . P^T                             (full)
// Both GEMMs use M = 128 (full tensor-core rate): slots for GEMM1, channels for GEMM2. The
// same swizzled KV stage is the K-major A operand of GEMM1 and the MN-major A of GEMM2.
// GEMM1 of block j+1 overlaps the softmax of block j (two S buffers, two KV stages).
//
// Warps: 0-3 softmax/epilogue (thread t = TMEM lane t), 4 producer (Q by 2D TMA, rows by
// TMA row gather), 5 MMA issuer and TMEM owner. Every wait is bounded; a cluster barrier at
// the end keeps both CTAs alive until neither can touch the other's shared memory.
#include <cstdlib>

#include "attn_common.cuh"
#include "tc_common.cuh"

namespace dsv4 {
namespace {

constexpr int A2_C = 512;               // channels of a row
constexpr int A2_CH = 256;              // channels per CTA
constexpr int A2_H = 64;                // heads per item
constexpr int A2_HO = 32;               // heads owned per CTA
constexpr int A2_BLK = 128;             // candidate slots per block
constexpr int A2_KCH = A2_CH / 64;      // 64-channel chunks per CTA
constexpr int A2_THREADS = 192;
constexpr uint32_t T2_S = 0;            // S buffers at columns 0 and 64
constexpr uint32_t T2_O = 128;          // O^T tiles at 128 + 64 q
constexpr uint32_t T2_COLS = 256;
constexpr float TAU2 = 8.f;
constexpr float LOG2E2 = 1.4426950408889634f;
constexpr float LN2_2 = 0.6931471805599453f;

struct Smem2 {
  uint8_t q[A2_KCH][A2_H * 128];              // 32 KiB
  uint8_t kv[2][A2_KCH][A2_BLK * 128];        // 128 KiB
  uint8_t p[2][A2_BLK * 128];                 // 32 KiB, P^T [slots][64 heads], MN-major SW128
  float xs[2][A2_BLK][A2_HO];                 // 32 KiB, peer's partial S for my heads
  float red[4][A2_HO];
  float mcur[A2_HO];
  float fac[2][A2_H];
  float inv[2][A2_H];
  uint64_t q_full, q_empty;
  uint64_t kv_full[2], kv_empty[2];
  uint64_t s_full[2], xs_full[2], fac_full[2], p_full[2];
  uint64_t o_blk[2], inv_full[2], drain;
  uint32_t tmem_base;
  int abort;
};
constexpr size_t A2_SMEM = sizeof(Smem2) + 1024;
static_assert(A2_SMEM <= 232448, "shared memory of the cluster attention kernel");

#ifdef DSV4_TRACE
// Phase timestamps (clock64) of cluster 0, first 4 items, first 8 blocks: a profiling aid
// compiled only into traced builds.
__device__ unsigned long long g_attn_trace[2][4][8][32];
#define A2_TRACE(ev, k_, j_)                                                   \
  do {                                                                         \
    if (cluster_id == 0 && (k_) < 4 && (j_) < 8)                               \
      g_attn_trace[rank][k_][j_][ev] = clock64();                              \
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
__device__ __forceinline__ void st_remote_v4(uint32_t addr, uint4 v) {
  asm volatile("st.shared::cluster.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y),
               "r"(v.z), "r"(v.w)
               : "memory");
}
__device__ __forceinline__ void st_remote_f32(uint32_t addr, float v) {
  asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(addr), "f"(v) : "memory");
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
__device__ __forceinline__ void fence_proxy_async_all() {
  asm volatile("fence.proxy.async;" ::: "memory");
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

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(A2_THREADS, 1)
    attn_tc2_kernel(const AttnArgs a, const __grid_constant__ CUtensorMap map_q,
                    const __grid_constant__ CUtensorMap map_pool,
                    const __grid_constant__ CUtensorMap map_local, int head_groups, int items,
                    float scale_log2, uint32_t spin) {
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
      tc::mbar_init(&s.kv_full[i], 1);
      tc::mbar_init(&s.kv_empty[i], 1);
      tc::mbar_init(&s.s_full[i], 1);
      tc::mbar_init(&s.xs_full[i], 128);
      tc::mbar_init(&s.fac_full[i], 128);
      tc::mbar_init(&s.p_full[i], 256);
      tc::mbar_init(&s.inv_full[i], 128);
    }
    tc::mbar_init(&s.o_blk[0], 1);
    tc::mbar_init(&s.o_blk[1], 1);
    tc::mbar_init(&s.drain, 1);
    s.abort = 0;
    tc::fence_barrier_init();
  }
  if (tid < A2_HO) s.mcur[tid] = -INFINITY;
  if (warp == 5) {
    tc::tmem_alloc(&s.tmem_base, T2_COLS);
    tc::tmem_relinquish();
  }
  tc::tc_fence_before();
  __syncthreads();
  cluster_sync();                       // the peer's barriers exist before any remote arrive
  tc::tc_fence_after();
  const uint32_t tmem = s.tmem_base;

  if (warp == 4) {
    // ------------------------------------------------------------------ producer
    int issued[2] = {0, 0};
    int q_issued = 0;
    if (lane == 0) {
      tc::prefetch_tensormap(&map_q);
      tc::prefetch_tensormap(&map_pool);
      tc::prefetch_tensormap(&map_local);
    }
    uint32_t G = 0;
    int k = 0;
    bool ok = true;
    for (int item = cluster_id; item < items && ok; item += nclusters, ++k) {
      const ItemInfo it = item_info(a, item, head_groups);
      if (lane == 0) {
        if (k > 0) ok = tc::mbar_wait(&s.q_empty, (uint32_t)((k - 1) & 1), spin, abort);
        if (ok) {
          tc::mbar_arrive_expect_tx(&s.q_full, A2_KCH * A2_H * 128);
          const int qrow = it.qi * a.H + it.hg * A2_H;
          for (int c = 0; c < A2_KCH; ++c)
            tc::tma_load_2d(s.q[c], &map_q, &s.q_full, (int)rank * A2_CH + 64 * c, qrow);
          q_issued = k + 1;
        }
      }
      ok = __shfl_sync(0xffffffffu, (int)ok, 0) != 0;
      for (int j = 0; j < it.nb && ok; ++j, ++G) {
        const int st = G & 1;
        Slot r[4];
        bool any_valid = false, bad = false;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          r[u] = slot_of(a, it.cs, it.nc4, j * A2_BLK + 4 * lane + u);
          any_valid |= r[u].valid;
          bad |= r[u].bad;
        }
        if (bad && rank == 0) flag_status(DSV4_ERR_DEVICE_BOUNDS);
        const CUtensorMap* map = &map_local;
        int32_t y[4];
        if (r[0].part == 0 && any_valid) {
          map = &map_pool;
          long long fill = 0;
#pragma unroll
          for (int u = 3; u >= 0; --u)
            if (r[u].valid) fill = r[u].row;
#pragma unroll
          for (int u = 0; u < 4; ++u) y[u] = (int32_t)(r[u].valid ? r[u].row : fill);
        } else {
#pragma unroll
          for (int u = 0; u < 4; ++u)
            y[u] = (int32_t)(r[u].part == 1 ? r[u].row : it.cs.local_base);
        }
        int w_ok = 1;
        if (lane == 0 && G >= 2) w_ok = tc::mbar_wait(&s.kv_empty[st], ((G >> 1) - 1) & 1, spin, abort);
        if (lane == 0) A2_TRACE(0, k, j);
        ok = __shfl_sync(0xffffffffu, w_ok, 0) != 0;
        if (!ok) break;
        if (lane == 0) tc::mbar_arrive_expect_tx(&s.kv_full[st], A2_KCH * A2_BLK * 128);
        __syncwarp();
#pragma unroll
        for (int c = 0; c < A2_KCH; ++c)
          tc::tma_gather4(s.kv[st][c] + 4 * lane * 128, map, &s.kv_full[st],
                          (int)rank * A2_CH + 64 * c, y[0], y[1], y[2], y[3]);
        if (lane == 0) A2_TRACE(1, k, j);
        issued[st] = (int)(G >> 1) + 1;
      }
    }
    if (*abort) {
      volatile int never = 0;
      for (int st = 0; st < 2; ++st)
        if (issued[st] > 0) tc::mbar_wait(&s.kv_full[st], (uint32_t)((issued[st] - 1) & 1), spin, &never);
      if (lane == 0 && q_issued > 0) tc::mbar_wait(&s.q_full, (uint32_t)((q_issued - 1) & 1), spin, &never);
    }
  } else if (warp == 5) {
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
        A2_TRACE(25, k, 0);
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
          ok = wait_cluster(&s.p_full[st], (G >> 1) & 1, spin, abort);
          A2_TRACE(4, k, j);
          if (!ok) break;
          tc::tc_fence_after();
          const uint32_t pb = tc::smem_u32(s.p[st]);
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
    const uint32_t lane_base = (uint32_t)(32 * warp) << 16;
    const uint32_t r_xs[2] = {mapa(tc::smem_u32(&s.xs[0][tid][0]), peer),
                              mapa(tc::smem_u32(&s.xs[1][tid][0]), peer)};
    const uint32_t r_p[2] = {mapa(tc::smem_u32(s.p[0] + tid * 128), peer),
                             mapa(tc::smem_u32(s.p[1] + tid * 128), peer)};
    const uint32_t r_fac[2] = {mapa(tc::smem_u32(&s.fac[0][0]), peer),
                               mapa(tc::smem_u32(&s.fac[1][0]), peer)};
    const uint32_t r_inv[2] = {mapa(tc::smem_u32(&s.inv[0][0]), peer),
                               mapa(tc::smem_u32(&s.inv[1][0]), peer)};
    const uint32_t rb_xs[2] = {mapa(tc::smem_u32(&s.xs_full[0]), peer),
                               mapa(tc::smem_u32(&s.xs_full[1]), peer)};
    const uint32_t rb_fac[2] = {mapa(tc::smem_u32(&s.fac_full[0]), peer),
                                mapa(tc::smem_u32(&s.fac_full[1]), peer)};
    const uint32_t rb_p[2] = {mapa(tc::smem_u32(&s.p_full[0]), peer),
                              mapa(tc::smem_u32(&s.p_full[1]), peer)};
    const uint32_t rb_inv[2] = {mapa(tc::smem_u32(&s.inv_full[0]), peer),
                                mapa(tc::smem_u32(&s.inv_full[1]), peer)};
    const int own0 = A2_HO * (int)rank, peer0 = A2_HO * (int)peer;
    uint32_t G = 0;
    int k = 0;
    bool ok = true;
    for (int item = cluster_id; item < items && ok; item += nclusters, ++k) {
      const ItemInfo it = item_info(a, item, head_groups);
      float l_part[A2_HO], l32[A2_HO];   // sums of bf16-rounded / exact probabilities
#pragma unroll
      for (int h = 0; h < A2_HO; ++h) l_part[h] = l32[h] = 0.f;
      for (int j = 0; j < it.nb; ++j, ++G) {
        const int st = G & 1;
        const uint32_t par = (G >> 1) & 1;
        const Slot sl = slot_of(a, it.cs, it.nc4, j * A2_BLK + tid);   // load overlaps the wait
        if (tid == 0) A2_TRACE(6, k, j);
        ok = tc::mbar_wait(&s.s_full[st], par, spin, abort);
        if (tid == 0) A2_TRACE(7, k, j);
        ok = !bar_red_or2(3, 128, !ok);
        if (!ok) break;
        tc::tc_fence_after();
        float vo[A2_HO], vp[A2_HO];            // partial S: owned heads, peer's heads
        tc::tmem_ld32(tmem + lane_base + T2_S + 64 * st + own0, vo);
        tc::tmem_ld32(tmem + lane_base + T2_S + 64 * st + peer0, vp);
        tc::tmem_wait_ld();
        // the peer's heads -> peer.xs[st][tid][*] (16-byte chunk c at c ^ (tid & 7))
#pragma unroll
        for (int c = 0; c < 8; ++c)
          st_remote_v4(r_xs[st] + 16 * (c ^ (tid & 7)),
                       make_uint4(__float_as_uint(vp[4 * c]), __float_as_uint(vp[4 * c + 1]),
                                  __float_as_uint(vp[4 * c + 2]), __float_as_uint(vp[4 * c + 3])));
        arrive_remote(rb_xs[st]);
        if (tid == 0) A2_TRACE(9, k, j);
        ok = wait_cluster(&s.xs_full[st], par, spin, abort);
        if (tid == 0) A2_TRACE(10, k, j);
        ok = !bar_red_or2(3, 128, !ok);
        if (!ok) break;
        float z[A2_HO];
        const float* xr = s.xs[st][tid];
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const float4 x4 = *reinterpret_cast<const float4*>(xr + 4 * (c ^ (tid & 7)));
          z[4 * c] = sl.valid ? (vo[4 * c] + x4.x) * scale_log2 : -INFINITY;
          z[4 * c + 1] = sl.valid ? (vo[4 * c + 1] + x4.y) * scale_log2 : -INFINITY;
          z[4 * c + 2] = sl.valid ? (vo[4 * c + 2] + x4.z) * scale_log2 : -INFINITY;
          z[4 * c + 3] = sl.valid ? (vo[4 * c + 3] + x4.w) * scale_log2 : -INFINITY;
        }
        float red[A2_HO];
#pragma unroll
        for (int h = 0; h < A2_HO; ++h) red[h] = z[h];
        s.red[warp][lane] = xpose_reduce32<true>(red);
        tc::named_barrier(1, 128);
        if (tid == 0) A2_TRACE(11, k, j);
        if (tid < A2_HO) {
          const float bm = fmaxf(fmaxf(s.red[0][tid], s.red[1][tid]), fmaxf(s.red[2][tid], s.red[3][tid]));
          const float mo = s.mcur[tid];
          float mn = mo, f = 1.f;
          if (mo == -INFINITY) {
            mn = bm;
            f = 0.f;
          } else if (bm > mo + TAU2) {
            mn = bm;
            f = exp2f(mo - mn);
          }
          s.mcur[tid] = mn;
          s.fac[st][own0 + tid] = f;
          st_remote_f32(r_fac[st] + 4 * (own0 + tid), f);
        }
        tc::named_barrier(1, 128);
        arrive_remote(rb_fac[st]);
        if (tid == 0) A2_TRACE(12, k, j);
        // probabilities of the owned heads, P^T columns to both CTAs
        uint32_t packed[A2_HO / 2];
#pragma unroll
        for (int h = 0; h < A2_HO; h += 2) {
          const float m0 = s.mcur[h], m1 = s.mcur[h + 1];
          const float p0 = exp2f(z[h] - (m0 == -INFINITY ? 0.f : m0));
          const float p1 = exp2f(z[h + 1] - (m1 == -INFINITY ? 0.f : m1));
          __nv_bfloat162 pb2 = __floats2bfloat162_rn(p0, p1);
          const float2 pr = __bfloat1622float2(pb2);
          const float f0 = s.fac[st][own0 + h], f1 = s.fac[st][own0 + h + 1];
          l_part[h] = fmaf(l_part[h], f0, pr.x);
          l_part[h + 1] = fmaf(l_part[h + 1], f1, pr.y);
          l32[h] = fmaf(l32[h], f0, p0);
          l32[h + 1] = fmaf(l32[h + 1], f1, p1);
          packed[h / 2] = *reinterpret_cast<uint32_t*>(&pb2);
        }
        uint8_t* prow = s.p[st] + tid * 128;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const uint32_t off = (uint32_t)(((4 * (int)rank + c) ^ (tid & 7)) << 4);
          const uint4 val = make_uint4(packed[4 * c], packed[4 * c + 1], packed[4 * c + 2], packed[4 * c + 3]);
          *reinterpret_cast<uint4*>(prow + off) = val;
          st_remote_v4(r_p[st] + off, val);
        }
        ok = wait_cluster(&s.fac_full[st], par, spin, abort);
        if (tid == 0) A2_TRACE(14, k, j);
        ok = !bar_red_or2(3, 128, !ok);
        if (!ok) break;
        // rescale O^T (all 64 heads of this CTA's channels) when any head's max grew
        bool any = false;
#pragma unroll
        for (int h = 0; h < A2_H; ++h) any |= (s.fac[st][h] != 1.f);
        if (any && j > 0) {
          // GEMM2 of the previous block must be done (its buffer's barrier, see below)
          ok = tc::mbar_wait(&s.o_blk[(G - 1) & 1], ((G - 1) >> 1) & 1, spin, abort);
          ok = !bar_red_or2(3, 128, !ok);
          if (!ok) break;
          tc::tc_fence_after();
#pragma unroll
          for (int q = 0; q < 2; ++q) {
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
              float o[32];
              const uint32_t addr = tmem + lane_base + T2_O + 64 * q + 32 * hh;
              tc::tmem_ld32(addr, o);
              tc::tmem_wait_ld();
#pragma unroll
              for (int u = 0; u < 32; ++u) o[u] *= s.fac[st][32 * hh + u];
              tc::tmem_st32(addr, o);
            }
          }
          tc::tmem_wait_st();
        }
        fence_proxy_async_all();
        if (tid == 0) A2_TRACE(16, k, j);
        tc::tc_fence_before();
        tc::mbar_arrive(&s.p_full[st]);
        arrive_remote(rb_p[st]);
        if (tid == 0) A2_TRACE(17, k, j);
      }
      if (!ok) break;
      // ---------------------------------------------------------------- epilogue
      // GEMM2 of the item's last block (hence every earlier one) is complete. One barrier per
      // S/KV parity keeps the phase of the waited GEMM2 unambiguous: GEMM1 of block G
      // completing implies GEMM2 of block G-2 completed (issued before it).
      ok = tc::mbar_wait(&s.o_blk[(G - 1) & 1], ((G - 1) >> 1) & 1, spin, abort);
      ok = !bar_red_or2(3, 128, !ok);
      if (tid == 0) A2_TRACE(20, k, 0);
      if (!ok) break;
      tc::tc_fence_after();
      // O is normalised by the sum of the same bf16 weights the PV product used; the LSE
      // uses the sum of the exact fp32 weights.
      s.red[warp][lane] = xpose_reduce32<false>(l32);
      tc::named_barrier(1, 128);
      float L32 = 0.f;
      if (tid < A2_HO) L32 = (s.red[0][tid] + s.red[1][tid]) + (s.red[2][tid] + s.red[3][tid]);
      tc::named_barrier(1, 128);
      s.red[warp][lane] = xpose_reduce32<false>(l_part);
      tc::named_barrier(1, 128);
      const int kb = k & 1;
      const int h0 = it.hg * A2_H;
      if (tid < A2_HO) {
        const float L = (s.red[0][tid] + s.red[1][tid]) + (s.red[2][tid] + s.red[3][tid]);
        const float m = s.mcur[tid];
        const int hgl = h0 + own0 + tid;
        const float s2 = a.sink ? a.sink[hgl] * LOG2E2 : -INFINITY;
        const float mf = fmaxf(m, s2);
        const float sk = a.sink ? exp2f(s2 - mf) : 0.f;
        const float em = m == -INFINITY ? 0.f : exp2f(m - mf);
        const float den = L * em + sk;
        const float den32 = L32 * em + sk;
        float inv = 0.f, lse = -INFINITY;
        if (den > 0.f && mf != -INFINITY) {
          inv = em / den;
          lse = (mf + log2f(den32)) * LN2_2;
        }
        s.inv[kb][own0 + tid] = inv;
        st_remote_f32(r_inv[kb] + 4 * (own0 + tid), inv);
        if (a.lse) a.lse[(long long)it.qi * a.H + hgl] = lse;
        s.mcur[tid] = -INFINITY;                    // next item starts fresh
      }
      tc::named_barrier(1, 128);
      arrive_remote(rb_inv[kb]);
      ok = wait_cluster(&s.inv_full[kb], (uint32_t)((k >> 1) & 1), spin, abort);
      if (tid == 0) A2_TRACE(22, k, 0);
      ok = !bar_red_or2(3, 128, !ok);
      if (!ok) break;
      __nv_bfloat16* O = reinterpret_cast<__nv_bfloat16*>(a.O) + ((long long)it.qi * a.H + h0) * A2_C +
                         (int)rank * A2_CH;
#pragma unroll
      for (int q = 0; q < 2; ++q) {
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          float o[32];
          tc::tmem_ld32(tmem + lane_base + T2_O + 64 * q + 32 * hh, o);
          tc::tmem_wait_ld();
#pragma unroll
          for (int u = 0; u < 32; ++u) {
            const int h = 32 * hh + u;
            O[(long long)h * A2_C + 128 * q + tid] = __float2bfloat16_rn(o[u] * s.inv[kb][h]);
          }
        }
      }
      if (tid == 0) A2_TRACE(23, k, 0);
      tc::tc_fence_before();
    }
  }
  tc::tc_fence_before();
  __syncthreads();
  cluster_sync();                       // no remote access may target an exited peer
  if (warp == 5) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, T2_COLS);
  }
}

}  // namespace

// Returns DSV4_OK with *used = false when the shape or the device does not fit this kernel.
int launch_attn_tc2(const AttnArgs& a, cudaStream_t st, bool* used) {
  *used = false;
  const char* off = std::getenv("DSV4_ATTN_V1");
  if (off && off[0] == '1') return DSV4_OK;
  const char* force = std::getenv("DSV4_FORCE_SIMT");
  if (force && force[0] == '1') return DSV4_OK;
  if (a.c != A2_C || a.H % A2_H != 0) return DSV4_OK;
  if (!aligned16(a.Q) || !aligned16(a.local) || (a.pool && !aligned16(a.pool))) return DSV4_OK;
  const long long nrows_q = (long long)a.B * a.nq * a.H;
  const long long nrows_local = (long long)a.B * a.R;
  const long long items = (long long)a.B * a.nq * (a.H / A2_H);
  if (nrows_q >= (1ll << 31) || nrows_local >= (1ll << 31) || a.pool_rows >= (1ll << 31) ||
      items >= (1ll << 31))
    return DSV4_OK;
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
    if (e != cudaSuccess) {
      cudaGetLastError();
      n = 0;
    }
    max_clusters = n;
  }
  if (max_clusters <= 0) return DSV4_OK;
  CUtensorMap mq, mpool, mlocal;
  int s = encode_tensor_map_2d(&mq, a.Q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, A2_C, nrows_q, 64,
                               A2_H, CU_TENSOR_MAP_SWIZZLE_128B);
  if (s != DSV4_OK) return s;
  s = encode_tensor_map_2d(&mlocal, a.local, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, A2_C,
                           nrows_local, 64, 1, CU_TENSOR_MAP_SWIZZLE_128B);
  if (s != DSV4_OK) return s;
  if (a.pool && a.pool_rows > 0)
    s = encode_tensor_map_2d(&mpool, a.pool, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, A2_C,
                             a.pool_rows, 64, 1, CU_TENSOR_MAP_SWIZZLE_128B);
  else
    mpool = mlocal;
  if (s != DSV4_OK) return s;
  const long long nclusters = items < max_clusters ? items : max_clusters;
  attn_tc2_kernel<<<(unsigned)(2 * nclusters), A2_THREADS, A2_SMEM, st>>>(
      a, mq, mpool, mlocal, a.H / A2_H, (int)items, a.scale * LOG2E2, spin_limit());
  *used = true;
  return launch_status("hybrid attention (tensor cores, 2-CTA cluster)");
}

}  // namespace dsv4

#ifdef DSV4_TRACE
extern "C" int dsv4_trace_read_attn(unsigned long long* host, size_t n) {
  return cudaMemcpyFromSymbol(host, dsv4::g_attn_trace, n * sizeof(unsigned long long)) == cudaSuccess ? 0 : 3;
}
#endif
