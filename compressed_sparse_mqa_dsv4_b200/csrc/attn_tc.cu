// Hybrid shared-KV MQA on the 5th-generation tensor cores (tcgen05 + TMEM + TMA gather).
//
// "CSA And HCA: Definition, State, And Cost Model": s3.2/s4 every candidate row is both
// key and value for all heads; s5.1 one candidate list (selected or all completed
// compressed entries, then the local window) under one softmax per head; s5.3 the sink
// logit joins the denominator only. Per-query valid counts follow pypto-lib PR #834.
//
// Because all heads share each KV row, the contraction for one query is dense with the
// candidates as one MMA dimension. The kernel uses the transposed form so that the MMA M
// dimension is 128 candidate slots (full tensor-core rate) and N is 64 heads:
//   GEMM1  S^T[128 slots x 64 heads] = KV[slots x c] . Q[heads x c]^T     (K = c = 512)
//   GEMM2  O^T[c x 64 heads]        += KV^T[c x slots] . P^T[slots x heads] (K = 128)
// The same shared-memory KV tile is the K-major A operand of GEMM1 and the MN-major A
// operand of GEMM2 (128-byte swizzle atoms of 8 slots x 64 channels). O^T lives in TMEM
// for the whole query (4 M-tiles x 64 columns); S^T takes 64 more columns.
//
// One CTA per (query, group of 64 heads), 6 warps:
//   warps 0-3  softmax + epilogue: thread t owns TMEM lane t (slot t of S^T, channel row t
//              of each O^T tile); per-head block maxima by a transposing butterfly over
//              the warp plus a 4-warp exchange; conditional rescaling of O^T (only when a
//              head's max grows by more than 2^8); P^T written to shared memory as bf16.
//   warp 4     producer: Q by 2D TMA, candidate rows by TMA row gather (4 rows per
//              instruction) per 64-channel chunk, with per-chunk full/empty mbarriers.
//   warp 5     MMA issuer (one thread) and TMEM owner.
// Candidate slots: [0, round4(n_comp)) compressed, then round4(n_local) local; slots past
// a part's count are masked (p = 0) and fetch an in-range row, so every value is finite.
// All waits are bounded (see tc_common.cuh).
#include <cstdlib>

#include "attn_common.cuh"
#include "tc_common.cuh"

namespace dsv4 {
namespace {

constexpr int AT_C = 512;
constexpr int AT_H = 64;
constexpr int AT_BLK = 128;
constexpr int AT_CHUNKS = AT_C / 64;
constexpr int AT_THREADS = 192;
constexpr uint32_t TM_S = 0;
constexpr uint32_t TM_O = 64;
constexpr uint32_t TM_COLS = 512;
constexpr float TAU = 8.f;                  // log2-domain growth tolerated before rescaling
constexpr float LOG2E = 1.4426950408889634f;
constexpr float LN2 = 0.6931471805599453f;

struct AttnSmem {
  uint8_t q[AT_CHUNKS][AT_H * 128];         // K-major SW128: [64 heads][64 ch] per chunk
  uint8_t kv[AT_CHUNKS][AT_BLK * 128];      // [128 slots][64 ch] per chunk
  uint8_t p[AT_BLK * 128];                  // MN-major SW128: [128 slots][64 heads]
  float red[4][AT_H];
  float mcur[AT_H];
  float fac[AT_H];
  float inv[AT_H];
  uint64_t q_full;
  uint64_t kv_full[AT_CHUNKS];
  uint64_t kv_empty[4];
  uint64_t s_full, p_full, o_done;
  uint32_t tmem_base;
  int abort;
};
constexpr size_t AT_SMEM = sizeof(AttnSmem) + 1024;

__device__ __forceinline__ float fmax_op(float a, float b) { return fmaxf(a, b); }
__device__ __forceinline__ float fadd_op(float a, float b) { return a + b; }

// Transposing butterfly: reduces 64 per-lane values across the 32 lanes of a warp; lane L
// ends with the reductions of heads 2L (v[0]) and 2L+1 (v[1]).
template <bool MAX>
__device__ __forceinline__ void xpose_reduce64(float (&v)[64]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int step = 0; step < 5; ++step) {
    const int half = 32 >> step;            // values kept after this step
    const int mask = 16 >> step;
    const bool up = (lane & mask) != 0;
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      if (i < half) {
        const float send = up ? v[i] : v[i + half];
        const float keep = up ? v[i + half] : v[i];
        const float recv = __shfl_xor_sync(0xffffffffu, send, mask);
        v[i] = MAX ? fmax_op(keep, recv) : fadd_op(keep, recv);
      }
    }
  }
}

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

__global__ void __launch_bounds__(AT_THREADS, 1)
    attn_tc_kernel(const AttnArgs a, const __grid_constant__ CUtensorMap map_q,
                   const __grid_constant__ CUtensorMap map_pool,
                   const __grid_constant__ CUtensorMap map_local, int head_groups,
                   float scale_log2, uint32_t spin) {
  extern __shared__ uint8_t smem_raw[];
  AttnSmem& s = *reinterpret_cast<AttnSmem*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int qi = blockIdx.x / head_groups;           // b * nq + i
  const int hg = blockIdx.x % head_groups;
  const int b = qi / a.nq, i = qi % a.nq;
  const CandidateSet cs = make_candidates(a, b, i);
  const int nc4 = (cs.n_comp + 3) & ~3;
  const int nl4 = (cs.n_local + 3) & ~3;
  const int nb = (nc4 + nl4 + AT_BLK - 1) / AT_BLK;
  volatile int* abort = &s.abort;

  if (tid == 0) {
    tc::mbar_init(&s.q_full, 1);
    for (int k = 0; k < AT_CHUNKS; ++k) tc::mbar_init(&s.kv_full[k], 1);
    for (int k = 0; k < 4; ++k) tc::mbar_init(&s.kv_empty[k], 1);
    tc::mbar_init(&s.s_full, 1);
    tc::mbar_init(&s.p_full, 128);
    tc::mbar_init(&s.o_done, 1);
    s.abort = 0;
    tc::fence_barrier_init();
  }
  if (tid < AT_H) s.mcur[tid] = -INFINITY;
  if (warp == 5) {
    tc::tmem_alloc(&s.tmem_base, TM_COLS);
    tc::tmem_relinquish();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = s.tmem_base;

  if (warp == 4) {
    // ------------------------------------------------------------------ producer
    int issued[AT_CHUNKS];
#pragma unroll
    for (int k = 0; k < AT_CHUNKS; ++k) issued[k] = 0;
    if (lane == 0) {
      tc::prefetch_tensormap(&map_q);
      tc::prefetch_tensormap(&map_pool);
      tc::prefetch_tensormap(&map_local);
      tc::mbar_arrive_expect_tx(&s.q_full, AT_CHUNKS * AT_H * 128);
      const int qrow = qi * a.H + hg * AT_H;
      for (int k = 0; k < AT_CHUNKS; ++k) tc::tma_load_2d(s.q[k], &map_q, &s.q_full, k * 64, qrow);
    }
    for (int j = 0; j < nb && !*abort; ++j) {
      // rows of this lane's group of 4 slots
      const int g0 = j * AT_BLK + 4 * lane;
      SlotRow r[4];
      bool any_valid = false, bad = false;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        r[u] = slot_row(a, cs, nc4, g0 + u);
        any_valid |= r[u].valid;
        bad |= r[u].bad_index;
      }
      if (bad) flag_status(DSV4_ERR_DEVICE_BOUNDS);
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
          y[u] = (int32_t)((r[u].part == 1) ? r[u].row : cs.local_base);
      }
      bool okw = true;
      for (int k = 0; k < AT_CHUNKS; ++k) {
        if (j > 0 && (k & 1) == 0) {
          int w_ok = 1;
          if (lane == 0) w_ok = tc::mbar_wait(&s.kv_empty[k >> 1], (uint32_t)((j - 1) & 1), spin, abort);
          okw = __shfl_sync(0xffffffffu, w_ok, 0) != 0;
          if (!okw) break;
        }
        if (lane == 0) tc::mbar_arrive_expect_tx(&s.kv_full[k], AT_BLK * 128);
        __syncwarp();
        tc::tma_gather4(s.kv[k] + 4 * lane * 128, map, &s.kv_full[k], k * 64, y[0], y[1], y[2],
                        y[3]);
        issued[k] = j + 1;
      }
      if (!okw) break;
    }
    if (*abort) {
      // drain this CTA's own loads before the shared memory can be released
      for (int k = 0; k < AT_CHUNKS; ++k)
        if (issued[k] > 0) {
          volatile int never = 0;
          tc::mbar_wait(&s.kv_full[k], (uint32_t)((issued[k] - 1) & 1), spin, &never);
        }
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t id1 = tc::idesc_bf16_f32(128, AT_H, 0, 0);   // A, B K-major
      const uint32_t id2 = tc::idesc_bf16_f32(128, AT_H, 1, 1);   // A, B MN-major
      bool ok = tc::mbar_wait(&s.q_full, 0, spin, abort);
      for (int j = 0; j < nb && ok; ++j) {
        for (int k = 0; k < AT_CHUNKS && ok; ++k) {
          ok = tc::mbar_wait(&s.kv_full[k], (uint32_t)(j & 1), spin, abort);
          if (!ok) break;
          tc::tc_fence_after();
          const uint32_t kvb = tc::smem_u32(s.kv[k]), qb = tc::smem_u32(s.q[k]);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            tc::mma_bf16_ss(tmem + TM_S, tc::sdesc_sw128(kvb + kk * 32, 16, 1024),
                            tc::sdesc_sw128(qb + kk * 32, 16, 1024), id1, (k | kk) != 0);
          }
        }
        if (!ok) break;
        tc::mma_commit(&s.s_full);
        ok = tc::mbar_wait(&s.p_full, (uint32_t)(j & 1), spin, abort);
        if (!ok) break;
        tc::tc_fence_after();
        const uint32_t pb = tc::smem_u32(s.p);
        for (int q = 0; q < 4; ++q) {
          const uint32_t kvb = tc::smem_u32(s.kv[2 * q]);
#pragma unroll
          for (int ks = 0; ks < AT_BLK / 16; ++ks) {
            tc::mma_bf16_ss(tmem + TM_O + 64 * q, tc::sdesc_sw128(kvb + ks * 2048, AT_BLK * 128, 1024),
                            tc::sdesc_sw128(pb + ks * 2048, AT_BLK * 128, 1024), id2,
                            (j > 0 || ks > 0) ? 1u : 0u);
          }
          tc::mma_commit(&s.kv_empty[q]);
        }
      }
      tc::mma_commit(&s.o_done);
      if (!ok) {
        volatile int never = 0;
        tc::mbar_wait(&s.o_done, 0, spin, &never);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------------ softmax warps
    const uint32_t lane_base = (uint32_t)(32 * warp) << 16;
    float l_part[AT_H];
#pragma unroll
    for (int h = 0; h < AT_H; ++h) l_part[h] = 0.f;
    bool ok = true;
    for (int j = 0; j < nb; ++j) {
      ok = tc::mbar_wait(&s.s_full, (uint32_t)(j & 1), spin, abort);
      ok = !bar_red_or(3, 128, !ok);          // all 128 threads take the same branch
      if (!ok) break;
      tc::tc_fence_after();
      float z[AT_H];
      {
        float t32[32];
        tc::tmem_ld32(tmem + lane_base + TM_S, t32);
#pragma unroll
        for (int h = 0; h < 32; ++h) z[h] = t32[h];
        tc::tmem_ld32(tmem + lane_base + TM_S + 32, t32);
#pragma unroll
        for (int h = 0; h < 32; ++h) z[32 + h] = t32[h];
        tc::tmem_wait_ld();
      }
      const SlotRow sr = slot_row(a, cs, nc4, j * AT_BLK + tid);
#pragma unroll
      for (int h = 0; h < AT_H; ++h) z[h] = sr.valid ? z[h] * scale_log2 : -INFINITY;
      float red[AT_H];
#pragma unroll
      for (int h = 0; h < AT_H; ++h) red[h] = z[h];
      xpose_reduce64<true>(red);
      s.red[warp][2 * lane] = red[0];
      s.red[warp][2 * lane + 1] = red[1];
      tc::named_barrier(1, 128);
      bool grow = false;
      if (tid < AT_H) {
        const float bm = fmaxf(fmaxf(s.red[0][tid], s.red[1][tid]), fmaxf(s.red[2][tid], s.red[3][tid]));
        const float mo = s.mcur[tid];
        float mn = mo, f = 1.f;
        if (mo == -INFINITY) {
          mn = bm;
          f = 0.f;
        } else if (bm > mo + TAU) {
          mn = bm;
          f = exp2f(mo - mn);
          grow = true;
        }
        s.mcur[tid] = mn;
        s.fac[tid] = f;
      }
      const bool rescale = bar_red_or(2, 128, grow) && j > 0;
      // probabilities, running partial sums, P^T row (bf16, 128-byte swizzle)
      uint32_t packed[AT_H / 2];
#pragma unroll
      for (int h = 0; h < AT_H; h += 2) {
        const float m0 = s.mcur[h], m1 = s.mcur[h + 1];
        const float p0 = exp2f(z[h] - (m0 == -INFINITY ? 0.f : m0));
        const float p1 = exp2f(z[h + 1] - (m1 == -INFINITY ? 0.f : m1));
        __nv_bfloat162 pb2 = __floats2bfloat162_rn(p0, p1);
        // the denominator sums the same bf16-rounded weights the PV product uses
        const float2 pr = __bfloat1622float2(pb2);
        l_part[h] = fmaf(l_part[h], s.fac[h], pr.x);
        l_part[h + 1] = fmaf(l_part[h + 1], s.fac[h + 1], pr.y);
        packed[h / 2] = *reinterpret_cast<uint32_t*>(&pb2);
      }
      uint8_t* prow = s.p + tid * 128;
#pragma unroll
      for (int c8 = 0; c8 < 8; ++c8) {
        *reinterpret_cast<uint4*>(prow + ((c8 ^ (tid & 7)) << 4)) =
            make_uint4(packed[4 * c8], packed[4 * c8 + 1], packed[4 * c8 + 2], packed[4 * c8 + 3]);
      }
      if (rescale) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            float v[32];
            const uint32_t addr = tmem + lane_base + TM_O + 64 * q + 32 * hh;
            tc::tmem_ld32(addr, v);
            tc::tmem_wait_ld();
#pragma unroll
            for (int u = 0; u < 32; ++u) v[u] *= s.fac[32 * hh + u];
            tc::tmem_st32(addr, v);
          }
        }
        tc::tmem_wait_st();
      }
      tc::fence_proxy_async_smem();
      tc::tc_fence_before();
      tc::mbar_arrive(&s.p_full);
    }
    // ---------------------------------------------------------------- epilogue
    if (ok) {
      ok = tc::mbar_wait(&s.o_done, 0, spin, abort);
      ok = !bar_red_or(3, 128, !ok);
    }
    if (ok) {
      tc::tc_fence_after();
      xpose_reduce64<false>(l_part);
      s.red[warp][2 * lane] = l_part[0];
      s.red[warp][2 * lane + 1] = l_part[1];
      tc::named_barrier(1, 128);
      const int h0 = hg * AT_H;
      if (tid < AT_H) {
        const float L = (s.red[0][tid] + s.red[1][tid]) + (s.red[2][tid] + s.red[3][tid]);
        const float m = s.mcur[tid];
        const float s2 = a.sink ? a.sink[h0 + tid] * LOG2E : -INFINITY;
        const float mf = fmaxf(m, s2);
        float den = (m == -INFINITY ? 0.f : L * exp2f(m - mf)) + (a.sink ? exp2f(s2 - mf) : 0.f);
        float inv = 0.f, lse = -INFINITY;
        if (den > 0.f && mf != -INFINITY) {
          inv = (m == -INFINITY ? 0.f : exp2f(m - mf)) / den;
          lse = (mf + log2f(den)) * LN2;
        }
        s.inv[tid] = inv;
        if (a.lse) a.lse[(long long)qi * a.H + h0 + tid] = lse;
      }
      tc::named_barrier(1, 128);
      __nv_bfloat16* O = reinterpret_cast<__nv_bfloat16*>(a.O) + ((long long)qi * a.H + h0) * AT_C;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          float v[32];
          tc::tmem_ld32(tmem + lane_base + TM_O + 64 * q + 32 * hh, v);
          tc::tmem_wait_ld();
#pragma unroll
          for (int u = 0; u < 32; ++u) {
            const int h = 32 * hh + u;
            O[(long long)h * AT_C + 128 * q + tid] = __float2bfloat16_rn(v[u] * s.inv[h]);
          }
        }
      }
    }
  }
  tc::tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, TM_COLS);
  }
}

}  // namespace

int launch_attn_tc(const AttnArgs& a, cudaStream_t st, bool* used) {
  *used = false;
  const char* force = std::getenv("DSV4_FORCE_SIMT");
  if (force && force[0] == '1') return DSV4_OK;
  if (a.c != AT_C || a.H % AT_H != 0) return DSV4_OK;
  if (!aligned16(a.Q) || !aligned16(a.local) || (a.pool && !aligned16(a.pool))) return DSV4_OK;
  const long long nrows_q = (long long)a.B * a.nq * a.H;
  const long long nrows_local = (long long)a.B * a.R;
  if (nrows_q >= (1ll << 31) || nrows_local >= (1ll << 31) || a.pool_rows >= (1ll << 31))
    return DSV4_OK;
  CUtensorMap mq, mpool, mlocal;
  int s = encode_tensor_map_2d(&mq, a.Q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, AT_C, nrows_q, 64,
                               AT_H, CU_TENSOR_MAP_SWIZZLE_128B);
  if (s != DSV4_OK) return s;
  s = encode_tensor_map_2d(&mlocal, a.local, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, AT_C,
                           nrows_local, 64, 1, CU_TENSOR_MAP_SWIZZLE_128B);
  if (s != DSV4_OK) return s;
  if (a.pool && a.pool_rows > 0)
    s = encode_tensor_map_2d(&mpool, a.pool, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, AT_C,
                             a.pool_rows, 64, 1, CU_TENSOR_MAP_SWIZZLE_128B);
  else
    mpool = mlocal;
  if (s != DSV4_OK) return s;
  const int head_groups = a.H / AT_H;
  const long long grid = (long long)a.B * a.nq * head_groups;
  if (grid >= (1ll << 31)) return DSV4_OK;
  cudaError_t e = cudaFuncSetAttribute(attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)AT_SMEM);
  if (e != cudaSuccess) return fail(DSV4_ERR_CUDA, "attn_tc: %s", cudaGetErrorString(e));
  attn_tc_kernel<<<(unsigned)grid, AT_THREADS, AT_SMEM, st>>>(a, mq, mpool, mlocal, head_groups,
                                                             a.scale * LOG2E, spin_limit());
  *used = true;
  return launch_status("hybrid attention (tensor cores)");
}

}  // namespace dsv4
