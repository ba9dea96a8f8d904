// Hybrid shared-KV MQA on CUDA cores: the general path (fp32 data, any head count and
// head dim); bf16 at V4 shapes takes the tensor-core kernel.
//
// "CSA And HCA: Definition, State, And Cost Model": s3.2/s4 shared K=V entries for all
// heads, s5.1 one candidate list (compressed ++ local window) under one softmax per
// head, s5.3 sink logit in the denominator only.
//
// One CTA per (query, group of 16 heads). Candidates stream through shared memory in
// chunks of 32 rows (converted to fp32, row stride c+1). Each chunk: logits for 16 heads
// x 32 rows, an online-softmax update per head (running max / denominator, rescale of
// the accumulator), then the weighted row sum into a 16 x c fp32 accumulator held in
// registers (each thread owns one head and c/16 strided channels).
#include "attn_common.cuh"

namespace dsv4 {

constexpr int AS_HG = 16;      // heads per CTA
constexpr int AS_NC = 32;      // candidate rows per chunk
constexpr int AS_THREADS = 256;
constexpr int AS_MAXC = 1024;  // largest head dim of this path

template <typename T>
__global__ void __launch_bounds__(AS_THREADS) attn_simt_kernel(AttnArgs a) {
  extern __shared__ float sm[];
  const int c = a.c, cp = a.c + 1;
  float* qs = sm;                         // [AS_HG][c]
  float* rows = qs + AS_HG * c;           // [AS_NC][c+1]
  float* zs = rows + AS_NC * cp;          // [AS_HG][AS_NC]
  float* mrun = zs + AS_HG * AS_NC;       // [AS_HG] running max
  float* lrun = mrun + AS_HG;             // [AS_HG] running denominator
  float* resc = lrun + AS_HG;             // [AS_HG] rescale of this chunk
  __shared__ int valid[AS_NC];

  const int qi = blockIdx.x;              // b * nq + i
  const int b = qi / a.nq, i = qi % a.nq;
  const int h0 = blockIdx.y * AS_HG;
  const int hn = min(AS_HG, a.H - h0);
  const T* Q = reinterpret_cast<const T*>(a.Q);
  const T* pool = reinterpret_cast<const T*>(a.pool);
  const T* local = reinterpret_cast<const T*>(a.local);
  const CandidateSet cs = make_candidates(a, b, i);
  const int N = cs.n_comp + cs.n_local;

  for (int e = threadIdx.x; e < AS_HG * c; e += blockDim.x) {
    const int h = e / c, d = e % c;
    qs[e] = h < hn ? to_f32(Q[(((long long)qi) * a.H + h0 + h) * c + d]) * a.scale : 0.f;
  }
  if (threadIdx.x < AS_HG) { mrun[threadIdx.x] = -INFINITY; lrun[threadIdx.x] = 0.f; }

  // accumulator: head ah, channels ac + 16*u
  const int ah = threadIdx.x / 16, ac = threadIdx.x % 16;
  const int nu = (c + 15) / 16;
  float acc[AS_MAXC / 16];
#pragma unroll
  for (int u = 0; u < AS_MAXC / 16; ++u) acc[u] = 0.f;

  for (int j0 = 0; j0 < N; j0 += AS_NC) {
    const int nr = min(AS_NC, N - j0);
    __syncthreads();
    if (threadIdx.x < AS_NC) {
      int ok = 0;
      if (threadIdx.x < nr) {
        bool is_local;
        const long long r = candidate_row(a, cs, j0 + threadIdx.x, is_local);
        ok = r >= 0 ? 1 + (is_local ? 1 : 0) : 0;
        if (r < 0) flag_status(DSV4_ERR_DEVICE_BOUNDS);
      }
      valid[threadIdx.x] = ok;
    }
    __syncthreads();
    for (int e = threadIdx.x; e < nr * c; e += blockDim.x) {
      const int r = e / c, d = e % c;
      float v = 0.f;
      if (valid[r]) {
        bool is_local;
        const long long row = candidate_row(a, cs, j0 + r, is_local);
        v = to_f32((is_local ? local : pool)[row * c + d]);
      }
      rows[r * cp + d] = v;
    }
    __syncthreads();
    // logits: thread -> (head zh, rows zr and zr + 16)
    {
      const int zh = threadIdx.x / 16, zr = threadIdx.x % 16;
      float d0 = 0.f, d1 = 0.f;
      const float* qh = qs + zh * c;
      const float* r0 = rows + zr * cp;
      const float* r1 = rows + (zr + 16) * cp;
      for (int d = 0; d < c; ++d) {
        const float qv = qh[d];
        d0 = fmaf(qv, r0[d], d0);
        d1 = fmaf(qv, r1[d], d1);
      }
      zs[zh * AS_NC + zr] = (zr < nr && valid[zr]) ? d0 : -INFINITY;
      zs[zh * AS_NC + zr + 16] = (zr + 16 < nr && valid[zr + 16]) ? d1 : -INFINITY;
    }
    __syncthreads();
    // online softmax per head (16 threads per head)
    {
      const int sh = threadIdx.x / 16, sl = threadIdx.x % 16;
      float* z = zs + sh * AS_NC;
      float mx = fmaxf(z[sl], z[sl + 16]);
#pragma unroll
      for (int off = 8; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off, 16));
      const float mold = mrun[sh];
      const float mnew = fmaxf(mold, mx);
      const float p0 = mnew == -INFINITY ? 0.f : expf(z[sl] - mnew);
      const float p1 = mnew == -INFINITY ? 0.f : expf(z[sl + 16] - mnew);
      float sum = p0 + p1;
#pragma unroll
      for (int off = 8; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off, 16);
      __syncwarp();
      z[sl] = p0;
      z[sl + 16] = p1;
      if (sl == 0) {
        const float r = mold == -INFINITY ? 0.f : expf(mold - mnew);
        resc[sh] = r;
        lrun[sh] = lrun[sh] * r + sum;
        mrun[sh] = mnew;
      }
    }
    __syncthreads();
    {
      const float r = resc[ah];
      const float* p = zs + ah * AS_NC;
#pragma unroll
      for (int u = 0; u < AS_MAXC / 16; ++u) {
        if (u < nu) {
          const int d = ac + 16 * u;
          if (d < c) {
            float v = acc[u] * r;
            for (int jr = 0; jr < nr; ++jr) v = fmaf(p[jr], rows[jr * cp + d], v);
            acc[u] = v;
          }
        }
      }
    }
  }
  __syncthreads();
  float mx = mrun[ah], den = lrun[ah];
  if (ah < hn && a.sink) {
    const float s = a.sink[h0 + ah];
    const float mnew = fmaxf(mx, s);
    den = den * expf(mx - mnew) + expf(s - mnew);
#pragma unroll
    for (int u = 0; u < AS_MAXC / 16; ++u) acc[u] *= expf(mx - mnew);
    mx = mnew;
  }
  const float inv = ah < hn ? 1.f / den : 0.f;
#pragma unroll
  for (int u = 0; u < AS_MAXC / 16; ++u) acc[u] *= inv;
  if (a.rope_out) {
    // inverse RoPE of the last rope_out channels at the query's position: the partner of
    // channel d (= ac + 16u) is d^1, held by thread ac^1 (c even, so both lie below c)
    const long long tpos = (long long)a.q_pos0[b] + i;
#pragma unroll
    for (int u = 0; u < AS_MAXC / 16; ++u) {
      if (u < nu) {
        const int d = ac + 16 * u;
        const float other = __shfl_xor_sync(0xffffffffu, acc[u], 1);
        if (d < c && d >= c - a.rope_out) {
          float cs, sn;
          rope_cos_sin(tpos, (d - (c - a.rope_out)) >> 1, a.rope_out, cs, sn);
          acc[u] = (d & 1) ? fmaf(acc[u], cs, -other * sn) : fmaf(acc[u], cs, other * sn);
        }
      }
    }
  }
  if (ah < hn) {
    T* O = reinterpret_cast<T*>(a.O) + ((long long)qi * a.H + h0 + ah) * c;
#pragma unroll
    for (int u = 0; u < AS_MAXC / 16; ++u) {
      const int d = ac + 16 * u;
      if (u < nu && d < c) O[d] = from_f32<T>(acc[u]);
    }
    if (a.lse && ac == 0) a.lse[(long long)qi * a.H + h0 + ah] = mx + logf(den);
  }
}

int launch_attn_simt(const AttnArgs& a, int dtype, cudaStream_t st) {
  if (a.c > AS_MAXC)
    return fail(DSV4_ERR_UNSUPPORTED, "dsv4_hybrid_sparse_attn: c=%d above %d on the CUDA-core path",
                a.c, AS_MAXC);
  const size_t smem = sizeof(float) * ((size_t)AS_HG * a.c + (size_t)AS_NC * (a.c + 1) +
                                       AS_HG * AS_NC + 3 * AS_HG);
  dim3 grid(a.B * a.nq, ceil_div(a.H, AS_HG));
  if (dtype == DSV4_F32) {
    cudaFuncSetAttribute(attn_simt_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)smem);
    attn_simt_kernel<float><<<grid, AS_THREADS, smem, st>>>(a);
  } else {
    cudaFuncSetAttribute(attn_simt_kernel<__nv_bfloat16>,
                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    attn_simt_kernel<__nv_bfloat16><<<grid, AS_THREADS, smem, st>>>(a);
  }
  return launch_status("hybrid attention (CUDA cores)");
}

}  // namespace dsv4
