// Incremental decode state ("CSA And HCA: Definition, State, And Cost Model", s7): per new
// token of every sequence, the local shared-KV ring slot write (step 1) and the compressor
// state machine (steps 2-4): the token's (C, Z) rows go to a bounded tail, and when t + 1
// is a multiple of the ratio m the completed entry (s2.1 / s2.2) is appended to the pool.
//
// The tail of a sequence holds the rows of its last T = m (HCA) or 2m (CSA: the current
// block plus the preceding block, whose stream-b half the next entry pools) positions,
// position p in slot p mod T. One CTA per sequence; a thread owns channel ch of both
// streams (columns ch and c + ch), so the rows it pools at an emission include the ones it
// has just written itself and no other thread's. Per channel the arithmetic is the one of
// the prefill compressor: an online softmax in fp32 over the preceding block's stream-b
// positions, then the current block's stream-a positions, in position order.
#include "dsv4_common.cuh"
#include "fp4_quant.cuh"
#include "fp8_kv.cuh"

namespace dsv4 {

// Where the emitted entry goes: a pool of dtype T, or -- through shared memory -- the
// production formats: the main-KV FP8 entry (fp8_kv.cuh) or the FP4 index key (fp4_quant.cuh).
// Either way the entry is rounded to T first and then quantised, so a packed pool holds
// exactly the quantisation of the T pool's row.
enum EmitMode { kEmitPool = 0, kEmitFp8 = 1, kEmitFp4 = 2 };

// Sequence b's token (one CTA of 256 threads): its (C, Z) rows into the tail and, when t + 1
// completes a block, the entry into the pool. FP8 / FP4: `entry` is shared memory of c floats;
// FP8: codes [rows, c - rope], scales fp32 [rows, (c - rope)/64], rope_out bf16 [rows, rope];
// FP4: codes [rows, c/2], scales E4M3 bytes [rows, c/16].
template <typename T, int MODE>
__device__ __forceinline__ void compress_decode_seq(
    int b, const T* __restrict__ C_new, const T* __restrict__ Z_new, const float* __restrict__ bias,
    T* __restrict__ tail, T* __restrict__ pool, const int64_t* __restrict__ pool_row_off,
    long long pool_rows, const int32_t* __restrict__ pos, int c, int m, int overlap,
    uint8_t* __restrict__ codes, void* __restrict__ scales_v, __nv_bfloat16* __restrict__ rope_out,
    int rope, float* entry) {
  constexpr bool FP8 = MODE == kEmitFp8;
  constexpr bool PACKED = MODE != kEmitPool;
  const int S = overlap ? 2 : 1;
  const int T_slots = S * m;
  const long long width = (long long)S * c;
  const int t = pos[b];
  if (t < 0) {
    if (threadIdx.x == 0) flag_status(DSV4_ERR_DEVICE_BOUNDS);
    return;
  }
  T* tail_b = tail + (long long)b * T_slots * 2 * width;     // [T, 2, S*c]
  // steps 2-3: the token's rows into slot t mod T
  T* slot = tail_b + (long long)(t % T_slots) * 2 * width;
  for (long long j = threadIdx.x; j < width; j += blockDim.x) {
    slot[j] = C_new[(long long)b * width + j];
    slot[width + j] = Z_new[(long long)b * width + j];
  }
  const long long t1 = (long long)t + 1;
  if (t1 % m != 0) return;                                   // incomplete block: no entry
  // step 4: entry i = (t+1)/m - 1 into pool row pool_row_off[b] + i
  const long long i = t1 / m - 1;
  const long long row = pool_row_off[b] + i;
  const bool row_ok = pool_row_off[b] >= 0 && row < pool_rows;
  if (!row_ok) {
    if (threadIdx.x == 0) flag_status(DSV4_ERR_DEVICE_BOUNDS);
    return;
  }
  constexpr int PF = 8;                                      // positions whose loads are in flight
  for (int ch = threadIdx.x; ch < c; ch += blockDim.x) {
    float mx = -INFINITY, den = 0.f, acc = 0.f;
    for (int half = (overlap && i > 0) ? 1 : 0; half >= 0; --half) {
      const long long tok0 = half ? m * (i - 1) : m * i;
      for (int p0 = 0; p0 < m; p0 += PF) {
        // the next PF positions' rows are loaded before any is used (a dependent load per
        // position made an emission latency-bound); the online softmax then takes them in
        // position order, as the prefill compressor does
        float xs[PF], ls[PF];
#pragma unroll
        for (int u = 0; u < PF; ++u) {
          xs[u] = 0.f;
          ls[u] = -INFINITY;
          if (p0 + u < m) {
            const T* r = tail_b + ((tok0 + p0 + u) % T_slots) * 2 * width + half * c + ch;
            xs[u] = to_f32(r[0]);
            ls[u] = to_f32(r[width]) + bias[((long long)half * m + p0 + u) * c + ch];
          }
        }
#pragma unroll
        for (int u = 0; u < PF; ++u) {
          if (p0 + u >= m) break;
          const float l = ls[u], x = xs[u];
          if (l > mx) {
            float e = expf(mx - l);
            den = den * e + 1.f; acc = acc * e + x; mx = l;
          } else {
            float e = expf(l - mx);
            den += e; acc = fmaf(e, x, acc);
          }
        }
      }
    }
    if constexpr (PACKED)
      entry[ch] = to_f32(from_f32<T>(acc / den));
    else
      pool[row * c + ch] = from_f32<T>(acc / den);
  }
  if constexpr (MODE == kEmitFp4) {
    __syncthreads();
    uint8_t* sc4 = static_cast<uint8_t*>(scales_v);
    for (int g = threadIdx.x; g < c / 16; g += blockDim.x) {
      float v[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) v[j] = entry[16 * g + j];
      uint32_t w0, w1, sb;
      fp4_quantize_group(v, w0, w1, sb);
      *reinterpret_cast<uint2*>(codes + row * (c / 2) + 8 * g) = make_uint2(w0, w1);
      sc4[row * (c / 16) + g] = (uint8_t)sb;
    }
  }
  if constexpr (FP8) {
    float* scales = static_cast<float*>(scales_v);
    __syncthreads();
    const int lane = threadIdx.x & 31, nw = blockDim.x >> 5;
    const int nf = c - rope, ng = nf / kFp8Group;
    for (int g = threadIdx.x >> 5; g < ng; g += nw) {
      const int ch = g * kFp8Group + 2 * lane;
      uint32_t code2;
      const float sc = fp8_group_quantize(entry[ch], entry[ch + 1], code2);
      *reinterpret_cast<uint16_t*>(codes + row * nf + ch) = (uint16_t)code2;
      if (lane == 0) scales[row * ng + g] = sc;
    }
    for (int d = threadIdx.x; d < rope; d += blockDim.x)
      rope_out[row * rope + d] = __float2bfloat16_rn(entry[nf + d]);
  }
}

template <typename T, int MODE>
__global__ void __launch_bounds__(256) compress_decode_kernel(
    const T* __restrict__ C_new, const T* __restrict__ Z_new, const float* __restrict__ bias,
    T* __restrict__ tail, T* __restrict__ pool, const int64_t* __restrict__ pool_row_off,
    long long pool_rows, const int32_t* __restrict__ pos, int c, int m, int overlap,
    uint8_t* __restrict__ codes, float* __restrict__ scales, __nv_bfloat16* __restrict__ rope_out,
    int rope) {
  extern __shared__ float entry[];                          // packed: the entry, c values
  compress_decode_seq<T, MODE>(blockIdx.x, C_new, Z_new, bias, tail, pool, pool_row_off, pool_rows,
                               pos, c, m, overlap, codes, scales, rope_out, rope, entry);
}

template <typename T>
__device__ __forceinline__ void ring_write_seq(int b, const T* __restrict__ kv_new,
                                               T* __restrict__ local, int R,
                                               const int32_t* __restrict__ pos, int c) {
  const int t = pos[b];
  if (t < 0) {
    if (threadIdx.x == 0) flag_status(DSV4_ERR_DEVICE_BOUNDS);
    return;
  }
  T* dst = local + ((long long)b * R + t % R) * c;
  for (int j = threadIdx.x; j < c; j += blockDim.x) dst[j] = kv_new[(long long)b * c + j];
}

template <typename T>
__global__ void __launch_bounds__(256) ring_write_kernel(const T* __restrict__ kv_new,
                                                         T* __restrict__ local, int R,
                                                         const int32_t* __restrict__ pos, int c) {
  ring_write_seq<T>(blockIdx.x, kv_new, local, R, pos, c);
}

// Every job of a token's state update in one launch: CTA (b, j) performs job j for sequence b.
struct DecodeJobs {
  dsv4_decode_job j[DSV4_DECODE_MAX_JOBS];
};

template <typename T>
__global__ void __launch_bounds__(256) decode_state_kernel(const __grid_constant__ DecodeJobs jobs,
                                                           const int32_t* __restrict__ pos) {
  extern __shared__ float entry[];                          // packed emissions: c values
  const dsv4_decode_job& jb = jobs.j[blockIdx.y];
  const T* x = static_cast<const T*>(jb.x_new);
  const T* z = static_cast<const T*>(jb.z_new);
  T* tail = static_cast<T*>(jb.tail);
  if (jb.kind == DSV4_JOB_RING)
    ring_write_seq<T>(blockIdx.x, x, static_cast<T*>(jb.out), jb.R, pos, jb.c);
  else if (jb.kind == DSV4_JOB_COMPRESS)
    compress_decode_seq<T, kEmitPool>(blockIdx.x, x, z, jb.bias, tail, static_cast<T*>(jb.out),
                                      jb.pool_row_off, jb.pool_rows, pos, jb.c, jb.m, jb.overlap,
                                      nullptr, nullptr, nullptr, 0, entry);
  else if (jb.kind == DSV4_JOB_COMPRESS_FP8)
    compress_decode_seq<T, kEmitFp8>(blockIdx.x, x, z, jb.bias, tail, nullptr, jb.pool_row_off,
                                     jb.pool_rows, pos, jb.c, jb.m, jb.overlap,
                                     static_cast<uint8_t*>(jb.out), jb.out_scales,
                                     static_cast<__nv_bfloat16*>(jb.out_rope), jb.rope_dims, entry);
  else
    compress_decode_seq<T, kEmitFp4>(blockIdx.x, x, z, jb.bias, tail, nullptr, jb.pool_row_off,
                                     jb.pool_rows, pos, jb.c, jb.m, jb.overlap,
                                     static_cast<uint8_t*>(jb.out), jb.out_scales, nullptr, 0, entry);
}

}  // namespace dsv4

extern "C" int dsv4_compress_decode(int dtype, const void* C_new, const void* Z_new,
                                    const float* bias, void* tail, void* pool,
                                    const int64_t* pool_row_off, int64_t pool_rows,
                                    const int32_t* pos, int B, int c, int m, int overlap,
                                    void* stream) {
  using namespace dsv4;
  if (B < 0 || c < 1 || m < 1 || (overlap != 0 && overlap != 1) || pool_rows < 0)
    return fail(DSV4_ERR_INVALID_ARG,
                "dsv4_compress_decode: bad sizes B=%d c=%d m=%d overlap=%d pool_rows=%lld", B, c,
                m, overlap, (long long)pool_rows);
  if (B == 0) return DSV4_OK;
  if (!C_new || !Z_new || !bias || !tail || !pool || !pool_row_off || !pos)
    return fail(DSV4_ERR_INVALID_ARG, "dsv4_compress_decode: NULL pointer");
  cudaStream_t st = (cudaStream_t)stream;
  if (dtype == DSV4_F32)
    compress_decode_kernel<float, kEmitPool><<<B, 256, 0, st>>>(
        (const float*)C_new, (const float*)Z_new, bias, (float*)tail, (float*)pool, pool_row_off,
        pool_rows, pos, c, m, overlap, nullptr, nullptr, nullptr, 0);
  else if (dtype == DSV4_BF16)
    compress_decode_kernel<__nv_bfloat16, kEmitPool><<<B, 256, 0, st>>>(
        (const __nv_bfloat16*)C_new, (const __nv_bfloat16*)Z_new, bias, (__nv_bfloat16*)tail,
        (__nv_bfloat16*)pool, pool_row_off, pool_rows, pos, c, m, overlap, nullptr, nullptr,
        nullptr, 0);
  else
    return fail(DSV4_ERR_INVALID_ARG, "dsv4_compress_decode: dtype %d not F32/BF16", dtype);
  return launch_status("dsv4_compress_decode");
}

extern "C" int dsv4_ring_write(int dtype, const void* kv_new, void* local, int R,
                               const int32_t* pos, int B, int c, void* stream) {
  using namespace dsv4;
  if (B < 0 || R < 1 || c < 1)
    return fail(DSV4_ERR_INVALID_ARG, "dsv4_ring_write: bad sizes B=%d R=%d c=%d", B, R, c);
  if (B == 0) return DSV4_OK;
  if (!kv_new || !local || !pos) return fail(DSV4_ERR_INVALID_ARG, "dsv4_ring_write: NULL pointer");
  cudaStream_t st = (cudaStream_t)stream;
  if (dtype == DSV4_F32)
    ring_write_kernel<float><<<B, 256, 0, st>>>((const float*)kv_new, (float*)local, R, pos, c);
  else if (dtype == DSV4_BF16)
    ring_write_kernel<__nv_bfloat16><<<B, 256, 0, st>>>((const __nv_bfloat16*)kv_new,
                                                        (__nv_bfloat16*)local, R, pos, c);
  else
    return fail(DSV4_ERR_INVALID_ARG, "dsv4_ring_write: dtype %d not F32/BF16", dtype);
  return launch_status("dsv4_ring_write");
}

extern "C" int dsv4_decode_state(int dtype, const dsv4_decode_job* jobs, int n_jobs,
                                 const int32_t* pos, int B, void* stream) {
  using namespace dsv4;
  if (B < 0 || n_jobs < 0 || n_jobs > DSV4_DECODE_MAX_JOBS)
    return fail(DSV4_ERR_INVALID_ARG, "dsv4_decode_state: bad sizes B=%d n_jobs=%d (at most %d)", B,
                n_jobs, DSV4_DECODE_MAX_JOBS);
  if (B == 0 || n_jobs == 0) return DSV4_OK;
  if (!jobs || !pos) return fail(DSV4_ERR_INVALID_ARG, "dsv4_decode_state: NULL pointer");
  if (dtype != DSV4_F32 && dtype != DSV4_BF16)
    return fail(DSV4_ERR_INVALID_ARG, "dsv4_decode_state: dtype %d not F32/BF16", dtype);
  DecodeJobs dj;
  int smem_c = 0;                                  // widest packed emission (floats)
  for (int i = 0; i < n_jobs; ++i) {
    const dsv4_decode_job& j = jobs[i];
    if (j.kind == DSV4_JOB_RING) {
      if (j.c < 1 || j.R < 1 || !j.x_new || !j.out)
        return fail(DSV4_ERR_INVALID_ARG, "dsv4_decode_state: ring job %d: c=%d R=%d or NULL pointer", i,
                    j.c, j.R);
    } else if (j.kind == DSV4_JOB_COMPRESS || j.kind == DSV4_JOB_COMPRESS_FP8 ||
               j.kind == DSV4_JOB_COMPRESS_FP4) {
      if (j.c < 1 || j.m < 1 || (j.overlap != 0 && j.overlap != 1) || j.pool_rows < 0 || !j.x_new ||
          !j.z_new || !j.bias || !j.tail || !j.out || !j.pool_row_off)
        return fail(DSV4_ERR_INVALID_ARG,
                    "dsv4_decode_state: compressor job %d: c=%d m=%d overlap=%d pool_rows=%lld or NULL "
                    "pointer", i, j.c, j.m, j.overlap, (long long)j.pool_rows);
      if (j.kind == DSV4_JOB_COMPRESS_FP8 &&
          (j.rope_dims < 0 || j.rope_dims > j.c || (j.rope_dims & 1) || (j.c - j.rope_dims) % kFp8Group != 0 ||
           j.c > 12 * 1024 || !j.out_scales || (j.rope_dims > 0 && !j.out_rope) ||
           (reinterpret_cast<uintptr_t>(j.out) & 1u)))
        return fail(DSV4_ERR_INVALID_ARG, "dsv4_decode_state: FP8 job %d: c=%d rope_dims=%d, scales/rope or "
                    "2-byte aligned codes", i, j.c, j.rope_dims);
      if (j.kind == DSV4_JOB_COMPRESS_FP4 &&
          (j.c % 16 != 0 || j.c > 12 * 1024 || !j.out_scales || (reinterpret_cast<uintptr_t>(j.out) & 7u)))
        return fail(DSV4_ERR_INVALID_ARG, "dsv4_decode_state: FP4 job %d: c=%d (c %% 16 == 0), scales or "
                    "8-byte aligned codes", i, j.c);
      if (j.kind != DSV4_JOB_COMPRESS && j.c > smem_c) smem_c = j.c;
    } else {
      return fail(DSV4_ERR_INVALID_ARG, "dsv4_decode_state: job %d has kind %d", i, j.kind);
    }
    dj.j[i] = j;
  }
  const size_t smem = sizeof(float) * (size_t)smem_c;
  cudaStream_t st = (cudaStream_t)stream;
  const dim3 grid((unsigned)B, (unsigned)n_jobs);
  if (dtype == DSV4_F32)
    decode_state_kernel<float><<<grid, 256, smem, st>>>(dj, pos);
  else
    decode_state_kernel<__nv_bfloat16><<<grid, 256, smem, st>>>(dj, pos);
  return launch_status("dsv4_decode_state");
}

extern "C" int dsv4_compress_decode_fp8(int dtype, const void* C_new, const void* Z_new,
                                        const float* bias, void* tail, uint8_t* codes,
                                        float* scales, void* rope_out, int rope,
                                        const int64_t* pool_row_off, int64_t pool_rows,
                                        const int32_t* pos, int B, int c, int m, int overlap,
                                        void* stream) {
  using namespace dsv4;
  if (B < 0 || c < 1 || m < 1 || (overlap != 0 && overlap != 1) || pool_rows < 0 || rope < 0 ||
      rope > c || (rope & 1) || (c - rope) % kFp8Group != 0 || c > 12 * 1024)
    return fail(DSV4_ERR_INVALID_ARG,
                "dsv4_compress_decode_fp8: bad sizes B=%d c=%d rope=%d m=%d overlap=%d pool_rows=%lld",
                B, c, rope, m, overlap, (long long)pool_rows);
  if (B == 0) return DSV4_OK;
  if (!C_new || !Z_new || !bias || !tail || !codes || !scales || (rope > 0 && !rope_out) ||
      !pool_row_off || !pos)
    return fail(DSV4_ERR_INVALID_ARG, "dsv4_compress_decode_fp8: NULL pointer");
  if (reinterpret_cast<uintptr_t>(codes) & 1u)
    return fail(DSV4_ERR_INVALID_ARG, "dsv4_compress_decode_fp8: codes must be 2-byte aligned");
  cudaStream_t st = (cudaStream_t)stream;
  const size_t smem = sizeof(float) * (size_t)c;
  if (dtype == DSV4_F32)
    compress_decode_kernel<float, kEmitFp8><<<B, 256, smem, st>>>(
        (const float*)C_new, (const float*)Z_new, bias, (float*)tail, nullptr, pool_row_off,
        pool_rows, pos, c, m, overlap, codes, scales, (__nv_bfloat16*)rope_out, rope);
  else if (dtype == DSV4_BF16)
    compress_decode_kernel<__nv_bfloat16, kEmitFp8><<<B, 256, smem, st>>>(
        (const __nv_bfloat16*)C_new, (const __nv_bfloat16*)Z_new, bias, (__nv_bfloat16*)tail,
        nullptr, pool_row_off, pool_rows, pos, c, m, overlap, codes, scales,
        (__nv_bfloat16*)rope_out, rope);
  else
    return fail(DSV4_ERR_INVALID_ARG, "dsv4_compress_decode_fp8: dtype %d not F32/BF16", dtype);
  return launch_status("dsv4_compress_decode_fp8");
}
