// dsv4_compress: learned softmax-gated pooling ("CSA And HCA: Definition, State, And Cost
// Model", s2.1 overlapping two-stream CSA compressor, s2.2 one-stream HCA compressor).
//
// HBM-bound streaming pass. One thread owns four consecutive channels of one output entry
// and walks the entry's positions with an online softmax per channel (running max, running
// denominator, running weighted sum; all fp32), with up to eight positions' loads in flight.
// Reads every input byte once (stream a of block i by entry i, stream b of block i by
// entry i+1), writes each entry once. Consecutive threads own consecutive channel groups of
// the same entry, so each position row is read contiguously across the warp. (Eight
// channels per thread needed 189 registers, one CTA per SM and reached ~0.7 TB/s.)
#include "dsv4_common.cuh"

namespace dsv4 {

template <typename T, int V>
struct OnlinePool {
  float mx[V], den[V], acc[V];
  __device__ __forceinline__ void init() {
#pragma unroll
    for (int j = 0; j < V; ++j) { mx[j] = -INFINITY; den[j] = 0.f; acc[j] = 0.f; }
  }
  __device__ __forceinline__ void add(const float (&z)[V], const float (&b)[V], const float (&x)[V]) {
#pragma unroll
    for (int j = 0; j < V; ++j) {
      float l = z[j] + b[j];
      if (l > mx[j]) {
        float r = expf(mx[j] - l);          // 0 on the first position (mx = -inf)
        den[j] = den[j] * r + 1.f;
        acc[j] = acc[j] * r + x[j];
        mx[j] = l;
      } else {
        float e = expf(l - mx[j]);
        den[j] += e;
        acc[j] = fmaf(e, x[j], acc[j]);
      }
    }
  }
};

// Four consecutive channels of T as raw bits (8 bytes of bf16, 16 of fp32), converted to fp32
// only where they are consumed, so the loads in flight cost 2 (4) registers each.
template <typename T> struct Raw4;
template <> struct Raw4<__nv_bfloat16> {
  uint2 r;
  __device__ __forceinline__ void load(const __nv_bfloat16* p) { r = __ldg(reinterpret_cast<const uint2*>(p)); }
  __device__ __forceinline__ void to_f32(float (&v)[4]) const {
    const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&r.x));
    const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&r.y));
    v[0] = a.x; v[1] = a.y; v[2] = b.x; v[3] = b.y;
  }
};
template <> struct Raw4<float> {
  uint4 r;
  __device__ __forceinline__ void load(const float* p) { r = __ldg(reinterpret_cast<const uint4*>(p)); }
  __device__ __forceinline__ void to_f32(float (&v)[4]) const {
    v[0] = __uint_as_float(r.x); v[1] = __uint_as_float(r.y); v[2] = __uint_as_float(r.z); v[3] = __uint_as_float(r.w);
  }
};

__device__ __forceinline__ void store4(float* p, const float (&v)[4]) {
  *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
}
__device__ __forceinline__ void store4(__nv_bfloat16* p, const float (&v)[4]) {
  __nv_bfloat162 a = __floats2bfloat162_rn(v[0], v[1]), b = __floats2bfloat162_rn(v[2], v[3]);
  *reinterpret_cast<uint2*>(p) = make_uint2(*reinterpret_cast<uint32_t*>(&a), *reinterpret_cast<uint32_t*>(&b));
}

// Vectorised kernel: requires c % 4 == 0 and C, Z, out aligned to 4 elements, bias to 16
// bytes. A thread owns 4 channels of one entry; CHUNK positions' C and Z vectors are loaded
// before any is consumed (memory-level parallelism per thread) and stay raw until use, and the
// bias is read at use: a small kernel, so that many CTAs per SM hide the rest of the latency.
template <typename T, int CHUNK>
__global__ void __launch_bounds__(256, 3) compress_vec_kernel(
    const T* __restrict__ C, const T* __restrict__ Z, const float* __restrict__ bias,
    T* __restrict__ out, int B, int n, int c, int m, int overlap, long long total_vecs) {
  constexpr int V = 4;
  const int vecs_per_entry = c / V;
  const int E = n / m;
  const int S = overlap ? 2 : 1;
  const long long row_stride = (long long)S * c;
  for (long long g = (long long)blockIdx.x * blockDim.x + threadIdx.x; g < total_vecs;
       g += (long long)gridDim.x * blockDim.x) {
    const int v = (int)(g % vecs_per_entry);
    const long long be = g / vecs_per_entry;
    const int i = (int)(be % E);
    const int b = (int)(be / E);
    const int ch = v * V;
    OnlinePool<T, V> pool;
    pool.init();
    // positions in order: the preceding block from stream b (CSA, i > 0), then the current
    // block from stream a; flattened, so that a chunk of loads spans both blocks when m is
    // small (CSA m = 4: all eight positions' loads are in flight at once)
    const int mb = (overlap && i > 0) ? m : 0;
    const long long tb = (long long)b * n + (long long)m * (i > 0 ? i - 1 : 0);
    const T* zb = Z + tb * row_stride + c + ch;                                 // stream b rows
    const T* cb = C + tb * row_stride + c + ch;
    const T* za = Z + ((long long)b * n + m * i) * row_stride + ch;             // stream a rows
    const T* ca = C + ((long long)b * n + m * i) * row_stride + ch;
    const int P = mb + m;
    for (int p0 = 0; p0 < P; p0 += CHUNK) {
      Raw4<T> zr[CHUNK], xr[CHUNK];
#pragma unroll
      for (int u = 0; u < CHUNK; ++u) {
        const int q = p0 + u;
        if (q < P) {
          const bool sb = q < mb;
          const long long off = (long long)(sb ? q : q - mb) * row_stride;
          zr[u].load((sb ? zb : za) + off);
          xr[u].load((sb ? cb : ca) + off);
        }
      }
#pragma unroll
      for (int u = 0; u < CHUNK; ++u) {
        const int q = p0 + u;
        if (q < P) {
          const bool sb = q < mb;
          float z[V], x[V], bb[V];
          zr[u].to_f32(z);
          xr[u].to_f32(x);
          const float4 t = __ldg(reinterpret_cast<const float4*>(
              bias + ((long long)(sb ? m + q : q - mb)) * c + ch));
          bb[0] = t.x; bb[1] = t.y; bb[2] = t.z; bb[3] = t.w;
          pool.add(z, bb, x);
        }
      }
    }
    float o[V];
#pragma unroll
    for (int j = 0; j < V; ++j) o[j] = pool.acc[j] / pool.den[j];
    store4(out + ((long long)b * E + i) * c + ch, o);
  }
}

// Scalar kernel for any c / alignment.
template <typename T>
__global__ void __launch_bounds__(256) compress_scalar_kernel(
    const T* __restrict__ C, const T* __restrict__ Z, const float* __restrict__ bias,
    T* __restrict__ out, int B, int n, int c, int m, int overlap, long long total) {
  const int E = n / m;
  const int S = overlap ? 2 : 1;
  const long long row_stride = (long long)S * c;
  for (long long g = (long long)blockIdx.x * blockDim.x + threadIdx.x; g < total;
       g += (long long)gridDim.x * blockDim.x) {
    const int ch = (int)(g % c);
    const long long be = g / c;
    const int i = (int)(be % E);
    const int b = (int)(be / E);
    float mx = -INFINITY, den = 0.f, acc = 0.f;
    for (int half = (overlap && i > 0) ? 1 : 0; half >= 0; --half) {
      const int tok0 = half ? m * (i - 1) : m * i;
      for (int p = 0; p < m; ++p) {
        const long long off = ((long long)b * n + tok0 + p) * row_stride + half * c + ch;
        float l = to_f32(Z[off]) + bias[((long long)half * m + p) * c + ch];
        float x = to_f32(C[off]);
        if (l > mx) {
          float r = expf(mx - l);
          den = den * r + 1.f; acc = acc * r + x; mx = l;
        } else {
          float e = expf(l - mx);
          den += e; acc = fmaf(e, x, acc);
        }
      }
    }
    out[((long long)b * E + i) * c + ch] = from_f32<T>(acc / den);
  }
}

template <typename T>
static int launch_compress(const void* C, const void* Z, const float* bias, void* out, int B,
                           int n, int c, int m, int overlap, cudaStream_t st) {
  const long long E = n / m;
  const uintptr_t al = 4 * sizeof(T) - 1;          // 4 elements
  const bool vec_ok = (c % 4 == 0) && !(reinterpret_cast<uintptr_t>(C) & al) &&
                      !(reinterpret_cast<uintptr_t>(Z) & al) && !(reinterpret_cast<uintptr_t>(out) & al) &&
                      aligned16(bias);
  int sms = 148;
  if (vec_ok) {
    const long long total = (long long)B * E * (c / 4);
    long long blocks = (total + 255) / 256;
    blocks = blocks < (long long)sms * 32 ? blocks : (long long)sms * 32;
    compress_vec_kernel<T, 8><<<(int)blocks, 256, 0, st>>>(
        (const T*)C, (const T*)Z, bias, (T*)out, B, n, c, m, overlap, total);
  } else {
    const long long total = (long long)B * E * c;
    long long blocks = (total + 255) / 256;
    blocks = blocks < (long long)sms * 16 ? blocks : (long long)sms * 16;
    compress_scalar_kernel<T><<<(int)blocks, 256, 0, st>>>(
        (const T*)C, (const T*)Z, bias, (T*)out, B, n, c, m, overlap, total);
  }
  return launch_status("dsv4_compress");
}

}  // namespace dsv4

extern "C" int dsv4_compress(int dtype, const void* C, const void* Z, const float* bias,
                             void* out, int B, int n, int c, int m, int overlap, void* stream) {
  using namespace dsv4;
  if (B < 0 || n < 0 || c < 1 || m < 1 || (overlap != 0 && overlap != 1))
    return fail(DSV4_ERR_INVALID_ARG, "dsv4_compress: bad sizes B=%d n=%d c=%d m=%d overlap=%d",
                B, n, c, m, overlap);
  if ((long long)B * (n / m) == 0) return DSV4_OK;
  if (!C || !Z || !bias || !out)
    return fail(DSV4_ERR_INVALID_ARG, "dsv4_compress: NULL tensor pointer");
  cudaStream_t st = (cudaStream_t)stream;
  if (dtype == DSV4_F32) return launch_compress<float>(C, Z, bias, out, B, n, c, m, overlap, st);
  if (dtype == DSV4_BF16)
    return launch_compress<__nv_bfloat16>(C, Z, bias, out, B, n, c, m, overlap, st);
  return fail(DSV4_ERR_INVALID_ARG, "dsv4_compress: dtype %d not F32/BF16", dtype);
}
