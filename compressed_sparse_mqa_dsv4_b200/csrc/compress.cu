// dsv4_compress: learned softmax-gated pooling ("CSA And HCA: Definition, State, And Cost
// Model", s2.1 overlapping two-stream CSA compressor, s2.2 one-stream HCA compressor).
//
// HBM-bound streaming pass. One thread owns one 16-byte channel vector (8 bf16 / 4 fp32
// channels) of one output entry and walks the entry's positions with an online softmax
// per channel (running max, running denominator, running weighted sum; all fp32).
// Reads every input byte once (stream a of block i by entry i, stream b of block i by
// entry i+1), writes each entry once. Consecutive threads own consecutive channel
// vectors of the same entry, so each position row is read as contiguous 16-byte
// vectors across the warp.
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

// Vectorised kernel: requires c % V == 0 and 16-byte aligned C, Z, out, bias rows.
template <typename T, int CHUNK>
__global__ void __launch_bounds__(256) compress_vec_kernel(
    const T* __restrict__ C, const T* __restrict__ Z, const float* __restrict__ bias,
    T* __restrict__ out, int B, int n, int c, int m, int overlap, long long total_vecs) {
  constexpr int V = Vec16<T>::N;
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
    // the preceding block from stream b (CSA, i > 0) then the current block from stream a
    for (int half = (overlap && i > 0) ? 1 : 0; half >= 0; --half) {
      const int tok0 = half ? m * (i - 1) : m * i;
      const T* zrow = Z + ((long long)b * n + tok0) * row_stride + half * c + ch;
      const T* crow = C + ((long long)b * n + tok0) * row_stride + half * c + ch;
      const float* brow = bias + (long long)half * m * c + ch;
      for (int p0 = 0; p0 < m; p0 += CHUNK) {
        float z[CHUNK][V], x[CHUNK][V], bb[CHUNK][V];
        const int cnt = min(CHUNK, m - p0);
#pragma unroll
        for (int u = 0; u < CHUNK; ++u) {
          if (u < cnt) {
            load16_f32(zrow + (long long)(p0 + u) * row_stride, z[u]);
            load16_f32(crow + (long long)(p0 + u) * row_stride, x[u]);
#pragma unroll
            for (int j = 0; j < V; j += 4) {
              float4 t = __ldg(reinterpret_cast<const float4*>(brow + (long long)(p0 + u) * c + j));
              bb[u][j] = t.x; bb[u][j + 1] = t.y; bb[u][j + 2] = t.z; bb[u][j + 3] = t.w;
            }
          }
        }
#pragma unroll
        for (int u = 0; u < CHUNK; ++u)
          if (u < cnt) pool.add(z[u], bb[u], x[u]);
      }
    }
    float o[V];
#pragma unroll
    for (int j = 0; j < V; ++j) o[j] = pool.acc[j] / pool.den[j];
    store16_f32(out + ((long long)b * E + i) * c + ch, o);
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
  constexpr int V = Vec16<T>::N;
  const long long E = n / m;
  const bool vec_ok = (c % V == 0) && (c % 4 == 0) && aligned16(C) && aligned16(Z) &&
                      aligned16(out) && aligned16(bias);
  int sms = 148;
  if (vec_ok) {
    const long long total = (long long)B * E * (c / V);
    long long blocks = (total + 255) / 256;
    blocks = blocks < (long long)sms * 16 ? blocks : (long long)sms * 16;
    if (m >= 16)
      compress_vec_kernel<T, 8><<<(int)blocks, 256, 0, st>>>(
          (const T*)C, (const T*)Z, bias, (T*)out, B, n, c, m, overlap, total);
    else
      compress_vec_kernel<T, 4><<<(int)blocks, 256, 0, st>>>(
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
