// Lightning-indexer scores on CUDA cores (any dtype, any c_I multiple of 16).
//
// I_{t,s} = sum_h w_{t,h} ReLU(q^I_{t,h} . K^I_s), s < floor((t+1)/m)
// ("CSA And HCA: Definition, State, And Cost Model", s3.1). This is the general path
// (fp32 operands, odd shapes); bf16 / FP4 operands at V4 shapes take the tensor-core
// kernel. One CTA scores one query against a tile of 64 entries: the query's heads are
// decoded to fp32 in shared memory, the key tile likewise (row stride c_I+1 so that
// 32 lanes reading 32 rows hit 32 banks); 4 thread groups split the heads and combine
// their weighted ReLU partial sums through shared memory.
#include "dsv4_common.cuh"
#include "index_common.cuh"

namespace dsv4 {

constexpr int IDX_TILE = 64;

template <int QD>
__global__ void __launch_bounds__(256) index_scores_simt_kernel(IndexArgs a, int q_begin,
                                                                int q_count) {
  extern __shared__ float smem[];
  const int cI = a.c_I, HI = a.H_I;
  float* qs = smem;                              // [HI][cI]
  float* ks = qs + HI * cI;                      // [IDX_TILE][cI+1]
  float* ws = ks + IDX_TILE * (cI + 1);          // [HI]
  float* part = ws + HI;                         // [4][IDX_TILE]
  const int qg = q_begin + blockIdx.x;           // global query id b*nq + i
  if ((int)blockIdx.x >= q_count) return;
  const int b = qg / a.nq, i = qg % a.nq;
  const int Et = visible_entries(a, b, i);
  const int s0 = blockIdx.y * IDX_TILE;
  if (s0 >= Et) return;
  const long long base = a.kv_row_off[b];
  if (base < 0 || base + Et > a.ki_rows) {
    if (threadIdx.x == 0 && blockIdx.y == 0) flag_status(DSV4_ERR_DEVICE_BOUNDS);
    return;
  }
  // stage the query heads and weights
  const long long qrow0 = (long long)qg * HI;
  for (int e = threadIdx.x; e < HI * cI; e += blockDim.x) {
    const int h = e / cI, d = e % cI;
    qs[e] = load_elem<QD>(a.qI, a.qI_scales, qrow0 + h, d, cI);
  }
  for (int h = threadIdx.x; h < HI; h += blockDim.x) ws[h] = a.w[qrow0 + h];
  const int ns = min(IDX_TILE, Et - s0);
  for (int e = threadIdx.x; e < ns * cI; e += blockDim.x) {
    const int r = e / cI, d = e % cI;
    ks[r * (cI + 1) + d] = load_elem<QD>(a.KI, a.KI_scales, base + s0 + r, d, cI);
  }
  __syncthreads();
  const int r = threadIdx.x % IDX_TILE, hg = threadIdx.x / IDX_TILE;
  float acc = 0.f;
  if (r < ns) {
    const float* kr = ks + r * (cI + 1);
    for (int h = hg; h < HI; h += 4) {
      const float* qh = qs + h * cI;
      float dot = 0.f;
      for (int d = 0; d < cI; ++d) dot = fmaf(qh[d], kr[d], dot);
      acc = fmaf(ws[h], fmaxf(dot, 0.f), acc);
    }
  }
  part[hg * IDX_TILE + r] = acc;
  __syncthreads();
  if (threadIdx.x < ns) {
    const int rr = threadIdx.x;
    const float s = ((part[rr] + part[IDX_TILE + rr]) + part[2 * IDX_TILE + rr]) +
                    part[3 * IDX_TILE + rr];
    a.scores[(long long)(qg - a.score_q0) * a.scores_ld + s0 + rr] = s;
  }
}

int launch_index_scores_simt(const IndexArgs& a, int q_begin, int q_count, int max_e,
                             cudaStream_t st) {
  const size_t smem = sizeof(float) * ((size_t)a.H_I * a.c_I + (size_t)IDX_TILE * (a.c_I + 1) +
                                       a.H_I + 4 * IDX_TILE);
  if (smem > 200 * 1024)
    return fail(DSV4_ERR_UNSUPPORTED, "dsv4_index_topk: H_I*c_I too large for the CUDA-core path");
  dim3 grid(q_count, ceil_div(max_e, IDX_TILE));
  if (grid.y == 0 || grid.x == 0) return DSV4_OK;
  if (grid.y > 65535)
    return fail(DSV4_ERR_UNSUPPORTED, "dsv4_index_topk: max_entries %d too large", max_e);
  switch (a.qdtype) {
    case DSV4_F32:
      cudaFuncSetAttribute(index_scores_simt_kernel<DSV4_F32>,
                           cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      index_scores_simt_kernel<DSV4_F32><<<grid, 256, smem, st>>>(a, q_begin, q_count);
      break;
    case DSV4_BF16:
      cudaFuncSetAttribute(index_scores_simt_kernel<DSV4_BF16>,
                           cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      index_scores_simt_kernel<DSV4_BF16><<<grid, 256, smem, st>>>(a, q_begin, q_count);
      break;
    default:
      cudaFuncSetAttribute(index_scores_simt_kernel<DSV4_FP4>,
                           cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      index_scores_simt_kernel<DSV4_FP4><<<grid, 256, smem, st>>>(a, q_begin, q_count);
      break;
  }
  return launch_status("index scores (CUDA cores)");
}

}  // namespace dsv4
