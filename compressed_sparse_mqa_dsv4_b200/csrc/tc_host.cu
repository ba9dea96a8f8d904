// Host helpers of the tensor-core kernels: tensor-map encoding through the driver entry
// point (no link-time dependency on libcuda) and the bounded-wait spin limit.
#include <cudaTypedefs.h>

#include <cstdlib>
#include <mutex>

#include "tc_common.cuh"

namespace dsv4 {

static PFN_cuTensorMapEncodeTiled_v12000 get_encode_fn() {
  static std::once_flag once;
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

int encode_tensor_map_2d(CUtensorMap* map, const void* base, CUtensorMapDataType dtype,
                         int elem_bytes, uint64_t cols, uint64_t rows, uint32_t box_cols,
                         uint32_t box_rows, CUtensorMapSwizzle swizzle) {
  auto fn = get_encode_fn();
  if (!fn) return fail(DSV4_ERR_CUDA, "cuTensorMapEncodeTiled entry point unavailable");
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * (cuuint64_t)elem_bytes};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, dtype, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS)
    return fail(DSV4_ERR_INVALID_ARG,
                "cuTensorMapEncodeTiled failed (%d): base %p, %llu x %llu, box %u x %u", (int)r,
                base, (unsigned long long)rows, (unsigned long long)cols, box_rows, box_cols);
  return DSV4_OK;
}

int encode_tensor_map_3d(CUtensorMap* map, const void* base, CUtensorMapDataType dtype,
                         const uint64_t dims[3], const uint64_t strides[2], const uint32_t box[3]) {
  auto fn = get_encode_fn();
  if (!fn) return fail(DSV4_ERR_CUDA, "cuTensorMapEncodeTiled entry point unavailable");
  cuuint64_t d[3] = {dims[0], dims[1], dims[2]};
  cuuint64_t st[2] = {strides[0], strides[1]};
  cuuint32_t bx[3] = {box[0], box[1], box[2]};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(map, dtype, 3, const_cast<void*>(base), d, st, bx, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS)
    return fail(DSV4_ERR_INVALID_ARG, "cuTensorMapEncodeTiled (3d) failed (%d): base %p, %llu x %llu x %llu",
                (int)r, base, (unsigned long long)dims[2], (unsigned long long)dims[1],
                (unsigned long long)dims[0]);
  return DSV4_OK;
}

// DSV4_SPIN_LIMIT=N sets the polls of every bounded wait (read once per process). N = 0
// leaves only the non-blocking first test, so any wait whose phase has not completed when
// it starts gives up at once: the way to exercise the abort path of the kernels.
uint32_t spin_limit() {
  static uint32_t lim = [] {
    const char* e = std::getenv("DSV4_SPIN_LIMIT");
    if (!e || !*e) return (uint32_t)(1u << 22);
    const long long v = std::atoll(e);
    return v >= 0 && v < (1ll << 32) ? (uint32_t)v : (uint32_t)(1u << 22);
  }();
  return lim;
}

}  // namespace dsv4
