// dsv4_index_topk_noalloc: the indexer top-k for callers that cannot allocate device
// memory themselves.
//
// dsv4_index_topk needs a scratch buffer for the per-query score rows. Most callers pass
// a workspace they allocated; some cannot: a runtime that hands kernels only buffers it
// planned ahead of time, plain C code with no device allocator of its own, or a serving
// loop that must not call cudaMalloc (it can synchronise the device and can fail once
// memory is fragmented). For them this entry point uses a fixed scratch array compiled
// into the library: a file-scope __device__ array of kNoAllocScratchBytes that every GPU
// which loads the library keeps until the process exits. Nothing is allocated per call.
//
// The work itself is the unchanged dsv4_index_topk path, handed that array as its
// workspace; it processes the queries in chunks whose score rows fit in the array.
#include <mutex>

#include "dsv4_common.cuh"

namespace {

constexpr size_t kNoAllocScratchBytes = 8u << 20;                  // 8 MiB of fp32 scores
constexpr long long kNoAllocMaxEntries = (long long)(kNoAllocScratchBytes / 4);

// Score scratch shared by every dsv4_index_topk_noalloc call on a device.
static __device__ __align__(256) float g_index_scratch[kNoAllocScratchBytes / sizeof(float)];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
float* g_scratch_ptr[kMaxDevices] = {};

// Device address of g_index_scratch on the current device, looked up once per device.
// (In host code the symbol name is only a host-side handle, not a device address.)
int scratch_address(float** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess)
    return dsv4::fail(DSV4_ERR_CUDA, "dsv4_index_topk_noalloc: cudaGetDevice: %s",
                      cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices)
    return dsv4::fail(DSV4_ERR_UNSUPPORTED, "dsv4_index_topk_noalloc: device %d", dev);
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_index_scratch);
    if (e != cudaSuccess || !p)
      return dsv4::fail(DSV4_ERR_CUDA, "dsv4_index_topk_noalloc: cudaGetSymbolAddress: %s",
                        cudaGetErrorString(e));
    g_scratch_ptr[dev] = static_cast<float*>(p);
  }
  *out = g_scratch_ptr[dev];
  return DSV4_OK;
}

}  // namespace

extern "C" int dsv4_index_topk_noalloc(int qdtype, const void* qI, const uint8_t* qI_scales,
                                       const float* w, const void* KI, const uint8_t* KI_scales,
                                       int64_t ki_rows, const int64_t* kv_row_off,
                                       const int32_t* q_pos0, int B, int nq, int H_I, int c_I,
                                       int m, int k, int max_entries, int32_t* idx,
                                       int32_t* counts, void* stream) {
  // One score row (rounded up to 4 entries) must fit in the fixed scratch.
  if ((long long)((max_entries + 3) / 4) * 4 > kNoAllocMaxEntries)
    return dsv4::fail(DSV4_ERR_INVALID_ARG,
                      "dsv4_index_topk_noalloc: max_entries %d exceeds the fixed scratch limit "
                      "of %lld entries (%zu bytes of scores); use dsv4_index_topk with a "
                      "workspace",
                      max_entries, kNoAllocMaxEntries, kNoAllocScratchBytes);
  float* scratch = nullptr;
  int s = scratch_address(&scratch);
  if (s != DSV4_OK) return s;
  return dsv4_index_topk(qdtype, qI, qI_scales, w, KI, KI_scales, ki_rows, kv_row_off, q_pos0,
                         B, nq, H_I, c_I, m, k, max_entries, idx, counts, nullptr, 0, scratch,
                         kNoAllocScratchBytes, stream);
}
