// gqa_static.cu -- gqa_decode_split_static: the split-KV decode with its
// scratch in a fixed array of device memory that belongs to the library.
//
// Who needs it: callers that may not allocate device memory while they decode.
// Examples are a host process whose device memory is owned by another memory
// manager (a serving engine that hands out every byte of HBM from its own
// pool), and latency-critical loops that must not enter the CUDA allocator.
// They still pass in q, the caches, the lengths and the output; only the
// scratch for partial softmax states comes from here.
//
// The array is GQA_STATIC_WORKSPACE_BYTES long and lives in the library's
// device module, so every GPU that loads the library keeps it until the
// process exits.  All calls share it: two calls whose kernels overlap on the
// GPU (on different streams, or from different host threads) race on it and
// must not be issued that way.  The kernels write every scratch word before
// reading it, so nothing in it has to start at zero and a call does not
// depend on what the previous call left there.
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "gqa.h"

namespace {

static __device__ __align__(256) unsigned char g_static_scratch[GQA_STATIC_WORKSPACE_BYTES];

constexpr int kMaxDevices = 64;
void *g_scratch_ptr[kMaxDevices] = {};
std::mutex g_scratch_mu;

// Device address of the array for the current device.  In host code the
// array's name is only a host-side handle, so the address is looked up once per
// device (with that device current) and cached.  The cache assumes the
// device's context lives as long as the process: after cudaDeviceReset (or a
// release and re-creation of the primary context) the module is loaded again
// elsewhere and the cached address is stale, so the library must not be used
// across a device reset.
int scratch_address(void **out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return GQA_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return GQA_ERR_DEVICE;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_ptr[dev] == nullptr) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || p == nullptr) return GQA_ERR_CUDA;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return GQA_OK;
}

}  // namespace

extern "C" int gqa_decode_split_static(const void *q, const void *k_cache, const void *v_cache,
                                       const int32_t *seqlens, const int32_t *page_table, float *out,
                                       const gqa_dims *dims, float scale, uint32_t *status,
                                       int32_t split_tokens, int32_t max_seqlen, void *stream) {
  const size_t need = gqa_decode_split_workspace_size(dims, max_seqlen, split_tokens);
  if (need == 0 || need > GQA_STATIC_WORKSPACE_BYTES) {
    // Invalid arguments, or a problem too large for the array: the regular
    // entry point, given no workspace, runs all of its checks in its own order
    // and stops at the workspace test at the latest (it launches nothing
    // without one), so an argument error is reported ahead of
    // GQA_ERR_WORKSPACE exactly as gqa_decode_split reports it.
    const int rc = gqa_decode_split(q, k_cache, v_cache, seqlens, page_table, out, dims, scale, status,
                                    split_tokens, max_seqlen, nullptr, 0, stream);
    return rc == GQA_OK ? GQA_ERR_WORKSPACE : rc;
  }
  void *scratch = nullptr;
  const int rc = scratch_address(&scratch);
  if (rc != GQA_OK) return rc;
  return gqa_decode_split(q, k_cache, v_cache, seqlens, page_table, out, dims, scale, status, split_tokens,
                          max_seqlen, scratch, GQA_STATIC_WORKSPACE_BYTES, stream);
}
