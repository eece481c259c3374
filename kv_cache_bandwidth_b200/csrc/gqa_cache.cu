// gqa_cache.cu -- the KV append step (one new token per sequence, written
// through the page table) and the host-side pool of page ids; see gqa_cache.h.
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>
#include <new>
#include <vector>

#include "gqa_cache.h"

namespace {

constexpr uint32_t kStatusBadSeqlen = 1u;
constexpr uint32_t kStatusBadPage = 2u;

struct AppendParams {
  const uint4 *k_new;      // [b, G, D/8] (8 bf16 per uint4)
  const uint4 *v_new;
  uint4 *k_cache;          // [pages, G, P, D/8]
  uint4 *v_cache;
  int32_t *seqlens;        // [b], incremented
  const int32_t *page_table;  // [b, max_pages] or null (contiguous)
  uint32_t *status;
  int G, P, num_pages, max_pages;
  long long capacity;
};

// One block per sequence: every thread reads the length, the block copies the
// sequence's G rows of K and of V (D/8 16-byte words each), and thread 0
// advances the length once the copies are issued and every thread has read it.
template <int D>
__global__ void __launch_bounds__(128) gqa_kv_append_kernel(const AppendParams p) {
  constexpr int kW = D / 8;
  // A decode launched right behind this kernel as its programmatic dependent
  // may be dispatched now; it waits for this grid to finish before it reads.
  if (threadIdx.x == 0) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int s = blockIdx.x;
  const int t = p.seqlens[s];
  if (t < 0 || static_cast<long long>(t) >= p.capacity) {
    if (threadIdx.x == 0 && p.status) atomicOr(p.status, kStatusBadSeqlen);
    return;
  }
  long long page;
  int row;
  if (p.page_table) {
    page = __ldg(p.page_table + static_cast<long long>(s) * p.max_pages + t / p.P);
    row = t % p.P;
    if (page < 0 || page >= p.num_pages) {
      if (threadIdx.x == 0 && p.status) atomicOr(p.status, kStatusBadPage);
      return;
    }
  } else {
    page = s;
    row = t;
  }
  const long long src0 = static_cast<long long>(s) * p.G * kW;
  for (int i = threadIdx.x; i < p.G * kW; i += blockDim.x) {
    const int g = i / kW, c = i % kW;
    const long long dst = ((page * p.G + g) * p.P + row) * kW + c;
    p.k_cache[dst] = __ldg(p.k_new + src0 + i);
    p.v_cache[dst] = __ldg(p.v_new + src0 + i);
  }
  __syncthreads();
  if (threadIdx.x == 0) p.seqlens[s] = t + 1;
}

bool aligned16(const void *x) { return (reinterpret_cast<uintptr_t>(x) & 15u) == 0; }

}  // namespace

struct gqa_page_pool {
  std::mutex mu;
  std::vector<int32_t> free_ids;  // a stack: the back is handed out next
  std::vector<uint8_t> in_use;
};

extern "C" {

int gqa_kv_append(const void *k_new, const void *v_new, void *k_cache, void *v_cache, int32_t *seqlens,
                  const int32_t *page_table, const gqa_dims *dims, uint32_t *status, void *stream) {
  if (!k_new || !v_new || !k_cache || !v_cache || !seqlens || !dims) return GQA_ERR_NULL_POINTER;
  if (!aligned16(k_new) || !aligned16(v_new) || !aligned16(k_cache) || !aligned16(v_cache) ||
      (reinterpret_cast<uintptr_t>(seqlens) & 3u) || (reinterpret_cast<uintptr_t>(page_table) & 3u) ||
      (reinterpret_cast<uintptr_t>(status) & 3u))
    return GQA_ERR_MISALIGNED;
  const gqa_dims &d = *dims;
  if (d.batch < 1 || d.batch > 0x7fffffff || d.num_heads < 1 || d.num_kv_heads < 1 || d.page_size < 1)
    return GQA_ERR_DIMS;
  if (d.num_heads % d.num_kv_heads != 0) return GQA_ERR_HEADS;
  if (d.head_dim != 64 && d.head_dim != 128) return GQA_ERR_HEAD_DIM;
  AppendParams p{};
  p.k_new = static_cast<const uint4 *>(k_new);
  p.v_new = static_cast<const uint4 *>(v_new);
  p.k_cache = static_cast<uint4 *>(k_cache);
  p.v_cache = static_cast<uint4 *>(v_cache);
  p.seqlens = seqlens;
  p.page_table = page_table;
  p.status = status;
  p.G = d.num_kv_heads;
  p.P = d.page_size;
  if (page_table) {
    if (d.page_size < 8 || d.page_size > (1 << 20) || (d.page_size & (d.page_size - 1))) return GQA_ERR_PAGE_SIZE;
    if (d.num_pages < 1 || d.max_pages_per_seq < 1) return GQA_ERR_DIMS;
    p.num_pages = d.num_pages;
    p.max_pages = d.max_pages_per_seq;
    p.capacity = static_cast<long long>(d.max_pages_per_seq) * d.page_size;
  } else {
    p.num_pages = d.batch;
    p.max_pages = 1;
    p.capacity = d.page_size;
  }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (d.head_dim == 128)
    gqa_kv_append_kernel<128><<<static_cast<unsigned>(d.batch), 128, 0, st>>>(p);
  else
    gqa_kv_append_kernel<64><<<static_cast<unsigned>(d.batch), 128, 0, st>>>(p);
  return cudaGetLastError() == cudaSuccess ? GQA_OK : GQA_ERR_CUDA;
}

gqa_page_pool *gqa_page_pool_create(int32_t num_pages) {
  if (num_pages < 1) return nullptr;
  gqa_page_pool *pool = new (std::nothrow) gqa_page_pool;
  if (!pool) return nullptr;
  try {
    pool->free_ids.resize(num_pages);
    for (int32_t i = 0; i < num_pages; ++i) pool->free_ids[i] = num_pages - 1 - i;  // 0 on top
    pool->in_use.assign(num_pages, 0);
  } catch (...) {
    delete pool;
    return nullptr;
  }
  return pool;
}

void gqa_page_pool_destroy(gqa_page_pool *pool) { delete pool; }

int32_t gqa_page_pool_available(const gqa_page_pool *pool) {
  if (!pool) return GQA_ERR_NULL_POINTER;
  std::lock_guard<std::mutex> lock(const_cast<gqa_page_pool *>(pool)->mu);
  return static_cast<int32_t>(pool->free_ids.size());
}

int gqa_page_pool_alloc(gqa_page_pool *pool, int32_t n, int32_t *ids) {
  if (!pool || (n > 0 && !ids)) return GQA_ERR_NULL_POINTER;
  if (n < 0) return GQA_ERR_DIMS;
  std::lock_guard<std::mutex> lock(pool->mu);
  if (static_cast<size_t>(n) > pool->free_ids.size()) return GQA_ERR_NO_PAGES;
  for (int32_t i = 0; i < n; ++i) {
    const int32_t id = pool->free_ids.back();
    pool->free_ids.pop_back();
    pool->in_use[id] = 1;
    ids[i] = id;
  }
  return GQA_OK;
}

int gqa_page_pool_free(gqa_page_pool *pool, const int32_t *ids, int32_t n) {
  if (!pool || (n > 0 && !ids)) return GQA_ERR_NULL_POINTER;
  if (n < 0) return GQA_ERR_DIMS;
  std::lock_guard<std::mutex> lock(pool->mu);
  const int32_t total = static_cast<int32_t>(pool->in_use.size());
  // check everything first: all or nothing
  for (int32_t i = 0; i < n; ++i) {
    const int32_t id = ids[i];
    if (id < 0 || id >= total || pool->in_use[id] != 1) {
      for (int32_t j = 0; j < i; ++j) pool->in_use[ids[j]] = 1;  // undo the duplicate marks
      return GQA_ERR_DIMS;
    }
    pool->in_use[id] = 2;  // marked: a second listing of the id fails the check above
  }
  for (int32_t i = 0; i < n; ++i) {
    pool->in_use[ids[i]] = 0;
    pool->free_ids.push_back(ids[i]);
  }
  return GQA_OK;
}

}  // extern "C"
