// gqa_api.cu -- the C ABI of libgqa (declared in include/gqa.h).
//
// Host side only: argument validation (before anything touches the GPU),
// TMA descriptor encoding for the K and V pools, the split / cluster plan and
// the kernel launches on the caller's stream.  No device memory is allocated
// here; the only state kept between calls is per-device attribute caches.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "gqa.h"
#include "gqa_cache.h"
#include "gqa_kernels.cuh"
#include "gqa_verify_tc.cuh"

static_assert(GQA_MERGE_IN_KERNEL_MAX_SPLITS == gqa::kSerialMergeMax,
              "the header's in-kernel merge limit is the kernels' serial-merge limit");

namespace {

using gqa::DecodeParams;
using gqa::CombineParams;
using gqa::Mode;

constexpr int kMaxDevices = 64;
constexpr int kSplitQuantum = 128;  // split_tokens granularity (a multiple of every tile)
constexpr int kMaxBalancedBlocks = 512;   // decode blocks of the balanced mode (workspace bound)
constexpr int kMaxBalancedBatch = 1024;   // longer batches use fixed splits
constexpr int kFallbackSplit = 4096;      // the fixed split used then

// ------------------------------------------------------------------ device info
struct DeviceInfo {
  int sms = 0;
  int major = 0;
  bool ok = false;
};

DeviceInfo g_dev[kMaxDevices];
std::mutex g_dev_mu;

int current_device_info(DeviceInfo *out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return GQA_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return GQA_ERR_DEVICE;
  std::lock_guard<std::mutex> lock(g_dev_mu);
  DeviceInfo &d = g_dev[dev];
  if (!d.ok) {
    if (cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&d.major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
      return GQA_ERR_CUDA;
    d.ok = true;
  }
  *out = d;
  return d.major == 10 ? GQA_OK : GQA_ERR_DEVICE;
}

// ------------------------------------------------------------------ TMA encode
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    cudaDriverEntryPointQueryResult q;
    void *ptr = nullptr;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

// A 4-D view [pages][G][rows_per_page][D] of a bf16 pool, boxes of 64 x box_rows.
int encode_pool(CUtensorMap *map, const void *base, int D, int rows_per_page, int G,
                long long pages, int box_rows) {
  auto fn = encode_fn();
  if (!fn) return GQA_ERR_CUDA;
  cuuint64_t dims[4] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(rows_per_page),
                        static_cast<cuuint64_t>(G), static_cast<cuuint64_t>(pages)};
  cuuint64_t strides[3] = {static_cast<cuuint64_t>(D) * 2,
                           static_cast<cuuint64_t>(rows_per_page) * D * 2,
                           static_cast<cuuint64_t>(G) * rows_per_page * D * 2};
  cuuint32_t box[4] = {64u, static_cast<cuuint32_t>(box_rows), 1u, 1u};
  cuuint32_t estride[4] = {1u, 1u, 1u, 1u};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(base), dims, strides,
                  box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? GQA_OK : GQA_ERR_CUDA;
}

// ------------------------------------------------------------------ validation
struct Shape {
  int b, H, G, r, D, P, num_pages, max_pages;
  bool mapped;  // group of each head from a table (r = the largest group)
  bool tc;      // the tcgen05 kernel: all rows of a group in one block (<= 128 rows at d = 128, 64 at d = 64)
  bool paged;
  long long capacity;
  int nt, nhb;  // kernel variant: n8 row tiles per consumer warp, row blocks of 8
  int nq, rq;   // query tokens per sequence and rows per group (nq * r, token-major)
  int rc, hs;   // rows per block (min(rq, 16)) and 16-row slices per group
  bool fma;     // q.k and p.v on CUDA cores instead of tensor cores
};

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Largest number of query tokens per sequence (speculative verification).
constexpr int kMaxQueryTokens = 64;

// group_of_head (host memory, num_heads entries) or null: with a table, H need
// not be a multiple of G and r becomes the largest group's size.
// Rows per group above which the automatic choice is the tcgen05 kernel
// (measured: with 64 and 128 rows it beats the 16-row mma.sync slices by 1.3x
// and 2.4x; with 32 or fewer its one-thread-per-row softmax leaves lanes idle).
constexpr int kTcAutoRows = GQA_TC_AUTO_ROWS;

int check_dims(const gqa_dims *dims, bool paged, Shape *sh, int nq = 1, const int32_t *group_of_head = nullptr,
               bool auto_tc = true) {
  if (!dims) return GQA_ERR_NULL_POINTER;
  const gqa_dims &d = *dims;
  if (d.batch < 1 || d.num_heads < 1 || d.num_kv_heads < 1 || d.page_size < 1) return GQA_ERR_DIMS;
  if (d.batch > 65535 || d.num_kv_heads > 16383) return GQA_ERR_DIMS;  // grid y/z limits (G x 4 slices)
  int r;
  if (group_of_head) {
    if (d.num_heads > gqa::kMaxMapHeads || d.num_kv_heads > gqa::kMaxMapGroups || nq != 1) return GQA_ERR_HEADS;
    int count[gqa::kMaxMapGroups] = {};
    for (int i = 0; i < d.num_heads; ++i) {
      if (group_of_head[i] < 0 || group_of_head[i] >= d.num_kv_heads) return GQA_ERR_HEADS;
      ++count[group_of_head[i]];
    }
    r = 1;
    for (int g = 0; g < d.num_kv_heads; ++g) r = std::max(r, count[g]);
  } else {
    if (d.num_heads % d.num_kv_heads != 0) return GQA_ERR_HEADS;
    r = d.num_heads / d.num_kv_heads;
  }
  if (r > GQA_MAX_GROUP_RATIO) return GQA_ERR_HEADS;
  if (d.head_dim != 64 && d.head_dim != 128) return GQA_ERR_HEAD_DIM;
  if (d.flags & ~(GQA_FLAG_CONTRACT_MMA | GQA_FLAG_CONTRACT_FMA | GQA_FLAG_CONTRACT_TCGEN05)) return GQA_ERR_DIMS;
  if (__builtin_popcount(d.flags) > 1) return GQA_ERR_DIMS;  // one contraction choice at most
  Shape s{};
  s.b = d.batch;
  s.H = d.num_heads;
  s.G = d.num_kv_heads;
  s.r = r;
  s.mapped = group_of_head != nullptr;
  s.D = d.head_dim;
  s.P = d.page_size;
  s.paged = paged;
  if (paged) {
    if (d.page_size < 8 || d.page_size > (1 << 20) || (d.page_size & (d.page_size - 1)))
      return GQA_ERR_PAGE_SIZE;
    if (d.num_pages < 1 || d.max_pages_per_seq < 1) return GQA_ERR_DIMS;
    s.num_pages = d.num_pages;
    s.max_pages = d.max_pages_per_seq;
    s.capacity = static_cast<long long>(d.max_pages_per_seq) * d.page_size;
  } else {
    s.num_pages = d.batch;
    s.max_pages = 1;
    s.capacity = d.page_size;
  }
  if (s.capacity > (1ll << 30)) return GQA_ERR_DIMS;
  if (nq < 1 || nq > kMaxQueryTokens) return GQA_ERR_DIMS;
  if (static_cast<long long>(s.b) * nq * s.H * s.D > (1ll << 31) - 1) return GQA_ERR_DIMS;
  // The rows of a group are its (query token, head) pairs, token-major.  A
  // block serves at most 16 rows (two row blocks of 8); larger groups are cut
  // into 16-row slices handled by separate blocks that stream the same KV
  // range (the repeats of a tile are L2 hits).
  s.nq = nq;
  s.rq = nq * r;
  s.rc = std::min(s.rq, 16);
  s.hs = (s.rq + s.rc - 1) / s.rc;
  s.nt = 1;
  s.nhb = (s.rc + 7) / 8;
  s.fma = (d.flags & GQA_FLAG_CONTRACT_FMA) != 0;
  // rows one tcgen05 block takes: 128 at d = 128, 64 at d = 64 (the spread layout)
  const int tc_rows = s.D == 128 ? gqa::TcTile::kM : gqa::TcTileSpread64::kQRows;
  s.tc = (d.flags & GQA_FLAG_CONTRACT_TCGEN05) != 0 ||
         (auto_tc && d.flags == 0 && s.rq > kTcAutoRows && s.rq <= tc_rows);
  if (s.tc) {
    // one block takes all rows of a group
    if (s.rq > tc_rows) return GQA_ERR_HEADS;
    s.rc = s.rq;
    s.hs = 1;
  }
  if (s.fma && (r > 2 || nq > 1 || s.mapped)) return GQA_ERR_HEADS;  // CUDA-core path: r <= 2, one token, no map
  *sh = s;
  return GQA_OK;
}

int check_inputs(const void *q, const void *k, const void *v, const int32_t *seqlens,
                 const uint32_t *status) {
  if (!q || !k || !v || !seqlens) return GQA_ERR_NULL_POINTER;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v)) return GQA_ERR_MISALIGNED;
  if ((reinterpret_cast<uintptr_t>(seqlens) & 3u) || (reinterpret_cast<uintptr_t>(status) & 3u))
    return GQA_ERR_MISALIGNED;
  return GQA_OK;
}

// ------------------------------------------------------------------ workspace
size_t round256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// Fixed splits: o [b, H, S, d], m and l [b, H, S], then one 64-bit arrival
// word per (sequence, group, head slice) unit for the decode kernel's own merge.
struct Workspace {
  size_t o_bytes, m_bytes, ctr_off, total;
};

long long units_of(const Shape &sh) { return static_cast<long long>(sh.b) * sh.G * sh.hs; }

Workspace workspace_layout(const Shape &sh, int num_splits) {
  Workspace w;
  const size_t rows = static_cast<size_t>(sh.b) * sh.nq * sh.H * num_splits;
  w.o_bytes = round256(rows * sh.D * sizeof(float));
  w.m_bytes = round256(rows * sizeof(float));
  w.ctr_off = w.o_bytes + 2 * w.m_bytes;
  w.total = w.ctr_off + round256(static_cast<size_t>(units_of(sh)) * sizeof(unsigned long long));
  return w;
}

// Tag of one call in the arrival words, in [1, 2^40 - 2]: never 0 or all ones,
// the two patterns a cleared or poisoned workspace holds.
unsigned long long next_epoch() {
  static std::atomic<unsigned long long> counter{0};
  return counter.fetch_add(1, std::memory_order_relaxed) % ((1ull << 40) - 2) + 1;
}

// Blocks per cluster for gqa_decode: 1 (one block per (sequence, group)
// unit) when the units give about 1.5 blocks per SM; otherwise the smallest
// power of two (at most 16, gqa::kMaxClusterBlocks) that does, never more
// blocks than 128-token tiles.
int cluster_plan(const Shape &sh, int sms) {
  const long long units = units_of(sh);
  const long long want = (3ll * sms + 1) / 2;
  const long long max_by_len = std::max<long long>(1, sh.capacity / 128);
  int c = 1;
  while (c < gqa::kMaxClusterBlocks && units * c < want && 2 * c <= max_by_len) c *= 2;
  return c;
}

// ------------------------------------------------------------------ launches
// Pipeline shape per variant.  For r <= 8 (the common GQA ratios) the block
// is small enough for several blocks per SM: "dual" runs two blocks of 3
// stages, "trio" three blocks of 2 stages, "solo" one block of 6 stages.
// Larger ratios run one block per SM with a 3- or 4-stage ring.
#ifndef GQA_PIPE_POLICY
#define GQA_PIPE_POLICY 0  // 0: automatic, 1: solo, 2: dual, 3: trio
#endif

enum class Pipe { kSolo, kDual, kTrio };

struct Launch {
  dim3 grid;
  int cluster;
  cudaStream_t stream;
  bool pdl = false;  // programmatic dependent launch (the kernel waits before its first global read)
  bool query = false;  // cluster mode: only ask whether every cluster of the grid is resident at once
};

template <int D, int NT, int NHB, int STAGES, bool PAGED, Mode MODE, int FMA = 0>
int launch_decode_t(const CUtensorMap &tk, const CUtensorMap &tv, const DecodeParams &p, Launch l) {
  constexpr int CH = (D == 64) ? 2 : 1;
  using TL = gqa::Tile<D, NT, NHB, CH, STAGES, MODE == Mode::kBalanced>;
  auto kernel = gqa::gqa_decode_kernel<D, NT, NHB, CH, STAGES, PAGED, MODE, FMA>;
  const int smem = TL::kSmemBytes;
  // The shared-memory limit is a per-device attribute of the function: set it
  // once per device (a repeat is harmless, so two threads racing here is too).
  static std::atomic<unsigned long long> attr_set{0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return GQA_ERR_CUDA;
  const unsigned long long bit = 1ull << (dev & 63);
  if (!(attr_set.load(std::memory_order_acquire) & bit)) {
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
      return GQA_ERR_CUDA;
    if (MODE == Mode::kCluster &&
        cudaFuncSetAttribute(kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) != cudaSuccess)
      return GQA_ERR_CUDA;
    attr_set.fetch_or(bit, std::memory_order_acq_rel);
  }
  if (MODE == Mode::kBalanced) {
    // one block per resident slot of the GPU: grid.x holds the SM count on
    // entry and becomes SMs x blocks per SM (capped by the workspace)
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, TL::kThreads, smem) != cudaSuccess ||
        per_sm < 1)
      return GQA_ERR_CUDA;
    l.grid.x = std::min<unsigned>(l.grid.x * per_sm, kMaxBalancedBlocks);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = l.grid;
    cfg.blockDim = dim3(TL::kThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = l.stream;
    cudaLaunchAttribute pdl[1];
    pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    pdl[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = pdl;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, kernel, tk, tv, p) != cudaSuccess) return GQA_ERR_CUDA;
    return static_cast<int>(l.grid.x);  // > 0: the number of decode blocks
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = l.grid;
  cfg.blockDim = dim3(TL::kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = l.stream;
  cudaLaunchAttribute attr[2];
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (MODE == Mode::kCluster) {
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = l.cluster;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    if (l.query) {
      // 1: one wave holds every cluster (a second wave would double the step)
      int n = 0;
      if (cudaOccupancyMaxActiveClusters(&n, kernel, &cfg) != cudaSuccess) return GQA_ERR_CUDA;
      return static_cast<long long>(n) >= static_cast<long long>(l.grid.y) * l.grid.z ? 1 : 0;
    }
    if (l.pdl) {
      attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
      attr[1].val.programmaticStreamSerializationAllowed = 1;
      cfg.numAttrs = 2;
    }
  } else if (l.pdl) {
    // items mode: may start while the previous kernel on the stream finishes
    // (the kernel waits for it before touching memory)
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
  } else {
    cfg.numAttrs = 0;
  }
  return cudaLaunchKernelEx(&cfg, kernel, tk, tv, p) == cudaSuccess ? GQA_OK : GQA_ERR_CUDA;
}

Pipe pick_pipe(const Shape &sh) {
  if (sh.nhb != 1) return Pipe::kDual;
  switch (GQA_PIPE_POLICY) {
    case 1: return Pipe::kSolo;
    case 3: return Pipe::kTrio;
    default: return Pipe::kDual;
  }
}

template <int D, bool PAGED, Mode MODE>
int launch_decode_d(const Shape &sh, const CUtensorMap &tk, const CUtensorMap &tv,
                    const DecodeParams &p, const Launch &l) {
  if (sh.fma)
    return sh.r == 1 ? launch_decode_t<D, 1, 1, 3, PAGED, MODE, 1>(tk, tv, p, l)
                     : launch_decode_t<D, 1, 1, 3, PAGED, MODE, 2>(tk, tv, p, l);
  if (sh.nhb == 2) {
    // 16 rows: two 288-thread blocks per SM get 96 registers a thread, too few
    // for the equal-work walker at d = 128 (it spilled 180-208 bytes), so
    // there equal-work ranges run one block per SM with a six-stage ring
    // (measured 7-8 % faster on paged 16-row batches).  At d = 64 the
    // two-block form, which spills only 12-20 bytes, stays: it measured 12 %
    // faster there.
    if constexpr (MODE == Mode::kBalanced && D == 128) return launch_decode_t<D, 1, 2, 6, PAGED, MODE>(tk, tv, p, l);
    else return launch_decode_t<D, 1, 2, 3, PAGED, MODE>(tk, tv, p, l);
  }
  switch (pick_pipe(sh)) {
    case Pipe::kTrio: return launch_decode_t<D, 1, 1, 2, PAGED, MODE>(tk, tv, p, l);
    case Pipe::kSolo: return launch_decode_t<D, 1, 1, 6, PAGED, MODE>(tk, tv, p, l);
    default: return launch_decode_t<D, 1, 1, 3, PAGED, MODE>(tk, tv, p, l);
  }
}

template <Mode MODE>
int launch_decode(const Shape &sh, const CUtensorMap &tk, const CUtensorMap &tv, const DecodeParams &p,
                  const Launch &l) {
  if (sh.D == 128)
    return sh.paged ? launch_decode_d<128, true, MODE>(sh, tk, tv, p, l)
                    : launch_decode_d<128, false, MODE>(sh, tk, tv, p, l);
  return sh.paged ? launch_decode_d<64, true, MODE>(sh, tk, tv, p, l)
                  : launch_decode_d<64, false, MODE>(sh, tk, tv, p, l);
}

int tile_tokens(const Shape &sh) { return sh.D == 64 ? 128 : 64; }

// The tcgen05 kernel (items mode; d = 128 with 64-token tiles, d = 64 with
// 128-token tiles, like the mma.sync kernel).
int launch_verify_tc(const Shape &sh, const CUtensorMap &tk, const CUtensorMap &tv, const DecodeParams &p,
                     const Launch &l) {
  // at most 64 rows: spread over the four lane quarters of tensor memory
  // (always at d = 64)
  const bool spread = sh.rc <= 64;
  auto kernel = sh.D == 64 ? (sh.paged ? gqa::gqa_verify_tc_kernel<true, true, 64>
                                       : gqa::gqa_verify_tc_kernel<false, true, 64>)
                : sh.paged ? (spread ? gqa::gqa_verify_tc_kernel<true, true> : gqa::gqa_verify_tc_kernel<true, false>)
                           : (spread ? gqa::gqa_verify_tc_kernel<false, true> : gqa::gqa_verify_tc_kernel<false, false>);
  const int smem = sh.D == 64 ? gqa::TcTileSpread64::kSmemBytes
                              : spread ? gqa::TcTileSpread::kSmemBytes : gqa::TcTile::kSmemBytes;
  static std::atomic<unsigned long long> attr_set{0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return GQA_ERR_CUDA;
  const unsigned long long bit = 1ull << (dev & 63);
  if (!(attr_set.load(std::memory_order_acquire) & bit)) {
    for (auto k : {gqa::gqa_verify_tc_kernel<true, true>, gqa::gqa_verify_tc_kernel<false, true>})
      if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, gqa::TcTileSpread::kSmemBytes) !=
          cudaSuccess)
        return GQA_ERR_CUDA;
    for (auto k : {gqa::gqa_verify_tc_kernel<true, false>, gqa::gqa_verify_tc_kernel<false, false>})
      if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, gqa::TcTile::kSmemBytes) !=
          cudaSuccess)
        return GQA_ERR_CUDA;
    for (auto k : {gqa::gqa_verify_tc_kernel<true, true, 64>, gqa::gqa_verify_tc_kernel<false, true, 64>})
      if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, gqa::TcTileSpread64::kSmemBytes) !=
          cudaSuccess)
        return GQA_ERR_CUDA;
    attr_set.fetch_or(bit, std::memory_order_acq_rel);
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = l.grid;
  cfg.blockDim = dim3(gqa::TcTile::kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = l.stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = l.pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kernel, tk, tv, p) == cudaSuccess ? GQA_OK : GQA_ERR_CUDA;
}

int encode_maps(const Shape &sh, const void *k, const void *v, CUtensorMap *tk, CUtensorMap *tv) {
  const int T = tile_tokens(sh);
  const int rows = sh.P;  // paged: page size; contiguous: capacity m
  const long long pages = sh.paged ? sh.num_pages : sh.b;
  const int box = sh.paged ? std::min(sh.P, T) : T;
  int rc = encode_pool(tk, k, sh.D, rows, sh.G, pages, box);
  if (rc == GQA_OK) rc = encode_pool(tv, v, sh.D, rows, sh.G, pages, box);
  return rc;
}

DecodeParams base_params(const Shape &sh, const void *q, const int32_t *seqlens, const int32_t *pt,
                         uint32_t *status, float scale) {
  DecodeParams p{};
  p.q = static_cast<const __nv_bfloat16 *>(q);
  p.seqlens = seqlens;
  p.page_table = pt;
  p.status = status;
  p.H = sh.H;
  p.G = sh.G;
  p.r = sh.r;
  p.nq = sh.nq;
  p.rq = sh.rq;
  p.rc = sh.rc;
  p.hs = sh.hs;
  p.page_size = sh.P;
  p.num_pages = sh.num_pages;
  p.max_pages = sh.max_pages;
  p.capacity = static_cast<int>(sh.capacity);
  p.scale_log2 = scale * 1.4426950408889634f;
  p.ups = sh.G * sh.hs;
  return p;
}

// Optional per-row outputs of the split entry points: the log-sum-exp of
// every final row, and whether a length of 0 is a valid (empty) sequence.
struct RowExtras {
  float *lse = nullptr;
  bool empty_ok = false;
  int nq = 1;  // query tokens per sequence
  bool force_pdl = false;  // dependent launch even for one item per unit (behind a short kernel)
  const int32_t *group_of_head = nullptr;  // host table of each head's KV group, or null
};

// The device form of a group table: heads sorted by group (stable), offsets,
// and the (group, slice of rc rows) units that hold rows.
void fill_group_map(const int32_t *group_of_head, int H, int G, int rc, gqa::GroupMap *m) {
  int count[gqa::kMaxMapGroups + 1] = {};
  for (int i = 0; i < H; ++i) ++count[group_of_head[i] + 1];
  m->off[0] = 0;
  for (int g = 0; g < G; ++g) m->off[g + 1] = static_cast<uint16_t>(m->off[g] + count[g + 1]);
  int fill[gqa::kMaxMapGroups] = {};
  for (int i = 0; i < H; ++i) {
    const int g = group_of_head[i];
    m->heads[m->off[g] + fill[g]++] = static_cast<uint8_t>(i);
  }
  int n = 0;
  for (int g = 0; g < G; ++g)
    for (int j = 0; j * rc < count[g + 1]; ++j) {  // at most H slices in all: each holds a row
      m->slice_g[n] = static_cast<uint8_t>(g);
      m->slice_j[n] = static_cast<uint8_t>(j);
      ++n;
    }
  m->n_slices = static_cast<uint16_t>(n);
}

// L2 a dependent launch may fill ahead of its wait: the first tiles of every
// block's piece, GQA_PREFETCH_L2_BYTES over the grid (about half of the L2),
// at most the piece.
#ifndef GQA_PREFETCH_L2_BYTES
#define GQA_PREFETCH_L2_BYTES (64ll << 20)
#endif
int prefetch_tiles(const Shape &sh, long long blocks, int piece_tokens) {
  const int T = tile_tokens(sh);
  const long long tile_bytes = 4ll * T * sh.D;  // K and V, bf16
  const long long per_block = GQA_PREFETCH_L2_BYTES / std::max<long long>(1, blocks / sh.hs) / tile_bytes;
  return static_cast<int>(std::min<long long>(per_block, (piece_tokens + T - 1) / T));
}

// The items kernel: one block per (sequence, group, split) item.
int run_items(const Shape &sh, const void *q, const void *k, const void *v, const int32_t *seqlens,
              const int32_t *pt, float *out, float scale, uint32_t *status, int split_tokens,
              int num_splits, int capacity, float *part_o, float *part_m, float *part_l,
              unsigned long long *unit_ctr, cudaStream_t stream, const RowExtras &ex = RowExtras()) {
  CUtensorMap tk, tv;
  int rc = encode_maps(sh, k, v, &tk, &tv);
  if (rc != GQA_OK) return rc;
  DecodeParams p = base_params(sh, q, seqlens, pt, status, scale);
  p.out = out;
  p.part_o = part_o;
  p.part_m = part_m;
  p.part_l = part_l;
  p.capacity = capacity;
  p.split_tokens = split_tokens;
  p.num_splits = num_splits;
  p.unit_ctr = unit_ctr;
  p.epoch = unit_ctr ? next_epoch() : 0;
  p.lse = ex.lse;
  p.empty_ok = ex.empty_ok ? 1 : 0;
  if (ex.group_of_head) {
    p.mapped = 1;
    fill_group_map(ex.group_of_head, sh.H, sh.G, sh.rc, &p.map);
  }
  const long long items = units_of(sh) * num_splits;
  if (items > (1ll << 31) - 1) return GQA_ERR_DIMS;
  // Programmatic dependent launch pays off when the grid follows a short or
  // partly idle kernel (a combine, a previous step's merge); with one item per
  // unit the mma.sync grid follows a full decode grid, where measured it cost
  // ~1-3 % (its early blocks only wait, and the grid no longer starts as one
  // wave); the tcgen05 grid of one item per unit gains ~1 % from it (its
  // blocks set up tensor memory and prefetch while the previous grid ends).
  Launch l{dim3(static_cast<unsigned>(items), 1, 1), 1, stream, num_splits > 1 || ex.force_pdl || sh.tc};
  if (l.pdl) p.prefetch_tiles = prefetch_tiles(sh, items, split_tokens);
  if (sh.tc) return launch_verify_tc(sh, tk, tv, p, l);
  return launch_decode<Mode::kItems>(sh, tk, tv, p, l);
}

// ------------------------------------------------------------------ balanced mode
// Workspace: a 256-byte header {decode blocks, capacity, total tiles} and one
// record per (sequence, group) unit {first block, last block, slot}, both
// written by the decode kernel for the combine, then the partial states
// o [blocks][2][r][d], m and l [blocks][2][r].
struct BalancedWorkspace {
  size_t meta_off, o_off, m_off, l_off, total;
};

BalancedWorkspace balanced_layout(const Shape &sh) {
  BalancedWorkspace w;
  const size_t rows = static_cast<size_t>(kMaxBalancedBlocks) * 2 * sh.rc;
  w.meta_off = 256;
  w.o_off = w.meta_off + round256(static_cast<size_t>(units_of(sh)) * 16);
  w.m_off = w.o_off + round256(rows * sh.D * sizeof(float));
  w.l_off = w.m_off + round256(rows * sizeof(float));
  w.total = w.l_off + round256(rows * sizeof(float));
  return w;
}

size_t auto_workspace_bytes(const Shape &sh, int max_seqlen) {
  const long long units = units_of(sh);
  const long long by_sms = 3ll * 256;  // one wave of up to three blocks per SM on GPUs of up to 256 SMs
  long long splits = std::max<long long>((max_seqlen + kFallbackSplit - 1) / kFallbackSplit,
                                         (by_sms + units - 1) / units);
  splits = std::min<long long>(splits, (max_seqlen + kSplitQuantum - 1) / kSplitQuantum);
  return std::max(balanced_layout(sh).total, workspace_layout(sh, static_cast<int>(splits)).total);
}

int run_balanced_decode(const Shape &sh, int sms, const void *q, const void *k, const void *v,
                        const int32_t *seqlens, const int32_t *pt, float *out, float scale,
                        uint32_t *status, int32_t max_seqlen, void *workspace, cudaStream_t stream,
                        const RowExtras &ex = RowExtras()) {
  CUtensorMap tk, tv;
  int rc = encode_maps(sh, k, v, &tk, &tv);
  if (rc != GQA_OK) return rc;
  const BalancedWorkspace ws = balanced_layout(sh);
  uint8_t *w = static_cast<uint8_t *>(workspace);
  DecodeParams p = base_params(sh, q, seqlens, pt, status, scale);
  p.out = out;
  p.ws_header = reinterpret_cast<int *>(w);
  p.ws_meta = reinterpret_cast<int4 *>(w + ws.meta_off);
  p.part_o = reinterpret_cast<float *>(w + ws.o_off);
  p.part_m = reinterpret_cast<float *>(w + ws.m_off);
  p.part_l = reinterpret_cast<float *>(w + ws.l_off);
  p.capacity = static_cast<int>(std::min<long long>(sh.capacity, max_seqlen));
  p.b = sh.b;
  p.lse = ex.lse;
  p.empty_ok = ex.empty_ok ? 1 : 0;
  if (ex.group_of_head) {
    p.mapped = 1;
    fill_group_map(ex.group_of_head, sh.H, sh.G, sh.rc, &p.map);
    p.ups = p.map.n_slices;
  }
  Launch l{dim3(static_cast<unsigned>(sms), 1, 1), 1, stream};
  rc = launch_decode<Mode::kBalanced>(sh, tk, tv, p, l);
  return rc < 0 ? rc : GQA_OK;
}

int run_balanced_combine(const Shape &sh, const int32_t *seqlens, float *out, uint32_t *status,
                         const void *workspace, cudaStream_t stream, const RowExtras &ex = RowExtras()) {
  const BalancedWorkspace ws = balanced_layout(sh);
  const uint8_t *w = static_cast<const uint8_t *>(workspace);
  CombineParams c{};
  c.seqlens = seqlens;
  c.out = out;
  c.ws_header = reinterpret_cast<const int *>(w);
  c.ws_meta = reinterpret_cast<const int4 *>(w + ws.meta_off);
  c.part_o = reinterpret_cast<const float *>(w + ws.o_off);
  c.part_m = reinterpret_cast<const float *>(w + ws.m_off);
  c.part_l = reinterpret_cast<const float *>(w + ws.l_off);
  c.status = status;
  c.b = sh.b;
  c.H = sh.H;
  c.G = sh.G;
  c.r = sh.r;
  c.rc = sh.rc;
  c.hs = sh.hs;
  c.nq = sh.nq;
  c.rq = sh.rq;
  c.lse = ex.lse;
  c.empty_ok = ex.empty_ok ? 1 : 0;
  c.ups = sh.G * sh.hs;
  if (ex.group_of_head) {
    c.mapped = 1;
    fill_group_map(ex.group_of_head, sh.H, sh.G, sh.rc, &c.map);
    c.ups = c.map.n_slices;
  }
  cudaLaunchConfig_t cfg = {};
  const int rows_per_block = 128 / (sh.D / 4);  // the combine's rows per block
  cfg.gridDim = dim3(static_cast<unsigned>(static_cast<long long>(sh.b) * c.ups *
                                           ((sh.rc + rows_per_block - 1) / rows_per_block)), 1, 1);
  cfg.blockDim = dim3(128, 1, 1);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = sh.D == 128 ? cudaLaunchKernelEx(&cfg, gqa::gqa_combine_balanced_kernel<128, 64>, c)
                              : cudaLaunchKernelEx(&cfg, gqa::gqa_combine_balanced_kernel<64, 128>, c);
  return e == cudaSuccess ? GQA_OK : GQA_ERR_CUDA;
}

// split_tokens == 0 in the split API: the library's choice, made from the
// dims, max_seqlen and the SM count only, so that gqa_split_partials and
// gqa_split_combine make the same one.  A paged pool (dims->max_pages_per_seq
// > 0) is the layout of choice for sequences of unequal lengths, so it gets
// equal-work ranges (for up to kMaxBalancedBatch sequences; fixed 4096-token
// splits beyond).  A contiguous cache gets fixed splits: one per (sequence,
// group) when the units already give 1.5 blocks per SM, else just enough
// splits for that.
struct AutoChoice {
  bool balanced;
  int split_tokens;
};

bool dims_paged(const gqa_dims *dims) { return dims->max_pages_per_seq > 0; }

// Equal-work ranges serve paged dims (with or without a group table), not the
// tcgen05 kernel (fixed splits only).
bool balanced_ok(const gqa_dims *dims, const Shape &sh) { return dims_paged(dims) && !sh.tc; }

int round_split(long long tokens) {
  tokens = (tokens + kSplitQuantum - 1) / kSplitQuantum * kSplitQuantum;
  return static_cast<int>(std::max<long long>(kSplitQuantum, tokens));
}

// Resident blocks per SM of the items kernel variant the shape runs (B200:
// shared memory allows two blocks of the 3-stage ring; the 288- and 544-thread
// variants for r > 16 fit once by registers).
int blocks_per_sm(const Shape &sh) {
  if (sh.tc) return 1;
  if (sh.fma || sh.nhb != 1) return 2;
  switch (pick_pipe(sh)) {
    case Pipe::kTrio: return 3;
    case Pipe::kSolo: return 1;
    default: return 2;
  }
}

constexpr int kNoSplitTokens = 256;

AutoChoice choose_auto(const Shape &sh, bool paged, int max_seqlen, int sms) {
  if (paged) {
    if (sh.b <= kMaxBalancedBatch) return {true, 0};
    return {false, kFallbackSplit};
  }
  // A unit of at most kNoSplitTokens is not split: merging two halves costs
  // more than the streaming they save (device-timed, graph replays: 256
  // tokens at d = 128 in one split 6.3-6.7 us against 7.8-8.3 in two, at
  // d = 64 4.8 against 6.7; from 512 tokens on, splits win).
  if (max_seqlen <= kNoSplitTokens) return {false, round_split(max_seqlen)};
  // One block per unit when the units fill three quarters of the resident
  // slots; otherwise as many splits as still fit one wave.
  const long long units = units_of(sh);
  const long long slots = static_cast<long long>(sms) * blocks_per_sm(sh);
  const long long splits = 4 * units >= 3 * slots ? 1 : std::max<long long>(1, slots / units);
  return {false, round_split((max_seqlen + splits - 1) / splits)};
}

// split_tokens == 0 in gqa_decode_split (and its verification, lse and group
// map forms): a contiguous cache whose (sequence, group) units are too few to
// fill the GPU one block each runs the cluster decomposition of gqa_decode
// instead of fixed splits when that fills at least three quarters of the
// resident blocks with portable clusters (<= 8 blocks): one kernel, the splits
// of a unit merged through distributed shared memory, no workspace.  The
// cluster kernel writes final rows (and their lse) only, so the partial-state
// entry points keep fixed splits; the tcgen05 and CUDA-core paths do too.
// Returns the blocks per cluster, or 0 for the fixed-split / equal-work plan.
int auto_cluster(const Shape &sh, bool paged, int sms) {
  if (paged || sh.tc || sh.fma) return 0;
  const int c = cluster_plan(sh, sms);
  if (c < 2 || c > 8) return 0;
  const long long blocks = units_of(sh) * c;
  const long long slots = static_cast<long long>(sms) * blocks_per_sm(sh);
  return (4 * blocks >= 3 * slots && 10 * blocks <= 9 * slots) ? c : 0;
}

// Whether the cluster decomposition's clusters all fit the current device at
// once (thread-block clusters must sit inside one GPC; on B200 eight blocks
// of one SM each fit 15 times, of half an SM each 33 times).
bool cluster_fits(const Shape &sh, int c) {
  CUtensorMap tk{}, tv{};
  DecodeParams p{};
  Launch l{dim3(c, sh.G * sh.hs, sh.b), c, nullptr, true};
  l.query = true;
  return launch_decode<Mode::kCluster>(sh, tk, tv, p, l) == 1;
}

// split_tokens == 0 in the split API: checks shared by its entry points.
int prepare_auto(const gqa_dims *dims, bool paged, int32_t max_seqlen, const void *workspace,
                 size_t workspace_bytes, Shape *sh, int nq = 1, const int32_t *group_of_head = nullptr) {
  int rc = check_dims(dims, paged, sh, nq, group_of_head);
  if (rc != GQA_OK) return rc;
  if (max_seqlen < 1) return GQA_ERR_DIMS;
  if (!workspace) return GQA_ERR_WORKSPACE;
  if (!aligned16(workspace)) return GQA_ERR_MISALIGNED;
  if (workspace_bytes < auto_workspace_bytes(*sh, max_seqlen)) return GQA_ERR_WORKSPACE;
  return GQA_OK;
}

struct SplitArgs {
  Shape sh;
  int split_tokens, num_splits;
  Workspace ws;
};

int prepare_split(const gqa_dims *dims, bool paged, int32_t split_tokens, int32_t max_seqlen,
                  const void *workspace, size_t workspace_bytes, int sms, SplitArgs *out, int nq = 1,
                  const int32_t *group_of_head = nullptr) {
  int rc = check_dims(dims, paged, &out->sh, nq, group_of_head);
  if (rc != GQA_OK) return rc;
  if (max_seqlen < 1) return GQA_ERR_DIMS;
  if (split_tokens <= 0 || split_tokens % kSplitQuantum != 0) return GQA_ERR_SPLIT;
  (void)sms;
  out->split_tokens = split_tokens;
  out->num_splits = (max_seqlen + split_tokens - 1) / split_tokens;
  if (out->num_splits > 65535) return GQA_ERR_SPLIT;
  out->ws = workspace_layout(out->sh, out->num_splits);
  if (!workspace) return GQA_ERR_WORKSPACE;
  if (!aligned16(workspace)) return GQA_ERR_MISALIGNED;
  if (workspace_bytes < out->ws.total) return GQA_ERR_WORKSPACE;
  return GQA_OK;
}

// merge_here: the decode kernel merges each unit's splits itself (the block
// that completes a unit does it); otherwise the partial states are left for
// gqa_split_combine.
int run_partials(const SplitArgs &a, const void *q, const void *k, const void *v,
                 const int32_t *seqlens, const int32_t *pt, float *out, float scale, uint32_t *status,
                 int32_t max_seqlen, void *workspace, bool merge_here, cudaStream_t stream,
                 const RowExtras &ex = RowExtras()) {
  uint8_t *w = static_cast<uint8_t *>(workspace);
  const int capacity = static_cast<int>(std::min<long long>(a.sh.capacity, max_seqlen));
  return run_items(a.sh, q, k, v, seqlens, pt, out, scale, status, a.split_tokens, a.num_splits,
                   capacity, reinterpret_cast<float *>(w), reinterpret_cast<float *>(w + a.ws.o_bytes),
                   reinterpret_cast<float *>(w + a.ws.o_bytes + a.ws.m_bytes),
                   merge_here ? reinterpret_cast<unsigned long long *>(w + a.ws.ctr_off) : nullptr, stream, ex);
}

int run_combine(const SplitArgs &a, const int32_t *seqlens, float *out, uint32_t *status,
                int32_t max_seqlen, const void *workspace, cudaStream_t stream,
                const RowExtras &ex = RowExtras()) {
  CombineParams c{};
  const uint8_t *w = static_cast<const uint8_t *>(workspace);
  c.seqlens = seqlens;
  c.out = out;
  c.part_o = reinterpret_cast<const float *>(w);
  c.part_m = reinterpret_cast<const float *>(w + a.ws.o_bytes);
  c.part_l = reinterpret_cast<const float *>(w + a.ws.o_bytes + a.ws.m_bytes);
  c.status = status;
  c.b = a.sh.b;
  c.H = a.sh.H;
  c.max_len = max_seqlen;
  c.split_tokens = a.split_tokens;
  c.num_splits = a.num_splits;
  c.lse = ex.lse;
  c.empty_ok = ex.empty_ok ? 1 : 0;
  c.nq = a.sh.nq;
  c.rq = a.sh.rq;
  const int rows = a.sh.b * a.sh.nq * a.sh.H;
  cudaLaunchConfig_t cfg = {};
  // many splits: 512 threads, so that every split's row loads in one round
  const bool wide = a.num_splits > gqa::kSerialMergeMax;
  cfg.gridDim = dim3(rows, 1, 1);
  cfg.blockDim = dim3(wide ? 512 : 128, 1, 1);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e;
  if (wide)
    e = a.sh.D == 128 ? cudaLaunchKernelEx(&cfg, gqa::gqa_combine_kernel<128, 512>, c)
                      : cudaLaunchKernelEx(&cfg, gqa::gqa_combine_kernel<64, 512>, c);
  else
    e = a.sh.D == 128 ? cudaLaunchKernelEx(&cfg, gqa::gqa_combine_kernel<128, 128>, c)
                      : cudaLaunchKernelEx(&cfg, gqa::gqa_combine_kernel<64, 128>, c);
  return e == cudaSuccess ? GQA_OK : GQA_ERR_CUDA;
}

// The cluster decomposition (gqa_decode, and gqa_decode_split's choice for
// contiguous caches with few units): grid (c, G x slices, b), clusters of c.
int run_cluster(const Shape &sh, int c, const void *q, const void *k, const void *v, const int32_t *seqlens,
                const int32_t *pt, float *out, float scale, uint32_t *status, cudaStream_t st,
                const RowExtras &ex = RowExtras()) {
  CUtensorMap tk, tv;
  int rc = encode_maps(sh, k, v, &tk, &tv);
  if (rc != GQA_OK) return rc;
  DecodeParams p = base_params(sh, q, seqlens, pt, status, scale);
  p.out = out;
  p.lse = ex.lse;
  p.empty_ok = ex.empty_ok ? 1 : 0;
  if (ex.group_of_head) {
    p.mapped = 1;
    fill_group_map(ex.group_of_head, sh.H, sh.G, sh.rc, &p.map);
  }
  // launched as a programmatic dependent: the blocks set themselves up while
  // the previous kernel on the stream finishes
  Launch l{dim3(c, sh.G * sh.hs, sh.b), c, st, true};
  p.prefetch_tiles = prefetch_tiles(sh, units_of(sh) * c, static_cast<int>((sh.capacity + c - 1) / c));
  return launch_decode<Mode::kCluster>(sh, tk, tv, p, l);
}

}  // namespace

namespace {

int decode_split_impl(const void *q, const void *k_cache, const void *v_cache, const int32_t *seqlens,
                      const int32_t *page_table, float *out, const gqa_dims *dims, float scale,
                      uint32_t *status, int32_t split_tokens, int32_t max_seqlen, void *workspace,
                      size_t workspace_bytes, void *stream, const RowExtras &ex) {
  int rc = check_inputs(q, k_cache, v_cache, seqlens, status);
  if (rc != GQA_OK) return rc;
  if (!out) return GQA_ERR_NULL_POINTER;
  if (!aligned16(out)) return GQA_ERR_MISALIGNED;
  if (!std::isfinite(scale)) return GQA_ERR_DIMS;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (split_tokens == 0) {
    Shape sh;
    if ((rc = prepare_auto(dims, page_table != nullptr, max_seqlen, workspace, workspace_bytes, &sh, ex.nq,
                           ex.group_of_head)) != GQA_OK)
      return rc;
    DeviceInfo dev;
    if ((rc = current_device_info(&dev)) != GQA_OK) return rc;
    const int c = auto_cluster(sh, dims_paged(dims), std::min(dev.sms, 256));
    if (c > 0 && cluster_fits(sh, c))
      return run_cluster(sh, c, q, k_cache, v_cache, seqlens, page_table, out, scale, status, st, ex);
    const AutoChoice ch = choose_auto(sh, balanced_ok(dims, sh), max_seqlen, std::min(dev.sms, 256));
    if (ch.balanced) {
      rc = run_balanced_decode(sh, dev.sms, q, k_cache, v_cache, seqlens, page_table, out, scale, status,
                               max_seqlen, workspace, st, ex);
      if (rc != GQA_OK) return rc;
      return run_balanced_combine(sh, seqlens, out, status, workspace, st, ex);
    }
    split_tokens = ch.split_tokens;
  }
  SplitArgs a;
  rc = prepare_split(dims, page_table != nullptr, split_tokens, max_seqlen, workspace,
                     workspace_bytes, 0, &a, ex.nq, ex.group_of_head);
  if (rc != GQA_OK) return rc;
  DeviceInfo dev;
  if ((rc = current_device_info(&dev)) != GQA_OK) return rc;
  // Up to kSerialMergeMax splits: one launch, single-split rows final in their
  // block and the others merged by the block that completes their unit.  More
  // splits: their merge is too much work for one block, the combine kernel
  // spreads it over one block per row.
  const bool merge_here = a.num_splits <= gqa::kSerialMergeMax;
  rc = run_partials(a, q, k_cache, v_cache, seqlens, page_table, out, scale, status, max_seqlen,
                    workspace, merge_here, st, ex);
  if (rc != GQA_OK || merge_here) return rc;
  return run_combine(a, seqlens, out, status, max_seqlen, workspace, st, ex);
}

}  // namespace

// ====================================================================== C ABI
extern "C" {

int32_t gqa_abi_version(void) { return (1 << 16) | 0; }

#ifdef GQA_TEST_HOOKS
// Test library only (not declared in gqa.h): the producer of decode block
// `block` leaves out the K/V tile at ring position `ring_pos` of its pipeline
// (-1, -1: none), so that a test can make a bounded wait run out.
int gqa_test_skip_tile(int32_t block, int32_t ring_pos) {
  const int v[2] = {block, ring_pos};
  return cudaMemcpyToSymbol(gqa::g_test_skip_tile, v, sizeof(v)) == cudaSuccess ? GQA_OK : GQA_ERR_CUDA;
}
#endif

const char *gqa_status_string(int code) {
  switch (code) {
    case GQA_OK: return "ok";
    case GQA_ERR_NULL_POINTER: return "a required pointer is NULL";
    case GQA_ERR_MISALIGNED: return "a buffer is not 16-byte aligned";
    case GQA_ERR_HEADS: return "num_heads is not a multiple of num_kv_heads, or the group ratio exceeds 64";
    case GQA_ERR_HEAD_DIM: return "head_dim must be 64 or 128";
    case GQA_ERR_PAGE_SIZE: return "page_size must be a power of two in [8, 2^20]";
    case GQA_ERR_DIMS: return "a size or flag is out of range";
    case GQA_ERR_SPLIT: return "split_tokens must be 0 or a positive multiple of 128";
    case GQA_ERR_WORKSPACE: return "workspace missing or too small";
    case GQA_ERR_CUDA: return "a CUDA call failed";
    case GQA_ERR_DEVICE: return "the current device is not an sm_100 (B200) GPU";
    case GQA_ERR_NO_PAGES: return "the page pool has fewer free pages than requested";
    default: return "unknown status";
  }
}

int gqa_decode(const void *q, const void *k_cache, const void *v_cache, const int32_t *seqlens,
               const int32_t *page_table, float *out, const gqa_dims *dims, float scale,
               uint32_t *status, void *stream) {
  Shape sh;
  int rc = check_dims(dims, page_table != nullptr, &sh, 1, nullptr, /*auto_tc=*/false);
  if (rc != GQA_OK) return rc;
  if (sh.tc) return GQA_ERR_DIMS;  // the tcgen05 kernel runs behind the split entry points only
  rc = check_inputs(q, k_cache, v_cache, seqlens, status);
  if (rc != GQA_OK) return rc;
  if (!out) return GQA_ERR_NULL_POINTER;
  if (!aligned16(out)) return GQA_ERR_MISALIGNED;
  if (!std::isfinite(scale)) return GQA_ERR_DIMS;
  DeviceInfo dev;
  if ((rc = current_device_info(&dev)) != GQA_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int c = cluster_plan(sh, dev.sms);
  if (c == 1) {
    // enough (sequence, group) units: one item each, final rows, no scratch
    const int split = static_cast<int>((sh.capacity + kSplitQuantum - 1) / kSplitQuantum * kSplitQuantum);
    return run_items(sh, q, k_cache, v_cache, seqlens, page_table, out, scale, status, split, 1,
                     static_cast<int>(sh.capacity), nullptr, nullptr, nullptr, nullptr, st);
  }
  return run_cluster(sh, c, q, k_cache, v_cache, seqlens, page_table, out, scale, status, st);
}

size_t gqa_decode_split_workspace_size(const gqa_dims *dims, int32_t max_seqlen, int32_t split_tokens) {
  Shape sh;  // only b, H and d matter here
  if (!dims || check_dims(dims, false, &sh) != GQA_OK) return 0;
  if (max_seqlen < 1 || split_tokens < 0 || split_tokens % kSplitQuantum != 0) return 0;
  if (split_tokens == 0) return auto_workspace_bytes(sh, max_seqlen);
  const int splits = (max_seqlen + split_tokens - 1) / split_tokens;
  return workspace_layout(sh, splits).total;
}

int32_t gqa_plan_split_tokens(const gqa_dims *dims, int32_t max_seqlen, int32_t num_sms) {
  Shape sh;
  if (!dims) return GQA_ERR_NULL_POINTER;
  int rc = check_dims(dims, false, &sh);
  if (rc != GQA_OK) return rc;
  if (max_seqlen < 1) return GQA_ERR_DIMS;
  if (num_sms <= 0) {
    DeviceInfo dev;
    if ((rc = current_device_info(&dev)) != GQA_OK) return rc;
    num_sms = dev.sms;
  }
  const AutoChoice ch = choose_auto(sh, balanced_ok(dims, sh), max_seqlen, std::min(num_sms, 256));
  return ch.balanced ? 0 : ch.split_tokens;
}

int32_t gqa_plan_decomposition(const gqa_dims *dims, int32_t max_seqlen, int32_t num_sms,
                               int32_t *split_tokens_out, int32_t *cluster_out) {
  return gqa_plan_decomposition_ex(dims, max_seqlen, 1, nullptr, num_sms, split_tokens_out, cluster_out);
}

int32_t gqa_plan_decomposition_ex(const gqa_dims *dims, int32_t max_seqlen, int32_t num_query_tokens,
                                  const int32_t *group_of_head, int32_t num_sms, int32_t *split_tokens_out,
                                  int32_t *cluster_out) {
  Shape sh;
  if (!dims) return GQA_ERR_NULL_POINTER;
  if (num_query_tokens < 1) return GQA_ERR_DIMS;
  int rc = check_dims(dims, dims_paged(dims), &sh, num_query_tokens, group_of_head);
  if (rc != GQA_OK) return rc;
  if (max_seqlen < 1) return GQA_ERR_DIMS;
  const bool on_device = num_sms <= 0;  // plan for the current device (its cluster occupancy included)
  if (on_device) {
    DeviceInfo dev;
    if ((rc = current_device_info(&dev)) != GQA_OK) return rc;
    num_sms = dev.sms;
  }
  num_sms = std::min(num_sms, 256);
  if (split_tokens_out) *split_tokens_out = 0;
  if (cluster_out) *cluster_out = 1;
  const int c = auto_cluster(sh, dims_paged(dims), num_sms);
  if (c > 0 && (!on_device || cluster_fits(sh, c))) {
    if (cluster_out) *cluster_out = c;
    return GQA_PLAN_CLUSTERS;
  }
  const AutoChoice ch = choose_auto(sh, balanced_ok(dims, sh), max_seqlen, num_sms);
  if (ch.balanced) return GQA_PLAN_EQUAL_WORK;
  if (split_tokens_out) *split_tokens_out = ch.split_tokens;
  return GQA_PLAN_FIXED_SPLITS;
}

int gqa_split_partials(const void *q, const void *k_cache, const void *v_cache,
                       const int32_t *seqlens, const int32_t *page_table, float *out,
                       const gqa_dims *dims, float scale, uint32_t *status, int32_t split_tokens,
                       int32_t max_seqlen, void *workspace, size_t workspace_bytes, void *stream) {
  int rc = check_inputs(q, k_cache, v_cache, seqlens, status);
  if (rc != GQA_OK) return rc;
  if (out && !aligned16(out)) return GQA_ERR_MISALIGNED;
  if (!std::isfinite(scale)) return GQA_ERR_DIMS;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (split_tokens == 0) {
    Shape sh;
    if ((rc = prepare_auto(dims, page_table != nullptr, max_seqlen, workspace, workspace_bytes, &sh)) != GQA_OK)
      return rc;
    DeviceInfo dev;
    if ((rc = current_device_info(&dev)) != GQA_OK) return rc;
    const AutoChoice ch = choose_auto(sh, balanced_ok(dims, sh), max_seqlen, std::min(dev.sms, 256));
    if (ch.balanced) {
      if (!out) return GQA_ERR_NULL_POINTER;  // whole units are finished straight into out
      return run_balanced_decode(sh, dev.sms, q, k_cache, v_cache, seqlens, page_table, out, scale,
                                 status, max_seqlen, workspace, st);
    }
    split_tokens = ch.split_tokens;
  }
  SplitArgs a;
  rc = prepare_split(dims, page_table != nullptr, split_tokens, max_seqlen, workspace, workspace_bytes,
                     0, &a);
  if (rc != GQA_OK) return rc;
  DeviceInfo dev;
  if ((rc = current_device_info(&dev)) != GQA_OK) return rc;
  return run_partials(a, q, k_cache, v_cache, seqlens, page_table, out, scale, status, max_seqlen,
                      workspace, false, st);
}

int gqa_split_combine(const int32_t *seqlens, float *out, const gqa_dims *dims, uint32_t *status,
                      int32_t split_tokens, int32_t max_seqlen, const void *workspace,
                      size_t workspace_bytes, void *stream) {
  if (!seqlens || !out) return GQA_ERR_NULL_POINTER;
  if (!aligned16(out)) return GQA_ERR_MISALIGNED;
  if ((reinterpret_cast<uintptr_t>(seqlens) & 3u) || (reinterpret_cast<uintptr_t>(status) & 3u))
    return GQA_ERR_MISALIGNED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int rc;
  if (split_tokens == 0) {
    Shape sh;  // the merge needs b, H, G and d only
    if ((rc = prepare_auto(dims, false, max_seqlen, workspace, workspace_bytes, &sh)) != GQA_OK) return rc;
    DeviceInfo dev;
    if ((rc = current_device_info(&dev)) != GQA_OK) return rc;
    const AutoChoice ch = choose_auto(sh, balanced_ok(dims, sh), max_seqlen, std::min(dev.sms, 256));
    if (ch.balanced) return run_balanced_combine(sh, seqlens, out, status, workspace, st);
    split_tokens = ch.split_tokens;
  }
  SplitArgs a;  // the merge needs b, H, d and the split geometry only
  rc = prepare_split(dims, false, split_tokens, max_seqlen, workspace, workspace_bytes, 0, &a);
  if (rc != GQA_OK) return rc;
  DeviceInfo dev;
  if ((rc = current_device_info(&dev)) != GQA_OK) return rc;
  return run_combine(a, seqlens, out, status, max_seqlen, workspace, st);
}

int gqa_decode_split(const void *q, const void *k_cache, const void *v_cache, const int32_t *seqlens,
                     const int32_t *page_table, float *out, const gqa_dims *dims, float scale,
                     uint32_t *status, int32_t split_tokens, int32_t max_seqlen, void *workspace,
                     size_t workspace_bytes, void *stream) {
  return decode_split_impl(q, k_cache, v_cache, seqlens, page_table, out, dims, scale, status, split_tokens,
                           max_seqlen, workspace, workspace_bytes, stream, RowExtras());
}

int gqa_decode_split_lse(const void *q, const void *k_cache, const void *v_cache, const int32_t *seqlens,
                         const int32_t *page_table, float *out, float *lse, const gqa_dims *dims, float scale,
                         uint32_t *status, int32_t split_tokens, int32_t max_seqlen, void *workspace,
                         size_t workspace_bytes, void *stream) {
  if (!lse) return GQA_ERR_NULL_POINTER;
  if (reinterpret_cast<uintptr_t>(lse) & 3u) return GQA_ERR_MISALIGNED;
  RowExtras ex;
  ex.lse = lse;
  ex.empty_ok = true;
  return decode_split_impl(q, k_cache, v_cache, seqlens, page_table, out, dims, scale, status, split_tokens,
                           max_seqlen, workspace, workspace_bytes, stream, ex);
}

int gqa_append_decode_split(const void *k_new, const void *v_new, const void *q, void *k_cache, void *v_cache,
                            int32_t *seqlens, const int32_t *page_table, float *out, const gqa_dims *dims,
                            float scale, uint32_t *status, int32_t split_tokens, int32_t max_seqlen,
                            void *workspace, size_t workspace_bytes, void *stream) {
  // every argument of the decode is checked before the append is launched
  Shape sh;
  int rc = check_dims(dims, page_table != nullptr, &sh);
  if (rc != GQA_OK) return rc;
  if ((rc = check_inputs(q, k_cache, v_cache, seqlens, status)) != GQA_OK) return rc;
  if (!out) return GQA_ERR_NULL_POINTER;
  if (!aligned16(out)) return GQA_ERR_MISALIGNED;
  if (!std::isfinite(scale) || max_seqlen < 1) return GQA_ERR_DIMS;
  if (split_tokens < 0 || split_tokens % kSplitQuantum != 0) return GQA_ERR_SPLIT;
  if (!workspace) return GQA_ERR_WORKSPACE;
  if (!aligned16(workspace)) return GQA_ERR_MISALIGNED;
  const size_t need = split_tokens == 0 ? auto_workspace_bytes(sh, max_seqlen)
                                        : workspace_layout(sh, (max_seqlen + split_tokens - 1) / split_tokens).total;
  if (workspace_bytes < need) return GQA_ERR_WORKSPACE;
  rc = gqa_kv_append(k_new, v_new, k_cache, v_cache, seqlens, page_table, dims, status, stream);
  if (rc != GQA_OK) return rc;
  RowExtras ex;
  ex.force_pdl = true;  // the decode's blocks are dispatched while the append runs
  return decode_split_impl(q, k_cache, v_cache, seqlens, page_table, out, dims, scale, status, split_tokens,
                           max_seqlen, workspace, workspace_bytes, stream, ex);
}

size_t gqa_decode_split_mapped_workspace_size(const gqa_dims *dims, const int32_t *group_of_head,
                                              int32_t max_seqlen, int32_t split_tokens) {
  Shape sh;
  if (!dims || !group_of_head || check_dims(dims, false, &sh, 1, group_of_head) != GQA_OK) return 0;
  if (max_seqlen < 1 || split_tokens < 0 || split_tokens % kSplitQuantum != 0) return 0;
  if (split_tokens == 0) return auto_workspace_bytes(sh, max_seqlen);
  return workspace_layout(sh, (max_seqlen + split_tokens - 1) / split_tokens).total;
}

int gqa_decode_split_mapped(const void *q, const void *k_cache, const void *v_cache, const int32_t *seqlens,
                            const int32_t *page_table, float *out, float *lse, const gqa_dims *dims,
                            const int32_t *group_of_head, float scale, uint32_t *status, int32_t split_tokens,
                            int32_t max_seqlen, void *workspace, size_t workspace_bytes, void *stream) {
  if (!group_of_head) return GQA_ERR_NULL_POINTER;
  if (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)) return GQA_ERR_MISALIGNED;
  RowExtras ex;
  ex.lse = lse;
  ex.group_of_head = group_of_head;
  return decode_split_impl(q, k_cache, v_cache, seqlens, page_table, out, dims, scale, status, split_tokens,
                           max_seqlen, workspace, workspace_bytes, stream, ex);
}

size_t gqa_decode_verify_workspace_size(const gqa_dims *dims, int32_t n_query, int32_t max_seqlen,
                                        int32_t split_tokens) {
  Shape sh;
  if (!dims || check_dims(dims, false, &sh, n_query) != GQA_OK) return 0;
  if (max_seqlen < 1 || split_tokens < 0 || split_tokens % kSplitQuantum != 0) return 0;
  if (split_tokens == 0) return auto_workspace_bytes(sh, max_seqlen);
  return workspace_layout(sh, (max_seqlen + split_tokens - 1) / split_tokens).total;
}

int gqa_decode_verify(const void *q, const void *k_cache, const void *v_cache, const int32_t *seqlens,
                      const int32_t *page_table, float *out, float *lse, const gqa_dims *dims, int32_t n_query,
                      float scale, uint32_t *status, int32_t split_tokens, int32_t max_seqlen, void *workspace,
                      size_t workspace_bytes, void *stream) {
  if (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)) return GQA_ERR_MISALIGNED;
  if (n_query < 1 || n_query > kMaxQueryTokens) return GQA_ERR_DIMS;
  RowExtras ex;
  ex.lse = lse;
  ex.nq = n_query;
  return decode_split_impl(q, k_cache, v_cache, seqlens, page_table, out, dims, scale, status, split_tokens,
                           max_seqlen, workspace, workspace_bytes, stream, ex);
}

int gqa_merge_lse(const float *o_parts, const float *lse_parts, int32_t n_parts, int64_t rows, int32_t head_dim,
                  float *out, float *lse_out, void *stream) {
  if (!o_parts || !lse_parts || !out) return GQA_ERR_NULL_POINTER;
  if (!aligned16(o_parts) || !aligned16(out) || (reinterpret_cast<uintptr_t>(lse_parts) & 3u) ||
      (reinterpret_cast<uintptr_t>(lse_out) & 3u))
    return GQA_ERR_MISALIGNED;
  if (head_dim != 64 && head_dim != 128) return GQA_ERR_HEAD_DIM;
  if (n_parts < 1 || rows < 1) return GQA_ERR_DIMS;
  const int rows_per_block = 128 / (head_dim / 4);
  const long long blocks = (rows + rows_per_block - 1) / rows_per_block;
  if (blocks > 0x7fffffffll) return GQA_ERR_DIMS;
  DeviceInfo dev;
  int rc = current_device_info(&dev);
  if (rc != GQA_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (head_dim == 128)
    gqa::gqa_merge_lse_kernel<128><<<static_cast<unsigned>(blocks), 128, 0, st>>>(o_parts, lse_parts, n_parts,
                                                                                    rows, out, lse_out);
  else
    gqa::gqa_merge_lse_kernel<64><<<static_cast<unsigned>(blocks), 128, 0, st>>>(o_parts, lse_parts, n_parts,
                                                                                   rows, out, lse_out);
  return cudaGetLastError() == cudaSuccess ? GQA_OK : GQA_ERR_CUDA;
}

}  // extern "C"
