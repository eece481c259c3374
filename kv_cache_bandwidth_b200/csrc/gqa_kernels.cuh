// gqa_kernels.cuh -- grouped-query attention decode kernels for B200 (sm_100a).
//
// The operation (see include/gqa.h): for every sequence s and query head i,
// out[s,i] = softmax_j(scale * q[s,i] . K[s,g(i),j]) V[s,g(i),j] with
// g(i) = i / (H/G), the group broadcast of the PyTorch module of
// "Grouped-Query Attention" (aiwiki) done inside the kernel instead of with
// repeat_interleave, as that page's closing note asks.
//
// One thread block owns one (sequence, KV group, row slice, token range)
// item.  The rows of a group are its r = H/G query heads (times the query
// tokens of a verification step, or the heads a group table assigns), cut
// into slices of at most 16.  The group's keys and values cross HBM once per
// slice and are shared on chip by the slice's rows:
//
//   * a producer warp bulk-copies the slice's q rows into shared memory and
//     streams K and V tiles of T tokens into a STAGES-deep shared-memory ring
//     with TMA (128-byte swizzle), translating logical pages through the page
//     table (a window of 32 page ids per warp, the next window prefetched);
//   * consumer warps (4 along the token axis x 1 or 2 row blocks of 8) run
//     the two small contractions on tensor cores with the roles of the
//     operands swapped so that the tile's tokens fill the M = 16 rows of
//     mma.m16n8k16 and the slice's rows the N = 8 columns:
//         S^T[tokens, heads] = K_tile q^T            (A = K from smem, B = q in registers)
//         O^T[d, heads]     += V_tile^T P^T           (A = V^T via ldmatrix.trans)
//     P^T goes from the accumulator layout of S^T to the B-operand layout with
//     movmatrix; it is split into a bf16 high part and a bf16 residual so that
//     the product keeps ~16 bits of the probabilities (a single bf16 rounding
//     would leave ~1e-3 relative error);
//   * online softmax in base 2: a running base (within 2^8 of the maximum) and
//     sum per head; the maximum is reduced across token rows with warp
//     shuffles and the accumulators rescaled by 2^(m_old - m_new) only when a
//     score passes the base by more than 8;
//   * at the end the consumer warps merge their states in shared memory and
//     write the normalised rows (a whole unit), or a split's partial state --
//     which the block completing the unit merges in place for up to 8 splits,
//     and a combine kernel otherwise -- or merge the blocks of a thread-block
//     cluster through distributed shared memory (cluster mode).
#pragma once

#include <cooperative_groups.h>
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#include "ptx.cuh"

namespace gqa {

namespace cg = cooperative_groups;

constexpr uint32_t kStatusBadSeqlen = 1u;
constexpr uint32_t kStatusBadPage = 2u;
constexpr uint32_t kStatusTimeout = 4u;

// Markers stored in the per-split sum l of the workspace instead of a sum.
constexpr float kLBadPage = -1.f;    // the split met a page id outside the pool
constexpr float kLBadLength = -2.f;  // split 0: the length is outside [1, capacity]
constexpr float kLFinal = -3.f;      // split 0: the only split already wrote the final row

// Largest thread-block cluster of the cluster mode (non-portable size).
constexpr int kMaxClusterBlocks = 16;

// kItems: one block per (sequence, group, split) item, blockIdx.x = item.
// kCluster: one block per cluster rank; the blocks of a cluster share one
// (sequence, group) and merge through distributed shared memory.
// kBalanced: stream-K.  The tiles of all (sequence, group) units, in that
// order, form one sequence that is cut into gridDim.x equal contiguous ranges;
// a block streams its range through one pipeline, finishing the units that lie
// wholly inside it and leaving partial states for the (at most two) units it
// shares with its neighbours.
enum class Mode { kItems, kCluster, kBalanced };

// Any query-head to KV-group table (items mode): the heads sorted by group
// (stable) and each group's first position in that order, so that group g
// serves heads map_heads[map_off[g] .. map_off[g + 1]).
constexpr int kMaxMapHeads = 256;
constexpr int kMaxMapGroups = 256;
struct GroupMap {
  uint8_t heads[kMaxMapHeads];
  uint16_t off[kMaxMapGroups + 1];
  // the (group, row slice) units that hold rows, in (group, slice) order:
  // equal-work ranges walk only these (a slice past a small group has none)
  uint8_t slice_g[kMaxMapHeads];
  uint8_t slice_j[kMaxMapHeads];
  uint16_t n_slices;
};

struct DecodeParams {
  const __nv_bfloat16 *q;     // [b, H, D]
  const int32_t *seqlens;     // [b]
  const int32_t *page_table;  // [b, max_pages] (paged) or nullptr
  float *out;                 // [b, H, D]; items mode: may be null (partials only)
  float *part_o;              // [b, H, S, D]; may be null when S == 1 and out is set
  float *part_m;              // [b, H, S]
  float *part_l;              // [b, H, S]
  uint32_t *status;           // optional
  int *ws_header;             // balanced mode: {decode blocks, capacity, W lo, W hi} for the combine
  int4 *ws_meta;              // balanced mode: per unit {first block, last block, slot in first block}
  float *lse;                 // [b, H] natural-log sum of exp(scale q.k) of each final row, or null
  int empty_ok;               // a length of 0 is valid: zero row, lse -inf, no status bit
  unsigned long long *unit_ctr;  // items mode: arrival word per unit, or null (the merge is left to the combine)
  unsigned long long epoch;      // items mode: this call's tag in the arrival words, 1 .. 2^40 - 2
  int H, G, r;                // query heads, KV groups, heads per group
  int nq, rq;                 // query tokens per sequence, rows per group (nq * r, token-major)
  int rc, hs;                 // rows per block (min(rq, 16)) and row slices per group (ceil(rq / rc))
  int page_size;              // paged: tokens per page; contiguous: capacity m
  int num_pages;              // paged: pages in the pool
  int max_pages;              // paged: page-table row stride
  int capacity;               // largest valid length
  int split_tokens;           // items mode: tokens per split
  int num_splits;             // items mode: S
  int b;                      // sequences
  float scale_log2;           // scale * log2(e)
  int mapped;                 // the group of each head comes from `map` (one query token)
  int ups;                    // balanced mode: units per sequence (G x hs, or the map's slices)
  int prefetch_tiles;         // items and cluster modes: tiles of the block's piece brought into L2
                              // before the wait for the previous kernel on the stream (0: none)
  GroupMap map;
};

struct CombineParams {
  const int32_t *seqlens;
  float *out;
  const float *part_o;
  const float *part_m;
  const float *part_l;
  uint32_t *status;
  int b, H, max_len, split_tokens, num_splits;
  int G, r, rc, hs;           // balanced mode
  int nq, rq;                 // query tokens per sequence, rows per group
  const int *ws_header;       // balanced mode: {decode blocks, capacity, W lo, W hi}
  const int4 *ws_meta;        // balanced mode: per unit {first block, last block, slot in first block}
  float *lse;                 // [b, H] or null, as in DecodeParams
  int empty_ok;
  int ups;                    // balanced mode: units per sequence
  int mapped;                 // balanced mode: rows resolve through `map`
  GroupMap map;
};

// Row of q / out ([b, nq, H] flattened) for row rho = t * r + h (query token t,
// head h of the group) of KV group g of sequence s.
__device__ __forceinline__ size_t out_row(int s, int g, int rho, int nq, int r, int H) {
  const int t = rho / r, h = rho - t * r;
  return (static_cast<size_t>(s) * nq + t) * H + static_cast<size_t>(g) * r + h;
}

// Row of q / out of row rho of KV group g of sequence s, with or without a
// group map.
__device__ __forceinline__ size_t row_of(const DecodeParams &p, int s, int g, int rho) {
  if (p.mapped) return static_cast<size_t>(s) * p.H + p.map.heads[p.map.off[g] + rho];
  return out_row(s, g, rho, p.nq, p.r, p.H);
}

// Rows of KV group g: nq * r, or the group's own size under a map.
__device__ __forceinline__ int group_rows(const DecodeParams &p, int g) {
  return p.mapped ? static_cast<int>(p.map.off[g + 1]) - static_cast<int>(p.map.off[g]) : p.rq;
}

// Group and row slice of unit u of a sequence (balanced mode): u = g hs + j,
// or the map's u-th slice that holds rows.
__device__ __forceinline__ void unit_gj(bool mapped, const GroupMap &map, int hs, int u, int *g, int *j) {
  if (mapped) {
    *g = map.slice_g[u];
    *j = map.slice_j[u];
  } else {
    *g = u / hs;
    *j = u % hs;
  }
}

// Natural-log sum of exp over a row from its base-2 state: the row's
// exponentials sum to L * 2^M, so ln(sum) = (M + log2 L) ln 2; -inf for a
// row without tokens.
__device__ __forceinline__ float lse_from_state(float M, float L) {
  const float kNegInf = -__int_as_float(0x7f800000);
  return (L > 0.f && M != kNegInf) ? (M + log2f(L)) * 0.6931471805599453f : kNegInf;
}

template <int D, int NT, int NHB, int CH, int STAGES, bool BAL = false>
struct Tile {
  static constexpr int kNWT = 4;                   // consumer warps along the token axis
  static constexpr int kHB = 8 * NT;               // query heads per consumer warp
  static constexpr int kNC = kNWT * NHB;           // consumer warps (NHB row blocks)
  static constexpr int kThreads = 32 * (kNC + 1);  // + one producer warp
  static constexpr int kT = kNWT * 16 * CH;        // tokens per pipeline stage
  static constexpr int kHalves = D / 64;           // 128-byte swizzle atoms per row
  static constexpr int kTileBytes = kT * D * 2;    // one K (or V) tile
  static constexpr int kStageBytes = 2 * kTileBytes;
  static constexpr int kRingBytes = STAGES * kStageBytes;
  static constexpr int kSteps = D / 16;            // k-steps of q.k, m-tiles of p.v
  static constexpr int kRPad = NHB * kHB;          // rows per block, padded
  static constexpr int kOStride = D + 4;           // padded merge row (floats)
  static constexpr int kQBytes = kRPad * D * 2;    // one q block
  static constexpr int kQSlots = BAL ? 2 : 1;      // double-buffered when pieces follow each other
  // Shared memory (after 1 KiB alignment): ring | [merge rows, balanced mode] |
  // q slots | per-warp m, l and per-head M, L | mbarriers | flags.  With one
  // piece per block the merge of the output accumulators reuses the ring once
  // every tile has been consumed; in balanced mode the ring is already taking
  // the next piece, so the merge rows have their own space.
  // One piece per block (items and cluster modes): once every tile has been
  // consumed the ring holds each consumer warp's raw O rows ([kNC][kHB]
  // [kOStride] floats from offset 0), then the block's merged rows (osum).
  // The cluster mode's receive area ([blocks][rows per owner][D + 4] floats,
  // blocks x rows <= kRPad + 16) reuses the warps' rows, which are dead by
  // then.  In balanced mode the ring is already taking the next piece, so the
  // merged rows have their own space after it.
  static constexpr int kWarpOBytes = kNC * kHB * kOStride * 4;
  static constexpr int kWarpOOff = 0;
  static constexpr int kOSumOff = BAL ? kRingBytes : kWarpOBytes;
  static constexpr int kRecvOff = 0;
  static_assert(BAL || kOSumOff + kRPad * kOStride * 4 <= kRingBytes, "warp rows and merged rows must fit in the ring");
  static_assert(BAL || (kRPad + 16) * (D + 4) * 4 <= kOSumOff, "cluster receive area must not reach the merged rows");
  static constexpr int kQOff = kRingBytes + (BAL ? kRPad * kOStride * 4 : 0);
  static constexpr int kMLOff = kQOff + kQSlots * kQBytes;
  static constexpr int kMLFloats = 2 * kNC * kHB + 2 * kRPad;
  static constexpr int kBarOff = (kMLOff + 4 * kMLFloats + 7) & ~7;
  static constexpr int kNumBars = 2 * STAGES + 2 * kQSlots;  // full, empty, q full, q empty
  static constexpr int kFlagOff = kBarOff + 8 * kNumBars;
  static constexpr int kNumFlags = STAGES + 3;     // bad tile per stage, abort, item bad, merge here
  static constexpr int kSmemBytes = 1024 + kFlagOff + 4 * kNumFlags;
  static constexpr int kMinBlocks = STAGES <= 2 ? 3 : (STAGES == 3 ? 2 : 1);

  static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");
};

// Byte offset of element (row, col) of a 128B-swizzled K/V tile (bf16, rows of
// D elements split into D/64 column halves of 128-byte rows).
template <int T>
__device__ __forceinline__ uint32_t swz_offset(int row, int col) {
  const int half = col >> 6;
  const int chunk = (col & 63) >> 3;
  return static_cast<uint32_t>(half * T * 128 + row * 128 + ((chunk ^ (row & 7)) << 4));
}

__device__ __forceinline__ uint32_t keep_halves(uint32_t v, bool keep_lo, bool keep_hi) {
  return (keep_lo ? (v & 0x0000ffffu) : 0u) | (keep_hi ? (v & 0xffff0000u) : 0u);
}

// One piece of work: the token range [t_begin, t_end) of KV group g of
// sequence s, and where its result goes.
struct Piece {
  int s, g, u, len, k, t_begin, t_end;  // u: balanced mode, the unit's index within its sequence
  int j, h0, nh;       // head slice j of the group: heads h0 .. h0 + nh - 1
  bool len_ok;
  bool final_row;      // balanced mode: the piece is the whole unit
  int slot;            // balanced mode: partial-state slot (2 per block)
  bool first_of_unit;  // balanced mode: the piece starts at the unit's first tile
  int last_block;      // balanced mode (first_of_unit): last block holding a tile of the unit
};

template <int T, Mode MODE>
__device__ __forceinline__ Piece make_item(const DecodeParams &p) {
  Piece it;
  if (MODE == Mode::kItems) {
    const int i = blockIdx.x;
    it.k = i % p.num_splits;
    const int t = i / p.num_splits;
    it.j = t % p.hs;
    const int sg = t / p.hs;
    it.g = sg % p.G;
    it.s = sg / p.G;
  } else {
    it.k = blockIdx.x;
    it.g = blockIdx.y / p.hs;
    it.j = blockIdx.y % p.hs;
    it.s = blockIdx.z;
  }
  it.h0 = it.j * p.rc;
  it.nh = min(p.rc, group_rows(p, it.g) - it.h0);  // <= 0: a slice past a small group (mapped)
  it.len = __ldg(p.seqlens + it.s);
  it.len_ok = it.len >= p.nq && it.len <= p.capacity;
  it.t_begin = 0;
  it.t_end = 0;
  it.final_row = false;
  it.slot = 0;
  it.first_of_unit = false;
  it.last_block = 0;
  if (it.len_ok) {
    if (MODE == Mode::kItems) {
      it.t_begin = it.k * p.split_tokens;
      it.t_end = min(it.len, it.t_begin + p.split_tokens);
    } else {
      const int tiles = (it.len + T - 1) / T;
      const long long c = gridDim.x;
      it.t_begin = static_cast<int>((it.k * static_cast<long long>(tiles)) / c) * T;
      it.t_end = min(it.len, static_cast<int>(((it.k + 1) * static_cast<long long>(tiles)) / c) * T);
    }
  }
  return it;
}

// Before the wait for the previous kernel on the stream (a programmatic
// dependent launch lets the block start while that kernel still runs): bring
// the first p.prefetch_tiles tiles of the block's piece into L2, so that the
// HBM reads of this step overlap the tail of the previous one (its last
// blocks' merges).  The length and page ids read here (relaxed loads) may
// still be written by that kernel, so they are only a hint: they pick the
// addresses to prefetch
// (page ids outside the pool are skipped, coordinates outside the cache are
// skipped by the tensor map) and nothing else; the piece itself is computed
// from the values read after the wait.  One slice per unit prefetches (the
// slices of a unit read the same tiles).  Called by one warp.
template <int D, int T, Mode MODE, bool PAGED>
__device__ __forceinline__ void prefetch_piece_l2(const CUtensorMap *tm_k, const CUtensorMap *tm_v,
                                                  const DecodeParams &p, int lane) {
  if (MODE == Mode::kBalanced || p.prefetch_tiles <= 0) return;
  int k, g, j, s;
  if (MODE == Mode::kItems) {
    const int i = blockIdx.x;
    k = i % p.num_splits;
    const int t = i / p.num_splits;
    j = t % p.hs;
    const int sg = t / p.hs;
    g = sg % p.G;
    s = sg / p.G;
  } else {
    k = blockIdx.x;
    g = blockIdx.y / p.hs;
    j = blockIdx.y % p.hs;
    s = blockIdx.z;
  }
  if (j != 0 || p.mapped) return;
  const int len = ld_relaxed_gpu(p.seqlens + s);
  if (len < p.nq || len > p.capacity) return;
  int t_begin, t_end;
  if (MODE == Mode::kItems) {
    t_begin = k * p.split_tokens;
    t_end = min(len, t_begin + p.split_tokens);
  } else {
    const int tiles = (len + T - 1) / T;
    const long long c = gridDim.x;
    t_begin = static_cast<int>((k * static_cast<long long>(tiles)) / c) * T;
    t_end = min(len, static_cast<int>(((k + 1) * static_cast<long long>(tiles)) / c) * T);
  }
  t_end = min(t_end, t_begin + p.prefetch_tiles * T);
  constexpr int kHalves = D / 64;  // 64-element (128-byte) columns of a row
  if (!PAGED) {
    // box i: tile i / (2 kHalves), column (i / 2) % kHalves, K or V
    const int n = (t_end - t_begin + T - 1) / T * 2 * kHalves;
    for (int i = lane; i < n; i += 32) {
      const int t0 = t_begin + (i / (2 * kHalves)) * T, h = (i >> 1) % kHalves;
      tma_prefetch_l2_4d((i & 1) ? tm_v : tm_k, h * 64, t0, g, s);
    }
  } else {
    // one lane per box of min(P, T) rows: a page, or a T-row window of a large page
    const int P = p.page_size;
    const int br = min(P, T);
    const int32_t *pt_row = p.page_table + static_cast<size_t>(s) * p.max_pages;
    for (int tb = t_begin + lane * br; tb < t_end; tb += 32 * br) {
      const int id = ld_relaxed_gpu(pt_row + tb / P);
      if (id < 0 || id >= p.num_pages) continue;
#pragma unroll
      for (int h = 0; h < kHalves; ++h) {
        tma_prefetch_l2_4d(tm_k, h * 64, tb % P, g, id);
        tma_prefetch_l2_4d(tm_v, h * 64, tb % P, g, id);
      }
    }
  }
}

// Tiles of each (sequence, group) unit of sequence s; 0 for an invalid length.
template <int T>
__device__ __forceinline__ int unit_tiles(const int32_t *seqlens, int capacity, int nq, int s, int *len_out) {
  const int len = __ldg(seqlens + s);
  *len_out = len;
  return (len >= nq && len <= capacity) ? (len + T - 1) / T : 0;
}

__device__ __forceinline__ long long warp_sum64(long long v) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
  return v;
}

// Total tiles of all units, and the position of global tile `start` in the
// unit order (sequence-major, group-minor).  Every lane of the warp calls it
// and gets the same answer.
template <int T>
__device__ __forceinline__ long long total_tiles(const int32_t *seqlens, int b, int units_per_seq,
                                                 int capacity, int nq, int lane) {
  long long tot = 0;
  for (int base = 0; base < b; base += 32) {
    const int s = base + lane;
    int len;
    tot += (s < b) ? unit_tiles<T>(seqlens, capacity, nq, s, &len) : 0;
  }
  return warp_sum64(tot) * units_per_seq;
}

// Walks the pieces of this block's range in balanced mode.
struct Walker {
  long long remaining;  // tiles of the range not handed out yet
  long long pos;        // global index of the next tile handed out
  long long W;          // tiles of all units
  int s, u, g, j, tile_in, tiles_s, len_s, count;  // u: unit within the sequence, (g, j) its group and slice
};

template <int T>
__device__ __forceinline__ void walker_init(Walker &wk, const DecodeParams &p, int lane) {
  const long long W = total_tiles<T>(p.seqlens, p.b, p.ups, p.capacity, p.nq, lane);
  const long long N = gridDim.x, c = blockIdx.x;
  const long long start = c * W / N;
  wk.remaining = (c + 1) * W / N - start;
  wk.pos = start;
  wk.W = W;
  wk.s = wk.u = wk.g = wk.j = wk.tile_in = wk.tiles_s = wk.len_s = wk.count = 0;
  if (wk.remaining <= 0) {
    wk.remaining = 0;
    return;
  }
  long long acc = 0;
  for (int base = 0; base < p.b; base += 32) {
    const int s = base + lane;
    int len = 0;
    const long long t =
        (s < p.b) ? static_cast<long long>(unit_tiles<T>(p.seqlens, p.capacity, p.nq, s, &len)) * p.ups : 0;
    long long inc = t;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const long long v = __shfl_up_sync(0xffffffffu, inc, off);
      if (lane >= off) inc += v;
    }
    const long long chunk = __shfl_sync(0xffffffffu, inc, 31);
    if (start < acc + chunk) {
      const unsigned hit = __ballot_sync(0xffffffffu, start < acc + inc);
      const int L = __ffs(hit) - 1;
      const long long before = acc + __shfl_sync(0xffffffffu, inc - t, L);
      wk.s = base + L;
      wk.len_s = __shfl_sync(0xffffffffu, len, L);
      wk.tiles_s = (wk.len_s + T - 1) / T;
      const long long in_seq = start - before;
      wk.u = static_cast<int>(in_seq / wk.tiles_s);
      unit_gj(p.mapped, p.map, p.hs, wk.u, &wk.g, &wk.j);
      wk.tile_in = static_cast<int>(in_seq % wk.tiles_s);
      return;
    }
    acc += chunk;
  }
  wk.remaining = 0;  // not reached: start < W
}

template <int T>
__device__ __forceinline__ bool walker_next(Walker &wk, const DecodeParams &p, Piece &pc) {
  if (wk.remaining <= 0) return false;
  const int take = static_cast<int>(min(static_cast<long long>(wk.tiles_s - wk.tile_in), wk.remaining));
  pc.s = wk.s;
  pc.u = wk.u;
  pc.g = wk.g;
  pc.j = wk.j;
  pc.h0 = wk.j * p.rc;
  pc.nh = min(p.rc, group_rows(p, wk.g) - pc.h0);
  pc.k = 0;
  pc.len = wk.len_s;
  pc.len_ok = true;
  pc.t_begin = wk.tile_in * T;
  pc.t_end = min(wk.len_s, (wk.tile_in + take) * T);
  pc.final_row = (wk.tile_in == 0 && take == wk.tiles_s);
  pc.slot = 2 * static_cast<int>(blockIdx.x) + (wk.count == 0 ? 0 : 1);
  // the block that holds a unit's first tile records which blocks share it
  pc.first_of_unit = (wk.tile_in == 0);
  if (pc.first_of_unit) {
    const long long N = gridDim.x;
    pc.last_block = static_cast<int>(((wk.pos + wk.tiles_s) * N - 1) / wk.W);
  }
  ++wk.count;
  wk.pos += take;
  wk.remaining -= take;
  wk.tile_in = 0;
  if (wk.remaining > 0) {
    do {
      if (++wk.u == p.ups) {
        wk.u = 0;
        ++wk.s;
        wk.tiles_s = unit_tiles<T>(p.seqlens, p.capacity, p.nq, wk.s, &wk.len_s);
      }
    } while (wk.tiles_s == 0);
    unit_gj(p.mapped, p.map, p.hs, wk.u, &wk.g, &wk.j);
  }
  return true;
}

// Merge the partial states (m_k, l_k, o_k) of one output row:
//   M = max_k m_k,  L = sum_k l_k 2^(m_k - M),  out = sum_k o_k 2^(m_k - M) / L.
// Built for latency: the contributions are taken in chunks of 512; for each
// chunk every thread resolves one contribution's slot and loads its m and l
// (all in flight together), the 128 threads reduce the maximum, each thread
// turns its m into a weight, and then kNG groups of D/4 threads (one float4 of
// the row each) add up the weighted o rows with precomputed addresses, several
// loads in flight per thread.  Chunks are merged online (rescaled by
// 2^(M_old - M_new)); the groups are summed in a fixed order, so the result is
// deterministic and the same wherever it runs (combine kernel or the decode
// kernel's own merge).  `slot(k)` is the index of contribution k in the m/l
// arrays (< 0: no contribution).  Any l < 0 (an invalid page) makes the row
// zero.  The partial states are read through L2 (they may come from other
// blocks of the same grid).  NTH threads (tid 0 .. NTH-1) take part; `sync`
// is their barrier and `sc` their shared scratch.
template <int D, int NTH = 128>
struct MergeScratch {
  static constexpr int kTPR = D / 4;        // threads per row (one float4 each)
  static constexpr int kNG = NTH / kTPR;    // row groups
  static constexpr int kNW = NTH / 32;      // warps
  static constexpr int kChunk = 512;        // contributions per round
  float4 acc[kNG][kTPR];
  long long ps[kChunk];
  float w[kChunk], l[kChunk];
  float wmax[kNW], L[kNG];
  int wbad[kNW];
};

template <int D, int NTH, typename SlotFn, typename SyncFn>
__device__ __forceinline__ void merge_row(const float *part_o, const float *part_m, const float *part_l,
                                          int n_contrib, SlotFn slot, float4 *dst, float *lse_dst, int tid,
                                          MergeScratch<D, NTH> &sc, SyncFn sync) {
  using SC = MergeScratch<D, NTH>;
  constexpr int kTPR = SC::kTPR;
  constexpr int kNG = SC::kNG;
  constexpr int kChunk = SC::kChunk;
  const float kNegInf = -__int_as_float(0x7f800000);
  const int grp = tid / kTPR, c4 = tid % kTPR;
  const int warp = tid >> 5, lane = tid & 31;

  float M = kNegInf;  // running maximum (the same in every thread)
  float L = 0.f;      // this group's running sum of l weights
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  int bad = 0;
  for (int base = 0; base < n_contrib && !bad; base += kChunk) {
    const int cnt = min(kChunk, n_contrib - base);
    float mx = kNegInf;
    int bd = 0;
    for (int i = tid; i < cnt; i += NTH) {
      const long long ps = slot(base + i);
      sc.ps[i] = ps;
      float m = kNegInf, l = 0.f;
      if (ps >= 0) {
        m = __ldcg(part_m + ps);
        l = __ldcg(part_l + ps);
      }
      sc.w[i] = m;
      sc.l[i] = l;
      mx = fmaxf(mx, m);
      bd |= l < 0.f;
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    bd = __any_sync(0xffffffffu, bd);
    if (lane == 0) {
      sc.wmax[warp] = mx;
      sc.wbad[warp] = bd;
    }
    sync();
    bad = 0;
#pragma unroll
    for (int w = 0; w < SC::kNW; ++w) {
      mx = fmaxf(mx, sc.wmax[w]);
      bad |= sc.wbad[w];
    }
    if (!bad && mx != kNegInf) {
      const float Mn = fmaxf(M, mx);
      const float rescale = (M == kNegInf) ? 0.f : ex2(M - Mn);
      L *= rescale;
      acc.x *= rescale;
      acc.y *= rescale;
      acc.z *= rescale;
      acc.w *= rescale;
      M = Mn;
      for (int i = tid; i < cnt; i += NTH) sc.w[i] = (sc.ps[i] >= 0) ? ex2(sc.w[i] - Mn) : 0.f;
      sync();
#pragma unroll 8
      for (int i = grp; i < cnt; i += kNG) {
        const long long ps = sc.ps[i];
        const float w = sc.w[i];
        if (ps >= 0) {
          const float4 v = __ldcg(reinterpret_cast<const float4 *>(part_o + ps * D) + c4);
          acc.x += v.x * w;
          acc.y += v.y * w;
          acc.z += v.z * w;
          acc.w += v.w * w;
          L += sc.l[i] * w;
        }
      }
    }
    sync();  // the chunk's shared arrays are reused
  }
  sc.acc[grp][c4] = acc;
  if (c4 == 0) sc.L[grp] = L;
  sync();
  if (grp == 0) {
    float4 t = make_float4(0.f, 0.f, 0.f, 0.f);
    float Lt = 0.f;
#pragma unroll
    for (int i = 0; i < kNG; ++i) {
      t.x += sc.acc[i][c4].x;
      t.y += sc.acc[i][c4].y;
      t.z += sc.acc[i][c4].z;
      t.w += sc.acc[i][c4].w;
      Lt += sc.L[i];
    }
    float4 res = make_float4(0.f, 0.f, 0.f, 0.f);
    if (!bad && Lt > 0.f) res = make_float4(t.x / Lt, t.y / Lt, t.z / Lt, t.w / Lt);
    *dst = res;
    if (lse_dst && c4 == 0) *lse_dst = bad ? kNegInf : lse_from_state(M, Lt);
  }
  sync();  // the scratch is free for the next row
}

// Items mode: the arrival word of a (sequence, group, head slice) unit with
// several splits holds {call tag: 40 bits, arrivals: 24 bits}.  Every block of
// the unit claims the word for its call when it starts: a word with another
// tag (an earlier call, or whatever the workspace held) is set to {tag, 0} by
// one compare-and-swap, and a word that already carries the tag is left alone.
// That happens microseconds before any block of the unit can finish, while the
// block's first K/V loads are in flight.  At the end every block counts its
// arrival with one atomic add, so arrivals that come together do not retry;
// the arrival that makes `need` resets the word to {tag, 0}, ready for a repeat
// of the same launch (a replayed CUDA graph keeps its tag).  The workspace
// therefore needs no clearing, and a word poisoned with any other tag is
// harmless.
__device__ __forceinline__ void unit_claim(unsigned long long *word, unsigned long long epoch) {
  unsigned long long cur = *reinterpret_cast<volatile unsigned long long *>(word);
  for (int i = 0; i < 64 && (cur >> 24) != epoch; ++i) {
    const unsigned long long prev = atomicCAS(word, cur, epoch << 24);
    if (prev == cur) return;
    cur = prev;  // another block of the unit claimed it first (or it changed): look again
  }
}

// Counts one split's arrival at its unit (after unit_claim by every block of
// the unit).  Returns true for the arrival that completes the unit.  A word
// that does not carry the call's tag (its claim gave up) sets the timeout bit
// and completes nothing.
__device__ __forceinline__ bool unit_arrive(unsigned long long *word, unsigned long long epoch, int need,
                                            uint32_t *status) {
  const unsigned long long old = atomicAdd(word, 1ull);
  if ((old >> 24) != epoch) {
    if (status) atomicOr(status, kStatusTimeout);
    return false;
  }
  const bool last = (old & 0xffffffull) + 1 == static_cast<unsigned long long>(need);
  if (last) atomicExch(word, epoch << 24);
  return last;
}

// NV float4 outputs (columns 4*c4 .. 4*c4+3 for c4 = c4_0 + i*c4_step, i < NV)
// of one merged row from the row's ns partial states at slots slot(0) ..
// slot(ns - 1) (a negative slot: no contribution; slot(0) is one), for rows
// with few splits (one round trip to L2 per kSerialMergeMax of them).  Every thread works
// alone (no barriers) and issues all its loads before it uses any, so the
// merge costs about one trip to L2; each output takes the contributions in
// ascending k with one accumulator, the same whatever NV is.  The decode
// kernel's own merge and the combine kernel both use it for such rows, so the
// two agree bit for bit.
constexpr int kSerialMergeMax = 8;

template <int D, int NV, bool CHUNKED = false, typename SlotFn>
__device__ __forceinline__ void merge_serial_at(const float *part_o, const float *part_m, const float *part_l,
                                                SlotFn slot, int ns, int c4_0, int c4_step, float4 *dst_row,
                                                float *lse_dst) {
  const float kNegInf = -__int_as_float(0x7f800000);
  const long long first = slot(0);
  float M = kNegInf;  // running maximum over the chunks so far
  float L = 0.f;
  float4 acc[NV];
#pragma unroll
  for (int i = 0; i < NV; ++i) acc[i] = make_float4(0.f, 0.f, 0.f, 0.f);
  bool bad = false;
  // chunks of kSerialMergeMax contributions (CHUNKED; otherwise ns <=
  // kSerialMergeMax, one chunk), merged online: the sums so far are rescaled
  // by 2^(M_old - M_new)
  const int k_end = CHUNKED ? ns : 1;
  for (int k0 = 0; k0 < k_end; k0 += kSerialMergeMax) {
    float m[kSerialMergeMax], l[kSerialMergeMax];
    float4 v[NV][kSerialMergeMax];
    bool use[kSerialMergeMax];
#pragma unroll
    for (int k = 0; k < kSerialMergeMax; ++k) {
      long long kk = k0 + k < ns ? slot(k0 + k) : -1;
      use[k] = kk >= 0;
      if (!use[k]) kk = first;  // every load issued (unused ones repeat the first)
      m[k] = __ldcg(part_m + kk);
      l[k] = __ldcg(part_l + kk);
#pragma unroll
      for (int i = 0; i < NV; ++i)
        v[i][k] = __ldcg(reinterpret_cast<const float4 *>(part_o + kk * D) + c4_0 + i * c4_step);
    }
    float Mc = M;
#pragma unroll
    for (int k = 0; k < kSerialMergeMax; ++k) {
      if (use[k]) {
        Mc = fmaxf(Mc, m[k]);
        bad |= l[k] < 0.f;
      }
    }
    if (bad || Mc == kNegInf) continue;
    if (M != Mc) {
      const float r = (M == kNegInf) ? 0.f : ex2(M - Mc);
      L *= r;
#pragma unroll
      for (int i = 0; i < NV; ++i) {
        acc[i].x *= r;
        acc[i].y *= r;
        acc[i].z *= r;
        acc[i].w *= r;
      }
      M = Mc;
    }
#pragma unroll
    for (int k = 0; k < kSerialMergeMax; ++k) {
      if (use[k]) {
        const float w = ex2(m[k] - M);
        L += l[k] * w;
#pragma unroll
        for (int i = 0; i < NV; ++i) {
          acc[i].x += v[i][k].x * w;
          acc[i].y += v[i][k].y * w;
          acc[i].z += v[i][k].z * w;
          acc[i].w += v[i][k].w * w;
        }
      }
    }
  }
#pragma unroll
  for (int i = 0; i < NV; ++i) {
    float4 res = make_float4(0.f, 0.f, 0.f, 0.f);
    if (!bad && L > 0.f) res = make_float4(acc[i].x / L, acc[i].y / L, acc[i].z / L, acc[i].w / L);
    dst_row[c4_0 + i * c4_step] = res;
  }
  if (lse_dst && c4_0 == 0) *lse_dst = bad ? kNegInf : lse_from_state(M, L);
}

// merge_serial_at over the ns consecutive slots base .. base + ns - 1.
template <int D, int NV>
__device__ __forceinline__ void merge_serial(const float *part_o, const float *part_m, const float *part_l,
                                             long long base, int ns, int c4_0, int c4_step, float4 *dst_row,
                                             float *lse_dst) {
  merge_serial_at<D, NV>(part_o, part_m, part_l, [base](int k) -> long long { return base + k; }, ns, c4_0, c4_step,
                         dst_row, lse_dst);
}

// Items mode with arrival words, for kernels whose rows' partial states are
// written by NTH threads: count this split's arrival at its unit and, in the
// block whose split completes the unit, merge the unit's splits into the
// output rows (two float4 columns of one row per thread, half a row apart).
// Called by all NTH threads (named barrier 1) after the partial states are
// written.
template <int D, int NTH>
__device__ __forceinline__ void merge_unit_by_last(const DecodeParams &p, const Piece &pc, int tid,
                                                   volatile int *merge_here) {
  named_barrier(1, NTH);
  const int ns = (pc.len + p.split_tokens - 1) / p.split_tokens;
  if (tid == 0) {
    __threadfence();
    const size_t u = (static_cast<size_t>(pc.s) * p.G + pc.g) * p.hs + pc.j;
    *merge_here = unit_arrive(p.unit_ctr + u, p.epoch, ns, p.status) ? 1 : 0;
    __threadfence();
  }
  named_barrier(1, NTH);
  if (*merge_here) {
    constexpr int kHalfRow = D / 8;      // two float4 columns per thread, half a row apart
    constexpr int kQuarterRow = D / 16;  // four float4 columns per thread, a quarter row apart
    if (pc.nh > NTH / kHalfRow) {
      // more rows than one pass of half rows: quarter rows, every load of
      // the merge in flight at once
      for (int rb = 0; rb < pc.nh; rb += NTH / kQuarterRow) {
        const int h = rb + tid / kQuarterRow, c4 = tid % kQuarterRow;
        if (h < pc.nh) {
          const size_t mrow = row_of(p, pc.s, pc.g, pc.h0 + h);
          merge_serial<D, 4>(p.part_o, p.part_m, p.part_l, static_cast<long long>(mrow) * p.num_splits, ns, c4,
                             kQuarterRow, reinterpret_cast<float4 *>(p.out + mrow * D),
                             p.lse ? p.lse + mrow : nullptr);
        }
      }
    } else {
      for (int rb = 0; rb < pc.nh; rb += NTH / kHalfRow) {
        const int h = rb + tid / kHalfRow, c4 = tid % kHalfRow;
        if (h < pc.nh) {
          const size_t mrow = row_of(p, pc.s, pc.g, pc.h0 + h);
          merge_serial<D, 2>(p.part_o, p.part_m, p.part_l, static_cast<long long>(mrow) * p.num_splits, ns, c4,
                             kHalfRow, reinterpret_cast<float4 *>(p.out + mrow * D),
                             p.lse ? p.lse + mrow : nullptr);
        }
      }
    }
  }
}

// The q.k and p.v contractions on CUDA cores (fp32 FMA) for group ratios
// r <= RMAX <= 2, as the alternative to the tensor-core path.  Same pipeline, same
// piece, same merge: this consumes the piece's tiles and leaves the warp's
// running maximum / sum in m_sm / l_sm (heads r..7 as -inf / 0) and its share
// of the output rows accumulated in osum, exactly as the tensor-core path does.
//
// Lane layout per 16-token chunk: for q.k two lanes per token (lane = 2 t +
// half), each covering half of d with the bf16 pairs of q held in registers;
// for p.v each lane owns d/32 consecutive dims and takes token t's
// probability from lane 2 t by shuffle.  Rows past the range are skipped, so
// whatever they hold (even NaN) never enters the sums.
template <int D, int T, int CH, int STAGES, bool PAGED, int NWT, int HB, int OSTRIDE, int RMAX>
__device__ __forceinline__ int consume_fma(const DecodeParams &p, const Piece &pc, uint32_t q_slot,
                                           uint8_t *smem, uint32_t bar_full, uint32_t bar_empty,
                                           uint32_t bar_qempty_slot, volatile int *tile_bad,
                                           volatile int *abort_flag, float *m_sm, float *l_sm, float *osum,
                                           int &tile, int warp, int lane, int nc) {
  constexpr int kRMax = RMAX;      // heads held by each lane (r <= RMAX)
  constexpr int kPairs = D / 4;   // bf16 pairs of q per lane (half of d)
  constexpr int kDpl = D / 32;    // output dims per lane
  const float kNegInf = -__int_as_float(0x7f800000);
  constexpr int kTileBytes = T * D * 2;
  const int ws = warp % NWT;
  const int tk = lane >> 1, half = lane & 1;
  const int r = pc.nh;
  const float sl = p.scale_log2;

  uint32_t qf[kRMax][kPairs];
#pragma unroll
  for (int h = 0; h < kRMax; ++h) {
#pragma unroll
    for (int i = 0; i < kPairs; ++i)
      qf[h][i] = (h < r) ? ld_shared_u32(q_slot + h * D * 2 + (half * (D / 2) + 2 * i) * 2) : 0u;
  }
  __syncwarp();
  if (lane == 0) mbar_arrive(bar_qempty_slot);

  float m_run[kRMax], l_run[kRMax], o[kRMax][kDpl];
#pragma unroll
  for (int h = 0; h < kRMax; ++h) {
    m_run[h] = kNegInf;
    l_run[h] = 0.f;
#pragma unroll
    for (int i = 0; i < kDpl; ++i) o[h][i] = 0.f;
  }
  int bad = 0;
  for (int t0 = pc.t_begin; t0 < pc.t_end && !*abort_flag; t0 += T, ++tile) {
    const int stage = tile % STAGES;
    bool ok = mbar_wait(bar_full + 8 * stage, (tile / STAGES) & 1);
    ok = __shfl_sync(0xffffffffu, ok, 0);
    if (!ok) {
      if (lane == 0) {
        *abort_flag = 1;
        if (p.status) atomicOr(p.status, kStatusTimeout);
      }
      break;
    }
    if (PAGED) bad |= tile_bad[stage];
    const uint32_t kbase = smem_addr(smem + stage * 2 * kTileBytes);
    const uint32_t vbase = kbase + kTileBytes;
#pragma unroll
    for (int c = 0; c < CH; ++c) {
      const int row0 = (ws * CH + c) * 16;
      // ---- q.k: this lane's half of d for token row0 + tk
      float acc[kRMax];
#pragma unroll
      for (int h = 0; h < kRMax; ++h) acc[h] = 0.f;
#pragma unroll
      for (int ch8 = 0; ch8 < D / 16; ++ch8) {
        uint32_t kw[4];
        const uint32_t addr = kbase + swz_offset<T>(row0 + tk, half * (D / 2) + 8 * ch8);
        asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                     : "=r"(kw[0]), "=r"(kw[1]), "=r"(kw[2]), "=r"(kw[3])
                     : "r"(addr)
                     : "memory");
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float k0 = __uint_as_float(kw[e] << 16), k1 = __uint_as_float(kw[e] & 0xffff0000u);
#pragma unroll
          for (int h = 0; h < kRMax; ++h) {
            const uint32_t qw = qf[h][ch8 * 4 + e];
            acc[h] = fmaf(__uint_as_float(qw << 16), k0, acc[h]);
            acc[h] = fmaf(__uint_as_float(qw & 0xffff0000u), k1, acc[h]);
          }
        }
      }
      const bool live = t0 + row0 + tk < pc.t_end;
      float pr[kRMax];
#pragma unroll
      for (int h = 0; h < kRMax; ++h) {
        const float sdot = acc[h] + __shfl_xor_sync(0xffffffffu, acc[h], 1);
        const float x = live ? sdot * sl : kNegInf;
        float mx = x;
#pragma unroll
        for (int off = 2; off < 32; off <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
        const float mn = fmaxf(m_run[h], mx);
        const float base = (mn == kNegInf) ? 0.f : mn;
        pr[h] = ex2(x - base);
        if (mn != m_run[h]) {  // uniform across the warp
          const float alpha = ex2(m_run[h] - base);
          l_run[h] *= alpha;
#pragma unroll
          for (int i = 0; i < kDpl; ++i) o[h][i] *= alpha;
        }
        l_run[h] += half == 0 ? pr[h] : 0.f;
        m_run[h] = mn;
      }
      // ---- p.v: this lane's dims, token by token (rows past the range skipped)
      const int n_live = min(16, pc.t_end - (t0 + row0));
      for (int tt = 0; tt < n_live; ++tt) {
        float pt[kRMax];
#pragma unroll
        for (int h = 0; h < kRMax; ++h) pt[h] = __shfl_sync(0xffffffffu, pr[h], 2 * tt);
        const int col = lane * kDpl;
        const uint32_t addr = vbase + swz_offset<T>(row0 + tt, col & ~7) + (col & 7) * 2;
        float v[kDpl];
        if (kDpl == 4) {
          uint32_t w0, w1;
          asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(w0), "=r"(w1) : "r"(addr) : "memory");
          v[0] = __uint_as_float(w0 << 16);
          v[1] = __uint_as_float(w0 & 0xffff0000u);
          v[2] = __uint_as_float(w1 << 16);
          v[3] = __uint_as_float(w1 & 0xffff0000u);
        } else {
          const uint32_t w0 = ld_shared_u32(addr);
          v[0] = __uint_as_float(w0 << 16);
          v[1] = __uint_as_float(w0 & 0xffff0000u);
        }
#pragma unroll
        for (int h = 0; h < kRMax; ++h) {
#pragma unroll
          for (int i = 0; i < kDpl; ++i) o[h][i] = fmaf(pt[h], v[i], o[h][i]);
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(bar_empty + 8 * stage);
  }

  // ---- this warp's state into the merge arrays
#pragma unroll
  for (int h = 0; h < kRMax; ++h) {
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) l_run[h] += __shfl_xor_sync(0xffffffffu, l_run[h], off);
  }
  if (lane < HB) {
    float mv = kNegInf, lv = 0.f;
#pragma unroll
    for (int h = 0; h < kRMax; ++h) {
      if (lane == h && h < r) {
        mv = m_run[h];
        lv = l_run[h];
      }
    }
    m_sm[warp * HB + lane] = mv;
    l_sm[warp * HB + lane] = lv;
  }
  named_barrier(1, nc * 32);
  float f[kRMax];
#pragma unroll
  for (int h = 0; h < kRMax; ++h) {
    float M = kNegInf;
#pragma unroll
    for (int w2 = 0; w2 < NWT; ++w2) M = fmaxf(M, m_sm[w2 * HB + h]);
    f[h] = (M == kNegInf) ? 0.f : ex2(m_run[h] - M);
  }
  // deterministic accumulation: token slice 0 stores, slices 1..3 add in order
#pragma unroll
  for (int step = 0; step < NWT; ++step) {
    if (ws == step) {
#pragma unroll
      for (int h = 0; h < kRMax; ++h) {
        if (h < r) {
#pragma unroll
          for (int i = 0; i < kDpl; ++i) {
            float *dst = osum + h * OSTRIDE + lane * kDpl + i;
            const float v = o[h][i] * f[h];
            *dst = (step == 0) ? v : (*dst + v);
          }
        }
      }
    }
    named_barrier(1, nc * 32);
  }
  return bad;
}

// FMA: 0 runs the contractions on tensor cores; 1 or 2 runs them on CUDA
// cores for group ratios up to that value.
template <int D, int NT, int NHB, int CH, int STAGES, bool PAGED, Mode MODE, int FMA = 0>
__global__ void __launch_bounds__(Tile<D, NT, NHB, CH, STAGES, MODE == Mode::kBalanced>::kThreads,
                                  Tile<D, NT, NHB, CH, STAGES, MODE == Mode::kBalanced>::kMinBlocks)
    gqa_decode_kernel(const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v, const DecodeParams p) {
  constexpr bool BAL = MODE == Mode::kBalanced;
  using TL = Tile<D, NT, NHB, CH, STAGES, BAL>;
  constexpr int T = TL::kT;
  constexpr int nc = TL::kNC;  // consumer warps
  constexpr int r_pad = TL::kRPad;
  constexpr int QS = TL::kQSlots;
  const float kNegInf = -__int_as_float(0x7f800000);

  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  float *osum = reinterpret_cast<float *>(smem + TL::kOSumOff);   // [r_pad][kOStride]
  const uint32_t q_sm = smem_addr(smem + TL::kQOff);              // QS x [r_pad][D] bf16
  float *m_sm = reinterpret_cast<float *>(smem + TL::kMLOff);     // [nc][kHB]
  float *l_sm = m_sm + nc * TL::kHB;                              // [nc][kHB]
  float *M_blk = l_sm + nc * TL::kHB;                             // [r_pad]
  float *L_blk = M_blk + r_pad;                                   // [r_pad]
  const uint32_t bar_full = smem_addr(smem + TL::kBarOff);
  const uint32_t bar_empty = bar_full + 8 * STAGES;
  const uint32_t bar_qfull = bar_empty + 8 * STAGES;
  const uint32_t bar_qempty = bar_qfull + 8 * QS;
  volatile int *tile_bad = reinterpret_cast<volatile int *>(smem + TL::kFlagOff);  // [STAGES]
  volatile int *abort_flag = tile_bad + STAGES;
  volatile int *item_bad = tile_bad + STAGES + 1;
  volatile int *merge_here = tile_bad + STAGES + 2;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // The block's own setup touches only shared memory and the kernel
  // parameters: it runs before the wait below.
  if (threadIdx.x == 0) {
    for (int i = 0; i < STAGES; ++i) {
      mbar_init(bar_full + 8 * i, 1);
      mbar_init(bar_empty + 8 * i, nc);
      tile_bad[i] = 0;
    }
    for (int i = 0; i < QS; ++i) {
      mbar_init(bar_qfull + 8 * i, 1);
      mbar_init(bar_qempty + 8 * i, nc);
    }
    *abort_flag = 0;
    *item_bad = 0;
    fence_mbarrier_init();
  }
  if (warp == nc) {
    if (lane == 0) {
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
    }
    prefetch_piece_l2<D, T, MODE, PAGED>(&tm_k, &tm_v, p, lane);
  }
  __syncthreads();

  // Launched as a programmatic dependent of the previous kernel on the stream
  // (items and balanced modes), the blocks may start while it finishes: wait
  // for it to complete (and its memory to be visible) before reading anything
  // it may have written (q, lengths, page table, cache, workspace).  A no-op
  // when the launch is an ordinary one.
  pdl_wait_primary();
  Piece pc;
  if (!BAL) pc = make_item<T, MODE>(p);
  if (MODE == Mode::kItems) {
    if (threadIdx.x == 0) pdl_launch_dependents();
    if (pc.nh <= 0) return;  // a slice past the rows of a small group (group map): no rows, nothing to do
    if (pc.t_begin >= pc.t_end) {
      // Nothing to read.  An invalid length is handled once, by split 0: zero
      // rows in `out` and a marker in split 0 for the combine.
      if (!pc.len_ok && pc.k == 0) {
        // (a length of 0 where empty sequences are allowed: the same zero row,
        // with lse -inf and no status bit)
        const bool empty = p.empty_ok && pc.len == 0;
        for (int idx = threadIdx.x; idx < pc.nh * (D / 4); idx += blockDim.x) {
          const int h = idx / (D / 4), c4 = idx % (D / 4);
          const size_t row = row_of(p, pc.s, pc.g, pc.h0 + h);
          if (p.out) reinterpret_cast<float4 *>(p.out + row * D)[c4] = make_float4(0.f, 0.f, 0.f, 0.f);
          if (c4 == 0 && p.part_l) p.part_l[row * p.num_splits] = kLBadLength;
          if (c4 == 0 && p.lse) p.lse[row] = kNegInf;
        }
        if (threadIdx.x == 0 && p.status && !empty) atomicOr(p.status, kStatusBadSeqlen);
      }
      return;
    }
  }
  if (MODE != Mode::kItems && threadIdx.x == 0) pdl_launch_dependents();
  // cluster mode, a slice past the rows of a small group (group map): every
  // block of the cluster has the same (group, slice), so all of them leave
  // here, before the cluster's barriers
  if (MODE == Mode::kCluster && pc.nh <= 0) return;
  // a unit with several splits: claim its arrival word for this call
  if (MODE == Mode::kItems && threadIdx.x == 0 && p.unit_ctr != nullptr &&
      (pc.len + p.split_tokens - 1) / p.split_tokens > 1)
    unit_claim(p.unit_ctr + (static_cast<size_t>(pc.s) * p.G + pc.g) * p.hs + pc.j, p.epoch);

  // Every warp walks the same sequence of pieces.
  Walker wk;
  bool have;
  if (BAL) {
    walker_init<T>(wk, p, lane);
    have = walker_next<T>(wk, p, pc);
  } else {
    have = pc.t_begin < pc.t_end;
  }

  if (warp == nc) {
    // =================================================================== producer
    const uint64_t policy = l2_policy_evict_first();
    const int P = p.page_size;
    const int ppt = PAGED ? max(1, T / P) : 1;  // pages per tile
    const int br = PAGED ? min(P, T) : T;        // rows per TMA box
    const uint32_t box_bytes = static_cast<uint32_t>(TL::kHalves * br * 128);
    int tile = 0;  // tiles issued (ring position)
    int n = 0;     // pieces started (q slot position)
    while (have) {
      // ---- q block of the piece's group
      const int qs = n % QS;
      if (n >= QS) {
        bool ok = mbar_wait(bar_qempty + 8 * qs, ((n / QS) - 1) & 1);
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok || *abort_flag) {
          if (lane == 0) {
            *abort_flag = 1;
            if (p.status) atomicOr(p.status, kStatusTimeout);
          }
          break;
        }
      }
      if (lane == 0) {
        const uint32_t q_bytes = static_cast<uint32_t>(pc.nh * D * 2);
        mbar_arrive_expect_tx(bar_qfull + 8 * qs, q_bytes);
        // the slice's rows, in runs of consecutive heads of one query token
        // (one run when there is one query token per sequence)
        for (int rho = 0; rho < pc.nh;) {
          const int a = pc.h0 + rho;
          const int run = p.mapped ? 1 : min(pc.nh - rho, p.r - a % p.r);  // mapped: one row per copy
          bulk_load(q_sm + qs * TL::kQBytes + rho * D * 2, p.q + row_of(p, pc.s, pc.g, a) * D,
                    static_cast<uint32_t>(run * D * 2), bar_qfull + 8 * qs);
          rho += run;
        }
      }
      ++n;
      // ---- K/V tiles
      const int32_t *pt_row = PAGED ? p.page_table + static_cast<size_t>(pc.s) * p.max_pages : nullptr;
      const int lp_end = PAGED ? (pc.t_end + P - 1) / P : 0;  // logical pages holding tokens < t_end
      int cur_w = -1, nxt_w = -1, win = -1, nxt = -1;
      bool stop = false;
      for (int t0 = pc.t_begin; t0 < pc.t_end; t0 += T, ++tile) {
        const int stage = tile % STAGES;
        const uint32_t full = bar_full + 8 * stage;
        if (tile >= STAGES) {
          bool ok = mbar_wait(bar_empty + 8 * stage, ((tile / STAGES) - 1) & 1);
          ok = __shfl_sync(0xffffffffu, ok, 0);
          if (!ok || *abort_flag) {
            if (lane == 0) {
              *abort_flag = 1;
              if (p.status) atomicOr(p.status, kStatusTimeout);
            }
            stop = true;
            break;
          }
        }
        const uint32_t dst_k = smem_addr(smem + stage * TL::kStageBytes);
        const uint32_t dst_v = dst_k + TL::kTileBytes;
        if (test_skip_tile(tile)) continue;  // test builds only
        if (PAGED) {
          const int lp0 = t0 / P;
          const int wnd = lp0 >> 5;
          if (wnd != cur_w) {
            const int idx = wnd * 32 + lane;
            win = (wnd == nxt_w) ? nxt : (idx < lp_end ? __ldg(pt_row + idx) : -1);
            cur_w = wnd;
            nxt_w = wnd + 1;
            const int nidx = nxt_w * 32 + lane;
            nxt = nidx < lp_end ? __ldg(pt_row + nidx) : -1;
          }
          const int n_here = min(ppt, lp_end - lp0);
          const int id = __shfl_sync(0xffffffffu, win, (lp0 & 31) + min(lane, ppt - 1));
          const bool mine = lane < n_here;
          const bool bad = mine && (id < 0 || id >= p.num_pages);
          const unsigned bad_mask = __ballot_sync(0xffffffffu, bad);
          const unsigned good_mask = __ballot_sync(0xffffffffu, mine && !bad);
          if (lane == 0) {
            tile_bad[stage] = bad_mask ? 1 : 0;
            if (bad_mask && p.status) atomicOr(p.status, kStatusBadPage);
            mbar_arrive_expect_tx(full, 2u * box_bytes * __popc(good_mask));
          }
          __syncwarp();
          if (mine && !bad) {
            const int row = (P >= T) ? (t0 % P) : 0;
            const uint32_t off = static_cast<uint32_t>(lane * br * 128);
#pragma unroll
            for (int h = 0; h < TL::kHalves; ++h) {
              tma_load_4d(dst_k + h * T * 128 + off, &tm_k, full, h * 64, row, pc.g, id, policy);
              tma_load_4d(dst_v + h * T * 128 + off, &tm_v, full, h * 64, row, pc.g, id, policy);
            }
          }
        } else if (lane == 0) {
          mbar_arrive_expect_tx(full, 2u * box_bytes);
#pragma unroll
          for (int h = 0; h < TL::kHalves; ++h) {
            tma_load_4d(dst_k + h * T * 128, &tm_k, full, h * 64, t0, pc.g, pc.s, policy);
            tma_load_4d(dst_v + h * T * 128, &tm_v, full, h * 64, t0, pc.g, pc.s, policy);
          }
        }
      }
      if (stop || !BAL) break;
      have = walker_next<T>(wk, p, pc);
    }
    // Never leave with copies in flight: wait (bounded) for the last tiles and
    // q blocks issued; on the normal path these phases completed long ago.
    if (lane == 0) {
      for (int t = max(0, tile - STAGES); t < tile; ++t)
        (void)mbar_wait(bar_full + 8 * (t % STAGES), (t / STAGES) & 1);
      for (int m = max(0, n - QS); m < n; ++m) (void)mbar_wait(bar_qfull + 8 * (m % QS), (m / QS) & 1);
    }
  } else {
    // =================================================================== consumers
    const int hb = warp / TL::kNWT;  // row block
    const int ws = warp % TL::kNWT;  // token slice within a tile
    const int g8 = lane >> 2;
    const int t4 = lane & 3;
    const int ctid = threadIdx.x;    // 0 .. nc*32-1
    const float sl = p.scale_log2;
    int tile = 0;
    int n = 0;
    if (BAL && blockIdx.x == 0 && ctid == 0) {
      p.ws_header[0] = static_cast<int>(gridDim.x);
      p.ws_header[1] = p.capacity;
      p.ws_header[2] = static_cast<int>(wk.W & 0xffffffff);
      p.ws_header[3] = static_cast<int>(wk.W >> 32);
    }
    if (MODE == Mode::kCluster && !have) {  // a block without tokens contributes nothing
      for (int h = ctid; h < r_pad; h += nc * 32) {
        M_blk[h] = kNegInf;
        L_blk[h] = 0.f;
      }
    }
    while (have) {
      // ---- q^T fragments (B operand of S^T = K q^T): head hb*kHB + j*8 + g8,
      // dims ks*16 + 2*t4 (+1) and ks*16 + 8 + 2*t4 (+1); padding heads are 0.
      const int qs = n % QS;
      if (!__shfl_sync(0xffffffffu, mbar_wait(bar_qfull + 8 * qs, (n / QS) & 1), 0)) {
        if (lane == 0) {
          *abort_flag = 1;
          if (p.status) atomicOr(p.status, kStatusTimeout);
        }
      }
      ++n;
      int bad = 0;
      if constexpr (FMA > 0) {
        bad = consume_fma<D, T, CH, STAGES, PAGED, TL::kNWT, TL::kHB, TL::kOStride, FMA>(
            p, pc, q_sm + qs * TL::kQBytes, smem, bar_full, bar_empty, bar_qempty + 8 * qs, tile_bad,
            abort_flag, m_sm, l_sm, osum, tile, warp, lane, nc);
      } else {
      uint32_t bq[TL::kSteps][NT][2];
#pragma unroll
      for (int j = 0; j < NT; ++j) {
        const int hl = hb * TL::kHB + j * 8 + g8;
        const bool valid = hl < pc.nh;
        const uint32_t qrow = q_sm + qs * TL::kQBytes + (valid ? hl : 0) * D * 2;
#pragma unroll
        for (int ks = 0; ks < TL::kSteps; ++ks) {
          bq[ks][j][0] = valid ? ld_shared_u32(qrow + (ks * 16 + 2 * t4) * 2) : 0u;
          bq[ks][j][1] = valid ? ld_shared_u32(qrow + (ks * 16 + 8 + 2 * t4) * 2) : 0u;
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_qempty + 8 * qs);

      float m_run[NT][2], l_run[NT][2];
      float o[TL::kSteps][NT][4];
#pragma unroll
      for (int j = 0; j < NT; ++j) {
        m_run[j][0] = m_run[j][1] = kNegInf;
        l_run[j][0] = l_run[j][1] = 0.f;
#pragma unroll
        for (int mt = 0; mt < TL::kSteps; ++mt) o[mt][j][0] = o[mt][j][1] = o[mt][j][2] = o[mt][j][3] = 0.f;
      }
      // End (exclusive) of the positions each of this lane's two rows sees in
      // the piece: with several query tokens per sequence, query token t sees
      // the cache up to and including itself, len - (nq - 1 - t); with one it
      // is the piece's end.
      int lim[NT][2];
#pragma unroll
      for (int j = 0; j < NT; ++j) {
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int rho = pc.h0 + hb * TL::kHB + j * 8 + 2 * t4 + e;
          lim[j][e] = min(pc.t_end, pc.len - (p.nq - 1 - rho / p.r));
        }
      }

      for (int t0 = pc.t_begin; t0 < pc.t_end; t0 += T, ++tile) {
        const int stage = tile % STAGES;
        // every lane polls the barrier; an abort elsewhere shows up here as a
        // wait that runs out
        const bool ok = __all_sync(0xffffffffu, mbar_wait(bar_full + 8 * stage, (tile / STAGES) & 1));
        if (!ok) {
          if (lane == 0) {
            *abort_flag = 1;
            if (p.status) atomicOr(p.status, kStatusTimeout);
          }
          break;
        }
        if (PAGED) bad |= tile_bad[stage];
        const uint32_t kbase = smem_addr(smem + stage * TL::kStageBytes);
        const uint32_t vbase = kbase + TL::kTileBytes;

#pragma unroll
        for (int c = 0; c < CH; ++c) {
          const int row0 = (ws * CH + c) * 16;
          // ---- S^T = K q^T for 16 tokens x kHB heads (four accumulator chains)
          constexpr int kChains = TL::kSteps >= 4 ? 4 : TL::kSteps;
          float sacc[kChains][NT][4];
#pragma unroll
          for (int c2 = 0; c2 < kChains; ++c2)
#pragma unroll
            for (int j = 0; j < NT; ++j) sacc[c2][j][0] = sacc[c2][j][1] = sacc[c2][j][2] = sacc[c2][j][3] = 0.f;
          {
            const int mi = lane >> 3;
            const int row = row0 + (mi & 1) * 8 + (lane & 7);
#pragma unroll
            for (int ks = 0; ks < TL::kSteps; ++ks) {
              uint32_t a[4];
              ldsm_x4(kbase + swz_offset<T>(row, ks * 16 + (mi >> 1) * 8), a);
#pragma unroll
              for (int j = 0; j < NT; ++j) mma_bf16_16816(sacc[ks % kChains][j], a, bq[ks][j][0], bq[ks][j][1]);
            }
          }
          // ---- mask, scale, online softmax, P^T fragments
          const int tok_a = t0 + row0 + g8;
          uint32_t bh[NT][2], bl[NT][2];
#pragma unroll
          for (int j = 0; j < NT; ++j) {
            float sum[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              sum[e] = sacc[0][j][e];
#pragma unroll
              for (int c2 = 1; c2 < kChains; ++c2) sum[e] += sacc[c2][j][e];
            }
            const float x0 = tok_a < lim[j][0] ? sum[0] * sl : kNegInf;      // token g8,   row 2*t4
            const float x1 = tok_a < lim[j][1] ? sum[1] * sl : kNegInf;      // token g8,   row 2*t4+1
            const float x2 = tok_a + 8 < lim[j][0] ? sum[2] * sl : kNegInf;  // token g8+8, row 2*t4
            const float x3 = tok_a + 8 < lim[j][1] ? sum[3] * sl : kNegInf;  // token g8+8, row 2*t4+1
            // The exponentials use a base m_run that may trail the true running
            // maximum by up to kSlack (p <= 2^kSlack): any base gives the same
            // normalised result as long as l and o share it.  Only when a score
            // passes the base by more than that is the maximum reduced across the
            // token rows and the accumulators rescaled to the new base.
            constexpr float kSlack = 8.f;
            const bool over = fmaxf(x0, x2) > m_run[j][0] + kSlack || fmaxf(x1, x3) > m_run[j][1] + kSlack;
            if (__any_sync(0xffffffffu, over)) {
              float mx_a = fmaxf(x0, x2), mx_b = fmaxf(x1, x3);
#pragma unroll
              for (int off = 4; off < 32; off <<= 1) {
                mx_a = fmaxf(mx_a, __shfl_xor_sync(0xffffffffu, mx_a, off));
                mx_b = fmaxf(mx_b, __shfl_xor_sync(0xffffffffu, mx_b, off));
              }
              const float mn_a = fmaxf(m_run[j][0], mx_a);
              const float mn_b = fmaxf(m_run[j][1], mx_b);
              const float alpha_a = (m_run[j][0] == kNegInf) ? 0.f : ex2(m_run[j][0] - mn_a);
              const float alpha_b = (m_run[j][1] == kNegInf) ? 0.f : ex2(m_run[j][1] - mn_b);
              l_run[j][0] *= alpha_a;
              l_run[j][1] *= alpha_b;
#pragma unroll
              for (int mt = 0; mt < TL::kSteps; ++mt) {
                o[mt][j][0] *= alpha_a;
                o[mt][j][1] *= alpha_b;
                o[mt][j][2] *= alpha_a;
                o[mt][j][3] *= alpha_b;
              }
              m_run[j][0] = mn_a;
              m_run[j][1] = mn_b;
            }
            const float base_a = (m_run[j][0] == kNegInf) ? 0.f : m_run[j][0];
            const float base_b = (m_run[j][1] == kNegInf) ? 0.f : m_run[j][1];
            const float p0 = ex2(x0 - base_a), p1 = ex2(x1 - base_b);
            const float p2 = ex2(x2 - base_a), p3 = ex2(x3 - base_b);
            l_run[j][0] += p0 + p2;
            l_run[j][1] += p1 + p3;
            // high and residual bf16 parts, transposed into the B layout
            uint32_t h01, l01, h23, l23;
            split_bf16x2(p0, p1, h01, l01);
            split_bf16x2(p2, p3, h23, l23);
            bh[j][0] = movmatrix_trans(h01);
            bh[j][1] = movmatrix_trans(h23);
            bl[j][0] = movmatrix_trans(l01);
            bl[j][1] = movmatrix_trans(l23);
          }
          // ---- O^T += V^T P^T
          const bool tail = t0 + row0 + 16 > pc.t_end;
          const int tok_lo = t0 + row0 + 2 * t4;
          const bool k0 = tok_lo < pc.t_end, k1 = tok_lo + 1 < pc.t_end;
          const bool k8 = tok_lo + 8 < pc.t_end, k9 = tok_lo + 9 < pc.t_end;
          {
            const int mi = lane >> 3;
            const int row = row0 + (mi >> 1) * 8 + (lane & 7);
#pragma unroll
            for (int mt = 0; mt < TL::kSteps; ++mt) {
              uint32_t a[4];
              ldsm_x4_trans(vbase + swz_offset<T>(row, mt * 16 + (mi & 1) * 8), a);
              if (tail) {  // rows past the range may hold anything (even NaN): zero them
                a[0] = keep_halves(a[0], k0, k1);
                a[1] = keep_halves(a[1], k0, k1);
                a[2] = keep_halves(a[2], k8, k9);
                a[3] = keep_halves(a[3], k8, k9);
              }
#pragma unroll
              for (int j = 0; j < NT; ++j) {
                mma_bf16_16816(o[mt][j], a, bh[j][0], bh[j][1]);
                mma_bf16_16816(o[mt][j], a, bl[j][0], bl[j][1]);
              }
            }
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(bar_empty + 8 * stage);
      }

      // ---- merge the consumer warps of each row block
#pragma unroll
      for (int j = 0; j < NT; ++j) {
#pragma unroll
        for (int e = 0; e < 2; ++e) {
#pragma unroll
          for (int off = 4; off < 32; off <<= 1)
            l_run[j][e] += __shfl_xor_sync(0xffffffffu, l_run[j][e], off);
        }
      }
      if (g8 == 0) {
#pragma unroll
        for (int j = 0; j < NT; ++j) {
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int hl = j * 8 + 2 * t4 + e;
            m_sm[warp * TL::kHB + hl] = m_run[j][e];
            l_sm[warp * TL::kHB + hl] = l_run[j][e];
          }
        }
      }
      if constexpr (BAL) {
        named_barrier(1, nc * 32);
        float f[NT][2];
#pragma unroll
        for (int j = 0; j < NT; ++j) {
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int hl = j * 8 + 2 * t4 + e;
            float M = kNegInf;
#pragma unroll
            for (int w2 = 0; w2 < TL::kNWT; ++w2) M = fmaxf(M, m_sm[(hb * TL::kNWT + w2) * TL::kHB + hl]);
            f[j][e] = (M == kNegInf) ? 0.f : ex2(m_run[j][e] - M);
          }
        }
        // deterministic accumulation: token slice 0 stores, slices 1..3 add in
        // order (each adding slice reads all its values before it writes any,
        // so that the loads are in flight together)
#pragma unroll
        for (int step = 0; step < TL::kNWT; ++step) {
          if (ws == step) {
            float prev[TL::kSteps][NT][4];
#pragma unroll
            for (int mt = 0; mt < TL::kSteps; ++mt)
#pragma unroll
              for (int j = 0; j < NT; ++j)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                  const int dim = mt * 16 + g8 + (e >> 1) * 8;
                  const int h = hb * TL::kHB + j * 8 + 2 * t4 + (e & 1);
                  prev[mt][j][e] = (step == 0) ? 0.f : osum[h * TL::kOStride + dim];
                }
#pragma unroll
            for (int mt = 0; mt < TL::kSteps; ++mt)
#pragma unroll
              for (int j = 0; j < NT; ++j)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                  const int dim = mt * 16 + g8 + (e >> 1) * 8;
                  const int h = hb * TL::kHB + j * 8 + 2 * t4 + (e & 1);
                  osum[h * TL::kOStride + dim] = prev[mt][j][e] + o[mt][j][e] * f[j][e & 1];
                }
          }
          named_barrier(1, nc * 32);
        }
      } else {
        // each warp's raw O rows into its own region of the ring (once every
        // warp is done with the last tile); the output pass below merges the
        // four token slices of every row in one go
        named_barrier(1, nc * 32);
        float *ow = reinterpret_cast<float *>(smem + TL::kWarpOOff) + warp * TL::kHB * TL::kOStride;
#pragma unroll
        for (int mt = 0; mt < TL::kSteps; ++mt)
#pragma unroll
          for (int j = 0; j < NT; ++j)
#pragma unroll
            for (int e = 0; e < 4; ++e)
              ow[(j * 8 + 2 * t4 + (e & 1)) * TL::kOStride + mt * 16 + g8 + (e >> 1) * 8] = o[mt][j][e];
      }
      }  // mma contraction
      if (FMA > 0 || BAL) {
        for (int h = ctid; h < r_pad; h += nc * 32) {
          const int hb2 = h / TL::kHB, hl = h % TL::kHB;
          float M = kNegInf;
          for (int w2 = 0; w2 < TL::kNWT; ++w2) M = fmaxf(M, m_sm[(hb2 * TL::kNWT + w2) * TL::kHB + hl]);
          float L = 0.f;
          if (M != kNegInf) {
            for (int w2 = 0; w2 < TL::kNWT; ++w2) {
              const int idx = (hb2 * TL::kNWT + w2) * TL::kHB + hl;
              L += l_sm[idx] * ex2(m_sm[idx] - M);
            }
          }
          M_blk[h] = M;
          L_blk[h] = L;
        }
      }
      if (MODE == Mode::kCluster && ctid == 0) *item_bad = bad;
      named_barrier(1, nc * 32);
      // ---- results of the piece
      if (BAL && ctid == 0) {
        if (pc.first_of_unit)
          p.ws_meta[static_cast<size_t>(pc.s) * p.ups + pc.u] =
              make_int4(static_cast<int>(blockIdx.x), pc.last_block, pc.slot & 1, 0);
      }
      constexpr bool kWarpRows = FMA == 0 && !BAL;  // the rows are still per warp (ow)
      if (kWarpRows) {
        // ---- one pass over the rows: merge the row's four token slices
        // (M = max m_w, weights 2^(m_w - M), in slice order: deterministic)
        // and write the result: final rows, a split's partial state, or
        // (cluster mode) the block's merged row for the cluster merge
        const int n4 = D / 4;
        const bool final_row = MODE == Mode::kItems &&
                               ((pc.len + p.split_tokens - 1) / p.split_tokens == 1) && p.out != nullptr;
        const float *ow = reinterpret_cast<const float *>(smem + TL::kWarpOOff);
        for (int idx = ctid; idx < pc.nh * n4; idx += nc * 32) {
          const int h = idx / n4, c4 = idx % n4;
          const int hb2 = h / TL::kHB, hl = h % TL::kHB;
          float mw[TL::kNWT];
          float M = kNegInf;
#pragma unroll
          for (int w2 = 0; w2 < TL::kNWT; ++w2) {
            mw[w2] = m_sm[(hb2 * TL::kNWT + w2) * TL::kHB + hl];
            M = fmaxf(M, mw[w2]);
          }
          float L = 0.f;
          float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
          for (int w2 = 0; w2 < TL::kNWT; ++w2) {
            const int wi = hb2 * TL::kNWT + w2;
            const float wt = (M == kNegInf) ? 0.f : ex2(mw[w2] - M);
            const float4 v = *reinterpret_cast<const float4 *>(ow + (wi * TL::kHB + hl) * TL::kOStride + 4 * c4);
            L += l_sm[wi * TL::kHB + hl] * wt;
            acc.x += v.x * wt;
            acc.y += v.y * wt;
            acc.z += v.z * wt;
            acc.w += v.w * wt;
          }
          if (MODE == Mode::kCluster) {
            *reinterpret_cast<float4 *>(osum + h * TL::kOStride + 4 * c4) = acc;
            if (c4 == 0) {
              M_blk[h] = M;
              L_blk[h] = L;
            }
            continue;
          }
          const size_t row = row_of(p, pc.s, pc.g, pc.h0 + h);
          if (final_row) {
            float4 res = make_float4(0.f, 0.f, 0.f, 0.f);
            if (!bad && L > 0.f) res = make_float4(acc.x / L, acc.y / L, acc.z / L, acc.w / L);
            reinterpret_cast<float4 *>(p.out + row * D)[c4] = res;
            if (c4 == 0 && p.lse) p.lse[row] = bad ? kNegInf : lse_from_state(M, L);
            if (c4 == 0 && p.part_l) p.part_l[row * p.num_splits] = kLFinal;
          } else {
            const size_t ps = row * p.num_splits + pc.k;
            reinterpret_cast<float4 *>(p.part_o + ps * D)[c4] = acc;
            if (c4 == 0) {
              p.part_m[ps] = M;
              p.part_l[ps] = bad ? kLBadPage : L;
            }
          }
        }
      }
      if (MODE != Mode::kCluster) {
        const int n4 = D / 4;
        // partial slot of a row: balanced mode, the block's slot (rc rows
        // each); fixed splits, split k of the output row ([b, nq, H, S])
        const bool final_row =
            BAL ? pc.final_row : (((pc.len + p.split_tokens - 1) / p.split_tokens == 1) && p.out != nullptr);
        for (int idx = ctid; !kWarpRows && idx < pc.nh * n4; idx += nc * 32) {
          const int h = idx / n4, c4 = idx % n4;
          const size_t row = row_of(p, pc.s, pc.g, pc.h0 + h);
          const float4 src = *reinterpret_cast<const float4 *>(osum + h * TL::kOStride + 4 * c4);
          if (final_row) {
            const float L = L_blk[h];
            float4 res = make_float4(0.f, 0.f, 0.f, 0.f);
            if (!bad && L > 0.f) res = make_float4(src.x / L, src.y / L, src.z / L, src.w / L);
            reinterpret_cast<float4 *>(p.out + row * D)[c4] = res;
            if (c4 == 0 && p.lse) p.lse[row] = bad ? kNegInf : lse_from_state(M_blk[h], L);
            if (!BAL && c4 == 0 && p.part_l) p.part_l[row * p.num_splits] = kLFinal;
          } else {
            const size_t ps = BAL ? static_cast<size_t>(pc.slot) * p.rc + h : row * p.num_splits + pc.k;
            reinterpret_cast<float4 *>(p.part_o + ps * D)[c4] = src;
            if (c4 == 0) {
              p.part_m[ps] = M_blk[h];
              p.part_l[ps] = bad ? kLBadPage : L_blk[h];
            }
          }
        }
        if (!BAL && p.unit_ctr != nullptr && !final_row) {
          // ---- the block whose split completes the unit merges its splits
          // (the combine kernel's arithmetic, in this grid): publish this
          // block's partial states, count the arrival, and if it was the last
          // one read everyone's states back through L2.
          // (the barrier orders every consumer thread's stores before thread
          // 0's fence, which makes them visible GPU-wide before its arrival;
          // its second fence orders the other blocks' states, published the
          // same way, before the merge's loads, which the barrier releases)
          named_barrier(1, nc * 32);
          const int ns = (pc.len + p.split_tokens - 1) / p.split_tokens;
          if (ctid == 0) {
            __threadfence();
            const size_t u = (static_cast<size_t>(pc.s) * p.G + pc.g) * p.hs + pc.j;
            *merge_here = unit_arrive(p.unit_ctr + u, p.epoch, ns, p.status) ? 1 : 0;
            __threadfence();
          }
          named_barrier(1, nc * 32);
          if (*merge_here) {
            // all rows at once: each thread takes two float4 columns of one
            // row (half a row apart), so rows x D/8 threads cover the block
            constexpr int kHalf = D / 8;
            static_assert(TL::kRPad * kHalf <= nc * 32, "one pass of the consumer threads");
            const int h = ctid / kHalf, c4 = ctid % kHalf;
            if (h < pc.nh) {
              const size_t row = row_of(p, pc.s, pc.g, pc.h0 + h);
              merge_serial<D, 2>(p.part_o, p.part_m, p.part_l, static_cast<long long>(row) * p.num_splits, ns,
                                 c4, kHalf, reinterpret_cast<float4 *>(p.out + row * D),
                                 p.lse ? p.lse + row : nullptr);
            }
          }
        }
      }
      if (*abort_flag || !BAL) break;
      have = walker_next<T>(wk, p, pc);
    }
  }

  if (MODE == Mode::kCluster) {
    // ---- merge the blocks of the cluster through distributed shared memory.
    // Block k of the nb blocks owns rows [k nh / nb, (k + 1) nh / nb).  Once
    // every block has its merged rows (osum, M_blk, L_blk), each block pushes
    // each of its rows into the owner's receive area with remote stores (no
    // round trip waits on them), one cluster barrier makes them visible, and
    // each owner merges its rows from its own shared memory, the blocks in
    // rank order (deterministic).  The receive area lies in the ring, past the
    // merged rows: at the first barrier every block is done with its ring.
    constexpr int kRS = D + 4;  // receive row: o[D], then M, L, bad
    cg::cluster_group cluster = cg::this_cluster();
    const int nb = static_cast<int>(cluster.num_blocks());
    const int rank = static_cast<int>(cluster.block_rank());
    const int rows_max = (pc.nh + nb - 1) / nb;  // rows per owner, at most
    float *recv = reinterpret_cast<float *>(smem + TL::kRecvOff);  // [nb][rows_max][kRS]
    cluster.sync();
    const int n4 = D / 4;
    const float bad_mine = static_cast<float>(*item_bad);
    for (int idx = threadIdx.x; idx < pc.nh * (n4 + 1); idx += blockDim.x) {
      const int h = idx / (n4 + 1), part = idx % (n4 + 1);
      const int k = (h * nb + nb - 1) / pc.nh;  // owner: the largest k with k nh / nb <= h
      const int k_own = (k * pc.nh / nb > h) ? k - 1 : k;
      const int r_lo_k = k_own * pc.nh / nb;
      float *dst = cluster.map_shared_rank(recv, k_own) + (rank * rows_max + (h - r_lo_k)) * kRS;
      if (part < n4)
        reinterpret_cast<float4 *>(dst)[part] = *reinterpret_cast<const float4 *>(osum + h * TL::kOStride + 4 * part);
      else
        reinterpret_cast<float4 *>(dst)[n4] = make_float4(M_blk[h], L_blk[h], bad_mine, 0.f);
    }
    cluster.sync();
    const int r_lo = rank * pc.nh / nb, r_hi = (rank + 1) * pc.nh / nb;
    for (int idx = threadIdx.x; idx < (r_hi - r_lo) * n4; idx += blockDim.x) {
      const int hr = idx / n4, c4 = idx % n4;
      float M = kNegInf;
      bool bad = false;
      for (int c = 0; c < nb; ++c) {
        const float4 meta = reinterpret_cast<const float4 *>(recv + (c * rows_max + hr) * kRS)[n4];
        M = fmaxf(M, meta.x);
        bad |= meta.z != 0.f;
      }
      float L = 0.f;
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
      if (pc.len_ok && !bad && M != kNegInf) {
        for (int c = 0; c < nb; ++c) {
          const float *src = recv + (c * rows_max + hr) * kRS;
          const float4 meta = reinterpret_cast<const float4 *>(src)[n4];
          if (meta.x == kNegInf) continue;  // a block without tokens contributes nothing
          const float wgt = ex2(meta.x - M);
          const float4 v = reinterpret_cast<const float4 *>(src)[c4];
          L += meta.y * wgt;
          acc.x += v.x * wgt;
          acc.y += v.y * wgt;
          acc.z += v.z * wgt;
          acc.w += v.w * wgt;
        }
      }
      float4 res = make_float4(0.f, 0.f, 0.f, 0.f);
      if (L > 0.f) res = make_float4(acc.x / L, acc.y / L, acc.z / L, acc.w / L);
      const size_t row = row_of(p, pc.s, pc.g, pc.h0 + r_lo + hr);
      reinterpret_cast<float4 *>(p.out + row * D)[c4] = res;
      if (c4 == 0 && p.lse) p.lse[row] = bad ? kNegInf : lse_from_state(M, L);
    }
    // (a length of 0 where empty sequences are allowed: zero rows, lse -inf,
    // no status bit)
    if (rank == 0 && threadIdx.x == 0 && !pc.len_ok && p.status && !(p.empty_ok && pc.len == 0))
      atomicOr(p.status, kStatusBadSeqlen);
  }
}

// Fixed splits: one block per (sequence, head) row merges the splits
// k < ceil(len / split_tokens) of that row.
template <int D, int NTH>
__global__ void __launch_bounds__(NTH) gqa_combine_kernel(const CombineParams p) {
  const int row = blockIdx.x;       // [b, nq, H] flattened
  const int s = row / (p.nq * p.H);
  const int len = __ldg(p.seqlens + s);
  float4 *dst = reinterpret_cast<float4 *>(p.out + static_cast<size_t>(row) * D) + threadIdx.x % (D / 4);
  // the next kernel on the stream (a dependent launch: the next step's decode)
  // may set itself up and prefetch while this one runs; it waits for this
  // grid to complete before touching memory
  if (threadIdx.x == 0) pdl_launch_dependents();
  pdl_wait_primary();  // the partial states below come from the preceding kernel
  float *lse_dst = p.lse ? p.lse + row : nullptr;
  if (len < p.nq || len > p.max_len) {
    if (threadIdx.x < D / 4) *dst = make_float4(0.f, 0.f, 0.f, 0.f);
    if (threadIdx.x == 0 && lse_dst) *lse_dst = -__int_as_float(0x7f800000);
    if (threadIdx.x == 0 && p.status && !(p.empty_ok && len == 0)) atomicOr(p.status, kStatusBadSeqlen);
    return;
  }
  const int ns = (len + p.split_tokens - 1) / p.split_tokens;
  const long long base = static_cast<long long>(row) * p.num_splits;
  // the decode kernel already wrote this row (a single split)
  if (ns == 1 && p.part_l[base] == kLFinal) return;
  if (ns <= kSerialMergeMax) {
    if (threadIdx.x < D / 4)
      merge_serial<D, 1>(p.part_o, p.part_m, p.part_l, base, ns, threadIdx.x, 0,
                         reinterpret_cast<float4 *>(p.out + static_cast<size_t>(row) * D), lse_dst);
    return;
  }
  __shared__ MergeScratch<D, NTH> sc;
  merge_row<D, NTH>(p.part_o, p.part_m, p.part_l, ns, [&](int k) -> long long { return base + k; }, dst, lse_dst,
               threadIdx.x, sc, [] { __syncthreads(); });
}

// Balanced mode: one block per (unit, group of 128 / (D / 4) rows), one
// float4 column of one row per thread.  The decode kernel recorded, for every
// unit, the first and last decode blocks holding its tiles and the slot the
// first one used; every later block holds the unit's first piece of its own
// range (slot 0), unless its range is empty.  Units one block covered whole
// are final already; units with an invalid length get zero rows here.  Up to
// 4 kSerialMergeMax contributions each thread merges its column alone
// (merge_serial_at: no barriers, kSerialMergeMax loads in flight at once);
// more, and the block merges its rows one after another with merge_row.
template <int D, int T>
__global__ void __launch_bounds__(128) gqa_combine_balanced_kernel(const CombineParams p) {
  constexpr int kTPR = D / 4;         // threads per row
  constexpr int kRPB = 128 / kTPR;    // rows per block
  const int rblocks = (p.rc + kRPB - 1) / kRPB;
  const int u = blockIdx.x / rblocks;  // unit: (sequence, group, head slice)
  const int h0 = (blockIdx.x % rblocks) * kRPB;
  const int s = u / p.ups;
  int g, j;
  unit_gj(p.mapped, p.map, p.hs, u % p.ups, &g, &j);
  // rows of the slice (the last slice of a group is narrower; a group table
  // gives each group its own size)
  const int slice_rows =
      min(p.rc, (p.mapped ? static_cast<int>(p.map.off[g + 1]) - static_cast<int>(p.map.off[g]) : p.rq) - j * p.rc);
  auto row_at = [&](int hh) -> size_t {
    return p.mapped ? static_cast<size_t>(s) * p.H + p.map.heads[p.map.off[g] + j * p.rc + hh]
                    : out_row(s, g, j * p.rc + hh, p.nq, p.r, p.H);
  };
  const int c4 = threadIdx.x % kTPR;
  const int h = h0 + threadIdx.x / kTPR;
  const bool row_ok = h < slice_rows;
  const size_t row = row_ok ? row_at(h) : 0;
  float4 *dst = reinterpret_cast<float4 *>(p.out + row * D);
  const int len = __ldg(p.seqlens + s);
  if (threadIdx.x == 0) pdl_launch_dependents();  // as in gqa_combine_kernel
  pdl_wait_primary();  // the header, unit records and partial states come from the decode kernel
  const int N = p.ws_header[0];
  const int capacity = p.ws_header[1];
  float *lse_dst = (p.lse && row_ok) ? p.lse + row : nullptr;
  if (len < p.nq || len > capacity) {
    if (row_ok) dst[c4] = make_float4(0.f, 0.f, 0.f, 0.f);
    if (c4 == 0 && lse_dst) *lse_dst = -__int_as_float(0x7f800000);
    if (threadIdx.x == 0 && h0 == 0 && p.status && !(p.empty_ok && len == 0)) atomicOr(p.status, kStatusBadSeqlen);
    return;
  }
  const long long W = static_cast<long long>(static_cast<unsigned>(p.ws_header[2])) |
                      (static_cast<long long>(p.ws_header[3]) << 32);
  const int4 meta = p.ws_meta[u];
  const int c_lo = meta.x, c_hi = meta.y, slot_lo = meta.z;
  if (c_lo == c_hi) return;  // one decode block covered the unit: its rows are final
  const int nc = c_hi - c_lo + 1;
  if (nc <= 4 * kSerialMergeMax) {
    if (row_ok)
      merge_serial_at<D, 1, true>(p.part_o, p.part_m, p.part_l,
                                  [&](int k) -> long long {
                              const long long c = c_lo + k;
                              if (k > 0 && (c * W / N) == ((c + 1) * W / N)) return -1;  // empty range
                              return (2 * c + (k == 0 ? slot_lo : 0)) * p.rc + h;
                            },
                            nc, c4, 0, dst, lse_dst);
    return;
  }
  __shared__ MergeScratch<D, 128> sc;
  for (int hh = h0; hh < h0 + kRPB && hh < slice_rows; ++hh) {  // (uniform in the block)
    const size_t row2 = row_at(hh);
    merge_row<D, 128>(p.part_o, p.part_m, p.part_l, nc,
                 [&](int k) -> long long {
                   const long long c = c_lo + k;
                   if (k > 0 && (c * W / N) == ((c + 1) * W / N)) return -1;  // empty range
                   return (2 * c + (k == 0 ? slot_lo : 0)) * p.rc + hh;
                 },
                 reinterpret_cast<float4 *>(p.out + row2 * D) + threadIdx.x % kTPR,
                 p.lse ? p.lse + row2 : nullptr, threadIdx.x, sc, [] { __syncthreads(); });
  }
}

// Merge of normalised partial results weighted by their log-sum-exp, e.g. the
// token shards of a sequence held by different GPUs, gathered into one buffer
// part-major: o_parts [n_parts][rows][D], lse_parts [n_parts][rows].  Per row,
//   LSE = ln sum_k e^(lse_k),  out = sum_k e^(lse_k - LSE) o_k,
// the same re-association of the softmax as the split merge, written for
// results that are already normalised.  Parts with lse = -inf (no tokens)
// weigh nothing; a row whose parts are all empty is zero with LSE -inf.  One
// thread per float4 of a row; the parts are taken in ascending order.
template <int D>
__global__ void __launch_bounds__(128)
    gqa_merge_lse_kernel(const float *o_parts, const float *lse_parts, int n_parts, long long rows, float *out,
                         float *lse_out) {
  constexpr int kTPR = D / 4;
  const float kNegInf = -__int_as_float(0x7f800000);
  const long long row = static_cast<long long>(blockIdx.x) * (128 / kTPR) + threadIdx.x / kTPR;
  const int c4 = threadIdx.x % kTPR;
  if (row >= rows) return;
  float mx = kNegInf;
  for (int k = 0; k < n_parts; ++k) mx = fmaxf(mx, __ldg(lse_parts + k * rows + row));
  float4 res = make_float4(0.f, 0.f, 0.f, 0.f);
  float lse = kNegInf;
  if (mx != kNegInf) {
    float S = 0.f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 4
    for (int k = 0; k < n_parts; ++k) {
      const float w = ex2((__ldg(lse_parts + k * rows + row) - mx) * 1.4426950408889634f);
      const float4 v = __ldg(reinterpret_cast<const float4 *>(o_parts + (k * rows + row) * D) + c4);
      S += w;
      acc.x += v.x * w;
      acc.y += v.y * w;
      acc.z += v.z * w;
      acc.w += v.w * w;
    }
    res = make_float4(acc.x / S, acc.y / S, acc.z / S, acc.w / S);
    lse = mx + logf(S);
  }
  reinterpret_cast<float4 *>(out + row * D)[c4] = res;
  if (lse_out && c4 == 0) lse_out[row] = lse;
}

}  // namespace gqa
