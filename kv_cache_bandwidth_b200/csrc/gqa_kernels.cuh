// gqa_kernels.cuh -- grouped-query attention decode kernels for B200 (sm_100a).
//
// The operation (see include/gqa.h): for every sequence s and query head i,
// out[s,i] = softmax_j(scale * q[s,i] . K[s,g(i),j]) V[s,g(i),j] with
// g(i) = i / (H/G), the group broadcast of the PyTorch module of
// "Grouped-Query Attention" (aiwiki) done inside the kernel instead of with
// repeat_interleave, as that page's closing note asks.
//
// One thread block owns one (sequence, KV group, token range) item.  Its keys
// and values cross HBM once and are shared on chip by the group's r = H/G
// query heads:
//
//   * a producer warp bulk-copies the group's q block into shared memory and
//     streams K and V tiles of T tokens into a STAGES-deep shared-memory ring
//     with TMA (128-byte swizzle), translating logical pages through the page
//     table (a window of 32 page ids per warp, the next window prefetched);
//   * consumer warps (4 along the token axis x head blocks of 8 or 16 heads)
//     run the two small contractions on tensor cores with the roles of the
//     operands swapped so that the tile's tokens fill the M = 16 rows of
//     mma.m16n8k16 and the group's heads the N = 8 columns:
//         S^T[tokens, heads] = K_tile q^T            (A = K from smem, B = q in registers)
//         O^T[d, heads]     += V_tile^T P^T           (A = V^T via ldmatrix.trans)
//     P^T goes from the accumulator layout of S^T to the B-operand layout with
//     movmatrix; it is split into a bf16 high part and a bf16 residual so that
//     the product keeps ~16 bits of the probabilities (a single bf16 rounding
//     would leave ~1e-3 relative error);
//   * online softmax in base 2: running maximum and sum per head, warp-shuffle
//     reductions over the token rows, accumulator rescaling by 2^(m_old - m_new);
//   * at the end the consumer warps merge their states in shared memory and
//     either write a split's partial state (split-KV mode) or merge the blocks
//     of a thread-block cluster through distributed shared memory and write the
//     normalised output (cluster mode).
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

// kItems: one block per (sequence, group, split) item, blockIdx.x = item.
// kCluster: one block per cluster rank; the blocks of a cluster share one
// (sequence, group) and merge through distributed shared memory.
enum class Mode { kItems, kCluster };

struct DecodeParams {
  const __nv_bfloat16 *q;     // [b, H, D]
  const int32_t *seqlens;     // [b]
  const int32_t *page_table;  // [b, max_pages] (paged) or nullptr
  float *out;                 // [b, H, D]; items mode: may be null (partials only)
  float *part_o;              // [b, H, S, D]; may be null when S == 1 and out is set
  float *part_m;              // [b, H, S]
  float *part_l;              // [b, H, S]
  uint32_t *status;           // optional
  int H, G, r;                // query heads, KV groups, heads per group
  int page_size;              // paged: tokens per page; contiguous: capacity m
  int num_pages;              // paged: pages in the pool
  int max_pages;              // paged: page-table row stride
  int capacity;               // largest valid length
  int split_tokens;           // items mode: tokens per split
  int num_splits;             // items mode: S
  float scale_log2;           // scale * log2(e)
};

struct CombineParams {
  const int32_t *seqlens;
  float *out;
  const float *part_o;
  const float *part_m;
  const float *part_l;
  uint32_t *status;
  int b, H, max_len, split_tokens, num_splits;
};

template <int D, int NT, int NHB, int CH, int STAGES>
struct Tile {
  static constexpr int kNWT = 4;                   // consumer warps along the token axis
  static constexpr int kHB = 8 * NT;               // query heads per consumer warp
  static constexpr int kNC = kNWT * NHB;           // consumer warps (NHB head blocks)
  static constexpr int kThreads = 32 * (kNC + 1);  // + one producer warp
  static constexpr int kT = kNWT * 16 * CH;        // tokens per pipeline stage
  static constexpr int kHalves = D / 64;           // 128-byte swizzle atoms per row
  static constexpr int kTileBytes = kT * D * 2;    // one K (or V) tile
  static constexpr int kStageBytes = 2 * kTileBytes;
  static constexpr int kRingBytes = STAGES * kStageBytes;
  static constexpr int kSteps = D / 16;            // k-steps of q.k, m-tiles of p.v
  static constexpr int kRPad = NHB * kHB;          // heads per block, padded
  static constexpr int kOStride = D + 4;           // padded merge row (floats)
  static constexpr int kQBytes = kRPad * D * 2;    // the group's q block
  // Shared memory (after 1 KiB alignment): ring | q block | per-warp m, l and
  // per-head M, L | mbarriers | flags.  The merge of the output accumulators
  // reuses the ring once every tile has been consumed.
  static constexpr int kQOff = kRingBytes;
  static constexpr int kMLOff = kQOff + kQBytes;
  static constexpr int kMLFloats = 2 * kNC * kHB + 2 * kRPad;
  static constexpr int kBarOff = (kMLOff + 4 * kMLFloats + 7) & ~7;
  static constexpr int kNumBars = 2 * STAGES + 1;  // full, empty, q
  static constexpr int kFlagOff = kBarOff + 8 * kNumBars;
  static constexpr int kNumFlags = STAGES + 2;     // bad tile per stage, abort, item bad
  static constexpr int kSmemBytes = 1024 + kFlagOff + 4 * kNumFlags;
  static constexpr int kMinBlocks = STAGES <= 2 ? 3 : (STAGES == 3 ? 2 : 1);
  static_assert(kRPad * kOStride * 4 <= kRingBytes, "merge rows must fit in the ring");
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

// One unit of work: the token range [t_begin, t_end) of KV group g of sequence s.
struct Item {
  int s, g, k, len, t_begin, t_end;
  bool len_ok;
};

template <int T, Mode MODE>
__device__ __forceinline__ Item make_item(const DecodeParams &p) {
  Item it;
  if (MODE == Mode::kItems) {
    const int i = blockIdx.x;
    it.k = i % p.num_splits;
    const int sg = i / p.num_splits;
    it.g = sg % p.G;
    it.s = sg / p.G;
  } else {
    it.k = blockIdx.x;
    it.g = blockIdx.y;
    it.s = blockIdx.z;
  }
  it.len = __ldg(p.seqlens + it.s);
  it.len_ok = it.len >= 1 && it.len <= p.capacity;
  it.t_begin = 0;
  it.t_end = 0;
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

template <int D, int NT, int NHB, int CH, int STAGES, bool PAGED, Mode MODE>
__global__ void __launch_bounds__(Tile<D, NT, NHB, CH, STAGES>::kThreads,
                                  Tile<D, NT, NHB, CH, STAGES>::kMinBlocks)
    gqa_decode_kernel(const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v, const DecodeParams p) {
  using TL = Tile<D, NT, NHB, CH, STAGES>;
  constexpr int T = TL::kT;
  constexpr int nc = TL::kNC;  // consumer warps
  constexpr int r_pad = TL::kRPad;
  const float kNegInf = -__int_as_float(0x7f800000);

  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  float *osum = reinterpret_cast<float *>(smem);                  // [r_pad][kOStride], after the loop
  const uint32_t q_sm = smem_addr(smem + TL::kQOff);              // [r][D] bf16
  float *m_sm = reinterpret_cast<float *>(smem + TL::kMLOff);     // [nc][kHB]
  float *l_sm = m_sm + nc * TL::kHB;                              // [nc][kHB]
  float *M_blk = l_sm + nc * TL::kHB;                             // [r_pad]
  float *L_blk = M_blk + r_pad;                                   // [r_pad]
  const uint32_t bar_full = smem_addr(smem + TL::kBarOff);
  const uint32_t bar_empty = bar_full + 8 * STAGES;
  const uint32_t bar_q = bar_empty + 8 * STAGES;
  volatile int *tile_bad = reinterpret_cast<volatile int *>(smem + TL::kFlagOff);  // [STAGES]
  volatile int *abort_flag = tile_bad + STAGES;
  volatile int *item_bad = tile_bad + STAGES + 1;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const Item w = make_item<T, MODE>(p);

  if (MODE == Mode::kItems) {
    if (threadIdx.x == 0) pdl_launch_dependents();
    if (w.t_begin >= w.t_end) {
      // Nothing to read.  An invalid length is handled once, by split 0: zero
      // rows in `out` and a marker in split 0 for the combine.
      if (!w.len_ok && w.k == 0) {
        for (int idx = threadIdx.x; idx < p.r * (D / 4); idx += blockDim.x) {
          const int h = idx / (D / 4), c4 = idx % (D / 4);
          const size_t row = static_cast<size_t>(w.s) * p.H + static_cast<size_t>(w.g) * p.r + h;
          if (p.out) reinterpret_cast<float4 *>(p.out + row * D)[c4] = make_float4(0.f, 0.f, 0.f, 0.f);
          if (c4 == 0 && p.part_l) p.part_l[row * p.num_splits] = kLBadLength;
        }
        if (threadIdx.x == 0 && p.status) atomicOr(p.status, kStatusBadSeqlen);
      }
      return;
    }
  }

  if (threadIdx.x == 0) {
    for (int i = 0; i < STAGES; ++i) {
      mbar_init(bar_full + 8 * i, 1);
      mbar_init(bar_empty + 8 * i, nc);
      tile_bad[i] = 0;
    }
    mbar_init(bar_q, 1);
    *abort_flag = 0;
    *item_bad = 0;
    fence_mbarrier_init();
  }
  __syncthreads();
  const int ntiles = w.t_end > w.t_begin ? (w.t_end - w.t_begin + T - 1) / T : 0;

  if (warp == nc) {
    // =================================================================== producer
    if (ntiles > 0) {
      if (lane == 0) {
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
        const uint32_t q_bytes = static_cast<uint32_t>(p.r * D * 2);
        mbar_arrive_expect_tx(bar_q, q_bytes);
        bulk_load(q_sm, p.q + (static_cast<size_t>(w.s) * p.H + static_cast<size_t>(w.g) * p.r) * D,
                  q_bytes, bar_q);
      }
      const uint64_t policy = l2_policy_evict_first();
      const int P = p.page_size;
      const int ppt = PAGED ? max(1, T / P) : 1;  // pages per tile
      const int br = PAGED ? min(P, T) : T;        // rows per TMA box
      const uint32_t box_bytes = static_cast<uint32_t>(TL::kHalves * br * 128);
      const int32_t *pt_row = PAGED ? p.page_table + static_cast<size_t>(w.s) * p.max_pages : nullptr;
      const int lp_end = PAGED ? (w.t_end + P - 1) / P : 0;  // logical pages holding tokens < t_end
      int cur_w = -1, nxt_w = -1, win = -1, nxt = -1;
      int tile = 0;
      for (; tile < ntiles; ++tile) {
        const int t0 = w.t_begin + tile * T;
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
            break;
          }
        }
        const uint32_t dst_k = smem_addr(smem + stage * TL::kStageBytes);
        const uint32_t dst_v = dst_k + TL::kTileBytes;
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
              tma_load_4d(dst_k + h * T * 128 + off, &tm_k, full, h * 64, row, w.g, id, policy);
              tma_load_4d(dst_v + h * T * 128 + off, &tm_v, full, h * 64, row, w.g, id, policy);
            }
          }
        } else if (lane == 0) {
          mbar_arrive_expect_tx(full, 2u * box_bytes);
#pragma unroll
          for (int h = 0; h < TL::kHalves; ++h) {
            tma_load_4d(dst_k + h * T * 128, &tm_k, full, h * 64, t0, w.g, w.s, policy);
            tma_load_4d(dst_v + h * T * 128, &tm_v, full, h * 64, t0, w.g, w.s, policy);
          }
        }
      }
      // Never leave with copies in flight: wait (bounded) for the last tiles
      // and the q block; on the normal path these phases completed long ago.
      if (lane == 0) {
        for (int t = max(0, tile - STAGES); t < tile; ++t)
          (void)mbar_wait(bar_full + 8 * (t % STAGES), (t / STAGES) & 1);
        (void)mbar_wait(bar_q, 0);
      }
    }
  } else if (ntiles > 0) {
    // =================================================================== consumers
    const int hb = warp / TL::kNWT;  // head block
    const int ws = warp % TL::kNWT;  // token slice within a tile
    const int g8 = lane >> 2;
    const int t4 = lane & 3;
    const int ctid = threadIdx.x;    // 0 .. nc*32-1
    const float sl = p.scale_log2;

    // ---- q^T fragments (B operand of S^T = K q^T): head hb*kHB + j*8 + g8,
    // dims ks*16 + 2*t4 (+1) and ks*16 + 8 + 2*t4 (+1); padding heads are 0.
    if (!__shfl_sync(0xffffffffu, mbar_wait(bar_q, 0), 0)) {
      if (lane == 0) {
        *abort_flag = 1;
        if (p.status) atomicOr(p.status, kStatusTimeout);
      }
    }
    uint32_t bq[TL::kSteps][NT][2];
#pragma unroll
    for (int j = 0; j < NT; ++j) {
      const int hl = hb * TL::kHB + j * 8 + g8;
      const bool valid = hl < p.r;
      const uint32_t qrow = q_sm + (valid ? hl : 0) * D * 2;
#pragma unroll
      for (int ks = 0; ks < TL::kSteps; ++ks) {
        bq[ks][j][0] = valid ? ld_shared_u32(qrow + (ks * 16 + 2 * t4) * 2) : 0u;
        bq[ks][j][1] = valid ? ld_shared_u32(qrow + (ks * 16 + 8 + 2 * t4) * 2) : 0u;
      }
    }

    float m_run[NT][2], l_run[NT][2];
    float o[TL::kSteps][NT][4];
#pragma unroll
    for (int j = 0; j < NT; ++j) {
      m_run[j][0] = m_run[j][1] = kNegInf;
      l_run[j][0] = l_run[j][1] = 0.f;
#pragma unroll
      for (int mt = 0; mt < TL::kSteps; ++mt) o[mt][j][0] = o[mt][j][1] = o[mt][j][2] = o[mt][j][3] = 0.f;
    }
    int bad = 0;

    for (int tile = 0; tile < ntiles && !*abort_flag; ++tile) {
      const int t0 = w.t_begin + tile * T;
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
      const uint32_t kbase = smem_addr(smem + stage * TL::kStageBytes);
      const uint32_t vbase = kbase + TL::kTileBytes;

#pragma unroll
      for (int c = 0; c < CH; ++c) {
        const int row0 = (ws * CH + c) * 16;
        // ---- S^T = K q^T for 16 tokens x kHB heads (two accumulator chains)
        float sacc[NT][4], sacc2[NT][4];
#pragma unroll
        for (int j = 0; j < NT; ++j) {
          sacc[j][0] = sacc[j][1] = sacc[j][2] = sacc[j][3] = 0.f;
          sacc2[j][0] = sacc2[j][1] = sacc2[j][2] = sacc2[j][3] = 0.f;
        }
        {
          const int mi = lane >> 3;
          const int row = row0 + (mi & 1) * 8 + (lane & 7);
#pragma unroll
          for (int ks = 0; ks < TL::kSteps; ++ks) {
            uint32_t a[4];
            ldsm_x4(kbase + swz_offset<T>(row, ks * 16 + (mi >> 1) * 8), a);
#pragma unroll
            for (int j = 0; j < NT; ++j) {
              if (ks & 1)
                mma_bf16_16816(sacc2[j], a, bq[ks][j][0], bq[ks][j][1]);
              else
                mma_bf16_16816(sacc[j], a, bq[ks][j][0], bq[ks][j][1]);
            }
          }
        }
        // ---- mask, scale, online softmax, P^T fragments
        const int tok_a = t0 + row0 + g8;
        const bool ok_a = tok_a < w.t_end;
        const bool ok_b = tok_a + 8 < w.t_end;
        uint32_t bh[NT][2], bl[NT][2];
#pragma unroll
        for (int j = 0; j < NT; ++j) {
          const float x0 = ok_a ? (sacc[j][0] + sacc2[j][0]) * sl : kNegInf;  // token g8,   head 2*t4
          const float x1 = ok_a ? (sacc[j][1] + sacc2[j][1]) * sl : kNegInf;  // token g8,   head 2*t4+1
          const float x2 = ok_b ? (sacc[j][2] + sacc2[j][2]) * sl : kNegInf;  // token g8+8, head 2*t4
          const float x3 = ok_b ? (sacc[j][3] + sacc2[j][3]) * sl : kNegInf;  // token g8+8, head 2*t4+1
          float mx_a = fmaxf(x0, x2), mx_b = fmaxf(x1, x3);
#pragma unroll
          for (int off = 4; off < 32; off <<= 1) {
            mx_a = fmaxf(mx_a, __shfl_xor_sync(0xffffffffu, mx_a, off));
            mx_b = fmaxf(mx_b, __shfl_xor_sync(0xffffffffu, mx_b, off));
          }
          const float mn_a = fmaxf(m_run[j][0], mx_a);
          const float mn_b = fmaxf(m_run[j][1], mx_b);
          const float base_a = (mn_a == kNegInf) ? 0.f : mn_a;
          const float base_b = (mn_b == kNegInf) ? 0.f : mn_b;
          const float p0 = ex2(x0 - base_a), p1 = ex2(x1 - base_b);
          const float p2 = ex2(x2 - base_a), p3 = ex2(x3 - base_b);
          // rescale only when a running maximum moved (rare after the first tiles)
          if (__any_sync(0xffffffffu, mn_a != m_run[j][0] || mn_b != m_run[j][1])) {
            const float alpha_a = ex2(m_run[j][0] - base_a);
            const float alpha_b = ex2(m_run[j][1] - base_b);
            l_run[j][0] *= alpha_a;
            l_run[j][1] *= alpha_b;
#pragma unroll
            for (int mt = 0; mt < TL::kSteps; ++mt) {
              o[mt][j][0] *= alpha_a;
              o[mt][j][1] *= alpha_b;
              o[mt][j][2] *= alpha_a;
              o[mt][j][3] *= alpha_b;
            }
          }
          l_run[j][0] += p0 + p2;
          l_run[j][1] += p1 + p3;
          m_run[j][0] = mn_a;
          m_run[j][1] = mn_b;
          // high and residual bf16 parts, transposed into the B layout
          bh[j][0] = movmatrix_trans(pack_bf16(p0, p1));
          bh[j][1] = movmatrix_trans(pack_bf16(p2, p3));
          bl[j][0] = movmatrix_trans(pack_bf16(p0 - bf16_round(p0), p1 - bf16_round(p1)));
          bl[j][1] = movmatrix_trans(pack_bf16(p2 - bf16_round(p2), p3 - bf16_round(p3)));
        }
        // ---- O^T += V^T P^T
        const bool tail = t0 + row0 + 16 > w.t_end;
        const int tok_lo = t0 + row0 + 2 * t4;
        const bool k0 = tok_lo < w.t_end, k1 = tok_lo + 1 < w.t_end;
        const bool k8 = tok_lo + 8 < w.t_end, k9 = tok_lo + 9 < w.t_end;
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

    // ---- merge the consumer warps of each head block (the ring is free now)
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
    // deterministic accumulation: token slice 0 stores, slices 1..3 add in order
#pragma unroll
    for (int step = 0; step < TL::kNWT; ++step) {
      if (ws == step) {
#pragma unroll
        for (int mt = 0; mt < TL::kSteps; ++mt) {
#pragma unroll
          for (int j = 0; j < NT; ++j) {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int dim = mt * 16 + g8 + (e >> 1) * 8;
              const int h = hb * TL::kHB + j * 8 + 2 * t4 + (e & 1);
              float *dst = osum + h * TL::kOStride + dim;
              const float v = o[mt][j][e] * f[j][e & 1];
              *dst = (step == 0) ? v : (*dst + v);
            }
          }
        }
      }
      named_barrier(1, nc * 32);
    }
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
    if (ctid == 0) *item_bad = bad;
    named_barrier(1, nc * 32);

    if (MODE == Mode::kItems) {
      const int n4 = D / 4;
      const int ns = (w.len + p.split_tokens - 1) / p.split_tokens;
      const bool final_row = (ns == 1) && p.out != nullptr;
      for (int idx = ctid; idx < p.r * n4; idx += nc * 32) {
        const int h = idx / n4, c4 = idx % n4;
        const size_t row = static_cast<size_t>(w.s) * p.H + static_cast<size_t>(w.g) * p.r + h;
        const float *src = osum + h * TL::kOStride + 4 * c4;
        if (final_row) {
          const float L = L_blk[h];
          float4 res = make_float4(0.f, 0.f, 0.f, 0.f);
          if (!bad && L > 0.f) res = make_float4(src[0] / L, src[1] / L, src[2] / L, src[3] / L);
          reinterpret_cast<float4 *>(p.out + row * D)[c4] = res;
          if (c4 == 0 && p.part_l) p.part_l[row * p.num_splits] = kLFinal;
        } else {
          const size_t ps = row * p.num_splits + w.k;
          reinterpret_cast<float4 *>(p.part_o + ps * D)[c4] = make_float4(src[0], src[1], src[2], src[3]);
          if (c4 == 0) {
            p.part_m[ps] = M_blk[h];
            p.part_l[ps] = bad ? kLBadPage : L_blk[h];
          }
        }
      }
    }
  }

  if (MODE == Mode::kCluster) {
    // ---- merge the blocks of the cluster through distributed shared memory
    if (ntiles == 0 && warp < nc) {  // a block without tokens contributes nothing
      for (int h = threadIdx.x; h < r_pad; h += nc * 32) {
        M_blk[h] = kNegInf;
        L_blk[h] = 0.f;
      }
    }
    cg::cluster_group cluster = cg::this_cluster();
    cluster.sync();
    if (cluster.block_rank() == 0) {
      const int nb = static_cast<int>(cluster.num_blocks());
      int bad = 0;
      if (w.len_ok)
        for (int c = 0; c < nb; ++c) bad |= *cluster.map_shared_rank(const_cast<int *>(item_bad), c);
      const int n4 = D / 4;
      for (int idx = threadIdx.x; idx < p.r * n4; idx += blockDim.x) {
        const int h = idx / n4, c4 = idx % n4;
        float L = 0.f;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        if (w.len_ok && !bad) {
          float M = kNegInf;
          for (int c = 0; c < nb; ++c) M = fmaxf(M, *cluster.map_shared_rank(M_blk + h, c));
          for (int c = 0; c < nb; ++c) {
            const float Mc = *cluster.map_shared_rank(M_blk + h, c);
            if (Mc == kNegInf) continue;  // a block without tokens
            const float wgt = ex2(Mc - M);
            L += *cluster.map_shared_rank(L_blk + h, c) * wgt;
            const float *src = cluster.map_shared_rank(osum + h * TL::kOStride + 4 * c4, c);
            acc.x += src[0] * wgt;
            acc.y += src[1] * wgt;
            acc.z += src[2] * wgt;
            acc.w += src[3] * wgt;
          }
        }
        float4 res = make_float4(0.f, 0.f, 0.f, 0.f);
        if (L > 0.f) res = make_float4(acc.x / L, acc.y / L, acc.z / L, acc.w / L);
        const size_t row = static_cast<size_t>(w.s) * p.H + static_cast<size_t>(w.g) * p.r + h;
        reinterpret_cast<float4 *>(p.out + row * D)[c4] = res;
      }
      if (threadIdx.x == 0 && !w.len_ok && p.status) atomicOr(p.status, kStatusBadSeqlen);
    }
    cluster.sync();
  }
}

// Merge the per-split partial states of every (sequence, head) row.  The
// D/4 threads of a row load the split maxima and sums cooperatively (one
// coalesced pass), reduce the maximum with warp shuffles, then accumulate the
// rescaled partial outputs with the loads of consecutive splits in flight
// together.
template <int D>
__global__ void __launch_bounds__(128) gqa_combine_kernel(const CombineParams p) {
  constexpr int kTPR = D / 4;         // threads per row (one float4 each)
  constexpr int kRPB = 128 / kTPR;    // rows per block
  const float kNegInf = -__int_as_float(0x7f800000);
  const int row = blockIdx.x * kRPB + threadIdx.x / kTPR;
  const int c4 = threadIdx.x % kTPR;
  const unsigned mask = (kTPR == 32) ? 0xffffffffu : (0xffffu << (threadIdx.x & 16));
  if (row >= p.b * p.H) return;  // whole row groups leave together
  const int s = row / p.H;
  const int len = __ldg(p.seqlens + s);
  pdl_wait_primary();  // the partial states below come from the preceding kernel
  float4 *dst = reinterpret_cast<float4 *>(p.out + static_cast<size_t>(row) * D) + c4;
  if (len < 1 || len > p.max_len) {
    *dst = make_float4(0.f, 0.f, 0.f, 0.f);
    if (c4 == 0 && p.status) atomicOr(p.status, kStatusBadSeqlen);
    return;
  }
  const int ns = (len + p.split_tokens - 1) / p.split_tokens;
  const float *mrow = p.part_m + static_cast<size_t>(row) * p.num_splits;
  const float *lrow = p.part_l + static_cast<size_t>(row) * p.num_splits;
  const float4 *orow = reinterpret_cast<const float4 *>(p.part_o + static_cast<size_t>(row) * p.num_splits * D);
  // Markers in l: the decode kernel already wrote this row (a single split),
  // or a split met an invalid page id / the length exceeds the capacity (the
  // row is zero).
  if (ns == 1 && lrow[0] == kLFinal) return;
  float M = kNegInf;
  bool bad = false;
  for (int k = c4; k < ns; k += kTPR) {
    M = fmaxf(M, mrow[k]);
    bad |= lrow[k] < 0.f;
  }
#pragma unroll
  for (int off = kTPR / 2; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(mask, M, off));
  bad = __any_sync(mask, bad);
  float L = 0.f;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  if (!bad && M != kNegInf) {
#pragma unroll 4
    for (int k = 0; k < ns; ++k) {
      const float w = ex2(mrow[k] - M);
      L += lrow[k] * w;
      const float4 v = orow[static_cast<size_t>(k) * kTPR + c4];
      acc.x += v.x * w;
      acc.y += v.y * w;
      acc.z += v.z * w;
      acc.w += v.w * w;
    }
  }
  float4 res = make_float4(0.f, 0.f, 0.f, 0.f);
  if (!bad && L > 0.f) res = make_float4(acc.x / L, acc.y / L, acc.z / L, acc.w / L);
  *dst = res;
}

}  // namespace gqa
