// gqa_verify_tc.cuh -- decode of many rows per KV group on the 5th-generation
// tensor cores (tcgen05): the rows of a verification step (n query tokens x r
// heads) or of a large group ratio, up to 128 per block at d = 128 (64-token
// tiles), up to 64 at d = 64 (128-token tiles: the same 16 KB of K per tile,
// S and P 128 columns wide).
//
// With more than 16 rows per group the mma.sync kernel has to cut the rows
// into 16-row slices, each with its own pass over the group's keys and values
// and its own share of the legacy tensor pipe's throughput.  Here one block
// takes all rows of its (sequence, group, split) item and the contractions
// become real matrix products on the tensor cores, with the accumulators in
// tensor memory:
//
//   S[rows, 64 tokens]  = Q[rows, 128] . K_tile[64, 128]^T        (M = 128, N = 64)
//   O[rows, 128]       += P[rows, 64] . V_tile[64, 128]            (M = 128, N = 128)
//
// With up to 128 rows (the layout described here) the rows are padded to
// M = 128; with up to 64 (the spread layout, see tc_softmax_spread; the only
// one at d = 64) both products have M = 64 and the rows sit in the first 16
// lanes of each tensor-memory lane quarter, four threads per row.  P enters
// as a bf16 high part and a bf16 residual (two MMAs), as in the mma.sync
// kernel, here both truncated (byte permutes, no conversions: P to within
// 2^-14 relative).  P is written to tensor memory over its own scores (each
// thread over the columns it has read) and the P.V product takes its A
// operand from there, which leaves shared memory to a 5-stage K/V ring (6 in
// the spread layout, whose Q is half as large).  Warp roles:
//   * warps 0-7: two threads per row (warps w and w+4 share the tensor-memory
//     lanes of rows 32(w%4) ..), each taking 32 of a tile's 64 tokens with a
//     softmax state of its own: its running base and sum, and its own O in
//     tensor memory (the P.V of its tokens accumulates there).  Each tile:
//     read the half-row of scores from tensor memory, mask (the row's own
//     causal limit among the drafts), online softmax in base 2 with the lazy
//     rescale (a half whose maximum moves by more than 2^8 rescales its O row
//     in tensor memory), write P to tensor memory.  The two halves of a row
//     meet once, at the end, as two partial states merged exactly;
//   * warp 8: the TMA producer of the K/V ring (as in the mma.sync kernel);
//   * warp 9: tensor-memory allocation; one thread issues the Q K^T products;
//   * warp 10: one thread issues the P.V products.  The two issuers run
//     concurrently (the tensor pipe overlaps their products) and signal
//     completion on mbarriers with tcgen05.commit.
// S and P share three tensor-memory buffers: the scores of tiles t+1 and t+2
// are computed and the softmax of t+1 runs while the P.V of tile t is on the
// tensor cores; a buffer takes new scores once the P.V that read it is done.
// The epilogue writes final rows or partial states in the layout of the
// mma.sync kernel, so the same merges (in this kernel for up to 8 splits, the
// combine kernel otherwise) apply.

#pragma once

#include <type_traits>

#include "gqa_kernels.cuh"
#include "tc05.cuh"

namespace gqa {

// Packed fp32 arithmetic (sm_100) for the softmax threads: two fp32 values in
// one 64-bit register pair, operated on by one instruction; each lane is
// rounded exactly as the scalar instruction rounds it.
__device__ __forceinline__ uint64_t f32x2(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}

__device__ __forceinline__ void f32x2_get(uint64_t v, float &lo, float &hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}

__device__ __forceinline__ uint64_t fma_f32x2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}

__device__ __forceinline__ uint64_t add_f32x2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

__device__ __forceinline__ uint64_t sub_f32x2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

// max(a, b, c) in one instruction (a NaN operand is ignored, as by fmaxf)
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// Maximum of N values (N even, >= 4): two independent chains of three-input
// maxima over the halves, joined at the end.
template <int N>
__device__ __forceinline__ float max_of(const float *x) {
  static_assert(N >= 4 && N % 2 == 0, "two chains of at least two values");
  constexpr int H = N / 2;
  float a = fmaxf(x[0], x[1]), b = fmaxf(x[H], x[H + 1]);
#pragma unroll
  for (int k = 2; k + 1 < H; k += 2) {
    a = fmax3(a, x[k], x[k + 1]);
    b = fmax3(b, x[H + k], x[H + k + 1]);
  }
  if (H % 2) {
    a = fmaxf(a, x[H - 1]);
    b = fmaxf(b, x[N - 1]);
  }
  return fmaxf(a, b);
}

// split_bf16x2_rz with the two residuals taken by one packed subtraction
// (the same bits: each residual is exact in fp32).
__device__ __forceinline__ void split_bf16x2_rz_x2(float a, float b, uint32_t &hi, uint32_t &lo) {
  const uint32_t ua = __float_as_uint(a), ub = __float_as_uint(b);
  hi = __byte_perm(ua, ub, 0x7632);
  float ra, rb;
  f32x2_get(sub_f32x2(f32x2(a, b), f32x2(__uint_as_float(ua & 0xffff0000u), __uint_as_float(ub & 0xffff0000u))),
            ra, rb);
  lo = __byte_perm(__float_as_uint(ra), __float_as_uint(rb), 0x7632);
}

// The waits of the single-thread roles (the TMA producer and the two MMA
// issuers), which spend most of each tile waiting: mbarrier.try_wait with a
// suspend-time hint, so that the waiting warp sleeps until the phase completes
// (or the hint runs out) instead of polling, and leaves the issue slots of its
// SM sub-partition to the two softmax warps there.  Bounded as mbar_wait is:
// false once the wait has run past kWaitLimitCycles.
constexpr uint32_t kRoleSuspendNs = 100000;

__device__ __forceinline__ bool mbar_try_wait_suspend(uint32_t bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(done)
      : "r"(bar), "r"(parity), "r"(kRoleSuspendNs)
      : "memory");
  return done != 0;
}

__device__ __forceinline__ bool mbar_wait_role(uint32_t bar, uint32_t parity) {
  if (mbar_try_wait_suspend(bar, parity)) return true;
  const long long start = clock64();
  while (!mbar_try_wait_suspend(bar, parity)) {
    if (clock64() - start > kWaitLimitCycles) return false;
  }
  return true;
}

// Shared-memory layout of the tcgen05 kernels: a STAGES-deep ring of K/V tiles
// of 64 tokens (32 KB per stage) and QBUFS buffers of Q (QROWS rows x d = 128).
// QROWS = 128: the Q K^T product has M = 128, row i in tensor-memory lane i.
// QROWS = 64 (at most 64 rows, SPREAD): M = 64, whose accumulator rows sit in
// the first 16 lanes of each 32-lane quarter (row m in lane m % 16 + 32 (m /
// 16)), exactly where the spread softmax reads them; Q then takes half the
// shared memory.  The P.V product takes P from tensor memory with the same
// M: with 64 rows its A operand and accumulator use that same lane layout
// (P written over the scores, O rows where the softmax threads read them),
// half the work of a 128-row product; with 128 rows lane = row.
template <int STAGES, int QBUFS, int QROWS, int D = 128>
struct TcLayout {
  static_assert(D == 64 || D == 128, "d = 64 or 128");
  static constexpr int kD = D;
  static constexpr int kT = D == 64 ? 128 : 64;        // tokens per tile (16 KB of K either way)
  static constexpr int kHalves = D / 64;               // 64-column (128-byte) halves of a row
  static constexpr int kM = 128;                       // rows at most (M of the 128-row products)
  static constexpr int kQRows = QROWS;                 // rows of the Q K^T product (padded)
  static constexpr int kStages = STAGES;
  static constexpr int kQBufs = QBUFS;
  static constexpr int kHalf = kT * 128;               // one 64-column half of a K or V tile
  static constexpr int kTileBytes = kHalves * kHalf;   // 16 KB
  static constexpr int kStageBytes = 2 * kTileBytes;   // K + V
  static constexpr int kQOff = kStages * kStageBytes;  // Q: kHalves halves of QROWS rows x 128 B per buffer
  static constexpr int kQHalf = kQRows * 128;
  static constexpr int kQBytes = kHalves * kQHalf;
  static constexpr int kBarOff = kQOff + kQBufs * kQBytes;
  static constexpr int kSP = 3;                        // S/P buffers in tensor memory
  // full[kStages], empty[kStages], s_full[kSP], p_full[kSP], pv_done[kSP],
  // drain[2] (one per MMA issuer: all its products done before teardown),
  // q_full[kQBufs], q_empty[kQBufs], o_free (O read out: the next unit's P.V may start)
  static constexpr int kNumBars = 2 * kStages + 3 * kSP + 2 + 2 * kQBufs + 1;
  static constexpr int kXOff = kBarOff + 8 * kNumBars;  // the halves' bases at the end: [2][kM] floats
  static constexpr int kLOff = kXOff + 4 * 2 * kM;      // the halves' sums at the end: [2][kM] floats
  static constexpr int kMiscOff = kLOff + 4 * 2 * kM;  // tmem base, tile_bad[kStages], abort, merge here, stop
  static constexpr int kSmemBytes = 1024 + kMiscOff + 4 * (kStages + 4);
  static constexpr int kSoftmaxWarps = 8;
  static constexpr int kThreads = 32 * (kSoftmaxWarps + 3);
  // S, then P over it (kSP x kT columns), then the two O of kD columns
  static constexpr uint32_t kOCol = D == 128 ? 256 : kSP * kT;
  static constexpr uint32_t kTmemCols = 512;
  static_assert(kSP * kT <= static_cast<int>(kOCol) && kOCol + 2 * kD <= kTmemCols, "tensor-memory columns");
  static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");
};
// One piece per block (up to 128 rows), and its SPREAD form (up to 64 rows,
// whose smaller Q leaves room for a sixth ring stage).
// d = 64 runs the SPREAD form only (128-token tiles).
using TcTile = TcLayout<5, 1, 128>;
using TcTileSpread = TcLayout<6, 1, 64>;
using TcTileSpread64 = TcLayout<6, 1, 64, 64>;
template <bool SPREAD, int D = 128>
using TcItemTile = typename std::conditional<D == 64, TcTileSpread64,
                                             typename std::conditional<SPREAD, TcTileSpread, TcTile>::type>::type;

struct TcBars {
  uint32_t full0, empty0, s_full0, p_full0, pv_done0, drain0, q_full0, q_empty0, o_free;
};

template <class TT>
__device__ __forceinline__ TcBars tc_bars(uint32_t sbase) {
  TcBars b;
  b.full0 = sbase + TT::kBarOff;
  b.empty0 = b.full0 + 8 * TT::kStages;
  b.s_full0 = b.empty0 + 8 * TT::kStages;
  b.p_full0 = b.s_full0 + 8 * TT::kSP;
  b.pv_done0 = b.p_full0 + 8 * TT::kSP;
  b.drain0 = b.pv_done0 + 8 * TT::kSP;
  b.q_full0 = b.drain0 + 16;
  b.q_empty0 = b.q_full0 + 8 * TT::kQBufs;
  b.o_free = b.q_empty0 + 8 * TT::kQBufs;
  return b;
}

// One thread initialises every barrier.  q_full_count: arrivals that make a Q
// buffer full (128 Q rows, or the producer warp's one arrival).
template <class TT>
__device__ __forceinline__ void tc_init_bars(const TcBars &b, volatile int *tile_bad, uint32_t q_full_count) {
  for (int i = 0; i < TT::kStages; ++i) {
    mbar_init(b.full0 + 8 * i, 1);
    mbar_init(b.empty0 + 8 * i, 1);  // one tcgen05.commit per use
    tile_bad[i] = 0;
  }
  for (int i = 0; i < TT::kSP; ++i) {
    mbar_init(b.s_full0 + 8 * i, 1);
    mbar_init(b.p_full0 + 8 * i, TT::kSoftmaxWarps);  // one arrival per softmax warp
    mbar_init(b.pv_done0 + 8 * i, 1);
  }
  mbar_init(b.drain0, 1);
  mbar_init(b.drain0 + 8, 1);
  for (int i = 0; i < TT::kQBufs; ++i) {
    mbar_init(b.q_full0 + 8 * i, q_full_count);
    mbar_init(b.q_empty0 + 8 * i, 1);
  }
  mbar_init(b.o_free, TT::kSoftmaxWarps);
}

// Row of the slice held by Q slot (row of the Q K^T product) r, or -1 for a
// padding slot.  SPREAD (64 slots, M = 64): slot r lands in lane r % 16 of
// quarter r / 16, which holds rows qd * rpq .. in its first rpq = ceil(nh / 4)
// lanes.
template <bool SPREAD>
__device__ __forceinline__ int tc_slot_row(int r, int nh) {
  if (SPREAD) {
    const int rpq = (nh + 3) / 4, li = r % 16, rho = (r / 16) * rpq + li;
    return (li < rpq && rho < nh) ? rho : -1;
  }
  return r < nh ? r : -1;
}

// Byte offset of 16-byte chunk c (of d / 8) of Q slot r: 64-column halves in
// the 128-byte swizzle TMA would write.
template <class TT>
__device__ __forceinline__ int tc_q_offset(int r, int c) {
  return (c >> 3) * TT::kQHalf + r * 128 + (((c & 7) ^ (r & 7)) << 4);
}

// TMA producer for one piece: K and V tiles of 64 tokens into the stage ring
// from ring position `tile` on (advanced past the piece), pages translated
// through the table as in the mma.sync kernel.  False if the block aborted.
template <class TT, bool PAGED>
__device__ __forceinline__ bool tc_produce_piece(const CUtensorMap *tm_k, const CUtensorMap *tm_v,
                                                 const DecodeParams &p, const Piece &pc, uint32_t sbase,
                                                 const TcBars &bars, volatile int *tile_bad,
                                                 volatile int *abort_flag, int lane, int &tile) {
  constexpr int T = TT::kT;
  constexpr int ST = TT::kStages;
  const uint64_t policy = l2_policy_evict_first();
  const int P = p.page_size;
  const int ppt = PAGED ? max(1, T / P) : 1;  // pages per tile
  const int br = PAGED ? min(P, T) : T;        // rows per TMA box
  const uint32_t box_bytes = static_cast<uint32_t>(TT::kHalves * br * 128);
  const int32_t *pt_row = PAGED ? p.page_table + static_cast<size_t>(pc.s) * p.max_pages : nullptr;
  const int lp_end = PAGED ? (pc.t_end + P - 1) / P : 0;
  int cur_w = -1, nxt_w = -1, win = -1, nxt = -1;
  for (int t0 = pc.t_begin; t0 < pc.t_end; t0 += T, ++tile) {
    const int stage = tile % ST;
    const uint32_t full = bars.full0 + 8 * stage;
    if (tile >= ST) {
      bool ok = mbar_wait_role(bars.empty0 + 8 * stage, ((tile / ST) - 1) & 1);
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok || *abort_flag) {
        if (lane == 0) {
          *abort_flag = 1;
          if (p.status) atomicOr(p.status, kStatusTimeout);
        }
        return false;
      }
    }
    const uint32_t dst_k = sbase + stage * TT::kStageBytes;
    const uint32_t dst_v = dst_k + TT::kTileBytes;
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
        for (int h = 0; h < TT::kHalves; ++h) {
          tma_load_4d(dst_k + h * TT::kHalf + off, tm_k, full, h * 64, row, pc.g, id, policy);
          tma_load_4d(dst_v + h * TT::kHalf + off, tm_v, full, h * 64, row, pc.g, id, policy);
        }
      }
    } else if (lane == 0) {
      mbar_arrive_expect_tx(full, 2u * box_bytes);
#pragma unroll
      for (int h = 0; h < TT::kHalves; ++h) {
        tma_load_4d(dst_k + h * TT::kHalf, tm_k, full, h * 64, t0, pc.g, pc.s, policy);
        tma_load_4d(dst_v + h * TT::kHalf, tm_v, full, h * 64, t0, pc.g, pc.s, policy);
      }
    }
  }
  return true;
}

// Never leave with copies in flight: wait (bounded) for the last tiles issued.
template <class TT>
__device__ __forceinline__ void tc_produce_drain(const TcBars &bars, int tile, int lane) {
  constexpr int ST = TT::kStages;
  if (lane == 0)
    for (int t = max(0, tile - ST); t < tile; ++t) (void)mbar_wait(bars.full0 + 8 * (t % ST), (t / ST) & 1);
}

// The block whose split completes the unit merges the unit's splits (as in
// the mma.sync kernel): the 256 softmax threads.
template <int D>
__device__ __forceinline__ void tc_merge_unit(const DecodeParams &p, const Piece &pc, int sm,
                                              volatile int *merge_here) {
  merge_unit_by_last<D, 32 * TcTile::kSoftmaxWarps>(p, pc, sm, merge_here);
}

// Where the rows of a piece go.  final_row: normalised rows into out (and
// lse).  Otherwise partial states: slot >= 0 is the block's partial slot of
// the equal-work mode (row rho at slot * rc + rho); slot < 0 is split k of the
// output row (items mode; the unit's last arrival merges it in this kernel
// when the call has arrival words).
struct TcDest {
  bool final_row;
  int slot;
};

__device__ __forceinline__ size_t tc_part_index(const DecodeParams &p, const Piece &pc, const TcDest &dst,
                                                size_t row, int rho) {
  return dst.slot >= 0 ? static_cast<size_t>(dst.slot) * p.rc + rho : row * p.num_splits + pc.k;
}

// After the rows of a piece are written: the softmax threads agree (through
// one barrier) on whether the block stops, so that they all take the same
// barriers in the next piece.
__device__ __forceinline__ bool tc_piece_done(volatile int *stop, volatile int *abort_flag, int sm, int n_threads) {
  if (sm == 0) *stop = *abort_flag;
  named_barrier(1, n_threads);
  return *stop == 0;
}

// Softmax warps with at most 64 rows (SPREAD), for one piece of n_tiles tiles
// starting at global tile gt0 of the block's pipeline: quarter qd = warp % 4 of
// the tensor-memory lanes holds rows qd * rpq .. in its first rpq <= 16 lanes
// (rpq = ceil(rows / 4)).  Warp w takes tokens [T/2 h, T/2 h + T/2) of every
// tile (T = 64, or 128 at d = 64), h = w / 4, and within it thread t the T/4
// tokens [T/2 h + T/4 (t / 16), + T/4) of lane t % 16 (the 16x32bx2 shape).  The two threads of a row in one
// warp share its running base (their maximum meets through one shuffle) and
// the row's O_h in tensor memory; the two warps of a quarter keep separate
// states and O_h, merged once at the end.  P's high part goes over the
// thread's first T/8 score columns, its residual over the next T/8.  Returns
// false once the block stops (a timeout).
template <class TT, bool PAGED>
__device__ __forceinline__ bool tc_softmax_spread(const DecodeParams &p, const Piece &pc, uint8_t *smem,
                                                  uint32_t tmem, const TcBars &bars, volatile int *tile_bad,
                                                  volatile int *abort_flag, volatile int *merge_here,
                                                  volatile int *stop, int gt0,
                                                  int n_tiles, const TcDest &dest, int warp, int lane) {
  constexpr int D = TT::kD;
  constexpr int T = TT::kT;
  constexpr int ST = TT::kStages;
  constexpr int SP = TT::kSP;
  constexpr int kSM = 32 * TT::kSoftmaxWarps;
  constexpr int HT = T / 2;                // tokens of a warp half
  constexpr int TPT = T / 4;               // tokens (score columns) of a thread: 16, or 32 at d = 64
  constexpr int CW = D / 4;                // output columns of a thread
  const float kNegInf = -__int_as_float(0x7f800000);
  const int sm = threadIdx.x;
  const int qd = warp % 4;                 // lane quarter
  const int half = warp / 4;               // tokens [HT half, HT half + HT) of every tile
  const int sub = lane >> 4;               // ... of which [TPT sub, TPT sub + TPT)
  const int li = lane & 15;                // lane within the quarter
  const int rpq = (pc.nh + 3) / 4;         // rows per quarter
  const int rho = qd * rpq + li;           // row of the slice
  const bool valid = li < rpq && rho < pc.nh;
  const bool warp_active = qd * rpq < pc.nh;
  const int slot = qd * 32 + li;           // tensor-memory lane of the row
  // the positions this row sees (a padding slot sees the whole piece: its
  // scores are 0 and its result unused)
  const int lim = valid ? min(pc.t_end, pc.len - (p.nq - 1 - (pc.h0 + rho) / p.r)) : pc.t_end;
  const uint32_t lane_tmem = tmem + (static_cast<uint32_t>(qd * 32) << 16);
  float *mbase = reinterpret_cast<float *>(smem + TT::kXOff);  // [half][slot]
  float *lsum = reinterpret_cast<float *>(smem + TT::kLOff);   // [half][slot]
  // |scale| log2(e): a negative scale's sign is folded into Q when it is
  // loaded, so that the maximum of the raw scores is the maximum of the
  // scaled ones and the exponent is one fma of the raw score
  const float sl = fabsf(p.scale_log2);
  float m_run = kNegInf, l_run = 0.f;  // this half's base (shared by the pair) and this thread's sum
  int bad = 0;
  bool ok = true;
  for (int t = 0; t < n_tiles; ++t) {
    const int gt = gt0 + t;
    const int t0 = pc.t_begin + t * T;
    const int st = gt % ST;
    const int b = gt % SP;
    ok = __all_sync(0xffffffffu, mbar_wait(bars.s_full0 + 8 * b, (gt / SP) & 1));
    if (!ok) break;
    tc_fence_after();
    uint32_t sv[TPT];
    tc_ld16x2_cols<TPT, TPT>(lane_tmem + b * T + half * HT, sv);
    tc_wait_ld();
    if (PAGED) bad |= tile_bad[st];
    // V rows past the piece's end may hold anything (even NaN): zero them so
    // that P = 0 there meets zeros
    const int valid_rows = min(T, pc.t_end - t0);
    if (valid_rows < T) {
      uint8_t *vt = smem + st * TT::kStageBytes + TT::kTileBytes;
      for (int idx = sm; idx < (T - valid_rows) * (D / 8); idx += kSM) {
        const int row = valid_rows + idx / (D / 8), c = idx % (D / 8);
        *reinterpret_cast<uint4 *>(vt + (c >> 3) * TT::kHalf + row * 128 + ((c & 7) << 4)) =
            make_uint4(0u, 0u, 0u, 0u);
      }
    }
    // raw scores (-inf past the row's limit)
    float x[TPT];
    const int tb = t0 + half * HT + sub * TPT;  // this thread's first token of the tile
    const bool edge = tb + TPT > lim;
    if (!edge) {
#pragma unroll
      for (int j = 0; j < TPT; ++j) x[j] = __uint_as_float(sv[j]);
    } else {
#pragma unroll
      for (int j = 0; j < TPT; ++j) x[j] = (tb + j < lim) ? __uint_as_float(sv[j]) : kNegInf;
    }
    float mx = max_of<TPT>(x);
    mx = (mx == kNegInf) ? kNegInf : mx * sl;              // the scaled maximum
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));  // the row's other TPT tokens of this half
    if (warp_active) {
      // lazy rescale: only when a score passes the base by more than 2^8 (the
      // same decision in both threads of the row)
      const bool need = mx > m_run + 8.f;
      if (__any_sync(0xffffffffu, need)) {
        const float mn = need ? fmaxf(m_run, mx) : m_run;
        const float alpha = need ? ((m_run == kNegInf) ? 0.f : ex2(m_run - mn)) : 1.f;
        l_run *= alpha;
        if (t > 0) {
          // O_h holds the piece's tiles 0 .. t-1: rescale it once their MMAs
          // are done; thread sub takes columns [D/2 sub, D/2 sub + D/2) of the row
          ok = __all_sync(0xffffffffu, mbar_wait(bars.pv_done0 + 8 * ((gt - 1) % SP), ((gt - 1) / SP) & 1));
          if (!ok) break;
          tc_fence_after();
#pragma unroll
          for (int c = 0; c < D / 64; ++c) {
            uint32_t ov[32];
            tc_ld16x2_x32<D / 2>(lane_tmem + TT::kOCol + half * D + c * 32, ov);
            tc_wait_ld();
#pragma unroll
            for (int j = 0; j < 32; ++j) ov[j] = __float_as_uint(__uint_as_float(ov[j]) * alpha);
            tc_st16x2_x32<D / 2>(lane_tmem + TT::kOCol + half * D + c * 32, ov);
          }
          tc_wait_st();
          tc_fence_before();
        }
        m_run = mn;
      }
      const float nb = (m_run == kNegInf) ? 0.f : -m_run;
      if (edge) {
        // the exponent of a masked score is -inf whatever the scale
#pragma unroll
        for (int j = 0; j < TPT; ++j) x[j] = (x[j] == kNegInf) ? kNegInf : fmaf(x[j], sl, nb);
      } else {
        // score * |scale| log2(e) - base, two scores per instruction
        const uint64_t sl2 = f32x2(sl, sl), nb2 = f32x2(nb, nb);
#pragma unroll
        for (int e = 0; e < TPT / 2; ++e)
          f32x2_get(fma_f32x2(f32x2(x[2 * e], x[2 * e + 1]), sl2, nb2), x[2 * e], x[2 * e + 1]);
      }
      uint32_t hi[TPT / 2], lo[TPT / 2];
      uint64_t ls2 = f32x2(0.f, 0.f);  // the tile's sum, even and odd columns apart
#pragma unroll
      for (int e = 0; e < TPT / 2; ++e) {
        const float p0 = ex2(x[2 * e]), p1 = ex2(x[2 * e + 1]);
        ls2 = add_f32x2(ls2, f32x2(p0, p1));
        split_bf16x2_rz_x2(p0, p1, hi[e], lo[e]);
      }
      {
        float la, lb;
        f32x2_get(ls2, la, lb);
        l_run += la + lb;
      }
      tc_st16x2_cols<TPT / 2, TPT>(lane_tmem + b * T + half * HT, hi);
      tc_st16x2_cols<TPT / 2, TPT>(lane_tmem + b * T + half * HT + TPT / 2, lo);
      tc_wait_st();
    }
    tc_fence_before();
    if (valid_rows < T) fence_proxy_async_smem();  // the zeroed V rows, for the tensor core
    __syncwarp();
    if (lane == 0) mbar_arrive(bars.p_full0 + 8 * b);
  }
  if (!ok && lane == 0) {
    *abort_flag = 1;
    if (p.status) atomicOr(p.status, kStatusTimeout);
  }
  l_run += __shfl_xor_sync(0xffffffffu, l_run, 16);  // the half's sum of the row
  // ---- the row's result: O from tensor memory once the last MMAs are done
  const int glast = gt0 + n_tiles - 1;
  const bool done = ok && __all_sync(0xffffffffu, mbar_wait(bars.pv_done0 + 8 * (glast % SP), (glast / SP) & 1));
  tc_fence_after();
  if (sub == 0) {
    mbase[half * 128 + slot] = m_run;
    lsum[half * 128 + slot] = l_run;
  }
  named_barrier(1, kSM);
  const float m0 = mbase[slot], m1 = mbase[128 + slot];
  const float m_row = fmaxf(m0, m1);
  const float w0 = (m0 == kNegInf) ? 0.f : ex2(m0 - m_row), w1 = (m1 == kNegInf) ? 0.f : ex2(m1 - m_row);
  const float l_row = lsum[slot] * w0 + lsum[128 + slot] * w1;
  const size_t row = valid ? row_of(p, pc.s, pc.g, pc.h0 + rho) : 0;
  const size_t ps = tc_part_index(p, pc, dest, row, rho);
  const float inv = (!bad && done && l_row > 0.f) ? 1.f / l_row : 0.f;
  const float s0 = dest.final_row ? w0 * inv : w0, s1 = dest.final_row ? w1 * inv : w1;
  // a final row without a valid result is zero (a select: O may hold anything
  // after a skipped page or a timeout)
  const bool zero_row = dest.final_row && inv == 0.f;
  {
    // this thread writes columns [D/2 half + CW sub, + CW) of the row
    uint32_t oa[CW], ob[CW];
    tc_ld16x2_cols<CW, CW>(lane_tmem + TT::kOCol + half * (D / 2), oa);
    tc_ld16x2_cols<CW, CW>(lane_tmem + TT::kOCol + D + half * (D / 2), ob);
    tc_wait_ld();
    if (valid) {
      const int col = half * (D / 2) + sub * CW;
      float4 *dst = reinterpret_cast<float4 *>((dest.final_row ? p.out + row * D : p.part_o + ps * D) + col);
#pragma unroll
      for (int j = 0; j < CW / 4; ++j) {
        float v[4];
#pragma unroll
        for (int e = 0; e < 4; ++e)
          v[e] = zero_row ? 0.f : __uint_as_float(oa[4 * j + e]) * s0 + __uint_as_float(ob[4 * j + e]) * s1;
        dst[j] = make_float4(v[0], v[1], v[2], v[3]);
      }
    }
  }
  if (valid && half == 0 && sub == 0) {
    if (dest.final_row) {
      if (p.lse) p.lse[row] = bad ? kNegInf : lse_from_state(m_row, l_row);
      if (dest.slot < 0 && p.part_l) p.part_l[row * p.num_splits] = kLFinal;
    } else {
      p.part_m[ps] = m_row;
      p.part_l[ps] = bad ? kLBadPage : l_row;
    }
  }
  tc_fence_before();
  if (dest.slot < 0 && p.unit_ctr != nullptr && !dest.final_row) tc_merge_unit<D>(p, pc, sm, merge_here);
  return tc_piece_done(stop, abort_flag, sm, kSM) && ok;
}

// Softmax warps with up to 128 rows, for one piece (as tc_softmax_spread):
// row i is lane i, two threads per row (warps w and w + 4 share the lanes of
// quarter w % 4), each on 32 of a tile's 64 tokens with a softmax state and an
// O of its own, merged once at the end.
template <class TT, bool PAGED>
__device__ __forceinline__ bool tc_softmax_wide(const DecodeParams &p, const Piece &pc, uint8_t *smem,
                                                uint32_t tmem, const TcBars &bars, volatile int *tile_bad,
                                                volatile int *abort_flag, volatile int *merge_here,
                                                  volatile int *stop, int gt0,
                                                int n_tiles, const TcDest &dest, int warp, int lane) {
  static_assert(TT::kD == 128, "the 128-row layout runs at d = 128");
  constexpr int D = TT::kD;
  constexpr int T = TT::kT;
  constexpr int ST = TT::kStages;
  constexpr int SP = TT::kSP;
  constexpr int kSM = 32 * TT::kSoftmaxWarps;  // softmax threads
  const float kNegInf = -__int_as_float(0x7f800000);
  const int sm = threadIdx.x;                  // 0 .. kSM-1
  const int half = sm / 128;                   // tokens [32 half, 32 half + 32) of every tile
  const int r = sm % 128;                      // row of the slice = tensor-memory lane
  const bool valid = r < pc.nh;
  const bool warp_active = (warp % 4) * 32 < pc.nh;
  // the positions this row sees: with several query tokens per sequence,
  // query token t sees the cache up to and including itself (a padding row,
  // q = 0, sees the whole piece: its scores are 0, its result unused, and it
  // keeps to the unmasked path of its warp)
  const int lim = valid ? min(pc.t_end, pc.len - (p.nq - 1 - (pc.h0 + r) / p.r)) : pc.t_end;
  const uint32_t lane_tmem = tmem + (static_cast<uint32_t>((warp % 4) * 32) << 16);
  float *mbase = reinterpret_cast<float *>(smem + TT::kXOff);  // [half][row]
  float *lsum = reinterpret_cast<float *>(smem + TT::kLOff);   // [half][row]
  const float sl = fabsf(p.scale_log2);  // (a negative scale's sign is in Q)
  float m_run = kNegInf, l_run = 0.f;  // this half's base and sum
  int bad = 0;
  bool ok = true;
  for (int t = 0; t < n_tiles; ++t) {
    const int gt = gt0 + t;
    const int t0 = pc.t_begin + t * T;
    const int st = gt % ST;
    const int b = gt % SP;
    ok = __all_sync(0xffffffffu, mbar_wait(bars.s_full0 + 8 * b, (gt / SP) & 1));
    if (!ok) break;
    tc_fence_after();
    uint32_t sv[32];
    tc_ld32(lane_tmem + b * 64 + half * 32, sv);
    tc_wait_ld();
    if (PAGED) bad |= tile_bad[st];
    // V rows past the piece's end may hold anything (even NaN): zero them so
    // that P = 0 there meets zeros
    const int valid_rows = min(T, pc.t_end - t0);
    if (valid_rows < T) {
      uint8_t *vt = smem + st * TT::kStageBytes + TT::kTileBytes;
      for (int idx = sm; idx < (T - valid_rows) * 16; idx += kSM) {
        const int row = valid_rows + idx / 16, c = idx % 16;
        *reinterpret_cast<uint4 *>(vt + (c >> 3) * TT::kHalf + row * 128 + ((c & 7) << 4)) =
            make_uint4(0u, 0u, 0u, 0u);
      }
    }
    float x[32];
    const int tb = t0 + half * 32;  // this thread's first token of the tile
    if (tb + 32 <= lim) {
      // all of them visible (every tile but the row's last)
#pragma unroll
      for (int j = 0; j < 32; ++j) x[j] = __uint_as_float(sv[j]) * sl;
    } else {
#pragma unroll
      for (int j = 0; j < 32; ++j) x[j] = (tb + j < lim) ? __uint_as_float(sv[j]) * sl : kNegInf;
    }
    float mx;
    {
      float m8[8];  // a tree, not a chain of 32 dependent steps
#pragma unroll
      for (int k = 0; k < 8; ++k) m8[k] = fmaxf(fmaxf(x[4 * k], x[4 * k + 1]), fmaxf(x[4 * k + 2], x[4 * k + 3]));
      mx = fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])), fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7])));
    }
    if (warp_active) {
      // lazy rescale: only when a score passes the base by more than 2^8
      const bool need = mx > m_run + 8.f;
      if (__any_sync(0xffffffffu, need)) {
        const float mn = need ? fmaxf(m_run, mx) : m_run;
        const float alpha = need ? ((m_run == kNegInf) ? 0.f : ex2(m_run - mn)) : 1.f;
        l_run *= alpha;
        if (t > 0) {
          // this half's O holds the piece's tiles 0 .. t-1: rescale it once their MMAs are done
          ok = __all_sync(0xffffffffu, mbar_wait(bars.pv_done0 + 8 * ((gt - 1) % SP), ((gt - 1) / SP) & 1));
          if (!ok) break;
          tc_fence_after();
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t ov[32];
            tc_ld32(lane_tmem + TT::kOCol + half * D + c * 32, ov);
            tc_wait_ld();
#pragma unroll
            for (int j = 0; j < 32; ++j) ov[j] = __float_as_uint(__uint_as_float(ov[j]) * alpha);
            tc_st32(lane_tmem + TT::kOCol + half * D + c * 32, ov);
          }
          tc_wait_st();
          tc_fence_before();
        }
        m_run = mn;
      }
      const float base = (m_run == kNegInf) ? 0.f : m_run;
      // P over this thread's own 32 score columns: high part in the first
      // 16, residual in the next 16 (the buffer's scores of tile t are no
      // longer needed, and the MMAs of tile t-SP that read it are done, since
      // the scores of tile t came after them)
      uint32_t hi[16], lo[16];
      uint64_t ls2 = f32x2(0.f, 0.f);  // the tile's sum, even and odd columns apart
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        const float p0 = ex2(x[2 * e] - base), p1 = ex2(x[2 * e + 1] - base);
        ls2 = add_f32x2(ls2, f32x2(p0, p1));
        split_bf16x2_rz_x2(p0, p1, hi[e], lo[e]);
      }
      {
        float la, lb;
        f32x2_get(ls2, la, lb);
        l_run += la + lb;
      }
      tc_st16(lane_tmem + b * 64 + half * 32, hi);
      tc_st16(lane_tmem + b * 64 + half * 32 + 16, lo);
      tc_wait_st();
    }
    // (p_full is one barrier per P buffer: a warp reaches tile t+SP only
    // after s_full of t+SP, and the scores of t+SP are issued only once the
    // P.V of tile t is done, so its next arrival on the same barrier cannot
    // fall into tile t's phase)
    tc_fence_before();
    if (valid_rows < T) fence_proxy_async_smem();  // the zeroed V rows, for the tensor core
    __syncwarp();
    if (lane == 0) mbar_arrive(bars.p_full0 + 8 * b);
  }
  if (!ok && lane == 0) {
    *abort_flag = 1;
    if (p.status) atomicOr(p.status, kStatusTimeout);
  }
  // ---- the row's result: O from tensor memory once the last MMAs are done
  const int glast = gt0 + n_tiles - 1;
  const bool done = ok && __all_sync(0xffffffffu, mbar_wait(bars.pv_done0 + 8 * (glast % SP), (glast / SP) & 1));
  tc_fence_after();
  // the row's two partial states, merged exactly: M = max(m0, m1), weights
  // 2^(m_h - M) (0 for a half that saw no position)
  mbase[half * 128 + r] = m_run;
  lsum[half * 128 + r] = l_run;
  named_barrier(1, kSM);
  const float m0 = mbase[r], m1 = mbase[128 + r];
  const float m_row = fmaxf(m0, m1);
  const float w0 = (m0 == kNegInf) ? 0.f : ex2(m0 - m_row), w1 = (m1 == kNegInf) ? 0.f : ex2(m1 - m_row);
  const float l_row = lsum[r] * w0 + lsum[128 + r] * w1;
  const size_t row = valid ? row_of(p, pc.s, pc.g, pc.h0 + r) : 0;
  const size_t ps = tc_part_index(p, pc, dest, row, r);
  const float inv = (!bad && done && l_row > 0.f) ? 1.f / l_row : 0.f;
  const float s0 = dest.final_row ? w0 * inv : w0, s1 = dest.final_row ? w1 * inv : w1;
  // a final row without a valid result is zero (a select: O may hold anything
  // after a skipped page or a timeout)
  const bool zero_row = dest.final_row && inv == 0.f;
#pragma unroll
  for (int c = 0; c < 2; ++c) {
    uint32_t oa[32], ob[32];
    const int col = half * 64 + c * 32;  // this thread writes columns [64 half, 64 half + 64)
    tc_ld32(lane_tmem + TT::kOCol + col, oa);
    tc_ld32(lane_tmem + TT::kOCol + D + col, ob);
    tc_wait_ld();
    if (valid) {
      float4 *dst = reinterpret_cast<float4 *>((dest.final_row ? p.out + row * D : p.part_o + ps * D) + col);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        float v[4];
#pragma unroll
        for (int e = 0; e < 4; ++e)
          v[e] = zero_row ? 0.f : __uint_as_float(oa[4 * j + e]) * s0 + __uint_as_float(ob[4 * j + e]) * s1;
        dst[j] = make_float4(v[0], v[1], v[2], v[3]);
      }
    }
  }
  if (valid && half == 0) {
    if (dest.final_row) {
      if (p.lse) p.lse[row] = bad ? kNegInf : lse_from_state(m_row, l_row);
      if (dest.slot < 0 && p.part_l) p.part_l[row * p.num_splits] = kLFinal;
    } else {
      p.part_m[ps] = m_row;
      p.part_l[ps] = bad ? kLBadPage : l_row;
    }
  }
  tc_fence_before();
  if (dest.slot < 0 && p.unit_ctr != nullptr && !dest.final_row) tc_merge_unit<128>(p, pc, sm, merge_here);
  return tc_piece_done(stop, abort_flag, sm, kSM) && ok;
}

// The Q K^T products of one piece (one thread): S[gt % SP] = Q K_gt^T for
// the piece's tiles, once K has landed and the buffer's last P.V is done.
template <class TT>
__device__ __forceinline__ bool tc_issue_qk(uint32_t sbase, uint32_t qbuf, uint32_t tmem, const TcBars &bars,
                                            int gt0, int n_tiles) {
  constexpr int D = TT::kD;
  constexpr int ST = TT::kStages;
  constexpr int SP = TT::kSP;
  constexpr int T = TT::kT;
  constexpr uint32_t kIdescQK = tc_idesc_bf16(TT::kQRows, T, false);
  // Q's descriptors are the same for every tile; a K-step adds to the
  // start-address field (addresses stay below 256 KB: no carry)
  uint64_t qd[D / 16];
#pragma unroll
  for (int ks = 0; ks < D / 16; ++ks)
    qd[ks] = tc_smem_desc(qbuf + (ks >> 2) * TT::kQHalf + (ks & 3) * 32, 16, 1024);
  for (int t = 0; t < n_tiles; ++t) {
    const int gt = gt0 + t;
    const int st = gt % ST;
    bool ok = mbar_wait_role(bars.full0 + 8 * st, (gt / ST) & 1);
    if (ok && gt >= SP) ok = mbar_wait_role(bars.pv_done0 + 8 * (gt % SP), ((gt / SP) - 1) & 1);
    if (!ok) return false;
    tc_fence_after();
    const uint64_t kd = tc_smem_desc(sbase + st * TT::kStageBytes, 16, 1024);
    const uint32_t d = tmem + (gt % SP) * T;
    tc_mma(d, qd[0], kd, kIdescQK, 0u);
#pragma unroll
    for (int ks = 1; ks < D / 16; ++ks)
      tc_mma(d, qd[ks], kd + ((static_cast<uint32_t>((ks >> 2) * TT::kHalf + (ks & 3) * 32)) >> 4), kIdescQK, 1u);
    tc_commit(bars.s_full0 + 8 * (gt % SP));
  }
  return true;
}

// The P.V products of one piece (one thread): O_h += P V for the piece's
// tiles, the high part and the residual of P read from tensor memory; the
// piece's first tile starts the accumulators afresh.
template <class TT, bool SPREAD>
__device__ __forceinline__ bool tc_issue_pv(uint32_t sbase, uint32_t tmem, const TcBars &bars, int gt0,
                                            int n_tiles) {
  constexpr int D = TT::kD;
  constexpr int T = TT::kT;
  constexpr int ST = TT::kStages;
  constexpr int SP = TT::kSP;
  constexpr uint32_t kIdescPV = tc_idesc_bf16(TT::kQRows, D, true);
  // each thread wrote the P of TPT tokens over its TPT score columns: the high
  // part over the first TPT/2, the residual over the next TPT/2 (SPREAD: four
  // threads per row, TPT = T/4; otherwise two, TPT = T/2)
  constexpr int TPT = SPREAD ? T / 4 : T / 2;
  for (int u = 0; u < n_tiles; ++u) {
    const int gt = gt0 + u;
    const int st = gt % ST;
    if (!mbar_wait_role(bars.p_full0 + 8 * (gt % SP), (gt / SP) & 1)) return false;
    tc_fence_after();
    const uint64_t vd = tc_smem_desc(sbase + st * TT::kStageBytes + TT::kTileBytes, TT::kHalf, 1024);
    const uint32_t pb = tmem + (gt % SP) * T;
#pragma unroll
    for (int ks = 0; ks < T / 16; ++ks) {
      // tokens 16 ks .. 16 ks + 15: those of thread group g = 16 ks / TPT, its
      // (16 ks % TPT) / 16-th 16 tokens; into the O of the half of the row
      // (tokens [T/2 h, T/2 h + T/2)) that owns them
      const uint64_t vdk = vd + ((ks * 16 * 128) >> 4);
      const int g = (16 * ks) / TPT, k2 = ((16 * ks) % TPT) / 16;
      const uint32_t pa = pb + g * TPT + 8 * k2;
      const int h = (16 * ks) / (T / 2);
      const uint32_t od = tmem + TT::kOCol + D * h;
      const bool first = (16 * ks) % (T / 2) == 0;  // the half's first tokens of the tile
      tc_mma_ts(od, pa, vdk, kIdescPV, (u > 0 || !first) ? 1u : 0u);
      tc_mma_ts(od, pa + TPT / 2, vdk, kIdescPV, 1u);
    }
    // K was read by the scores of this tile, done before its P existed; V and
    // P by these products
    tc_commit(bars.empty0 + 8 * st);
    tc_commit(bars.pv_done0 + 8 * (gt % SP));
  }
  return true;
}

// An issuer's last step: every product it issued is done before the block
// tears down (on an early exit, products already issued may still be running).
__device__ __forceinline__ void tc_issuer_drain(uint32_t drain_bar, const DecodeParams &p) {
  tc_commit(drain_bar);
  if (!mbar_wait(drain_bar, 0) && p.status) atomicOr(p.status, kStatusTimeout);
}

__device__ __forceinline__ void tc_abort(const DecodeParams &p, volatile int *abort_flag) {
  *abort_flag = 1;
  if (p.status) atomicOr(p.status, kStatusTimeout);
}

// SPREAD (at most 64 rows): the rows sit in the first 16 lanes of each of the
// four tensor-memory lane quarters, ceil(rows / 4) per quarter, so that the
// softmax work is shared by all four SM sub-partitions; four threads take
// each row (two warps, 16 tokens each of their 32), through the 16-lane
// tensor-memory shapes.  Otherwise (up to 128 rows) row i is lane i and two
// threads take each row.
template <bool PAGED, bool SPREAD, int DH = 128>
__global__ void __launch_bounds__(TcTile::kThreads, 1)
    gqa_verify_tc_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                         const DecodeParams p) {
  static_assert(DH == 128 || SPREAD, "d = 64 runs the spread layout (at most 64 rows)");
  using TT = TcItemTile<SPREAD, DH>;
  constexpr int D = TT::kD;
  constexpr int T = TT::kT;
  const float kNegInf = -__int_as_float(0x7f800000);

  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_addr(smem);
  const TcBars bars = tc_bars<TT>(sbase);
  volatile uint32_t *tmem_slot = reinterpret_cast<volatile uint32_t *>(smem + TT::kMiscOff);
  volatile int *tile_bad = reinterpret_cast<volatile int *>(smem + TT::kMiscOff + 4);  // [ST]
  volatile int *abort_flag = tile_bad + TT::kStages;
  volatile int *merge_here = tile_bad + TT::kStages + 1;
  volatile int *stop = tile_bad + TT::kStages + 2;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // The block's own setup (barriers, tensor memory) touches no global memory:
  // it runs before the wait for the previous kernel on the stream.
  constexpr int kProducerWarp = TT::kSoftmaxWarps;  // then the Q K^T issuer (allocates), the P.V issuer
  constexpr int kMmaWarp = TT::kSoftmaxWarps + 1, kPvWarp = TT::kSoftmaxWarps + 2;
  if (threadIdx.x == 0) {
    tc_init_bars<TT>(bars, tile_bad, TT::kQRows);  // one arrival per Q slot
    *abort_flag = 0;
    *merge_here = 0;
    *stop = 0;
    fence_mbarrier_init();
  }
  if (warp == kMmaWarp) {
    tc_alloc(smem_addr(const_cast<uint32_t *>(tmem_slot)), TT::kTmemCols);
    tc_relinquish();
  }
  if (warp == kProducerWarp) {
    if (lane == 0) {
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
    }
    prefetch_piece_l2<D, T, Mode::kItems, PAGED>(&tm_k, &tm_v, p, lane);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  pdl_wait_primary();
  const Piece pc = make_item<T, Mode::kItems>(p);
  if (threadIdx.x == 0) pdl_launch_dependents();
  if (pc.nh <= 0 || pc.t_begin >= pc.t_end) {
    // nothing to read; an invalid length is handled once, by split 0
    if (pc.nh > 0 && !pc.len_ok && pc.k == 0) {
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
    if (warp == kMmaWarp) tc_dealloc(tmem, TT::kTmemCols);
    return;
  }
  // a unit with several splits: claim its arrival word for this call
  if (threadIdx.x == 0 && p.unit_ctr != nullptr && (pc.len + p.split_tokens - 1) / p.split_tokens > 1)
    unit_claim(p.unit_ctr + (static_cast<size_t>(pc.s) * p.G + pc.g) * p.hs + pc.j, p.epoch);
  if (threadIdx.x < TT::kQRows) {
    // the q row of this thread's slot into Q (padding slots are zero), while
    // the producer already streams K and V; the Q K^T issuer waits for all
    // the slots
    const int r = threadIdx.x;
    const int rho = tc_slot_row<SPREAD>(r, pc.nh);
    const uint4 *src = rho >= 0 ? reinterpret_cast<const uint4 *>(p.q + row_of(p, pc.s, pc.g, pc.h0 + rho) * D)
                                : nullptr;
    // (a negative scale: the sign goes into q, exactly, so that the softmax
    // threads scale by |scale|)
    const uint32_t flip = p.scale_log2 < 0.f ? 0x80008000u : 0u;
#pragma unroll
    for (int c = 0; c < D / 8; ++c) {
      uint4 v = rho >= 0 ? __ldg(src + c) : make_uint4(0u, 0u, 0u, 0u);
      v.x ^= flip;
      v.y ^= flip;
      v.z ^= flip;
      v.w ^= flip;
      *reinterpret_cast<uint4 *>(smem + TT::kQOff + tc_q_offset<TT>(r, c)) = v;
    }
    fence_proxy_async_smem();
    mbar_arrive(bars.q_full0);
  }
  const int n_tiles = (pc.t_end - pc.t_begin + T - 1) / T;

  if (warp == kProducerWarp) {
    // ============================================================ producer
    int tile = 0;
    (void)tc_produce_piece<TT, PAGED>(&tm_k, &tm_v, p, pc, sbase, bars, tile_bad, abort_flag, lane, tile);
    tc_produce_drain<TT>(bars, tile, lane);
  } else if (warp == kMmaWarp) {
    // ============================================================ Q K^T issuer
    if (lane == 0) {
      const bool ok = mbar_wait_role(bars.q_full0, 0) && tc_issue_qk<TT>(sbase, sbase + TT::kQOff, tmem, bars, 0, n_tiles);
      if (!ok) tc_abort(p, abort_flag);
      tc_issuer_drain(bars.drain0, p);
    }
  } else if (warp == kPvWarp) {
    // ============================================================ P.V issuer
    if (lane == 0) {
      if (!tc_issue_pv<TT, SPREAD>(sbase, tmem, bars, 0, n_tiles)) tc_abort(p, abort_flag);
      tc_issuer_drain(bars.drain0 + 8, p);
    }
  } else {
    // ============================================================ softmax rows
    const TcDest dest{((pc.len + p.split_tokens - 1) / p.split_tokens == 1) && p.out != nullptr, -1};
    if constexpr (SPREAD)
      (void)tc_softmax_spread<TT, PAGED>(p, pc, smem, tmem, bars, tile_bad, abort_flag, merge_here, stop, 0,
                                         n_tiles, dest, warp, lane);
    else
      (void)tc_softmax_wide<TT, PAGED>(p, pc, smem, tmem, bars, tile_bad, abort_flag, merge_here, stop, 0,
                                       n_tiles, dest, warp, lane);
  }

  // ---- teardown: every tensor-memory access is done before the columns go
  // back (the two issuers waited above for their last products to finish)
  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tc_dealloc(tmem, TT::kTmemCols);
  }
}

}  // namespace gqa
