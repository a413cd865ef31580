// Backward of the prefill over the flat, deduplicated packed layout.  The
// flat layout has to give the gradients of running every [prefix; s_i] on
// its own, so the prefix K/V collect the gradients of every suffix that sees
// them ("KV-0 redundancy prefix sharing attention mask design", PrefixSharing
// PR #50: design summary and test plan -- gradient equivalence).  For a query
// row with upstream gradient dO and the visible keys of the tile schedule:
//   P = exp(scale q.k - LSE), D = dO . O,
//   dV += P^T dO,  dS = P (dO V^T - D),  dQ += scale dS K,  dK += scale dS^T Q.
//
// Three launches, no atomics:
//   prep     -D and -LSE (log2 domain) per (row, head), stored head-major so a
//            tile of 64 rows is one contiguous 256-byte run; stored negated so
//            two adjacent columns feed a paired fp32 add as one 8-byte load.
//   dq pass  row-major over the forward's kind of schedule (blocks of 128
//            rows, KV tiles of 64 keys): a CTA owns one (row block, query
//            head) and streams the K and V tiles its rows see.
//   dkdv     key-major over the schedule of the transposed spec (blocks of
//            128 keys, query tiles of 64 rows): a CTA owns one (key block, KV
//            head) and streams the Q / dO tiles (with their LSE and D) of
//            every query head of the group that sees it.
// Both passes are one kernel template on the 5th-generation tensor cores.
// With X1, X2 the unit's 128-row block operands and Y1, Y2 a streamed tile
// (dq: X = Q, dO and Y = K, V; dkdv: X = K, V and Y = Q, dO):
//   S  = X1 Y1^T and dP = X2 Y2^T      tcgen05 SS MMAs into TMEM (M = 128,
//                                      N = 64), double-buffered per tile;
//   P, dS from S and dP                one thread per block row (= TMEM lane)
//                                      writes them back to TMEM as bf16;
//   dq:   dQ += dS Y1                  tcgen05 TS MMAs (A from TMEM), the
//   dkdv: dV += P^T Y2, dK += dS^T Y1  accumulators stay in TMEM per unit.
// Warps: 0 TMA producer (128-byte swizzle, no multicast), 1 MMA issuer and
// TMEM owner, 4-7 and 8-11 two compute warpgroups that split every tile's
// columns (while they work on tile t the tensor pipe runs tile t+1's S and
// dP), and both run the unit's epilogue.  Every wait is bounded and reports
// PSA_ERR_TIMEOUT instead of hanging; TMEM is freed on every exit path.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <type_traits>

#include "psa_debug.cuh"
#include "psa_device.cuh"
#include "psa_internal.h"

namespace psa {
namespace {

constexpr int BR = 64;             // rows of a half-block (the schedule's rectangle ranges)
constexpr int BLK = 2 * BR;        // rows (or keys) per schedule block = TMEM lanes
constexpr int BT = 64;             // columns per streamed tile
constexpr int kThreads = 384;      // 12 warps
// streamed tiles in flight: the tiles the MMAs still read (two TMEM
// buffers' worth) plus one being prefetched
constexpr int kStages = 3;
constexpr uint32_t kTmemCols = 512;

enum { kDq = 0, kDkdv = 1 };

__device__ __forceinline__ bool sched_ok(const int32_t* sch, int64_t len) {
  const int32_t n_items = __ldg(sch + 1), n_kv = __ldg(sch + 2), n_rect = __ldg(sch + 3);
  return __ldg(sch + 0) == 0x50534132 && __ldg(sch + 4) == BLK && __ldg(sch + 5) == BT &&
         n_items >= 0 && n_kv >= 0 && n_rect >= 0 &&
         8 + 4 * int64_t(n_items) + 8 * int64_t(n_kv) + 5 * int64_t(n_rect) <= len;
}

// Columns [c0, c0 + BT) of row `row` that the copied rectangles [rb, rb + rc)
// make visible, as a 64-bit mask.  Rows and columns are in the schedule's
// orientation (keys are rows in the transposed spec, whose causal rectangles
// carry causal == 2: row sees col iff col - k0 >= row - q0).
__device__ __forceinline__ uint64_t rect_mask(const int32_t* rects, int rb, int rc, int row,
                                              int c0, int32_t n_rect, int32_t* status) {
  uint64_t m = 0;
  if (!psa_in_bounds(rb >= 0 && rc >= 0 && int64_t(rb) + rc <= n_rect, status)) return 0;
  for (int i = 0; i < rc; ++i) {
    const int32_t* r = rects + 5 * (rb + i);
    const int q0 = __ldg(r), q1 = __ldg(r + 1), k0 = __ldg(r + 2), k1 = __ldg(r + 3);
    const int c = __ldg(r + 4);
    if (row < q0 || row >= q1) continue;
    int lo = k0, hi = k1;
    if (c == 1) hi = min(hi, k0 + (row - q0) + 1);
    if (c == 2) lo = max(lo, k0 + (row - q0));
    lo = max(lo - c0, 0);
    hi = min(hi - c0, BT);
    if (lo >= hi) continue;
    const uint64_t upto_hi = hi >= 64 ? ~0ull : ((1ull << hi) - 1ull);
    const uint64_t below_lo = (1ull << lo) - 1ull;
    m |= upto_hi & ~below_lo;
  }
  return m;
}

// ---------------------------------------------------------------- prep

__global__ void __launch_bounds__(256) bwd_prep_kernel(const __nv_bfloat16* __restrict__ o,
                                                       const __nv_bfloat16* __restrict__ dout,
                                                       const float* __restrict__ lse,
                                                       float* __restrict__ lse2_t,
                                                       float* __restrict__ delta_t, int T, int Tp,
                                                       int Hq, int D) {
  const int gw = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  if (gw >= T * Hq) return;
  const int t = gw / Hq, h = gw % Hq;
  const __nv_bfloat16* op = o + (size_t(t) * Hq + h) * D;
  const __nv_bfloat16* dp = dout + (size_t(t) * Hq + h) * D;
  float s = 0.f;
  for (int e = lane * 2; e < D; e += 64) {
    const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(op + e));
    const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(dp + e));
    s += a.x * b.x + a.y * b.y;
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
  if (lane == 0) {
    delta_t[size_t(h) * Tp + t] = -s;
    lse2_t[size_t(h) * Tp + t] = -lse[size_t(t) * Hq + h] * kLog2e;
  }
}

// ---------------------------------------------------------------- the tensor-core passes

struct BwdParams {
  const int32_t* sched;
  int64_t sched_len;
  const float* lse2_t;        // [Hq, Tp], -LSE * log2(e)
  const float* delta_t;       // [Hq, Tp], -D
  __nv_bfloat16* dq;          // [T, Hq, D]
  __nv_bfloat16* dk;          // [T, Hkv, D]
  __nv_bfloat16* dv;
  int32_t T, Tp, Hq, Hkv, G;  // Tp: T rounded up to a multiple of 4 (row stride of the stats)
  float scale, scale_log2;
  int32_t* status;
};

template <int D, int MODE>
struct TcCfg {
  static constexpr int NST = kStages;
  static constexpr int NPART = D / 64;              // 128-byte swizzle atoms across d
  static constexpr uint32_t BLOCK = BLK * D * 2;    // one block operand
  static constexpr uint32_t TILE = BT * D * 2;      // one tile operand
  // dkdv: + LSE and D of the tile, BT + 4 floats each (the copy starts at the
  // tile's first row rounded down to a multiple of 4 so the TMA x coordinate
  // stays 16-byte aligned), each on a 512-byte slot; stages stay 1 KB aligned.
  static constexpr uint32_t STAT = (BT + 4) * 4;
  static constexpr uint32_t STAT_SLOT = 512;
  static constexpr uint32_t STAGE = 2 * TILE + (MODE == kDkdv ? 2 * STAT_SLOT : 0u);
  static constexpr uint32_t STAGE_TX = 2 * TILE + (MODE == kDkdv ? 2 * STAT : 0u);
  static constexpr uint32_t OFF_BLK = 0;
  static constexpr uint32_t OFF_RING = 2 * BLOCK;
  static constexpr uint32_t OFF_BAR = OFF_RING + NST * STAGE;
  static constexpr int NBAR = 2 + 2 * NST + 3 + 3 + 2;
  // at least 116 KB, so that one CTA (holding all 512 TMEM columns) fits per SM
  static constexpr uint32_t SMEM_USED = 1024 + OFF_BAR + NBAR * 8 + 16;
  static constexpr uint32_t SMEM = SMEM_USED > 116u * 1024 ? SMEM_USED : 116u * 1024;
  // TMEM columns: buffer b holds S at 128 b and dP at 128 b + 64 (P and dS
  // overwrite their first 32 columns as packed bf16); the accumulators follow.
  // Two buffers: the MMA issuer runs one tile ahead of the P / dS warps.
  // (dq has TMEM room for a third; with a deeper ring to match it measured
  // the same, the tensor pipe being the limit there.)
  static constexpr int NBUF = 2;
  static constexpr uint32_t T_ACC = NBUF * 128;  // dkdv: dV then dK; dq: dQ
  static_assert(T_ACC + (MODE == kDq ? D : 2 * D) <= kTmemCols, "TMEM budget");
};

// Column (within a 64-column S or dP region of TMEM) of the packed bf16 P or
// dS that k-step ks (16 tile columns) of the accumulating products reads:
// the warpgroup that made tile columns 32 w .. 32 w + 31 packs them over the
// first 16 of the fp32 columns it read, at 32 w.
__host__ __device__ constexpr uint32_t a_col(int ks) { return (ks >> 1) * 32 + (ks & 1) * 8; }

struct Bars {
  uint64_t *blk_full, *blk_empty, *ring_full, *ring_empty, *s_full, *p_full, *acc_full,
      *acc_free;
};

// Unit of this CTA in round r.  Units are listed longest first; odd rounds
// hand them out in reverse CTA order, so the CTAs that got the longest units
// of one round get the shortest of the next.
__device__ __forceinline__ int snake_unit(int r) {
  const int lane_in_round = (r & 1) ? int(gridDim.x) - 1 - int(blockIdx.x) : int(blockIdx.x);
  return r * int(gridDim.x) + lane_in_round;
}

// The unit's schedule item and head (dq: query head; dkdv: KV head) and its
// number of streamed tiles (dkdv: every query head of the group).
template <int MODE>
__device__ __forceinline__ int unit_tiles(const BwdParams& p, const int4* items, int32_t n_kv,
                                          int u, int4& it, int& head) {
  const int H = MODE == kDq ? p.Hq : p.Hkv;
  it = __ldg(items + u / H);
  head = u % H;
  // a block outside the schedule or the tokens becomes an empty one for
  // every role (debug build)
  if (!psa_in_bounds(it.x >= 0 && it.y >= 0 && it.y <= BLK && int64_t(it.x) + it.y <= p.T &&
                         it.z >= 0 && it.w >= 0 && int64_t(it.z) + it.w <= n_kv,
                     p.status))
    it = make_int4(0, 0, 0, 0);
  return MODE == kDq ? it.w : it.w * p.G;
}

template <int D, int MODE>
__global__ void __launch_bounds__(kThreads, 1)
    bwd_tc_kernel(const __grid_constant__ CUtensorMap tm_x1, const __grid_constant__ CUtensorMap tm_x2,
                  const __grid_constant__ CUtensorMap tm_y1, const __grid_constant__ CUtensorMap tm_y2,
                  const __grid_constant__ CUtensorMap tm_lse, const __grid_constant__ CUtensorMap tm_dlt,
                  BwdParams p) {
  using C = TcCfg<D, MODE>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  __shared__ int abort_flag;
  __shared__ uint32_t tmem_slot;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int32_t* sch = p.sched;
  if (!sched_ok(sch, p.sched_len)) {
    if (threadIdx.x == 0) report_status(p.status, PSA_ERR_INVALID_ARG);
    return;
  }
  const int32_t n_items = __ldg(sch + 1), n_kv = __ldg(sch + 2), n_rect = __ldg(sch + 3);
  const int4* items = reinterpret_cast<const int4*>(sch + 8);
  const int32_t* tiles = sch + 8 + 4 * n_items;  // the column tiles of each block
  const int32_t* rects = tiles + 8 * n_kv;
  const int units = n_items * (MODE == kDq ? p.Hq : p.Hkv);

  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  Bars B;
  B.blk_full = bar;
  B.blk_empty = bar + 1;
  B.ring_full = bar + 2;
  B.ring_empty = B.ring_full + C::NST;
  B.s_full = B.ring_empty + C::NST;
  B.p_full = B.s_full + C::NBUF;
  B.acc_full = B.p_full + C::NBUF;
  B.acc_free = B.acc_full + 1;
  if (threadIdx.x == 0) {
    abort_flag = 0;
    mbar_init(B.blk_full, 1);
    mbar_init(B.blk_empty, 1);
    for (int i = 0; i < C::NST; ++i) {
      mbar_init(B.ring_full + i, 1);
      mbar_init(B.ring_empty + i, 1);
    }
    for (int i = 0; i < C::NBUF; ++i) {
      mbar_init(B.s_full + i, 1);
      mbar_init(B.p_full + i, 8);  // both compute warpgroups (half a tile each)
    }
    mbar_init(B.acc_full, 1);
    mbar_init(B.acc_free, 8);      // both compute warpgroups
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;

  if (warp == 0) {
    // ================================================================ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tm_x1);
      tma_prefetch_desc(&tm_x2);
      tma_prefetch_desc(&tm_y1);
      tma_prefetch_desc(&tm_y2);
      uint32_t n = 0, ub = 0;
      bool ok = true;
      for (int r = 0; ok; ++r) {
        const int u = snake_unit(r);
        if (u >= units) break;
        int4 it;
        int head;
        const int nt = unit_tiles<MODE>(p, items, n_kv, u, it, head);
        if (nt == 0) continue;
        // block operands X1, X2 (rows it.x .. it.x + 127 of this head)
        if (!mbar_wait(B.blk_empty, (ub & 1) ^ 1, &abort_flag, p.status)) break;
        mbar_arrive_expect_tx(B.blk_full, 2 * C::BLOCK);
#pragma unroll
        for (int part = 0; part < C::NPART; ++part) {
          tma_load_3d(smem + C::OFF_BLK + part * BLK * 128, &tm_x1, B.blk_full, part * 64, head,
                      it.x);
          tma_load_3d(smem + C::OFF_BLK + C::BLOCK + part * BLK * 128, &tm_x2, B.blk_full,
                      part * 64, head, it.x);
        }
        for (int t = 0; t < nt; ++t, ++n) {
          const int j = MODE == kDq ? t : t % it.w;
          const int yh = MODE == kDq ? head / p.G : head * p.G + t / it.w;
          const int c0 = __ldg(tiles + 8 * (it.z + j));
          const int s = n % C::NST;
          if (!mbar_wait(B.ring_empty + s, ((n / C::NST) & 1) ^ 1, &abort_flag, p.status)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(B.ring_full + s, C::STAGE_TX);
          uint8_t* dst = smem + C::OFF_RING + s * C::STAGE;
#pragma unroll
          for (int part = 0; part < C::NPART; ++part) {
            tma_load_3d(dst + part * BT * 128, &tm_y1, B.ring_full + s, part * 64, yh, c0);
            tma_load_3d(dst + C::TILE + part * BT * 128, &tm_y2, B.ring_full + s, part * 64, yh,
                        c0);
          }
          if constexpr (MODE == kDkdv) {
            tma_load_2d(dst + 2 * C::TILE, &tm_lse, B.ring_full + s, c0 & ~3, yh);
            tma_load_2d(dst + 2 * C::TILE + C::STAT_SLOT, &tm_dlt, B.ring_full + s, c0 & ~3, yh);
          }
        }
        ++ub;
      }
      if (!ok || abort_flag) {
        // let copies in flight land before the CTA exits
        const uint64_t t0 = globaltimer();
        while (globaltimer() - t0 < 1000000ull) {
        }
      }
    }
  } else if (warp == 1) {
    // ================================================================ MMA issuer
    if (lane == 0) {
      const uint32_t idesc_s = umma_idesc_bf16(BLK, BT, false, false);
      const uint32_t idesc_acc = umma_idesc_bf16(BLK, D, false, true);
      const uint32_t sX = smem_u32(smem + C::OFF_BLK);
      const uint32_t sR = smem_u32(smem + C::OFF_RING);
      static_assert(C::OFF_RING + C::NST * C::STAGE < (1u << 18), "descriptor address field");
      uint32_t n = 0, ub = 0;
      bool ok = true;
      // Descriptors are built once; a k-step or stage moves only the start
      // address field (bits 0..13, in 16-byte units), so it is a plain add.
      const uint64_t dX = umma_desc_sw128(sX, 16, 1024);
      const uint64_t dR = umma_desc_sw128(sR, 16, 1024);          // K-major tile rows
      const uint64_t dRmn = umma_desc_sw128(sR, BT * 128, 1024);  // MN-major tile rows
      // S = X1 Y1^T and dP = X2 Y2^T of global tile m into TMEM buffer m % NBUF
      auto issue_s = [&](uint32_t m) -> bool {
        const int s = m % C::NST;
        if (!mbar_wait(B.ring_full + s, (m / C::NST) & 1, &abort_flag, p.status)) return false;
        tc_fence_after();
        const uint32_t tb = tmem + (m % C::NBUF) * 128;
        const uint64_t dY = dR + ((s * C::STAGE) >> 4);
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const uint32_t ox = ((ks >> 2) * (BLK * 128) + (ks & 3) * 32) >> 4;
          const uint32_t oy = ((ks >> 2) * (BT * 128) + (ks & 3) * 32) >> 4;
          umma_ss(tb, dX + ox, dY + oy, idesc_s, ks > 0 ? 1u : 0u);
        }
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const uint32_t ox = (C::BLOCK + (ks >> 2) * (BLK * 128) + (ks & 3) * 32) >> 4;
          const uint32_t oy = (C::TILE + (ks >> 2) * (BT * 128) + (ks & 3) * 32) >> 4;
          umma_ss(tb + 64, dX + ox, dY + oy, idesc_s, ks > 0 ? 1u : 0u);
        }
        umma_commit(B.s_full + (m % C::NBUF));
        return true;
      };
      // the accumulating products of global tile m (the unit's tile t)
      auto issue_acc = [&](uint32_t m, int t) -> bool {
        if (!mbar_wait(B.p_full + (m % C::NBUF), (m / C::NBUF) & 1, &abort_flag, p.status))
          return false;
        if (t == 0 && !mbar_wait(B.acc_free, (ub & 1) ^ 1, &abort_flag, p.status)) return false;
        tc_fence_after();
        const uint32_t tb = tmem + (m % C::NBUF) * 128;
        const uint64_t dY = dRmn + (((m % C::NST) * C::STAGE) >> 4);
        // B operands: the tile's rows are the contraction, D the N dimension
#pragma unroll
        for (int ks = 0; ks < BT / 16; ++ks) {
          const uint32_t acc = (t > 0 || ks > 0) ? 1u : 0u;
          if constexpr (MODE == kDq) {
            // dQ += dS K_t
            umma_ts(tmem + C::T_ACC, tb + 64 + a_col(ks), dY + ks * (2048 >> 4), idesc_acc, acc);
          } else {
            // dV += P^T dO_t, dK += dS^T Q_t
            umma_ts(tmem + C::T_ACC, tb + a_col(ks), dY + ((C::TILE + ks * 2048) >> 4), idesc_acc,
                    acc);
            umma_ts(tmem + C::T_ACC + D, tb + 64 + a_col(ks), dY + ks * (2048 >> 4), idesc_acc,
                    acc);
          }
        }
        umma_commit(B.ring_empty + (m % C::NST));
        return true;
      };
      for (int r = 0; ok; ++r) {
        const int u = snake_unit(r);
        if (u >= units) break;
        int4 it;
        int head;
        const int nt = unit_tiles<MODE>(p, items, n_kv, u, it, head);
        if (nt == 0) continue;
        if (!mbar_wait(B.blk_full, ub & 1, &abort_flag, p.status)) break;
        // S runs NBUF - 1 tiles ahead of the accumulating products: the
        // tensor pipe works on later tiles while tile t's P and dS are made
        constexpr int L = C::NBUF - 1;
        for (int t = 0; t < L && t < nt && ok; ++t) ok = issue_s(n + t);
        for (int t = 0; t < nt && ok; ++t) {
          if (t + L < nt) ok = issue_s(n + t + L);
          if (ok) ok = issue_acc(n + t, t);
        }
        if (!ok) break;
        umma_commit(B.blk_empty);
        umma_commit(B.acc_full);
        n += nt;
        ++ub;
      }
      if (!ok || abort_flag) {
        // give MMAs already issued time to finish before TMEM is freed
        const uint64_t t0 = globaltimer();
        while (globaltimer() - t0 < 1000000ull) {
        }
      }
    }
  } else if (warp >= 4) {
    // ================================================================ P, dS and the epilogue
    const int wg = (warp - 4) >> 2;       // takes the tiles m with m % 2 == wg
    const int quarter = warp & 3;         // TMEM lane quarter
    const int row = quarter * 32 + lane;  // row of the block
    const int half = row / BR;
    const uint32_t tlane = tmem + (uint32_t(quarter * 32) << 16);
    uint32_t n = 0, ub = 0;
    bool ok = true;
    for (int r = 0; ok; ++r) {
      const int u = snake_unit(r);
      if (u >= units) break;
      int4 it;
      int head;
      const int nt = unit_tiles<MODE>(p, items, n_kv, u, it, head);
      const int grow = it.x + row;                 // this thread's row (query or key)
      const bool rvalid = row < it.y;
      // epilogue targets: dq writes dQ [T, Hq, D]; dkdv writes dV (wg 0) and dK (wg 1)
      __nv_bfloat16* out = MODE == kDq ? p.dq : (wg == 0 ? p.dv : p.dk);
      const int Hout = MODE == kDq ? p.Hq : p.Hkv;
      const float oscale = (MODE == kDkdv && wg == 0) ? 1.f : p.scale;
      constexpr int OCOLS = MODE == kDq ? D / 2 : D;  // columns this warpgroup writes
      const int ocol0 = MODE == kDq ? wg * (D / 2) : 0;
      const uint32_t tacc = tlane + C::T_ACC + (MODE == kDq ? ocol0 : wg * D);
      if (nt == 0) {
        // nothing in this block sees (or is seen by) anything: zero gradient
        if (rvalid) {
          __nv_bfloat16* dst = out + (size_t(grow) * Hout + head) * D + ocol0;
      const bool out_al32 = (reinterpret_cast<uintptr_t>(out) & 31u) == 0;
          for (int c = 0; c < OCOLS; c += 8)
            *reinterpret_cast<uint4*>(dst + c) = make_uint4(0u, 0u, 0u, 0u);
        }
        continue;
      }
      float lse_row = 0.f, dlt_row = 0.f;  // negated, as stored
      if (MODE == kDq && rvalid) {
        lse_row = __ldg(p.lse2_t + size_t(head) * p.Tp + grow);
        dlt_row = __ldg(p.delta_t + size_t(head) * p.Tp + grow);
      }
      for (int t = 0; t < nt; ++t) {
        const uint32_t m = n + t;

        const int j = MODE == kDq ? t : t % it.w;
        const int32_t* e = tiles + 8 * (it.z + j);
        const int c0 = __ldg(e), clen = __ldg(e + 1), flags = __ldg(e + 6);
        uint64_t vis = 0;
        if (rvalid && (flags & (1 << half))) {
          if (flags & (4 << half))
            vis = clen >= 64 ? ~0ull : ((1ull << clen) - 1ull);
          else
            vis = rect_mask(rects, __ldg(e + 2 + 2 * half), __ldg(e + 3 + 2 * half), grow, c0,
                            n_rect, p.status);
        }
        const float* lse_col = nullptr;  // negated, as stored
        const float* dlt_col = nullptr;
        if constexpr (MODE == kDkdv) {
          const uint8_t* st = smem + C::OFF_RING + (m % C::NST) * C::STAGE + 2 * C::TILE;
          lse_col = reinterpret_cast<const float*>(st) + (c0 & 3);
          dlt_col = reinterpret_cast<const float*>(st + C::STAT_SLOT) + (c0 & 3);
        }
        // the tile's stats came with its TMA copies: observe that phase
        // directly before reading them (dkdv), then wait for S and dP
        if (MODE == kDkdv && !mbar_wait(B.ring_full + (m % C::NST), (m / C::NST) & 1,
                                        &abort_flag, p.status)) {
          ok = false;
          break;
        }
        const int buf = m % C::NBUF;
        if (!mbar_wait(B.s_full + buf, (m / C::NBUF) & 1, &abort_flag, p.status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t tS = tlane + buf * 128, tP = tS + 64;
        // every column visible (the common case): no per-element mask
        const bool all_vis = vis == ~0ull;
        const uint64_t sc2 = f2_pack(p.scale_log2, p.scale_log2), zero2 = f2_pack(0.f, 0.f);
        const uint64_t nl_row2 = f2_pack(lse_row, lse_row), nd_row2 = f2_pack(dlt_row, dlt_row);
        // x = scale_log2 s - lse, P = 2^x, dS = P (dP - D), two columns at a time;
        // PAIRS: the dkdv stats of columns (c, c + 1) are one aligned 8-byte load
        auto tile = [&](auto pairs_tag) {
          [[maybe_unused]] constexpr bool PAIRS = decltype(pairs_tag)::value;
          {
            const int ch = wg;  // this warpgroup's half of the tile: columns 32 ch ..
            uint32_t s[32], dp[32];
            tmem_ld32(tS + ch * 32, s);
            tmem_ld32(tP + ch * 32, dp);
            tmem_wait_ld();
            const uint32_t vm = uint32_t(vis >> (32 * ch));
            uint32_t pk[16], dk[16];
#pragma unroll
            for (int i = 0; i < 32; i += 2) {
              [[maybe_unused]] const int col = ch * 32 + i;
              uint64_t nl2, nd2;
              if constexpr (MODE == kDq) {
                nl2 = nl_row2;
                nd2 = nd_row2;
              } else if constexpr (PAIRS) {
                nl2 = *reinterpret_cast<const uint64_t*>(lse_col + col);
                nd2 = *reinterpret_cast<const uint64_t*>(dlt_col + col);
              } else {
                nl2 = f2_pack(lse_col[col], lse_col[col + 1]);
                nd2 = f2_pack(dlt_col[col], dlt_col[col + 1]);
              }
              const uint64_t x2 =
                  f2_fma(f2_pack(__uint_as_float(s[i]), __uint_as_float(s[i + 1])), sc2, nl2);
              float x0, x1;
              f2_unpack(x2, x0, x1);
              float p0 = fast_exp2(x0), p1 = fast_exp2(x1);
              if (!all_vis) {
                p0 = (vm >> i) & 1u ? p0 : 0.f;
                p1 = (vm >> (i + 1)) & 1u ? p1 : 0.f;
              }
              const uint64_t g2 =
                  f2_add(f2_pack(__uint_as_float(dp[i]), __uint_as_float(dp[i + 1])), nd2);
              float ds0, ds1;
              f2_unpack(f2_fma(f2_pack(p0, p1), g2, zero2), ds0, ds1);
              pk[i / 2] = pack_bf16(p0, p1);
              dk[i / 2] = pack_bf16(ds0, ds1);
            }
            // packed over columns this thread has read itself (32 ch ..)
            if constexpr (MODE == kDkdv) tmem_st16(tS + ch * 32, pk);
            tmem_st16(tP + ch * 32, dk);
          }
        };
        // the stats slot is 512-byte aligned and starts at column -(c0 & 3)
        if (MODE == kDq || ((c0 & 3) & 1) == 0)
          tile(std::true_type{});
        else
          tile(std::false_type{});
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(B.p_full + buf);
      }
      if (!ok) break;
      // epilogue: this warpgroup's accumulator columns of the unit
      if (!mbar_wait(B.acc_full, ub & 1, &abort_flag, p.status)) break;
      tc_fence_after();
      __nv_bfloat16* dst = out + (size_t(grow) * Hout + head) * D + ocol0;
      const bool out_al32 = (reinterpret_cast<uintptr_t>(out) & 31u) == 0;
#pragma unroll
      for (int c = 0; c < OCOLS; c += 32) {
        uint32_t a[32];
        tmem_ld32(tacc + c, a);
        tmem_wait_ld();
        if (rvalid) {
          if (out_al32) {
            // 32-byte stores (a thread's row is its own, so a warp store
            // touches 32 rows; fewer, wider stores halve the instructions)
#pragma unroll
            for (int v = 0; v < 32; v += 16) {
              uint32_t w[8];
#pragma unroll
              for (int i = 0; i < 8; ++i)
                w[i] = pack_bf16(__uint_as_float(a[v + 2 * i]) * oscale,
                                 __uint_as_float(a[v + 2 * i + 1]) * oscale);
              asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(
                               dst + c + v),
                           "r"(w[0]), "r"(w[1]), "r"(w[2]), "r"(w[3]), "r"(w[4]), "r"(w[5]),
                           "r"(w[6]), "r"(w[7])
                           : "memory");
            }
          } else {
#pragma unroll
            for (int v = 0; v < 32; v += 8) {
              uint4 w;
              w.x = pack_bf16(__uint_as_float(a[v]) * oscale, __uint_as_float(a[v + 1]) * oscale);
              w.y = pack_bf16(__uint_as_float(a[v + 2]) * oscale, __uint_as_float(a[v + 3]) * oscale);
              w.z = pack_bf16(__uint_as_float(a[v + 4]) * oscale, __uint_as_float(a[v + 5]) * oscale);
              w.w = pack_bf16(__uint_as_float(a[v + 6]) * oscale, __uint_as_float(a[v + 7]) * oscale);
              *reinterpret_cast<uint4*>(dst + c + v) = w;
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(B.acc_free);
      n += nt;
      ++ub;
    }
  }
  // warps 2 and 3 have no role; every warp meets here before TMEM is freed
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

template <int D>
int launch_bwd_d(const BackwardArgs& a) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return PSA_ERR_CUDA;
  const int sms = sm_count(dev);
  if (sms <= 0) return PSA_ERR_CUDA;
  {
    const int warps = a.T * a.Hq;
    bwd_prep_kernel<<<(warps + 7) / 8, 256, 0, a.stream>>>(
        static_cast<const __nv_bfloat16*>(a.o), static_cast<const __nv_bfloat16*>(a.dout), a.lse,
        a.lse2_t, a.delta_t, a.T, (a.T + 3) / 4 * 4, a.Hq, D);
    if (cudaGetLastError() != cudaSuccess) return PSA_ERR_CUDA;
  }
  CUtensorMap q_blk, do_blk, k_t, v_t, k_blk, v_blk, q_t, do_t, tl, td;
  auto map3 = [&](CUtensorMap* m, const void* base, int H, int rows) {
    const uint64_t dims[3] = {uint64_t(D), uint64_t(H), uint64_t(a.T)};
    const uint64_t strides[2] = {uint64_t(D) * 2, uint64_t(H) * D * 2};
    const uint32_t box[3] = {64u, 1u, uint32_t(rows)};
    return encode_tmap(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, base, dims, strides, box,
                       CU_TENSOR_MAP_SWIZZLE_128B);
  };
  auto map2 = [&](CUtensorMap* m, const float* base) {
    const uint64_t dims[2] = {uint64_t(a.T), uint64_t(a.Hq)};
    const uint64_t strides[1] = {uint64_t((a.T + 3) / 4 * 4) * 4};
    const uint32_t box[2] = {uint32_t(BT + 4), 1u};
    return encode_tmap(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, base, dims, strides, box,
                       CU_TENSOR_MAP_SWIZZLE_NONE);
  };
  int rc = map3(&q_blk, a.q, a.Hq, BLK);
  if (rc == PSA_OK) rc = map3(&do_blk, a.dout, a.Hq, BLK);
  if (rc == PSA_OK) rc = map3(&k_t, a.k, a.Hkv, BT);
  if (rc == PSA_OK) rc = map3(&v_t, a.v, a.Hkv, BT);
  if (rc == PSA_OK) rc = map3(&k_blk, a.k, a.Hkv, BLK);
  if (rc == PSA_OK) rc = map3(&v_blk, a.v, a.Hkv, BLK);
  if (rc == PSA_OK) rc = map3(&q_t, a.q, a.Hq, BT);
  if (rc == PSA_OK) rc = map3(&do_t, a.dout, a.Hq, BT);
  if (rc == PSA_OK) rc = map2(&tl, a.lse2_t);
  if (rc == PSA_OK) rc = map2(&td, a.delta_t);
  if (rc != PSA_OK) return rc;

  BwdParams p;
  p.lse2_t = a.lse2_t;
  p.delta_t = a.delta_t;
  p.dq = static_cast<__nv_bfloat16*>(a.dq);
  p.dk = static_cast<__nv_bfloat16*>(a.dk);
  p.dv = static_cast<__nv_bfloat16*>(a.dv);
  p.T = a.T;
  p.Tp = (a.T + 3) / 4 * 4;
  p.Hq = a.Hq;
  p.Hkv = a.Hkv;
  p.G = a.Hq / a.Hkv;
  p.scale = a.scale;
  p.scale_log2 = a.scale * kLog2e;
  p.status = a.status;

  {
    p.sched = a.sched_q;
    p.sched_len = a.sched_q_len;
    auto kern = bwd_tc_kernel<D, kDq>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             int(TcCfg<D, kDq>::SMEM)) != cudaSuccess)
      return PSA_ERR_CUDA;
    // persistent over units; the unit count lives in the device schedule
    kern<<<sms, kThreads, TcCfg<D, kDq>::SMEM, a.stream>>>(q_blk, do_blk, k_t, v_t, tl, td, p);
    if (cudaGetLastError() != cudaSuccess) return PSA_ERR_CUDA;
  }
  {
    p.sched = a.sched_kv;
    p.sched_len = a.sched_kv_len;
    auto kern = bwd_tc_kernel<D, kDkdv>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             int(TcCfg<D, kDkdv>::SMEM)) != cudaSuccess)
      return PSA_ERR_CUDA;
    kern<<<sms, kThreads, TcCfg<D, kDkdv>::SMEM, a.stream>>>(k_blk, v_blk, q_t, do_t, tl, td, p);
    if (cudaGetLastError() != cudaSuccess) return PSA_ERR_CUDA;
  }
  return PSA_OK;
}

}  // namespace

int launch_backward(const BackwardArgs& a) {
  switch (a.D) {
    case 64:
      return launch_bwd_d<64>(a);
    case 128:
      return launch_bwd_d<128>(a);
    default:
      return PSA_ERR_UNSUPPORTED;
  }
}

}  // namespace psa
