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
//   prep     D and the log2-domain LSE per (row, head), stored head-major so a
//            tile of 64 rows is one contiguous 256-byte run.
//   dq pass  row-major over the forward's kind of schedule (blocks of 128
//            rows = two halves of 64, KV tiles of 64 keys): a CTA owns one
//            (row block, query head), streams the K and V tiles its rows see
//            and accumulates dQ in registers.
//   dkdv     key-major over the schedule of the transposed spec (blocks of
//            128 keys = two halves of 64, query tiles of 64 rows): a CTA owns
//            one (key block, KV head), holds its K and V block in shared
//            memory, streams the Q / dO tiles (and their LSE / D) of every
//            query head of the group that sees it, and accumulates dK, dV
//            in registers.
// Both passes: eight warps of 16 rows (or keys) each doing warp-level MMAs;
// lane 0 of warp 0 also feeds a TMA ring between its tiles (128-byte
// swizzle, no multicast).
// Every wait is bounded and reports PSA_ERR_TIMEOUT instead of hanging.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "psa_device.cuh"
#include "psa_internal.h"

namespace psa {
namespace {

constexpr int BR = 64;             // rows (or keys) per half
constexpr int BLK = 2 * BR;        // rows (or keys) per schedule block
constexpr int BT = 64;             // columns per streamed tile
constexpr int kConsumers = 8;      // 16-row warps: four per half
constexpr int kThreads = kConsumers * 32;
constexpr int kStages = 3;

__device__ __forceinline__ bool sched_ok(const int32_t* sch, int64_t len) {
  const int32_t n_items = __ldg(sch + 1), n_kv = __ldg(sch + 2), n_rect = __ldg(sch + 3);
  return __ldg(sch + 0) == 0x50534132 && __ldg(sch + 4) == BLK && __ldg(sch + 5) == BT &&
         n_items >= 0 && n_kv >= 0 && n_rect >= 0 &&
         8 + 4 * int64_t(n_items) + 8 * int64_t(n_kv) + 5 * int64_t(n_rect) <= len;
}

// Is (row, col) inside one of the copied rectangles [rb, rb + rc)?  Rows and
// columns are in the schedule's orientation (keys are rows in the transposed
// spec, whose causal rectangles carry causal == 2).
__device__ __forceinline__ bool in_rects(const int32_t* rects, int rb, int rc, int row, int col) {
  for (int i = 0; i < rc; ++i) {
    const int32_t* r = rects + 5 * (rb + i);
    const int q0 = __ldg(r), q1 = __ldg(r + 1), k0 = __ldg(r + 2), k1 = __ldg(r + 3);
    const int c = __ldg(r + 4);
    if (row < q0 || row >= q1 || col < k0 || col >= k1) continue;
    if (c == 1 && col - k0 > row - q0) continue;
    if (c == 2 && col - k0 < row - q0) continue;
    return true;
  }
  return false;
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
    delta_t[size_t(h) * Tp + t] = s;
    lse2_t[size_t(h) * Tp + t] = lse[size_t(t) * Hq + h] * kLog2e;
  }
}

// ---------------------------------------------------------------- shared pieces

struct BwdParams {
  const int32_t* sched;
  int64_t sched_len;
  const __nv_bfloat16* q;     // [T, Hq, D]
  const __nv_bfloat16* k;     // [T, Hkv, D]
  const __nv_bfloat16* v;
  const __nv_bfloat16* dout;  // [T, Hq, D]
  const float* lse2_t;        // [Hq, Tp]
  const float* delta_t;       // [Hq, Tp]
  __nv_bfloat16* dq;          // [T, Hq, D]
  __nv_bfloat16* dk;          // [T, Hkv, D]
  __nv_bfloat16* dv;
  int32_t T, Tp, Hq, Hkv, G;  // Tp: T rounded up to a multiple of 4 (row stride of the stats)
  float scale, scale_log2;
  int32_t* status;
};

// A fragments of 16 rows x D of a [T, H, D] bf16 tensor (rows past T are 0).
template <int D>
__device__ __forceinline__ void load_rows_a(const __nv_bfloat16* base, int H, int head, int r0,
                                            int T, uint32_t (&a)[D / 16][4]) {
  const int lane = threadIdx.x & 31, g = lane >> 2, c = lane & 3;
  const int ra = r0 + g, rb = r0 + g + 8;
  const __nv_bfloat16* pa = base + (size_t(ra) * H + head) * D;
  const __nv_bfloat16* pb = base + (size_t(rb) * H + head) * D;
#pragma unroll
  for (int ks = 0; ks < D / 16; ++ks) {
    const int col = ks * 16 + 2 * c;
    a[ks][0] = ra < T ? __ldg(reinterpret_cast<const uint32_t*>(pa + col)) : 0u;
    a[ks][1] = rb < T ? __ldg(reinterpret_cast<const uint32_t*>(pb + col)) : 0u;
    a[ks][2] = ra < T ? __ldg(reinterpret_cast<const uint32_t*>(pa + col + 8)) : 0u;
    a[ks][3] = rb < T ? __ldg(reinterpret_cast<const uint32_t*>(pb + col + 8)) : 0u;
  }
}

// acc[4 n-tiles] = A(16 x D, registers) . X^T for 32 columns of a swizzled
// tile X (rows = columns of the product, D contiguous): X rows col0 .. col0+31.
template <int D>
__device__ __forceinline__ void gemm_a_xt(const uint32_t (&a)[D / 16][4], uint32_t xbase,
                                          uint32_t part_stride, int col0, float (&acc)[4][4]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int nt = 0; nt < 4; ++nt) {
    acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
    const uint32_t row = col0 + nt * 8 + (lane & 7);
#pragma unroll
    for (int ks = 0; ks < D / 16; ks += 2) {
      const uint32_t chunk = ks * 2 + (lane >> 3);
      const uint32_t addr = xbase + (chunk >> 3) * part_stride + sw128(row, chunk & 7);
      uint32_t b0, b1, b2, b3;
      ldmatrix_x4(addr, b0, b1, b2, b3);
      mma_bf16_16816(acc[nt], a[ks], b0, b1);
      mma_bf16_16816(acc[nt], a[ks + 1], b2, b3);
    }
  }
}

// acc[4 n-tiles] = A(16 rows of a swizzled tile Y: rows y0 .. y0+15) . X^T
// for 32 columns of a swizzled tile X (rows col0 .. col0+31).
template <int D>
__device__ __forceinline__ void gemm_y_xt(uint32_t ybase, uint32_t ypart, int y0, uint32_t xbase,
                                          uint32_t xpart, int col0, float (&acc)[4][4]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int nt = 0; nt < 4; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
#pragma unroll
  for (int ks = 0; ks < D / 16; ++ks) {
    uint32_t a[4];
    {
      const uint32_t row = y0 + (lane & 7) + ((lane >> 3) & 1) * 8;
      const uint32_t chunk = ks * 2 + (lane >> 4);
      ldmatrix_x4(ybase + (chunk >> 3) * ypart + sw128(row, chunk & 7), a[0], a[1], a[2], a[3]);
    }
#pragma unroll
    for (int np = 0; np < 2; ++np) {
      // two n-tiles per ldmatrix_x4: rows col0 + 16 np + (0..15), one k-step
      const uint32_t row = col0 + np * 16 + (lane & 7) + ((lane >> 4) << 3);
      const uint32_t chunk = ks * 2 + ((lane >> 3) & 1);
      uint32_t b0, b1, b2, b3;
      ldmatrix_x4(xbase + (chunk >> 3) * xpart + sw128(row, chunk & 7), b0, b1, b2, b3);
      mma_bf16_16816(acc[2 * np], a, b0, b1);
      mma_bf16_16816(acc[2 * np + 1], a, b2, b3);
    }
  }
}

// acc[D/8 n-tiles] += A(16 x 32: two k-steps given as packed fragments) .
// X(32 rows x D) of a swizzled tile X (rows x0 .. x0+31, D contiguous).
template <int D>
__device__ __forceinline__ void gemm_p_x(const uint32_t (&pa)[2][4], uint32_t xbase,
                                         uint32_t part_stride, int x0, float (&acc)[D / 8][4]) {
  const int lane = threadIdx.x & 31;
  const int mi = lane >> 3;
#pragma unroll
  for (int kk = 0; kk < 2; ++kk) {
    const uint32_t row = x0 + kk * 16 + (mi & 1) * 8 + (lane & 7);
#pragma unroll
    for (int dt = 0; dt < D / 8; dt += 2) {
      const uint32_t chunk = dt + (mi >> 1);
      const uint32_t addr = xbase + (chunk >> 3) * part_stride + sw128(row, chunk & 7);
      uint32_t b0, b1, b2, b3;
      ldmatrix_x4_trans(addr, b0, b1, b2, b3);
      mma_bf16_16816(acc[dt], pa[kk], b0, b1);
      mma_bf16_16816(acc[dt + 1], pa[kk], b2, b3);
    }
  }
}

// Packs 4 n-tiles of fp32 C fragments (16 x 32) into two bf16 A fragments.
__device__ __forceinline__ void pack_a(const float (&c)[4][4], uint32_t (&pa)[2][4]) {
#pragma unroll
  for (int kk = 0; kk < 2; ++kk) {
    pa[kk][0] = pack_bf16(c[2 * kk][0], c[2 * kk][1]);
    pa[kk][1] = pack_bf16(c[2 * kk][2], c[2 * kk][3]);
    pa[kk][2] = pack_bf16(c[2 * kk + 1][0], c[2 * kk + 1][1]);
    pa[kk][3] = pack_bf16(c[2 * kk + 1][2], c[2 * kk + 1][3]);
  }
}

// Stores a 16 x D fp32 accumulator (times s) as bf16 rows of [T, H, D].
template <int D>
__device__ __forceinline__ void store_rows(__nv_bfloat16* base, int H, int head, int r0, int rend,
                                           const float (&acc)[D / 8][4], float s) {
  const int lane = threadIdx.x & 31, g = lane >> 2, c = lane & 3;
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const int r = r0 + g + 8 * i;
    if (r >= rend) continue;
    __nv_bfloat16* p = base + (size_t(r) * H + head) * D;
#pragma unroll
    for (int dt = 0; dt < D / 8; ++dt)
      *reinterpret_cast<uint32_t*>(p + dt * 8 + 2 * c) =
          pack_bf16(acc[dt][2 * i] * s, acc[dt][2 * i + 1] * s);
  }
}

// Unit of this CTA in round r.  Units are listed longest first; odd rounds
// hand them out in reverse CTA order, so the CTAs that got the longest units
// of one round get the shortest of the next.
__device__ __forceinline__ int snake_unit(int r) {
  const int lane_in_round = (r & 1) ? int(gridDim.x) - 1 - int(blockIdx.x) : int(blockIdx.x);
  return r * int(gridDim.x) + lane_in_round;
}

// ---------------------------------------------------------------- dq pass

// The ring is fed by lane 0 of warp 0 between its own tiles (no separate
// producer warp: eight warps keep two per sub-partition, so each thread may
// hold up to 255 registers).  Load n goes to slot n % kStages once every
// warp has released the tile that used the slot before.

template <int D>
struct DqCfg {
  static constexpr uint32_t TILE = BT * D * 2;          // one K (or V) tile
  static constexpr uint32_t STAGE = 2 * TILE;
  static constexpr uint32_t OFF_BAR = kStages * STAGE;
  static constexpr uint32_t SMEM = 1024 + OFF_BAR + 2 * kStages * 8 + 16;
};

// Walks the (round, KV tile) sequence of one CTA for the dq pass.
struct DqCursor {
  int r, j;
};

template <int D>
__device__ __forceinline__ bool dq_issue(const BwdParams& p, const int4* items,
                                         const int32_t* kvs, int units, DqCursor& cur,
                                         uint32_t n, uint8_t* smem, uint64_t* full,
                                         uint64_t* empty, const CUtensorMap* tk,
                                         const CUtensorMap* tv, int* abort_flag) {
  using C = DqCfg<D>;
  int u = snake_unit(cur.r);
  while (u < units) {
    const int4 it = __ldg(items + u / p.Hq);
    if (cur.j < it.w) break;
    u = snake_unit(++cur.r);
    cur.j = 0;
  }
  if (u >= units) return true;  // nothing left to load
  const int4 it = __ldg(items + u / p.Hq);
  const int kvh = (u % p.Hq) / p.G;
  const int k0 = __ldg(kvs + 8 * (it.z + cur.j));
  const int s = n % kStages;
  if (!mbar_wait(empty + s, ((n / kStages) & 1) ^ 1, abort_flag, p.status)) return false;
  mbar_arrive_expect_tx(full + s, C::STAGE);
  uint8_t* dst = smem + s * C::STAGE;
#pragma unroll
  for (int part = 0; part < D / 64; ++part) {
    tma_load_3d(dst + part * BT * 128, tk, full + s, part * 64, kvh, k0);
    tma_load_3d(dst + C::TILE + part * BT * 128, tv, full + s, part * 64, kvh, k0);
  }
  ++cur.j;
  return true;
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    bwd_dq_kernel(const __grid_constant__ CUtensorMap tmap_k,
                  const __grid_constant__ CUtensorMap tmap_v, BwdParams p) {
  using C = DqCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  __shared__ int abort_flag;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int32_t* sch = p.sched;
  if (!sched_ok(sch, p.sched_len)) {
    if (threadIdx.x == 0) report_status(p.status, PSA_ERR_INVALID_ARG);
    return;
  }
  const int32_t n_items = __ldg(sch + 1), n_kv = __ldg(sch + 2);
  const int4* items = reinterpret_cast<const int4*>(sch + 8);
  const int32_t* kvs = sch + 8 + 4 * n_items;
  const int32_t* rects = kvs + 8 * n_kv;
  const int units = n_items * p.Hq;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* empty = full + kStages;
  if (threadIdx.x == 0) {
    abort_flag = 0;
    for (int i = 0; i < kStages; ++i) {
      mbar_init(full + i, 1);
      mbar_init(empty + i, kConsumers);
    }
    fence_barrier_init();
  }
  __syncthreads();
  const bool producer = warp == 0 && lane == 0;
  DqCursor cur{0, 0};
  uint32_t issued = 0;
  bool ok = true;
  if (producer) {
    tma_prefetch_desc(&tmap_k);
    tma_prefetch_desc(&tmap_v);
    for (int i = 0; i < kStages && ok; ++i) {
      const DqCursor before = cur;
      ok = dq_issue<D>(p, items, kvs, units, cur, issued, smem, full, empty, &tmap_k, &tmap_v,
                       &abort_flag);
      if (ok && (cur.r != before.r || cur.j != before.j)) ++issued;
    }
  }

  const int x = warp >> 2;  // half of the row block
  const int g = lane >> 2, c = lane & 3;
  uint32_t n = 0;
  for (int rnd = 0; ok; ++rnd) {
    const int u = snake_unit(rnd);
    if (u >= units) break;
    const int4 it = __ldg(items + u / p.Hq);
    const int h = u % p.Hq;
    const int r0 = it.x + x * BR + (warp & 3) * 16;  // this warp's 16 rows
    const int rend = it.x + it.y;                    // past the block's last row
    uint32_t qa[D / 16][4], da[D / 16][4];
    load_rows_a<D>(p.q, p.Hq, h, r0, rend, qa);
    load_rows_a<D>(p.dout, p.Hq, h, r0, rend, da);
    float lse2[2], dl[2];
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const int r = r0 + g + 8 * i;
      lse2[i] = r < rend ? __ldg(p.lse2_t + size_t(h) * p.Tp + r) : 0.f;
      dl[i] = r < rend ? __ldg(p.delta_t + size_t(h) * p.Tp + r) : 0.f;
    }
    float acc[D / 8][4];
#pragma unroll
    for (int i = 0; i < D / 8; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
    for (int j = 0; j < it.w; ++j, ++n) {
      const int s = n % kStages;
      if (!mbar_wait(full + s, (n / kStages) & 1, &abort_flag, p.status)) {
        ok = false;
        break;
      }
      const int32_t* e = kvs + 8 * (it.z + j);
      const int k0 = __ldg(e), klen = __ldg(e + 1), flags = __ldg(e + 6);
      const int rb = __ldg(e + 2 + 2 * x), rc = __ldg(e + 3 + 2 * x);
      if ((flags & (1 << x)) && r0 < rend) {
        const uint32_t kb = smem_u32(smem + s * C::STAGE), vb = kb + C::TILE;
        const bool full_vis = (flags & (4 << x)) != 0;
#pragma unroll
        for (int kh = 0; kh < 2; ++kh) {
          float sc[4][4], dp[4][4];
          gemm_a_xt<D>(qa, kb, BT * 128, kh * 32, sc);
          gemm_a_xt<D>(da, vb, BT * 128, kh * 32, dp);
#pragma unroll
          for (int nt = 0; nt < 4; ++nt)
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const int col = kh * 32 + nt * 8 + 2 * c + (q & 1);
              const int row = r0 + g + 8 * (q >> 1);
              bool vis = col < klen && row < rend;
              if (vis && !full_vis) vis = in_rects(rects, rb, rc, row, k0 + col);
              const float pr = vis ? fast_exp2(sc[nt][q] * p.scale_log2 - lse2[q >> 1]) : 0.f;
              sc[nt][q] = pr * (dp[nt][q] - dl[q >> 1]);  // dS
            }
          uint32_t pa[2][4];
          pack_a(sc, pa);
          gemm_p_x<D>(pa, kb, BT * 128, kh * 32, acc);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(empty + s);
      if (producer) {
        // refill the slot just released once every warp has released it
        const DqCursor before = cur;
        ok = dq_issue<D>(p, items, kvs, units, cur, issued, smem, full, empty, &tmap_k, &tmap_v,
                         &abort_flag);
        if (ok && (cur.r != before.r || cur.j != before.j)) ++issued;
      }
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0 && ok;
    }
    if (!ok) break;
    store_rows<D>(p.dq, p.Hq, h, r0, rend, acc, p.scale);
  }
  if (!ok && producer) {
    // let copies in flight land before the CTA exits
    const uint64_t t0 = globaltimer();
    while (globaltimer() - t0 < 1000000ull) {
    }
  }
}

// ---------------------------------------------------------------- dk / dv pass

template <int D>
struct KvCfg {
  static constexpr uint32_t BLOCK = BLK * D * 2;        // the unit's K (or V) block
  static constexpr uint32_t TILE = BT * D * 2;          // one Q (or dO) tile
  // + LSE and D of the tile: BT + 4 floats each (the copy starts at the
  // tile's first row rounded down to a multiple of 4, keeping the TMA x
  // coordinate 16-byte aligned).  Each copy lands on a 128-byte aligned
  // slot of STAT_SLOT bytes, and the stage is padded to stay 1 KB aligned.
  static constexpr uint32_t STAT = (BT + 4) * 4;
  static constexpr uint32_t STAT_SLOT = 512;
  static constexpr uint32_t STAGE = 2 * TILE + 2 * STAT_SLOT;
  static constexpr uint32_t OFF_KV = 0;
  static constexpr uint32_t OFF_RING = 2 * BLOCK;
  static constexpr uint32_t OFF_BAR = OFF_RING + kStages * STAGE;
  static constexpr uint32_t SMEM = 1024 + OFF_BAR + (2 * kStages + 2) * 8 + 16;
};

// Walks the (round, query head, query tile) sequence of one CTA.
struct KvCursor {
  int r, gq, j;
};

struct KvMaps {
  const CUtensorMap *q, *dout, *lse, *delta;
};

template <int D>
__device__ __forceinline__ bool kv_issue(const BwdParams& p, const int4* items,
                                         const int32_t* qts, int units, KvCursor& cur,
                                         uint32_t n, uint8_t* smem, uint64_t* full,
                                         uint64_t* empty, const KvMaps& m, int* abort_flag) {
  using C = KvCfg<D>;
  int u = snake_unit(cur.r);
  while (u < units) {
    const int4 it = __ldg(items + u / p.Hkv);
    if (cur.j < it.w) break;
    cur.j = 0;
    if (++cur.gq == p.G) {
      cur.gq = 0;
      u = snake_unit(++cur.r);
    }
  }
  if (u >= units) return true;
  const int4 it = __ldg(items + u / p.Hkv);
  const int h = (u % p.Hkv) * p.G + cur.gq;
  const int q0 = __ldg(qts + 8 * (it.z + cur.j));
  const int s = n % kStages;
  if (!mbar_wait(empty + s, ((n / kStages) & 1) ^ 1, abort_flag, p.status)) return false;
  mbar_arrive_expect_tx(full + s, 2 * C::TILE + 2 * C::STAT);
  uint8_t* dst = smem + C::OFF_RING + s * C::STAGE;
#pragma unroll
  for (int part = 0; part < D / 64; ++part) {
    tma_load_3d(dst + part * BT * 128, m.q, full + s, part * 64, h, q0);
    tma_load_3d(dst + C::TILE + part * BT * 128, m.dout, full + s, part * 64, h, q0);
  }
  tma_load_2d(dst + 2 * C::TILE, m.lse, full + s, q0 & ~3, h);
  tma_load_2d(dst + 2 * C::TILE + C::STAT_SLOT, m.delta, full + s, q0 & ~3, h);
  ++cur.j;
  return true;
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tmap_k,
                    const __grid_constant__ CUtensorMap tmap_v,
                    const __grid_constant__ CUtensorMap tmap_q,
                    const __grid_constant__ CUtensorMap tmap_do,
                    const __grid_constant__ CUtensorMap tmap_lse,
                    const __grid_constant__ CUtensorMap tmap_delta, BwdParams p) {
  using C = KvCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  __shared__ int abort_flag;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int32_t* sch = p.sched;
  if (!sched_ok(sch, p.sched_len)) {
    if (threadIdx.x == 0) report_status(p.status, PSA_ERR_INVALID_ARG);
    return;
  }
  const int32_t n_items = __ldg(sch + 1), n_kv = __ldg(sch + 2);
  const int4* items = reinterpret_cast<const int4*>(sch + 8);
  const int32_t* qts = sch + 8 + 4 * n_items;  // query tiles of each key block
  const int32_t* rects = qts + 8 * n_kv;
  const int units = n_items * p.Hkv;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* empty = full + kStages;
  uint64_t* kv_full = empty + kStages;
  uint64_t* kv_empty = kv_full + 1;
  if (threadIdx.x == 0) {
    abort_flag = 0;
    for (int i = 0; i < kStages; ++i) {
      mbar_init(full + i, 1);
      mbar_init(empty + i, kConsumers);
    }
    mbar_init(kv_full, 1);
    mbar_init(kv_empty, kConsumers);
    fence_barrier_init();
  }
  __syncthreads();
  const bool producer = warp == 0 && lane == 0;
  const KvMaps maps{&tmap_q, &tmap_do, &tmap_lse, &tmap_delta};
  KvCursor cur{0, 0, 0};
  uint32_t issued = 0;
  bool ok = true;
  // the K and V block of unit u (the previous unit must have released it)
  auto load_block = [&](int u, uint32_t uc) -> bool {
    if (u >= units) return true;
    if (!mbar_wait(kv_empty, (uc & 1) ^ 1, &abort_flag, p.status)) return false;
    const int4 it = __ldg(items + u / p.Hkv);
    const int kvh = u % p.Hkv;
    mbar_arrive_expect_tx(kv_full, 2 * C::BLOCK);
#pragma unroll
    for (int part = 0; part < D / 64; ++part) {
      tma_load_3d(smem + C::OFF_KV + part * BLK * 128, &tmap_k, kv_full, part * 64, kvh, it.x);
      tma_load_3d(smem + C::OFF_KV + C::BLOCK + part * BLK * 128, &tmap_v, kv_full, part * 64,
                  kvh, it.x);
    }
    return true;
  };
  auto issue = [&]() -> bool {
    const KvCursor before = cur;
    const bool r = kv_issue<D>(p, items, qts, units, cur, issued, smem, full, empty, maps,
                               &abort_flag);
    if (r && (cur.r != before.r || cur.gq != before.gq || cur.j != before.j)) ++issued;
    return r;
  };
  if (producer) {
    tma_prefetch_desc(&tmap_q);
    tma_prefetch_desc(&tmap_do);
    ok = load_block(snake_unit(0), 0);
    for (int i = 0; i < kStages && ok; ++i) ok = issue();
  }
  ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;

  const int x = warp >> 2;  // half of the key block
  const int g = lane >> 2, c = lane & 3;
  const uint32_t kblk = smem_u32(smem + C::OFF_KV), vblk = kblk + C::BLOCK;
  uint32_t n = 0, uc = 0;
  for (int rnd = 0; ok; ++rnd, ++uc) {
    const int u = snake_unit(rnd);
    if (u >= units) break;
    const int4 it = __ldg(items + u / p.Hkv);
    const int kvh = u % p.Hkv;
    const int kl0 = x * BR + (warp & 3) * 16;  // this warp's 16 keys within the block
    const int key0 = it.x + kl0;
    const int kend = it.x + it.y;
    float dka[D / 8][4], dva[D / 8][4];
#pragma unroll
    for (int i = 0; i < D / 8; ++i) {
      dka[i][0] = dka[i][1] = dka[i][2] = dka[i][3] = 0.f;
      dva[i][0] = dva[i][1] = dva[i][2] = dva[i][3] = 0.f;
    }
    ok = mbar_wait(kv_full, uc & 1, &abort_flag, p.status);
    for (int gq = 0; gq < p.G && ok; ++gq) {
      for (int j = 0; j < it.w; ++j, ++n) {
        const int s = n % kStages;
        if (!mbar_wait(full + s, (n / kStages) & 1, &abort_flag, p.status)) {
          ok = false;
          break;
        }
        const int32_t* e = qts + 8 * (it.z + j);
        const int q0 = __ldg(e), qlen = __ldg(e + 1), flags = __ldg(e + 6);
        const int rb = __ldg(e + 2 + 2 * x), rc = __ldg(e + 3 + 2 * x);
        if ((flags & (1 << x)) && key0 < kend) {
          const uint32_t qb = smem_u32(smem + C::OFF_RING + s * C::STAGE), db = qb + C::TILE;
          const float* lse2 = reinterpret_cast<const float*>(smem + C::OFF_RING + s * C::STAGE +
                                                             2 * C::TILE) + (q0 & 3);
          const float* dlt = lse2 + C::STAT_SLOT / 4;
          const bool full_vis = (flags & (4 << x)) != 0;
#pragma unroll
          for (int rh = 0; rh < 2; ++rh) {
            float st[4][4], dpt[4][4];
            gemm_y_xt<D>(kblk, BLK * 128, kl0, qb, BT * 128, rh * 32, st);
            gemm_y_xt<D>(vblk, BLK * 128, kl0, db, BT * 128, rh * 32, dpt);
            float pt[4][4];
#pragma unroll
            for (int nt = 0; nt < 4; ++nt)
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                const int col = rh * 32 + nt * 8 + 2 * c + (q & 1);  // query within the tile
                const int key = key0 + g + 8 * (q >> 1);
                bool vis = col < qlen && key < kend;
                if (vis && !full_vis) vis = in_rects(rects, rb, rc, key, q0 + col);
                const float pr = vis ? fast_exp2(st[nt][q] * p.scale_log2 - lse2[col]) : 0.f;
                pt[nt][q] = pr;
                st[nt][q] = pr * (dpt[nt][q] - dlt[col]);  // dS^T
              }
            uint32_t pa[2][4];
            pack_a(pt, pa);
            gemm_p_x<D>(pa, db, BT * 128, rh * 32, dva);
            pack_a(st, pa);
            gemm_p_x<D>(pa, qb, BT * 128, rh * 32, dka);
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(empty + s);
        if (producer) ok = issue();
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0 && ok;
      }
    }
    if (!ok) break;
    __syncwarp();
    if (lane == 0) mbar_arrive(kv_empty);
    store_rows<D>(p.dk, p.Hkv, kvh, key0, kend, dka, p.scale);
    store_rows<D>(p.dv, p.Hkv, kvh, key0, kend, dva, 1.f);
    if (producer) ok = load_block(snake_unit(rnd + 1), uc + 1);
    ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0 && ok;
  }
  if (!ok && producer) {
    const uint64_t t0 = globaltimer();
    while (globaltimer() - t0 < 1000000ull) {
    }
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
  CUtensorMap tk, tv, tq, tdo, tk_blk, tv_blk, tl, td;
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
  int rc = map3(&tk, a.k, a.Hkv, BT);
  if (rc == PSA_OK) rc = map3(&tv, a.v, a.Hkv, BT);
  if (rc == PSA_OK) rc = map3(&tk_blk, a.k, a.Hkv, BLK);
  if (rc == PSA_OK) rc = map3(&tv_blk, a.v, a.Hkv, BLK);
  if (rc == PSA_OK) rc = map3(&tq, a.q, a.Hq, BT);
  if (rc == PSA_OK) rc = map3(&tdo, a.dout, a.Hq, BT);
  if (rc == PSA_OK) rc = map2(&tl, a.lse2_t);
  if (rc == PSA_OK) rc = map2(&td, a.delta_t);
  if (rc != PSA_OK) return rc;

  BwdParams p;
  p.q = static_cast<const __nv_bfloat16*>(a.q);
  p.k = static_cast<const __nv_bfloat16*>(a.k);
  p.v = static_cast<const __nv_bfloat16*>(a.v);
  p.dout = static_cast<const __nv_bfloat16*>(a.dout);
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
    auto kern = bwd_dq_kernel<D>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             int(DqCfg<D>::SMEM)) != cudaSuccess)
      return PSA_ERR_CUDA;
    // persistent over units; the unit count lives in the device schedule
    kern<<<sms, kThreads, DqCfg<D>::SMEM, a.stream>>>(tk, tv, p);
    {
      if (cudaGetLastError() != cudaSuccess) return PSA_ERR_CUDA;
    }
  }
  {
    p.sched = a.sched_kv;
    p.sched_len = a.sched_kv_len;
    auto kern = bwd_dkdv_kernel<D>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             int(KvCfg<D>::SMEM)) != cudaSuccess)
      return PSA_ERR_CUDA;
    kern<<<sms, kThreads, KvCfg<D>::SMEM, a.stream>>>(tk_blk, tv_blk, tq, tdo, tl, td, p);
    {
      if (cudaGetLastError() != cudaSuccess) return PSA_ERR_CUDA;
    }
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
