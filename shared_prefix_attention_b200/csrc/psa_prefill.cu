// Prefill over the flat, deduplicated packed layout: one forward pass of
// softmax attention in which the prefix K/V is stored once and every suffix
// sees it through the tile schedule ("KV-0 redundancy prefix sharing
// attention mask design", PrefixSharing PR #50: design summary -- flat
// dedup layout, block-causal rectangle spec instead of a dense mask, one
// forward that is mathematically equivalent to running each [prefix; s_i]).
//
// sm_100a design.  One CTA per SM, persistent over units (Q block of 256
// rows, query head).  The host schedule lists the blocks longest-first and
// the producer hands units out through a global counter, so long suffix
// blocks start first and short prefix blocks fill the tail (per KV head when
// each KV head has units for two waves, so the CTAs in flight share its K/V
// in L2).  A block is two
// 128-row halves A and B that share every K/V tile load:
//   warps 0, 2   TMA producers (Q and K; V): the Q block, then the K and V
//                tiles of the block's visible KV tiles only (invisible tiles
//                are never touched), 128-byte swizzle, no multicast.
//   warp 1       tcgen05 issuer (one thread).  Per half X: S_X = Q_X K^T
//                into TMEM, then O_X += P_X V with P_X read from TMEM where
//                the softmax left it (aliasing S_X).  Issue order
//                PV_A(j), QK_A(j+1), PV_B(j), QK_B(j+1): while one half's
//                softmax runs, the tensor pipe works on the other half.
//   warps 4..7   softmax of half A, warps 8..11 softmax of half B: one query
//                row per thread (= TMEM lane), the whole 128-column S row
//                read in one TMEM load (setmaxnreg moves registers from the
//                producer/MMA warpgroup to the softmax warpgroups).  Masks
//                partial tiles from the
//                copied rectangles, keeps the running max in the log2 domain
//                with lazy rescaling (O is rescaled in TMEM only when the
//                max grows by more than 2^8), writes P as bf16 over its S
//                columns, and runs the epilogue (O / l, LSE) from TMEM.
// Every wait is bounded: a stuck pipeline reports PSA_ERR_TIMEOUT through
// the status word, the CTA unwinds and frees its TMEM.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "psa_debug.cuh"
#include "psa_device.cuh"
#include "psa_internal.h"
#include "psa_tmem_wide.cuh"

namespace psa {
namespace {

constexpr int BM = 128;            // query rows per half
constexpr int BLOCK_M = 2 * BM;    // query rows per schedule block
constexpr int BN = 128;            // keys per tile
constexpr int kThreads = 384;      // 12 warps
constexpr float kRescaleLog2 = 8.f;
constexpr uint32_t kTmemCols = 512;  // per half: S at X*256, O at X*256 + 128
constexpr int kSchedSlots = 4;       // units the producer may fetch ahead
constexpr int kSchedReaders = 10;    // V producer, MMA thread, eight softmax warps

template <int D>
struct Cfg {
  static constexpr int NPART = D / 64;  // 128-byte swizzle atoms across d
  static constexpr uint32_t Q_BYTES = BM * D * 2;   // one half
  static constexpr uint32_t KV_BYTES = BN * D * 2;
  // K is needed a whole tile before V (QK_{j+1} is issued right after
  // PV_j), so its ring is one slot deeper.
  static constexpr int NSK = D == 128 ? 3 : 4;
  static constexpr int NSV = D == 128 ? 2 : 4;
  static constexpr uint32_t OFF_Q = 0;
  static constexpr uint32_t OFF_K = OFF_Q + 2 * Q_BYTES;
  static constexpr uint32_t OFF_V = OFF_K + NSK * KV_BYTES;
  static constexpr uint32_t OFF_BAR = OFF_V + NSV * KV_BYTES;
  static constexpr uint32_t NBAR = 2 + 2 * NSK + 2 * NSV + 8 + 2 * kSchedSlots;
  static constexpr uint32_t SMEM = 1024 + OFF_BAR + NBAR * 8 + 16;
};

struct Params {
  const int32_t* sched;
  int64_t sched_len;
  void* o;
  float* lse;
  int32_t T, Hq, Hkv, G;
  float scale_log2;
  int32_t* status;
  int32_t* counter;  // next unit to hand out (zeroed before every launch)
};

struct Bars {
  uint64_t *q_full, *q_empty, *k_full, *k_empty, *v_full, *v_empty;
  uint64_t *s_full, *p_full, *pv_done, *o_free;  // [2] each, one per half
  uint64_t *sch_full, *sch_empty;
};

__device__ __forceinline__ void set_bits(uint32_t (&m)[4], int a, int b) {
#pragma unroll
  for (int w = 0; w < 4; ++w) {
    const int lo = max(a, 32 * w), hi = min(b, 32 * w + 32);
    if (lo < hi) {
      const uint32_t n = uint32_t(hi - lo);
      const uint32_t bits = n == 32 ? 0xffffffffu : ((1u << n) - 1u);
      m[w] |= bits << (lo - 32 * w);
    }
  }
}

// Register split between warpgroups: the launch gives every thread 168
// registers (384 x 168 = 64512); warpgroup 0 (the two producers, the MMA
// issuer, one idle warp) drops to 104, the least that keeps the MMA issuer
// free of spills, so the two softmax warpgroups can hold a whole 128-column
// S row in registers (2 x 128 x 200 + 128 x 104 = 64512).
__device__ __forceinline__ void regs_dec() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 104;" ::: "memory");
}
__device__ __forceinline__ void regs_inc() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 200;" ::: "memory");
}

// Unit u -> (schedule block, query head).  When every KV head has at least
// two waves of units, the order is KV-head-major (blocks longest-first within
// a KV head, its G query heads adjacent), so the CTAs in flight all stream
// the same KV head's K/V tiles and L2 serves the re-reads; otherwise it is
// block-major with the query heads adjacent.
__device__ __forceinline__ void unit_block_head(int u, int n_items, int Hq, int G, int& item,
                                                int& h) {
  if (int64_t(n_items) * G >= 2 * int64_t(gridDim.x)) {
    const int per_kv = n_items * G;
    const int kvh = u / per_kv, rem = u - kvh * per_kv;
    item = rem / G;
    h = kvh * G + (rem - item * G);
  } else {
    item = u / Hq;
    h = u - item * Hq;
  }
}

// Header check shared by both prefill kernels (uniform across threads).
__device__ __forceinline__ bool schedule_ok(const int32_t* sch, int64_t len) {
  const int32_t n_items = __ldg(sch + 1), n_kv = __ldg(sch + 2), n_rect = __ldg(sch + 3);
  return __ldg(sch + 0) == 0x50534132 && __ldg(sch + 4) == BLOCK_M && __ldg(sch + 5) == BN &&
         n_items >= 0 && n_kv >= 0 && n_rect >= 0 &&
         8 + 4 * int64_t(n_items) + 8 * int64_t(n_kv) + 5 * int64_t(n_rect) <= len;
}

// One schedule KV entry as seen by half x (its rectangle range selected
// without indexing, so the entry stays in registers).
struct KvEntry {
  int k0, klen, rb, rc, flags;
};

__device__ __forceinline__ KvEntry load_kv(const int32_t* kvs, int idx, int x) {
  const int4 a = __ldg(reinterpret_cast<const int4*>(kvs) + 2 * idx);
  const int4 b = __ldg(reinterpret_cast<const int4*>(kvs) + 2 * idx + 1);
  KvEntry e;
  e.k0 = a.x;
  e.klen = a.y;
  e.rb = x ? b.x : a.z;
  e.rc = x ? b.y : a.w;
  e.flags = b.z;
  return e;
}

// A schedule block as the kernels use it: its rows inside [0, T) and its
// tile entries inside the schedule's tile list (checked in the debug build).
__device__ __forceinline__ bool item_in_bounds(const int4& it, int32_t n_kv, int32_t T) {
  return it.x >= 0 && it.y >= 0 && it.y <= BLOCK_M && int64_t(it.x) + it.y <= T && it.z >= 0 &&
         it.w >= 0 && int64_t(it.z) + it.w <= n_kv;
}

// Visible keys of row q inside KV tile e for half x, as a 128-bit mask.
__device__ __forceinline__ void row_visibility(const KvEntry& e, int x, int q,
                                               const int32_t* rects, int32_t n_rect,
                                               int32_t* status, uint32_t (&vis)[4]) {
  vis[0] = vis[1] = vis[2] = vis[3] = 0u;
  if (e.flags & (4 << x)) {
    set_bits(vis, 0, e.klen);
    return;
  }
  if (!psa_in_bounds(e.rb >= 0 && e.rc >= 0 && int64_t(e.rb) + e.rc <= n_rect, status)) return;
  for (int ri = 0; ri < e.rc; ++ri) {
    const int32_t* rc = rects + 5 * (e.rb + ri);
    const int rq0 = __ldg(rc), rq1 = __ldg(rc + 1), rk0 = __ldg(rc + 2), rk1 = __ldg(rc + 3),
              causal = __ldg(rc + 4);
    if (q < rq0 || q >= rq1) continue;
    int hi = causal ? min(rk1, rk0 + (q - rq0) + 1) : rk1;
    hi = min(hi, e.k0 + e.klen);
    const int lo = max(rk0, e.k0);
    if (lo < hi) set_bits(vis, lo - e.k0, hi - e.k0);
  }
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    prefill_kernel(const __grid_constant__ CUtensorMap tmap_q,
                   const __grid_constant__ CUtensorMap tmap_k,
                   const __grid_constant__ CUtensorMap tmap_v, Params p) {
  using C = Cfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  __shared__ uint32_t tmem_base_slot;
  __shared__ int abort_flag;
  __shared__ int sch_unit[kSchedSlots];
  __shared__ int4 sch_item[kSchedSlots];  // the unit's schedule block, fetched once

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  const int32_t* sch = p.sched;
  if (!schedule_ok(sch, p.sched_len)) {
    if (threadIdx.x == 0) report_status(p.status, PSA_ERR_INVALID_ARG);
    return;
  }
  const int32_t n_items = __ldg(sch + 1), n_kv = __ldg(sch + 2), n_rect = __ldg(sch + 3);
  const int4* items = reinterpret_cast<const int4*>(sch + 8);
  const int32_t* kvs = sch + 8 + 4 * n_items;
  const int32_t* rects = kvs + 8 * n_kv;
  const int units = n_items * p.Hq;

  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  Bars B;
  B.q_full = bar + 0;
  B.q_empty = bar + 1;
  B.k_full = bar + 2;
  B.k_empty = B.k_full + C::NSK;
  B.v_full = B.k_empty + C::NSK;
  B.v_empty = B.v_full + C::NSV;
  B.s_full = B.v_empty + C::NSV;
  B.p_full = B.s_full + 2;
  B.pv_done = B.p_full + 2;
  B.o_free = B.pv_done + 2;
  B.sch_full = B.o_free + 2;
  B.sch_empty = B.sch_full + kSchedSlots;

  if (threadIdx.x == 0) {
    abort_flag = 0;
    mbar_init(B.q_full, 1);
    mbar_init(B.q_empty, 1);
    for (int i = 0; i < C::NSK; ++i) {
      mbar_init(B.k_full + i, 1);
      mbar_init(B.k_empty + i, 1);
    }
    for (int i = 0; i < C::NSV; ++i) {
      mbar_init(B.v_full + i, 1);
      mbar_init(B.v_empty + i, 1);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(B.s_full + x, 1);
      mbar_init(B.p_full + x, 4);
      mbar_init(B.pv_done + x, 1);
      mbar_init(B.o_free + x, 4);
    }
    for (int i = 0; i < kSchedSlots; ++i) {
      mbar_init(B.sch_full + i, 1);
      mbar_init(B.sch_empty + i, kSchedReaders);
    }
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&tmem_base_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_slot;

  if (warp < 4) {
    regs_dec();
    if (warp == 0 || warp == 2) {
    // ================================================================ producers
    // warp 0 fetches units and loads Q and K; warp 2 loads V.  The two rings
    // advance independently, so a K load never waits behind a V slot.
    if (lane == 0) {
      const bool kprod = warp == 0;
      if (kprod) {
        tma_prefetch_desc(&tmap_q);
        tma_prefetch_desc(&tmap_k);
      } else {
        tma_prefetch_desc(&tmap_v);
      }
      uint32_t kc = 0, uc = 0;
      bool ok = true;
      for (uint32_t i = 0; ok; ++i) {
        const int slot_s = i % kSchedSlots;
        const uint32_t sph = (i / kSchedSlots) & 1;
        int u;
        int4 it = make_int4(0, 0, 0, 0);
        if (kprod) {
          if (!mbar_wait(B.sch_empty + slot_s, sph ^ 1, &abort_flag, p.status)) break;
          u = atomicAdd(p.counter, 1);
          if (u < units) {
            int item, hh;
            unit_block_head(u, n_items, p.Hq, p.G, item, hh);
            it = __ldg(items + item);
          }
          // a block outside the schedule or the tokens becomes an empty one
          // for every role (debug build)
          if (!psa_in_bounds(item_in_bounds(it, n_kv, p.T), p.status)) it = make_int4(0, 0, 0, 0);
          sch_item[slot_s] = it;
          sch_unit[slot_s] = u;
          mbar_arrive(B.sch_full + slot_s);
        } else {
          if (!mbar_wait(B.sch_full + slot_s, sph, &abort_flag, p.status)) break;
          u = sch_unit[slot_s];
          it = sch_item[slot_s];
          mbar_arrive(B.sch_empty + slot_s);
        }
        if (u >= units) break;
        int item_u, h;
        unit_block_head(u, n_items, p.Hq, p.G, item_u, h);
        const int kvh = h / p.G;
        if (it.w == 0) continue;
        if (kprod) {
          if (!mbar_wait(B.q_empty, (uc & 1) ^ 1, &abort_flag, p.status)) break;
          mbar_arrive_expect_tx(B.q_full, 2 * C::Q_BYTES);
#pragma unroll
          for (int x = 0; x < 2; ++x)
#pragma unroll
            for (int part = 0; part < C::NPART; ++part)
              tma_load_3d(smem + C::OFF_Q + x * C::Q_BYTES + part * BM * 128, &tmap_q,
                          B.q_full, part * 64, h, it.x + x * BM);
        }
        for (int j = 0; j < it.w; ++j) {
          const int k0 = __ldg(kvs + 8 * (it.z + j));
          const int ns = kprod ? C::NSK : C::NSV;
          const int slot = kc % ns;
          const uint32_t ph = (kc / ns) & 1;
          uint64_t* empty = kprod ? B.k_empty : B.v_empty;
          uint64_t* full = kprod ? B.k_full : B.v_full;
          if (!mbar_wait(empty + slot, ph ^ 1, &abort_flag, p.status)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(full + slot, C::KV_BYTES);
          uint8_t* dst = smem + (kprod ? C::OFF_K : C::OFF_V) + slot * C::KV_BYTES;
          const CUtensorMap* tm = kprod ? &tmap_k : &tmap_v;
#pragma unroll
          for (int part = 0; part < C::NPART; ++part)
            tma_load_3d(dst + part * BN * 128, tm, full + slot, part * 64, kvh, k0);
          ++kc;
        }
        ++uc;
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
      const uint32_t idesc_qk = umma_idesc_bf16(BM, BN, false, false);
      const uint32_t idesc_pv = umma_idesc_bf16(BM, D, false, true);
      const uint32_t sQ = smem_u32(smem + C::OFF_Q);
      const uint32_t sK = smem_u32(smem + C::OFF_K);
      const uint32_t sV = smem_u32(smem + C::OFF_V);
      uint32_t kc = 0, uc = 0;
      uint32_t pvc[2] = {0, 0};  // PVs issued per half (all units)
      uint32_t uhc[2] = {0, 0};  // units in which the half had work
      bool ok = true;

      // S_X = Q_X K_t^T into the S columns of half x
      auto issue_qk = [&](int x, uint32_t t_glob) -> bool {
        const int slot = t_glob % C::NSK;
        if (!mbar_wait(B.k_full + slot, (t_glob / C::NSK) & 1, &abort_flag, p.status))
          return false;
        tc_fence_after();
        const uint32_t qbase = sQ + x * C::Q_BYTES, kbase = sK + slot * C::KV_BYTES;
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const uint32_t off = (ks >> 2) * (BM * 128) + (ks & 3) * 32;
          umma_ss(tmem + x * 256, umma_desc_sw128(qbase + off, 16, 1024),
                  umma_desc_sw128(kbase + off, 16, 1024), idesc_qk, ks > 0 ? 1u : 0u);
        }
        umma_commit(B.s_full + x);
        return true;
      };
      // O_X += P_X V_t, P_X in TMEM over the first 64 columns of S_X
      auto issue_pv = [&](int x, uint32_t t_glob, bool first) -> bool {
        if (!mbar_wait(B.p_full + x, pvc[x] & 1, &abort_flag, p.status)) return false;
        const int slot = t_glob % C::NSV;
        if (!mbar_wait(B.v_full + slot, (t_glob / C::NSV) & 1, &abort_flag, p.status))
          return false;
        if (first && !mbar_wait(B.o_free + x, (uhc[x] & 1) ^ 1, &abort_flag, p.status))
          return false;
        tc_fence_after();
        const uint32_t vbase = sV + slot * C::KV_BYTES;
#pragma unroll
        for (int ks = 0; ks < BN / 16; ++ks)
          umma_ts(tmem + x * 256 + 128, tmem + x * 256 + ks * 8,
                  umma_desc_sw128(vbase + ks * 2048, BN * 128, 1024), idesc_pv,
                  (first && ks == 0) ? 0u : 1u);
        umma_commit(B.pv_done + x);
        ++pvc[x];
        return true;
      };

      for (uint32_t i = 0; ok; ++i) {
        const int slot_s = i % kSchedSlots;
        if (!mbar_wait(B.sch_full + slot_s, (i / kSchedSlots) & 1, &abort_flag, p.status)) break;
        const int u = sch_unit[slot_s];
        const int4 it = sch_item[slot_s];
        mbar_arrive(B.sch_empty + slot_s);
        if (u >= units) break;
        const int n = it.w;
        if (n == 0) continue;
        // tile flags (which halves see the tile) are read two tiles ahead so
        // their latency hides behind the waits
        int f = __ldg(kvs + 8 * it.z + 6);
        int fn = n > 1 ? __ldg(kvs + 8 * (it.z + 1) + 6) : 0;
        if (!mbar_wait(B.q_full, uc & 1, &abort_flag, p.status)) break;
        bool started[2] = {false, false};
        // prologue: QK of tile 0 for each half that takes part in it
#pragma unroll
        for (int x = 0; x < 2; ++x)
          if (ok && (f & (1 << x))) ok = issue_qk(x, kc);
        if (!ok) break;
        umma_commit(B.k_empty + (kc % C::NSK));
        if (n == 1) umma_commit(B.q_empty);
        for (int j = 0; j < n && ok; ++j) {
          const int fnn = j + 2 < n ? __ldg(kvs + 8 * (it.z + j + 2) + 6) : 0;
          const uint32_t t = kc + j;
#pragma unroll
          for (int x = 0; x < 2; ++x) {
            if (ok && (f & (1 << x))) {
              ok = issue_pv(x, t, !started[x]);
              started[x] = true;
            }
            if (ok && (fn & (1 << x))) ok = issue_qk(x, t + 1);
          }
          if (!ok) break;
          umma_commit(B.v_empty + (t % C::NSV));
          if (j + 1 < n) {
            umma_commit(B.k_empty + ((t + 1) % C::NSK));
            if (j + 2 == n) umma_commit(B.q_empty);
          }
          f = fn;
          fn = fnn;
        }
        if (!ok) break;
        kc += n;
#pragma unroll
        for (int x = 0; x < 2; ++x)
          if (started[x]) ++uhc[x];
        ++uc;
      }
      if (!ok || abort_flag) {
        // give MMAs already issued time to finish before TMEM is freed
        const uint64_t t0 = globaltimer();
        while (globaltimer() - t0 < 1000000ull) {
        }
      }
    }
    }
  } else {
    regs_inc();
    // ================================================================ softmax + epilogue
    const int x = (warp - 4) >> 2;      // half
    const int quarter = warp & 3;       // TMEM lane quarter
    const int r = quarter * 32 + lane;  // row within the half
    const uint32_t trow = tmem + (uint32_t(quarter * 32) << 16) + x * 256;
    const uint32_t tS = trow, tO = trow + 128;
    uint32_t sc_count = 0;  // S tiles of this half consumed (all units)
    bool ok = true;
    for (uint32_t i = 0; ok; ++i) {
      const int slot_s = i % kSchedSlots;
      if (!mbar_wait(B.sch_full + slot_s, (i / kSchedSlots) & 1, &abort_flag, p.status)) break;
      const int u = sch_unit[slot_s];
      const int4 it = sch_item[slot_s];
      __syncwarp();
      if (lane == 0) mbar_arrive(B.sch_empty + slot_s);
      if (u >= units) break;
      int item_u, h;
      unit_block_head(u, n_items, p.Hq, p.G, item_u, h);
      const int q = it.x + x * BM + r;
      const bool valid = x * BM + r < it.y;
      __nv_bfloat16* orow = static_cast<__nv_bfloat16*>(p.o) + (size_t(q) * p.Hq + h) * D;

      float m_run = -INFINITY, l_run = 0.f;
      int nt = 0;  // tiles of this half in this unit
      // the next tile's schedule entry is read one tile ahead
      KvEntry e_next{0, 0, 0, 0, 0};
      if (it.w > 0) e_next = load_kv(kvs, it.z, x);
      for (int j = 0; j < it.w; ++j) {
        const KvEntry e = e_next;
        if (j + 1 < it.w) e_next = load_kv(kvs, it.z + j + 1, x);
        if (!(e.flags & (1 << x))) continue;
        if (!mbar_wait(B.s_full + x, sc_count & 1, &abort_flag, p.status)) {
          ok = false;
          break;
        }
        tc_fence_after();

        const bool need_mask = !(e.flags & (4 << x)) || e.klen < BN;
        uint32_t vis[4] = {0xffffffffu, 0xffffffffu, 0xffffffffu, 0xffffffffu};
        if (need_mask) row_visibility(e, x, q, rects, n_rect, p.status, vis);

        // the whole S row in one TMEM load
        uint32_t sr[BN];
        tmem_ld128(tS, sr);
        tmem_wait_ld();
        if (need_mask) {
#pragma unroll
          for (int k = 0; k < BN; ++k)
            if (!((vis[k >> 5] >> (k & 31)) & 1u)) sr[k] = __float_as_uint(-INFINITY);
        }
        // row max of the raw logits (scale > 0 commutes with max)
        float mx8[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) mx8[k] = __uint_as_float(sr[k]);
#pragma unroll
        for (int k = 8; k < BN; ++k) mx8[k & 7] = fmaxf(mx8[k & 7], __uint_as_float(sr[k]));
        const float mx = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                               fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7]))) *
                         p.scale_log2;
        const float m_new = fmaxf(m_run, mx);
        const bool resc = m_new > m_run + kRescaleLog2;
        // O (the PVs of earlier tiles) is rescaled after P is stored, when the
        // S row no longer occupies registers; it only has to happen before
        // this tile's PV, which waits for p_full.
        const bool rescale_o = __any_sync(0xffffffffu, resc) && nt > 0;
        float alpha = 1.f;
        if (resc) {
          alpha = fast_exp2(m_run - m_new);
          l_run *= alpha;
          m_run = m_new;
        }
        const float neg_m = m_run == -INFINITY ? 0.f : -m_run;

        // P = exp2(s * scale - m) as bf16, written over the S columns (masked
        // logits are -inf and give exactly 0)
        const uint64_t sc2 = f2_pack(p.scale_log2, p.scale_log2), nm2 = f2_pack(neg_m, neg_m);
        uint64_t acc2[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
        for (int k = 0; k < BN / 2; ++k) {
          float x0, x1;
          f2_unpack(f2_fma(f2_pack(__uint_as_float(sr[2 * k]), __uint_as_float(sr[2 * k + 1])),
                           sc2, nm2),
                    x0, x1);
          const float p0 = fast_exp2(x0), p1 = fast_exp2(x1);
          acc2[k & 3] = f2_add(acc2[k & 3], f2_pack(p0, p1));
          sr[k] = pack_bf16(p0, p1);  // packed pairs go into consumed registers (k <= 2k)
        }
        float ls8[8];
#pragma unroll
        for (int k = 0; k < 4; ++k) f2_unpack(acc2[k], ls8[2 * k], ls8[2 * k + 1]);
        tmem_st64(tS, *reinterpret_cast<uint32_t(*)[BN / 2]>(sr));
        l_run += ((ls8[0] + ls8[1]) + (ls8[2] + ls8[3])) + ((ls8[4] + ls8[5]) + (ls8[6] + ls8[7]));
        if (rescale_o) {
          // wait for the latest PV into O, then scale O by alpha in place
          if (!mbar_wait(B.pv_done + x, (sc_count - 1) & 1, &abort_flag, p.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t rr[32];
            tmem_ld32(tO + c * 32, rr);
            tmem_wait_ld();
#pragma unroll
            for (int k = 0; k < 32; ++k) rr[k] = __float_as_uint(__uint_as_float(rr[k]) * alpha);
            tmem_st32(tO + c * 32, rr);
          }
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(B.p_full + x);
        ++sc_count;
        ++nt;
      }
      if (!ok) break;

      if (nt == 0) {
        // this half sees nothing in the block (rows past the group end)
        if (valid) {
          for (int c = 0; c < D; ++c) orow[c] = __float2bfloat16(0.f);
          if (p.lse) p.lse[size_t(q) * p.Hq + h] = -INFINITY;
        }
        continue;
      }
      // ---- epilogue: O / l straight from TMEM, LSE
      if (!mbar_wait(B.pv_done + x, (sc_count - 1) & 1, &abort_flag, p.status)) break;
      tc_fence_after();
      const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
      {
        uint32_t orr[D];
        if constexpr (D == 128) {
          tmem_ld128(tO, orr);
        } else {
          tmem_ld64(tO, orr);
        }
        tmem_wait_ld();
        if (valid) {
          // the row as 32-byte stores when the output is 32-byte aligned (half
          // the store instructions of 16-byte ones; each thread's row is its
          // own, so a warp store touches 32 rows)
          if ((reinterpret_cast<uintptr_t>(p.o) & 31u) == 0) {
#pragma unroll
            for (int k = 0; k < D / 16; ++k) {
              uint32_t w[8];
#pragma unroll
              for (int i = 0; i < 8; ++i)
                w[i] = pack_bf16(__uint_as_float(orr[16 * k + 2 * i]) * inv,
                                 __uint_as_float(orr[16 * k + 2 * i + 1]) * inv);
              asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(
                               orow + 16 * k),
                           "r"(w[0]), "r"(w[1]), "r"(w[2]), "r"(w[3]), "r"(w[4]), "r"(w[5]),
                           "r"(w[6]), "r"(w[7])
                           : "memory");
            }
          } else {
            uint4* dst = reinterpret_cast<uint4*>(orow);
#pragma unroll
            for (int k = 0; k < D / 8; ++k)
              dst[k] = make_uint4(
                  pack_bf16(__uint_as_float(orr[8 * k]) * inv, __uint_as_float(orr[8 * k + 1]) * inv),
                  pack_bf16(__uint_as_float(orr[8 * k + 2]) * inv,
                            __uint_as_float(orr[8 * k + 3]) * inv),
                  pack_bf16(__uint_as_float(orr[8 * k + 4]) * inv,
                            __uint_as_float(orr[8 * k + 5]) * inv),
                  pack_bf16(__uint_as_float(orr[8 * k + 6]) * inv,
                            __uint_as_float(orr[8 * k + 7]) * inv));
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(B.o_free + x);
      if (valid && p.lse)
        p.lse[size_t(q) * p.Hq + h] = l_run > 0.f ? (m_run + __log2f(l_run)) * kLn2 : -INFINITY;
    }
  }

  // ---- teardown: every role has finished issuing; free TMEM
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, kTmemCols);
}

// fp32 I/O path: the same schedule and visibility, fp32 CUDA-core
// arithmetic throughout (no rounding of the fp32 inputs).  One warp per
// (query row, head); lanes split the head dimension.  It serves small fp32
// problems; the bf16 tensor-core kernel above is the throughput path.
template <int D>
__global__ void __launch_bounds__(256) prefill_f32_kernel(
    const float* __restrict__ q, const float* __restrict__ k, const float* __restrict__ v,
    float* __restrict__ o, float* __restrict__ lse, const int32_t* __restrict__ sch,
    int64_t sched_len, int32_t T, int32_t Hq, int32_t G, float scale_log2, int32_t* status) {
  constexpr int E = D / 32;
  if (!schedule_ok(sch, sched_len)) {
    if (blockIdx.x == 0 && threadIdx.x == 0) report_status(status, PSA_ERR_INVALID_ARG);
    return;
  }
  const int32_t n_items = __ldg(sch + 1), n_kv = __ldg(sch + 2), n_rect = __ldg(sch + 3);
  const int4* items = reinterpret_cast<const int4*>(sch + 8);
  const int32_t* kvs = sch + 8 + 4 * n_items;
  const int32_t* rects = kvs + 8 * n_kv;
  const int lane = threadIdx.x & 31;
  const int64_t total = int64_t(n_items) * BLOCK_M * Hq;
  const int64_t nwarps = int64_t(gridDim.x) * (blockDim.x >> 5);
  const int Hkv = Hq / G;
  for (int64_t u = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5; u < total;
       u += nwarps) {
    const int item = int(u / (int64_t(BLOCK_M) * Hq));
    const int rem = int(u % (int64_t(BLOCK_M) * Hq));
    const int r = rem / Hq, h = rem % Hq;
    const int4 it = __ldg(items + item);
    if (!psa_in_bounds(item_in_bounds(it, n_kv, T), lane == 0 ? status : nullptr)) continue;
    if (r >= it.y) continue;
    const int x = r / BM;
    const int qi = it.x + r, kvh = h / G;
    float qv[E], acc[E];
#pragma unroll
    for (int e = 0; e < E; ++e) {
      qv[e] = q[(size_t(qi) * Hq + h) * D + lane * E + e];
      acc[e] = 0.f;
    }
    float m = -INFINITY, l = 0.f;
    for (int j = 0; j < it.w; ++j) {
      const KvEntry ent = load_kv(kvs, it.z + j, x);
      if (!(ent.flags & (1 << x))) continue;
      uint32_t vis[4];
      row_visibility(ent, x, qi, rects, n_rect, status, vis);
      for (int kk = 0; kk < ent.klen; ++kk) {
        if (!((vis[kk >> 5] >> (kk & 31)) & 1u)) continue;
        const int key = ent.k0 + kk;
        const float* kr = k + (size_t(key) * Hkv + kvh) * D + lane * E;
        float d = 0.f;
#pragma unroll
        for (int e = 0; e < E; ++e) d = fmaf(qv[e], kr[e], d);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) d += __shfl_xor_sync(0xffffffffu, d, off);
        const float sv = d * scale_log2;
        const float mn = fmaxf(m, sv);
        const float alpha = exp2f(m - mn);
        const float pe = exp2f(sv - mn);
        l = l * alpha + pe;
        const float* vr = v + (size_t(key) * Hkv + kvh) * D + lane * E;
#pragma unroll
        for (int e = 0; e < E; ++e) acc[e] = fmaf(acc[e], alpha, pe * vr[e]);
        m = mn;
      }
    }
    const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
    for (int e = 0; e < E; ++e) o[(size_t(qi) * Hq + h) * D + lane * E + e] = acc[e] * inv;
    if (lse && lane == 0) lse[size_t(qi) * Hq + h] = l > 0.f ? (m + log2f(l)) * kLn2 : -INFINITY;
  }
}

template <int D>
int launch_prefill_f32_d(const PrefillArgs& a) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return PSA_ERR_CUDA;
  const int grid = 4 * sm_count(dev);
  if (grid <= 0) return PSA_ERR_CUDA;
  prefill_f32_kernel<D><<<grid, 256, 0, a.stream>>>(
      static_cast<const float*>(a.q), static_cast<const float*>(a.k),
      static_cast<const float*>(a.v), static_cast<float*>(a.o), a.lse, a.sched, a.sched_len,
      a.T, a.Hq, a.Hq / a.Hkv, a.scale * kLog2e, a.status);
  return cudaGetLastError() == cudaSuccess ? PSA_OK : PSA_ERR_CUDA;
}

template <int D>
int launch_prefill_d(const PrefillArgs& a) {
  using C = Cfg<D>;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return PSA_ERR_CUDA;
  CUtensorMap tq, tk, tv;
  const uint32_t box[3] = {64u, 1u, uint32_t(BM)};
  {
    const uint64_t dims[3] = {uint64_t(D), uint64_t(a.Hq), uint64_t(a.T)};
    const uint64_t strides[2] = {uint64_t(D) * 2, uint64_t(a.Hq) * D * 2};
    int rc = encode_tmap(&tq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, a.q, dims, strides, box,
                         CU_TENSOR_MAP_SWIZZLE_128B);
    if (rc != PSA_OK) return rc;
  }
  {
    const uint64_t dims[3] = {uint64_t(D), uint64_t(a.Hkv), uint64_t(a.T)};
    const uint64_t strides[2] = {uint64_t(D) * 2, uint64_t(a.Hkv) * D * 2};
    int rc = encode_tmap(&tk, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, a.k, dims, strides, box,
                         CU_TENSOR_MAP_SWIZZLE_128B);
    if (rc != PSA_OK) return rc;
    rc = encode_tmap(&tv, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, a.v, dims, strides, box,
                     CU_TENSOR_MAP_SWIZZLE_128B);
    if (rc != PSA_OK) return rc;
  }
  Params p;
  p.sched = a.sched;
  p.sched_len = a.sched_len;
  p.o = a.o;
  p.lse = a.lse;
  p.T = a.T;
  p.Hq = a.Hq;
  p.Hkv = a.Hkv;
  p.G = a.Hq / a.Hkv;
  p.scale_log2 = a.scale * kLog2e;
  p.status = a.status;
  p.counter = a.counter;
  auto kern = prefill_kernel<D>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(C::SMEM)) !=
      cudaSuccess)
    return PSA_ERR_CUDA;
  const int grid = sm_count(dev);
  if (grid <= 0) return PSA_ERR_CUDA;
  if (cudaMemsetAsync(a.counter, 0, sizeof(int32_t), a.stream) != cudaSuccess)
    return PSA_ERR_CUDA;
  kern<<<grid, kThreads, C::SMEM, a.stream>>>(tq, tk, tv, p);
  return cudaGetLastError() == cudaSuccess ? PSA_OK : PSA_ERR_CUDA;
}

}  // namespace

int launch_prefill(const PrefillArgs& a) {
  if (a.out_f32) {
    switch (a.D) {
      case 64:
        return launch_prefill_f32_d<64>(a);
      case 128:
        return launch_prefill_f32_d<128>(a);
      default:
        return PSA_ERR_UNSUPPORTED;
    }
  }
  switch (a.D) {
    case 64:
      return launch_prefill_d<64>(a);
    case 128:
      return launch_prefill_d<128>(a);
    default:
      return PSA_ERR_UNSUPPORTED;
  }
}

}  // namespace psa
