// Prefill over the flat, deduplicated packed layout: one forward pass of
// softmax attention in which the prefix K/V is stored once and every suffix
// sees it through the tile schedule ("KV-0 redundancy prefix sharing
// attention mask design", PrefixSharing PR #50: design summary -- flat
// dedup layout, block-causal rectangle spec instead of a dense mask, one
// forward that is mathematically equivalent to running each [prefix; s_i]).
//
// sm_100a design (one CTA per SM, persistent over (Q tile, query head)
// units; the host schedule lists them longest-first and the producer hands
// them out dynamically through a global counter, so the long suffix tiles
// start first and the short prefix tiles fill the tail):
//   warp 0      TMA producer: Q tile once per unit; K and V tiles of the
//               unit's visible KV tiles only (invisible tiles are never
//               touched) into two-slot rings, 128-byte swizzle, no multicast.
//   warp 1      tcgen05 issuer (one thread): S = Q K^T into a double-
//               buffered TMEM S, then O += P V into a TMEM O accumulator,
//               ordered QK_0, QK_1, PV_0, QK_2, PV_1, ... so the tensor
//               pipe computes the next S while the softmax works.
//   warps 4..7  softmax warpgroup, one query row per thread (= TMEM lane):
//               masks partial tiles from the copied rectangles, keeps the
//               running max in the log2 domain with lazy rescaling (O is
//               rescaled only when the max grows by more than 2^8), writes
//               P as bf16 into a double-buffered swizzled shared tile that
//               the next MMA reads as its K-major A operand, and runs the
//               epilogue (O / l, LSE) straight from TMEM.
// Every wait is bounded: a stuck pipeline reports PSA_ERR_TIMEOUT through
// the status word, the CTA unwinds and frees its TMEM.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "psa_device.cuh"
#include "psa_internal.h"

namespace psa {
namespace {

constexpr int BM = 128;            // query rows per tile
constexpr int BN = 128;            // keys per tile
constexpr int kThreads = 256;      // 8 warps
constexpr int kSoftmaxWarp0 = 4;   // warps 4..7 own TMEM lanes 0..127
constexpr float kRescaleLog2 = 8.f;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kSCol0 = 0, kSCol1 = 128, kOCol = 256;
constexpr int kSchedSlots = 4;  // units the producer may fetch ahead

template <int D>
struct Cfg {
  static constexpr int NPART = D / 64;  // 128-byte swizzle atoms across d
  static constexpr uint32_t Q_BYTES = BM * D * 2;
  static constexpr uint32_t KV_BYTES = BN * D * 2;
  static constexpr uint32_t P_BYTES = BM * BN * 2;
  static constexpr int NS = D == 128 ? 2 : 4;  // K and V ring slots
  static constexpr uint32_t OFF_Q = 0;
  static constexpr uint32_t OFF_K = OFF_Q + Q_BYTES;
  static constexpr uint32_t OFF_V = OFF_K + NS * KV_BYTES;
  static constexpr uint32_t OFF_P = OFF_V + NS * KV_BYTES;
  static constexpr uint32_t OFF_BAR = OFF_P + 2 * P_BYTES;
  static constexpr uint32_t NBAR = 2 + 4 * NS + 8 + 2 + 2 * kSchedSlots;
  static constexpr uint32_t SMEM = 1024 + OFF_BAR + NBAR * 8 + 16;
};

struct Params {
  const int32_t* sched;
  int64_t sched_len;
  void* o;
  float* lse;
  int32_t T, Hq, Hkv, G;
  int32_t out_f32;
  float scale_log2;
  int32_t* status;
  int32_t* counter;  // next unit to hand out (zeroed before every launch)
};

struct Bars {
  uint64_t *q_full, *q_empty, *k_full, *k_empty, *v_full, *v_empty;
  uint64_t *s_full, *s_free, *p_full, *p_free, *o_full, *o_free;
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

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // ---- schedule header (every thread reads it; the decision is uniform)
  const int32_t* sch = p.sched;
  const int32_t n_items = __ldg(sch + 1), n_kv = __ldg(sch + 2), n_rect = __ldg(sch + 3);
  const bool bad = __ldg(sch + 0) != 0x50534131 || __ldg(sch + 4) != BM ||
                   __ldg(sch + 5) != BN || n_items < 0 || n_kv < 0 || n_rect < 0 ||
                   8 + 4 * int64_t(n_items) + 4 * int64_t(n_kv) + 5 * int64_t(n_rect) >
                       p.sched_len;
  if (bad) {
    if (threadIdx.x == 0) report_status(p.status, PSA_ERR_INVALID_ARG);
    return;
  }
  const int4* items = reinterpret_cast<const int4*>(sch + 8);
  const int4* kvs = reinterpret_cast<const int4*>(sch + 8 + 4 * n_items);
  const int32_t* rects = sch + 8 + 4 * n_items + 4 * n_kv;
  const int units = n_items * p.Hq;

  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  Bars B;
  B.q_full = bar + 0;
  B.q_empty = bar + 1;
  B.k_full = bar + 2;
  B.k_empty = B.k_full + C::NS;
  B.v_full = B.k_empty + C::NS;
  B.v_empty = B.v_full + C::NS;
  B.s_full = B.v_empty + C::NS;
  B.s_free = B.s_full + 2;
  B.p_full = B.s_free + 2;
  B.p_free = B.p_full + 2;
  B.o_full = B.p_free + 2;
  B.o_free = B.o_full + 1;
  B.sch_full = B.o_free + 1;
  B.sch_empty = B.sch_full + kSchedSlots;

  if (threadIdx.x == 0) {
    abort_flag = 0;
    mbar_init(B.q_full, 1);
    mbar_init(B.q_empty, 1);
    for (int i = 0; i < C::NS; ++i) {
      mbar_init(B.k_full + i, 1);
      mbar_init(B.k_empty + i, 1);
      mbar_init(B.v_full + i, 1);
      mbar_init(B.v_empty + i, 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(B.s_full + i, 1);
      mbar_init(B.s_free + i, 4);
      mbar_init(B.p_full + i, 4);
      mbar_init(B.p_free + i, 1);
    }
    mbar_init(B.o_full, 1);
    mbar_init(B.o_free, 4);
    for (int i = 0; i < kSchedSlots; ++i) {
      mbar_init(B.sch_full + i, 1);
      mbar_init(B.sch_empty + i, 5);  // the MMA thread and the four softmax warps
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

  const uint32_t sQ = smem_u32(smem + C::OFF_Q);
  const uint32_t sK = smem_u32(smem + C::OFF_K);
  const uint32_t sV = smem_u32(smem + C::OFF_V);
  const uint32_t sP = smem_u32(smem + C::OFF_P);

  if (warp == 0) {
    // ================================================================ producer
    if (lane == 0) {
      tma_prefetch_desc(&tmap_q);
      tma_prefetch_desc(&tmap_k);
      tma_prefetch_desc(&tmap_v);
      uint32_t kc = 0, uc = 0;
      bool ok = true;
      for (uint32_t i = 0; ok; ++i) {
        // dynamic scheduler: hand the next unit to every role through smem
        const int slot = i % kSchedSlots;
        if (!mbar_wait(B.sch_empty + slot, ((i / kSchedSlots) & 1) ^ 1, &abort_flag, p.status))
          break;
        const int u = atomicAdd(p.counter, 1);
        sch_unit[slot] = u;
        mbar_arrive(B.sch_full + slot);
        if (u >= units) break;
        const int4 it = __ldg(items + u / p.Hq);
        const int h = u % p.Hq, kvh = h / p.G;
        if (it.w == 0) continue;
        if (!mbar_wait(B.q_empty, (uc & 1) ^ 1, &abort_flag, p.status)) break;
        mbar_arrive_expect_tx(B.q_full, C::Q_BYTES);
#pragma unroll
        for (int part = 0; part < C::NPART; ++part)
          tma_load_3d(smem + C::OFF_Q + part * BM * 128, &tmap_q, B.q_full, part * 64, h, it.x);
        for (int j = 0; j < it.w; ++j) {
          const int k0 = __ldg(&kvs[it.z + j].x);
          const int slot = kc % C::NS;
          const uint32_t ph = (kc / C::NS) & 1;
          if (!mbar_wait(B.k_empty + slot, ph ^ 1, &abort_flag, p.status)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(B.k_full + slot, C::KV_BYTES);
#pragma unroll
          for (int part = 0; part < C::NPART; ++part)
            tma_load_3d(smem + C::OFF_K + slot * C::KV_BYTES + part * BN * 128, &tmap_k,
                        B.k_full + slot, part * 64, kvh, k0);
          if (!mbar_wait(B.v_empty + slot, ph ^ 1, &abort_flag, p.status)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(B.v_full + slot, C::KV_BYTES);
#pragma unroll
          for (int part = 0; part < C::NPART; ++part)
            tma_load_3d(smem + C::OFF_V + slot * C::KV_BYTES + part * BN * 128, &tmap_v,
                        B.v_full + slot, part * 64, kvh, k0);
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
      uint32_t kc = 0, vc = 0, tg = 0, uc = 0;
      bool ok = true;

      auto issue_pv = [&](uint32_t t, bool first, bool last) -> bool {
        const uint32_t pb = t & 1;
        if (!mbar_wait(B.p_full + pb, (t >> 1) & 1, &abort_flag, p.status)) return false;
        const int slot = vc % C::NS;
        if (!mbar_wait(B.v_full + slot, (vc / C::NS) & 1, &abort_flag, p.status)) return false;
        if (first && !mbar_wait(B.o_free, (uc & 1) ^ 1, &abort_flag, p.status)) return false;
        tc_fence_after();
        const uint32_t pbase = sP + pb * C::P_BYTES;
        const uint32_t vbase = sV + slot * C::KV_BYTES;
#pragma unroll
        for (int ks = 0; ks < BN / 16; ++ks) {
          const uint64_t a = umma_desc_sw128(pbase + (ks >> 2) * (BM * 128) + (ks & 3) * 32, 16,
                                             1024);
          const uint64_t b = umma_desc_sw128(vbase + ks * 2048, BN * 128, 1024);
          umma_ss(tmem + kOCol, a, b, idesc_pv, (first && ks == 0) ? 0u : 1u);
        }
        umma_commit(B.p_free + pb);
        umma_commit(B.v_empty + slot);
        if (last) umma_commit(B.o_full);
        ++vc;
        return true;
      };

      for (uint32_t i = 0; ok; ++i) {
        const int slot_s = i % kSchedSlots;
        if (!mbar_wait(B.sch_full + slot_s, (i / kSchedSlots) & 1, &abort_flag, p.status)) break;
        const int u = sch_unit[slot_s];
        mbar_arrive(B.sch_empty + slot_s);
        if (u >= units) break;
        const int4 it = __ldg(items + u / p.Hq);
        if (it.w == 0) continue;
        if (!mbar_wait(B.q_full, uc & 1, &abort_flag, p.status)) break;
        for (int j = 0; j < it.w; ++j) {
          const int slot = kc % C::NS;
          const uint32_t sb = tg & 1;
          if (!mbar_wait(B.k_full + slot, (kc / C::NS) & 1, &abort_flag, p.status) ||
              !mbar_wait(B.s_free + sb, ((tg >> 1) & 1) ^ 1, &abort_flag, p.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t kbase = sK + slot * C::KV_BYTES;
#pragma unroll
          for (int ks = 0; ks < D / 16; ++ks) {
            const uint32_t off = (ks >> 2) * (BM * 128) + (ks & 3) * 32;
            const uint64_t a = umma_desc_sw128(sQ + off, 16, 1024);
            const uint64_t b = umma_desc_sw128(kbase + off, 16, 1024);
            umma_ss(tmem + (sb ? kSCol1 : kSCol0), a, b, idesc_qk, ks > 0 ? 1u : 0u);
          }
          umma_commit(B.s_full + sb);
          umma_commit(B.k_empty + slot);
          if (j == it.w - 1) umma_commit(B.q_empty);
          ++kc;
          if (j > 0 && !issue_pv(tg - 1, j == 1, false)) {
            ok = false;
            break;
          }
          ++tg;
        }
        if (!ok) break;
        if (!issue_pv(tg - 1, it.w == 1, true)) break;
        ++uc;
      }
      if (!ok || abort_flag) {
        // wait (bounded) for every MMA already issued before TMEM is freed
        uint64_t* drain = B.o_free;  // reuse: arrive count is irrelevant for a commit
        (void)drain;
        const uint64_t t0 = globaltimer();
        while (globaltimer() - t0 < 1000000ull) {
        }
      }
    }
  } else if (warp >= kSoftmaxWarp0) {
    // ================================================================ softmax + epilogue
    const int quarter = warp - kSoftmaxWarp0;
    const int r = quarter * 32 + lane;  // row within the Q tile = TMEM lane
    const uint32_t trow = tmem + (uint32_t(quarter * 32) << 16);
    uint32_t tg = 0, uc = 0;
    bool ok = true;
    for (uint32_t i = 0; ok; ++i) {
      const int slot_s = i % kSchedSlots;
      if (!mbar_wait(B.sch_full + slot_s, (i / kSchedSlots) & 1, &abort_flag, p.status)) break;
      const int u = sch_unit[slot_s];
      __syncwarp();
      if (lane == 0) mbar_arrive(B.sch_empty + slot_s);
      if (u >= units) break;
      const int4 it = __ldg(items + u / p.Hq);
      const int h = u % p.Hq;
      const int q = it.x + r;
      const bool valid = r < it.y;
      if (it.w == 0) {
        if (valid) {
          if (p.out_f32) {
            float* dst = static_cast<float*>(p.o) + (size_t(q) * p.Hq + h) * D;
            for (int c = 0; c < D; ++c) dst[c] = 0.f;
          } else {
            __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(p.o) + (size_t(q) * p.Hq + h) * D;
            for (int c = 0; c < D; ++c) dst[c] = __float2bfloat16(0.f);
          }
          if (p.lse) p.lse[size_t(q) * p.Hq + h] = -INFINITY;
        }
        continue;
      }
      float m_run = -INFINITY, l_run = 0.f;
      for (int j = 0; j < it.w; ++j) {
        const int4 e = __ldg(kvs + it.z + j);  // k0, k_len, rect_begin, rect_count
        const uint32_t sb = tg & 1;
        if (!mbar_wait(B.s_full + sb, (tg >> 1) & 1, &abort_flag, p.status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        float s[BN];
        {
          uint32_t rr[32];
#pragma unroll
          for (int c = 0; c < BN / 32; ++c) {
            tmem_ld32(trow + (sb ? kSCol1 : kSCol0) + c * 32, rr);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) s[c * 32 + i] = __uint_as_float(rr[i]);
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(B.s_free + sb);

        // visibility of this row inside the tile
        const bool need_mask = e.w > 0 || e.y < BN;
        uint32_t vis[4] = {0xffffffffu, 0xffffffffu, 0xffffffffu, 0xffffffffu};
        if (need_mask) {
          vis[0] = vis[1] = vis[2] = vis[3] = 0u;
          if (e.w == 0) {
            set_bits(vis, 0, e.y);
          } else {
            for (int ri = 0; ri < e.w; ++ri) {
              const int32_t* rc = rects + 5 * (e.z + ri);
              const int rq0 = __ldg(rc), rq1 = __ldg(rc + 1), rk0 = __ldg(rc + 2),
                        rk1 = __ldg(rc + 3), causal = __ldg(rc + 4);
              if (q < rq0 || q >= rq1) continue;
              int hi = causal ? min(rk1, rk0 + (q - rq0) + 1) : rk1;
              hi = min(hi, e.x + e.y);
              const int lo = max(rk0, e.x);
              if (lo < hi) set_bits(vis, lo - e.x, hi - e.x);
            }
          }
        }
        // raw logits stay unscaled (scale > 0 commutes with max); masked
        // entries become -inf.  Eight independent max chains.
        if (need_mask) {
#pragma unroll
          for (int i = 0; i < BN; ++i)
            s[i] = ((vis[i >> 5] >> (i & 31)) & 1u) ? s[i] : -INFINITY;
        }
        float mx8[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) mx8[k] = s[k];
#pragma unroll
        for (int i = 8; i < BN; ++i) mx8[i & 7] = fmaxf(mx8[i & 7], s[i]);
        const float mx = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                               fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7]))) *
                         p.scale_log2;
        const float m_new = fmaxf(m_run, mx);
        const bool resc = m_new > m_run + kRescaleLog2;
        if (__any_sync(0xffffffffu, resc) && j > 0) {
          // O holds PV of earlier tiles: wait for the latest, rescale in TMEM
          const uint32_t tp = tg - 1;
          if (!mbar_wait(B.p_free + (tp & 1), (tp >> 1) & 1, &abort_flag, p.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const float alpha = resc ? fast_exp2(m_run - m_new) : 1.f;
          uint32_t rr[32];
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            tmem_ld32(trow + kOCol + c * 32, rr);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) rr[i] = __float_as_uint(__uint_as_float(rr[i]) * alpha);
            tmem_st32(trow + kOCol + c * 32, rr);
          }
          tmem_wait_st();
        }
        if (resc) {
          l_run *= fast_exp2(m_run - m_new);
          m_run = m_new;
        }
        const float m_use = m_run == -INFINITY ? 0.f : m_run;

        // P buffer sb is free once the PV two tiles back has completed
        if (!mbar_wait(B.p_free + sb, ((tg >> 1) & 1) ^ 1, &abort_flag, p.status)) {
          ok = false;
          break;
        }
        const uint32_t prow = sP + sb * C::P_BYTES + r * 128;
        const float sc = p.scale_log2, neg_m = -m_use;
        float ls8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int c = 0; c < BN / 8; ++c) {
          uint32_t w[4];
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const float p0 = fast_exp2(fmaf(s[c * 8 + 2 * k], sc, neg_m));
            const float p1 = fast_exp2(fmaf(s[c * 8 + 2 * k + 1], sc, neg_m));
            ls8[2 * k] += p0;
            ls8[2 * k + 1] += p1;
            w[k] = pack_bf16(p0, p1);
          }
          const uint32_t addr = prow + (c >> 3) * (BM * 128) + (((c & 7) ^ (r & 7)) << 4);
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(w[0]),
                       "r"(w[1]), "r"(w[2]), "r"(w[3])
                       : "memory");
        }
        const float lsum = ((ls8[0] + ls8[1]) + (ls8[2] + ls8[3])) +
                           ((ls8[4] + ls8[5]) + (ls8[6] + ls8[7]));
        l_run += lsum;
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(B.p_full + sb);
        ++tg;
      }
      if (!ok) break;

      // ---- epilogue: O / l straight from TMEM, LSE
      if (!mbar_wait(B.o_full, uc & 1, &abort_flag, p.status)) break;
      tc_fence_after();
      const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
      uint32_t rr[32];
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        tmem_ld32(trow + kOCol + c * 32, rr);
        tmem_wait_ld();
        if (valid) {
          if (p.out_f32) {
            float4* dst = reinterpret_cast<float4*>(static_cast<float*>(p.o) +
                                                    (size_t(q) * p.Hq + h) * D + c * 32);
#pragma unroll
            for (int k = 0; k < 8; ++k)
              dst[k] = make_float4(__uint_as_float(rr[4 * k]) * inv,
                                   __uint_as_float(rr[4 * k + 1]) * inv,
                                   __uint_as_float(rr[4 * k + 2]) * inv,
                                   __uint_as_float(rr[4 * k + 3]) * inv);
          } else {
            uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.o) +
                                                  (size_t(q) * p.Hq + h) * D + c * 32);
#pragma unroll
            for (int k = 0; k < 4; ++k)
              dst[k] = make_uint4(
                  pack_bf16(__uint_as_float(rr[8 * k]) * inv, __uint_as_float(rr[8 * k + 1]) * inv),
                  pack_bf16(__uint_as_float(rr[8 * k + 2]) * inv,
                            __uint_as_float(rr[8 * k + 3]) * inv),
                  pack_bf16(__uint_as_float(rr[8 * k + 4]) * inv,
                            __uint_as_float(rr[8 * k + 5]) * inv),
                  pack_bf16(__uint_as_float(rr[8 * k + 6]) * inv,
                            __uint_as_float(rr[8 * k + 7]) * inv));
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(B.o_free);
      if (valid && p.lse)
        p.lse[size_t(q) * p.Hq + h] =
            l_run > 0.f ? (m_run + __log2f(l_run)) * kLn2 : -INFINITY;
      ++uc;
    }
  }

  // ---- teardown: every role has finished issuing; free TMEM
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, kTmemCols);
}

template <int D>
__global__ void __launch_bounds__(256) prefill_f32_kernel(
    const float* __restrict__ q, const float* __restrict__ k, const float* __restrict__ v,
    float* __restrict__ o, float* __restrict__ lse, const int32_t* __restrict__ sch,
    int64_t sched_len, int32_t Hq, int32_t G, float scale_log2, int32_t* status) {
  constexpr int E = D / 32;
  const int32_t n_items = __ldg(sch + 1), n_kv = __ldg(sch + 2), n_rect = __ldg(sch + 3);
  const bool bad = __ldg(sch + 0) != 0x50534131 || __ldg(sch + 4) != BM ||
                   __ldg(sch + 5) != BN || n_items < 0 || n_kv < 0 || n_rect < 0 ||
                   8 + 4 * int64_t(n_items) + 4 * int64_t(n_kv) + 5 * int64_t(n_rect) >
                       sched_len;
  if (bad) {
    if (blockIdx.x == 0 && threadIdx.x == 0) report_status(status, PSA_ERR_INVALID_ARG);
    return;
  }
  const int4* items = reinterpret_cast<const int4*>(sch + 8);
  const int4* kvs = reinterpret_cast<const int4*>(sch + 8 + 4 * n_items);
  const int32_t* rects = sch + 8 + 4 * n_items + 4 * n_kv;
  const int lane = threadIdx.x & 31;
  const int64_t total = int64_t(n_items) * BM * Hq;
  const int64_t nwarps = int64_t(gridDim.x) * (blockDim.x >> 5);
  for (int64_t u = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5; u < total;
       u += nwarps) {
    const int item = int(u / (int64_t(BM) * Hq));
    const int rem = int(u % (int64_t(BM) * Hq));
    const int r = rem / Hq, h = rem % Hq;
    const int4 it = __ldg(items + item);
    if (r >= it.y) continue;
    const int qi = it.x + r, kvh = h / G;
    const int Hkv = Hq / G;
    float qv[E], acc[E];
#pragma unroll
    for (int e = 0; e < E; ++e) {
      qv[e] = q[(size_t(qi) * Hq + h) * D + lane * E + e];
      acc[e] = 0.f;
    }
    float m = -INFINITY, l = 0.f;
    for (int j = 0; j < it.w; ++j) {
      const int4 ent = __ldg(kvs + it.z + j);
      for (int kk = ent.x; kk < ent.x + ent.y; ++kk) {
        bool on = ent.w == 0;
        for (int ri = 0; ri < ent.w && !on; ++ri) {
          const int32_t* rc = rects + 5 * (ent.z + ri);
          const int rq0 = rc[0], rq1 = rc[1], rk0 = rc[2], rk1 = rc[3], causal = rc[4];
          on = qi >= rq0 && qi < rq1 && kk >= rk0 && kk < rk1 && (!causal || kk - rk0 <= qi - rq0);
        }
        if (!on) continue;
        const float* kr = k + (size_t(kk) * Hkv + kvh) * D + lane * E;
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
        const float* vr = v + (size_t(kk) * Hkv + kvh) * D + lane * E;
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
      a.Hq, a.Hq / a.Hkv, a.scale * kLog2e, a.status);
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
  p.out_f32 = a.out_f32 ? 1 : 0;
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
