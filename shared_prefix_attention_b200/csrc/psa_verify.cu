// Speculative-verify attention: split-KV over the cached prefix (stage 1)
// and a log-sum-exp combine that folds in the causal draft block (stage 2).
// "Split-KV flash-decode attention for EAGLE target-verify" (sglang PR
// #27382), implementation breakdown item 1 and motivation (the pre-split
// verify path reached about 8% of HBM bandwidth at 16k context).
//
// Stage 1 is an HBM stream.  A persistent CTA walks work units
// (request b, split s, block of KV heads); for each unit one producer
// thread streams 16-token K/V tiles with TMA (128-byte swizzle, no
// multicast) into a ring of shared-memory stages, and one consumer warp per
// (KV head, 16-row m-tile) forms S = Q K^T and O += P V with warp MMAs.
// The 16 rows of an m-tile are all query heads of the KV head's group times
// all draft tokens, so each shared K/V row is read from HBM once for every
// query head that uses it (GQA/MQA grouping).  The output of a unit is the
// normalised partial O and its log2-domain LSE in the workspace.
//
// Stage 2 has one warp per (draft row, query head): it scores the draft
// keys 0..j (or the row of a tree mask), then merges them with every split
// by LSE weights.
//
// The extend form of the same call: a paged prefix (a page table of one
// token per page; the PAGED instantiation gathers each key's row of HB heads
// with one bulk copy, issued by four producer warps, into a padded row
// layout), ragged draft counts (rows mapped through qo_indptr; units with no
// live row skipped) and per-request tree masks (stage 2).
#include <cuda_bf16.h>
#include <cuda_runtime.h>


#include "psa_debug.cuh"
#include "psa_device.cuh"
#include "psa_internal.h"

namespace psa {

template <int D>
int launch_combine_d(const VerifyArgs& a);

namespace {

// Plain (untiled) bulk copy of `bytes` contiguous global bytes into shared
// memory, completing on `bar`'s transaction count.  Both addresses and the
// size must be multiples of 16 bytes.
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes,
                                          uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
      ::"r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

constexpr int kTileKeys = 16;      // keys per pipeline stage
// Consumer warps per CTA: with the producer warp, 9 warps leave each warp
// 168 registers; head_dim 256 needs more, so it runs 4 consumer warps.
__host__ __device__ constexpr int max_consumer_warps(int D) { return D > 128 ? 4 : 8; }

struct Stage1Params {
  const __nv_bfloat16* q;  // [nrows, Hq, D]
  const int32_t* indptr;   // [B+1]
  // Page table (nullable): prefix position t is cache row kv_indices[t];
  // those rows are gathered with cp.async instead of TMA tiles.
  const int32_t* kv_indices;
  const __nv_bfloat16* kc;  // [ntok, Hkv, D], read directly only when paged
  const __nv_bfloat16* vc;
  int64_t ntok;
  const int32_t* qo_indptr;  // nullable: request b's draft rows are b*Ld + [0, Ld)
  int32_t nrows;             // draft rows in all
  float* part_o;
  float* part_lse;
  int32_t B, Ld, Hq, Hkv, G, R;
  int32_t MT;   // m-tiles per CTA for each KV head
  int32_t nrb;  // row blocks: a head's m-tiles are split over nrb CTAs
  int32_t HB, nhb, nsplit;
  float scale_log2;
  int32_t* status;
  int32_t nstage;
};

struct Unit {
  int b, s, rb, hb;
};

// Work units are ordered so that consecutive units stream adjacent memory.
__device__ __forceinline__ Unit decode_unit(const Stage1Params& p, int u) {
  Unit x;
  x.hb = u % p.nhb;
  u /= p.nhb;
  x.rb = u % p.nrb;
  u /= p.nrb;
  x.s = u % p.nsplit;
  x.b = u / p.nsplit;
  return x;
}

// First draft row and draft count of request b (Ld is the maximum count).
// A count above Ld is reported and clamped; a decreasing qo_indptr or rows
// outside [0, nrows) are reported and the request is treated as empty.
__device__ __forceinline__ void request_rows(const int32_t* qo_indptr, int Ld, int nrows, int b,
                                             int& q0, int& Lb, int32_t* status) {
  if (!qo_indptr) {
    q0 = b * Ld;
    Lb = Ld;
    return;
  }
  q0 = __ldg(qo_indptr + b);
  Lb = __ldg(qo_indptr + b + 1) - q0;
  if (Lb > Ld) {
    report_status(status, PSA_ERR_INVALID_ARG);
    Lb = Ld;
  }
  if (Lb < 0 || q0 < 0 || q0 > nrows - Lb) {
    report_status(status, PSA_ERR_INVALID_ARG);
    Lb = 0;
  }
}

// A unit does work only if its row block holds a draft row of the request.
__device__ __forceinline__ bool unit_live(const Stage1Params& p, const Unit& x, int Lb) {
  return x.rb * p.MT * 16 < Lb * p.G;
}

__device__ __forceinline__ void split_range(const Stage1Params& p, int b, int s, int32_t& t0,
                                            int32_t& t1) {
  const int32_t a = __ldg(p.indptr + b), e = __ldg(p.indptr + b + 1);
  int32_t L = e - a;
  // a paged prefix must lie inside the page table, whose length is indptr[B]
  const bool in_table = !p.kv_indices || e <= __ldg(p.indptr + p.B);
  if (L < 0 || a < 0 || !in_table) L = 0;
  // debug build: an offset outside the page table or (contiguous) the cache
  // is reported and the request's prefix left out
  if (!psa_in_bounds(e >= a && a >= 0 && in_table && (p.kv_indices || int64_t(e) <= p.ntok),
                     p.status))
    L = 0;
  int32_t c = (L + p.nsplit - 1) / p.nsplit;
  c = (c + kTileKeys - 1) / kTileKeys * kTileKeys;
  t0 = a + min(L, s * c);
  t1 = a + min(L, (s + 1) * c);
}

// Shared-memory layout of one stage (K then V, 16 keys each):
//  - contiguous prefix: TMA tiles with 128-byte swizzling, [D/64][HB][key][64];
//  - paged prefix: one bulk copy per key of its HB heads (HB*D*2 bytes), rows
//    padded by 16 bytes so the 8 rows an ldmatrix reads fall in distinct banks.
// Producer warps of the paged layout: bulk copies issued by the lanes of one
// warp go out one after another, so the keys of a tile are spread over
// several warps (each fills kTileKeys / kPagedProducers keys, K and V).
constexpr int kPagedProducers = 4;

template <bool PAGED>
__host__ __device__ constexpr int producer_warps() { return PAGED ? kPagedProducers : 1; }

template <int D, bool PAGED>
__device__ __forceinline__ uint32_t kv_row_stride(int HB) {
  return PAGED ? uint32_t(HB) * D * 2 + 16 : 0u;
}

template <int D, bool PAGED>
__host__ __device__ constexpr uint32_t stage_kv_bytes(int HB) {
  return PAGED ? uint32_t(kTileKeys) * (uint32_t(HB) * D * 2 + 16)
               : uint32_t(D / 64) * HB * kTileKeys * 128;
}

template <int D, bool PAGED>
__global__ void __launch_bounds__((max_consumer_warps(D) + producer_warps<PAGED>()) * 32, 1)
    verify_stage1_kernel(const __grid_constant__ CUtensorMap tmap_k,
                         const __grid_constant__ CUtensorMap tmap_v, Stage1Params p) {
  constexpr int KSTEPS = D / 16;  // MMA k-steps over the head dimension
  constexpr int NPART = D / 64;   // 128-byte swizzle atoms across the head dimension
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  __shared__ int abort_flag;

  const int NW = p.HB * p.MT;
  const uint32_t head_bytes = kTileKeys * 128;                // one head, one part
  const uint32_t kv_bytes = stage_kv_bytes<D, PAGED>(p.HB);    // K (or V) per stage
  const uint32_t stage_bytes = 2 * kv_bytes;
  const uint32_t row_stride = kv_row_stride<D, PAGED>(p.HB);   // paged layout only
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + p.nstage * stage_bytes);
  uint64_t* empty = full + p.nstage;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    abort_flag = 0;
    for (int i = 0; i < p.nstage; ++i) {
      // one arrival with the byte count per producer warp
      mbar_init(&full[i], producer_warps<PAGED>());
      mbar_init(&empty[i], NW);
    }
    fence_barrier_init();
  }
  __syncthreads();

  const int units = p.B * p.nsplit * p.nrb * p.nhb;

  if (warp >= NW) {
    // ------------------------------------------------------------ producer
    if constexpr (PAGED) {
      // Paged prefix: producer warp pw fills keys [pw*TPW, (pw+1)*TPW) of
      // each tile; its lane l < TPW copies key l's K row, lane TPW + l its V
      // row (the key's HB heads, one bulk copy).  A key past the split end,
      // or a cache row outside [0, ntok) (reported), is written as zeros.
      constexpr int TPW = kTileKeys / kPagedProducers;
      const int pw = warp - NW;
      const bool active = lane < 2 * TPW;
      const int tok = pw * TPW + lane % TPW;
      const bool is_v = (lane / TPW) & 1;
      const uint32_t row_bytes = uint32_t(p.HB) * D * 2;
      const __nv_bfloat16* cache = is_v ? p.vc : p.kc;
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      int last_phase[8];
      for (int i = 0; i < 8; ++i) last_phase[i] = -1;
      for (int u = blockIdx.x; u < units && ok; u += gridDim.x) {
        const Unit x = decode_unit(p, u);
        int q0, Lb;
        request_rows(p.qo_indptr, p.Ld, p.nrows, x.b, q0, Lb, p.status);
        if (!unit_live(p, x, Lb)) continue;
        int32_t t0, t1;
        split_range(p, x.b, x.s, t0, t1);
        // The page-table entries are read kPrefetch tiles ahead, so a
        // stage's copies never wait on the latency of its own lookups.
        constexpr int kPrefetch = 8;
        int32_t cur[kPrefetch], nxt[kPrefetch];
        auto lookup = [&](int32_t tb, int32_t (&dst)[kPrefetch]) {
#pragma unroll
          for (int k = 0; k < kPrefetch; ++k) {
            const int32_t pos = tb + k * kTileKeys + tok;
            dst[k] = pos < t1 ? __ldg(p.kv_indices + pos) : -1;
          }
        };
        lookup(t0, cur);
        for (int32_t tb = t0; tb < t1 && ok; tb += kPrefetch * kTileKeys) {
          if (tb + kPrefetch * kTileKeys < t1) lookup(tb + kPrefetch * kTileKeys, nxt);
#pragma unroll
          for (int k = 0; k < kPrefetch; ++k) {
            if (tb + k * kTileKeys >= t1) break;
            // every lane acquires the released stage before writing into it
            const bool w = mbar_wait(&empty[stage], phase ^ 1, &abort_flag, p.status);
            if (!__all_sync(0xffffffffu, w)) {
              ok = false;
              break;
            }
            last_phase[stage] = int(phase);
            int32_t slot = cur[k];
            if (slot >= p.ntok || (slot < 0 && tb + k * kTileKeys + tok < t1)) {
              report_status(p.status, PSA_ERR_INVALID_ARG);
              slot = -1;
            }
            uint8_t* dst =
                smem + stage * stage_bytes + (is_v ? kv_bytes : 0u) + tok * row_stride;
            if (active && slot < 0) {
              const uint4 z = make_uint4(0u, 0u, 0u, 0u);
              for (uint32_t o = 0; o < row_bytes; o += 16)
                *reinterpret_cast<uint4*>(dst + o) = z;
              fence_proxy_async_smem();  // later bulk copies land after these stores
            }
            // one arrival per warp announces the bytes of all its copies,
            // before any of them is issued
            const uint32_t copies = __popc(__ballot_sync(0xffffffffu, active && slot >= 0));
            if (lane == 0) mbar_arrive_expect_tx(&full[stage], copies * row_bytes);
            __syncwarp();
            if (active && slot >= 0)
              bulk_load(dst, cache + (size_t(slot) * p.Hkv + x.hb * p.HB) * D, row_bytes,
                        &full[stage]);
            if (++stage == p.nstage) {
              stage = 0;
              phase ^= 1;
            }
          }
#pragma unroll
          for (int k = 0; k < kPrefetch; ++k) cur[k] = nxt[k];
        }
      }
      if (!ok && lane == 0 && pw == 0) {
        // Let copies already in flight land before the CTA exits.
        for (int i = 0; i < p.nstage; ++i) {
          if (last_phase[i] < 0) continue;
          const uint64_t w0 = globaltimer();
          while (!mbar_try_wait(&full[i], uint32_t(last_phase[i])) &&
                 globaltimer() - w0 < kWaitTimeoutNs) {
          }
        }
      }
    } else if (lane == 0) {
      tma_prefetch_desc(&tmap_k);
      tma_prefetch_desc(&tmap_v);
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      int last_phase[8];
      for (int i = 0; i < 8; ++i) last_phase[i] = -1;
      for (int u = blockIdx.x; u < units && ok; u += gridDim.x) {
        const Unit x = decode_unit(p, u);
        const int hb = x.hb;
        int q0, Lb;
        request_rows(p.qo_indptr, p.Ld, p.nrows, x.b, q0, Lb, nullptr);
        if (!unit_live(p, x, Lb)) continue;
        int32_t t0, t1;
        split_range(p, x.b, x.s, t0, t1);
        for (int32_t t = t0; t < t1; t += kTileKeys) {
          if (!mbar_wait(&empty[stage], phase ^ 1, &abort_flag, p.status)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full[stage], stage_bytes);
          last_phase[stage] = int(phase);
          uint8_t* kdst = smem + stage * stage_bytes;
          uint8_t* vdst = kdst + kv_bytes;
#pragma unroll
          for (int part = 0; part < NPART; ++part) {
            tma_load_3d(kdst + part * p.HB * head_bytes, &tmap_k, &full[stage], part * 64, t,
                        hb * p.HB);
            tma_load_3d(vdst + part * p.HB * head_bytes, &tmap_v, &full[stage], part * 64, t,
                        hb * p.HB);
          }
          if (++stage == p.nstage) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      if (!ok) {
        // Let copies already in flight land before the CTA exits.
        for (int i = 0; i < p.nstage; ++i) {
          if (last_phase[i] < 0) continue;
          const uint64_t w0 = globaltimer();
          while (!mbar_try_wait(&full[i], uint32_t(last_phase[i])) &&
                 globaltimer() - w0 < kWaitTimeoutNs) {
          }
        }
      }
    }
    return;
  }

  // -------------------------------------------------------------- consumers
  const int hh = warp / p.MT;  // KV head within the block
  const int mt = warp % p.MT;  // 16-row m-tile of that head's rows
  const int g = lane >> 2, c = lane & 3;
  const int BL = p.nrows;
  int stage = 0;
  uint32_t phase = 0;

  for (int u = blockIdx.x; u < units; u += gridDim.x) {
    const Unit x = decode_unit(p, u);
    const int b = x.b, s = x.s;
    const int kvh = x.hb * p.HB + hh;
    int q0, Lb;
    request_rows(p.qo_indptr, p.Ld, p.nrows, b, q0, Lb, nullptr);
    if (!unit_live(p, x, Lb)) continue;
    int32_t t0, t1;
    split_range(p, b, s, t0, t1);

    // rows of this thread: g and g + 8 of the m-tile
    int rrow[2], rqh[2];
    bool rvalid[2];
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const int rr = (x.rb * p.MT + mt) * 16 + g + 8 * i;
      rvalid[i] = rr < Lb * p.G;
      const int j = rvalid[i] ? rr / p.G : 0;
      rqh[i] = kvh * p.G + (rvalid[i] ? rr % p.G : 0);
      rrow[i] = q0 + j;
    }

    // Q fragments for every k-step (A operand, row-major 16x16 per step)
    uint32_t qa[KSTEPS][4];
    {
      const __nv_bfloat16* q0 = p.q + (size_t(rrow[0]) * p.Hq + rqh[0]) * D;
      const __nv_bfloat16* q1 = p.q + (size_t(rrow[1]) * p.Hq + rqh[1]) * D;
#pragma unroll
      for (int ks = 0; ks < KSTEPS; ++ks) {
        const int col = ks * 16 + 2 * c;
        qa[ks][0] = rvalid[0] ? __ldg(reinterpret_cast<const uint32_t*>(q0 + col)) : 0u;
        qa[ks][1] = rvalid[1] ? __ldg(reinterpret_cast<const uint32_t*>(q1 + col)) : 0u;
        qa[ks][2] = rvalid[0] ? __ldg(reinterpret_cast<const uint32_t*>(q0 + col + 8)) : 0u;
        qa[ks][3] = rvalid[1] ? __ldg(reinterpret_cast<const uint32_t*>(q1 + col + 8)) : 0u;
      }
    }

    float acc[D / 8][4];
#pragma unroll
    for (int i = 0; i < D / 8; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
    float m_run[2] = {-INFINITY, -INFINITY};
    float l_run[2] = {0.f, 0.f};
    bool ok = true;

    for (int32_t t = t0; t < t1; t += kTileKeys) {
      if (!mbar_wait(&full[stage], phase, &abort_flag, p.status)) {
        ok = false;
        break;
      }
      const uint32_t kbase =
          smem_u32(smem + stage * stage_bytes) + hh * (PAGED ? uint32_t(D) * 2 : head_bytes);
      const uint32_t vbase = kbase + kv_bytes;
      // byte address of 16-byte chunk `chunk` of key `key` in a K or V tile
      auto at = [&](uint32_t base, uint32_t key, uint32_t chunk) {
        return PAGED ? base + key * row_stride + chunk * 16
                     : base + (chunk >> 3) * (p.HB * head_bytes) + sw128(key, chunk & 7);
      };

      // S = Q K^T over 16 keys: two n-tiles of 8 keys
      float sc[2][4];
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        sc[nt][0] = sc[nt][1] = sc[nt][2] = sc[nt][3] = 0.f;
        const uint32_t key = nt * 8 + (lane & 7);
#pragma unroll
        for (int ks = 0; ks < KSTEPS; ks += 2) {
          const uint32_t chunk = ks * 2 + (lane >> 3);  // 16-byte chunk of the head dim
          const uint32_t addr = at(kbase, key, chunk);
          uint32_t b0, b1, b2, b3;
          ldmatrix_x4(addr, b0, b1, b2, b3);
          mma_bf16_16816(sc[nt], qa[ks], b0, b1);
          mma_bf16_16816(sc[nt], qa[ks + 1], b2, b3);
        }
      }

      // online softmax in the log2 domain; keys past the split end are masked
      float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int32_t key = t + nt * 8 + 2 * c + (e & 1);
          float v = sc[nt][e] * p.scale_log2;
          v = key < t1 ? v : -INFINITY;
          sc[nt][e] = v;
          mx[e >> 1] = fmaxf(mx[e >> 1], v);
        }
      float alpha[2];
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        mx[i] = fmaxf(mx[i], __shfl_xor_sync(0xffffffffu, mx[i], 1));
        mx[i] = fmaxf(mx[i], __shfl_xor_sync(0xffffffffu, mx[i], 2));
        const float mn = fmaxf(m_run[i], mx[i]);
        alpha[i] = fast_exp2(m_run[i] - mn);
        m_run[i] = mn;
      }
      float ps[2][4];
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) ps[nt][e] = fast_exp2(sc[nt][e] - m_run[e >> 1]);
      l_run[0] = l_run[0] * alpha[0] + ps[0][0] + ps[0][1] + ps[1][0] + ps[1][1];
      l_run[1] = l_run[1] * alpha[1] + ps[0][2] + ps[0][3] + ps[1][2] + ps[1][3];
#pragma unroll
      for (int i = 0; i < D / 8; ++i) {
        acc[i][0] *= alpha[0];
        acc[i][1] *= alpha[0];
        acc[i][2] *= alpha[1];
        acc[i][3] *= alpha[1];
      }

      // O += P V: P as the A operand (16 rows x 16 keys), V^T via ldmatrix.trans
      uint32_t pa[4];
      pa[0] = pack_bf16(ps[0][0], ps[0][1]);
      pa[1] = pack_bf16(ps[0][2], ps[0][3]);
      pa[2] = pack_bf16(ps[1][0], ps[1][1]);
      pa[3] = pack_bf16(ps[1][2], ps[1][3]);
      {
        const int mi = lane >> 3;
        const uint32_t key = (mi & 1) * 8 + (lane & 7);
#pragma unroll
        for (int dt = 0; dt < D / 8; dt += 2) {
          const uint32_t chunk = dt + (mi >> 1);
          const uint32_t addr = at(vbase, key, chunk);
          uint32_t b0, b1, b2, b3;
          ldmatrix_x4_trans(addr, b0, b1, b2, b3);
          mma_bf16_16816(acc[dt], pa, b0, b1);
          mma_bf16_16816(acc[dt + 1], pa, b2, b3);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[stage]);
      if (++stage == p.nstage) {
        stage = 0;
        phase ^= 1;
      }
    }
    if (!ok) return;

    // normalise and write this split's partial
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      l_run[i] += __shfl_xor_sync(0xffffffffu, l_run[i], 1);
      l_run[i] += __shfl_xor_sync(0xffffffffu, l_run[i], 2);
    }
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      if (!rvalid[i]) continue;
      const float inv = l_run[i] > 0.f ? 1.f / l_run[i] : 0.f;
      const size_t prow = (size_t(s) * BL + rrow[i]) * p.Hq + rqh[i];
      float* dst = p.part_o + prow * D;
#pragma unroll
      for (int dt = 0; dt < D / 8; ++dt) {
        float2 v = make_float2(acc[dt][2 * i] * inv, acc[dt][2 * i + 1] * inv);
        *reinterpret_cast<float2*>(dst + dt * 8 + 2 * c) = v;
      }
      if (c == 0)
        p.part_lse[prow] = l_run[i] > 0.f ? m_run[i] + __log2f(l_run[i]) : -INFINITY;
    }
  }
}

struct Stage2Params {
  const __nv_bfloat16* q;
  const __nv_bfloat16* kd;
  const __nv_bfloat16* vd;
  const float* part_o;
  const float* part_lse;
  __nv_bfloat16* o;
  float* lse;
  const uint8_t* dmask;  // nullable: causal draft block; else a tree mask per request
  const int32_t* qo_indptr;    // nullable: request b's draft rows are b*Ld + [0, Ld)
  const int32_t* mask_indptr;  // nullable: request b's mask starts at b*Ld*Ld
  int32_t B, Ld, Hq, Hkv, G, nsplit, nrows;
  float scale_log2;
  int32_t* status;
};

template <int D>
__global__ void __launch_bounds__(256) verify_stage2_kernel(Stage2Params p) {
  constexpr int E = D / 32;  // head-dim elements per lane
  const int gw = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const int BL = p.nrows;
  if (gw >= BL * p.Hq) return;
  const int row = gw / p.Hq, qh = gw % p.Hq;
  int b;
  if (p.qo_indptr) {
    // the last request whose first row is <= row (empty requests are passed over)
    int lo = 0, hi = p.B;
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (__ldg(p.qo_indptr + mid) <= row) lo = mid; else hi = mid;
    }
    b = lo;
  } else {
    b = row / p.Ld;
  }
  int q0, Lb;
  request_rows(p.qo_indptr, p.Ld, p.nrows, b, q0, Lb, lane == 0 ? p.status : nullptr);
  const int j = row - q0;
  if (j >= Lb) return;  // only after a reported inconsistent qo_indptr
  const int kvh = qh / p.G;

  float qv[E];
  {
    const __nv_bfloat16* qp = p.q + (size_t(row) * p.Hq + qh) * D + lane * E;
#pragma unroll
    for (int e = 0; e < E; ++e) qv[e] = __bfloat162float(qp[e]);
  }

  // draft keys 0..j (the causal draft-draft block), log2-domain logits
  auto draft_logit = [&](int i) {
    const __nv_bfloat16* kp = p.kd + (size_t(q0 + i) * p.Hkv + kvh) * D + lane * E;
    float sdot = 0.f;
#pragma unroll
    for (int e = 0; e < E; ++e) sdot += qv[e] * __bfloat162float(kp[e]);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) sdot += __shfl_xor_sync(0xffffffffu, sdot, off);
    return sdot * p.scale_log2;
  };
  // the draft block: drafts 0..j, or the tree mask's row (the same for every head)
  const uint8_t* mrow = nullptr;
  bool mask_ok = true;
  if (p.dmask) {
    const int64_t moff = p.mask_indptr ? int64_t(__ldg(p.mask_indptr + b)) : int64_t(q0) * Lb;
    // debug build: request b's Lb x Lb block must lie inside the mask, whose
    // length is mask_indptr[B]; otherwise no draft is seen
    mask_ok = psa_in_bounds(!p.mask_indptr || (moff >= 0 && moff + int64_t(Lb) * Lb <=
                                                                 __ldg(p.mask_indptr + p.B)),
                            lane == 0 ? p.status : nullptr);
    mrow = p.dmask + size_t(moff) + size_t(j) * Lb;
  }
  auto sees = [&](int i) { return mrow ? __ldg(mrow + i) != 0 : i <= j; };
  const int nd = !mask_ok ? 0 : mrow ? Lb : j + 1;
  // The draft logits, computed once: lane i keeps draft i's (nd <= 16).
  float M = -INFINITY, dlog = -INFINITY;
  for (int i = 0; i < nd; ++i) {
    if (!sees(i)) continue;
    const float l = draft_logit(i);
    if (lane == i) dlog = l;
    M = fmaxf(M, l);
  }
  // The splits' LSEs, all loaded up front: split s sits in lane s % 32 of
  // slot s / 32 (nsplit <= 256), so the combine below waits on no load to
  // learn a weight.
  constexpr int kSlots = 8;
  float lsv[kSlots];
#pragma unroll
  for (int k = 0; k < kSlots; ++k) {
    const int s = k * 32 + lane;
    lsv[k] = s < p.nsplit ? p.part_lse[(size_t(s) * BL + row) * p.Hq + qh] : -INFINITY;
    M = fmaxf(M, lsv[k]);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
  if (M == -INFINITY) {
    // no visible key (an empty prefix and an empty tree-mask row)
    __nv_bfloat16* op = p.o + (size_t(row) * p.Hq + qh) * D + lane * E;
#pragma unroll
    for (int e = 0; e < E; ++e) op[e] = __float2bfloat16(0.f);
    if (p.lse && lane == 0) p.lse[size_t(row) * p.Hq + qh] = -INFINITY;
    return;
  }

  float acc[E];
#pragma unroll
  for (int e = 0; e < E; ++e) acc[e] = 0.f;
  float wsum = 0.f;  // this lane's splits; summed over the warp below
  // Partial O rows, four splits per step: the weights come from the
  // registers above by shuffle and the four loads are in flight together.
  // An empty split (LSE -inf, weight 0) is not read.
#pragma unroll
  for (int k = 0; k < kSlots; ++k) {
    if (k * 32 >= p.nsplit) break;
    const float wk = fast_exp2(lsv[k] - M);  // empty or absent split: exp2(-inf) = 0
    wsum += wk;
    const int nj = min(32, p.nsplit - k * 32);
    for (int j0 = 0; j0 < nj; j0 += 4) {
      float w[4];
      float v[4][E];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int jj = j0 + u;
        w[u] = __shfl_sync(0xffffffffu, wk, jj & 31);
        if (jj >= nj) w[u] = 0.f;
        const size_t prow = (size_t(k * 32 + jj) * BL + row) * p.Hq + qh;
        const float* op = p.part_o + prow * D + lane * E;
#pragma unroll
        for (int e = 0; e < E; e += 2) {
          float2 x = make_float2(0.f, 0.f);
          if (w[u] != 0.f) x = *reinterpret_cast<const float2*>(op + e);
          v[u][e] = x.x;
          v[u][e + 1] = x.y;
        }
      }
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int e = 0; e < E; ++e) acc[e] += w[u] * v[u][e];
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) wsum += __shfl_xor_sync(0xffffffffu, wsum, off);
  for (int i = 0; i < nd; ++i) {
    if (!sees(i)) continue;
    const float w = fast_exp2(__shfl_sync(0xffffffffu, dlog, i) - M);
    const __nv_bfloat16* vp = p.vd + (size_t(q0 + i) * p.Hkv + kvh) * D + lane * E;
#pragma unroll
    for (int e = 0; e < E; ++e) acc[e] += w * __bfloat162float(vp[e]);
    wsum += w;
  }
  const float inv = wsum > 0.f ? 1.f / wsum : 0.f;  // no visible key at all: O = 0
  __nv_bfloat16* op = p.o + (size_t(row) * p.Hq + qh) * D + lane * E;
#pragma unroll
  for (int e = 0; e < E; e += 2)
    *reinterpret_cast<__nv_bfloat162*>(op + e) = __floats2bfloat162_rn(acc[e] * inv, acc[e + 1] * inv);
  if (p.lse && lane == 0)
    p.lse[size_t(row) * p.Hq + qh] = wsum > 0.f ? (M + __log2f(wsum)) * kLn2 : -INFINITY;
}

template <int D>
int launch_verify_d(const VerifyArgs& a, int HB, int MT, int NRB) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return PSA_ERR_CUDA;
  const int G = a.Hq / a.Hkv;
  const int R = a.Ld * G;
  const int nhb = a.Hkv / HB;

  CUtensorMap tk, tv;
  // a tensor map needs a non-empty extent (an empty cache is never read)
  const uint64_t rows = a.n_cache_tokens > 0 ? uint64_t(a.n_cache_tokens) : 1u;
  const uint64_t dims[3] = {uint64_t(D), rows, uint64_t(a.Hkv)};
  const uint64_t strides[2] = {uint64_t(a.Hkv) * D * 2, uint64_t(D) * 2};
  const uint32_t box[3] = {64u, uint32_t(kTileKeys), uint32_t(HB)};
  int rc = encode_tmap(&tk, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, a.kc, dims, strides, box,
                       CU_TENSOR_MAP_SWIZZLE_128B);
  if (rc != PSA_OK) return rc;
  rc = encode_tmap(&tv, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, a.vc, dims, strides, box,
                   CU_TENSOR_MAP_SWIZZLE_128B);
  if (rc != PSA_OK) return rc;

  Stage1Params p1;
  p1.q = static_cast<const __nv_bfloat16*>(a.q);
  p1.indptr = a.indptr;
  p1.kv_indices = a.kv_indices;
  p1.kc = static_cast<const __nv_bfloat16*>(a.kc);
  p1.vc = static_cast<const __nv_bfloat16*>(a.vc);
  p1.ntok = a.n_cache_tokens;
  p1.qo_indptr = a.qo_indptr;
  p1.nrows = a.qo_indptr ? a.n_rows : a.B * a.Ld;
  p1.part_o = a.part_o;
  p1.part_lse = a.part_lse;
  p1.B = a.B;
  p1.Ld = a.Ld;
  p1.Hq = a.Hq;
  p1.Hkv = a.Hkv;
  p1.G = G;
  p1.R = R;
  p1.MT = MT;
  p1.nrb = NRB;
  p1.HB = HB;
  p1.nhb = nhb;
  p1.nsplit = a.nsplit;
  p1.scale_log2 = a.scale * kLog2e;
  p1.status = a.status;

  const bool paged = a.kv_indices != nullptr;
  const size_t stage_bytes =
      size_t(2) * (paged ? stage_kv_bytes<D, true>(HB) : stage_kv_bytes<D, false>(HB));
  const size_t budget = 200 * 1024;
  int nstage = int(budget / stage_bytes);
  nstage = nstage > 8 ? 8 : nstage;
  if (nstage < 2) return PSA_ERR_UNSUPPORTED;
  p1.nstage = nstage;
  const size_t smem = 1024 + nstage * stage_bytes + 2 * nstage * sizeof(uint64_t);
  auto k1 = paged ? verify_stage1_kernel<D, true> : verify_stage1_kernel<D, false>;
  if (cudaFuncSetAttribute(k1, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)) !=
      cudaSuccess)
    return PSA_ERR_CUDA;
  const int units = a.B * a.nsplit * NRB * nhb;
  int grid = sm_count(dev);
  if (grid <= 0) return PSA_ERR_CUDA;
  grid = units < grid ? units : grid;
  const int threads = (HB * MT + (paged ? producer_warps<true>() : 1)) * 32;
  if (units > 0) {
    k1<<<grid, threads, smem, a.stream>>>(tk, tv, p1);
    if (cudaGetLastError() != cudaSuccess) return PSA_ERR_CUDA;
  }
  return launch_combine_d<D>(a);
}

}  // namespace

// Stage 2 on its own: merge the split partials of a.part_o / a.part_lse with
// the causal draft block (shared with the shared-prefix verify).
template <int D>
int launch_combine_d(const VerifyArgs& a) {
  const int G = a.Hq / a.Hkv;
  Stage2Params p2;
  p2.q = static_cast<const __nv_bfloat16*>(a.q);
  p2.kd = static_cast<const __nv_bfloat16*>(a.kd);
  p2.vd = static_cast<const __nv_bfloat16*>(a.vd);
  p2.part_o = a.part_o;
  p2.part_lse = a.part_lse;
  p2.o = static_cast<__nv_bfloat16*>(a.o);
  p2.lse = a.lse;
  p2.dmask = a.dmask;
  p2.qo_indptr = a.qo_indptr;
  p2.mask_indptr = a.mask_indptr;
  p2.nrows = a.qo_indptr ? a.n_rows : a.B * a.Ld;
  p2.status = a.status;
  p2.B = a.B;
  p2.Ld = a.Ld;
  p2.Hq = a.Hq;
  p2.Hkv = a.Hkv;
  p2.G = G;
  p2.nsplit = a.nsplit;
  p2.scale_log2 = a.scale * kLog2e;
  const int warps = p2.nrows * a.Hq;
  const int blocks = (warps + 7) / 8;
  if (blocks > 0) {
    verify_stage2_kernel<D><<<blocks, 256, 0, a.stream>>>(p2);
    if (cudaGetLastError() != cudaSuccess) return PSA_ERR_CUDA;
  }
  return PSA_OK;
}

int launch_verify_combine(const VerifyArgs& a) {
  switch (a.D) {
    case 64:
      return launch_combine_d<64>(a);
    case 128:
      return launch_combine_d<128>(a);
    case 256:
      return launch_combine_d<256>(a);
    default:
      return PSA_ERR_UNSUPPORTED;
  }
}

int verify_plan(int32_t Ld, int32_t Hq, int32_t Hkv, int32_t D, int32_t* heads_per_block,
                int32_t* mtiles, int32_t* row_blocks) {
  if (Hkv <= 0 || Hq % Hkv != 0 || Ld <= 0 || Ld > 16) return 0;
  if (D != 64 && D != 128 && D != 256) return 0;
  const int R = Ld * (Hq / Hkv);
  if (R > 128) return 0;
  const int MT = (R + 15) / 16;
  const int maxw = max_consumer_warps(D);
  if (MT > maxw) {
    // one KV head per CTA; its m-tiles are spread over several CTAs
    *heads_per_block = 1;
    *mtiles = maxw;
    *row_blocks = (MT + maxw - 1) / maxw;
    return 1;
  }
  // largest divisor of Hkv that fits the warp budget and a <= 64 KB stage
  int best = 0;
  for (int hb = 1; hb <= Hkv; ++hb) {
    if (Hkv % hb) continue;
    if (hb * MT > maxw) continue;
    if (size_t(2) * (D / 64) * hb * kTileKeys * 128 > 64 * 1024) continue;
    best = hb;
  }
  if (!best) return 0;
  *heads_per_block = best;
  *mtiles = MT;
  *row_blocks = 1;
  return 1;
}

int launch_verify(const VerifyArgs& a) {
  int HB = 0, MT = 0, NRB = 0;
  if (!verify_plan(a.Ld, a.Hq, a.Hkv, a.D, &HB, &MT, &NRB)) return PSA_ERR_UNSUPPORTED;
  switch (a.D) {
    case 64:
      return launch_verify_d<64>(a, HB, MT, NRB);
    case 128:
      return launch_verify_d<128>(a, HB, MT, NRB);
    case 256:
      return launch_verify_d<256>(a, HB, MT, NRB);
    default:
      return PSA_ERR_UNSUPPORTED;
  }
}

}  // namespace psa

// ---------------------------------------------------------------------------
// Verify without a caller workspace: the partials live in a fixed file-scope
// device array.  Host code cannot use the array's name as a device address,
// so every call looks the address up in the context that is current for the
// call.  The lookup allocates nothing and costs little; caching it per device
// ordinal would hand a stale address to a caller that switched contexts on
// the same device (a driver-API context of its own, or a context rebuilt
// after cudaDeviceReset), and the kernels would then fault.

namespace psa {
namespace {

static __device__ __align__(256) uint8_t g_verify_scratch[PSA_VERIFY_NOALLOC_SCRATCH_BYTES];

int scratch_address(void** out) {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_verify_scratch) != cudaSuccess || !p) {
    (void)cudaGetLastError();
    return PSA_ERR_CUDA;
  }
  *out = p;
  return PSA_OK;
}

}  // namespace
}  // namespace psa

extern "C" int psa_verify_fwd_noalloc(const void* q_draft, const void* k_draft,
                                      const void* v_draft, const void* k_cache,
                                      const void* v_cache, int64_t n_cache_tokens,
                                      const int32_t* dev_kv_indptr, int64_t max_prefix_len,
                                      const int32_t* kv_indices, void* o, float* lse, int32_t B,
                                      int32_t Ld, int32_t Hq, int32_t Hkv, int32_t head_dim,
                                      float scale, int32_t nsplit,
                                      const psa_verify_features* features, int32_t* dev_status,
                                      void* stream) {
  int32_t ns = nsplit;
  if (ns == 0 && B > 0) ns = psa_verify_auto_splits(B, max_prefix_len, Hkv, head_dim);
  if (B > 0 && ns >= 1 && ns <= 256 &&
      psa_verify_workspace_size(B, Ld, Hq, head_dim, ns) > PSA_VERIFY_NOALLOC_SCRATCH_BYTES)
    return PSA_ERR_WORKSPACE;
  void* scratch = nullptr;
  const int rc = psa::scratch_address(&scratch);
  if (rc != PSA_OK) return rc;
  return psa_verify_fwd(q_draft, k_draft, v_draft, k_cache, v_cache, n_cache_tokens,
                        dev_kv_indptr, max_prefix_len, kv_indices, o, lse, B, Ld, Hq, Hkv,
                        head_dim, scale, ns, features, scratch, PSA_VERIFY_NOALLOC_SCRATCH_BYTES,
                        dev_status, stream);
}
