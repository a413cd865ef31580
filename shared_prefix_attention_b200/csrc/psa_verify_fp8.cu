// Split-KV verify over an fp8 (e4m3) prefix cache with per-tensor scales
// ("Split-KV flash-decode attention for EAGLE target-verify", sglang PR
// #27382: implementation item 1 -- stage 1 streams the cached prefix in
// chunks and applies the fp8 scales k_scale / v_scale; stage 2 merges the
// chunks with the causal draft block by LSE weight).  A cached key stands for
// k_scale * e4m3 and a cached value for v_scale * e4m3; draft keys and values
// are bf16 and unscaled.
//
// The prefix is HBM-bound, so one byte per element halves the traffic of the
// bf16 stream.  Stage 1 keeps the bf16 kernel's shape (TMA ring of 16-key
// tiles of a group of KV heads, one producer warp, one consumer warp per
// (KV head, 16-row m-tile) doing warp-level MMAs) with three changes:
//   - the ring holds e4m3 tiles (128 bytes per key and head, 128-byte
//     swizzle);
//   - each consumer warp reads its K fragments straight from the e4m3 tile
//     (two bytes per register, widened to f16 in registers, exact for e4m3)
//     and widens its head's V tile into a private f16 tile laid out like the
//     bf16 path's, so ldmatrix.trans can feed the PV warp MMAs;
//   - k_scale is folded into the logit scale and v_scale into the partial
//     output, so the inner loop never multiplies by a scale.
// Q is widened from bf16 to f16 for the f16 MMAs (exact for |q| < 65504 and
// above the f16 subnormal range) and P is rounded to f16 (finer than bf16).
// Stage 2 is the bf16 verify's combine kernel, unchanged.
// The same kernel serves the verify entry's other forms: a paged prefix (the
// PAGED instantiation gathers each key's e4m3 row with a bulk copy into a
// padded row layout) and ragged draft counts (units whose rows are all past
// their request's count are skipped); tree masks live in the combine.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "psa_debug.cuh"
#include "psa_device.cuh"
#include "psa_internal.h"

namespace psa {
namespace {

constexpr int D8 = 128;           // head dim of the fp8 path (one swizzle atom of bytes)
constexpr int kKeys = 16;         // keys per ring stage
constexpr int kMaxWarps = 8;      // consumer warps per CTA
constexpr uint32_t kHeadTile8 = kKeys * D8;        // e4m3 bytes of one head's K (or V) tile
constexpr uint32_t kPrivBytes = 2 * kKeys * 128;  // f16 V tile, two d-parts

struct P8Params {
  const __nv_bfloat16* q;  // [B*Ld, Hq, D]
  const int32_t* indptr;   // [B+1]
  // Page table (paged instantiation only): prefix position t is cache row
  // kv_indices[t], gathered with one bulk copy per key.
  const int32_t* kv_indices;
  const uint8_t* kc8;      // [ntok, Hkv, 128] e4m3
  const uint8_t* vc8;
  int64_t ntok;
  float* part_o;
  float* part_lse;
  // Extend form (nullable): request b's draft rows are [qo_indptr[b],
  // qo_indptr[b+1]); Ld is then the largest draft count, nrows the total.
  const int32_t* qo_indptr;
  int32_t nrows;
  int32_t B, Ld, Hq, Hkv, G, R;
  int32_t MT, nrb, HB, nhb, nsplit, nstage;
  float logit_scale_log2;  // scale * k_scale * log2(e)
  float v_scale;
  int32_t* status;
};

struct Unit8 {
  int b, s, rb, hb;
};

__device__ __forceinline__ Unit8 decode_unit8(const P8Params& p, int u) {
  Unit8 x;
  x.hb = u % p.nhb;
  u /= p.nhb;
  x.rb = u % p.nrb;
  u /= p.nrb;
  x.s = u % p.nsplit;
  x.b = u / p.nsplit;
  return x;
}

// First draft row and draft count of request b (a count above Ld is
// reported and clamped; rows outside [0, nrows) empty the request).
__device__ __forceinline__ void request_rows8(const P8Params& p, int b, int& q0, int& Lb,
                                              int32_t* status) {
  if (!p.qo_indptr) {
    q0 = b * p.Ld;
    Lb = p.Ld;
    return;
  }
  q0 = __ldg(p.qo_indptr + b);
  Lb = __ldg(p.qo_indptr + b + 1) - q0;
  if (Lb > p.Ld) {
    report_status(status, PSA_ERR_INVALID_ARG);
    Lb = p.Ld;
  }
  if (Lb < 0 || q0 < 0 || q0 > p.nrows - Lb) {
    report_status(status, PSA_ERR_INVALID_ARG);
    Lb = 0;
  }
}

// A unit does work only if its row block holds a draft row of the request.
__device__ __forceinline__ bool unit_live8(const P8Params& p, const Unit8& x, int Lb) {
  return x.rb * p.MT * 16 < Lb * p.G;
}

__device__ __forceinline__ void split_range8(const P8Params& p, int b, int s, int32_t& t0,
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
  c = (c + kKeys - 1) / kKeys * kKeys;
  t0 = a + min(L, s * c);
  t1 = a + min(L, (s + 1) * c);
}

__device__ __forceinline__ void mma_f16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                              uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
      "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Two e4m3 values (low byte -> low half) widened to an f16 pair; exact.
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t two) {
  uint32_t r;
  asm("{\n\t.reg .b16 t;\n\tcvt.u16.u32 t, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, t;\n\t}"
      : "=r"(r)
      : "r"(two));
  return r;
}

__device__ __forceinline__ uint32_t bf16x2_to_f16x2(uint32_t v) {
  const float lo = __uint_as_float(v << 16), hi = __uint_as_float(v & 0xffff0000u);
  __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ uint32_t pack_f16(float lo, float hi) {
  __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

// Paged prefix: producer warps of the gathered layout (each fills
// kKeys / kPagedProducers8 keys, K and V, one bulk copy per key and tensor)
// and the byte address of 16-byte chunk `chunk` of key `key` in a K or V
// tile: 128-byte swizzled TMA tile [head][key][128], or rows of HB heads
// padded by 16 bytes (row stride rs) so an 8-key access hits 8 bank groups.
constexpr int kPagedProducers8 = 4;

template <bool PAGED>
__device__ __forceinline__ uint32_t tile_at(uint32_t base, uint32_t key, uint32_t chunk,
                                            uint32_t rs) {
  return PAGED ? base + key * rs + chunk * 16 : base + sw128(key, chunk);
}

// One lane widens 64 e4m3 values (half a key row) of an e4m3 tile into the
// f16 tile: key row `key`, d half `half` (d = 64 half .. 64 half + 63 is the
// f16 tile's d-part `half`).
template <bool PAGED>
__device__ __forceinline__ void widen_row(uint32_t src_tile, uint32_t dst_tile, int key,
                                          int half, uint32_t rs) {
  uint32_t w[16];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t addr = tile_at<PAGED>(src_tile, key, half * 4 + i, rs);
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(w[4 * i]), "=r"(w[4 * i + 1]), "=r"(w[4 * i + 2]), "=r"(w[4 * i + 3])
                 : "r"(addr));
  }
  const uint32_t part = dst_tile + half * (kKeys * 128);
#pragma unroll
  for (int ch = 0; ch < 8; ++ch) {
    // f16 chunk ch holds d = 8 ch .. 8 ch + 7 of this part: e4m3 bytes 8 ch .. 8 ch + 7
    const uint32_t lo = w[2 * ch], hi = w[2 * ch + 1];
    const uint32_t a0 = e4m3x2_to_f16x2(lo & 0xffffu), a1 = e4m3x2_to_f16x2(lo >> 16);
    const uint32_t a2 = e4m3x2_to_f16x2(hi & 0xffffu), a3 = e4m3x2_to_f16x2(hi >> 16);
    asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(part + sw128(key, ch)),
                 "r"(a0), "r"(a1), "r"(a2), "r"(a3)
                 : "memory");
  }
}

// Plain (untiled) bulk copy of `bytes` contiguous global bytes into shared
// memory, completing on `bar`'s transaction count (16-byte multiples).
__device__ __forceinline__ void bulk_load8(void* dst, const void* src, uint32_t bytes,
                                           uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
      ::"r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

template <bool PAGED>
__global__ void __launch_bounds__((kMaxWarps + (PAGED ? kPagedProducers8 : 1)) * 32, 1)
    verify_stage1_fp8_kernel(const __grid_constant__ CUtensorMap tmap_k,
                             const __grid_constant__ CUtensorMap tmap_v, P8Params p) {
  constexpr int KSTEPS = D8 / 16;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  __shared__ int abort_flag;

  const int NW = p.HB * p.MT;
  // K (or V) bytes per stage, and the paged layout's row stride
  const uint32_t rs = PAGED ? uint32_t(p.HB) * D8 + 16 : 0u;
  const uint32_t kv_bytes = PAGED ? kKeys * rs : uint32_t(p.HB) * kHeadTile8;
  const uint32_t stage_bytes = 2 * kv_bytes;
  uint8_t* priv = smem + p.nstage * stage_bytes;           // kPrivBytes per consumer warp
  uint64_t* full = reinterpret_cast<uint64_t*>(priv + NW * kPrivBytes);
  uint64_t* empty = full + p.nstage;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    abort_flag = 0;
    for (int i = 0; i < p.nstage; ++i) {
      // one arrival with the byte count per producer warp
      mbar_init(&full[i], PAGED ? kPagedProducers8 : 1);
      mbar_init(&empty[i], NW);
    }
    fence_barrier_init();
  }
  __syncthreads();

  const int units = p.B * p.nsplit * p.nrb * p.nhb;

  if (warp >= NW) {
    // ------------------------------------------------------------ producer
    if constexpr (PAGED) {
      // producer warp pw fills keys [pw*TPW, (pw+1)*TPW) of each tile: lane
      // l < TPW copies key l's K row, lane TPW + l its V row (HB heads); a key
      // past the split end, or a cache row outside [0, ntok) (reported), is
      // written as zeros.  Table entries are read eight tiles ahead.
      constexpr int TPW = kKeys / kPagedProducers8;
      const int pw = warp - NW;
      const bool active = lane < 2 * TPW;
      const int tok = pw * TPW + lane % TPW;
      const bool is_v = (lane / TPW) & 1;
      const uint32_t row_bytes = uint32_t(p.HB) * D8;
      const uint8_t* cache = is_v ? p.vc8 : p.kc8;
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      int last_phase[16];
      for (int i = 0; i < 16; ++i) last_phase[i] = -1;
      for (int u = blockIdx.x; u < units && ok; u += gridDim.x) {
        const Unit8 x = decode_unit8(p, u);
        int q0, Lb;
        request_rows8(p, x.b, q0, Lb, nullptr);
        if (!unit_live8(p, x, Lb)) continue;
        int32_t t0, t1;
        split_range8(p, x.b, x.s, t0, t1);
        constexpr int kPrefetch = 8;
        int32_t cur[kPrefetch], nxt[kPrefetch];
        auto lookup = [&](int32_t tb, int32_t (&dst)[kPrefetch]) {
#pragma unroll
          for (int k = 0; k < kPrefetch; ++k) {
            const int32_t pos = tb + k * kKeys + tok;
            dst[k] = pos < t1 ? __ldg(p.kv_indices + pos) : -1;
          }
        };
        lookup(t0, cur);
        for (int32_t tb = t0; tb < t1 && ok; tb += kPrefetch * kKeys) {
          if (tb + kPrefetch * kKeys < t1) lookup(tb + kPrefetch * kKeys, nxt);
#pragma unroll
          for (int k = 0; k < kPrefetch; ++k) {
            if (tb + k * kKeys >= t1) break;
            // every lane acquires the released stage before writing into it
            const bool w = mbar_wait(&empty[stage], phase ^ 1, &abort_flag, p.status);
            if (!__all_sync(0xffffffffu, w)) {
              ok = false;
              break;
            }
            last_phase[stage] = int(phase);
            int32_t slot = cur[k];
            if (slot >= p.ntok || (slot < 0 && tb + k * kKeys + tok < t1)) {
              report_status(p.status, PSA_ERR_INVALID_ARG);
              slot = -1;
            }
            uint8_t* dst = smem + stage * stage_bytes + (is_v ? kv_bytes : 0u) + tok * rs;
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
              bulk_load8(dst, cache + (size_t(slot) * p.Hkv + x.hb * p.HB) * D8, row_bytes,
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
      int last_phase[16];
      for (int i = 0; i < 16; ++i) last_phase[i] = -1;
      for (int u = blockIdx.x; u < units && ok; u += gridDim.x) {
        const Unit8 x = decode_unit8(p, u);
        int q0, Lb;
        request_rows8(p, x.b, q0, Lb, nullptr);
        if (!unit_live8(p, x, Lb)) continue;
        int32_t t0, t1;
        split_range8(p, x.b, x.s, t0, t1);
        for (int32_t t = t0; t < t1; t += kKeys) {
          if (!mbar_wait(&empty[stage], phase ^ 1, &abort_flag, p.status)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full[stage], stage_bytes);
          last_phase[stage] = int(phase);
          uint8_t* kdst = smem + stage * stage_bytes;
          tma_load_3d(kdst, &tmap_k, &full[stage], 0, t, x.hb * p.HB);
          tma_load_3d(kdst + kv_bytes, &tmap_v, &full[stage], 0, t, x.hb * p.HB);
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
  const int hh = warp / p.MT;  // KV head within the group
  const int mt = warp % p.MT;  // 16-row m-tile of that head's rows
  const int g = lane >> 2, c = lane & 3;
  const int BL = p.nrows;
  const uint32_t vpriv = smem_u32(priv + warp * kPrivBytes);
  int stage = 0;
  uint32_t phase = 0;

  for (int u = blockIdx.x; u < units; u += gridDim.x) {
    const Unit8 x = decode_unit8(p, u);
    const int b = x.b, s = x.s;
    const int kvh = x.hb * p.HB + hh;
    int q0, Lb;
    request_rows8(p, b, q0, Lb, nullptr);
    if (!unit_live8(p, x, Lb)) continue;
    int32_t t0, t1;
    split_range8(p, b, s, t0, t1);

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

    // Q fragments (A operand) widened to f16
    uint32_t qa[KSTEPS][4];
    {
      const __nv_bfloat16* q0 = p.q + (size_t(rrow[0]) * p.Hq + rqh[0]) * D8;
      const __nv_bfloat16* q1 = p.q + (size_t(rrow[1]) * p.Hq + rqh[1]) * D8;
#pragma unroll
      for (int ks = 0; ks < KSTEPS; ++ks) {
        const int col = ks * 16 + 2 * c;
        const uint32_t z = 0u;
        qa[ks][0] = bf16x2_to_f16x2(rvalid[0] ? __ldg(reinterpret_cast<const uint32_t*>(q0 + col)) : z);
        qa[ks][1] = bf16x2_to_f16x2(rvalid[1] ? __ldg(reinterpret_cast<const uint32_t*>(q1 + col)) : z);
        qa[ks][2] = bf16x2_to_f16x2(rvalid[0] ? __ldg(reinterpret_cast<const uint32_t*>(q0 + col + 8)) : z);
        qa[ks][3] = bf16x2_to_f16x2(rvalid[1] ? __ldg(reinterpret_cast<const uint32_t*>(q1 + col + 8)) : z);
      }
    }

    float acc[D8 / 8][4];
#pragma unroll
    for (int i = 0; i < D8 / 8; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
    float m_run[2] = {-INFINITY, -INFINITY};
    float l_run[2] = {0.f, 0.f};
    bool ok = true;

    for (int32_t t = t0; t < t1; t += kKeys) {
      if (!mbar_wait(&full[stage], phase, &abort_flag, p.status)) {
        ok = false;
        break;
      }
      const uint32_t k8 =
          smem_u32(smem + stage * stage_bytes) + hh * (PAGED ? uint32_t(D8) : kHeadTile8);
      // widen this head's V tile into the warp's private f16 tile (the PV
      // operand needs it transposed, which ldmatrix.trans does on 16-bit data)
      widen_row<PAGED>(k8 + kv_bytes, vpriv, lane >> 1, lane & 1, rs);

      // S = Q K^T over 16 keys: two n-tiles of 8 keys; the B fragments come
      // straight from the e4m3 tile: key g, d = 16 ks + 2c (+1) and + 8 (+9)
      float sc[2][4];
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        sc[nt][0] = sc[nt][1] = sc[nt][2] = sc[nt][3] = 0.f;
        const uint32_t key = nt * 8 + g;
#pragma unroll
        for (int ks = 0; ks < KSTEPS; ++ks) {
          const uint32_t addr = tile_at<PAGED>(k8, key, ks, rs) + 2 * c;
          uint32_t x0, x1;
          asm volatile("ld.shared.u16 %0, [%1];" : "=r"(x0) : "r"(addr));
          asm volatile("ld.shared.u16 %0, [%1];" : "=r"(x1) : "r"(addr + 8));
          mma_f16_16816(sc[nt], qa[ks], e4m3x2_to_f16x2(x0), e4m3x2_to_f16x2(x1));
        }
      }
      // the e4m3 tile is no longer needed: hand the ring slot back
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[stage]);
      if (++stage == p.nstage) {
        stage = 0;
        phase ^= 1;
      }

      // online softmax in the log2 domain; keys past the split end are masked
      float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int32_t key = t + nt * 8 + 2 * c + (e & 1);
          float v = sc[nt][e] * p.logit_scale_log2;
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
      for (int i = 0; i < D8 / 8; ++i) {
        acc[i][0] *= alpha[0];
        acc[i][1] *= alpha[0];
        acc[i][2] *= alpha[1];
        acc[i][3] *= alpha[1];
      }

      // O += P V: P as the A operand (f16), V^T via ldmatrix.trans on the f16 tile
      uint32_t pa[4];
      pa[0] = pack_f16(ps[0][0], ps[0][1]);
      pa[1] = pack_f16(ps[0][2], ps[0][3]);
      pa[2] = pack_f16(ps[1][0], ps[1][1]);
      pa[3] = pack_f16(ps[1][2], ps[1][3]);
      {
        const int mi = lane >> 3;
        const uint32_t key = (mi & 1) * 8 + (lane & 7);
#pragma unroll
        for (int dt = 0; dt < D8 / 8; dt += 2) {
          const uint32_t chunk = dt + (mi >> 1);
          const uint32_t addr = vpriv + (chunk >> 3) * (kKeys * 128) + sw128(key, chunk & 7);
          uint32_t b0, b1, b2, b3;
          ldmatrix_x4_trans(addr, b0, b1, b2, b3);
          mma_f16_16816(acc[dt], pa, b0, b1);
          mma_f16_16816(acc[dt + 1], pa, b2, b3);
        }
      }
      __syncwarp();  // the private tiles are rewritten by the next tile
    }
    if (!ok) return;

    // normalise, apply v_scale and write this split's partial
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      l_run[i] += __shfl_xor_sync(0xffffffffu, l_run[i], 1);
      l_run[i] += __shfl_xor_sync(0xffffffffu, l_run[i], 2);
    }
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      if (!rvalid[i]) continue;
      const float inv = l_run[i] > 0.f ? p.v_scale / l_run[i] : 0.f;
      const size_t prow = (size_t(s) * BL + rrow[i]) * p.Hq + rqh[i];
      float* dst = p.part_o + prow * D8;
#pragma unroll
      for (int dt = 0; dt < D8 / 8; ++dt) {
        float2 v = make_float2(acc[dt][2 * i] * inv, acc[dt][2 * i + 1] * inv);
        *reinterpret_cast<float2*>(dst + dt * 8 + 2 * c) = v;
      }
      if (c == 0)
        p.part_lse[prow] = l_run[i] > 0.f ? m_run[i] + __log2f(l_run[i]) : -INFINITY;
    }
  }
}

}  // namespace

int launch_verify_fp8(const VerifyArgs& a, float k_scale, float v_scale) {
  if (a.D != D8) return PSA_ERR_UNSUPPORTED;
  int HB = 0, MT = 0, NRB = 0;
  if (!verify_plan(a.Ld, a.Hq, a.Hkv, a.D, &HB, &MT, &NRB)) return PSA_ERR_UNSUPPORTED;
  if (HB * MT > kMaxWarps || HB > 16) return PSA_ERR_UNSUPPORTED;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return PSA_ERR_CUDA;
  const int G = a.Hq / a.Hkv;

  CUtensorMap tk, tv;
  // a tensor map needs a non-empty extent (an empty cache is never read)
  const uint64_t rows = a.n_cache_tokens > 0 ? uint64_t(a.n_cache_tokens) : 1u;
  const uint64_t dims[3] = {uint64_t(D8), rows, uint64_t(a.Hkv)};
  const uint64_t strides[2] = {uint64_t(a.Hkv) * D8, uint64_t(D8)};
  const uint32_t box[3] = {uint32_t(D8), uint32_t(kKeys), uint32_t(HB)};
  int rc = encode_tmap(&tk, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, a.kc, dims, strides, box,
                       CU_TENSOR_MAP_SWIZZLE_128B);
  if (rc != PSA_OK) return rc;
  rc = encode_tmap(&tv, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, a.vc, dims, strides, box,
                   CU_TENSOR_MAP_SWIZZLE_128B);
  if (rc != PSA_OK) return rc;

  P8Params p;
  p.q = static_cast<const __nv_bfloat16*>(a.q);
  p.indptr = a.indptr;
  p.kv_indices = a.kv_indices;
  p.qo_indptr = a.qo_indptr;
  p.nrows = a.qo_indptr ? a.n_rows : a.B * a.Ld;
  p.kc8 = static_cast<const uint8_t*>(a.kc);
  p.vc8 = static_cast<const uint8_t*>(a.vc);
  p.ntok = a.n_cache_tokens;
  p.part_o = a.part_o;
  p.part_lse = a.part_lse;
  p.B = a.B;
  p.Ld = a.Ld;
  p.Hq = a.Hq;
  p.Hkv = a.Hkv;
  p.G = G;
  p.R = a.Ld * G;
  p.MT = MT;
  p.nrb = NRB;
  p.HB = HB;
  p.nhb = a.Hkv / HB;
  p.nsplit = a.nsplit;
  p.logit_scale_log2 = a.scale * k_scale * kLog2e;
  p.v_scale = v_scale;
  p.status = a.status;

  const int NW = HB * MT;
  const bool paged = a.kv_indices != nullptr;
  const size_t stage_bytes =
      size_t(2) * (paged ? size_t(kKeys) * (size_t(HB) * D8 + 16) : size_t(HB) * kHeadTile8);
  const size_t priv_bytes = size_t(NW) * kPrivBytes;
  const size_t budget = 200 * 1024;
  int nstage = int((budget - priv_bytes) / stage_bytes);
  nstage = nstage > 16 ? 16 : nstage;
  if (nstage < 2) return PSA_ERR_UNSUPPORTED;
  p.nstage = nstage;
  const size_t smem = 1024 + nstage * stage_bytes + priv_bytes + 2 * nstage * sizeof(uint64_t);
  auto k1 = paged ? verify_stage1_fp8_kernel<true> : verify_stage1_fp8_kernel<false>;
  if (cudaFuncSetAttribute(k1, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)) !=
      cudaSuccess)
    return PSA_ERR_CUDA;
  const int units = a.B * a.nsplit * NRB * p.nhb;
  int grid = sm_count(dev);
  if (grid <= 0) return PSA_ERR_CUDA;
  grid = units < grid ? units : grid;
  if (units > 0) {
    k1<<<grid, (NW + (paged ? kPagedProducers8 : 1)) * 32, smem, a.stream>>>(tk, tv, p);
    if (cudaGetLastError() != cudaSuccess) return PSA_ERR_CUDA;
  }
  return launch_verify_combine(a);
}

}  // namespace psa
