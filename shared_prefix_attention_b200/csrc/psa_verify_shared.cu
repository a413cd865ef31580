// Speculative verify against ONE prefix shared by every request.  The prefix
// K/V is stored once ("KV-0 redundancy prefix sharing attention mask
// design", PrefixSharing PR #50: design summary) and every draft row of every
// request attends to all of it plus its own causal draft block
// ("Split-KV flash-decode attention for EAGLE target-verify", sglang PR
// #27382: implementation breakdown item 1).
//
// With the prefix shared, all B * Ld draft tokens of a KV head's G query heads
// read the same keys, so stage 1 is a dense tensor-core product instead of a
// per-request stream: the rows (token t, head g) of one KV head are stacked
// into 128-row halves, the prefix is cut into nsplit chunks of whole 128-key
// tiles, and each unit (chunk s, KV head h, block of 256 rows) computes the
// normalised partial O and the log2-domain LSE of its rows over its chunk.
// The combine stage of the per-request verify then merges the chunks and the
// causal draft block unchanged.
//
// sm_100a design (one CTA per SM, static round-robin over units):
//   warps 0, 2   TMA producers: the two Q halves of the unit (a 3-D box of
//                {64 d, G heads, 128 / G tokens} = 128 rows x 128 bytes per
//                swizzle atom), then the chunk's K and V tiles, 128-byte
//                swizzle, no multicast.
//   warp 1       tcgen05 issuer (one thread): S_X = Q_X K^T into TMEM, then
//                O_X += P_X V with P_X read from TMEM where the softmax left
//                it.  Issue order PV_A(j), QK_A(j+1), PV_B(j), QK_B(j+1).
//   warps 4..7 / 8..11  softmax of half A / B (one row per thread = TMEM
//                lane), lazy O rescaling in TMEM, epilogue straight from TMEM
//                into the fp32 partials.
// Every wait is bounded: a stuck pipeline reports PSA_ERR_TIMEOUT through the
// status word, the CTA unwinds and frees its TMEM.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>

#include "psa_device.cuh"
#include "psa_internal.h"
#include "psa_tmem_wide.cuh"

namespace psa {
namespace {

constexpr int BM = 128;             // rows per half
constexpr int BLOCK_M = 2 * BM;     // rows per unit
constexpr int BN = 128;             // keys per tile
constexpr int kThreads = 384;       // 12 warps
constexpr float kRescaleLog2 = 8.f;
constexpr uint32_t kTmemCols = 512;  // per half: S at X*256, O at X*256 + 128

template <int D>
struct SCfg {
  static constexpr int NPART = D / 64;
  static constexpr uint32_t Q_BYTES = BM * D * 2;  // one half
  static constexpr uint32_t KV_BYTES = BN * D * 2;
  static constexpr int NSK = D == 128 ? 3 : 4;
  static constexpr int NSV = D == 128 ? 2 : 4;
  static constexpr uint32_t OFF_Q = 0;
  static constexpr uint32_t OFF_K = OFF_Q + 2 * Q_BYTES;
  static constexpr uint32_t OFF_V = OFF_K + NSK * KV_BYTES;
  static constexpr uint32_t OFF_BAR = OFF_V + NSV * KV_BYTES;
  static constexpr uint32_t NBAR = 2 + 2 * NSK + 2 * NSV + 8;
  static constexpr uint32_t SMEM = 1024 + OFF_BAR + NBAR * 8 + 16;
};

struct SParams {
  float* part_o;    // [nsplit][BL][Hq][D]
  float* part_lse;  // [nsplit][BL][Hq], log2 domain
  int32_t L, BL, Hq, Hkv, G, nsplit, chunk, nblocks, units;
  float scale_log2;
  int32_t* status;
};

struct SBars {
  uint64_t *q_full, *q_empty, *k_full, *k_empty, *v_full, *v_empty;
  uint64_t *s_full, *p_full, *pv_done, *o_free;  // [2] each, one per half
};

// Register split (as in the prefill kernel): warpgroup 0 drops to 104, the
// two softmax warpgroups rise to 200 (2 x 128 x 200 + 128 x 104 = 64512).
__device__ __forceinline__ void sregs_dec() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 104;" ::: "memory");
}
__device__ __forceinline__ void sregs_inc() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 200;" ::: "memory");
}

// Unit u -> (chunk s, KV head h, row block rb); its key range [kb, ke).
struct Unit {
  int s, h, rb, kb, ke, ntiles;
};

__device__ __forceinline__ Unit decode_unit(const SParams& p, int u) {
  Unit w;
  w.rb = u % p.nblocks;
  const int sh = u / p.nblocks;
  w.h = sh % p.Hkv;
  w.s = sh / p.Hkv;
  w.kb = min(p.L, w.s * p.chunk);
  w.ke = min(p.L, w.kb + p.chunk);
  w.ntiles = (w.ke - w.kb + BN - 1) / BN;
  return w;
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    verify_shared_stage1(const __grid_constant__ CUtensorMap tmap_q,
                         const __grid_constant__ CUtensorMap tmap_k,
                         const __grid_constant__ CUtensorMap tmap_v, SParams p) {
  using C = SCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  __shared__ uint32_t tmem_base_slot;
  __shared__ int abort_flag;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int R = p.BL * p.G;  // rows of one KV head

  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  SBars B;
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
    sregs_dec();
    if (warp == 0 || warp == 2) {
      // ============================================================ producers
      // warp 0 loads Q and K, warp 2 loads V; units of empty chunks load nothing
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
        for (int u = blockIdx.x; u < p.units && ok; u += gridDim.x) {
          const Unit w = decode_unit(p, u);
          if (w.ntiles == 0) continue;
          if (kprod) {
            if (!mbar_wait(B.q_empty, (uc & 1) ^ 1, &abort_flag, p.status)) break;
            mbar_arrive_expect_tx(B.q_full, 2 * C::Q_BYTES);
#pragma unroll
            for (int x = 0; x < 2; ++x) {
              const int t0 = (w.rb * BLOCK_M + x * BM) / p.G;
#pragma unroll
              for (int part = 0; part < C::NPART; ++part)
                tma_load_3d(smem + C::OFF_Q + x * C::Q_BYTES + part * BM * 128, &tmap_q,
                            B.q_full, part * 64, w.h * p.G, t0);
            }
          }
          for (int j = 0; j < w.ntiles; ++j) {
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
              tma_load_3d(dst + part * BN * 128, tm, full + slot, part * 64, w.h, w.kb + j * BN);
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
      // ============================================================ MMA issuer
      if (lane == 0) {
        const uint32_t idesc_qk = umma_idesc_bf16(BM, BN, false, false);
        const uint32_t idesc_pv = umma_idesc_bf16(BM, D, false, true);
        const uint32_t sQ = smem_u32(smem + C::OFF_Q);
        const uint32_t sK = smem_u32(smem + C::OFF_K);
        const uint32_t sV = smem_u32(smem + C::OFF_V);
        uint32_t kc = 0, uc = 0;
        uint32_t pvc0 = 0, pvc1 = 0, uhc0 = 0, uhc1 = 0;
        bool ok = true;

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
        auto issue_pv = [&](int x, uint32_t t_glob, bool first, uint32_t& pvc,
                            uint32_t uhc) -> bool {
          if (!mbar_wait(B.p_full + x, pvc & 1, &abort_flag, p.status)) return false;
          const int slot = t_glob % C::NSV;
          if (!mbar_wait(B.v_full + slot, (t_glob / C::NSV) & 1, &abort_flag, p.status))
            return false;
          if (first && !mbar_wait(B.o_free + x, (uhc & 1) ^ 1, &abort_flag, p.status))
            return false;
          tc_fence_after();
          const uint32_t vbase = sV + slot * C::KV_BYTES;
#pragma unroll
          for (int ks = 0; ks < BN / 16; ++ks)
            umma_ts(tmem + x * 256 + 128, tmem + x * 256 + ks * 8,
                    umma_desc_sw128(vbase + ks * 2048, BN * 128, 1024), idesc_pv,
                    (first && ks == 0) ? 0u : 1u);
          umma_commit(B.pv_done + x);
          ++pvc;
          return true;
        };

        for (int u = blockIdx.x; u < p.units && ok; u += gridDim.x) {
          const Unit w = decode_unit(p, u);
          const int n = w.ntiles;
          if (n == 0) continue;
          const bool act0 = w.rb * BLOCK_M < R, act1 = w.rb * BLOCK_M + BM < R;
          if (!mbar_wait(B.q_full, uc & 1, &abort_flag, p.status)) break;
          if (act0) ok = issue_qk(0, kc);
          if (ok && act1) ok = issue_qk(1, kc);
          if (!ok) break;
          umma_commit(B.k_empty + (kc % C::NSK));
          if (n == 1) umma_commit(B.q_empty);
          for (int j = 0; j < n && ok; ++j) {
            const uint32_t t = kc + j;
            if (act0) ok = issue_pv(0, t, j == 0, pvc0, uhc0);
            if (ok && act0 && j + 1 < n) ok = issue_qk(0, t + 1);
            if (ok && act1) ok = issue_pv(1, t, j == 0, pvc1, uhc1);
            if (ok && act1 && j + 1 < n) ok = issue_qk(1, t + 1);
            if (!ok) break;
            umma_commit(B.v_empty + (t % C::NSV));
            if (j + 1 < n) {
              umma_commit(B.k_empty + ((t + 1) % C::NSK));
              if (j + 2 == n) umma_commit(B.q_empty);
            }
          }
          if (!ok) break;
          kc += n;
          if (act0) ++uhc0;
          if (act1) ++uhc1;
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
    sregs_inc();
    // ============================================================== softmax + epilogue
    const int x = (warp - 4) >> 2;
    const int quarter = warp & 3;
    const int r_in = quarter * 32 + lane;  // row within the half
    const uint32_t trow = tmem + (uint32_t(quarter * 32) << 16) + x * 256;
    const uint32_t tS = trow, tO = trow + 128;
    uint32_t sc_count = 0;  // S tiles of this half consumed (all units)
    bool ok = true;
    for (int u = blockIdx.x; u < p.units && ok; u += gridDim.x) {
      const Unit w = decode_unit(p, u);
      const int row = w.rb * BLOCK_M + x * BM + r_in;  // row = token * G + head-in-group
      const bool valid = row < R;
      const int tok = row / p.G, qh = w.h * p.G + row % p.G;
      const size_t prow = (size_t(w.s) * p.BL + tok) * p.Hq + qh;
      if (w.ntiles == 0) {
        // empty chunk: a partial that carries no weight
        if (valid) {
          float4* dst = reinterpret_cast<float4*>(p.part_o + prow * D);
#pragma unroll 4
          for (int k = 0; k < D / 4; ++k) dst[k] = make_float4(0.f, 0.f, 0.f, 0.f);
          p.part_lse[prow] = -INFINITY;
        }
        continue;
      }
      if (w.rb * BLOCK_M + x * BM >= R) continue;  // the whole half is past the last row

      float m_run = -INFINITY, l_run = 0.f;
      for (int j = 0; j < w.ntiles; ++j) {
        if (!mbar_wait(B.s_full + x, sc_count & 1, &abort_flag, p.status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const int klen = min(BN, w.ke - (w.kb + j * BN));  // keys of this tile in the chunk

        uint32_t sr[BN];
        tmem_ld128(tS, sr);
        tmem_wait_ld();
        if (klen < BN) {
#pragma unroll
          for (int k = 0; k < BN; ++k)
            if (k >= klen) sr[k] = __float_as_uint(-INFINITY);
        }
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
        const bool rescale_o = __any_sync(0xffffffffu, resc) && j > 0;
        float alpha = 1.f;
        if (resc) {
          alpha = fast_exp2(m_run - m_new);
          l_run *= alpha;
          m_run = m_new;
        }
        const float neg_m = m_run == -INFINITY ? 0.f : -m_run;

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
      }
      if (!ok) break;

      // ---- epilogue: normalised partial O (fp32) and log2-domain LSE
      if (!mbar_wait(B.pv_done + x, (sc_count - 1) & 1, &abort_flag, p.status)) break;
      tc_fence_after();
      const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t rr[32];
        tmem_ld32(tO + c * 32, rr);
        tmem_wait_ld();
        if (valid) {
          float4* dst = reinterpret_cast<float4*>(p.part_o + prow * D + c * 32);
#pragma unroll
          for (int k = 0; k < 8; ++k)
            dst[k] = make_float4(
                __uint_as_float(rr[4 * k]) * inv, __uint_as_float(rr[4 * k + 1]) * inv,
                __uint_as_float(rr[4 * k + 2]) * inv, __uint_as_float(rr[4 * k + 3]) * inv);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(B.o_free + x);
      if (valid) p.part_lse[prow] = l_run > 0.f ? m_run + __log2f(l_run) : -INFINITY;
    }
  }

  // ---- teardown: every role has finished issuing; free TMEM
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, kTmemCols);
}

template <int D>
int launch_shared_stage1(const VerifySharedArgs& a, int nblocks) {
  using C = SCfg<D>;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return PSA_ERR_CUDA;
  const int G = a.Hq / a.Hkv;
  const int BL = a.B * a.Ld;
  CUtensorMap tq, tk, tv;
  {
    // q_draft [BL, Hq, D] viewed as (d, head, token); a box is G heads x
    // 128 / G tokens = 128 stacked rows of one KV head
    const uint32_t box[3] = {64u, uint32_t(G), uint32_t(BM / G)};
    const uint64_t dims[3] = {uint64_t(D), uint64_t(a.Hq), uint64_t(BL)};
    const uint64_t strides[2] = {uint64_t(D) * 2, uint64_t(a.Hq) * D * 2};
    int rc = encode_tmap(&tq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, a.q, dims, strides, box,
                         CU_TENSOR_MAP_SWIZZLE_128B);
    if (rc != PSA_OK) return rc;
  }
  {
    const uint32_t box[3] = {64u, 1u, uint32_t(BN)};
    const uint64_t dims[3] = {uint64_t(D), uint64_t(a.Hkv), uint64_t(a.L)};
    const uint64_t strides[2] = {uint64_t(D) * 2, uint64_t(a.Hkv) * D * 2};
    int rc = encode_tmap(&tk, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, a.kp, dims, strides, box,
                         CU_TENSOR_MAP_SWIZZLE_128B);
    if (rc != PSA_OK) return rc;
    rc = encode_tmap(&tv, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, a.vp, dims, strides, box,
                     CU_TENSOR_MAP_SWIZZLE_128B);
    if (rc != PSA_OK) return rc;
  }
  SParams p;
  p.part_o = a.part_o;
  p.part_lse = a.part_lse;
  p.L = int32_t(a.L);
  p.BL = BL;
  p.Hq = a.Hq;
  p.Hkv = a.Hkv;
  p.G = G;
  p.nsplit = a.nsplit;
  p.chunk = a.chunk;
  p.nblocks = nblocks;
  p.units = a.nsplit * a.Hkv * nblocks;
  p.scale_log2 = a.scale * kLog2e;
  p.status = a.status;
  auto kern = verify_shared_stage1<D>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(C::SMEM)) !=
      cudaSuccess)
    return PSA_ERR_CUDA;
  const int grid = std::min(sm_count(dev), p.units);
  if (grid <= 0) return PSA_ERR_CUDA;
  kern<<<grid, kThreads, C::SMEM, a.stream>>>(tq, tk, tv, p);
  return cudaGetLastError() == cudaSuccess ? PSA_OK : PSA_ERR_CUDA;
}

}  // namespace

int launch_verify_shared(const VerifySharedArgs& a) {
  const int G = a.Hq / a.Hkv;
  const int R = a.B * a.Ld * G;
  const int nblocks = (R + BLOCK_M - 1) / BLOCK_M;
  if (a.L > 0) {
    int rc = PSA_ERR_UNSUPPORTED;
    if (a.D == 64) rc = launch_shared_stage1<64>(a, nblocks);
    if (a.D == 128) rc = launch_shared_stage1<128>(a, nblocks);
    if (rc != PSA_OK) return rc;
  }
  VerifyArgs c{};
  c.q = a.q;
  c.kd = a.kd;
  c.vd = a.vd;
  c.o = a.o;
  c.lse = a.lse;
  c.B = a.B;
  c.Ld = a.Ld;
  c.Hq = a.Hq;
  c.Hkv = a.Hkv;
  c.D = a.D;
  c.scale = a.scale;
  c.nsplit = a.L > 0 ? a.nsplit : 0;
  c.part_o = a.part_o;
  c.part_lse = a.part_lse;
  c.status = a.status;
  c.stream = a.stream;
  c.dmask = a.dmask;
  return launch_verify_combine(c);
}

}  // namespace psa
