// Shared-latent sparse attention: every query attends to the latent rows its
// own index list names, and the one 512-wide latent serves as both K and V
// for all heads ("SM8x sparse-MLA prefill fallback re-reads the shared MLA
// latent once per head", vLLM issue write-up: environment -- index_topk
// 2048, 64 heads, kv_lora_rank 512, no rope part; analysis -- the per-head
// program re-reads the shared latent, and head-blocked 2-D tiles are what
// make the kernel fast).
//
// sm_100a design: one CTA per SM, persistent over queries (heaviest first).
// All heads of a query share every latent row the CTA gathers, and the
// gathered rows are used twice -- as K and as V -- from one shared-memory
// copy.  The products are computed transposed so the key dimension fills
// the 128 rows of a tcgen05 MMA:
//   S^T [128 keys x H]   = Lat_tile [128 x 512] . Q_t^T [512 x H]
//   O^T [512 x H]       += Lat_tile^T [512 x 128] . P^T [128 x H]
// The latent tile is gathered by cp.async (whole 128-byte rows per group of
// eight threads, zero fill for -1 entries) in eight 64-column parts; a part
// is released for the next tile as soon as the O^T block that reads it has
// completed.  Q_t^T arrives by TMA.
//   warps 0..3   gather producers and the Q^T load
//   warp 4       tcgen05 issuer (one thread)
//   warps 8..11  softmax over keys (one key per thread = TMEM lane) with
//                per-head max / sum reductions across lanes, P^T written to
//                shared memory, lazy O^T rescaling, and the epilogue (one
//                latent dimension per thread and M-block).
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "psa_device.cuh"
#include "psa_internal.h"
#include "psa_tmem_wide.cuh"

namespace psa {
namespace {

constexpr int DL = 512;          // latent width
constexpr int KT = 128;          // keys per tile (MMA M for S^T)
constexpr int NPART = DL / 64;   // 64-column parts of a latent tile
constexpr int HMAX = 64;         // heads per CTA pass (MMA N)
constexpr int kThreads = 384;
constexpr float kRescaleLog2 = 8.f;
constexpr uint32_t kTmemCols = 512;  // S^T at 0, O^T M-blocks at 128 + 64 * mb

constexpr uint32_t PART_BYTES = KT * 128;       // 16 KB
constexpr uint32_t QPART_BYTES = HMAX * 128;    // 8 KB
constexpr uint32_t OFF_LAT = 0;
constexpr uint32_t OFF_Q = OFF_LAT + NPART * PART_BYTES;     // 128 KB
constexpr uint32_t OFF_P = OFF_Q + NPART * QPART_BYTES;      // +64 KB
constexpr uint32_t OFF_RED = OFF_P + KT * 128;               // +16 KB
constexpr uint32_t RED_BYTES = 2 * 4 * HMAX * 4;             // max and sum: [4 warps][64]
constexpr uint32_t OFF_HEAD = OFF_RED + RED_BYTES;           // per-head state
constexpr uint32_t HEAD_BYTES = 4 * HMAX * 4;                // m, l, alpha, 1/l
constexpr uint32_t OFF_BAR = OFF_HEAD + HEAD_BYTES;
constexpr uint32_t NBAR = 2 * NPART + 2 + 5;
constexpr uint32_t SMEM = 1024 + OFF_BAR + NBAR * 8 + 64;

struct Params {
  const __nv_bfloat16* q;
  const __nv_bfloat16* lat;
  const int32_t* idx;
  __nv_bfloat16* o;
  float* lse;
  int32_t T, Tk, H, topk;
  float scale_log2;
  int32_t* status;
};

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src),
               "r"(src_bytes)
               : "memory");
}

// Arrives on `bar` once every cp.async this thread issued so far has landed.
__device__ __forceinline__ void cp_async_arrive(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void named_bar_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// A group barrier that every member skips once the CTA has aborted (a member
// that gave up on a bounded wait never reaches the barrier); the `break`
// leaves the enclosing loop.
#define GROUP_SYNC(id)                 \
  if (*(volatile int*)&abort_flag) {   \
    ok = false;                        \
    break;                             \
  } else                               \
    named_bar_sync((id), 128)

// Reduces v[0..63] across the 32 lanes of the warp (max or sum); afterwards
// lane L holds the results for entries 2L and 2L+1 in r0, r1.
template <bool MAX>
__device__ __forceinline__ void warp_transpose_reduce64(const float (&v)[64], int lane, float& r0,
                                                        float& r1) {
  float w32[32];
  {
    const bool hi = lane & 16;
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      const float mine = hi ? v[32 + i] : v[i];
      const float other = hi ? v[i] : v[32 + i];
      const float got = __shfl_xor_sync(0xffffffffu, other, 16);
      w32[i] = MAX ? fmaxf(mine, got) : mine + got;
    }
  }
  float w16[16];
  {
    const bool hi = lane & 8;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const float mine = hi ? w32[16 + i] : w32[i];
      const float other = hi ? w32[i] : w32[16 + i];
      const float got = __shfl_xor_sync(0xffffffffu, other, 8);
      w16[i] = MAX ? fmaxf(mine, got) : mine + got;
    }
  }
  float w8[8];
  {
    const bool hi = lane & 4;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float mine = hi ? w16[8 + i] : w16[i];
      const float other = hi ? w16[i] : w16[8 + i];
      const float got = __shfl_xor_sync(0xffffffffu, other, 4);
      w8[i] = MAX ? fmaxf(mine, got) : mine + got;
    }
  }
  float w4[4];
  {
    const bool hi = lane & 2;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float mine = hi ? w8[4 + i] : w8[i];
      const float other = hi ? w8[i] : w8[4 + i];
      const float got = __shfl_xor_sync(0xffffffffu, other, 2);
      w4[i] = MAX ? fmaxf(mine, got) : mine + got;
    }
  }
  {
    const bool hi = lane & 1;
    float w2[2];
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const float mine = hi ? w4[2 + i] : w4[i];
      const float other = hi ? w4[i] : w4[2 + i];
      const float got = __shfl_xor_sync(0xffffffffu, other, 1);
      w2[i] = MAX ? fmaxf(mine, got) : mine + got;
    }
    r0 = w2[0];
    r1 = w2[1];
  }
}

__device__ __forceinline__ bool key_ok(int32_t k, int32_t Tk) { return k >= 0 && k < Tk; }

// Register split: 384 threads x 168 at launch = 64512.  The producer and
// MMA warpgroups drop to 80 so the softmax warpgroup can keep a key's 64
// logits, its 64 probabilities and the reduction scratch in registers
// (2 x 128 x 80 + 128 x 256 = 53248).
__device__ __forceinline__ void regs_dec80() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 80;" ::: "memory");
}
__device__ __forceinline__ void regs_inc256() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 256;" ::: "memory");
}

__global__ void __launch_bounds__(kThreads, 1)
    sparse_latent_kernel(const __grid_constant__ CUtensorMap tmap_q, Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  __shared__ uint32_t tmem_base_slot;
  __shared__ int abort_flag;
  __shared__ int q_ntiles;
  __shared__ int prod_ntiles;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
  uint64_t* part_full = bar;                 // [8] 128 producer copy arrivals
  uint64_t* part_empty = bar + NPART;        // [8] MMA commit
  uint64_t* q_full = bar + 2 * NPART;        // producer arrive (tile count) + TMA bytes
  uint64_t* q_empty = q_full + 1;            // MMA commit
  uint64_t* s_full = q_empty + 1;            // MMA commit
  uint64_t* p_full = s_full + 1;             // 4 softmax warps
  uint64_t* pv_done = p_full + 1;            // MMA commit
  uint64_t* o_full = pv_done + 1;            // MMA commit
  uint64_t* o_free = o_full + 1;             // 4 softmax warps
  float* red_max = reinterpret_cast<float*>(smem + OFF_RED);  // [4 warps][64]
  float* red_sum = red_max + 4 * HMAX;                         // [4 warps][64]
  float* h_m = reinterpret_cast<float*>(smem + OFF_HEAD);  // running max (log2 domain)
  float* h_l = h_m + HMAX;                                 // running sum
  float* h_alpha = h_l + HMAX;                             // this tile's rescale factor
  float* h_inv = h_alpha + HMAX;                           // 1 / l for the epilogue
  __shared__ int h_flagw[2];                               // a head-owner warp rescaled

  if (threadIdx.x == 0) {
    abort_flag = 0;
    for (int i = 0; i < NPART; ++i) {
      mbar_init(part_full + i, 128);
      mbar_init(part_empty + i, 1);
    }
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    mbar_init(s_full, 1);
    mbar_init(p_full, 4);
    mbar_init(pv_done, 1);
    mbar_init(o_full, 1);
    mbar_init(o_free, 4);
    fence_barrier_init();
  }
  if (threadIdx.x >= 256 && threadIdx.x < 256 + HMAX) h_m[threadIdx.x - 256] = -INFINITY;
  if (warp == 4) {
    tmem_alloc(&tmem_base_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_slot;
  const int tiles_max = (p.topk + KT - 1) / KT;

  // queries heaviest first: the last rows have the longest index lists
  auto query_of = [&](int i) { return p.T - 1 - (int(blockIdx.x) + i * int(gridDim.x)); };

  if (warp < 4) {
    regs_dec80();
    // ============================================================ producers
    // Warps 0..3 gather the latent tile with cp.async: eight threads cover
    // one 128-byte row of a part, so every warp instruction moves four whole
    // rows.  Lane 0 of warp 0 loads Q^T with TMA and publishes the tile count.
    const int pt = threadIdx.x;      // 0..127
    const int chunk = pt & 7;        // 16-byte piece of a part row
    const int rsub = pt >> 3;        // 0..15: row within a round of 16
    if (pt == 0) {
      tma_prefetch_desc(&tmap_q);
    }
    uint32_t tile_glob = 0;
    bool ok = true;
    for (int qi = 0; ok; ++qi) {
      const int t = query_of(qi);
      if (t < 0) break;
      const int32_t* qidx = p.idx + size_t(t) * p.topk;
      int ntiles = 0;
      if (warp == 0) {
        int last = -1;
        for (int sl = lane; sl < p.topk; sl += 32)
          if (key_ok(__ldg(qidx + sl), p.Tk)) last = sl;
        for (int off = 16; off > 0; off >>= 1)
          last = max(last, __shfl_xor_sync(0xffffffffu, last, off));
        ntiles = (last + KT) / KT;
        if (!mbar_wait(q_empty, (qi & 1) ^ 1, &abort_flag, p.status)) ntiles = -1;
        if (lane == 0 && ntiles >= 0) {
          q_ntiles = ntiles;  // published by the arrive below
          mbar_arrive_expect_tx(q_full, NPART * QPART_BYTES);
#pragma unroll
          for (int part = 0; part < NPART; ++part)
            tma_load_2d(smem + OFF_Q + part * QPART_BYTES, &tmap_q, q_full, part * 64, t * p.H);
        }
        if (lane == 0) prod_ntiles = ntiles;
      }
      if (*(volatile int*)&abort_flag) break;
      named_bar_sync(1, 128);
      ntiles = prod_ntiles;
      if (*(volatile int*)&abort_flag) break;
      named_bar_sync(1, 128);
      if (ntiles < 0) break;
      for (int j = 0; j < ntiles && ok; ++j, ++tile_glob) {
        const __nv_bfloat16* src[8];
        uint32_t sz[8];
#pragma unroll
        for (int it = 0; it < 8; ++it) {
          const int sl = j * KT + it * 16 + rsub;
          const int32_t k = sl < p.topk ? __ldg(qidx + sl) : -1;
          if (k >= p.Tk) report_status(p.status, PSA_ERR_INVALID_ARG);
          const bool valid = key_ok(k, p.Tk);
          src[it] = p.lat + size_t(valid ? k : 0) * DL + chunk * 8;
          sz[it] = valid ? 16u : 0u;  // zero fill for skipped slots
        }
        for (int part = 0; part < NPART; ++part) {
          if (!mbar_wait(part_empty + part, (tile_glob & 1) ^ 1, &abort_flag, p.status)) {
            ok = false;
            break;
          }
          const uint32_t base = smem_u32(smem + OFF_LAT + part * PART_BYTES);
#pragma unroll
          for (int it = 0; it < 8; ++it) {
            const int row = it * 16 + rsub;
            cp_async16(base + row * 128 + ((chunk ^ (row & 7)) << 4), src[it] + part * 64,
                       sz[it]);
          }
          cp_async_arrive(part_full + part);
        }
      }
    }
    // let every copy this thread issued land before the CTA can exit
    asm volatile("cp.async.wait_all;" ::: "memory");
  } else if (warp < 8) {
    regs_dec80();
    // ============================================================ MMA issuer
    if (warp == 4 && lane == 0) {
      const uint32_t idesc_s = umma_idesc_bf16(KT, HMAX, false, false);
      const uint32_t idesc_o = umma_idesc_bf16(128, HMAX, true, true);
      const uint32_t sLat = smem_u32(smem + OFF_LAT);
      const uint32_t sQ = smem_u32(smem + OFF_Q);
      const uint32_t sP = smem_u32(smem + OFF_P);
      uint32_t tile_glob = 0;
      uint32_t oq = 0;  // queries with at least one tile (O^T produced)
      bool ok = true;
      for (int qi = 0; ok; ++qi) {
        const int t = query_of(qi);
        if (t < 0) break;
        if (!mbar_wait(q_full, qi & 1, &abort_flag, p.status)) break;
        const int ntiles = q_ntiles;
        if (ntiles == 0) {
          umma_commit(q_empty);
          continue;
        }
        for (int j = 0; j < ntiles && ok; ++j, ++tile_glob) {
          // S^T = Lat_tile . Q^T, accumulated over the eight parts
          for (int part = 0; part < NPART && ok; ++part) {
            if (!mbar_wait(part_full + part, tile_glob & 1, &abort_flag, p.status)) {
              ok = false;
              break;
            }
            tc_fence_after();
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
              umma_ss(tmem, umma_desc_sw128(sLat + part * PART_BYTES + ks * 32, 16, 1024),
                      umma_desc_sw128(sQ + part * QPART_BYTES + ks * 32, 16, 1024), idesc_s,
                      (part | ks) ? 1u : 0u);
          }
          if (!ok) break;
          umma_commit(s_full);
          if (j == ntiles - 1) umma_commit(q_empty);
          // O^T += Lat^T . P^T once the softmax has written P^T
          if (!mbar_wait(p_full, tile_glob & 1, &abort_flag, p.status) ||
              (j == 0 && !mbar_wait(o_free, (oq & 1) ^ 1, &abort_flag, p.status))) {
            ok = false;
            break;
          }
          tc_fence_after();
          for (int mb = 0; mb < 4; ++mb) {
#pragma unroll
            for (int ks = 0; ks < KT / 16; ++ks)
              umma_ss(tmem + 128 + mb * 64,
                      umma_desc_sw128(sLat + 2 * mb * PART_BYTES + ks * 2048, PART_BYTES, 1024),
                      umma_desc_sw128(sP + ks * 2048, 8192, 1024), idesc_o,
                      (j > 0 || ks > 0) ? 1u : 0u);
            umma_commit(part_empty + 2 * mb);
            umma_commit(part_empty + 2 * mb + 1);
          }
          umma_commit(pv_done);
          if (j == ntiles - 1) umma_commit(o_full);
        }
        ++oq;
      }
      if (!ok || abort_flag) {
        const uint64_t t0 = globaltimer();
        while (globaltimer() - t0 < 1000000ull) {
        }
      }
    }
  } else {
    regs_inc256();
    // ============================================================ softmax + epilogue
    // One key per thread.  The 64 running maxima (log2 domain) live in shared
    // memory, each thread keeps its own 64 partial row sums in registers; a
    // tile only needs
    // a cross-key max when some logit would exceed its head's running max by
    // more than 2^8 (the first tile of a query always does), detected with
    // one OR-reduction barrier.  The partial sums meet once per query.
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;  // key slot (TMEM lane); latent dim in the epilogue
    const int tid = threadIdx.x - 256;  // 0..127 within the group
    const uint32_t trow = tmem + (uint32_t(quarter * 32) << 16);
    uint32_t tile_glob = 0;
    uint32_t oq = 0;  // queries with at least one tile
    bool ok = true;
    for (int qi = 0; ok; ++qi) {
      const int t = query_of(qi);
      if (t < 0) break;
      const int32_t* qidx = p.idx + size_t(t) * p.topk;
      // index of this thread's key slot in tile 0, fetched before the wait
      int32_t kidx_next = r < p.topk ? __ldg(qidx + r) : -1;
      if (!mbar_wait(q_full, qi & 1, &abort_flag, p.status)) break;
      const int ntiles = q_ntiles;
      float lpart[HMAX];
#pragma unroll
      for (int h = 0; h < HMAX; ++h) lpart[h] = 0.f;
      for (int j = 0; j < ntiles && ok; ++j, ++tile_glob) {
        const bool valid = key_ok(kidx_next, p.Tk);
        {
          const int sl = (j + 1) * KT + r;  // prefetch the next tile's index
          kidx_next = sl < p.topk ? __ldg(qidx + sl) : -1;
        }
        if (!mbar_wait(s_full, tile_glob & 1, &abort_flag, p.status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        float v[HMAX];
        {
          uint32_t raw[HMAX];
          tmem_ld64(trow, raw);
          tmem_wait_ld();
#pragma unroll
          for (int h = 0; h < HMAX; ++h)
            v[h] = valid ? __uint_as_float(raw[h]) * p.scale_log2 : -INFINITY;
        }
        // does any logit of this tile outgrow its head's running max?
        float over = -INFINITY;
#pragma unroll
        for (int h = 0; h < HMAX; ++h) over = fmaxf(over, v[h] - h_m[h]);
        if (*(volatile int*)&abort_flag) {
          ok = false;
          break;
        }
        uint32_t any_over;
        asm volatile(
            "{\n\t.reg .pred pi, po;\n\t"
            "setp.gt.f32 pi, %1, %2;\n\t"
            "bar.red.or.pred po, 2, 128, pi;\n\t"
            "selp.u32 %0, 1, 0, po;\n\t}"
            : "=r"(any_over)
            : "f"(over), "f"(kRescaleLog2)
            : "memory");
        if (any_over) {
          // cross-key max per head: across lanes, then across warps
          float a0, a1;
          warp_transpose_reduce64<true>(v, lane, a0, a1);
          red_max[quarter * HMAX + 2 * lane] = a0;
          red_max[quarter * HMAX + 2 * lane + 1] = a1;
          GROUP_SYNC(2);
          if (tid < HMAX) {
            const float mt = fmaxf(fmaxf(red_max[tid], red_max[HMAX + tid]),
                                   fmaxf(red_max[2 * HMAX + tid], red_max[3 * HMAX + tid]));
            const float mo = h_m[tid];
            const float mn = fmaxf(mo, mt);
            float alpha = 1.f;
            if (mn > mo + kRescaleLog2) {
              alpha = fast_exp2(mo - mn);  // 0 when mo = -inf
              h_m[tid] = mn;
            }
            h_alpha[tid] = alpha;
            const bool any = __any_sync(0xffffffffu, alpha != 1.f && j > 0);
            if (lane == 0) h_flagw[quarter] = any ? 1 : 0;
          }
          GROUP_SYNC(2);
#pragma unroll
          for (int h = 0; h < HMAX; ++h) lpart[h] *= h_alpha[h];
          if (h_flagw[0] | h_flagw[1]) {
            // lazy O^T rescale: column h of every M-block times alpha_h, once
            // the previous O^T product has landed
            if (!mbar_wait(pv_done, (tile_glob - 1) & 1, &abort_flag, p.status)) {
              ok = false;
              break;
            }
            tc_fence_after();
#pragma unroll 1
            for (int mb = 0; mb < 4; ++mb) {
              uint32_t ov[HMAX];
              tmem_ld64(trow + 128 + mb * 64, ov);
              tmem_wait_ld();
#pragma unroll
              for (int h = 0; h < HMAX; ++h)
                ov[h] = __float_as_uint(__uint_as_float(ov[h]) * h_alpha[h]);
              tmem_st64(trow + 128 + mb * 64, ov);
            }
            tmem_wait_st();
          }
        }
        // P^T row of this key: exp2(s * scale - m_h)
#pragma unroll
        for (int h = 0; h < HMAX; ++h) {
          const float m = h_m[h];
          v[h] = fast_exp2(v[h] - (m == -INFINITY ? 0.f : m));
          lpart[h] += v[h];
        }
        // the previous O^T product must be done before P^T is overwritten
        if (j > 0 && !mbar_wait(pv_done, (tile_glob - 1) & 1, &abort_flag, p.status)) {
          ok = false;
          break;
        }
        {
          const uint32_t prow = smem_u32(smem + OFF_P) + r * 128;
#pragma unroll
          for (int c = 0; c < HMAX / 8; ++c) {
            const uint32_t w0 = pack_bf16(v[8 * c], v[8 * c + 1]);
            const uint32_t w1 = pack_bf16(v[8 * c + 2], v[8 * c + 3]);
            const uint32_t w2 = pack_bf16(v[8 * c + 4], v[8 * c + 5]);
            const uint32_t w3 = pack_bf16(v[8 * c + 6], v[8 * c + 7]);
            asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(
                             prow + ((c ^ (r & 7)) << 4)),
                         "r"(w0), "r"(w1), "r"(w2), "r"(w3)
                         : "memory");
          }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(p_full);
      }
      if (!ok) break;
      // per-head sums: the partial sums of all keys meet once per query
      {
        float a0, a1;
        warp_transpose_reduce64<false>(lpart, lane, a0, a1);
        red_sum[quarter * HMAX + 2 * lane] = a0;
        red_sum[quarter * HMAX + 2 * lane + 1] = a1;
      }
      GROUP_SYNC(2);
      if (tid < HMAX) {
        const float l = (red_sum[tid] + red_sum[HMAX + tid]) +
                        (red_sum[2 * HMAX + tid] + red_sum[3 * HMAX + tid]);
        h_l[tid] = l;
        h_inv[tid] = l > 0.f ? 1.f / l : 0.f;
      }
      GROUP_SYNC(2);  // h_l, h_inv final
      if (ntiles > 0) {
        if (!mbar_wait(o_full, oq & 1, &abort_flag, p.status)) break;
        tc_fence_after();
      }
      // epilogue: per M-block, thread d = r scales its O^T lane by 1/l_h and
      // stages it as [head][128 dims] in the (now idle) P^T buffer; the block
      // then goes out as contiguous 16-byte rows.
      __nv_bfloat16* stage = reinterpret_cast<__nv_bfloat16*>(smem + OFF_P);
#pragma unroll 1
      for (int mb = 0; mb < 4; ++mb) {
        uint32_t ov[HMAX];
        if (ntiles > 0) {
          tmem_ld64(trow + 128 + mb * 64, ov);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int h = 0; h < HMAX; ++h) ov[h] = 0u;
        }
#pragma unroll
        for (int h = 0; h < HMAX; ++h)
          stage[h * 128 + r] = __float2bfloat16(__uint_as_float(ov[h]) * h_inv[h]);
        GROUP_SYNC(2);
#pragma unroll
        for (int k = 0; k < (HMAX * 16) / 128; ++k) {
          const int c = k * 128 + tid;  // 16-byte chunk: head c / 16, piece c % 16
          const int h = c >> 4, piece = c & 15;
          if (h < p.H)
            *reinterpret_cast<uint4*>(p.o + (size_t(t) * p.H + h) * DL + mb * 128 + piece * 8) =
                *reinterpret_cast<const uint4*>(stage + h * 128 + piece * 8);
        }
        GROUP_SYNC(2);
      }
      if (!ok) break;
      tc_fence_before();
      __syncwarp();
      if (ntiles > 0) {
        if (lane == 0) mbar_arrive(o_free);
        ++oq;
      }
      if (tid < p.H && p.lse) {
        const float l = h_l[tid];
        p.lse[size_t(t) * p.H + tid] = l > 0.f ? (h_m[tid] + __log2f(l)) * kLn2 : -INFINITY;
      }
      if (tid < HMAX) h_m[tid] = -INFINITY;  // fresh running max for the next query
      GROUP_SYNC(2);
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 4) tmem_dealloc(tmem, kTmemCols);
}

}  // namespace

int launch_sparse_latent(const SparseArgs& a) {
  if (a.dl != DL || a.H > HMAX || a.H <= 0) return PSA_ERR_UNSUPPORTED;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return PSA_ERR_CUDA;
  Params p;
  p.q = static_cast<const __nv_bfloat16*>(a.q);
  p.lat = static_cast<const __nv_bfloat16*>(a.latent);
  p.idx = a.idx;
  p.o = static_cast<__nv_bfloat16*>(a.o);
  p.lse = a.lse;
  p.T = a.T;
  p.Tk = a.Tk;
  p.H = a.H;
  p.topk = a.topk;
  p.scale_log2 = a.scale * kLog2e;
  p.status = a.status;
  CUtensorMap tq;
  {
    const uint64_t dims[2] = {uint64_t(DL), uint64_t(a.T) * a.H};
    const uint64_t strides[1] = {uint64_t(DL) * 2};
    const uint32_t box[2] = {64u, uint32_t(HMAX)};
    const int rc = encode_tmap(&tq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.q, dims, strides, box,
                               CU_TENSOR_MAP_SWIZZLE_128B);
    if (rc != PSA_OK) return rc;
  }
  if (cudaFuncSetAttribute(sparse_latent_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           int(SMEM)) != cudaSuccess)
    return PSA_ERR_CUDA;
  int grid = sm_count(dev);
  if (grid <= 0) return PSA_ERR_CUDA;
  if (grid > a.T) grid = a.T;
  if (grid == 0) return PSA_OK;
  sparse_latent_kernel<<<grid, kThreads, SMEM, a.stream>>>(tq, p);
  return cudaGetLastError() == cudaSuccess ? PSA_OK : PSA_ERR_CUDA;
}

}  // namespace psa
