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
// The latent tile is gathered with 16-byte cp.async copies straight into
// the 128-byte-swizzled layout the MMA reads (eight threads per 128-byte
// row segment, zero fill for a -1 entry or an index past the latent).  Every
// part is spread over all 256 producer threads, four copies each, so a freed
// part refills after about one L2 round trip.  (Measured and not kept: the
// tensor-memory accelerator's four-row gather, one copy per four rows,
// stalls its issuing warp for over a thousand cycles per instruction.)  A
// part is released for the next tile as soon as the O^T block that reads it
// has completed, so the next tile's gather overlaps this tile's O^T.  Q_t^T
// arrives by TMA.
//   warps 0..7    gather producers, 32 rows per round of eight threads each
//                 (warp 0 also loads Q^T and publishes the tile count)
//   warp 8        tcgen05 issuer (one thread) and TMEM owner
//   warps 9..11   idle (they complete warp 8's register warpgroup)
//   warps 12..19  softmax over keys: TMEM lane quadrant (warp % 4) picks 32
//                 keys, warps 12..15 take heads 0..31 and warps 16..19 heads
//                 32..63; per-head max / sum reductions across lanes, P^T
//                 written to shared memory, lazy O^T rescaling, and the
//                 epilogue (one latent dimension per thread and M-block).
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "psa_device.cuh"
#include "psa_internal.h"

namespace psa {
namespace {

constexpr int DL = 512;          // latent width
constexpr int KT = 128;          // keys per tile (MMA M for S^T)
constexpr int NPART = DL / 64;   // 64-column parts of a latent tile
constexpr int HMAX = 64;         // heads per CTA pass (MMA N)
constexpr int HW = 32;           // heads per softmax warp
constexpr int kThreads = 640;
constexpr int kSoftmaxWarp0 = 12;     // first softmax warp (a warpgroup boundary)
constexpr int kSoftmaxThreads = 256;
constexpr int kMmaWarp = 8;
// Register split: 640 threads x 96 at launch = 61440.  The producer
// warpgroups (8 warps) drop to PROD and the MMA warpgroup (4 warps) to MMA,
// so each softmax thread can keep a key's 32 logits, 32 partial sums and the
// reduction scratch in registers: 8 x 32 x PROD + 4 x 32 x MMA + 8 x 32 x
// SOFTMAX must not exceed 61440.  The launcher checks the compiled register
// count against this before the first launch.
constexpr int kRegsProd = 48;
constexpr int kRegsMma = 64;
constexpr int kRegsSoftmax = 160;
constexpr int kRegsNeeded = 8 * 32 * kRegsProd + 4 * 32 * kRegsMma + 8 * 32 * kRegsSoftmax;
static_assert(kRegsNeeded <= 640 * 96, "register split exceeds the launch registers");
constexpr float kRescaleLog2 = 8.f;
constexpr uint32_t kTmemCols = 512;  // S^T at 0, O^T M-blocks at 128 + 64 * mb

constexpr uint32_t PART_BYTES = KT * 128;       // 16 KB
constexpr uint32_t QPART_BYTES = HMAX * 128;    // 8 KB
constexpr uint32_t OFF_LAT = 0;
constexpr uint32_t OFF_Q = OFF_LAT + NPART * PART_BYTES;     // 128 KB
constexpr uint32_t OFF_P = OFF_Q + NPART * QPART_BYTES;      // +64 KB
constexpr uint32_t OFF_RED = OFF_P + KT * 128;               // +16 KB
constexpr uint32_t RED_BYTES = 2 * 4 * HMAX * 4;             // max and sum: [4 quadrants][64]
constexpr uint32_t OFF_HEAD = OFF_RED + RED_BYTES;           // per-head state
constexpr uint32_t HEAD_BYTES = 4 * HMAX * 4;                // m, l, alpha, 1/l
constexpr uint32_t OFF_BAR = OFF_HEAD + HEAD_BYTES;
constexpr uint32_t NBAR = 2 * NPART + 2 + 6;
constexpr uint32_t SMEM = 1024 + OFF_BAR + NBAR * 8 + 64;

struct Params {
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

// Bounded wait as mbar_wait, retrying with the hardware's default
// try_wait time limit instead of a long suspend hint: a waiter here is on
// the critical path of the next tile and must resume as soon as the phase
// completes.
__device__ __forceinline__ bool mbar_wait_hot(uint64_t* bar, uint32_t parity,
                                              volatile int* abort_flag, int32_t* dev_status) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 63u) == 0) {
      if (*abort_flag) return false;
      if (globaltimer() - t0 > kWaitTimeoutNs) {
        *abort_flag = 1;
        report_status(dev_status, PSA_ERR_TIMEOUT);
        return false;
      }
    }
  }
}

// Reduces v[0..31] across the 32 lanes of the warp (max or sum); afterwards
// lane L holds the result for entry L.  Each step keeps the half of the
// entries its lane bit selects and folds in the partner's copy of them.
template <bool MAX>
__device__ __forceinline__ float warp_transpose_reduce32(const float (&v)[32], int lane) {
  float w16[16];
  {
    const bool hi = lane & 16;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const float mine = hi ? v[16 + i] : v[i];
      const float other = hi ? v[i] : v[16 + i];
      const float got = __shfl_xor_sync(0xffffffffu, other, 16);
      w16[i] = MAX ? fmaxf(mine, got) : mine + got;
    }
  }
  float w8[8];
  {
    const bool hi = lane & 8;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float mine = hi ? w16[8 + i] : w16[i];
      const float other = hi ? w16[i] : w16[8 + i];
      const float got = __shfl_xor_sync(0xffffffffu, other, 8);
      w8[i] = MAX ? fmaxf(mine, got) : mine + got;
    }
  }
  float w4[4];
  {
    const bool hi = lane & 4;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float mine = hi ? w8[4 + i] : w8[i];
      const float other = hi ? w8[i] : w8[4 + i];
      const float got = __shfl_xor_sync(0xffffffffu, other, 4);
      w4[i] = MAX ? fmaxf(mine, got) : mine + got;
    }
  }
  float w2[2];
  {
    const bool hi = lane & 2;
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const float mine = hi ? w4[2 + i] : w4[i];
      const float other = hi ? w4[i] : w4[2 + i];
      const float got = __shfl_xor_sync(0xffffffffu, other, 2);
      w2[i] = MAX ? fmaxf(mine, got) : mine + got;
    }
  }
  const bool hi = lane & 1;
  const float mine = hi ? w2[1] : w2[0];
  const float other = hi ? w2[0] : w2[1];
  const float got = __shfl_xor_sync(0xffffffffu, other, 1);
  return MAX ? fmaxf(mine, got) : mine + got;
}

__device__ __forceinline__ bool key_ok(int32_t k, int32_t Tk) { return k >= 0 && k < Tk; }

__device__ __forceinline__ void regs_dec_prod() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsProd) : "memory");
}
__device__ __forceinline__ void regs_dec_mma() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsMma) : "memory");
}
__device__ __forceinline__ void regs_inc_softmax() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsSoftmax) : "memory");
}

// The 32 per-head values v[h] - m[h] need the running maxima of this warp's
// heads: eight 16-byte shared loads instead of 32 scalar ones.
__device__ __forceinline__ void load_heads32(const float* src, float (&m)[32]) {
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float4 x = reinterpret_cast<const float4*>(src)[i];
    m[4 * i] = x.x;
    m[4 * i + 1] = x.y;
    m[4 * i + 2] = x.z;
    m[4 * i + 3] = x.w;
  }
}

__global__ void __launch_bounds__(kThreads, 1)
    sparse_latent_kernel(const __grid_constant__ CUtensorMap tmap_q, Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  __shared__ uint32_t tmem_base_slot;
  __shared__ int abort_flag;
  __shared__ int q_ntiles;
  __shared__ int over_tile;  // 1 + the last tile whose logits outgrew a running max

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
  uint64_t* part_full = bar;                 // [8] 256 producer copy arrivals
  uint64_t* part_empty = bar + NPART;        // [8] MMA commit
  uint64_t* q_full = bar + 2 * NPART;        // producer expect_tx (tile count) + TMA bytes
  uint64_t* q_empty = q_full + 1;            // MMA commit
  uint64_t* s_full = q_empty + 1;            // MMA commit
  uint64_t* p_full = s_full + 1;             // 8 softmax warps
  uint64_t* pv_done = p_full + 1;            // MMA commit
  uint64_t* o_full = pv_done + 1;            // MMA commit
  uint64_t* o_free = o_full + 1;             // 8 softmax warps
  uint64_t* grp = o_free + 1;                // the softmax group's rendezvous (8 warps)
  float* red_max = reinterpret_cast<float*>(smem + OFF_RED);  // [4 quadrants][64]
  float* red_sum = red_max + 4 * HMAX;                         // [4 quadrants][64]
  float* h_m = reinterpret_cast<float*>(smem + OFF_HEAD);  // running max (log2 domain)
  float* h_l = h_m + HMAX;                                 // running sum
  float* h_alpha = h_l + HMAX;                             // this tile's rescale factor
  float* h_inv = h_alpha + HMAX;                           // 1 / l for the epilogue
  __shared__ int h_flagw[2];                               // a head-owner warp rescaled

  if (threadIdx.x == 0) {
    abort_flag = 0;
    for (int i = 0; i < NPART; ++i) {
      mbar_init(part_full + i, 32 * kMmaWarp);  // every producer thread's copies
      mbar_init(part_empty + i, 1);
    }
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    mbar_init(s_full, 1);
    mbar_init(p_full, kSoftmaxThreads / 32);
    mbar_init(pv_done, 1);
    mbar_init(o_full, 1);
    mbar_init(o_free, kSoftmaxThreads / 32);
    mbar_init(grp, kSoftmaxThreads / 32);
    over_tile = 0;
    fence_barrier_init();
  }
  if (threadIdx.x >= 32 * kSoftmaxWarp0 && threadIdx.x < 32 * kSoftmaxWarp0 + HMAX)
    h_m[threadIdx.x - 32 * kSoftmaxWarp0] = -INFINITY;
  if (warp == kMmaWarp) {
    tmem_alloc(&tmem_base_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_slot;

  // queries heaviest first: the last rows have the longest index lists
  auto query_of = [&](int i) { return p.T - 1 - (int(blockIdx.x) + i * int(gridDim.x)); };

  if (warp < kMmaWarp) {
    regs_dec_prod();
    // ============================================================ producers
    // Thread pt copies the 16-byte piece pt % 8 of rows pt / 8 + 32 i
    // (i = 0..3) of every part: each warp instruction moves four whole
    // 128-byte row segments.
    const int pt = threadIdx.x;   // 0..255
    const int chunk = pt & 7;
    const int rsub = pt >> 3;     // 0..31
    if (warp == 0 && lane == 0) tma_prefetch_desc(&tmap_q);
    uint32_t tile_glob = 0;
    bool ok = true;
    for (int qi = 0; ok; ++qi) {
      const int t = query_of(qi);
      if (t < 0) break;
      const int32_t* qidx = p.idx + size_t(t) * p.topk;
      // the last listed row: 32-slot chunks scanned from the end (a full
      // list stops at the first chunk)
      int last = -1;
      for (int base = ((p.topk - 1) >> 5) << 5; base >= 0; base -= 32) {
        const int sl = base + lane;
        const bool v = sl < p.topk && key_ok(__ldg(qidx + sl), p.Tk);
        const uint32_t b = __ballot_sync(0xffffffffu, v);
        if (b) {
          last = base + 31 - __clz(b);
          break;
        }
      }
      const int ntiles = (last + KT) / KT;
      if (warp == 0) {
        int got = 1;
        if (lane == 0) got = mbar_wait_hot(q_empty, (qi & 1) ^ 1, &abort_flag, p.status) ? 1 : 0;
        if (!__shfl_sync(0xffffffffu, got, 0)) break;
        if (lane == 0) {
          q_ntiles = ntiles;  // published by the arrive below
          mbar_arrive_expect_tx(q_full, NPART * QPART_BYTES);
#pragma unroll
          for (int qp = 0; qp < NPART; ++qp)
            tma_load_2d(smem + OFF_Q + qp * QPART_BYTES, &tmap_q, q_full, qp * 64, t * p.H);
        }
        __syncwarp();
      }
      for (int j = 0; j < ntiles && ok; ++j, ++tile_glob) {
        const __nv_bfloat16* src[4];
        uint32_t sz[4];
#pragma unroll
        for (int it = 0; it < 4; ++it) {
          const int sl = j * KT + it * 32 + rsub;
          const int32_t k = sl < p.topk ? __ldg(qidx + sl) : -1;
          if (k >= p.Tk) report_status(p.status, PSA_ERR_INVALID_ARG);
          const bool valid = key_ok(k, p.Tk);
          src[it] = p.lat + size_t(valid ? k : 0) * DL + chunk * 8;
          sz[it] = valid ? 16u : 0u;  // zero fill for skipped slots
        }
        for (int part = 0; part < NPART; ++part) {
          int free_ok = 1;
          if (lane == 0)
            free_ok = mbar_wait_hot(part_empty + part, (tile_glob & 1) ^ 1, &abort_flag,
                                    p.status)
                          ? 1
                          : 0;
          if (!__shfl_sync(0xffffffffu, free_ok, 0)) {
            ok = false;
            break;
          }
          const uint32_t base = smem_u32(smem + OFF_LAT + part * PART_BYTES);
#pragma unroll
          for (int it = 0; it < 4; ++it) {
            const int row = it * 32 + rsub;
            cp_async16(base + row * 128 + ((chunk ^ (row & 7)) << 4), src[it] + part * 64,
                       sz[it]);
          }
          cp_async_arrive(part_full + part);
        }
      }
    }
    // let every copy this thread issued land before the CTA can exit
    asm volatile("cp.async.wait_all;" ::: "memory");
    if (!ok || abort_flag) {
      // give copies still in flight time to land before the CTA can exit
      const uint64_t t0 = globaltimer();
      while (globaltimer() - t0 < 1000000ull) {
      }
    }
  } else if (warp < kSoftmaxWarp0) {
    regs_dec_mma();
    // ============================================================ MMA issuer
    if (warp == kMmaWarp && lane == 0) {
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
        if (!mbar_wait_hot(q_full, qi & 1, &abort_flag, p.status)) break;
        const int ntiles = q_ntiles;
        if (ntiles == 0) {
          umma_commit(q_empty);
          continue;
        }
        for (int j = 0; j < ntiles && ok; ++j, ++tile_glob) {
          // S^T = Lat_tile . Q^T, accumulated over the eight parts
          for (int part = 0; part < NPART && ok; ++part) {
            if (!mbar_wait_hot(part_full + part, tile_glob & 1, &abort_flag, p.status)) {
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
          if (!mbar_wait_hot(p_full, tile_glob & 1, &abort_flag, p.status) ||
              (j == 0 && !mbar_wait_hot(o_free, (oq & 1) ^ 1, &abort_flag, p.status))) {
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
    regs_inc_softmax();
    // ============================================================ softmax + epilogue
    // One key per thread and 32 heads per warp.  The 64 running maxima (log2
    // domain) live in shared memory; each thread keeps its own 32 partial
    // row sums in registers.  A tile only needs a cross-key max when some
    // logit would exceed its head's running max by more than 2^8 (the first
    // tile of a query always does), detected with one OR-reduction barrier.
    // The partial sums meet once per query.
    const int quad = warp & 3;
    const int hb = ((warp - kSoftmaxWarp0) >> 2) * HW;  // first head of this warp
    const int r = quad * 32 + lane;  // key slot (TMEM lane); latent dim in the epilogue
    const int tid = threadIdx.x - 32 * kSoftmaxWarp0;  // 0..255 within the group
    const uint32_t trow = tmem + (uint32_t(quad * 32) << 16);
    uint32_t tile_glob = 0;
    uint32_t oq = 0;  // queries with at least one tile
    bool ok = true;
    // The group's rendezvous: an 8-warp mbarrier with the bounded wait, so
    // a member that gave up cannot leave the others waiting.
    uint32_t gphase = 0;
    auto group_sync = [&]() -> bool {
      __syncwarp();
      if (lane == 0) mbar_arrive(grp);
      const bool got = mbar_wait_hot(grp, gphase & 1, &abort_flag, p.status);
      ++gphase;
      return got;
    };
    for (int qi = 0; ok; ++qi) {
      const int t = query_of(qi);
      if (t < 0) break;
      const int32_t* qidx = p.idx + size_t(t) * p.topk;
      // index of this thread's key slot in tile 0, fetched before the wait
      int32_t kidx_next = r < p.topk ? __ldg(qidx + r) : -1;
      if (!mbar_wait_hot(q_full, qi & 1, &abort_flag, p.status)) break;
      const int ntiles = q_ntiles;
      float lpart[HW];
#pragma unroll
      for (int h = 0; h < HW; ++h) lpart[h] = 0.f;
      for (int j = 0; j < ntiles && ok; ++j, ++tile_glob) {
        const bool valid = key_ok(kidx_next, p.Tk);
        {
          const int sl = (j + 1) * KT + r;  // prefetch the next tile's index
          kidx_next = sl < p.topk ? __ldg(qidx + sl) : -1;
        }
        if (!mbar_wait_hot(s_full, tile_glob & 1, &abort_flag, p.status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        float v[HW];
        {
          uint32_t raw[HW];
          tmem_ld32(trow + hb, raw);
          tmem_wait_ld();
#pragma unroll
          for (int h = 0; h < HW; ++h)
            v[h] = valid ? __uint_as_float(raw[h]) * p.scale_log2 : -INFINITY;
        }
        // does any logit of this tile outgrow its head's running max?
        float over = -INFINITY;
        {
          float m[HW];
          load_heads32(h_m + hb, m);
#pragma unroll
          for (int h = 0; h < HW; ++h) over = fmaxf(over, v[h] - m[h]);
        }
        // the group's OR of "some logit outgrew its head's running max":
        // a warp that saw one marks this tile, then everyone meets
        if (__any_sync(0xffffffffu, over > kRescaleLog2) && lane == 0)
          atomicMax(&over_tile, int(tile_glob) + 1);
        if (!group_sync()) {
          ok = false;
          break;
        }
        const bool any_over = *(volatile int*)&over_tile == int(tile_glob) + 1;
        if (any_over) {
          // cross-key max per head: across lanes, then across quadrants
          red_max[quad * HMAX + hb + lane] = warp_transpose_reduce32<true>(v, lane);
          if (!group_sync()) {
            ok = false;
            break;
          }
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
            if (lane == 0) h_flagw[tid >> 5] = any ? 1 : 0;
          }
          if (!group_sync()) {
            ok = false;
            break;
          }
          {
            float a[HW];
            load_heads32(h_alpha + hb, a);
#pragma unroll
            for (int h = 0; h < HW; ++h) lpart[h] *= a[h];
            if (h_flagw[0] | h_flagw[1]) {
              // lazy O^T rescale: column h of every M-block times alpha_h,
              // once the previous O^T product has landed
              if (!mbar_wait_hot(pv_done, (tile_glob - 1) & 1, &abort_flag, p.status)) {
                ok = false;
                break;
              }
              tc_fence_after();
#pragma unroll 1
              for (int mb = 0; mb < 4; ++mb) {
                uint32_t ov[HW];
                tmem_ld32(trow + 128 + mb * 64 + hb, ov);
                tmem_wait_ld();
#pragma unroll
                for (int h = 0; h < HW; ++h)
                  ov[h] = __float_as_uint(__uint_as_float(ov[h]) * a[h]);
                tmem_st32(trow + 128 + mb * 64 + hb, ov);
              }
              tmem_wait_st();
            }
          }
        }
        // P^T row of this key: exp2(s * scale - m_h)
        {
          float m[HW];
          load_heads32(h_m + hb, m);
#pragma unroll
          for (int h = 0; h < HW; ++h) {
            v[h] = fast_exp2(v[h] - (m[h] == -INFINITY ? 0.f : m[h]));
            lpart[h] += v[h];
          }
        }
        // the previous O^T product must be done before P^T is overwritten
        if (j > 0 && !mbar_wait_hot(pv_done, (tile_glob - 1) & 1, &abort_flag, p.status)) {
          ok = false;
          break;
        }
        {
          // this warp's 32 heads are 16-byte chunks hb/8 .. hb/8 + 3 of the
          // key's 128-byte P^T row (128-byte swizzle)
          const uint32_t prow = smem_u32(smem + OFF_P) + r * 128;
#pragma unroll
          for (int c = 0; c < HW / 8; ++c) {
            const uint32_t w0 = pack_bf16(v[8 * c], v[8 * c + 1]);
            const uint32_t w1 = pack_bf16(v[8 * c + 2], v[8 * c + 3]);
            const uint32_t w2 = pack_bf16(v[8 * c + 4], v[8 * c + 5]);
            const uint32_t w3 = pack_bf16(v[8 * c + 6], v[8 * c + 7]);
            const int chunk = hb / 8 + c;
            asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(
                             prow + ((chunk ^ (r & 7)) << 4)),
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
      red_sum[quad * HMAX + hb + lane] = warp_transpose_reduce32<false>(lpart, lane);
      if (!group_sync()) {
        ok = false;
        break;
      }
      if (tid < HMAX) {
        const float l = (red_sum[tid] + red_sum[HMAX + tid]) +
                        (red_sum[2 * HMAX + tid] + red_sum[3 * HMAX + tid]);
        h_l[tid] = l;
        h_inv[tid] = l > 0.f ? 1.f / l : 0.f;
      }
      if (!group_sync()) break;  // h_l, h_inv final
      if (ntiles > 0) {
        if (!mbar_wait_hot(o_full, oq & 1, &abort_flag, p.status)) break;
        tc_fence_after();
      }
      // epilogue: per M-block, thread d = r scales its O^T lane by 1/l_h for
      // its warp's heads and stages it as [head][128 dims] in the (now idle)
      // P^T buffer; the block then goes out as contiguous 16-byte rows.
      __nv_bfloat16* stage = reinterpret_cast<__nv_bfloat16*>(smem + OFF_P);
      float inv[HW];
      load_heads32(h_inv + hb, inv);
#pragma unroll 1
      for (int mb = 0; mb < 4; ++mb) {
        uint32_t ov[HW];
        if (ntiles > 0) {
          tmem_ld32(trow + 128 + mb * 64 + hb, ov);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int h = 0; h < HW; ++h) ov[h] = 0u;
        }
#pragma unroll
        for (int h = 0; h < HW; ++h)
          stage[(hb + h) * 128 + r] = __float2bfloat16(__uint_as_float(ov[h]) * inv[h]);
        if (!group_sync()) {
          ok = false;
          break;
        }
#pragma unroll
        for (int k = 0; k < (HMAX * 16) / kSoftmaxThreads; ++k) {
          const int c = k * kSoftmaxThreads + tid;  // 16-byte chunk: head c / 16, piece c % 16
          const int h = c >> 4, piece = c & 15;
          if (h < p.H)
            *reinterpret_cast<uint4*>(p.o + (size_t(t) * p.H + h) * DL + mb * 128 + piece * 8) =
                *reinterpret_cast<const uint4*>(stage + h * 128 + piece * 8);
        }
        if (!group_sync()) {
          ok = false;
          break;
        }
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
      if (!group_sync()) {
        ok = false;
        break;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kMmaWarp) tmem_dealloc(tmem, kTmemCols);
}

}  // namespace

int launch_sparse_latent(const SparseArgs& a) {
  if (a.dl != DL || a.H > HMAX || a.H <= 0) return PSA_ERR_UNSUPPORTED;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return PSA_ERR_CUDA;
  Params p;
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
    // Q_t^T: rows (token, head), 64-column boxes of 64 head rows
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
  {
    // setmaxnreg.inc waits until the block's launch registers cover the
    // split, so a build with fewer registers per thread must not launch
    cudaFuncAttributes fa;
    if (cudaFuncGetAttributes(&fa, sparse_latent_kernel) != cudaSuccess) return PSA_ERR_CUDA;
    if (fa.numRegs * kThreads < kRegsNeeded) return PSA_ERR_UNSUPPORTED;
  }
  int grid = sm_count(dev);
  if (grid <= 0) return PSA_ERR_CUDA;
  if (grid > a.T) grid = a.T;
  if (grid == 0) return PSA_OK;
  sparse_latent_kernel<<<grid, kThreads, SMEM, a.stream>>>(tq, p);
  return cudaGetLastError() == cudaSuccess ? PSA_OK : PSA_ERR_CUDA;
}

}  // namespace psa
