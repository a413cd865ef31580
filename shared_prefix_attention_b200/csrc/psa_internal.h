// Internal launchers shared between the C-ABI layer (psa_api.cpp) and the
// kernel translation units.  Not part of the public ABI.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "psa.h"

namespace psa {

// Encodes a tiled TMA descriptor through the driver entry point (no link
// dependency on libcuda).  rank <= 5; dims/strides innermost first; strides
// are in bytes for dims 1..rank-1.  Returns PSA_OK or PSA_ERR_CUDA.
int encode_tmap(CUtensorMap* map, CUtensorMapDataType dtype, int rank, const void* base,
                const uint64_t* dims, const uint64_t* strides_bytes, const uint32_t* box,
                CUtensorMapSwizzle swizzle);

int sm_count(int device);

// ---------------------------------------------------------------- verify

struct VerifyArgs {
  const void* q;
  const void* kd;
  const void* vd;
  const void* kc;
  const void* vc;
  const int32_t* indptr;
  int64_t n_cache_tokens;
  void* o;
  float* lse;
  int32_t B, Ld, Hq, Hkv, D;
  float scale;
  int32_t nsplit;
  float* part_o;    // [nsplit][B*Ld][Hq][D]
  float* part_lse;  // [nsplit][B*Ld][Hq], log2 domain
  int32_t* status;
  cudaStream_t stream;
  const uint8_t* dmask = nullptr;  // tree verify: [B*Ld, Ld] draft mask (device)
  // Extend form (all null for uniform draft counts and a contiguous prefix):
  const int32_t* kv_indices = nullptr;   // prefix position t -> cache row kv_indices[t]
  const int32_t* qo_indptr = nullptr;    // [B+1] draft rows per request; Ld is their maximum
  const int32_t* mask_indptr = nullptr;  // [B+1] start of request b's Lb x Lb mask in dmask
  int32_t n_rows = 0;                    // draft rows in all (qo_indptr[B]); B*Ld when uniform
};

// KV heads per CTA, 16-row m-tiles per CTA and row blocks per KV head;
// returns 0 if the shape is unsupported.
int verify_plan(int32_t Ld, int32_t Hq, int32_t Hkv, int32_t D, int32_t* heads_per_block,
                int32_t* mtiles, int32_t* row_blocks);
int launch_verify(const VerifyArgs& a);
// Stage 2 alone: merge a.nsplit partials with the causal draft block.
int launch_verify_combine(const VerifyArgs& a);
// The verify with e4m3 caches in a.kc / a.vc (head_dim 128): cached key =
// k_scale * e4m3, cached value = v_scale * e4m3.
int launch_verify_fp8(const VerifyArgs& a, float k_scale, float v_scale);

// Verify against one prefix shared by every request.
struct VerifySharedArgs {
  const void* q;   // bf16 [B*Ld, Hq, D]
  const void* kd;  // bf16 [B*Ld, Hkv, D]
  const void* vd;
  const void* kp;  // bf16 [L, Hkv, D], the shared prefix
  const void* vp;
  int64_t L;
  void* o;
  float* lse;
  int32_t B, Ld, Hq, Hkv, D;
  float scale;
  int32_t nsplit, chunk;  // chunk: prefix keys per split, a multiple of 128
  float* part_o;          // [nsplit][B*Ld][Hq][D]
  float* part_lse;        // [nsplit][B*Ld][Hq], log2 domain
  int32_t* status;
  cudaStream_t stream;
  const uint8_t* dmask = nullptr;  // tree verify: [B*Ld, Ld] draft mask (device)
};
int launch_verify_shared(const VerifySharedArgs& a);

// ---------------------------------------------------------------- prefill

struct PrefillArgs {
  const void* q;  // bf16 [T, Hq, D]
  const void* k;  // bf16 [T, Hkv, D]
  const void* v;
  void* o;        // [T, Hq, D], bf16, or fp32 when out_f32 (then q/k/v are fp32 too)
  bool out_f32;
  float* lse;
  int32_t T, Hq, Hkv, D;
  float scale;
  const int32_t* sched;  // device copy of a psa_build_schedule result
  int64_t sched_len;
  int32_t* counter;      // device word for the dynamic tile scheduler
  int32_t* status;
  cudaStream_t stream;
};
int launch_prefill(const PrefillArgs& a);

// ---------------------------------------------------------------- backward

struct BackwardArgs {
  const void* q;     // bf16 [T, Hq, D]
  const void* k;     // bf16 [T, Hkv, D]
  const void* v;
  const void* o;     // bf16 [T, Hq, D], the forward output
  const float* lse;  // [T, Hq], natural log, the forward's
  const void* dout;  // bf16 [T, Hq, D]
  void* dq;          // bf16 [T, Hq, D] (written)
  void* dk;          // bf16 [T, Hkv, D] (written)
  void* dv;
  int32_t T, Hq, Hkv, D;
  float scale;
  const int32_t* sched_q;   // psa_build_schedule(spec, ...), blocks of 128 rows, tiles of 64
  int64_t sched_q_len;
  const int32_t* sched_kv;  // psa_build_schedule(transposed spec, ...), same tile sizes
  int64_t sched_kv_len;
  float* lse2_t;            // workspace [Hq, Tp], -LSE * log2(e); Tp = T rounded up to 4
  float* delta_t;           // workspace [Hq, Tp], -rowsum(dO * O)
  int32_t* status;
  cudaStream_t stream;
};
int launch_backward(const BackwardArgs& a);

// ---------------------------------------------------------------- sparse latent

struct SparseArgs {
  const void* q;       // bf16 [T, H, dl]
  const void* latent;  // bf16 [Tk, dl]
  const int32_t* idx;  // [T, topk]
  void* o;
  float* lse;
  int32_t T, Tk, H, dl, topk;
  float scale;
  int32_t* status;
  cudaStream_t stream;
};
int launch_sparse_latent(const SparseArgs& a);

}  // namespace psa
