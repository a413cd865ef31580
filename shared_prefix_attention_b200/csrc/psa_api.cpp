// C-ABI layer of libpsa: argument validation, workspace sizing and kernel
// launches.  No allocation, no host synchronisation (psa_read_status
// excepted), no fallback: an unsupported case returns PSA_ERR_UNSUPPORTED.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "psa.h"
#include "psa_internal.h"

namespace psa {

namespace {

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

int encode_tmap(CUtensorMap* map, CUtensorMapDataType dtype, int rank, const void* base,
                const uint64_t* dims, const uint64_t* strides_bytes, const uint32_t* box,
                CUtensorMapSwizzle swizzle) {
  EncodeTiledFn fn = get_encode_fn();
  if (!fn) return PSA_ERR_CUDA;
  cuuint64_t d[5], st[4];
  cuuint32_t bx[5], es[5];
  for (int i = 0; i < rank; ++i) {
    d[i] = dims[i];
    bx[i] = box[i];
    es[i] = 1;
  }
  for (int i = 0; i + 1 < rank; ++i) st[i] = strides_bytes[i];
  CUresult r = fn(map, dtype, cuuint32_t(rank), const_cast<void*>(base), d, st, bx, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? PSA_OK : PSA_ERR_CUDA;
}

int sm_count(int device) {
  static int cached[64] = {0};
  if (device < 0 || device >= 64) return 0;
  if (cached[device] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, device) != cudaSuccess)
      return 0;
    cached[device] = n;
  }
  return cached[device];
}

}  // namespace psa

using namespace psa;

extern "C" int psa_version(void) { return PSA_VERSION; }

extern "C" const char* psa_status_string(int status) {
  switch (status) {
    case PSA_OK:
      return "ok";
    case PSA_ERR_INVALID_ARG:
      return "invalid argument";
    case PSA_ERR_UNSUPPORTED:
      return "unsupported case (no fallback path exists)";
    case PSA_ERR_WORKSPACE:
      return "workspace missing or too small";
    case PSA_ERR_CUDA:
      return "CUDA call failed";
    case PSA_ERR_TIMEOUT:
      return "device-side wait timed out";
    case PSA_ERR_CAPACITY:
      return "output capacity too small";
    case PSA_ERR_BOUNDS:
      return "device bounds check failed (debug build)";
    default:
      return "unknown status";
  }
}

extern "C" int psa_read_status(const int32_t* dev_status, int32_t* host_out, void* stream) {
  if (!dev_status || !host_out) return PSA_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaMemcpyAsync(host_out, dev_status, sizeof(int32_t), cudaMemcpyDeviceToHost, s) !=
      cudaSuccess)
    return PSA_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return PSA_ERR_CUDA;
  return PSA_OK;
}

// ------------------------------------------------------------------ verify

extern "C" int32_t psa_verify_auto_splits(int32_t B, int64_t max_prefix_len, int32_t Hkv,
                                          int32_t head_dim) {
  (void)Hkv;
  (void)head_dim;
  if (B <= 0 || max_prefix_len <= 0) return 1;
  // Aim for about four (request, split) units per SM of a 148-SM part, but
  // keep every split at least 256 keys long so each unit streams enough.
  const int64_t target_units = 4 * 148;
  int64_t n = (target_units + B - 1) / B;
  const int64_t by_len = max_prefix_len / 256;
  if (n > by_len) n = by_len;
  if (n < 1) n = 1;
  if (n > 256) n = 256;
  return int32_t(n);
}

extern "C" size_t psa_verify_workspace_size(int32_t B, int32_t Ld, int32_t Hq,
                                            int32_t head_dim, int32_t nsplit) {
  if (B <= 0 || Ld <= 0 || Hq <= 0 || head_dim <= 0 || nsplit <= 0) return 0;
  const size_t rows = size_t(nsplit) * B * Ld * Hq;
  const size_t o_bytes = (rows * head_dim * sizeof(float) + 255) / 256 * 256;
  const size_t l_bytes = (rows * sizeof(float) + 255) / 256 * 256;
  return o_bytes + l_bytes;
}

static int verify_common(const void* q_draft, const void* k_draft, const void* v_draft,
                              const void* k_cache, const void* v_cache, int64_t n_cache_tokens,
                              const int32_t* dev_kv_indptr, int64_t max_prefix_len,
                              const int32_t* kv_indices, void* o, float* lse, int32_t B,
                              int32_t Ld, int32_t Hq, int32_t Hkv, int32_t head_dim, float scale,
                              int32_t nsplit, const psa_verify_features* features,
                              void* workspace, size_t ws_bytes, int32_t* dev_status,
                              void* stream, const uint8_t* dmask,
                              const int32_t* qo_indptr = nullptr, int32_t n_rows = 0,
                              const int32_t* mask_indptr = nullptr,
                              const psa_kv_scales* e4m3 = nullptr) {
  // The split-KV path's gating ("can_handle"): everything else is refused;
  // a custom draft mask only through the entries that pass dmask, ragged
  // draft counts only through the extend entry, which passes qo_indptr.
  if (features) {
    if ((features->has_custom_mask && !dmask) || !features->is_causal ||
        features->sliding_window > 0 ||
        features->has_sinks || features->logit_cap != 0.f ||
        features->xai_temperature_len > 0 || (features->ragged_extend && !qo_indptr))
      return PSA_ERR_UNSUPPORTED;
  }
  if (B < 0 || Ld <= 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || n_cache_tokens < 0 ||
      max_prefix_len < 0 || n_cache_tokens > INT32_MAX || !(scale > 0.f))
    return PSA_ERR_INVALID_ARG;
  // rows of the partials: every draft row once
  const int64_t rows_all = qo_indptr ? int64_t(n_rows) : int64_t(B) * Ld;
  if (qo_indptr && (n_rows < 0 || int64_t(n_rows) > int64_t(B) * Ld)) return PSA_ERR_INVALID_ARG;
  if (rows_all * Hq > INT32_MAX) return PSA_ERR_INVALID_ARG;
  if (e4m3 && (!(e4m3->k_scale > 0.f) || !(e4m3->v_scale > 0.f) ||
               !std::isfinite(e4m3->k_scale) || !std::isfinite(e4m3->v_scale)))
    return PSA_ERR_INVALID_ARG;
  if (e4m3 ? head_dim != 128 : (head_dim != 64 && head_dim != 128 && head_dim != 256))
    return PSA_ERR_UNSUPPORTED;
  if (B == 0 || rows_all == 0) return PSA_OK;
  if (!q_draft || !k_draft || !v_draft || !k_cache || !v_cache || !dev_kv_indptr || !o)
    return PSA_ERR_INVALID_ARG;
  if (!aligned16(q_draft) || !aligned16(k_draft) || !aligned16(v_draft) ||
      !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(o) ||
      (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)))
    return PSA_ERR_INVALID_ARG;
  int32_t HB = 0, MT = 0, NRB = 0;
  if (!verify_plan(Ld, Hq, Hkv, head_dim, &HB, &MT, &NRB)) return PSA_ERR_UNSUPPORTED;
  if (nsplit == 0) nsplit = psa_verify_auto_splits(B, max_prefix_len, Hkv, head_dim);
  if (nsplit < 1 || nsplit > 256) return PSA_ERR_INVALID_ARG;
  const size_t need = psa_verify_workspace_size(1, int32_t(rows_all), Hq, head_dim, nsplit);
  if (!workspace || ws_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return PSA_ERR_WORKSPACE;

  VerifyArgs a;
  a.q = q_draft;
  a.kd = k_draft;
  a.vd = v_draft;
  a.kc = k_cache;
  a.vc = v_cache;
  a.indptr = dev_kv_indptr;
  a.n_cache_tokens = n_cache_tokens;
  a.o = o;
  a.lse = lse;
  a.B = B;
  a.Ld = Ld;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.D = head_dim;
  a.scale = scale;
  a.nsplit = nsplit;
  const size_t rows = size_t(nsplit) * size_t(rows_all) * Hq;
  const size_t o_bytes = (rows * head_dim * sizeof(float) + 255) / 256 * 256;
  a.part_o = static_cast<float*>(workspace);
  a.part_lse = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + o_bytes);
  a.status = dev_status;
  a.stream = static_cast<cudaStream_t>(stream);
  a.dmask = dmask;
  a.kv_indices = kv_indices;
  a.qo_indptr = qo_indptr;
  a.mask_indptr = mask_indptr;
  a.n_rows = int32_t(rows_all);
  return e4m3 ? launch_verify_fp8(a, e4m3->k_scale, e4m3->v_scale) : launch_verify(a);
}

extern "C" int psa_verify_fwd(const void* q_draft, const void* k_draft, const void* v_draft,
                              const void* k_cache, const void* v_cache, int64_t n_cache_tokens,
                              const int32_t* dev_kv_indptr, int64_t max_prefix_len,
                              const int32_t* kv_indices, void* o, float* lse, int32_t B,
                              int32_t Ld, int32_t Hq, int32_t Hkv, int32_t head_dim, float scale,
                              int32_t nsplit, const psa_verify_features* features,
                              void* workspace, size_t ws_bytes, int32_t* dev_status,
                              void* stream) {
  return verify_common(q_draft, k_draft, v_draft, k_cache, v_cache, n_cache_tokens,
                       dev_kv_indptr, max_prefix_len, kv_indices, o, lse, B, Ld, Hq, Hkv,
                       head_dim, scale, nsplit, features, workspace, ws_bytes, dev_status, stream,
                       nullptr);
}

extern "C" int psa_verify_tree_fwd(const void* q_draft, const void* k_draft, const void* v_draft,
                                   const void* k_cache, const void* v_cache,
                                   int64_t n_cache_tokens, const int32_t* dev_kv_indptr,
                                   int64_t max_prefix_len, const int32_t* kv_indices,
                                   const uint8_t* dev_draft_mask, void* o, float* lse, int32_t B,
                                   int32_t Ld, int32_t Hq, int32_t Hkv, int32_t head_dim,
                                   float scale, int32_t nsplit,
                                   const psa_verify_features* features, void* workspace,
                                   size_t ws_bytes, int32_t* dev_status, void* stream) {
  if (B > 0 && !dev_draft_mask) return PSA_ERR_INVALID_ARG;
  return verify_common(q_draft, k_draft, v_draft, k_cache, v_cache, n_cache_tokens,
                       dev_kv_indptr, max_prefix_len, kv_indices, o, lse, B, Ld, Hq, Hkv,
                       head_dim, scale, nsplit, features, workspace, ws_bytes, dev_status, stream,
                       dev_draft_mask);
}

extern "C" int psa_verify_extend_fwd(
    const void* q_draft, const void* k_draft, const void* v_draft, const void* k_cache,
    const void* v_cache, int64_t n_cache_tokens, const int32_t* dev_qo_indptr, int32_t n_rows,
    int32_t max_draft_len, const int32_t* dev_kv_indptr, int64_t max_prefix_len,
    const int32_t* dev_kv_indices, const uint8_t* dev_draft_mask,
    const int32_t* dev_mask_indptr, const psa_kv_scales* e4m3_scales, void* o, float* lse,
    int32_t B, int32_t Hq, int32_t Hkv,
    int32_t head_dim, float scale, int32_t nsplit, const psa_verify_features* features,
    void* workspace, size_t ws_bytes, int32_t* dev_status, void* stream) {
  if (B > 0 && !dev_qo_indptr) return PSA_ERR_INVALID_ARG;
  if (dev_draft_mask && !dev_mask_indptr) return PSA_ERR_INVALID_ARG;
  return verify_common(q_draft, k_draft, v_draft, k_cache, v_cache, n_cache_tokens,
                       dev_kv_indptr, max_prefix_len, dev_kv_indices, o, lse, B, max_draft_len,
                       Hq, Hkv, head_dim, scale, nsplit, features, workspace, ws_bytes,
                       dev_status, stream, dev_draft_mask, B > 0 ? dev_qo_indptr : nullptr,
                       n_rows, dev_mask_indptr, e4m3_scales);
}

extern "C" int psa_verify_fp8_fwd(const void* q_draft, const void* k_draft, const void* v_draft,
                                  const void* k_cache, const void* v_cache,
                                  int64_t n_cache_tokens, const int32_t* dev_kv_indptr,
                                  int64_t max_prefix_len, const int32_t* kv_indices,
                                  float k_scale, float v_scale, void* o, float* lse, int32_t B,
                                  int32_t Ld, int32_t Hq, int32_t Hkv, int32_t head_dim,
                                  float scale, int32_t nsplit,
                                  const psa_verify_features* features, void* workspace,
                                  size_t ws_bytes, int32_t* dev_status, void* stream) {
  const psa_kv_scales sc{k_scale, v_scale};
  return verify_common(q_draft, k_draft, v_draft, k_cache, v_cache, n_cache_tokens,
                       dev_kv_indptr, max_prefix_len, kv_indices, o, lse, B, Ld, Hq, Hkv,
                       head_dim, scale, nsplit, features, workspace, ws_bytes, dev_status, stream,
                       nullptr, nullptr, 0, nullptr, &sc);
}

// ------------------------------------------------------- shared-prefix verify

extern "C" int32_t psa_verify_shared_auto_splits(int32_t B, int32_t Ld, int32_t Hq,
                                                 int32_t Hkv, int64_t prefix_len) {
  if (B <= 0 || Ld <= 0 || Hkv <= 0 || Hq <= 0 || prefix_len <= 0) return 1;
  // One wave of units (chunk, KV head, 256-row block) on a 148-SM part:
  // a unit's fixed cost (Q load, epilogue) is high, so fewer, longer units
  // beat more waves; every chunk keeps at least four 128-key tiles.
  const int64_t rows = int64_t(B) * Ld * (Hq / Hkv);
  const int64_t per_split = int64_t(Hkv) * ((rows + 255) / 256);
  int64_t n = 148 / per_split;
  const int64_t by_len = prefix_len / 512;
  if (n > by_len) n = by_len;
  if (n < 1) n = 1;
  if (n > 256) n = 256;
  return int32_t(n);
}

static int verify_shared_common(const void* q_draft, const void* k_draft, const void* v_draft,
                                const void* k_prefix, const void* v_prefix, int64_t prefix_len,
                                void* o, float* lse, int32_t B, int32_t Ld, int32_t Hq,
                                int32_t Hkv, int32_t head_dim, float scale, int32_t nsplit,
                                void* workspace, size_t ws_bytes, int32_t* dev_status,
                                void* stream, const uint8_t* dmask) {
  if (B < 0 || Ld <= 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || prefix_len < 0 ||
      prefix_len > (int64_t(1) << 30) || !(scale > 0.f))
    return PSA_ERR_INVALID_ARG;
  if (head_dim != 64 && head_dim != 128) return PSA_ERR_UNSUPPORTED;
  // the combine holds a row's draft block in one warp's registers
  if (Ld > 16) return PSA_ERR_UNSUPPORTED;
  const int32_t G = Hq / Hkv;
  if (G > 128 || 128 % G != 0) return PSA_ERR_UNSUPPORTED;  // 128-row halves of whole tokens
  if (int64_t(B) * Ld > INT32_MAX / Hq) return PSA_ERR_INVALID_ARG;
  if (B == 0) return PSA_OK;
  if (!q_draft || !k_draft || !v_draft || !o) return PSA_ERR_INVALID_ARG;
  if (prefix_len > 0 && (!k_prefix || !v_prefix)) return PSA_ERR_INVALID_ARG;
  if (!aligned16(q_draft) || !aligned16(k_draft) || !aligned16(v_draft) || !aligned16(o) ||
      (prefix_len > 0 && (!aligned16(k_prefix) || !aligned16(v_prefix))) ||
      (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)))
    return PSA_ERR_INVALID_ARG;
  if (nsplit == 0) nsplit = psa_verify_shared_auto_splits(B, Ld, Hq, Hkv, prefix_len);
  if (nsplit < 1 || nsplit > 256) return PSA_ERR_INVALID_ARG;
  const size_t need = psa_verify_workspace_size(B, Ld, Hq, head_dim, nsplit);
  if (!workspace || ws_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return PSA_ERR_WORKSPACE;

  VerifySharedArgs a;
  a.q = q_draft;
  a.kd = k_draft;
  a.vd = v_draft;
  a.kp = k_prefix;
  a.vp = v_prefix;
  a.L = prefix_len;
  a.o = o;
  a.lse = lse;
  a.B = B;
  a.Ld = Ld;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.D = head_dim;
  a.scale = scale;
  a.nsplit = nsplit;
  // whole 128-key tiles per chunk; trailing chunks may be empty
  const int64_t per = (prefix_len + nsplit - 1) / nsplit;
  a.chunk = int32_t((per + 127) / 128 * 128);
  const size_t rows = size_t(nsplit) * B * Ld * Hq;
  const size_t o_bytes = (rows * head_dim * sizeof(float) + 255) / 256 * 256;
  a.part_o = static_cast<float*>(workspace);
  a.part_lse = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + o_bytes);
  a.status = dev_status;
  a.stream = static_cast<cudaStream_t>(stream);
  a.dmask = dmask;
  return launch_verify_shared(a);
}

extern "C" int psa_verify_shared_fwd(const void* q_draft, const void* k_draft,
                                     const void* v_draft, const void* k_prefix,
                                     const void* v_prefix, int64_t prefix_len, void* o,
                                     float* lse, int32_t B, int32_t Ld, int32_t Hq, int32_t Hkv,
                                     int32_t head_dim, float scale, int32_t nsplit,
                                     void* workspace, size_t ws_bytes, int32_t* dev_status,
                                     void* stream) {
  return verify_shared_common(q_draft, k_draft, v_draft, k_prefix, v_prefix, prefix_len, o, lse,
                              B, Ld, Hq, Hkv, head_dim, scale, nsplit, workspace, ws_bytes,
                              dev_status, stream, nullptr);
}

extern "C" int psa_verify_shared_tree_fwd(const void* q_draft, const void* k_draft,
                                          const void* v_draft, const void* k_prefix,
                                          const void* v_prefix, int64_t prefix_len,
                                          const uint8_t* dev_draft_mask, void* o, float* lse,
                                          int32_t B, int32_t Ld, int32_t Hq, int32_t Hkv,
                                          int32_t head_dim, float scale, int32_t nsplit,
                                          void* workspace, size_t ws_bytes, int32_t* dev_status,
                                          void* stream) {
  if (B > 0 && !dev_draft_mask) return PSA_ERR_INVALID_ARG;
  return verify_shared_common(q_draft, k_draft, v_draft, k_prefix, v_prefix, prefix_len, o, lse,
                              B, Ld, Hq, Hkv, head_dim, scale, nsplit, workspace, ws_bytes,
                              dev_status, stream, dev_draft_mask);
}

// ------------------------------------------------------------------ backward

extern "C" int psa_prefill_bwd_tiles(int32_t head_dim, int32_t* tile_m, int32_t* tile_n) {
  if (!tile_m || !tile_n) return PSA_ERR_INVALID_ARG;
  if (head_dim != 64 && head_dim != 128) return PSA_ERR_UNSUPPORTED;
  *tile_m = 128;  // two halves of 64 rows (keys in the transposed schedule)
  *tile_n = 64;
  return PSA_OK;
}

extern "C" size_t psa_prefill_bwd_workspace_size(int32_t T, int32_t Hq) {
  if (T <= 0 || Hq <= 0) return 0;
  const size_t tp = (size_t(T) + 3) / 4 * 4;
  return 2 * ((tp * Hq * sizeof(float) + 255) / 256 * 256);
}

extern "C" int psa_prefill_bwd(const void* q, const void* k, const void* v, const void* o,
                               const float* lse, const void* dout, void* dq, void* dk, void* dv,
                               int32_t T, int32_t Hq, int32_t Hkv, int32_t head_dim, float scale,
                               const int32_t* dev_schedule, int64_t sched_len,
                               const int32_t* dev_schedule_kv, int64_t sched_kv_len,
                               void* workspace, size_t ws_bytes, int32_t* dev_status,
                               void* stream) {
  if (T < 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || !(scale > 0.f))
    return PSA_ERR_INVALID_ARG;
  if (head_dim != 64 && head_dim != 128) return PSA_ERR_UNSUPPORTED;
  if (T == 0) return PSA_OK;
  if (!q || !k || !v || !o || !lse || !dout || !dq || !dk || !dv || !dev_schedule ||
      !dev_schedule_kv || sched_len < 8 || sched_kv_len < 8)
    return PSA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(dout) ||
      !aligned16(dq) || !aligned16(dk) || !aligned16(dv) ||
      (reinterpret_cast<uintptr_t>(lse) & 3u))
    return PSA_ERR_INVALID_ARG;
  const size_t need = psa_prefill_bwd_workspace_size(T, Hq);
  if (!workspace || ws_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return PSA_ERR_WORKSPACE;
  BackwardArgs a;
  a.q = q;
  a.k = k;
  a.v = v;
  a.o = o;
  a.lse = lse;
  a.dout = dout;
  a.dq = dq;
  a.dk = dk;
  a.dv = dv;
  a.T = T;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.D = head_dim;
  a.scale = scale;
  a.sched_q = dev_schedule;
  a.sched_q_len = sched_len;
  a.sched_kv = dev_schedule_kv;
  a.sched_kv_len = sched_kv_len;
  a.lse2_t = static_cast<float*>(workspace);
  a.delta_t = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + need / 2);
  a.status = dev_status;
  a.stream = static_cast<cudaStream_t>(stream);
  return launch_backward(a);
}

// ------------------------------------------------------------------ prefill

extern "C" int psa_prefill_tiles(int32_t head_dim, int32_t* tile_m, int32_t* tile_n) {
  if (!tile_m || !tile_n) return PSA_ERR_INVALID_ARG;
  if (head_dim != 64 && head_dim != 128) return PSA_ERR_UNSUPPORTED;
  *tile_m = 256;  // two 128-row halves per block
  *tile_n = 128;
  return PSA_OK;
}

extern "C" size_t psa_prefill_workspace_size(int dtype, int32_t T, int32_t Hq, int32_t Hkv,
                                             int32_t head_dim) {
  (void)dtype;
  (void)T;
  (void)Hq;
  (void)Hkv;
  (void)head_dim;
  return 256;  // the tile scheduler's counter
}

extern "C" int psa_prefill_fwd(const void* q, const void* k, const void* v, void* o,
                               float* lse, int dtype, int32_t T, int32_t Hq, int32_t Hkv,
                               int32_t head_dim, float scale, const int32_t* dev_schedule,
                               int64_t sched_len, void* workspace, size_t ws_bytes,
                               int32_t* dev_status, void* stream) {
  if (dtype != PSA_BF16 && dtype != PSA_F32) return PSA_ERR_INVALID_ARG;
  if (T < 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || !(scale > 0.f))
    return PSA_ERR_INVALID_ARG;
  if (head_dim != 64 && head_dim != 128) return PSA_ERR_UNSUPPORTED;
  if (T == 0) return PSA_OK;
  if (!q || !k || !v || !o || !dev_schedule || sched_len < 8) return PSA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) ||
      !aligned16(dev_schedule) || (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)))
    return PSA_ERR_INVALID_ARG;
  const size_t need = psa_prefill_workspace_size(dtype, T, Hq, Hkv, head_dim);
  if (!workspace || ws_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return PSA_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);

  PrefillArgs a;
  a.q = q;
  a.k = k;
  a.v = v;
  a.o = o;
  a.out_f32 = dtype == PSA_F32;
  a.lse = lse;
  a.T = T;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.D = head_dim;
  a.scale = scale;
  a.sched = dev_schedule;
  a.sched_len = sched_len;
  a.status = dev_status;
  a.stream = s;
  a.counter = static_cast<int32_t*>(workspace);
  return launch_prefill(a);
}

// ------------------------------------------------------------------ sparse latent

extern "C" int psa_sparse_latent_fwd(const void* q, const void* latent, const int32_t* idx,
                                     void* o, float* lse, int32_t T, int32_t Tk, int32_t H,
                                     int32_t dl, int32_t topk, float scale,
                                     int32_t* dev_status, void* stream) {
  if (T < 0 || Tk <= 0 || H <= 0 || topk <= 0 || !(scale > 0.f)) return PSA_ERR_INVALID_ARG;
  if (dl != 512 || H > 64) return PSA_ERR_UNSUPPORTED;
  if (T == 0) return PSA_OK;
  if (!q || !latent || !idx || !o) return PSA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(latent) || !aligned16(o) ||
      (reinterpret_cast<uintptr_t>(idx) & 3u) ||
      (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)))
    return PSA_ERR_INVALID_ARG;
  SparseArgs a;
  a.q = q;
  a.latent = latent;
  a.idx = idx;
  a.o = o;
  a.lse = lse;
  a.T = T;
  a.Tk = Tk;
  a.H = H;
  a.dl = dl;
  a.topk = topk;
  a.scale = scale;
  a.status = dev_status;
  a.stream = static_cast<cudaStream_t>(stream);
  return launch_sparse_latent(a);
}
