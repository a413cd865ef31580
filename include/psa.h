/*
 * psa.h -- C ABI of libpsa: shared-prefix attention over a flat,
 * deduplicated packed layout, for NVIDIA B200 (sm_100a).
 *
 * Page references are by title and section:
 *   [PS]  "KV-0 redundancy prefix sharing attention mask design"
 *         (PrefixSharing PR #50)
 *   [SKV] "Split-KV flash-decode attention for EAGLE target-verify"
 *         (sglang PR #27382)
 *   [MLA] "SM8x sparse-MLA prefill fallback re-reads the shared MLA latent
 *         once per head" (vLLM issue write-up)
 *
 * Conventions shared by every call:
 *   - Every function returns an int status (psa_status).  Nothing throws
 *     across this boundary.
 *   - Pointers named dev_* or documented as "device" are CUDA device
 *     pointers; all other pointers are host memory.  All buffers are owned
 *     by the caller; the library allocates and frees nothing and never
 *     synchronises the host with the device.
 *   - GPU work is enqueued on the caller's stream (a cudaStream_t passed as
 *     void*; NULL = the legacy default stream) and returns before it runs.
 *   - Tensors are dense, row-major and token-major, as documented per call.
 *     Every device pointer must be 16-byte aligned.
 *   - dev_status (nullable) is a device int32 the caller zeroes; a kernel
 *     that gives up on a bounded wait writes PSA_ERR_TIMEOUT there instead
 *     of hanging.  Read it with psa_read_status after the stream drains.
 *   - Arithmetic: bf16 inputs, fp32 accumulation, bf16 output; LSE is fp32
 *     natural-log of the sum of exp(scale * q.k) over visible keys.
 *   - GQA: query head h reads KV head h / (Hq / Hkv).
 */
#ifndef PSA_H
#define PSA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif
#if defined(__GNUC__)
#pragma GCC visibility push(default) /* the ABI stays visible under -fvisibility=hidden */
#endif

#define PSA_VERSION 1

typedef enum psa_status {
    PSA_OK = 0,
    PSA_ERR_INVALID_ARG = 1,  /* null pointer, bad size, misaligned, inconsistent shapes */
    PSA_ERR_UNSUPPORTED = 2,  /* a feature outside what the kernels implement */
    PSA_ERR_WORKSPACE = 3,    /* workspace missing or smaller than *_workspace_size */
    PSA_ERR_CUDA = 4,         /* a CUDA runtime/driver call failed */
    PSA_ERR_TIMEOUT = 5,      /* a device-side bounded wait gave up (via dev_status) */
    PSA_ERR_CAPACITY = 6,     /* a host output array is too small; *nout holds the need */
    PSA_ERR_BOUNDS = 7        /* debug build (libpsa_debug.so) only, via dev_status: a
                                 device-side bounds check found an index taken from caller
                                 data (a schedule entry, a prefix or mask offset) outside
                                 its buffer; the access was skipped, the results are void */
} psa_status;

typedef enum psa_dtype {
    PSA_BF16 = 0,
    PSA_F32 = 1
} psa_dtype;

/* Library version (PSA_VERSION) and a static string for a status code. */
int psa_version(void);
const char *psa_status_string(int status);

/* ------------------------------------------------------------------------
 * Mask spec (host only)                                      [PS] key changes s.2
 * --------------------------------------------------------------------- */

/* One segment of the flat layout: `len` tokens; `parent` is the global
 * index of the parent segment or -1 for a root.  Segments are listed in
 * flat order, parents before children; consecutive segments are adjacent
 * in the flat token range. */
typedef struct psa_segment {
    int32_t len;
    int32_t parent;
} psa_segment;

/* A visibility rectangle over flat token indices: queries [q0, q1) see keys
 * [k0, k1); if causal == 1, only where q - q0 >= k - k0 (top-left aligned).
 * causal == 2 appears only in transposed specs (psa_transpose_spec), where
 * the rows are keys: row r sees column c iff c - c0 >= r - r0. */
typedef struct psa_rect {
    int32_t q0, q1, k0, k1;
    int32_t causal;  /* 0: full; 1: causal; 2: transposed causal (psa_transpose_spec) */
} psa_rect;

/* Segments of the flat GRPO layout [PS] design summary: one prefix of P
 * tokens stored once, then N suffixes of S tokens, each child of the
 * prefix.  P == 0 gives N independent roots.  Writes N+1 (or N) segments.
 * Returns PSA_ERR_CAPACITY (with *nout set) if cap is too small. */
int psa_spec_flat(int32_t P, int32_t N, int32_t S, psa_segment *out, int32_t cap,
                  int32_t *nout);

/* Rectangle spec from a segment forest [PS] design summary ("a rectangle
 * spec rather than a full mask") and key changes s.2 (flat GRPO and
 * multi-level tree / chain cases).  Each segment sees every ancestor
 * segment fully and itself causally, so the rectangles are disjoint and
 * together cover exactly the visible (q, k) pairs.  No dense mask is ever
 * formed.  segs: nseg segments (flat order, all groups back to back).
 * Returns PSA_ERR_INVALID_ARG for a parent that does not precede its child
 * or a non-positive length; PSA_ERR_CAPACITY if cap < the rect count. */
int psa_build_spec(const psa_segment *segs, int32_t nseg, psa_rect *out, int32_t cap,
                   int32_t *nout);

/* Tile schedule for psa_prefill_fwd (host int32 array).  Q blocks of
 * tile_m rows (even; each block is two halves of tile_m/2 rows that one CTA
 * processes side by side) and KV tiles of tile_n keys are cut per group
 * (cu_seqlens, host, ngroups+1 entries).  For every Q block it lists only
 * the KV tiles in which at least one half has a visible pair, and for each
 * half whether it takes part, whether every pair is visible, and -- for a
 * partially visible half -- copies of the rectangles that cut it.  Q blocks
 * are ordered longest-first (most KV tiles first).
 *
 * Layout (int32):  [0] magic 0x50534132  [1] n_items  [2] n_kv  [3] n_rect
 *   [4] tile_m  [5] tile_n  [6] total tokens  [7] max KV tiles per item
 *   items  at 8:                  {q0, q_len, kv_begin, kv_count} x n_items
 *   kv     at 8 + 4*n_items:      {k0, k_len, a_rect_begin, a_rect_count,
 *                                  b_rect_begin, b_rect_count, flags, 0} x n_kv
 *          flags: bit 0 / 1 = half A / B has visible pairs in the tile,
 *                 bit 2 / 3 = every pair of half A / B is visible
 *   rects  at 8 + 4*n_items + 8*n_kv: {q0, q1, k0, k1, causal} x n_rect
 *          causal: 0 full, 1 causal (k - k0 <= q - q0), 2 transposed causal
 *          (k - k0 >= q - q0; see psa_transpose_spec)
 * Returns PSA_ERR_CAPACITY (with *nout = needed length) if cap is short. */
int psa_build_schedule(const psa_rect *rects, int32_t nrect, const int32_t *cu_seqlens,
                       int32_t ngroups, int32_t tile_m, int32_t tile_n, int32_t *out,
                       int64_t cap, int64_t *nout);

/* The transpose of a spec, for schedules that walk keys as rows (the
 * backward's dK / dV pass): rectangle r becomes {k0, k1, q0, q1} with
 * causal 1 turned into 2 and 2 into 1, where causal == 2 marks a
 * transposed causal rectangle (row r sees column c iff c - c0 >= r - r0).
 * out may alias rects.  PSA_ERR_INVALID_ARG for a causal value outside
 * 0..2. */
int psa_transpose_spec(const psa_rect *rects, int32_t nrect, psa_rect *out);

/* The block and tile sizes psa_prefill_fwd expects in its schedule:
 * tile_m query rows per block (two halves), tile_n keys per KV tile. */
int psa_prefill_tiles(int32_t head_dim, int32_t *tile_m, int32_t *tile_n);

/* ------------------------------------------------------------------------
 * Prefill over the packed layout          [PS] design summary, key changes
 * --------------------------------------------------------------------- */

/* Workspace bytes psa_prefill_fwd needs (PSA_F32 inputs are converted to
 * bf16 into it; the tile scheduler keeps its counter there). */
size_t psa_prefill_workspace_size(int dtype, int32_t T, int32_t Hq, int32_t Hkv,
                                  int32_t head_dim);

/* One forward pass of softmax attention over the flat layout with the
 * visibility described by dev_schedule (device copy of a
 * psa_build_schedule result, sched_len int32).
 *   q   device [T, Hq, d]      dtype (PSA_BF16 or PSA_F32)
 *   k,v device [T, Hkv, d]     dtype
 *   o   device [T, Hq, d]      dtype (written)
 *   lse device [T, Hq] fp32    (written; nullable)
 * d in {64, 128}; Hq % Hkv == 0.  Rows with no visible key (none occur for
 * a valid spec) are written as O = 0, LSE = -inf.
 * workspace: device, >= psa_prefill_workspace_size bytes, 256-B aligned. */
int psa_prefill_fwd(const void *q, const void *k, const void *v, void *o, float *lse,
                    int dtype, int32_t T, int32_t Hq, int32_t Hkv, int32_t head_dim,
                    float scale, const int32_t *dev_schedule, int64_t sched_len,
                    void *workspace, size_t ws_bytes, int32_t *dev_status, void *stream);

/* ------------------------------------------------------------------------
 * Backward of the prefill        [PS] design summary and test plan (the flat
 * layout gives the gradients of running each [prefix; s_i] separately, the
 * prefix K/V collecting the gradients of every suffix that sees them)
 * --------------------------------------------------------------------- */

/* Block and tile sizes of both backward schedules: tile_m rows per block
 * (two halves), tile_n columns per tile.  The dQ pass uses
 * psa_build_schedule(spec, ...) and the dK / dV pass
 * psa_build_schedule(psa_transpose_spec(spec), ...) with these sizes. */
int psa_prefill_bwd_tiles(int32_t head_dim, int32_t *tile_m, int32_t *tile_n);

/* Workspace bytes psa_prefill_bwd needs: the log2-domain LSE and
 * D = rowsum(dO * O) per (row, head), head-major. */
size_t psa_prefill_bwd_workspace_size(int32_t T, int32_t Hq);

/*
 * Gradients of O = psa_prefill_fwd(q, k, v) for the upstream gradient dout.
 *   q, dout    device [T, Hq, d] bf16
 *   k, v       device [T, Hkv, d] bf16
 *   o, lse     device, the forward's outputs for the same inputs and
 *              schedule ([T, Hq, d] bf16 and [T, Hq] fp32)
 *   dq         device [T, Hq, d] bf16 (written)
 *   dk, dv     device [T, Hkv, d] bf16 (written; every row, zero where no
 *              query sees the key)
 *   dev_schedule     device copy of psa_build_schedule(spec, cu_seqlens, ngroups,
 *                    tile_m, tile_n) with psa_prefill_bwd_tiles' sizes
 *   dev_schedule_kv  device copy of the same for psa_transpose_spec(spec)
 * dQ = scale dS K and dK = scale dS^T Q with dS = P (dO V^T - D); dV = P^T dO.
 * d in {64, 128}; Hq % Hkv == 0.  No atomics: each output row is written
 * once, by one CTA.  workspace: device, >= psa_prefill_bwd_workspace_size
 * bytes, 256-B aligned.
 */
int psa_prefill_bwd(const void *q, const void *k, const void *v, const void *o,
                    const float *lse, const void *dout, void *dq, void *dk, void *dv, int32_t T,
                    int32_t Hq, int32_t Hkv, int32_t head_dim, float scale,
                    const int32_t *dev_schedule, int64_t sched_len,
                    const int32_t *dev_schedule_kv, int64_t sched_kv_len, void *workspace,
                    size_t ws_bytes, int32_t *dev_status, void *stream);

/* ------------------------------------------------------------------------
 * Speculative verify: split-KV over the cached prefix, then an LSE combine
 * that folds in the causal draft block.   [SKV] implementation item 1
 * --------------------------------------------------------------------- */

/* Features of the general extend-attention call that the split-KV path
 * does not implement ([SKV] key code: can_handle).  Pass NULL for the
 * supported case; any non-default field makes psa_verify_fwd return
 * PSA_ERR_UNSUPPORTED (there is no fallback path). */
typedef struct psa_verify_features {
    int32_t has_custom_mask;     /* tree drafts (topk > 1) carry a custom mask */
    int32_t is_causal;           /* must be 1 */
    int32_t sliding_window;      /* must be <= 0 */
    int32_t has_sinks;           /* must be 0 */
    float logit_cap;             /* must be 0 */
    int32_t xai_temperature_len; /* must be <= 0 */
    int32_t ragged_extend;       /* per-request draft counts differ: must be 0 */
} psa_verify_features;

/* Per-tensor scales of an e4m3 KV cache ([SKV] the verify entry's k_scale /
 * v_scale): a cached key stands for k_scale * e4m3, a cached value for
 * v_scale * e4m3.  Both finite and > 0. */
typedef struct psa_kv_scales {
    float k_scale;
    float v_scale;
} psa_kv_scales;

/* Split count chosen when nsplit == 0: enough (request, split) units to
 * fill the GPU, each covering a whole number of key tiles. */
int32_t psa_verify_auto_splits(int32_t B, int64_t max_prefix_len, int32_t Hkv,
                               int32_t head_dim);

/* Workspace bytes for the split partials: nsplit * B*Ld*Hq * (d + 1) fp32,
 * plus alignment padding (B*Ld is the number of draft rows: pass B = 1 and
 * Ld = n_rows for psa_verify_extend_fwd).  Size it for the largest batch you
 * will run and reuse it ([SKV] review: key scratch by the maximum batch, not
 * by the current one). */
size_t psa_verify_workspace_size(int32_t B, int32_t Ld, int32_t Hq, int32_t head_dim,
                                 int32_t nsplit);

/*
 *   q_draft          device [B*Ld, Hq, d] bf16   draft-token queries, request-major
 *   k_draft, v_draft device [B*Ld, Hkv, d] bf16  draft-token keys/values
 *   k_cache, v_cache device [Ntok, Hkv, d] bf16  the KV cache (token rows)
 *   n_cache_tokens   host value Ntok (rows of k_cache / v_cache)
 *   dev_kv_indptr    device int32 [B+1]         request b's prefix positions are
 *                                                [indptr[b], indptr[b+1])
 *   max_prefix_len   host value >= every prefix length (no device sync is made)
 *   kv_indices       NULL: prefix position t is cache row t (one contiguous
 *                    range per request, streamed with TMA tiles); else device
 *                    int32 [indptr[B]], a page table with one token per page:
 *                    position t is cache row kv_indices[t] ([SKV] the verify
 *                    entry's kv_indptr / kv_indices pair).  Rows are gathered
 *                    with 16-byte copies; a row outside [0, Ntok) reads as
 *                    zeros and sets PSA_ERR_INVALID_ARG in dev_status.
 *   o                device [B*Ld, Hq, d] bf16   (written)
 *   lse              device [B*Ld, Hq] fp32      (written; nullable)
 * Draft j of request b sees the whole prefix of b plus drafts 0..j.
 * d in {64, 128, 256}; Hq % Hkv == 0; Ld * Hq / Hkv <= 128.
 * nsplit in [1, 256], or 0 for psa_verify_auto_splits.  Split s of request
 * b covers prefix tokens [s*c, min((s+1)*c, L_b)) with c = ceil(L_b/nsplit)
 * rounded up to the key tile; empty splits contribute nothing.
 */
int psa_verify_fwd(const void *q_draft, const void *k_draft, const void *v_draft,
                   const void *k_cache, const void *v_cache, int64_t n_cache_tokens,
                   const int32_t *dev_kv_indptr,
                   int64_t max_prefix_len, const int32_t *kv_indices, void *o, float *lse,
                   int32_t B, int32_t Ld, int32_t Hq, int32_t Hkv, int32_t head_dim,
                   float scale, int32_t nsplit, const psa_verify_features *features,
                   void *workspace, size_t ws_bytes, int32_t *dev_status, void *stream);

/*
 * Tree verify: psa_verify_fwd with the draft block given by a custom mask
 * instead of the causal chain ([SKV] key code, can_handle: EAGLE trees with
 * topk > 1 bring a custom mask; the prefix is not masked, so every draft
 * still sees the whole cached prefix).
 *   dev_draft_mask  device uint8 [B*Ld, Ld]: draft j of request b sees draft
 *                   i of b iff dev_draft_mask[(b*Ld + j)*Ld + i] != 0
 *                   (required when B > 0: PSA_ERR_INVALID_ARG otherwise)
 * features->has_custom_mask may be set here; every other argument, layout,
 * gate and status is that of psa_verify_fwd.  A draft row that sees no key
 * (empty prefix and an empty mask row) gets O = 0 and LSE = -inf.
 */
int psa_verify_tree_fwd(const void *q_draft, const void *k_draft, const void *v_draft,
                        const void *k_cache, const void *v_cache, int64_t n_cache_tokens,
                        const int32_t *dev_kv_indptr, int64_t max_prefix_len,
                        const int32_t *kv_indices, const uint8_t *dev_draft_mask, void *o,
                        float *lse, int32_t B, int32_t Ld, int32_t Hq, int32_t Hkv,
                        int32_t head_dim, float scale, int32_t nsplit,
                        const psa_verify_features *features, void *workspace, size_t ws_bytes,
                        int32_t *dev_status, void *stream);

/*
 * Verify in the general extend form ([SKV] the verify entry's signature:
 * qo_indptr, kv_indptr, kv_indices, custom_mask, mask_indptr; can_handle
 * names ragged extend and custom masks as what its split path leaves out):
 * per-request draft counts, an optional page table and optional tree masks.
 *   q_draft          device [n_rows, Hq, d] bf16   draft rows, request-major
 *   k_draft, v_draft device [n_rows, Hkv, d] bf16
 *   dev_qo_indptr    device int32 [B+1]: request b's drafts are rows
 *                    [qo_indptr[b], qo_indptr[b+1]); qo_indptr[B] == n_rows
 *   n_rows           host value, the total draft rows
 *   max_draft_len    host value >= every draft count (the m-tile plan uses
 *                    it: max_draft_len * Hq / Hkv <= 128).  A count above it
 *                    or a decreasing qo_indptr sets PSA_ERR_INVALID_ARG in
 *                    dev_status; those rows are not written.
 *   dev_kv_indptr, max_prefix_len, dev_kv_indices: as psa_verify_fwd
 *   dev_draft_mask   NULL: each request's draft block is causal; else device
 *                    uint8, request b's Lb x Lb block (row-major, Lb its draft
 *                    count) starting at dev_draft_mask[mask_indptr[b]]: draft
 *                    j sees draft i iff its (j, i) byte is non-zero
 *   dev_mask_indptr  device int32 [B+1] (required with a mask)
 *   e4m3_scales      NULL: k_cache / v_cache are bf16; else they hold e4m3
 *                    bytes standing for k_scale * e4m3 and v_scale * e4m3
 *                    (as psa_verify_fp8_fwd; head_dim must be 128)
 *   o, lse           device [n_rows, Hq, d] bf16 / [n_rows, Hq] fp32
 * features->ragged_extend and ->has_custom_mask may be set here.  The
 * workspace holds the partials of n_rows rows:
 * psa_verify_workspace_size(1, n_rows, Hq, d, nsplit) bytes.  Every draft row
 * sees its request's whole prefix; a row that sees no key gets O = 0 and
 * LSE = -inf.  Other arguments and statuses as psa_verify_fwd.
 */
int psa_verify_extend_fwd(const void *q_draft, const void *k_draft, const void *v_draft,
                          const void *k_cache, const void *v_cache, int64_t n_cache_tokens,
                          const int32_t *dev_qo_indptr, int32_t n_rows, int32_t max_draft_len,
                          const int32_t *dev_kv_indptr, int64_t max_prefix_len,
                          const int32_t *dev_kv_indices, const uint8_t *dev_draft_mask,
                          const int32_t *dev_mask_indptr, const psa_kv_scales *e4m3_scales,
                          void *o, float *lse, int32_t B, int32_t Hq, int32_t Hkv,
                          int32_t head_dim, float scale,
                          int32_t nsplit, const psa_verify_features *features,
                          void *workspace, size_t ws_bytes, int32_t *dev_status, void *stream);

/* Size of the library's fixed device scratch used by psa_verify_fwd_noalloc:
 * 16 MiB, held by every GPU that loads the library until the process exits. */
#define PSA_VERIFY_NOALLOC_SCRATCH_BYTES (16u << 20)

/*
 * psa_verify_fwd without a caller workspace.  The pages have no counterpart
 * of this call; it exists for callers that cannot allocate device memory
 * where they call attention -- for example a host whose device memory is
 * owned by another allocator (a framework's caching allocator or a serving
 * engine's preallocated pool) that must not see cudaMalloc behind its back,
 * or a latency-critical loop where cudaMalloc's implicit device-wide
 * synchronisation, or its failure under memory pressure, is unacceptable.
 *
 * The split partials go to one file-scope device array of
 * PSA_VERIFY_NOALLOC_SCRATCH_BYTES instead of a workspace.  Arguments,
 * layouts and results are those of psa_verify_fwd (minus workspace and
 * ws_bytes); the caller still owns every input and output.
 *   - Returns PSA_ERR_WORKSPACE when the call would need more than
 *     PSA_VERIFY_NOALLOC_SCRATCH_BYTES, that is when
 *     psa_verify_workspace_size(B, Ld, Hq, head_dim, nsplit) exceeds it
 *     (nsplit == 0 is resolved with psa_verify_auto_splits first).
 *   - Allocates and frees nothing, directly or through any library.
 *   - Every call looks up the array's device address in the context that is
 *     current for the call (cudaGetSymbolAddress; no allocation), so a caller
 *     that switches contexts on a device, or rebuilds its context after a
 *     device reset, still gets the array of the context it calls from.  The
 *     first call in a context also loads the library's module there; make it
 *     before any stream capture in that context.
 *   - Every call on a device shares the one array, which keeps whatever the
 *     last call left there.  Nothing in it needs to start at zero (stage 1
 *     writes every partial that stage 2 reads).  Calls whose GPU work
 *     overlaps -- on different streams, or from different host threads --
 *     race on the array and corrupt each other's results; order them.
 */
int psa_verify_fwd_noalloc(const void *q_draft, const void *k_draft, const void *v_draft,
                           const void *k_cache, const void *v_cache, int64_t n_cache_tokens,
                           const int32_t *dev_kv_indptr, int64_t max_prefix_len,
                           const int32_t *kv_indices, void *o, float *lse, int32_t B,
                           int32_t Ld, int32_t Hq, int32_t Hkv, int32_t head_dim, float scale,
                           int32_t nsplit, const psa_verify_features *features,
                           int32_t *dev_status, void *stream);

/*
 * psa_verify_fwd with an fp8 prefix cache ([SKV] implementation item 1:
 * stage 1 applies the fp8 scales k_scale / v_scale of the cache).
 *   k_cache, v_cache device [Ntok, Hkv, d] e4m3 bytes ("E4M3FN": bias 7,
 *                    3 mantissa bits, no infinities); a cached key stands for
 *                    k_scale * e4m3, a cached value for v_scale * e4m3
 *   k_scale, v_scale host values, finite and > 0
 * Draft keys and values stay bf16 and are not scaled.  Every other argument,
 * layout and status is that of psa_verify_fwd (kv_indices included: NULL for
 * a contiguous prefix, else the token-granular page table), except that
 * head_dim must be 128 (PSA_ERR_UNSUPPORTED otherwise).  The prefix read is
 * half the bytes of the bf16 cache.  Q is widened to f16 for the tensor
 * cores: |q| must stay below 65504.
 */
int psa_verify_fp8_fwd(const void *q_draft, const void *k_draft, const void *v_draft,
                       const void *k_cache, const void *v_cache, int64_t n_cache_tokens,
                       const int32_t *dev_kv_indptr, int64_t max_prefix_len,
                       const int32_t *kv_indices, float k_scale, float v_scale, void *o,
                       float *lse, int32_t B, int32_t Ld, int32_t Hq, int32_t Hkv,
                       int32_t head_dim, float scale, int32_t nsplit,
                       const psa_verify_features *features, void *workspace, size_t ws_bytes,
                       int32_t *dev_status, void *stream);

/* ------------------------------------------------------------------------
 * Speculative verify against one prefix shared by every request.
 *   [PS] design summary (the prefix K/V is stored once and every sequence
 *   built on it sees all of it) + [SKV] implementation item 1 (a draft row
 *   sees the prefix plus drafts 0..j of its own request).
 * --------------------------------------------------------------------- */

/* nsplit chosen by psa_verify_shared_fwd when it is passed 0: as many
 * units (chunk, KV head, 256 stacked rows) as fit one wave of 148 SMs,
 * chunks of >= 512 keys. */
int32_t psa_verify_shared_auto_splits(int32_t B, int32_t Ld, int32_t Hq, int32_t Hkv,
                                      int64_t prefix_len);

/*
 * The B requests share ONE cached prefix instead of owning one each, so the
 * prefix is read once for all of them: the B * Ld * (Hq / Hkv) draft rows of
 * a KV head are stacked into 128-row tensor-core tiles and multiplied
 * against each prefix chunk, then the chunks and each row's causal draft
 * block are merged by log-sum-exp weight exactly as in psa_verify_fwd.
 *   q_draft          device [B*Ld, Hq, d] bf16   draft queries, request-major
 *   k_draft, v_draft device [B*Ld, Hkv, d] bf16  draft keys / values
 *   k_prefix,        device [L, Hkv, d] bf16     the shared prefix (nullable
 *   v_prefix                                     when L == 0)
 *   prefix_len       host value L, 0 <= L <= 2^30
 *   o                device [B*Ld, Hq, d] bf16   (written)
 *   lse              device [B*Ld, Hq] fp32      (written; nullable)
 * Draft j of request b sees prefix tokens 0..L-1 and drafts 0..j of b; the
 * result equals psa_verify_fwd on a cache holding B copies of the prefix.
 * d in {64, 128}; Hq / Hkv must divide 128; 1 <= Ld <= 16 (the combine
 * holds a row's draft block in one warp's registers; PSA_ERR_UNSUPPORTED
 * above).  nsplit: 1..256, or 0 for
 * psa_verify_shared_auto_splits; the prefix is cut into nsplit chunks of
 * ceil(L / nsplit) keys rounded up to 128 (trailing chunks may be empty).
 * workspace: device, >= psa_verify_workspace_size(B, Ld, Hq, d, nsplit)
 * bytes, 256-B aligned (PSA_ERR_WORKSPACE otherwise).  Statuses as for
 * psa_verify_fwd.
 */
int psa_verify_shared_fwd(const void *q_draft, const void *k_draft, const void *v_draft,
                          const void *k_prefix, const void *v_prefix, int64_t prefix_len,
                          void *o, float *lse, int32_t B, int32_t Ld, int32_t Hq, int32_t Hkv,
                          int32_t head_dim, float scale, int32_t nsplit, void *workspace,
                          size_t ws_bytes, int32_t *dev_status, void *stream);

/*
 * psa_verify_shared_fwd with the draft block given by a custom mask (tree
 * verify against one shared prefix: [SKV] key code, can_handle -- EAGLE
 * trees with topk > 1 bring a custom mask; [PS] design summary -- the prefix
 * stored once).  dev_draft_mask: device uint8 [B*Ld, Ld], draft j of request
 * b sees draft i of b iff dev_draft_mask[(b*Ld + j)*Ld + i] != 0 (required
 * when B > 0: PSA_ERR_INVALID_ARG otherwise); every draft sees the whole
 * prefix.  A row that sees no key gets O = 0 and LSE = -inf.  Everything
 * else as psa_verify_shared_fwd.
 */
int psa_verify_shared_tree_fwd(const void *q_draft, const void *k_draft, const void *v_draft,
                               const void *k_prefix, const void *v_prefix, int64_t prefix_len,
                               const uint8_t *dev_draft_mask, void *o, float *lse, int32_t B,
                               int32_t Ld, int32_t Hq, int32_t Hkv, int32_t head_dim,
                               float scale, int32_t nsplit, void *workspace, size_t ws_bytes,
                               int32_t *dev_status, void *stream);

/* ------------------------------------------------------------------------
 * Shared-latent sparse attention                     [MLA] environment,
 * analysis (head-blocked tiles; the latent is shared by every head)
 * --------------------------------------------------------------------- */

/*
 *   q       device [T, H, dl] bf16     queries, all heads of a token together
 *   latent  device [Tk, dl] bf16       the one shared latent: K = V = latent
 *   idx     device [T, topk] int32     per-query key rows; -1 entries are
 *                                      skipped; an entry >= Tk is skipped too
 *                                      and sets PSA_ERR_INVALID_ARG in
 *                                      dev_status
 *   o       device [T, H, dl] bf16     (written)
 *   lse     device [T, H] fp32         (written; nullable)
 * dl == 512, H <= 64, topk >= 1.  Row t attends to the listed latent rows
 * only; a row whose list is all -1 gets O = 0 and LSE = -inf.
 */
int psa_sparse_latent_fwd(const void *q, const void *latent, const int32_t *idx, void *o,
                          float *lse, int32_t T, int32_t Tk, int32_t H, int32_t dl,
                          int32_t topk, float scale, int32_t *dev_status, void *stream);

/* ------------------------------------------------------------------------
 * Status word
 * --------------------------------------------------------------------- */

/* Copies the device status word to *host_out after draining `stream`.
 * This is the one call that waits on the device. */
int psa_read_status(const int32_t *dev_status, int32_t *host_out, void *stream);

/* Failure-detection self-test of the bounded device wait every kernel uses
 * (no counterpart on the pages).  Launches one warp on `stream` that waits
 * on a shared-memory barrier expecting one arrival.
 *   arrive != 0: the barrier is arrived at first; the wait completes at once
 *                and *dev_status is left unchanged.
 *   arrive == 0: nothing arrives; after the library's wait budget (2 s) the
 *                wait gives up, writes PSA_ERR_TIMEOUT to *dev_status (when
 *                it still holds 0) and the kernel returns normally, leaving
 *                the context usable.
 * dev_status (device int32, required) is owned by the caller, who zeroes it.
 * Returns PSA_ERR_INVALID_ARG for a null dev_status, PSA_ERR_CUDA if the
 * launch fails, else PSA_OK. */
int psa_wait_selftest(int32_t arrive, int32_t *dev_status, void *stream);

#if defined(__GNUC__)
#pragma GCC visibility pop
#endif
#ifdef __cplusplus
}
#endif

#endif /* PSA_H */
