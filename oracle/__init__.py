"""fp64 CPU oracle for shared-prefix attention.

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg may import this package; the product package
never does.  The arithmetic lives in ``oracle.c`` (plain C, fp64, built with
gcc by :func:`build`); this module only marshals numpy arrays.

Every function takes the exact input values the GPU consumed (bf16 tensors
widened to fp32 without rounding) and returns fp64 results:

* :func:`prefill` -- dense masked softmax attention over the flat packed
  layout [prefix; s_1; ...; s_N] with visibility from the segment tree
  ("KV-0 redundancy prefix sharing attention mask design", design summary
  and key changes section 2).
* :func:`verify` -- each draft row sees the whole cached prefix of its
  request plus drafts 0..j ("Split-KV flash-decode attention for EAGLE
  target-verify", implementation breakdown item 1).
* :func:`sparse_latent` -- each query attends to the latent rows named by
  its index list, K = V = latent ("SM8x sparse-MLA prefill fallback re-reads
  the shared MLA latent once per head", environment section).
* :func:`visibility` -- the dense visibility matrix from the same
  definition, for checking the mask builder bit-exactly.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(mutant: int = 0, out: str | None = None) -> str:
    """Compile oracle.c with gcc.  ``mutant`` > 0 builds a deliberately broken
    copy (the tests use these to show that the pins catch planted mistakes)."""
    out = out or _LIB_PATH
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-pthread",
           f"-DORACLE_MUTANT={int(mutant)}", _SRC, "-o", out, "-lm"]
    subprocess.run(cmd, check=True)
    return out


def _needs_build(path: str) -> bool:
    return (not os.path.exists(path)) or os.path.getmtime(path) < os.path.getmtime(_SRC)


def load(path: str | None = None):
    """Load (building first if stale) the oracle library."""
    global _lib
    if path is None:
        if _lib is not None:
            return _lib
        if _needs_build(_LIB_PATH):
            build()
        path = _LIB_PATH
    lib = ctypes.CDLL(path)
    P = ctypes.c_void_p
    I = ctypes.c_int
    D = ctypes.c_double
    lib.oracle_prefill.argtypes = [P, P, P, I, I, I, I, D, P, P, P, I, P, I, P, P, I]
    lib.oracle_verify.argtypes = [P, P, P, P, P, P, I, I, I, I, I, D, P, I, P, P, I]
    lib.oracle_prefill_bwd.argtypes = [P, P, P, P, I, I, I, I, D, P, P, P, I, P, P, P, I]
    lib.oracle_prefill_bwd_dq.argtypes = [P, P, P, P, I, I, I, I, D, P, P, P, I, P, I, P, I]
    lib.oracle_verify_tree.argtypes = [P, P, P, P, P, P, P, I, I, I, I, I, D, P, I, P, P, I]
    lib.oracle_verify_extend.argtypes = [P] * 10 + [I, I, I, I, D, P, I, P, P, I]
    lib.oracle_verify_shared.argtypes = [P, P, P, P, P, ctypes.c_int64, I, I, I, I, I, D, P, I,
                                         P, P, I]
    lib.oracle_verify_fp8.argtypes = [P, P, P, P, P, D, D, P, I, I, I, I, I, D, P, I, P, P, I]
    lib.oracle_verify_shared_tree.argtypes = [P, P, P, P, P, ctypes.c_int64, P, I, I, I, I, I, D,
                                              P, I, P, P, I]
    lib.oracle_verify_fp8_paged.argtypes = [P, P, P, P, P, D, D, P, P, I, I, I, I, I, D, P, I,
                                            P, P, I]
    lib.oracle_decode_e4m3.argtypes = [P, P, ctypes.c_int64]
    lib.oracle_sparse_latent.argtypes = [P, P, P, I, I, I, I, I, D, P, I, P, P, I]
    lib.oracle_visibility.argtypes = [P, P, P, I, I, I, I, P]
    for f in (lib.oracle_prefill, lib.oracle_prefill_bwd, lib.oracle_prefill_bwd_dq,
              lib.oracle_verify, lib.oracle_verify_tree, lib.oracle_verify_extend,
              lib.oracle_verify_shared, lib.oracle_verify_shared_tree,
              lib.oracle_verify_fp8, lib.oracle_verify_fp8_paged, lib.oracle_decode_e4m3, lib.oracle_sparse_latent,
              lib.oracle_visibility):
        f.restype = I
    if path == _LIB_PATH:
        _lib = lib
    return lib


def _f32(a) -> np.ndarray:
    """Widen to a C-contiguous fp32 array.  Accepts numpy arrays and CPU
    torch tensors (bf16 widens exactly)."""
    if hasattr(a, "detach"):
        a = a.detach().float().cpu().numpy()
    return np.ascontiguousarray(np.asarray(a, dtype=np.float32))


def _i32(a) -> np.ndarray:
    if hasattr(a, "detach"):
        a = a.detach().cpu().numpy()
    return np.ascontiguousarray(np.asarray(a, dtype=np.int32))


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def default_threads() -> int:
    return max(1, os.cpu_count() or 1)


def segment_arrays(segments: Sequence[tuple[int, int]]):
    """(len, parent) list in flat order -> (start, len, parent) int32 arrays.
    Parents are global segment indices, -1 for a root."""
    lens = np.array([s[0] for s in segments], dtype=np.int32)
    parent = np.array([s[1] for s in segments], dtype=np.int32)
    start = np.zeros_like(lens)
    if len(lens):
        start[1:] = np.cumsum(lens)[:-1]
    return start, lens, parent


def visibility(segments, row0: int = 0, nrows: int | None = None, lib=None) -> np.ndarray:
    """Dense [nrows, T] uint8 visibility matrix from the segment-tree definition."""
    lib = lib or load()
    start, lens, parent = segment_arrays(segments)
    T = int(lens.sum())
    nrows = T - row0 if nrows is None else nrows
    out = np.zeros((nrows, T), dtype=np.uint8)
    rc = lib.oracle_visibility(_ptr(start), _ptr(lens), _ptr(parent), len(lens), T,
                               row0, nrows, _ptr(out))
    assert rc == 0
    return out


def prefill(q, k, v, segments, scale: float, rows=None, nthreads: int | None = None,
            lib=None):
    """O [nrows, Hq, d] and LSE [nrows, Hq] (fp64) for flat rows ``rows``
    (all rows when None).  q [T, Hq, d]; k, v [T, Hkv, d]."""
    lib = lib or load()
    q, k, v = _f32(q), _f32(k), _f32(v)
    T, Hq, d = q.shape
    Hkv = k.shape[1]
    start, lens, parent = segment_arrays(segments)
    rows = np.arange(T, dtype=np.int32) if rows is None else _i32(rows)
    o = np.zeros((len(rows), Hq, d), dtype=np.float64)
    lse = np.zeros((len(rows), Hq), dtype=np.float64)
    rc = lib.oracle_prefill(_ptr(q), _ptr(k), _ptr(v), T, Hq, Hkv, d, float(scale),
                            _ptr(start), _ptr(lens), _ptr(parent), len(lens),
                            _ptr(rows), len(rows), _ptr(o), _ptr(lse),
                            nthreads or default_threads())
    assert rc == 0, "oracle_prefill rejected its arguments"
    return o, lse


def prefill_bwd(q, k, v, dout, segments, scale: float, nthreads: int | None = None, lib=None):
    """Gradients (dq [T, Hq, d], dk, dv [T, Hkv, d], fp64) of the prefill
    output O with upstream gradient dout [T, Hq, d]."""
    lib = lib or load()
    q, k, v, do = _f32(q), _f32(k), _f32(v), _f32(dout)
    T, Hq, d = q.shape
    Hkv = k.shape[1]
    start, lens, parent = segment_arrays(segments)
    dq = np.zeros((T, Hq, d), dtype=np.float64)
    dk = np.zeros((T, Hkv, d), dtype=np.float64)
    dv = np.zeros((T, Hkv, d), dtype=np.float64)
    rc = lib.oracle_prefill_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(do), T, Hq, Hkv, d, float(scale),
                                _ptr(start), _ptr(lens), _ptr(parent), len(lens), _ptr(dq),
                                _ptr(dk), _ptr(dv), nthreads or default_threads())
    assert rc == 0, "oracle_prefill_bwd rejected its arguments"
    return dq, dk, dv


def prefill_bwd_dq(q, k, v, dout, segments, scale: float, rows, nthreads: int | None = None,
                   lib=None):
    """dq [nrows, Hq, d] (fp64) of the selected flat rows only."""
    lib = lib or load()
    q, k, v, do = _f32(q), _f32(k), _f32(v), _f32(dout)
    T, Hq, d = q.shape
    Hkv = k.shape[1]
    start, lens, parent = segment_arrays(segments)
    rows = _i32(rows)
    dq = np.zeros((len(rows), Hq, d), dtype=np.float64)
    rc = lib.oracle_prefill_bwd_dq(_ptr(q), _ptr(k), _ptr(v), _ptr(do), T, Hq, Hkv, d,
                                   float(scale), _ptr(start), _ptr(lens), _ptr(parent), len(lens),
                                   _ptr(rows), len(rows), _ptr(dq), nthreads or default_threads())
    assert rc == 0, "oracle_prefill_bwd_dq rejected its arguments"
    return dq


def verify(q_draft, k_draft, v_draft, k_cache, v_cache, kv_indptr, Ld: int,
           scale: float, rows=None, nthreads: int | None = None, lib=None):
    """O [nrows, Hq, d] and LSE [nrows, Hq] for draft rows b*Ld + j."""
    lib = lib or load()
    qd, kd, vd = _f32(q_draft), _f32(k_draft), _f32(v_draft)
    kc, vc = _f32(k_cache), _f32(v_cache)
    indptr = np.ascontiguousarray(np.asarray(
        kv_indptr.cpu().numpy() if hasattr(kv_indptr, "cpu") else kv_indptr, dtype=np.int64))
    BL, Hq, d = qd.shape
    Hkv = kd.shape[1]
    B = BL // Ld
    rows = np.arange(BL, dtype=np.int32) if rows is None else _i32(rows)
    o = np.zeros((len(rows), Hq, d), dtype=np.float64)
    lse = np.zeros((len(rows), Hq), dtype=np.float64)
    rc = lib.oracle_verify(_ptr(qd), _ptr(kd), _ptr(vd), _ptr(kc), _ptr(vc), _ptr(indptr),
                           B, Ld, Hq, Hkv, d, float(scale), _ptr(rows), len(rows),
                           _ptr(o), _ptr(lse), nthreads or default_threads())
    assert rc == 0, "oracle_verify rejected its arguments"
    return o, lse


def verify_tree(q_draft, k_draft, v_draft, k_cache, v_cache, kv_indptr, draft_mask, Ld: int,
                scale: float, rows=None, nthreads: int | None = None, lib=None):
    """As verify, with the draft block given by draft_mask [B*Ld, Ld] (row
    b*Ld + j lists the drafts of request b that draft j sees)."""
    lib = lib or load()
    qd, kd, vd = _f32(q_draft), _f32(k_draft), _f32(v_draft)
    kc, vc = _f32(k_cache), _f32(v_cache)
    dm = _u8(draft_mask)
    indptr = np.ascontiguousarray(np.asarray(
        kv_indptr.cpu().numpy() if hasattr(kv_indptr, "cpu") else kv_indptr, dtype=np.int64))
    BL, Hq, d = qd.shape
    Hkv = kd.shape[1]
    B = BL // Ld
    assert dm.shape == (BL, Ld)
    rows = np.arange(BL, dtype=np.int32) if rows is None else _i32(rows)
    o = np.zeros((len(rows), Hq, d), dtype=np.float64)
    lse = np.zeros((len(rows), Hq), dtype=np.float64)
    rc = lib.oracle_verify_tree(_ptr(qd), _ptr(kd), _ptr(vd), _ptr(kc), _ptr(vc), _ptr(indptr),
                                _ptr(dm), B, Ld, Hq, Hkv, d, float(scale), _ptr(rows), len(rows),
                                _ptr(o), _ptr(lse), nthreads or default_threads())
    assert rc == 0, "oracle_verify_tree rejected its arguments"
    return o, lse


def _i64(x):
    return np.ascontiguousarray(np.asarray(x.cpu().numpy() if hasattr(x, "cpu") else x,
                                           dtype=np.int64))


def verify_extend(q_draft, k_draft, v_draft, k_cache, v_cache, qo_indptr, kv_indptr, scale: float,
                  kv_indices=None, draft_mask=None, mask_indptr=None, rows=None,
                  nthreads: int | None = None, lib=None):
    """Verify in the extend form: ragged draft counts (qo_indptr), a paged
    prefix (kv_indices: prefix position t is cache row kv_indices[t]) and an
    optional per-request draft mask (request b's Lb x Lb block starts at
    draft_mask[mask_indptr[b]], flat uint8).  O [nrows, Hq, d], LSE [nrows, Hq]."""
    lib = lib or load()
    qd, kd, vd = _f32(q_draft), _f32(k_draft), _f32(v_draft)
    kc, vc = _f32(k_cache), _f32(v_cache)
    qo, kvp = _i64(qo_indptr), _i64(kv_indptr)
    B = len(qo) - 1
    assert len(kvp) == B + 1
    idx = None if kv_indices is None else _i32(kv_indices)
    dm = None if draft_mask is None else _u8(draft_mask).reshape(-1)
    mi = None if mask_indptr is None else _i64(mask_indptr)
    NR, Hq, d = qd.shape
    Hkv = kd.shape[1]
    assert qo[-1] == NR
    rows = np.arange(NR, dtype=np.int32) if rows is None else _i32(rows)
    o = np.zeros((len(rows), Hq, d), dtype=np.float64)
    lse = np.zeros((len(rows), Hq), dtype=np.float64)
    nul = ctypes.c_void_p(0)
    rc = lib.oracle_verify_extend(_ptr(qd), _ptr(kd), _ptr(vd), _ptr(kc), _ptr(vc), _ptr(qo),
                                  _ptr(kvp), nul if idx is None else _ptr(idx),
                                  nul if dm is None else _ptr(dm), nul if mi is None else _ptr(mi),
                                  B, Hq, Hkv, d, float(scale), _ptr(rows), len(rows), _ptr(o),
                                  _ptr(lse), nthreads or default_threads())
    assert rc == 0, "oracle_verify_extend rejected its arguments"
    return o, lse


def verify_shared(q_draft, k_draft, v_draft, k_prefix, v_prefix, Ld: int, scale: float,
                  rows=None, nthreads: int | None = None, lib=None, draft_mask=None):
    """O [nrows, Hq, d] and LSE [nrows, Hq] for draft rows b*Ld + j when every
    request sees the same prefix k_prefix/v_prefix [L, Hkv, d]."""
    lib = lib or load()
    qd, kd, vd = _f32(q_draft), _f32(k_draft), _f32(v_draft)
    kp, vp = _f32(k_prefix), _f32(v_prefix)
    BL, Hq, d = qd.shape
    Hkv = kd.shape[1]
    B = BL // Ld
    rows = np.arange(BL, dtype=np.int32) if rows is None else _i32(rows)
    o = np.zeros((len(rows), Hq, d), dtype=np.float64)
    lse = np.zeros((len(rows), Hq), dtype=np.float64)
    if draft_mask is None:
        rc = lib.oracle_verify_shared(_ptr(qd), _ptr(kd), _ptr(vd), _ptr(kp), _ptr(vp),
                                      int(kp.shape[0]), B, Ld, Hq, Hkv, d, float(scale),
                                      _ptr(rows), len(rows), _ptr(o), _ptr(lse),
                                      nthreads or default_threads())
    else:
        dm = _u8(draft_mask)
        assert dm.shape == (BL, Ld)
        rc = lib.oracle_verify_shared_tree(_ptr(qd), _ptr(kd), _ptr(vd), _ptr(kp), _ptr(vp),
                                           int(kp.shape[0]), _ptr(dm), B, Ld, Hq, Hkv, d,
                                           float(scale), _ptr(rows), len(rows), _ptr(o),
                                           _ptr(lse), nthreads or default_threads())
    assert rc == 0, "oracle_verify_shared rejected its arguments"
    return o, lse


def _u8(x):
    if hasattr(x, "cpu"):
        import torch
        x = x.cpu()
        if x.dtype != torch.uint8:
            x = x.view(torch.uint8)
        x = x.numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.uint8))


def decode_e4m3(codes, lib=None):
    """fp64 values of e4m3 bytes (any shape)."""
    lib = lib or load()
    c = _u8(codes)
    out = np.zeros(c.shape, dtype=np.float64)
    lib.oracle_decode_e4m3(_ptr(c), _ptr(out), c.size)
    return out


def verify_fp8(q_draft, k_draft, v_draft, k_cache8, v_cache8, k_scale: float, v_scale: float,
               kv_indptr, Ld: int, scale: float, rows=None, nthreads: int | None = None,
               lib=None, kv_indices=None):
    """As verify, with e4m3 caches (uint8 or float8 tensors) standing for
    k_scale * e4m3 and v_scale * e4m3; with kv_indices, prefix position t of
    the flat kv_indptr range is cache row kv_indices[t]."""
    lib = lib or load()
    qd, kd, vd = _f32(q_draft), _f32(k_draft), _f32(v_draft)
    kc, vc = _u8(k_cache8), _u8(v_cache8)
    indptr = np.ascontiguousarray(np.asarray(
        kv_indptr.cpu().numpy() if hasattr(kv_indptr, "cpu") else kv_indptr, dtype=np.int64))
    BL, Hq, d = qd.shape
    Hkv = kd.shape[1]
    B = BL // Ld
    rows = np.arange(BL, dtype=np.int32) if rows is None else _i32(rows)
    o = np.zeros((len(rows), Hq, d), dtype=np.float64)
    lse = np.zeros((len(rows), Hq), dtype=np.float64)
    if kv_indices is None:
        rc = lib.oracle_verify_fp8(_ptr(qd), _ptr(kd), _ptr(vd), _ptr(kc), _ptr(vc),
                                   float(k_scale), float(v_scale), _ptr(indptr), B, Ld, Hq, Hkv,
                                   d, float(scale), _ptr(rows), len(rows), _ptr(o), _ptr(lse),
                                   nthreads or default_threads())
    else:
        idx = _i32(kv_indices)
        rc = lib.oracle_verify_fp8_paged(_ptr(qd), _ptr(kd), _ptr(vd), _ptr(kc), _ptr(vc),
                                         float(k_scale), float(v_scale), _ptr(indptr), _ptr(idx),
                                         B, Ld, Hq, Hkv, d, float(scale), _ptr(rows), len(rows),
                                         _ptr(o), _ptr(lse), nthreads or default_threads())
    assert rc == 0, "oracle_verify_fp8 rejected its arguments"
    return o, lse


def sparse_latent(q, latent, idx, scale: float, rows=None, nthreads: int | None = None,
                  lib=None):
    """O [nrows, H, dl] and LSE [nrows, H]; q [T, H, dl], latent [Tk, dl],
    idx [T, topk] int32 with -1 padding.  An index outside [-1, Tk) names no
    latent row: ValueError, before anything is read through it."""
    lib = lib or load()
    q, lat, idx = _f32(q), _f32(latent), _i32(idx)
    T, H, dl = q.shape
    Tk = lat.shape[0]
    if lat.shape[1] != dl or idx.shape[0] != T:
        raise ValueError("sparse_latent: latent [Tk, dl] and idx [T, topk] must match q")
    topk = idx.shape[1]
    rows = np.arange(T, dtype=np.int32) if rows is None else _i32(rows)
    o = np.zeros((len(rows), H, dl), dtype=np.float64)
    lse = np.zeros((len(rows), H), dtype=np.float64)
    rc = lib.oracle_sparse_latent(_ptr(q), _ptr(lat), _ptr(idx), T, Tk, H, dl, topk,
                                  float(scale), _ptr(rows), len(rows), _ptr(o), _ptr(lse),
                                  nthreads or default_threads())
    if rc == -2:
        raise ValueError("sparse_latent: an index entry is outside [-1, Tk) or a row "
                         "outside [0, T)")
    assert rc == 0, "oracle_sparse_latent rejected its arguments"
    return o, lse
