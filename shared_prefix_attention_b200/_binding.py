"""ctypes binding of libpsa.  Argument marshalling only: every step of the
attention path runs in the library's CUDA kernels; PyTorch supplies device
memory and the current stream.  There is no CPU fallback -- if the library
is missing, importing a call raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Sequence

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libpsa.so")
# The same library built with device-side bounds checks (PSA_DEBUG): an index
# taken from caller data outside its buffer is reported as PSA_ERR_BOUNDS
# through the status word instead of being followed.
DEBUG_LIB_PATH = os.path.join(_HERE, "libpsa_debug.so")

PSA_OK = 0
PSA_ERR_INVALID_ARG = 1
PSA_ERR_UNSUPPORTED = 2
PSA_ERR_WORKSPACE = 3
PSA_ERR_CUDA = 4
PSA_ERR_TIMEOUT = 5
PSA_ERR_CAPACITY = 6
PSA_ERR_BOUNDS = 7
PSA_BF16 = 0
PSA_F32 = 1

# Every symbol include/psa.h declares.
EXPORTS = [
    "psa_version", "psa_status_string", "psa_spec_flat", "psa_build_spec",
    "psa_build_schedule", "psa_prefill_tiles", "psa_prefill_workspace_size",
    "psa_prefill_fwd", "psa_verify_auto_splits", "psa_verify_workspace_size",
    "psa_verify_fwd", "psa_verify_fwd_noalloc", "psa_sparse_latent_fwd", "psa_read_status",
    "psa_wait_selftest", "psa_verify_shared_auto_splits", "psa_verify_shared_fwd",
    "psa_verify_shared_tree_fwd",
    "psa_verify_fp8_fwd", "psa_transpose_spec", "psa_prefill_bwd_tiles",
    "psa_prefill_bwd_workspace_size", "psa_prefill_bwd", "psa_verify_tree_fwd",
    "psa_verify_extend_fwd",
]


class PsaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} (status {status})")


class Segment(ctypes.Structure):
    _fields_ = [("len", ctypes.c_int32), ("parent", ctypes.c_int32)]


class Rect(ctypes.Structure):
    _fields_ = [("q0", ctypes.c_int32), ("q1", ctypes.c_int32), ("k0", ctypes.c_int32),
                ("k1", ctypes.c_int32), ("causal", ctypes.c_int32)]


class VerifyFeatures(ctypes.Structure):
    _fields_ = [("has_custom_mask", ctypes.c_int32), ("is_causal", ctypes.c_int32),
                ("sliding_window", ctypes.c_int32), ("has_sinks", ctypes.c_int32),
                ("logit_cap", ctypes.c_float), ("xai_temperature_len", ctypes.c_int32),
                ("ragged_extend", ctypes.c_int32)]


class KvScales(ctypes.Structure):
    """psa_kv_scales: per-tensor scales of an e4m3 KV cache."""
    _fields_ = [("k_scale", ctypes.c_float), ("v_scale", ctypes.c_float)]


_lib = None


def lib():
    """The loaded libpsa (raises if it has not been built)."""
    global _lib
    if _lib is None:
        _lib = load(LIB_PATH)
    return _lib


class use_library:
    """Context manager: the binding's calls go to the library at ``path``
    (e.g. DEBUG_LIB_PATH) inside the block, and back to the previous one
    after it."""

    def __init__(self, path: str):
        self.path = path

    def __enter__(self):
        global _lib
        self.saved = _lib
        _lib = load(self.path)
        return _lib

    def __exit__(self, *exc):
        global _lib
        _lib = self.saved
        return False


_loaded: dict = {}


def load(path: str):
    """Load a build of libpsa and declare its C signatures (cached per path;
    raises if the file is missing)."""
    if path in _loaded:
        return _loaded[path]
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is missing: build it with "
                           "`python -m shared_prefix_attention_b200.build`")
    L = ctypes.CDLL(path)
    P, I32, I64, SZ, F = (ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t,
                          ctypes.c_float)
    sig = {
        "psa_version": ([], ctypes.c_int),
        "psa_status_string": ([ctypes.c_int], ctypes.c_char_p),
        "psa_spec_flat": ([I32, I32, I32, P, I32, P], ctypes.c_int),
        "psa_build_spec": ([P, I32, P, I32, P], ctypes.c_int),
        "psa_build_schedule": ([P, I32, P, I32, I32, I32, P, I64, P], ctypes.c_int),
        "psa_prefill_tiles": ([I32, P, P], ctypes.c_int),
        "psa_prefill_workspace_size": ([ctypes.c_int, I32, I32, I32, I32], SZ),
        "psa_prefill_fwd": ([P, P, P, P, P, ctypes.c_int, I32, I32, I32, I32, F, P, I64, P, SZ,
                             P, P], ctypes.c_int),
        "psa_verify_auto_splits": ([I32, I64, I32, I32], I32),
        "psa_verify_workspace_size": ([I32, I32, I32, I32, I32], SZ),
        "psa_verify_fwd": ([P, P, P, P, P, I64, P, I64, P, P, P, I32, I32, I32, I32, I32, F, I32,
                            P, P, SZ, P, P], ctypes.c_int),
        "psa_verify_fwd_noalloc": ([P, P, P, P, P, I64, P, I64, P, P, P, I32, I32, I32, I32, I32,
                                    F, I32, P, P, P], ctypes.c_int),
        "psa_sparse_latent_fwd": ([P, P, P, P, P, I32, I32, I32, I32, I32, F, P, P],
                                  ctypes.c_int),
        "psa_read_status": ([P, P, P], ctypes.c_int),
        "psa_wait_selftest": ([I32, P, P], ctypes.c_int),
        "psa_verify_shared_auto_splits": ([I32, I32, I32, I32, I64], I32),
        "psa_transpose_spec": ([P, I32, P], ctypes.c_int),
        "psa_prefill_bwd_tiles": ([I32, P, P], ctypes.c_int),
        "psa_verify_tree_fwd": ([P, P, P, P, P, I64, P, I64, P, P, P, P, I32, I32, I32, I32, I32,
                                 F, I32, P, P, SZ, P, P], ctypes.c_int),
        "psa_verify_extend_fwd": ([P, P, P, P, P, I64, P, I32, I32, P, I64, P, P, P, P, P, P,
                                   I32, I32, I32, I32, F, I32, P, P, SZ, P, P], ctypes.c_int),
        "psa_prefill_bwd_workspace_size": ([I32, I32], SZ),
        "psa_prefill_bwd": ([P, P, P, P, P, P, P, P, P, I32, I32, I32, I32, F, P, I64, P, I64, P,
                             SZ, P, P], ctypes.c_int),
        "psa_verify_fp8_fwd": ([P, P, P, P, P, I64, P, I64, P, F, F, P, P, I32, I32, I32, I32,
                                I32, F, I32, P, P, SZ, P, P], ctypes.c_int),
        "psa_verify_shared_tree_fwd": ([P, P, P, P, P, I64, P, P, P, I32, I32, I32, I32, I32, F,
                                        I32, P, ctypes.c_size_t, P, P], ctypes.c_int),
        "psa_verify_shared_fwd": ([P, P, P, P, P, I64, P, P, I32, I32, I32, I32, I32, F, I32, P,
                                   ctypes.c_size_t, P, P], ctypes.c_int),
    }
    for name, (args, res) in sig.items():
        fn = getattr(L, name)
        fn.argtypes = args
        fn.restype = res
    _loaded[path] = L
    return L


def status_string(status: int) -> str:
    return lib().psa_status_string(int(status)).decode()


def _check(rc: int, where: str):
    if rc != PSA_OK:
        raise PsaError(rc, where)


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, np.ndarray):
        return t.ctypes.data_as(ctypes.c_void_p)
    return ctypes.c_void_p(t.data_ptr())


def _stream(device) -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _require_cuda(*ts):
    for t in ts:
        if t is not None and not t.is_cuda:
            raise ValueError("psa kernels take CUDA tensors; there is no CPU path")
        if t is not None and not t.is_contiguous():
            raise ValueError("psa kernels take contiguous tensors")


# ---------------------------------------------------------------- host spec

def spec_flat(P: int, N: int, S: int) -> list[tuple[int, int]]:
    n = ctypes.c_int32(0)
    lib().psa_spec_flat(P, N, S, None, 0, ctypes.byref(n))
    arr = (Segment * max(1, n.value))()
    _check(lib().psa_spec_flat(P, N, S, arr, n.value, ctypes.byref(n)), "psa_spec_flat")
    return [(arr[i].len, arr[i].parent) for i in range(n.value)]


def build_spec(segments: Sequence[tuple[int, int]]) -> np.ndarray:
    """Rectangles [n, 5] int32 (q0, q1, k0, k1, causal) for a segment forest."""
    segs = (Segment * max(1, len(segments)))(*[Segment(int(a), int(b)) for a, b in segments])
    n = ctypes.c_int32(0)
    rc = lib().psa_build_spec(segs, len(segments), None, 0, ctypes.byref(n))
    if rc not in (PSA_OK, PSA_ERR_CAPACITY):
        _check(rc, "psa_build_spec")
    out = np.zeros((max(1, n.value), 5), dtype=np.int32)
    _check(lib().psa_build_spec(segs, len(segments), _ptr(out), n.value, ctypes.byref(n)),
           "psa_build_spec")
    return out[:n.value]


def prefill_tiles(head_dim: int) -> tuple[int, int]:
    m, n = ctypes.c_int32(0), ctypes.c_int32(0)
    _check(lib().psa_prefill_tiles(head_dim, ctypes.byref(m), ctypes.byref(n)),
           "psa_prefill_tiles")
    return m.value, n.value


def build_schedule(rects: np.ndarray, cu_seqlens: Sequence[int], tile_m: int,
                   tile_n: int) -> np.ndarray:
    """Tile schedule (host int32 array) for :func:`prefill`."""
    rects = np.ascontiguousarray(rects, dtype=np.int32)
    cu = np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int32))
    n = ctypes.c_int64(0)
    ng = len(cu) - 1
    rc = lib().psa_build_schedule(_ptr(rects), len(rects), _ptr(cu), ng, tile_m, tile_n, None, 0,
                                  ctypes.byref(n))
    if rc not in (PSA_OK, PSA_ERR_CAPACITY):
        _check(rc, "psa_build_schedule")
    out = np.zeros(n.value, dtype=np.int32)
    _check(lib().psa_build_schedule(_ptr(rects), len(rects), _ptr(cu), ng, tile_m, tile_n,
                                    _ptr(out), n.value, ctypes.byref(n)), "psa_build_schedule")
    return out


def transpose_spec(rects: np.ndarray) -> np.ndarray:
    """Rectangles with rows and columns swapped (keys become rows)."""
    rects = np.ascontiguousarray(rects, dtype=np.int32)
    out = np.zeros_like(rects)
    _check(lib().psa_transpose_spec(_ptr(rects), len(rects), _ptr(out)), "psa_transpose_spec")
    return out


def plan_prefill(segments, cu_seqlens, head_dim: int, device="cuda") -> torch.Tensor:
    """Spec + schedule for a segment forest, uploaded to ``device``."""
    tm, tn = prefill_tiles(head_dim)
    sched = build_schedule(build_spec(segments), cu_seqlens, tm, tn)
    return torch.from_numpy(sched).to(device)


# ---------------------------------------------------------------- kernels

def prefill(q, k, v, schedule: torch.Tensor, scale: float, out=None, lse=None,
            workspace=None, status=None):
    """O [T, Hq, d] (q's dtype) and LSE [T, Hq] fp32 over the flat layout."""
    _require_cuda(q, k, v, schedule)
    T, Hq, d = q.shape
    Hkv = k.shape[1]
    dtype = {torch.bfloat16: PSA_BF16, torch.float32: PSA_F32}[q.dtype]
    out = torch.empty_like(q) if out is None else out
    lse = torch.empty((T, Hq), dtype=torch.float32, device=q.device) if lse is None else lse
    if workspace is None:
        nbytes = lib().psa_prefill_workspace_size(dtype, T, Hq, Hkv, d)
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=q.device)
    rc = lib().psa_prefill_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), dtype, T, Hq,
                               Hkv, d, float(scale), _ptr(schedule), schedule.numel(),
                               _ptr(workspace), workspace.numel(), _ptr(status),
                               _stream(q.device))
    _check(rc, "psa_prefill_fwd")
    return out, lse


def verify_workspace_size(B: int, Ld: int, Hq: int, head_dim: int, nsplit: int) -> int:
    return int(lib().psa_verify_workspace_size(B, Ld, Hq, head_dim, nsplit))


def verify_auto_splits(B: int, max_prefix_len: int, Hkv: int, head_dim: int) -> int:
    return int(lib().psa_verify_auto_splits(B, max_prefix_len, Hkv, head_dim))


def verify(q_draft, k_draft, v_draft, k_cache, v_cache, kv_indptr: torch.Tensor,
           max_prefix_len: int, scale: float, Ld: int, nsplit: int = 0, out=None, lse=None,
           workspace=None, status=None, features: VerifyFeatures | None = None,
           kv_indices=None):
    """Split-KV verify.  kv_indptr: device int32 [B+1] prefix offsets."""
    _require_cuda(q_draft, k_draft, v_draft, k_cache, v_cache, kv_indptr)
    BL, Hq, d = q_draft.shape
    Hkv = k_cache.shape[1]
    B = BL // Ld
    if nsplit == 0:
        nsplit = verify_auto_splits(B, max_prefix_len, Hkv, d)
    out = torch.empty_like(q_draft) if out is None else out
    lse = torch.empty((BL, Hq), dtype=torch.float32, device=q_draft.device) if lse is None else lse
    if workspace is None:
        workspace = torch.empty(max(256, verify_workspace_size(B, Ld, Hq, d, nsplit)),
                                dtype=torch.uint8, device=q_draft.device)
    rc = lib().psa_verify_fwd(_ptr(q_draft), _ptr(k_draft), _ptr(v_draft), _ptr(k_cache),
                              _ptr(v_cache), k_cache.shape[0], _ptr(kv_indptr),
                              int(max_prefix_len), _ptr(kv_indices), _ptr(out), _ptr(lse), B,
                              Ld, Hq, Hkv, d, float(scale), nsplit,
                              ctypes.byref(features) if features is not None else None,
                              _ptr(workspace), workspace.numel(), _ptr(status),
                              _stream(q_draft.device))
    _check(rc, "psa_verify_fwd")
    return out, lse


def verify_noalloc(q_draft, k_draft, v_draft, k_cache, v_cache, kv_indptr: torch.Tensor,
                   max_prefix_len: int, scale: float, Ld: int, nsplit: int = 0, out=None,
                   lse=None, status=None):
    """Split-KV verify through psa_verify_fwd_noalloc: the library's fixed
    device scratch replaces the workspace (for callers that cannot allocate
    device memory at the call site).  Outputs are allocated here only for
    convenience; pass ``out`` / ``lse`` to avoid that too."""
    _require_cuda(q_draft, k_draft, v_draft, k_cache, v_cache, kv_indptr)
    BL, Hq, d = q_draft.shape
    Hkv = k_cache.shape[1]
    if Ld <= 0 or BL % Ld != 0:
        raise ValueError(f"verify_noalloc: {BL} draft rows are not a whole number of "
                         f"requests of {Ld} drafts")
    B = BL // Ld
    out = torch.empty_like(q_draft) if out is None else out
    lse = torch.empty((BL, Hq), dtype=torch.float32, device=q_draft.device) if lse is None else lse
    rc = lib().psa_verify_fwd_noalloc(_ptr(q_draft), _ptr(k_draft), _ptr(v_draft),
                                      _ptr(k_cache), _ptr(v_cache), k_cache.shape[0],
                                      _ptr(kv_indptr), int(max_prefix_len), None, _ptr(out),
                                      _ptr(lse), B, Ld, Hq, Hkv, d, float(scale), nsplit, None,
                                      _ptr(status), _stream(q_draft.device))
    _check(rc, "psa_verify_fwd_noalloc")
    return out, lse


def sparse_latent(q, latent, idx, scale: float, out=None, lse=None, status=None):
    """Shared-latent sparse attention: O [T, H, dl] bf16, LSE [T, H] fp32."""
    _require_cuda(q, latent, idx)
    T, H, dl = q.shape
    out = torch.empty_like(q) if out is None else out
    lse = torch.empty((T, H), dtype=torch.float32, device=q.device) if lse is None else lse
    rc = lib().psa_sparse_latent_fwd(_ptr(q), _ptr(latent), _ptr(idx), _ptr(out), _ptr(lse), T,
                                     latent.shape[0], H, dl, idx.shape[1], float(scale),
                                     _ptr(status), _stream(q.device))
    _check(rc, "psa_sparse_latent_fwd")
    return out, lse


def read_status(status: torch.Tensor) -> int:
    v = ctypes.c_int32(0)
    _check(lib().psa_read_status(_ptr(status), ctypes.byref(v), _stream(status.device)),
           "psa_read_status")
    return v.value


def wait_selftest(status: torch.Tensor, arrive: bool) -> None:
    """Launches the library's bounded-wait self-test on ``status``'s device:
    with ``arrive`` the wait completes at once, without it the wait gives up
    after the library's budget and writes PSA_ERR_TIMEOUT to ``status``."""
    _check(lib().psa_wait_selftest(1 if arrive else 0, _ptr(status), _stream(status.device)),
           "psa_wait_selftest")


def verify_shared_auto_splits(B: int, Ld: int, Hq: int, Hkv: int, prefix_len: int) -> int:
    return int(lib().psa_verify_shared_auto_splits(B, Ld, Hq, Hkv, int(prefix_len)))


def verify_shared(q_draft, k_draft, v_draft, k_prefix, v_prefix, scale: float, Ld: int,
                  nsplit: int = 0, out=None, lse=None, workspace=None, status=None,
                  draft_mask=None):
    """Verify against one prefix shared by every request: O [B*Ld, Hq, d]
    bf16 and LSE [B*Ld, Hq] fp32; k_prefix/v_prefix [L, Hkv, d].  With
    draft_mask (device uint8 [B*Ld, Ld]) the draft block is that tree mask."""
    _require_cuda(q_draft, k_draft, v_draft, k_prefix, v_prefix)
    BL, Hq, d = q_draft.shape
    Hkv = k_draft.shape[1]
    B = BL // Ld
    L = k_prefix.shape[0]
    ns = nsplit or verify_shared_auto_splits(B, Ld, Hq, Hkv, L)
    out = torch.empty_like(q_draft) if out is None else out
    lse = torch.empty((BL, Hq), dtype=torch.float32, device=q_draft.device) if lse is None else lse
    if workspace is None:
        workspace = torch.empty(max(verify_workspace_size(B, Ld, Hq, d, ns), 256),
                                dtype=torch.uint8, device=q_draft.device)
    kp, vp = (_ptr(k_prefix) if L else None), (_ptr(v_prefix) if L else None)
    if draft_mask is None:
        rc = lib().psa_verify_shared_fwd(_ptr(q_draft), _ptr(k_draft), _ptr(v_draft), kp, vp, L,
                                         _ptr(out), _ptr(lse), B, Ld, Hq, Hkv, d, float(scale), ns,
                                         _ptr(workspace), workspace.numel(), _ptr(status),
                                         _stream(q_draft.device))
        _check(rc, "psa_verify_shared_fwd")
    else:
        rc = lib().psa_verify_shared_tree_fwd(_ptr(q_draft), _ptr(k_draft), _ptr(v_draft), kp, vp,
                                              L, _ptr(draft_mask), _ptr(out), _ptr(lse), B, Ld,
                                              Hq, Hkv, d, float(scale), ns, _ptr(workspace),
                                              workspace.numel(), _ptr(status),
                                              _stream(q_draft.device))
        _check(rc, "psa_verify_shared_tree_fwd")
    return out, lse


def verify_fp8(q_draft, k_draft, v_draft, k_cache8, v_cache8, k_scale: float, v_scale: float,
               kv_indptr: torch.Tensor, max_prefix_len: int, scale: float, Ld: int,
               nsplit: int = 0, out=None, lse=None, workspace=None, status=None,
               kv_indices=None):
    """Split-KV verify over an e4m3 prefix cache (uint8 or float8_e4m3fn
    tensors [Ntok, Hkv, d]) standing for k_scale * e4m3 and v_scale * e4m3;
    kv_indices: optional token-granular page table (device int32)."""
    _require_cuda(q_draft, k_draft, v_draft, k_cache8, v_cache8, kv_indptr)
    BL, Hq, d = q_draft.shape
    Hkv = k_draft.shape[1]
    B = BL // Ld
    ns = nsplit or verify_auto_splits(B, max_prefix_len, Hkv, d)
    out = torch.empty_like(q_draft) if out is None else out
    lse = torch.empty((BL, Hq), dtype=torch.float32, device=q_draft.device) if lse is None else lse
    if workspace is None:
        workspace = torch.empty(max(verify_workspace_size(B, Ld, Hq, d, ns), 256),
                                dtype=torch.uint8, device=q_draft.device)
    rc = lib().psa_verify_fp8_fwd(_ptr(q_draft), _ptr(k_draft), _ptr(v_draft), _ptr(k_cache8),
                                  _ptr(v_cache8), k_cache8.shape[0], _ptr(kv_indptr),
                                  int(max_prefix_len), _ptr(kv_indices), float(k_scale),
                                  float(v_scale),
                                  _ptr(out), _ptr(lse), B, Ld, Hq, Hkv, d, float(scale), ns, None,
                                  _ptr(workspace), workspace.numel(), _ptr(status),
                                  _stream(q_draft.device))
    _check(rc, "psa_verify_fp8_fwd")
    return out, lse


def prefill_bwd_tiles(head_dim: int):
    tm, tn = ctypes.c_int32(0), ctypes.c_int32(0)
    _check(lib().psa_prefill_bwd_tiles(head_dim, ctypes.byref(tm), ctypes.byref(tn)),
           "psa_prefill_bwd_tiles")
    return tm.value, tn.value


def plan_prefill_bwd(segments, cu_seqlens, head_dim: int, device="cuda"):
    """The two backward schedules (row-major for dQ, key-major for dK / dV)
    for a segment forest, uploaded to ``device``."""
    tm, tn = prefill_bwd_tiles(head_dim)
    spec = build_spec(segments)
    sq = build_schedule(spec, cu_seqlens, tm, tn)
    skv = build_schedule(transpose_spec(spec), cu_seqlens, tm, tn)
    return torch.from_numpy(sq).to(device), torch.from_numpy(skv).to(device)


def prefill_bwd(q, k, v, o, lse, dout, schedules, scale: float, dq=None, dk=None, dv=None,
                workspace=None, status=None):
    """Gradients (dq, dk, dv) of the prefill output for upstream gradient
    ``dout``; ``schedules`` from :func:`plan_prefill_bwd`."""
    sq, skv = schedules
    _require_cuda(q, k, v, o, lse, dout, sq, skv)
    T, Hq, d = q.shape
    Hkv = k.shape[1]
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    if workspace is None:
        workspace = torch.empty(max(int(lib().psa_prefill_bwd_workspace_size(T, Hq)), 256),
                                dtype=torch.uint8, device=q.device)
    rc = lib().psa_prefill_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(dout),
                               _ptr(dq), _ptr(dk), _ptr(dv), T, Hq, Hkv, d, float(scale),
                               _ptr(sq), sq.numel(), _ptr(skv), skv.numel(), _ptr(workspace),
                               workspace.numel(), _ptr(status), _stream(q.device))
    _check(rc, "psa_prefill_bwd")
    return dq, dk, dv


def verify_tree(q_draft, k_draft, v_draft, k_cache, v_cache, kv_indptr: torch.Tensor,
                max_prefix_len: int, draft_mask: torch.Tensor, scale: float, Ld: int,
                nsplit: int = 0, out=None, lse=None, workspace=None, status=None,
                kv_indices=None):
    """Split-KV verify with a custom draft mask (device uint8 [B*Ld, Ld])."""
    _require_cuda(q_draft, k_draft, v_draft, k_cache, v_cache, kv_indptr, draft_mask)
    BL, Hq, d = q_draft.shape
    Hkv = k_draft.shape[1]
    B = BL // Ld
    ns = nsplit or verify_auto_splits(B, max_prefix_len, Hkv, d)
    out = torch.empty_like(q_draft) if out is None else out
    lse = torch.empty((BL, Hq), dtype=torch.float32, device=q_draft.device) if lse is None else lse
    if workspace is None:
        workspace = torch.empty(max(verify_workspace_size(B, Ld, Hq, d, ns), 256),
                                dtype=torch.uint8, device=q_draft.device)
    feat = VerifyFeatures(1, 1, -1, 0, 0.0, -1, 0)
    rc = lib().psa_verify_tree_fwd(_ptr(q_draft), _ptr(k_draft), _ptr(v_draft), _ptr(k_cache),
                                   _ptr(v_cache), k_cache.shape[0], _ptr(kv_indptr),
                                   int(max_prefix_len), _ptr(kv_indices), _ptr(draft_mask),
                                   _ptr(out),
                                   _ptr(lse), B, Ld, Hq, Hkv, d, float(scale), ns,
                                   ctypes.byref(feat), _ptr(workspace), workspace.numel(),
                                   _ptr(status), _stream(q_draft.device))
    _check(rc, "psa_verify_tree_fwd")
    return out, lse


def verify_extend(q_draft, k_draft, v_draft, k_cache, v_cache, qo_indptr: torch.Tensor,
                  max_draft_len: int, kv_indptr: torch.Tensor, max_prefix_len: int,
                  scale: float, kv_indices=None, draft_mask=None, mask_indptr=None,
                  nsplit: int = 0, out=None, lse=None, workspace=None, status=None,
                  k_scale: float | None = None, v_scale: float | None = None):
    """Verify in the extend form: ragged draft counts (qo_indptr, device int32
    [B+1]), an optional page table (kv_indices: prefix position t is cache row
    kv_indices[t]) and optional per-request tree masks (flat device uint8,
    request b's Lb x Lb block at mask_indptr[b]).  With k_scale / v_scale the
    caches hold e4m3 bytes standing for k_scale * e4m3 and v_scale * e4m3."""
    _require_cuda(q_draft, k_draft, v_draft, k_cache, v_cache, qo_indptr, kv_indptr)
    NR, Hq, d = q_draft.shape
    Hkv = k_draft.shape[1]
    B = qo_indptr.numel() - 1
    ns = nsplit or verify_auto_splits(B, max_prefix_len, Hkv, d)
    out = torch.empty_like(q_draft) if out is None else out
    lse = torch.empty((NR, Hq), dtype=torch.float32, device=q_draft.device) if lse is None else lse
    if workspace is None:
        workspace = torch.empty(max(verify_workspace_size(1, NR, Hq, d, ns), 256),
                                dtype=torch.uint8, device=q_draft.device)
    feat = VerifyFeatures(int(draft_mask is not None), 1, -1, 0, 0.0, -1, 1)
    sc = None
    if k_scale is not None or v_scale is not None:
        sc = ctypes.byref(KvScales(float(k_scale), float(v_scale)))
    rc = lib().psa_verify_extend_fwd(_ptr(q_draft), _ptr(k_draft), _ptr(v_draft),
                                     _ptr(k_cache), _ptr(v_cache), k_cache.shape[0],
                                     _ptr(qo_indptr), NR, int(max_draft_len), _ptr(kv_indptr),
                                     int(max_prefix_len), _ptr(kv_indices), _ptr(draft_mask),
                                     _ptr(mask_indptr), sc, _ptr(out), _ptr(lse), B, Hq, Hkv, d,
                                     float(scale), ns, ctypes.byref(feat), _ptr(workspace),
                                     workspace.numel(), _ptr(status), _stream(q_draft.device))
    _check(rc, "psa_verify_extend_fwd")
    return out, lse
