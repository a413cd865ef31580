"""psa_verify_fwd_noalloc: split-KV verify for callers that cannot allocate
device memory where they call attention (a host whose device memory belongs
to another allocator, or a loop that cannot afford cudaMalloc's implicit
device synchronisation).  Its partials live in the library's fixed 16 MiB
device array instead of a caller workspace.

This file is collected last on purpose, so a run that stops at the first
failure has already run every other test.  It must pass both alone in a
fresh process and after the other tests (which leave the array holding the
previous call's data -- nothing in it needs to start at zero)."""
import ctypes

import numpy as np
import pytest
import torch

import oracle

import shared_prefix_attention_b200 as psa
from shared_prefix_attention_b200 import workloads as W
from parity import errors, O_MAX_ABS, O_REL_FRO, LSE_MAX_ABS

pytestmark = pytest.mark.gpu


def _inputs(seed, lens):
    wl = W.VerifyWorkload("noalloc", B=len(lens), L=0, Ld=4, Hq=16, Hkv=4, d=128, nsplit=8,
                          prefix_lens=lens, seed=seed)
    dev = "cuda"
    q, kd, vd, kc, vc = (t.to(dev) for t in wl.make("cpu"))
    indptr = torch.tensor(wl.kv_indptr(), dtype=torch.int32, device=dev)
    return wl, (q, kd, vd, kc, vc), indptr


def _noalloc_call(wl, ts, indptr, status):
    """Straight through the C ABI (ctypes), as a non-Python caller would."""
    q, kd, vd, kc, vc = ts
    o = torch.empty_like(q)
    lse = torch.empty(q.shape[:2], dtype=torch.float32, device=q.device)
    P = ctypes.c_void_p
    rc = psa.lib().psa_verify_fwd_noalloc(
        P(q.data_ptr()), P(kd.data_ptr()), P(vd.data_ptr()), P(kc.data_ptr()),
        P(vc.data_ptr()), kc.shape[0], P(indptr.data_ptr()), max(wl.lens()), None,
        P(o.data_ptr()), P(lse.data_ptr()), wl.B, wl.Ld, wl.Hq, wl.Hkv, wl.d, wl.scale,
        wl.nsplit, None, P(status.data_ptr()),
        P(torch.cuda.current_stream().cuda_stream))
    assert rc == psa.PSA_OK, psa.status_string(rc)
    return o, lse


def test_noalloc_matches_workspace_entry_on_two_calls():
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    # two calls in a row with different shapes and data: the second reuses
    # the array the first one filled.  Both entries run the same kernels with
    # the same split count on the same inputs, so their results are
    # bit-identical; a stale split row left in the array would break that.
    for seed, lens in ((21, [700, 64, 1500]), (22, [33, 2048])):
        wl, ts, indptr = _inputs(seed, lens)
        o_na, l_na = _noalloc_call(wl, ts, indptr, status)
        o_ws, l_ws = psa.verify(*ts, indptr, max(wl.lens()), wl.scale, wl.Ld,
                                nsplit=wl.nsplit)
        torch.cuda.synchronize()
        assert psa.read_status(status) == 0
        assert torch.equal(o_na, o_ws)
        assert torch.equal(l_na, l_ws)
        # and pinned to the fp64 oracle directly
        q, kd, vd, kc, vc = (t.cpu() for t in ts)
        ro, rl = oracle.verify(q, kd, vd, kc, vc, np.array(wl.kv_indptr(), dtype=np.int64),
                               wl.Ld, wl.scale)
        e = errors(o_na, l_na, ro, rl)
        assert e["o_max_abs"] <= O_MAX_ABS and e["o_rel_fro"] <= O_REL_FRO, e
        assert e["lse_max_abs"] <= LSE_MAX_ABS, e


def test_noalloc_python_wrapper_matches_workspace_entry():
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    wl, ts, indptr = _inputs(24, [300, 1024, 5])
    o_na, l_na = psa.verify_noalloc(*ts, indptr, max(wl.lens()), wl.scale, wl.Ld,
                                    nsplit=wl.nsplit, status=status)
    o_ws, l_ws = psa.verify(*ts, indptr, max(wl.lens()), wl.scale, wl.Ld, nsplit=wl.nsplit)
    torch.cuda.synchronize()
    assert psa.read_status(status) == 0
    assert torch.equal(o_na, o_ws) and torch.equal(l_na, l_ws)
    with pytest.raises(ValueError):
        psa.verify_noalloc(ts[0][:-1], *ts[1:], indptr, max(wl.lens()), wl.scale, wl.Ld)


def test_noalloc_rejects_calls_beyond_the_scratch():
    wl, ts, indptr = _inputs(23, [64])
    q, kd, vd, kc, vc = ts
    # 256 splits x 4096 rows x 129 floats is far beyond 16 MiB
    big_B = 64
    need = psa.verify_workspace_size(big_B, 4, 16, 128, 256)
    assert need > (16 << 20)
    P = ctypes.c_void_p
    rc = psa.lib().psa_verify_fwd_noalloc(
        P(q.data_ptr()), P(kd.data_ptr()), P(vd.data_ptr()), P(kc.data_ptr()),
        P(vc.data_ptr()), kc.shape[0], P(indptr.data_ptr()), 64, None, P(q.data_ptr()),
        None, big_B, 4, 16, 4, 128, wl.scale, 256, None, None, None)
    assert rc == psa.PSA_ERR_WORKSPACE
