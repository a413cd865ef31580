"""The C-ABI library loads and exports every symbol include/psa.h declares;
host-side validation returns the documented statuses before any GPU work.
No call here launches a kernel, so these run without a GPU."""
import ctypes
import os
import re

import pytest

import shared_prefix_attention_b200 as psa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_symbols():
    text = open(os.path.join(ROOT, "include", "psa.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(psa_[a-z0-9_]+)\s*\(", text)))


def test_library_exports_every_declared_symbol():
    L = psa.lib()
    declared = _declared_symbols()
    assert declared, "no declarations parsed"
    assert set(declared) == set(psa.EXPORTS)
    for name in declared:
        assert hasattr(L, name), name


def test_version_and_status_strings():
    assert psa.lib().psa_version() == 1
    for code in range(7):
        assert psa.status_string(code)
    assert "unsupported" in psa.status_string(psa.PSA_ERR_UNSUPPORTED)


def _verify_call(**kw):
    """psa_verify_fwd with dummy (never dereferenced) pointers: every case
    below is refused on the host before any CUDA call."""
    args = dict(q=16, kd=16, vd=16, kc=16, vc=16, ntok=64, indptr=16, maxlen=64, kvi=None,
                o=16, lse=None, B=1, Ld=4, Hq=8, Hkv=2, d=128, scale=0.1, nsplit=1,
                feat=None, ws=None, wsb=0)
    args.update(kw)
    a = args
    P = ctypes.c_void_p
    return psa.lib().psa_verify_fwd(
        P(a["q"]), P(a["kd"]), P(a["vd"]), P(a["kc"]), P(a["vc"]), a["ntok"], P(a["indptr"]),
        a["maxlen"], P(a["kvi"]) if a["kvi"] else None, P(a["o"]), None, a["B"], a["Ld"],
        a["Hq"], a["Hkv"], a["d"], a["scale"], a["nsplit"],
        ctypes.byref(a["feat"]) if a["feat"] is not None else None,
        P(a["ws"]) if a["ws"] else None, a["wsb"], None, None)


@pytest.mark.parametrize("field,value", [
    ("has_custom_mask", 1), ("is_causal", 0), ("sliding_window", 128), ("has_sinks", 1),
    ("logit_cap", 30.0), ("xai_temperature_len", 5), ("ragged_extend", 1)])
def test_verify_gating_refuses_unsupported_features(field, value):
    """Split-KV verify gating ("can_handle" in the split-KV verify PR's key
    code): each unsupported feature is refused with PSA_ERR_UNSUPPORTED."""
    f = psa.VerifyFeatures(0, 1, -1, 0, 0.0, -1, 0)
    setattr(f, field, value)
    assert _verify_call(feat=f) == psa.PSA_ERR_UNSUPPORTED


def test_verify_host_validation():
    assert _verify_call(kvi=16) == psa.PSA_ERR_WORKSPACE            # paged: passes the gate
    assert _verify_call(d=96) == psa.PSA_ERR_UNSUPPORTED             # head dim
    assert _verify_call(Hq=6, Hkv=4) == psa.PSA_ERR_INVALID_ARG      # Hq % Hkv
    assert _verify_call(scale=0.0) == psa.PSA_ERR_INVALID_ARG
    assert _verify_call(q=8) == psa.PSA_ERR_INVALID_ARG              # misaligned
    assert _verify_call(Ld=17) == psa.PSA_ERR_UNSUPPORTED            # draft block too big
    assert _verify_call(nsplit=257) == psa.PSA_ERR_INVALID_ARG
    assert _verify_call(ws=None) == psa.PSA_ERR_WORKSPACE
    need = psa.verify_workspace_size(1, 4, 8, 128, 1)
    assert _verify_call(ws=256, wsb=need - 1) == psa.PSA_ERR_WORKSPACE
    assert _verify_call(ws=8, wsb=need) == psa.PSA_ERR_WORKSPACE     # alignment
    assert _verify_call(B=0) == psa.PSA_OK                           # nothing to do


def _shared_call(**kw):
    """psa_verify_shared_fwd with dummy (never dereferenced) pointers: every
    case below is refused on the host before any CUDA call."""
    a = dict(q=16, kd=16, vd=16, kp=16, vp=16, L=512, o=16, B=2, Ld=4, Hq=8, Hkv=2, d=128,
             scale=0.1, nsplit=2, ws=None, wsb=0)
    a.update(kw)
    P = ctypes.c_void_p
    return psa.lib().psa_verify_shared_fwd(
        P(a["q"]), P(a["kd"]), P(a["vd"]), P(a["kp"]) if a["kp"] else None,
        P(a["vp"]) if a["vp"] else None, a["L"], P(a["o"]), None, a["B"], a["Ld"], a["Hq"],
        a["Hkv"], a["d"], a["scale"], a["nsplit"], P(a["ws"]) if a["ws"] else None, a["wsb"],
        None, None)


def test_verify_shared_host_validation():
    assert _shared_call(d=256) == psa.PSA_ERR_UNSUPPORTED             # head dim
    assert _shared_call(Hq=24, Hkv=1) == psa.PSA_ERR_UNSUPPORTED      # 24 rows per token
    assert _shared_call(Ld=17) == psa.PSA_ERR_UNSUPPORTED             # draft block too big
    assert _shared_call(Hq=6, Hkv=4) == psa.PSA_ERR_INVALID_ARG       # Hq % Hkv
    assert _shared_call(scale=0.0) == psa.PSA_ERR_INVALID_ARG
    assert _shared_call(L=-1) == psa.PSA_ERR_INVALID_ARG
    assert _shared_call(L=(1 << 30) + 1) == psa.PSA_ERR_INVALID_ARG
    assert _shared_call(kp=None) == psa.PSA_ERR_INVALID_ARG            # prefix missing
    assert _shared_call(q=8) == psa.PSA_ERR_INVALID_ARG                # misaligned
    assert _shared_call(nsplit=257) == psa.PSA_ERR_INVALID_ARG
    assert _shared_call(ws=None) == psa.PSA_ERR_WORKSPACE
    need = psa.verify_workspace_size(2, 4, 8, 128, 2)
    assert _shared_call(ws=256, wsb=need - 1) == psa.PSA_ERR_WORKSPACE
    assert _shared_call(ws=8, wsb=need) == psa.PSA_ERR_WORKSPACE       # alignment
    assert _shared_call(B=0) == psa.PSA_OK                             # nothing to do


def test_verify_shared_auto_splits():
    n = psa.verify_shared_auto_splits(32, 4, 32, 8, 16384)
    assert 1 <= n <= 256
    # one wave of (chunk, KV head, 256-row block) units on a 148-SM part
    units = n * 8 * 2
    assert 74 < units <= 148
    assert psa.verify_shared_auto_splits(32, 4, 32, 8, 100) == 1     # short prefix
    assert psa.verify_shared_auto_splits(1, 1, 1, 1, 1 << 20) <= 256


def test_verify_tree_needs_a_mask():
    P = ctypes.c_void_p
    f = psa.VerifyFeatures(1, 1, -1, 0, 0.0, -1, 0)
    rc = psa.lib().psa_verify_tree_fwd(P(16), P(16), P(16), P(16), P(16), 64, P(16), 64, None,
                                       None, P(16), None, 1, 4, 8, 2, 128, 0.1, 1,
                                       ctypes.byref(f), None, 0, None, None)
    assert rc == psa.PSA_ERR_INVALID_ARG
    # with a mask the custom-mask feature passes the gate (then the workspace is missing)
    rc = psa.lib().psa_verify_tree_fwd(P(16), P(16), P(16), P(16), P(16), 64, P(16), 64, None,
                                       P(16), P(16), None, 1, 4, 8, 2, 128, 0.1, 1,
                                       ctypes.byref(f), None, 0, None, None)
    assert rc == psa.PSA_ERR_WORKSPACE


def _extend_call(**kw):
    args = dict(qo=16, nrows=6, maxld=4, B=2, mask=None, mi=None, feat=None, ws=None, wsb=0,
                sc=None, d=128)
    args.update(kw)
    a = args
    P = ctypes.c_void_p
    opt = lambda v: P(v) if v else None  # noqa: E731
    sc = ctypes.byref(a["sc"]) if a["sc"] is not None else None
    return psa.lib().psa_verify_extend_fwd(
        P(16), P(16), P(16), P(16), P(16), 64, opt(a["qo"]), a["nrows"], a["maxld"], P(16), 64,
        None, opt(a["mask"]), opt(a["mi"]), sc, P(16), None, a["B"], 8, 2, a["d"], 0.1, 1,
        ctypes.byref(a["feat"]) if a["feat"] is not None else None, opt(a["ws"]), a["wsb"],
        None, None)


def test_verify_extend_host_validation():
    """The extend entry takes ragged draft counts and tree masks (can_handle's
    two refusals) and checks what the host can see."""
    ragged_tree = psa.VerifyFeatures(1, 1, -1, 0, 0.0, -1, 1)
    assert _extend_call(feat=ragged_tree, mask=16, mi=16) == psa.PSA_ERR_WORKSPACE
    assert _extend_call(qo=None) == psa.PSA_ERR_INVALID_ARG          # qo_indptr required
    assert _extend_call(mask=16) == psa.PSA_ERR_INVALID_ARG          # mask without mask_indptr
    assert _extend_call(feat=ragged_tree) == psa.PSA_ERR_UNSUPPORTED  # custom mask flag, no mask
    assert _extend_call(nrows=9) == psa.PSA_ERR_INVALID_ARG          # more rows than B * max
    assert _extend_call(maxld=17) == psa.PSA_ERR_UNSUPPORTED         # m-tile plan: 17 * 4 > 128
    assert _extend_call(nrows=0) == psa.PSA_OK                       # no draft rows
    # an e4m3 cache: head_dim 128 only, finite positive scales
    assert _extend_call(sc=psa.KvScales(0.5, 0.25)) == psa.PSA_ERR_WORKSPACE
    assert _extend_call(sc=psa.KvScales(0.5, 0.25), d=64) == psa.PSA_ERR_UNSUPPORTED
    assert _extend_call(sc=psa.KvScales(0.0, 0.25)) == psa.PSA_ERR_INVALID_ARG
    assert _extend_call(sc=psa.KvScales(0.5, float("inf"))) == psa.PSA_ERR_INVALID_ARG


def test_verify_fp8_host_validation():
    P = ctypes.c_void_p

    def call(d=128, ks=0.1, vs=0.1, B=1, kvi=None):
        return psa.lib().psa_verify_fp8_fwd(P(16), P(16), P(16), P(16), P(16), 64, P(16), 64,
                                            P(kvi) if kvi else None, ks, vs, P(16), None, B, 4,
                                            8, 2, d, 0.1, 1, None, None, 0, None, None)
    assert call(d=64) == psa.PSA_ERR_UNSUPPORTED       # e4m3 path is head_dim 128 only
    assert call(kvi=16) == psa.PSA_ERR_WORKSPACE       # paged cache: passes the gate
    assert call(ks=0.0) == psa.PSA_ERR_INVALID_ARG
    assert call(vs=float("inf")) == psa.PSA_ERR_INVALID_ARG
    assert call() == psa.PSA_ERR_WORKSPACE
    assert call(B=0) == psa.PSA_OK


def test_verify_workspace_size_formula():
    B, Ld, Hq, d, ns = 32, 4, 32, 128, 32
    rows = ns * B * Ld * Hq
    assert psa.verify_workspace_size(B, Ld, Hq, d, ns) >= rows * (d + 1) * 4
    assert psa.verify_workspace_size(0, Ld, Hq, d, ns) == 0


def test_auto_splits_bounds():
    assert 1 <= psa.verify_auto_splits(32, 16384, 8, 128) <= 256
    assert psa.verify_auto_splits(1, 100, 8, 128) == 1
    assert psa.verify_auto_splits(1, 1 << 20, 8, 128) <= 256


def test_prefill_and_sparse_host_validation():
    L = psa.lib()
    P = ctypes.c_void_p
    assert L.psa_prefill_fwd(P(16), P(16), P(16), P(16), None, 0, 10, 4, 3, 128, 0.1, P(16), 8,
                             None, 0, None, None) == psa.PSA_ERR_INVALID_ARG
    assert L.psa_prefill_fwd(P(16), P(16), P(16), P(16), None, 0, 10, 4, 2, 96, 0.1, P(16), 8,
                             None, 0, None, None) == psa.PSA_ERR_UNSUPPORTED
    assert L.psa_prefill_fwd(P(16), P(16), P(16), P(16), None, 7, 10, 4, 2, 128, 0.1, P(16), 8,
                             None, 0, None, None) == psa.PSA_ERR_INVALID_ARG
    assert L.psa_sparse_latent_fwd(P(16), P(16), P(16), P(16), None, 4, 8, 64, 256, 16, 0.1,
                                   None, None) == psa.PSA_ERR_UNSUPPORTED
    assert L.psa_sparse_latent_fwd(P(16), P(16), P(16), P(16), None, 4, 8, 64, 512, 0, 0.1,
                                   None, None) == psa.PSA_ERR_INVALID_ARG
    assert psa.prefill_tiles(128) == (256, 128)
    with pytest.raises(psa.PsaError):
        psa.prefill_tiles(80)


def test_python_binding_refuses_cpu_tensors():
    """No CPU fallback: every compute entry of the binding refuses host
    tensors before any library call."""
    import torch
    x = torch.zeros(4, 2, 64, dtype=torch.bfloat16)
    i32 = torch.zeros(3, dtype=torch.int32)
    with pytest.raises(ValueError):
        psa.sparse_latent(x, x[:, 0], torch.zeros(4, 1, dtype=torch.int32), 0.1)
    with pytest.raises(ValueError):
        psa.verify(x, x, x, x, x, i32, 8, 0.1, 2)
    with pytest.raises(ValueError):
        psa.verify_tree(x, x, x, x, x, i32, 8, torch.ones(4, 2, dtype=torch.uint8), 0.1, 2)
    with pytest.raises(ValueError):
        psa.verify_extend(x, x, x, x, x, i32, 2, i32, 8, 0.1)
    with pytest.raises(ValueError):
        psa.verify_shared(x, x, x, x, x, 0.1, 2)
    with pytest.raises(ValueError):
        psa.verify_fp8(x, x, x, x, x, 1.0, 1.0, i32, 8, 0.1, 2)
