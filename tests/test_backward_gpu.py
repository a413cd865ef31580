"""Backward of the prefill on the GPU against the fp64 oracle backward
("KV-0 redundancy prefix sharing attention mask design": design summary and
test plan -- the flat layout's gradients equal those of the separate
[prefix; s_i] sequences, which pins the oracle).  Every call goes through the
C ABI.

Tolerance: the kernels round P and dS to bf16 for the tensor cores (relative
error 2^-9 each) and read the forward's bf16 O for D = rowsum(dO * O); dS is
a difference dP - D that cancels where P is large, so the gradients carry a
few times the forward's relative error.  Bar: relative Frobenius error
<= 2e-2 and max |err| <= 2e-2 * max |reference| per gradient."""
import numpy as np
import pytest
import torch

import oracle
import shared_prefix_attention_b200 as psa
from shared_prefix_attention_b200 import workloads as W

pytestmark = pytest.mark.gpu

REL_FRO = 2e-2
MAX_ABS_REL = 2e-2


def _grad_errors(got, ref):
    g = got.float().cpu().numpy().astype(np.float64)
    d = g - ref
    return (float(np.linalg.norm(d) / max(np.linalg.norm(ref), 1e-30)),
            float(np.abs(d).max() / max(np.abs(ref).max(), 1e-30)))


def _run(segs, cu, T, Hq, Hkv, d, seed=100):
    gen = torch.Generator().manual_seed(seed)
    draw = lambda shape: (torch.randn(shape, generator=gen) * 0.5).to(torch.bfloat16)
    q, k, v = draw((T, Hq, d)), draw((T, Hkv, d)), draw((T, Hkv, d))
    dout = draw((T, Hq, d))
    scale = 1.0 / np.sqrt(d)
    qg, kg, vg, dog = (t.cuda() for t in (q, k, v, dout))
    sched = psa.plan_prefill(segs, cu, d, "cuda")
    o, lse = psa.prefill(qg, kg, vg, sched, scale)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    dq, dk, dv = psa.prefill_bwd(qg, kg, vg, o, lse, dog, psa.plan_prefill_bwd(segs, cu, d),
                                 scale, status=status)
    torch.cuda.synchronize()
    assert psa.read_status(status) == 0
    rq, rk, rv = oracle.prefill_bwd(q, k, v, dout, segs, scale)
    return (dq, dk, dv), (rq, rk, rv)


def _check(got, ref, what):
    for name, g, r in zip(("dq", "dk", "dv"), got, ref):
        fro, mx = _grad_errors(g, r)
        assert np.isfinite(g.float().cpu().numpy()).all(), f"{what} {name}: non-finite"
        assert fro <= REL_FRO and mx <= MAX_ABS_REL, f"{what} {name}: fro={fro:.3e} max={mx:.3e}"


@pytest.mark.parametrize("P,N,S,Hq,Hkv,d,groups", [
    (64, 4, 32, 2, 2, 128, 1),     # tile-aligned prefix, suffixes of half a tile
    (100, 3, 37, 4, 2, 64, 1),     # ragged everywhere, GQA 2:1, d = 64
    (128, 2, 64, 2, 1, 128, 2),    # two packed groups, MQA
    (5, 7, 3, 2, 2, 128, 1),       # rows and keys far below one tile
    (300, 2, 41, 2, 2, 128, 1),    # several KV blocks, partial diagonal tiles
    # long units: a prefix key block collects 1024 + 4 * 256 query rows of
    # each of its two query heads, far more ring slots and tiles than above
    (1024, 4, 256, 4, 2, 128, 1),
    (512, 4, 128, 4, 2, 128, 2),   # two packed groups with GQA 2:1
])
def test_backward_parity_flat(P, N, S, Hq, Hkv, d, groups):
    wl = W.PrefillWorkload("t", P=P, N=N, S=S, Hq=Hq, Hkv=Hkv, d=d, groups=groups)
    got, ref = _run(wl.segments(), wl.cu_seqlens(), wl.T, Hq, Hkv, d)
    _check(got, ref, f"P={P} N={N} S={S}")


def test_backward_parity_random_trees():
    g = torch.Generator().manual_seed(12)
    for i in range(3):
        segs = W.random_tree_segments(g, nseg=6, max_len=70, groups=1)
        T = sum(s[0] for s in segs)
        got, ref = _run(segs, [0, T], T, 2, 1, 128, seed=200 + i)
        _check(got, ref, f"tree {i}")


def test_backward_full_size_grpo():
    """The GRPO group (P=2048, N=8, S=512, 16 heads, d=128): dq on sampled
    rows against the oracle, and two identities that hold at any size and
    involve every key: sum_k dV[k] = sum over the group's query heads and
    rows of dO (each row's P sums to one), and sum_k dK[k] = 0 (each row's
    dS sums to zero)."""
    wl = W.GRPO
    q, k, v = (t.cuda() for t in wl.make("cpu"))
    gen = torch.Generator().manual_seed(300)
    dout = (torch.randn((wl.T, wl.Hq, wl.d), generator=gen) * 0.5).to(torch.bfloat16)
    dog = dout.cuda()
    sched = psa.plan_prefill(wl.segments(), wl.cu_seqlens(), wl.d, "cuda")
    o, lse = psa.prefill(q, k, v, sched, wl.scale)
    dq, dk, dv = psa.prefill_bwd(q, k, v, o, lse, dog,
                                 psa.plan_prefill_bwd(wl.segments(), wl.cu_seqlens(), wl.d),
                                 wl.scale)
    torch.cuda.synchronize()
    rows = np.array([0, 1, 127, 128, 2047, 2048, 2100, 2559, 2560, 4000, wl.T - 1],
                    dtype=np.int32)
    rq = oracle.prefill_bwd_dq(q.cpu(), k.cpu(), v.cpu(), dout, wl.segments(), wl.scale, rows)
    fro, mx = _grad_errors(dq[torch.as_tensor(rows).long().cuda()], rq)
    assert fro <= REL_FRO and mx <= MAX_ABS_REL, f"dq rows: fro={fro:.3e} max={mx:.3e}"
    G = wl.Hq // wl.Hkv
    sv = dv.double().sum(0)                                   # [Hkv, d]
    want = dog.double().sum(0).view(wl.Hkv, G, wl.d).sum(1)   # [Hkv, d]
    assert (sv - want).norm() <= REL_FRO * want.norm()
    sk = dk.double().sum(0)
    assert sk.norm() <= 0.05 * dk.double().norm()


def test_backward_full_size_grpo_heads_elementwise():
    """The GRPO group at full size (T = 6144, 16 heads, d = 128), through the
    same call as above, with every element of dq, dk and dv of two whole
    heads checked against the oracle.  With 16 query heads over 16 KV heads
    a head's gradients depend on that head's Q, K, V and dO only, so the
    oracle runs on the head slice; every prefix key block's unit streams
    all 2048 + 8 * 512 query rows that see it."""
    wl = W.GRPO
    q, k, v = wl.make("cpu")
    gen = torch.Generator().manual_seed(301)
    dout = (torch.randn((wl.T, wl.Hq, wl.d), generator=gen) * 0.5).to(torch.bfloat16)
    qg, kg, vg, dog = (t.cuda() for t in (q, k, v, dout))
    sched = psa.plan_prefill(wl.segments(), wl.cu_seqlens(), wl.d, "cuda")
    o, lse = psa.prefill(qg, kg, vg, sched, wl.scale)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    dq, dk, dv = psa.prefill_bwd(qg, kg, vg, o, lse, dog,
                                 psa.plan_prefill_bwd(wl.segments(), wl.cu_seqlens(), wl.d),
                                 wl.scale, status=status)
    torch.cuda.synchronize()
    assert psa.read_status(status) == 0
    assert wl.Hq == wl.Hkv
    for h in (0, wl.Hq - 1):
        sl = lambda t: t[:, h:h + 1].contiguous()  # noqa: E731
        rq, rk, rv = oracle.prefill_bwd(sl(q), sl(k), sl(v), sl(dout), wl.segments(), wl.scale)
        _check((dq[:, h:h + 1], dk[:, h:h + 1], dv[:, h:h + 1]), (rq, rk, rv),
               f"GRPO head {h}")


def test_backward_outputs_only_16_byte_aligned():
    """dq / dk / dv that start 16 bytes past a 32-byte boundary (allowed: the
    entry asks for 16-byte alignment) take the epilogue's 16-byte stores; the
    gradients are the same bytes as with aligned outputs."""
    segs, cu = psa.spec_flat(100, 3, 37), [0, 100 + 3 * 37]
    T, Hq, Hkv, d = cu[1], 4, 2, 64
    gen = torch.Generator().manual_seed(101)
    draw = lambda shape: (torch.randn(shape, generator=gen) * 0.5).to(torch.bfloat16).cuda()
    q, k, v, dout = draw((T, Hq, d)), draw((T, Hkv, d)), draw((T, Hkv, d)), draw((T, Hq, d))
    scale = 1.0 / np.sqrt(d)
    o, lse = psa.prefill(q, k, v, psa.plan_prefill(segs, cu, d, "cuda"), scale)
    sch = psa.plan_prefill_bwd(segs, cu, d)

    def offset_like(t):
        buf = torch.zeros(t.numel() + 16, dtype=t.dtype, device="cuda")
        assert buf.data_ptr() % 32 == 0
        return buf[8:8 + t.numel()].view(t.shape)  # 16 bytes past the boundary

    got = psa.prefill_bwd(q, k, v, o, lse, dout, sch, scale, dq=offset_like(q),
                          dk=offset_like(k), dv=offset_like(v))
    ref = psa.prefill_bwd(q, k, v, o, lse, dout, sch, scale)
    torch.cuda.synchronize()
    for g, r in zip(got, ref):
        assert r.data_ptr() % 32 == 0 and g.data_ptr() % 32 == 16
        assert torch.equal(g, r)
