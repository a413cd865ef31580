"""Prefill over the flat packed layout on the GPU against the fp64 oracle.

"KV-0 redundancy prefix sharing attention mask design" (PrefixSharing PR
#50): design summary (dedup flat layout, rectangle spec, one forward) and
key changes section 2 (flat GRPO and tree / chain masks).  Every call goes
through the C ABI; the oracle reads the same input bytes."""
import numpy as np
import pytest
import torch

import oracle
import shared_prefix_attention_b200 as psa
from shared_prefix_attention_b200 import workloads as W
from parity import assert_parity

pytestmark = pytest.mark.gpu


def _run(segs, cu, q, k, v, scale, rows=None):
    dev = "cuda"
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    sched = psa.plan_prefill(segs, cu, q.shape[2], dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    o, lse = psa.prefill(qd, kd, vd, sched, scale, status=status)
    torch.cuda.synchronize()
    assert psa.read_status(status) == 0
    ro, rl = oracle.prefill(q, k, v, segs, scale, rows=rows)
    if rows is not None:
        idx = torch.as_tensor(rows, device=dev).long()
        o, lse = o[idx], lse[idx]
    return o, lse, ro, rl


def _inputs(T, Hq, Hkv, d, seed, dtype=torch.bfloat16, sigma=0.5):
    g = torch.Generator().manual_seed(seed)
    mk = lambda h: (torch.randn((T, h, d), generator=g) * sigma).to(dtype)
    return mk(Hq), mk(Hkv), mk(Hkv)


def test_prefill_tiny_fp32_workload():
    """The tiny fp32 workload (P=64, N=4, S=32, 2 heads, d=64), every row."""
    wl = W.TINY
    q, k, v = wl.make("cpu")
    o, lse, ro, rl = _run(wl.segments(), wl.cu_seqlens(), q, k, v, wl.scale)
    assert o.dtype == torch.float32
    assert_parity(o, lse, ro, rl, "tiny fp32")


def test_prefill_tiny_bf16_d64():
    wl = W.TINY
    q, k, v = _inputs(wl.T, 2, 2, 64, 5)
    o, lse, ro, rl = _run(wl.segments(), wl.cu_seqlens(), q, k, v, wl.scale)
    assert_parity(o, lse, ro, rl, "tiny bf16")


@pytest.mark.parametrize("P,N,S,groups,Hq,Hkv,d", [
    (100, 3, 37, 1, 4, 1, 128),     # ragged tails, MQA
    (256, 4, 128, 1, 8, 2, 128),    # tile-aligned, GQA 4:1
    (300, 5, 200, 2, 4, 4, 128),    # two groups, tiles straddle segments
    (0, 4, 150, 1, 2, 2, 128),      # no prefix: varlen causal
    (500, 1, 300, 1, 2, 1, 64),     # N = 1: plain causal
    (129, 9, 1, 1, 2, 2, 64),       # one-token suffixes
    (1, 3, 130, 1, 2, 2, 128),      # one-token prefix
])
def test_prefill_parity_shapes(P, N, S, groups, Hq, Hkv, d):
    wl = W.PrefillWorkload("t", P=P, N=N, S=S, Hq=Hq, Hkv=Hkv, d=d, groups=groups)
    q, k, v = _inputs(wl.T, Hq, Hkv, d, P + N + S)
    o, lse, ro, rl = _run(wl.segments(), wl.cu_seqlens(), q, k, v, wl.scale)
    assert_parity(o, lse, ro, rl, f"P={P} N={N} S={S}")


def test_prefill_random_trees_and_chain():
    g = torch.Generator().manual_seed(3)
    for i in range(3):
        segs = W.random_tree_segments(g, nseg=6, max_len=150, groups=1)
        T = sum(s[0] for s in segs)
        q, k, v = _inputs(T, 4, 2, 128, 50 + i)
        o, lse, ro, rl = _run(segs, [0, T], q, k, v, 128 ** -0.5)
        assert_parity(o, lse, ro, rl, f"tree {i}")
    segs = W.chain_segments([90, 200, 17, 300])
    T = sum(s[0] for s in segs)
    q, k, v = _inputs(T, 2, 2, 64, 60)
    o, lse, ro, rl = _run(segs, [0, T], q, k, v, 64 ** -0.5)
    assert_parity(o, lse, ro, rl, "chain")


def _sample_rows(wl, extra=64, seed=0):
    """Segment and tile boundaries plus random rows."""
    rows = set()
    start = 0
    for n, _ in wl.segments():
        for r in (start, start + 1, start + n - 2, start + n - 1):
            if 0 <= r < wl.T:
                rows.add(r)
        start += n
    for t in range(0, wl.T, 128):
        rows.update((t, min(wl.T - 1, t + 127)))
    rng = np.random.default_rng(seed)
    rows.update(int(x) for x in rng.integers(0, wl.T, extra))
    return sorted(rows)


@pytest.mark.parametrize("wl", [W.GRPO, W.LARGE], ids=["grpo", "large"])
def test_prefill_full_size_sampled_rows(wl):
    """Full-size workloads on device-generated inputs (as the benchmark
    times them), checked on boundary and random rows."""
    dev = "cuda"
    q, k, v = wl.make(dev)
    sched = psa.plan_prefill(wl.segments(), wl.cu_seqlens(), wl.d, dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    o, lse = psa.prefill(q, k, v, sched, wl.scale, status=status)
    torch.cuda.synchronize()
    assert psa.read_status(status) == 0
    rows = _sample_rows(wl, extra=32 if wl is W.LARGE else 64)
    if wl is W.LARGE:
        rows = rows[::3]
    ro, rl = oracle.prefill(q.cpu(), k.cpu(), v.cpu(), wl.segments(), wl.scale, rows=rows)
    idx = torch.tensor(rows, device=dev)
    assert_parity(o[idx], lse[idx], ro, rl, wl.name)
    assert torch.isfinite(o.float()).all() and torch.isfinite(lse).all()


def test_prefill_repeatable_and_independent_of_output_contents():
    wl = W.PrefillWorkload("t", P=333, N=3, S=111, Hq=4, Hkv=2, d=128)
    q, k, v = (t.cuda() for t in _inputs(wl.T, 4, 2, 128, 9))
    sched = psa.plan_prefill(wl.segments(), wl.cu_seqlens(), 128)
    o1 = torch.full_like(q, float("nan"))
    o1, l1 = psa.prefill(q, k, v, sched, wl.scale, out=o1)
    o2, l2 = psa.prefill(q, k, v, sched, wl.scale)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_prefill_output_only_16_byte_aligned():
    """An output that starts 16 bytes past a 32-byte boundary (allowed: the
    entry asks for 16-byte alignment) takes the epilogue's 16-byte stores;
    the result is the same bytes as an aligned output's, and matches the
    oracle."""
    wl = W.PrefillWorkload("t", P=300, N=3, S=170, Hq=8, Hkv=2, d=128)
    q, k, v = _inputs(wl.T, 8, 2, 128, 13)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    sched = psa.plan_prefill(wl.segments(), wl.cu_seqlens(), 128)
    buf = torch.zeros(qd.numel() + 16, dtype=qd.dtype, device="cuda")
    assert buf.data_ptr() % 32 == 0
    o_off = buf[8:8 + qd.numel()].view(qd.shape)  # 16 bytes past the boundary
    o_off, l_off = psa.prefill(qd, kd, vd, sched, wl.scale, out=o_off)
    o_al, l_al = psa.prefill(qd, kd, vd, sched, wl.scale)
    torch.cuda.synchronize()
    assert o_al.data_ptr() % 32 == 0
    assert torch.equal(o_off, o_al) and torch.equal(l_off, l_al)
    ro, rl = oracle.prefill(q, k, v, wl.segments(), wl.scale)
    assert_parity(o_off, l_off, ro, rl, "16-byte-aligned output")
