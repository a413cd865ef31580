"""Host mask builder: the rectangle spec is bit-exact against the oracle's
brute-force visibility matrix, and the tile schedule lists exactly the tiles
with a visible pair, flags full tiles correctly and reproduces the mask of
every partial tile.  ("KV-0 redundancy prefix sharing attention mask
design": design summary -- rectangle spec, no dense mask; key changes
section 2 -- flat GRPO and multi-level tree / chain construction.)"""
import itertools

import numpy as np
import pytest
import torch

import oracle
import shared_prefix_attention_b200 as psa
from shared_prefix_attention_b200 import workloads as W


def _expand(rects, T, row0=0, nrows=None):
    nrows = T - row0 if nrows is None else nrows
    m = np.zeros((nrows, T), dtype=np.uint8)
    for q0, q1, k0, k1, causal in rects:
        a, b = max(q0, row0), min(q1, row0 + nrows)
        if a >= b:
            continue
        for q in range(a, b):
            lo, hi = k0, k1
            if causal == 1:      # k - k0 <= q - q0
                hi = min(k1, k0 + (q - q0) + 1)
            elif causal == 2:    # transposed: k - k0 >= q - q0
                lo = max(k0, k0 + (q - q0))
            if hi > lo:
                assert not m[q - row0, lo:hi].any(), "rectangles overlap"
                m[q - row0, lo:hi] = 1
    return m


def _check_spec(segs):
    rects = psa.build_spec(segs)
    T = sum(s[0] for s in segs)
    assert np.array_equal(_expand(rects, T), oracle.visibility(segs))
    return rects


def test_spec_flat_matches_helper():
    assert psa.spec_flat(64, 4, 32) == W.grpo_segments(64, 4, 32)
    assert psa.spec_flat(0, 3, 5) == W.grpo_segments(0, 3, 5)


def test_spec_bit_exact_all_small_grpo():
    """Every flat GRPO layout with P <= 8, 1 <= N <= 8, 1 <= S <= 8."""
    for P, N, S in itertools.product(range(0, 9), range(1, 9), range(1, 9)):
        _check_spec(W.grpo_segments(P, N, S))


def test_spec_bit_exact_random_trees_and_chains():
    g = torch.Generator().manual_seed(7)
    for _ in range(40):
        _check_spec(W.random_tree_segments(g, nseg=7, max_len=9, groups=3))
    _check_spec(W.chain_segments([3, 1, 4, 1, 5, 9, 2, 6]))


def test_spec_rect_counts_of_the_workloads():
    assert len(psa.build_spec(W.TINY.segments())) == 9
    assert len(psa.build_spec(W.GRPO.segments())) == 17
    assert len(psa.build_spec(W.LARGE.segments())) == 66


@pytest.mark.parametrize("wl", [W.TINY, W.GRPO], ids=["tiny", "grpo"])
def test_spec_bit_exact_workloads(wl):
    _check_spec(wl.segments())


def test_spec_bit_exact_large_blockwise():
    """The two-group 49152-token layout, checked in row blocks."""
    segs = W.LARGE.segments()
    rects = psa.build_spec(segs)
    T = W.LARGE.T
    rng = np.random.default_rng(0)
    for row0 in list(range(0, T, 8192)) + [int(x) for x in rng.integers(0, T - 512, 4)]:
        n = 512
        assert np.array_equal(_expand(rects, T, row0, n), oracle.visibility(segs, row0, n))


def test_spec_rejects_bad_trees():
    with pytest.raises(psa.PsaError):
        psa.build_spec([(4, -1), (3, 1)])   # parent does not precede
    with pytest.raises(psa.PsaError):
        psa.build_spec([(0, -1)])           # empty segment


def _decode(sched):
    assert sched[0] == 0x50534132
    ni, nk, nr, tm, tn, T, maxkv = (int(x) for x in sched[1:8])
    items = sched[8:8 + 4 * ni].reshape(ni, 4)
    kvs = sched[8 + 4 * ni:8 + 4 * ni + 8 * nk].reshape(nk, 8)
    rects = sched[8 + 4 * ni + 8 * nk:8 + 4 * ni + 8 * nk + 5 * nr].reshape(nr, 5)
    assert len(sched) == 8 + 4 * ni + 8 * nk + 5 * nr
    return items, kvs, rects, tm, tn, T, maxkv


def _check_schedule(segs, cu, tm, tn, transpose=False):
    """Every Q block (two halves of tm/2 rows) lists exactly the KV tiles in
    which some half has a visible pair; per half the active / full flags
    and the copied rectangles reproduce the visibility of the box.  With
    transpose, the spec is transposed first and the rows are keys: the
    schedule must then reproduce the transposed visibility."""
    rects = psa.build_spec(segs)
    if transpose:
        rects = psa.transpose_spec(rects)
    sched = psa.build_schedule(rects, cu, tm, tn)
    items, kvs, trects, tm2, tn2, T, maxkv = _decode(sched)
    assert (tm2, tn2, T) == (tm, tn, cu[-1])
    vis = oracle.visibility(segs).astype(bool)
    if transpose:
        vis = vis.T.copy()
    counts = [int(it[3]) for it in items]
    assert counts == sorted(counts, reverse=True)          # longest first
    assert maxkv == max(counts)
    half = tm // 2
    covered = np.zeros_like(vis)
    seen_q = []
    for q0, ql, kb, kc in items:
        seen_q.append((int(q0), int(ql)))
        g = max(i for i in range(len(cu) - 1) if cu[i] <= q0)
        listed = {int(e[0]): e for e in kvs[kb:kb + kc]}
        assert len(listed) == kc
        for ka in range(cu[g], cu[g + 1], tn):
            kl = min(cu[g + 1], ka + tn) - ka
            boxes = []
            for h in range(2):
                a, b = q0 + h * half, min(q0 + ql, q0 + (h + 1) * half)
                boxes.append(vis[a:b, ka:ka + kl] if a < b else np.zeros((0, kl), bool))
            if not any(bx.any() for bx in boxes):
                assert ka not in listed
                continue
            e = listed[ka]
            assert int(e[1]) == kl
            flags = int(e[6])
            for h in range(2):
                bx = boxes[h]
                active = bool(bx.any())
                assert bool(flags & (1 << h)) == active
                if not active:
                    continue
                full = bool(bx.all())
                assert bool(flags & (4 << h)) == full
                if not full:
                    rb, rc = int(e[2 + 2 * h]), int(e[3 + 2 * h])
                    assert rc > 0
                    a = q0 + h * half
                    sub = _expand(trects[rb:rb + rc], T)[a:a + bx.shape[0], ka:ka + kl]
                    assert np.array_equal(sub.astype(bool), bx)
                covered[q0 + h * half:q0 + h * half + bx.shape[0], ka:ka + kl] = True
    assert sorted(seen_q) == sorted(
        (a, min(cu[i + 1], a + tm) - a) for i in range(len(cu) - 1)
        for a in range(cu[i], cu[i + 1], tm))
    assert not (vis & ~covered).any()


@pytest.mark.parametrize("P,N,S,groups,tm,tn", [
    (64, 4, 32, 1, 256, 128), (2048, 8, 512, 1, 256, 128), (100, 3, 37, 2, 256, 128),
    (5, 7, 3, 1, 8, 4), (0, 4, 50, 1, 32, 16), (300, 2, 1, 3, 128, 64), (700, 3, 300, 1, 256, 128)])
def test_schedule_tiles(P, N, S, groups, tm, tn):
    wl = W.PrefillWorkload("t", P=P, N=N, S=S, Hq=1, Hkv=1, d=64, groups=groups)
    _check_schedule(wl.segments(), wl.cu_seqlens(), tm, tn)


@pytest.mark.parametrize("P,N,S,groups,tm,tn", [
    (64, 4, 32, 1, 128, 64), (100, 3, 37, 2, 128, 64), (5, 7, 3, 1, 8, 4), (0, 4, 50, 1, 32, 16)])
def test_transposed_schedule_tiles(P, N, S, groups, tm, tn):
    """The key-major schedule of the backward's dK / dV pass (keys as rows)."""
    wl = W.PrefillWorkload("t", P=P, N=N, S=S, Hq=1, Hkv=1, d=64, groups=groups)
    _check_schedule(wl.segments(), wl.cu_seqlens(), tm, tn, transpose=True)


def test_transpose_spec_round_trip():
    rects = psa.build_spec(W.grpo_segments(10, 3, 4))
    t = psa.transpose_spec(rects)
    assert set(int(c) for c in t[:, 4]) <= {0, 2}
    assert np.array_equal(psa.transpose_spec(t), rects)


def test_schedule_random_trees():
    g = torch.Generator().manual_seed(11)
    for _ in range(10):
        segs = W.random_tree_segments(g, nseg=6, max_len=40, groups=1)
        T = sum(s[0] for s in segs)
        _check_schedule(segs, [0, T], 32, 32)


def test_schedule_tile_counts_grpo():
    """Visible 128x128 tiles per head: 728 for P=2048/N=8/S=512 (16*17/2 +
    8 * (4*16 + 10)) and 10848 per group of the two-group P=8192 layout,
    counted as (half, KV tile) pairs that take part."""
    for wl, want in ((W.GRPO, 728), (W.LARGE, 2 * 10848)):
        rects = psa.build_spec(wl.segments())
        sched = psa.build_schedule(rects, wl.cu_seqlens(), 256, 128)
        items, kvs, *_ = _decode(sched)
        active = sum(bin(int(f) & 3).count("1") for f in kvs[:, 6])
        assert active == want
