"""The seeded input generators hold no arithmetic of the method, but the
structure they promise (the pages' workload shapes, valid draft trees, a
page table of distinct pool rows) is what the parity tests rely on."""
import numpy as np
import torch

from shared_prefix_attention_b200 import workloads as W


def _blocks(wl, mask):
    mi = wl.mask_indptr()
    return [mask[mi[b]:mi[b + 1]].reshape(n, n).numpy() for b, n in enumerate(wl.draft_lens)]


def test_extend_workload_indptrs_and_shapes():
    wl = W.ExtendVerifyWorkload("t", draft_lens=[3, 0, 5, 1], prefix_lens=[29, 11, 0, 40], Hq=4,
                                Hkv=2, d=16, seed=3)
    q, kd, vd, kp, vp, idx, mask = wl.make()
    assert wl.qo_indptr() == [0, 3, 3, 8, 9] and wl.kv_indptr() == [0, 29, 40, 40, 80]
    assert wl.mask_indptr() == [0, 9, 9, 34, 35]
    assert q.shape == (9, 4, 16) and kd.shape == vd.shape == (9, 2, 16)
    assert kp.shape[0] == vp.shape[0] == wl.pool_rows() == 100
    assert idx.dtype == torch.int32 and idx.shape == (80,)
    assert mask.dtype == torch.uint8 and mask.shape == (35,)


def test_extend_page_table_is_distinct_pool_rows():
    wl = W.ExtendVerifyWorkload("t", draft_lens=[2] * 6, prefix_lens=[300, 1, 77, 0, 512, 64],
                                Hq=2, Hkv=1, d=8, seed=5)
    _, _, _, kp, _, idx, _ = wl.make()
    rows = idx.numpy()
    assert len(np.unique(rows)) == len(rows)
    assert rows.min() >= 0 and rows.max() < kp.shape[0]


def test_extend_trees_are_ancestor_closed():
    """Each draft sees itself; whatever it sees is an earlier draft; the set
    it sees is its parent's set plus itself (parent = its latest ancestor)."""
    wl = W.ExtendVerifyWorkload("t", draft_lens=[1, 4, 8, 16], prefix_lens=[5] * 4, Hq=2, Hkv=1,
                                d=8, seed=9)
    *_, mask = wl.make()
    for m in _blocks(wl, mask):
        n = m.shape[0]
        for j in range(n):
            assert m[j, j] == 1
            assert not m[j, j + 1:].any()
            anc = np.flatnonzero(m[j, :j])
            if len(anc):
                par = anc.max()
                expect = m[par].copy()
                expect[j] = 1
                assert np.array_equal(m[j], expect)


def test_extend_generator_is_seeded():
    wl = W.ExtendVerifyWorkload("t", draft_lens=[3, 2], prefix_lens=[20, 30], Hq=2, Hkv=1, d=8,
                                seed=4)
    a, b = wl.make(), wl.make()
    for x, y in zip(a, b):
        assert torch.equal(x, y)
    c = wl.make(seed=5)
    assert not torch.equal(a[0], c[0])


def test_benchmark_extend_workload_shape():
    """The timed extend workload: 32 requests, 16384-token prefixes, 1..8
    drafts each (every count present), trees on, the verify shapes."""
    wl = W.VERIFY_PAGED
    assert wl.B == 32 and set(wl.prefix_lens) == {16384}
    assert sorted(set(wl.draft_lens)) == list(range(1, 9)) and wl.max_draft_len == 8
    assert (wl.Hq, wl.Hkv, wl.d, wl.nsplit, wl.tree) == (32, 8, 128, 32, True)
    assert wl.prefix_kv_bytes() == 32 * 16384 * 8 * 128 * 2 * 2
