"""Verify in the extend form on the GPU against the fp64 oracle ("Split-KV
flash-decode attention for EAGLE target-verify": the verify entry's
qo_indptr / kv_indptr / kv_indices / custom_mask / mask_indptr arguments,
and can_handle's refusals of ragged extend and custom masks): a prefix read
through a token-granular page table, ragged draft counts, per-request trees."""
import numpy as np
import pytest
import torch

import oracle
import shared_prefix_attention_b200 as psa
from shared_prefix_attention_b200 import workloads as W
from parity import assert_parity

pytestmark = pytest.mark.gpu


def _dev(xs):
    return torch.tensor(xs, dtype=torch.int32, device="cuda")


def _run_extend(wl, rows=None):
    q, kd, vd, kp, vp, idx, mask = wl.make("cpu")
    g = [t.cuda() for t in (q, kd, vd, kp, vp, idx)]
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    o, lse = psa.verify_extend(g[0], g[1], g[2], g[3], g[4], _dev(wl.qo_indptr()),
                               wl.max_draft_len, _dev(wl.kv_indptr()), wl.max_prefix_len,
                               wl.scale, kv_indices=g[5],
                               draft_mask=None if mask is None else mask.cuda(),
                               mask_indptr=None if mask is None else _dev(wl.mask_indptr()),
                               nsplit=wl.nsplit, status=status)
    torch.cuda.synchronize()
    assert psa.read_status(status) == 0
    ro, rl = oracle.verify_extend(q, kd, vd, kp, vp, wl.qo_indptr(), wl.kv_indptr(), wl.scale,
                                  kv_indices=idx, draft_mask=mask,
                                  mask_indptr=None if mask is None else wl.mask_indptr(),
                                  rows=rows)
    if rows is not None:
        o, lse = o[torch.as_tensor(rows).long().cuda()], lse[torch.as_tensor(rows).long().cuda()]
    return o, lse, ro, rl


@pytest.mark.parametrize("drafts,prefixes,Hq,Hkv,d,nsplit,tree", [
    ([3, 0, 5, 1], [300, 77, 0, 1000], 32, 8, 128, 4, True),     # ragged both ways, an empty one
    ([8, 8, 2], [2048, 15, 513], 32, 8, 128, 16, False),         # ragged drafts, causal blocks
    ([16, 1, 7], [700, 700, 64], 8, 8, 128, 3, True),            # MHA, the largest block
    ([4, 2], [333, 1500], 16, 2, 64, 5, True),                   # head_dim 64
    ([4, 3], [640, 129], 8, 2, 256, 2, True),                    # head_dim 256
])
def test_verify_extend_parity(drafts, prefixes, Hq, Hkv, d, nsplit, tree):
    wl = W.ExtendVerifyWorkload("t", draft_lens=drafts, prefix_lens=prefixes, Hq=Hq, Hkv=Hkv,
                                d=d, nsplit=nsplit, tree=tree, seed=sum(drafts) + d)
    o, lse, ro, rl = _run_extend(wl)
    assert_parity(o, lse, ro, rl, f"drafts={drafts} prefixes={prefixes} d={d}")


def test_verify_extend_full_size_sampled_rows():
    """The benchmark's extend workload (B = 32, 16384-token prefixes through a
    page table, 1..8 drafts per request in trees), rows sampled across it."""
    wl = W.VERIFY_PAGED
    qo = wl.qo_indptr()
    rows = sorted({0, 1, qo[5], qo[5] + 1, qo[17] - 1, qo[31], wl.n_rows - 1, 77, 100})
    o, lse, ro, rl = _run_extend(wl, rows=np.array(rows, dtype=np.int32))
    assert_parity(o, lse, ro, rl, "extend full size")


def test_paged_verify_equals_contiguous():
    """The page table only moves where the rows are read from: scattering the
    prefix over a pool and reading it back through the table gives the
    contiguous verify's bytes exactly (same tiles, same arithmetic)."""
    wl = W.VerifyWorkload("t", B=3, L=900, Ld=4, Hq=32, Hkv=8, d=128, nsplit=7, seed=95,
                          prefix_lens=[900, 31, 400])
    q, kd, vd, kc, vc = (t.cuda() for t in wl.make("cpu"))
    ntok = kc.shape[0]
    gen = torch.Generator().manual_seed(5)
    idx = torch.randperm(2 * ntok, generator=gen)[:ntok].to(torch.int32).cuda()
    kp = torch.zeros((2 * ntok,) + tuple(kc.shape[1:]), dtype=kc.dtype, device="cuda")
    vp = torch.zeros_like(kp)
    kp[idx.long()] = kc
    vp[idx.long()] = vc
    indptr = torch.tensor(wl.kv_indptr(), dtype=torch.int32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    o1, l1 = psa.verify(q, kd, vd, kc, vc, indptr, wl.L, wl.scale, wl.Ld, nsplit=wl.nsplit)
    o2, l2 = psa.verify(q, kd, vd, kp, vp, indptr, wl.L, wl.scale, wl.Ld, nsplit=wl.nsplit,
                        kv_indices=idx, status=status)
    torch.cuda.synchronize()
    assert psa.read_status(status) == 0
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    # tree verify through the same table
    mask = torch.from_numpy(np.tile(np.array([[1, 0, 0, 0], [1, 1, 0, 0], [1, 0, 1, 0],
                                              [1, 1, 0, 1]], np.uint8), (3, 1))).cuda()
    o3, l3 = psa.verify_tree(q, kd, vd, kp, vp, indptr, wl.L, mask, wl.scale, wl.Ld,
                             nsplit=wl.nsplit, kv_indices=idx)
    torch.cuda.synchronize()
    ro, rl = oracle.verify_tree(q.cpu(), kd.cpu(), vd.cpu(), kc.cpu(), vc.cpu(),
                                np.array(wl.kv_indptr(), dtype=np.int64), mask.cpu().numpy(),
                                wl.Ld, wl.scale)
    assert_parity(o3, l3, ro, rl, "paged tree verify")


def test_paged_row_outside_the_cache_is_reported():
    """A page-table entry outside the cache is caught by the gather's bounds
    check: the row reads as zeros and PSA_ERR_INVALID_ARG lands in the status."""
    wl = W.VerifyWorkload("t", B=2, L=64, Ld=2, Hq=8, Hkv=2, d=128, nsplit=2, seed=96)
    q, kd, vd, kc, vc = (t.cuda() for t in wl.make("cpu"))
    idx = torch.arange(128, dtype=torch.int32, device="cuda")
    idx[70] = 128                          # one past the last cache row
    indptr = torch.tensor(wl.kv_indptr(), dtype=torch.int32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    o, _ = psa.verify(q, kd, vd, kc, vc, indptr, wl.L, wl.scale, wl.Ld, nsplit=wl.nsplit,
                      kv_indices=idx, status=status)
    torch.cuda.synchronize()
    assert psa.read_status(status) == psa.PSA_ERR_INVALID_ARG
    assert bool(torch.isfinite(o.float()).all())


def test_verify_extend_row_that_sees_nothing():
    """The degenerate case: a request with an empty prefix whose mask row is
    empty sees no key at all, so O = 0 and LSE = -inf (both sides); every
    other row matches the oracle."""
    wl = W.ExtendVerifyWorkload("t", draft_lens=[3, 4], prefix_lens=[0, 200], Hq=8, Hkv=2,
                                d=128, nsplit=3, tree=True, seed=97)
    q, kd, vd, kp, vp, idx, mask = wl.make("cpu")
    mask = mask.clone()
    mask[1 * 3:2 * 3] = 0            # request 0, draft 1: sees nothing
    g = [t.cuda() for t in (q, kd, vd, kp, vp, idx)]
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    o, lse = psa.verify_extend(g[0], g[1], g[2], g[3], g[4], _dev(wl.qo_indptr()),
                               wl.max_draft_len, _dev(wl.kv_indptr()), wl.max_prefix_len,
                               wl.scale, kv_indices=g[5], draft_mask=mask.cuda(),
                               mask_indptr=_dev(wl.mask_indptr()), nsplit=wl.nsplit,
                               status=status)
    torch.cuda.synchronize()
    assert psa.read_status(status) == 0
    ro, rl = oracle.verify_extend(q, kd, vd, kp, vp, wl.qo_indptr(), wl.kv_indptr(), wl.scale,
                                  kv_indices=idx, draft_mask=mask,
                                  mask_indptr=wl.mask_indptr())
    assert np.all(np.isneginf(rl[1])) and not np.any(ro[1])
    assert bool(torch.all(o[1] == 0)) and bool(torch.all(torch.isneginf(lse[1])))
    keep = [r for r in range(wl.n_rows) if r != 1]
    assert_parity(o[keep], lse[keep], ro[keep], rl[keep], "rows that see keys")


@pytest.mark.parametrize("drafts,prefixes,Hq,Hkv,nsplit,tree", [
    ([3, 0, 5, 1], [300, 77, 0, 1000], 32, 8, 4, True),   # ragged, paged, trees, an empty one
    ([8, 8, 2], [2048, 15, 513], 16, 2, 16, False),      # ragged drafts, causal blocks
])
def test_verify_extend_e4m3(drafts, prefixes, Hq, Hkv, nsplit, tree):
    """The extend form over an e4m3 cache ([SKV]: the verify entry takes
    k_scale / v_scale with the page table and the masks).  Reference: the
    oracle's extend form on the decoded, scaled cache (the fp8 verify equals
    the float verify on that cache, a pinned identity)."""
    wl = W.ExtendVerifyWorkload("t", draft_lens=drafts, prefix_lens=prefixes, Hq=Hq, Hkv=Hkv,
                                d=128, nsplit=nsplit, tree=tree, seed=sum(drafts) + 31)
    q, kd, vd, kp, vp, idx, mask = wl.make("cpu")
    ks, vs = 1.0 / 96, 1.0 / 80
    kp8 = (kp.float() / ks).to(torch.float8_e4m3fn).view(torch.uint8)
    vp8 = (vp.float() / vs).to(torch.float8_e4m3fn).view(torch.uint8)
    g = [t.cuda() for t in (q, kd, vd, kp8, vp8, idx)]
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    o, lse = psa.verify_extend(g[0], g[1], g[2], g[3], g[4], _dev(wl.qo_indptr()),
                               wl.max_draft_len, _dev(wl.kv_indptr()), wl.max_prefix_len,
                               wl.scale, kv_indices=g[5],
                               draft_mask=None if mask is None else mask.cuda(),
                               mask_indptr=None if mask is None else _dev(wl.mask_indptr()),
                               nsplit=nsplit, status=status, k_scale=ks, v_scale=vs)
    torch.cuda.synchronize()
    assert psa.read_status(status) == 0
    kdec = torch.from_numpy(oracle.decode_e4m3(kp8) * ks)
    vdec = torch.from_numpy(oracle.decode_e4m3(vp8) * vs)
    ro, rl = oracle.verify_extend(q, kd, vd, kdec, vdec, wl.qo_indptr(), wl.kv_indptr(),
                                  wl.scale, kv_indices=idx, draft_mask=mask,
                                  mask_indptr=None if mask is None else wl.mask_indptr())
    assert_parity(o, lse, ro, rl, f"e4m3 drafts={drafts} prefixes={prefixes}")
