"""Tree verify on the GPU against the fp64 oracle ("Split-KV flash-decode
attention for EAGLE target-verify", key code can_handle: EAGLE trees with
topk > 1 bring a custom draft mask; the prefix stays fully visible).  The
split-KV prefix stage is unchanged; the combine stage takes the mask."""
import numpy as np
import pytest
import torch

import oracle
import shared_prefix_attention_b200 as psa
from shared_prefix_attention_b200 import workloads as W
from parity import assert_parity

pytestmark = pytest.mark.gpu


def _tree_mask(B, Ld, seed):
    """Per request a random draft tree in topological order: draft j's parent
    is an earlier draft (or the prefix); j sees its ancestors and itself."""
    rng = np.random.default_rng(seed)
    m = np.zeros((B * Ld, Ld), dtype=np.uint8)
    for b in range(B):
        parent = [-1] + [int(rng.integers(-1, j)) for j in range(1, Ld)]
        for j in range(Ld):
            a = j
            while a >= 0:
                m[b * Ld + j, a] = 1
                a = parent[a]
    return m


def _run(wl, mask):
    q, kd, vd, kc, vc = (t.cuda() for t in wl.make("cpu"))
    indptr = torch.tensor(wl.kv_indptr(), dtype=torch.int32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    o, lse = psa.verify_tree(q, kd, vd, kc, vc, indptr, max(wl.lens() + [0]),
                             torch.from_numpy(mask).cuda(), wl.scale, wl.Ld, nsplit=wl.nsplit,
                             status=status)
    torch.cuda.synchronize()
    assert psa.read_status(status) == 0
    ro, rl = oracle.verify_tree(q.cpu(), kd.cpu(), vd.cpu(), kc.cpu(), vc.cpu(),
                                np.array(wl.kv_indptr(), dtype=np.int64), mask, wl.Ld, wl.scale)
    return o, lse, ro, rl


@pytest.mark.parametrize("lens,Ld,nsplit,seed", [
    ([300, 300, 300], 4, 4, 1),
    ([37, 513, 1000], 8, 8, 2),      # deeper trees, ragged prefixes
    ([2048, 17], 16, 32, 3),         # the largest draft block
])
def test_verify_tree_parity(lens, Ld, nsplit, seed):
    wl = W.VerifyWorkload("t", B=len(lens), L=max(lens), Ld=Ld, Hq=32, Hkv=8, d=128,
                          nsplit=nsplit, seed=80 + seed, prefix_lens=lens)
    o, lse, ro, rl = _run(wl, _tree_mask(len(lens), Ld, seed))
    assert_parity(o, lse, ro, rl, f"lens={lens} Ld={Ld}")


def test_verify_tree_row_without_drafts():
    """A draft row whose mask row is empty still sees the whole prefix."""
    wl = W.VerifyWorkload("t", B=2, L=200, Ld=4, Hq=8, Hkv=2, d=128, nsplit=3, seed=90)
    m = _tree_mask(2, 4, 7)
    m[1] = 0
    o, lse, ro, rl = _run(wl, m)
    assert_parity(o, lse, ro, rl, "empty mask row")


def test_verify_tree_causal_mask_equals_chain_verify():
    wl = W.VerifyWorkload("t", B=3, L=700, Ld=4, Hq=32, Hkv=8, d=128, nsplit=5, seed=91)
    q, kd, vd, kc, vc = (t.cuda() for t in wl.make("cpu"))
    indptr = torch.tensor(wl.kv_indptr(), dtype=torch.int32, device="cuda")
    causal = torch.from_numpy(np.tile(np.tril(np.ones((4, 4), np.uint8)), (3, 1))).cuda()
    o1, l1 = psa.verify_tree(q, kd, vd, kc, vc, indptr, wl.L, causal, wl.scale, wl.Ld,
                             nsplit=wl.nsplit)
    o2, l2 = psa.verify(q, kd, vd, kc, vc, indptr, wl.L, wl.scale, wl.Ld, nsplit=wl.nsplit)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
