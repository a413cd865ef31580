"""Split-KV verify on the GPU against the fp64 oracle.

"Split-KV flash-decode attention for EAGLE target-verify" (sglang PR
#27382): implementation item 1 (stage-1 split over the cached prefix, stage-2
LSE combine with the causal draft block), test section (head_dim 256 with
4096-token prefixes; GQA ratios 32:1, 16:2, 8:2 on 2048-token prefixes; 4
draft tokens).  Every call goes through the C ABI."""
import math

import numpy as np
import pytest
import torch

import oracle
import shared_prefix_attention_b200 as psa
from shared_prefix_attention_b200 import workloads as W
from parity import assert_parity

pytestmark = pytest.mark.gpu


def _run(wl, nsplit=None, rows=None, seed=None):
    dev = "cuda"
    q, kd, vd, kc, vc = (t.to(dev) for t in wl.make("cpu", seed))
    indptr = torch.tensor(wl.kv_indptr(), dtype=torch.int32, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    ns = wl.nsplit if nsplit is None else nsplit
    o, lse = psa.verify(q, kd, vd, kc, vc, indptr, max(wl.lens() + [0]), wl.scale, wl.Ld,
                        nsplit=ns, status=status)
    torch.cuda.synchronize()
    assert psa.read_status(status) == 0
    ro, rl = oracle.verify(q.cpu(), kd.cpu(), vd.cpu(), kc.cpu(), vc.cpu(),
                           np.array(wl.kv_indptr(), dtype=np.int64), wl.Ld, wl.scale, rows=rows)
    if rows is not None:
        o, lse = o[torch.as_tensor(rows).long().to(dev)], lse[torch.as_tensor(rows).long().to(dev)]
    return o, lse, ro, rl


def _wl(B=3, L=300, Ld=4, Hq=32, Hkv=8, d=128, nsplit=4, lens=None, seed=40):
    return W.VerifyWorkload("t", B=B, L=L, Ld=Ld, Hq=Hq, Hkv=Hkv, d=d, nsplit=nsplit,
                            seed=seed, prefix_lens=lens)


@pytest.mark.parametrize("lens,nsplit", [
    ([300, 300, 300], 4),            # several tiles per split
    ([37, 513, 1000], 8),            # ragged prefixes, tail tiles
    ([0, 5, 16], 3),                 # empty prefix, empty splits
    ([2048, 17, 1], 32),             # many splits, most empty for short prefixes
    ([640], 1),                      # one split
    ([4096, 100], 256),              # maximum split count
])
def test_verify_parity_ragged(lens, nsplit):
    o, lse, ro, rl = _run(_wl(B=len(lens), lens=lens, nsplit=nsplit))
    assert_parity(o, lse, ro, rl, f"lens={lens} nsplit={nsplit}")


@pytest.mark.parametrize("Hq,Hkv,d,L", [
    (16, 2, 256, 4096),   # head_dim 256, 4096-token prefixes
    (32, 1, 128, 2048),   # MQA 32:1 (128 rows per KV head: several row blocks)
    (32, 1, 256, 2048),
    (16, 2, 128, 2048),
    (8, 2, 128, 2048),
    (8, 8, 64, 1000),
])
def test_verify_parity_head_shapes(Hq, Hkv, d, L):
    o, lse, ro, rl = _run(_wl(B=2, L=L, Hq=Hq, Hkv=Hkv, d=d, nsplit=8))
    assert_parity(o, lse, ro, rl, f"Hq={Hq} Hkv={Hkv} d={d}")


@pytest.mark.parametrize("Ld", [1, 2, 7, 16])
def test_verify_parity_draft_counts(Ld):
    o, lse, ro, rl = _run(_wl(B=2, L=777, Ld=Ld, Hq=8, Hkv=2, nsplit=5))
    assert_parity(o, lse, ro, rl, f"Ld={Ld}")


def test_verify_auto_split_count():
    wl = _wl(B=2, L=3000, nsplit=0)
    o, lse, ro, rl = _run(wl, nsplit=0)
    assert_parity(o, lse, ro, rl, "auto splits")


def test_verify_full_size_sampled_rows():
    """The full 32-request, 16384-token, 32-split workload (device-generated
    inputs, as the benchmark times it), checked on sampled draft rows."""
    wl = W.VERIFY
    dev = "cuda"
    q, kd, vd, kc, vc = wl.make(dev)
    indptr = torch.tensor(wl.kv_indptr(), dtype=torch.int32, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    o, lse = psa.verify(q, kd, vd, kc, vc, indptr, wl.L, wl.scale, wl.Ld, nsplit=wl.nsplit,
                        status=status)
    torch.cuda.synchronize()
    assert psa.read_status(status) == 0
    rows = [0, 3, 4 * 7 + 1, 4 * 15 + 2, 4 * 31 + 3, 4 * 31]
    ro, rl = [], []
    for r in rows:
        # the oracle sees only request b's slice of the cache
        b, j = divmod(r, wl.Ld)
        p0, p1 = b * wl.L, (b + 1) * wl.L
        sl = slice(b * wl.Ld, (b + 1) * wl.Ld)
        o1, l1 = oracle.verify(q[sl].cpu(), kd[sl].cpu(), vd[sl].cpu(), kc[p0:p1].cpu(),
                               vc[p0:p1].cpu(), np.array([0, wl.L], dtype=np.int64), wl.Ld,
                               wl.scale, rows=[j])
        ro.append(o1)
        rl.append(l1)
    idx = torch.tensor(rows, device=dev)
    assert_parity(o[idx], lse[idx], np.concatenate(ro), np.concatenate(rl), "full size")
    assert torch.isfinite(o.float()).all()


def test_verify_repeatable():
    """Two calls on the same inputs give identical bytes (no state leaks
    between calls through the workspace)."""
    wl = _wl(B=2, L=900, nsplit=6)
    dev = "cuda"
    q, kd, vd, kc, vc = (t.to(dev) for t in wl.make("cpu"))
    indptr = torch.tensor(wl.kv_indptr(), dtype=torch.int32, device=dev)
    ws = torch.full((psa.verify_workspace_size(2, 4, 32, 128, 6),), 255, dtype=torch.uint8,
                    device=dev)
    o1, l1 = psa.verify(q, kd, vd, kc, vc, indptr, 900, wl.scale, 4, nsplit=6, workspace=ws)
    o2, l2 = psa.verify(q, kd, vd, kc, vc, indptr, 900, wl.scale, 4, nsplit=6, workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
