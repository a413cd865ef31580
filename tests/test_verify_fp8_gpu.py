"""Split-KV verify over an e4m3 prefix cache on the GPU against the fp64
oracle ("Split-KV flash-decode attention for EAGLE target-verify",
implementation item 1: stage 1 applies the cache's fp8 scales k_scale /
v_scale).  Both sides read the same e4m3 bytes and scales; every call goes
through the C ABI."""
import numpy as np
import pytest
import torch

import oracle
import shared_prefix_attention_b200 as psa
from shared_prefix_attention_b200 import workloads as W
from parity import assert_parity

pytestmark = pytest.mark.gpu


def _wl(B=3, L=300, Ld=4, Hq=32, Hkv=8, nsplit=4, lens=None, seed=70):
    return W.VerifyWorkload("t", B=B, L=L, Ld=Ld, Hq=Hq, Hkv=Hkv, d=128, nsplit=nsplit,
                            seed=seed, prefix_lens=lens)


def _run(wl, rows=None):
    q, kd, vd, kc8, vc8 = (t.cuda() for t in wl.make_fp8("cpu"))
    indptr = torch.tensor(wl.kv_indptr(), dtype=torch.int32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    o, lse = psa.verify_fp8(q, kd, vd, kc8, vc8, wl.k_scale, wl.v_scale, indptr,
                            max(wl.lens() + [0]), wl.scale, wl.Ld, nsplit=wl.nsplit,
                            status=status)
    torch.cuda.synchronize()
    assert psa.read_status(status) == 0
    ro, rl = oracle.verify_fp8(q.cpu(), kd.cpu(), vd.cpu(), kc8.cpu(), vc8.cpu(), wl.k_scale,
                               wl.v_scale, np.array(wl.kv_indptr(), dtype=np.int64), wl.Ld,
                               wl.scale, rows=rows)
    if rows is not None:
        idx = torch.as_tensor(rows).long().cuda()
        o, lse = o[idx], lse[idx]
    return o, lse, ro, rl


@pytest.mark.parametrize("lens,nsplit", [
    ([300, 300, 300], 4),            # several tiles per split
    ([37, 513, 1000], 8),            # ragged prefixes, tail tiles
    ([0, 5, 16], 3),                 # empty prefix, empty splits
    ([2048, 17, 1], 32),             # many splits, most empty for short prefixes
    ([4096, 100], 256),              # maximum split count
])
def test_verify_fp8_parity_ragged(lens, nsplit):
    o, lse, ro, rl = _run(_wl(B=len(lens), lens=lens, nsplit=nsplit))
    assert_parity(o, lse, ro, rl, f"lens={lens} nsplit={nsplit}")


@pytest.mark.parametrize("Hq,Hkv,L,Ld", [
    (32, 1, 2048, 4),     # MQA: 128 rows per KV head, several row blocks
    (16, 2, 1024, 4),
    (8, 2, 777, 2),
    (32, 8, 512, 16),     # longest draft block
])
def test_verify_fp8_parity_gqa(Hq, Hkv, L, Ld):
    o, lse, ro, rl = _run(_wl(B=2, L=L, Ld=Ld, Hq=Hq, Hkv=Hkv, nsplit=5))
    assert_parity(o, lse, ro, rl, f"H={Hq}/{Hkv} L={L} Ld={Ld}")


def test_verify_fp8_full_size_sampled():
    """The 32-request, 16384-token workload, checked on every draft row of a
    spread of requests."""
    wl = W.VERIFY_FP8
    rows = sorted({b * wl.Ld + j for b in (0, 7, 19, 31) for j in range(wl.Ld)})
    o, lse, ro, rl = _run(wl, rows=rows)
    assert_parity(o, lse, ro, rl, "full size")


def test_verify_fp8_matches_bf16_path_on_decoded_cache():
    """With power-of-two scales the decoded, scaled cache is exact in bf16, so
    the fp8 path and the bf16 verify on that cache compute the same thing."""
    wl = W.VerifyWorkload("t", B=4, L=1500, Ld=4, Hq=32, Hkv=8, d=128, nsplit=6, seed=72,
                          k_scale=0.25, v_scale=0.5)
    q, kd, vd, kc8, vc8 = (t.cuda() for t in wl.make_fp8("cpu"))
    indptr = torch.tensor(wl.kv_indptr(), dtype=torch.int32, device="cuda")
    o8, l8 = psa.verify_fp8(q, kd, vd, kc8, vc8, wl.k_scale, wl.v_scale, indptr, wl.L, wl.scale,
                            wl.Ld, nsplit=wl.nsplit)
    kc = (kc8.view(torch.float8_e4m3fn).float() * wl.k_scale).to(torch.bfloat16)
    vc = (vc8.view(torch.float8_e4m3fn).float() * wl.v_scale).to(torch.bfloat16)
    o2, l2 = psa.verify(q, kd, vd, kc, vc, indptr, wl.L, wl.scale, wl.Ld, nsplit=wl.nsplit)
    torch.cuda.synchronize()
    assert (o8.float() - o2.float()).abs().max().item() <= 1e-2
    assert (l8 - l2).abs().max().item() <= 1e-3


@pytest.mark.parametrize("lens,Hq,Hkv,Ld,nsplit", [
    ([300, 37, 1000], 32, 8, 4, 4),      # ragged prefixes, tail tiles, GQA 4:1
    ([0, 700, 16], 16, 2, 8, 3),         # an empty prefix; 8 drafts
    ([2048, 129], 32, 1, 4, 32),         # MQA: several row blocks
])
def test_verify_fp8_paged(lens, Hq, Hkv, Ld, nsplit):
    """The e4m3 prefix read through a token-granular page table ([SKV] the
    verify entry's kv_indices with its fp8 scales): against the oracle on
    the same pool and table, and byte-identical to the contiguous cache."""
    wl = _wl(B=len(lens), lens=lens, Hq=Hq, Hkv=Hkv, Ld=Ld, nsplit=nsplit, seed=75)
    q, kd, vd, kc8, vc8 = (t.cuda() for t in wl.make_fp8("cpu"))
    ntok = kc8.shape[0]
    gen = torch.Generator().manual_seed(11)
    table = torch.randperm(2 * ntok + 3, generator=gen)[:ntok].to(torch.int32)
    kp = torch.zeros((2 * ntok + 3,) + tuple(kc8.shape[1:]), dtype=torch.uint8)
    vp = torch.zeros_like(kp)
    kp[table.long()] = kc8.cpu()
    vp[table.long()] = vc8.cpu()
    indptr = torch.tensor(wl.kv_indptr(), dtype=torch.int32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    o, lse = psa.verify_fp8(q, kd, vd, kp.cuda(), vp.cuda(), wl.k_scale, wl.v_scale, indptr,
                            max(lens), wl.scale, wl.Ld, nsplit=nsplit, status=status,
                            kv_indices=table.cuda())
    o2, l2 = psa.verify_fp8(q, kd, vd, kc8, vc8, wl.k_scale, wl.v_scale, indptr, max(lens),
                            wl.scale, wl.Ld, nsplit=nsplit)
    torch.cuda.synchronize()
    assert psa.read_status(status) == 0
    assert torch.equal(o, o2) and torch.equal(lse, l2)
    ro, rl = oracle.verify_fp8(q.cpu(), kd.cpu(), vd.cpu(), kp, vp, wl.k_scale, wl.v_scale,
                               np.array(wl.kv_indptr(), dtype=np.int64), wl.Ld, wl.scale,
                               kv_indices=table)
    assert_parity(o, lse, ro, rl, f"paged lens={lens}")
