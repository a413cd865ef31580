"""The debug build (libpsa_debug.so, compiled with PSA_DEBUG=1): the same
kernels with device-side bounds checks on every index they take from caller
data -- schedule items, tile entries and rectangle ranges, prefix offsets
and tree-mask offsets.  A failed check writes PSA_ERR_BOUNDS to the status
word and the access is skipped; nothing traps.

On the GPU the debug build must give the release build's results on valid
inputs, and must turn each corrupted input below into PSA_ERR_BOUNDS while
the context stays usable.  Corrupted inputs are only ever given to the debug
build: the release build trusts the schedule and offsets it is handed."""
import ctypes
import os

import numpy as np
import pytest
import torch

import oracle
import shared_prefix_attention_b200 as psa
from shared_prefix_attention_b200 import _binding as B
from shared_prefix_attention_b200 import workloads as W
from parity import assert_parity

DEBUG = psa.DEBUG_LIB_PATH
needs_debug_lib = pytest.mark.skipif(not os.path.exists(DEBUG),
                                     reason="libpsa_debug.so not built")


# ----------------------------------------------------------------- host only

@needs_debug_lib
def test_debug_library_exports_every_symbol():
    L = ctypes.CDLL(DEBUG)
    for name in psa.EXPORTS:
        assert hasattr(L, name), name


@needs_debug_lib
def test_bounds_status_has_a_message_in_both_builds():
    for path in (psa.LIB_PATH, DEBUG):
        with psa.use_library(path):
            assert "bounds" in psa.status_string(psa.PSA_ERR_BOUNDS)
    assert psa.lib() is B.load(psa.LIB_PATH)


# ----------------------------------------------------------------- GPU

def _status():
    return torch.zeros(1, dtype=torch.int32, device="cuda")


def _prefill_case(seed=41):
    wl = W.PrefillWorkload("dbg", P=300, N=3, S=170, Hq=8, Hkv=2, d=128, seed=seed)
    q, k, v = wl.make("cpu")
    tm, tn = psa.prefill_tiles(wl.d)
    sched = B.build_schedule(B.build_spec(wl.segments()), wl.cu_seqlens(), tm, tn)
    return wl, (q, k, v), sched


def _sched_parts(sched):
    n_items, n_kv, n_rect = int(sched[1]), int(sched[2]), int(sched[3])
    items = sched[8:8 + 4 * n_items].reshape(n_items, 4)
    kvs = sched[8 + 4 * n_items:8 + 4 * n_items + 8 * n_kv].reshape(n_kv, 8)
    return n_items, n_kv, n_rect, items, kvs


@pytest.mark.gpu
@needs_debug_lib
def test_debug_build_matches_the_oracle_on_valid_inputs():
    with psa.use_library(DEBUG):
        # prefill, bf16 and fp32 I/O
        wl, (q, k, v), sched = _prefill_case()
        st = _status()
        o, lse = psa.prefill(q.cuda(), k.cuda(), v.cuda(), torch.from_numpy(sched).cuda(),
                             wl.scale, status=st)
        torch.cuda.synchronize()
        assert psa.read_status(st) == 0
        ro, rl = oracle.prefill(q, k, v, wl.segments(), wl.scale)
        assert_parity(o, lse, ro, rl, "debug prefill")
        tw = W.TINY
        q32, k32, v32 = tw.make("cpu")
        o, lse = psa.prefill(q32.cuda(), k32.cuda(), v32.cuda(),
                             psa.plan_prefill(tw.segments(), tw.cu_seqlens(), tw.d), tw.scale,
                             status=st)
        torch.cuda.synchronize()
        assert psa.read_status(st) == 0
        ro, rl = oracle.prefill(q32, k32, v32, tw.segments(), tw.scale)
        assert_parity(o, lse, ro, rl, "debug prefill fp32")

        # backward
        gen = torch.Generator().manual_seed(3)
        dout = (torch.randn(q.shape, generator=gen) * 0.5).to(torch.bfloat16)
        qg, kg, vg = q.cuda(), k.cuda(), v.cuda()
        o, lse = psa.prefill(qg, kg, vg, torch.from_numpy(sched).cuda(), wl.scale)
        dq, dk, dv = psa.prefill_bwd(qg, kg, vg, o, lse, dout.cuda(),
                                     psa.plan_prefill_bwd(wl.segments(), wl.cu_seqlens(), wl.d),
                                     wl.scale, status=st)
        torch.cuda.synchronize()
        assert psa.read_status(st) == 0
        for got, ref in zip((dq, dk, dv), oracle.prefill_bwd(q, k, v, dout, wl.segments(),
                                                             wl.scale)):
            g = got.double().cpu().numpy()
            assert np.linalg.norm(g - ref) <= 2e-2 * np.linalg.norm(ref)

        # split-KV verify (contiguous), its e4m3 form and the shared-prefix form
        vw = W.VerifyWorkload("dbg", B=3, L=0, Ld=4, Hq=16, Hkv=4, d=128, nsplit=4,
                              prefix_lens=[200, 37, 513], seed=11)
        q, kd, vd, kc, vc = vw.make("cpu")
        indptr = torch.tensor(vw.kv_indptr(), dtype=torch.int32, device="cuda")
        o, lse = psa.verify(q.cuda(), kd.cuda(), vd.cuda(), kc.cuda(), vc.cuda(), indptr, 513,
                            vw.scale, vw.Ld, nsplit=4, status=st)
        torch.cuda.synchronize()
        assert psa.read_status(st) == 0
        ro, rl = oracle.verify(q, kd, vd, kc, vc, np.array(vw.kv_indptr()), vw.Ld, vw.scale)
        assert_parity(o, lse, ro, rl, "debug verify")
        q, kd, vd, kc8, vc8 = vw.make_fp8("cpu")
        o, lse = psa.verify_fp8(q.cuda(), kd.cuda(), vd.cuda(), kc8.cuda(), vc8.cuda(),
                                vw.k_scale, vw.v_scale, indptr, 513, vw.scale, vw.Ld, nsplit=4,
                                status=st)
        torch.cuda.synchronize()
        assert psa.read_status(st) == 0
        ro, rl = oracle.verify_fp8(q, kd, vd, kc8, vc8, vw.k_scale, vw.v_scale,
                                   np.array(vw.kv_indptr()), vw.Ld, vw.scale)
        assert_parity(o, lse, ro, rl, "debug verify fp8")
        sw = W.SharedVerifyWorkload("dbg", B=5, L=700, Ld=4, Hq=16, Hkv=4, d=128, seed=7)
        q, kd, vd, kp, vp = sw.make("cpu")
        o, lse = psa.verify_shared(q.cuda(), kd.cuda(), vd.cuda(), kp.cuda(), vp.cuda(),
                                   sw.scale, sw.Ld, status=st)
        torch.cuda.synchronize()
        assert psa.read_status(st) == 0
        ro, rl = oracle.verify_shared(q, kd, vd, kp, vp, sw.Ld, sw.scale)
        assert_parity(o, lse, ro, rl, "debug verify shared")

        # extend form: page table, ragged drafts, tree masks
        ew = W.ExtendVerifyWorkload("dbg", draft_lens=[3, 0, 5], prefix_lens=[300, 77, 1000],
                                    Hq=16, Hkv=4, d=128, nsplit=4, seed=9)
        q, kd, vd, kp, vp, idx, mask = ew.make("cpu")
        dev = lambda xs: torch.tensor(xs, dtype=torch.int32, device="cuda")  # noqa: E731
        o, lse = psa.verify_extend(q.cuda(), kd.cuda(), vd.cuda(), kp.cuda(), vp.cuda(),
                                   dev(ew.qo_indptr()), ew.max_draft_len, dev(ew.kv_indptr()),
                                   ew.max_prefix_len, ew.scale, kv_indices=idx.cuda(),
                                   draft_mask=mask.cuda(), mask_indptr=dev(ew.mask_indptr()),
                                   nsplit=4, status=st)
        torch.cuda.synchronize()
        assert psa.read_status(st) == 0
        ro, rl = oracle.verify_extend(q, kd, vd, kp, vp, ew.qo_indptr(), ew.kv_indptr(),
                                      ew.scale, kv_indices=idx, draft_mask=mask,
                                      mask_indptr=ew.mask_indptr())
        assert_parity(o, lse, ro, rl, "debug verify extend")

        # shared-latent sparse
        spw = W.SparseLatentWorkload("dbg", T=300, H=64, dl=512, topk=256, seed=5)
        q, lat, sidx = spw.make("cpu")
        o, lse = psa.sparse_latent(q.cuda(), lat.cuda(), sidx.cuda(), spw.scale, status=st)
        torch.cuda.synchronize()
        assert psa.read_status(st) == 0
        ro, rl = oracle.sparse_latent(q, lat, sidx, spw.scale)
        assert_parity(o, lse, ro, rl, "debug sparse")


@pytest.mark.gpu
@needs_debug_lib
def test_debug_build_reports_corrupted_inputs():
    with psa.use_library(DEBUG):
        wl, (q, k, v), sched = _prefill_case()
        qg, kg, vg = q.cuda(), k.cuda(), v.cuda()
        n_items, n_kv, n_rect, items, kvs = _sched_parts(sched)

        # a schedule block whose tile entries run past the tile list
        bad = sched.copy()
        _, _, _, bitems, _ = _sched_parts(bad)
        bitems[0, 2] = n_kv + 1000
        st = _status()
        psa.prefill(qg, kg, vg, torch.from_numpy(bad).cuda(), wl.scale, status=st)
        torch.cuda.synchronize()
        assert psa.read_status(st) == psa.PSA_ERR_BOUNDS

        # a partially visible tile whose rectangle range runs past the list
        part = np.nonzero(((kvs[:, 6] & 1) != 0) & ((kvs[:, 6] & 4) == 0) & (kvs[:, 3] > 0))[0]
        assert len(part)
        bad = sched.copy()
        _, _, _, _, bkvs = _sched_parts(bad)
        bkvs[part[0], 2] = n_rect + 50
        st = _status()
        psa.prefill(qg, kg, vg, torch.from_numpy(bad).cuda(), wl.scale, status=st)
        torch.cuda.synchronize()
        assert psa.read_status(st) == psa.PSA_ERR_BOUNDS

        # the backward's dQ schedule with a block past the tokens
        o, lse = psa.prefill(qg, kg, vg, torch.from_numpy(sched).cuda(), wl.scale)
        tm, tn = psa.prefill_bwd_tiles(wl.d)
        spec = B.build_spec(wl.segments())
        sq = B.build_schedule(spec, wl.cu_seqlens(), tm, tn)
        skv = B.build_schedule(B.transpose_spec(spec), wl.cu_seqlens(), tm, tn)
        _, _, _, qitems, _ = _sched_parts(sq)
        qitems[0, 0] = wl.T + 512
        st = _status()
        psa.prefill_bwd(qg, kg, vg, o, lse, qg, (torch.from_numpy(sq).cuda(),
                                                  torch.from_numpy(skv).cuda()),
                        wl.scale, status=st)
        torch.cuda.synchronize()
        assert psa.read_status(st) == psa.PSA_ERR_BOUNDS

        # a contiguous prefix that ends past the cache
        vw = W.VerifyWorkload("dbg", B=2, L=0, Ld=4, Hq=16, Hkv=4, d=128, nsplit=4,
                              prefix_lens=[200, 300], seed=12)
        q, kd, vd, kc, vc = (t.cuda() for t in vw.make("cpu"))
        indptr = torch.tensor([0, 200, 300 + kc.shape[0]], dtype=torch.int32, device="cuda")
        st = _status()
        psa.verify(q, kd, vd, kc, vc, indptr, 300 + kc.shape[0], vw.scale, vw.Ld, nsplit=4,
                   status=st)
        torch.cuda.synchronize()
        assert psa.read_status(st) == psa.PSA_ERR_BOUNDS

        # a tree-mask offset past the mask (mask_indptr[B], its length, intact)
        ew = W.ExtendVerifyWorkload("dbg", draft_lens=[3, 4, 2], prefix_lens=[100, 50, 70],
                                    Hq=16, Hkv=4, d=128, nsplit=2, seed=13)
        q, kd, vd, kp, vp, idx, mask = ew.make("cpu")
        mi = list(ew.mask_indptr())
        mi[1] = mi[-1] + 4096
        dev = lambda xs: torch.tensor(xs, dtype=torch.int32, device="cuda")  # noqa: E731
        st = _status()
        psa.verify_extend(q.cuda(), kd.cuda(), vd.cuda(), kp.cuda(), vp.cuda(),
                          dev(ew.qo_indptr()), ew.max_draft_len, dev(ew.kv_indptr()),
                          ew.max_prefix_len, ew.scale, kv_indices=idx.cuda(),
                          draft_mask=mask.cuda(), mask_indptr=dev(mi), nsplit=2, status=st)
        torch.cuda.synchronize()
        assert psa.read_status(st) == psa.PSA_ERR_BOUNDS

        # the context is still good: a valid call after all of the above
        st = _status()
        o, lse = psa.prefill(qg, kg, vg, torch.from_numpy(sched).cuda(), wl.scale, status=st)
        torch.cuda.synchronize()
        assert psa.read_status(st) == 0
        ro, rl = oracle.prefill(*(t for t in (qg.cpu(), kg.cpu(), vg.cpu())), wl.segments(),
                                wl.scale)
        assert_parity(o, lse, ro, rl, "after the corrupted calls")
