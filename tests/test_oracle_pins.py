"""Pins for the fp64 oracle: each check ties the oracle to something other
than itself -- hand-derived golden values, closed forms, brute force, an
independent library routine (torch SDPA in fp64) or an identity the pages
state.  The last test builds deliberately broken copies of the oracle and
shows that every planted mistake fails at least one pin.

Page references are by title and section:
  [PS]  "KV-0 redundancy prefix sharing attention mask design" (PrefixSharing PR #50)
  [SKV] "Split-KV flash-decode attention for EAGLE target-verify" (sglang PR #27382)
  [MLA] "SM8x sparse-MLA prefill fallback re-reads the shared MLA latent once per head"
"""
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from shared_prefix_attention_b200 import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _load_matrix(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append([float(x) for x in line.split()])
    return np.array(rows)


def _rand(shape, seed, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(shape, generator=g) * scale).to(torch.bfloat16).float()


def _expand_kv(k, Hq):
    """Repeat each KV head Hq/Hkv times, contiguous (GQA -> MHA)."""
    return k.repeat_interleave(Hq // k.shape[1], dim=1)


def _sdpa(q, k, v, mask, scale):
    """torch SDPA in fp64.  q [Tq,H,d], k/v [Tk,H,d], mask [Tq,Tk] bool (True = visible)
    or the string 'causal'."""
    qq = q.double().permute(1, 0, 2)[None]
    kk = k.double().permute(1, 0, 2)[None]
    vv = v.double().permute(1, 0, 2)[None]
    if isinstance(mask, str):
        out = F.scaled_dot_product_attention(qq, kk, vv, is_causal=True, scale=scale)
    else:
        out = F.scaled_dot_product_attention(qq, kk, vv, attn_mask=mask, scale=scale)
    return out[0].permute(1, 0, 2).numpy()


def _python_visibility(segments, T):
    """Brute-force visibility written independently of the oracle: walk each
    query's ancestor chain in Python."""
    start, lens, parent = oracle.segment_arrays(segments)
    seg = np.full(T, -1)
    for s, (a, n) in enumerate(zip(start, lens)):
        seg[a:a + n] = s
    vis = np.zeros((T, T), dtype=bool)
    for qi in range(T):
        anc = set()
        s = seg[qi]
        while s >= 0:
            anc.add(s)
            s = parent[s]
        for kj in range(qi + 1):
            vis[qi, kj] = seg[kj] in anc
    return vis


# ---------------------------------------------------------------- pin checks
# Each returns True when the oracle (``lib``) agrees with the pin.

def pin_golden_masks(lib):
    ok = True
    m = _load_matrix("mask_P2_N2_S2.txt").astype(np.uint8)
    ok &= np.array_equal(oracle.visibility(W.grpo_segments(2, 2, 2), lib=lib), m)
    m = _load_matrix("mask_chain_1_2_1.txt").astype(np.uint8)
    ok &= np.array_equal(oracle.visibility(W.chain_segments([1, 2, 1]), lib=lib), m)
    return bool(ok)


def pin_golden_tiny_attention(lib):
    g = _load_matrix("attn_tiny_hand.txt")
    q = torch.tensor([2.0, 1.0, 1.0]).view(3, 1, 1)
    k = torch.tensor([0.0, math.log(3.0), math.log(7.0)]).view(3, 1, 1)
    v = torch.tensor([1.0, 5.0, 100.0]).view(3, 1, 1)
    o, lse = oracle.prefill(q, k, v, W.grpo_segments(1, 2, 1), 1.0, lib=lib)
    return bool(np.allclose(o[:, 0, 0], g[:, 1], rtol=1e-6, atol=1e-6)
                and np.allclose(lse[:, 0], g[:, 2], atol=1e-6))


def pin_equivalence_route(lib):
    """[PS] design summary: the flat forward equals running [prefix; s_i]
    separately under ordinary causal attention (the physical-copy route)."""
    P, N, S, Hq, Hkv, d = 24, 3, 10, 4, 2, 16
    T = P + N * S
    q, k, v = _rand((T, Hq, d), 1), _rand((T, Hkv, d), 2), _rand((T, Hkv, d), 3)
    scale = 1 / math.sqrt(d)
    o, lse = oracle.prefill(q, k, v, W.grpo_segments(P, N, S), scale, lib=lib)
    ke, ve = _expand_kv(k, Hq), _expand_kv(v, Hq)
    ok = np.allclose(o[:P], _sdpa(q[:P], ke[:P], ve[:P], "causal", scale), atol=1e-12)
    for i in range(N):
        sl = slice(P + i * S, P + (i + 1) * S)
        qi = torch.cat([q[:P], q[sl]])
        ki = torch.cat([ke[:P], ke[sl]])
        vi = torch.cat([ve[:P], ve[sl]])
        ref = _sdpa(qi, ki, vi, "causal", scale)[P:]
        ok &= np.allclose(o[sl], ref, atol=1e-12)
    return bool(ok)


def pin_sdpa_random_trees(lib):
    """Library cross-check on random segment forests with an explicit mask
    built by the independent Python walker."""
    ok = True
    for seed in range(3):
        g = torch.Generator().manual_seed(100 + seed)
        segs = W.random_tree_segments(g, nseg=6, max_len=7, groups=2)
        T = sum(s[0] for s in segs)
        Hq, Hkv, d = 4, 2, 8
        q, k, v = _rand((T, Hq, d), seed), _rand((T, Hkv, d), seed + 10), _rand((T, Hkv, d), seed + 20)
        o, _ = oracle.prefill(q, k, v, segs, 0.3, lib=lib)
        mask = torch.from_numpy(_python_visibility(segs, T))
        ref = _sdpa(q, _expand_kv(k, Hq), _expand_kv(v, Hq), mask, 0.3)
        ok &= np.allclose(o, ref, atol=1e-12)
        ok &= np.array_equal(oracle.visibility(segs, lib=lib).astype(bool),
                             _python_visibility(segs, T))
    return bool(ok)


def pin_closed_forms(lib):
    """Q = 0: O is the mean of the visible V rows and LSE = ln(#visible).
    One-hot V rows: O is the softmax row itself, which sums to 1 and is zero
    on invisible keys."""
    P, N, S, d = 5, 3, 4, 32
    segs = W.grpo_segments(P, N, S)
    T = P + N * S
    vis = _python_visibility(segs, T)
    v = _rand((T, 1, d), 7)
    q = torch.zeros((T, 1, d))
    k = _rand((T, 1, d), 8)
    o, lse = oracle.prefill(q, k, v, segs, 0.5, lib=lib)
    cnt = vis.sum(1)
    mean = (vis.astype(np.float64) @ v[:, 0].double().numpy()) / cnt[:, None]
    ok = np.allclose(o[:, 0], mean, atol=1e-12) and np.allclose(lse[:, 0], np.log(cnt), atol=1e-12)
    onehot = torch.eye(T, d)[:, None, :]          # d >= T: row j is e_j
    q2 = _rand((T, 1, d), 9)
    o2, _ = oracle.prefill(q2, k, onehot, segs, 0.5, lib=lib)
    w = o2[:, 0, :T]
    ok &= np.allclose(w.sum(1), 1.0, atol=1e-12)
    ok &= bool(np.all(w[~vis] == 0.0)) and bool(np.all(w[vis] > 0.0))
    return bool(ok)


def pin_special_cases(lib):
    """N = 1 is plain causal attention over P + S; P = 0 is N independent
    causal sequences (varlen); GQA equals MHA with KV heads repeated."""
    d, Hq, Hkv = 16, 4, 2
    ok = True
    T = 20
    q, k, v = _rand((T, Hq, d), 11), _rand((T, Hkv, d), 12), _rand((T, Hkv, d), 13)
    ke, ve = _expand_kv(k, Hq), _expand_kv(v, Hq)
    o, _ = oracle.prefill(q, k, v, W.grpo_segments(12, 1, 8), 0.25, lib=lib)
    ok &= np.allclose(o, _sdpa(q, ke, ve, "causal", 0.25), atol=1e-12)
    o, _ = oracle.prefill(q, k, v, W.grpo_segments(0, 4, 5), 0.25, lib=lib)
    for i in range(4):
        sl = slice(5 * i, 5 * i + 5)
        ok &= np.allclose(o[sl], _sdpa(q[sl], ke[sl], ve[sl], "causal", 0.25), atol=1e-12)
    o_mha, _ = oracle.prefill(q, ke, ve, W.grpo_segments(6, 2, 7), 0.25, lib=lib)
    o_gqa, _ = oracle.prefill(q, k, v, W.grpo_segments(6, 2, 7), 0.25, lib=lib)
    ok &= np.allclose(o_mha, o_gqa, atol=1e-13)
    return bool(ok)


def pin_brute_force_python(lib):
    """Pure-Python loops on a tiny input (T = 7, d = 3)."""
    segs = W.grpo_segments(3, 2, 2)
    T, H, d, scale = 7, 2, 3, 0.7
    q, k, v = _rand((T, H, d), 21), _rand((T, 1, d), 22), _rand((T, 1, d), 23)
    vis = _python_visibility(segs, T)
    o, lse = oracle.prefill(q, k, v, segs, scale, lib=lib)
    ok = True
    for qi in range(T):
        for h in range(H):
            zs = [(scale * sum(float(q[qi, h, c]) * float(k[kj, 0, c]) for c in range(d)), kj)
                  for kj in range(T) if vis[qi, kj]]
            m = max(z for z, _ in zs)
            den = sum(math.exp(z - m) for z, _ in zs)
            for c in range(d):
                num = sum(math.exp(z - m) * float(v[kj, 0, c]) for z, kj in zs)
                ok &= abs(o[qi, h, c] - num / den) < 1e-12
            ok &= abs(lse[qi, h] - (m + math.log(den))) < 1e-12
    return bool(ok)


def _verify_case(seed=31, lens=(37, 0, 64), Ld=3, Hq=4, Hkv=2, d=16):
    B = len(lens)
    ntok = sum(lens)
    q = _rand((B * Ld, Hq, d), seed)
    kd, vd = _rand((B * Ld, Hkv, d), seed + 1), _rand((B * Ld, Hkv, d), seed + 2)
    kc, vc = _rand((ntok, Hkv, d), seed + 3), _rand((ntok, Hkv, d), seed + 4)
    indptr = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    return q, kd, vd, kc, vc, indptr, Ld


def pin_verify_against_sdpa(lib):
    """[SKV] implementation item 1: draft row j of request b sees the whole
    cached prefix of b plus drafts 0..j."""
    q, kd, vd, kc, vc, indptr, Ld = _verify_case()
    Hq, d = q.shape[1], q.shape[2]
    scale = 1 / math.sqrt(d)
    o, _ = oracle.verify(q, kd, vd, kc, vc, indptr, Ld, scale, lib=lib)
    ok = True
    for b in range(len(indptr) - 1):
        p0, p1 = int(indptr[b]), int(indptr[b + 1])
        ks = torch.cat([kc[p0:p1], kd[b * Ld:(b + 1) * Ld]])
        vs = torch.cat([vc[p0:p1], vd[b * Ld:(b + 1) * Ld]])
        L = p1 - p0
        mask = torch.ones((Ld, L + Ld), dtype=torch.bool)
        mask[:, L:] = torch.tril(torch.ones((Ld, Ld), dtype=torch.bool))
        ref = _sdpa(q[b * Ld:(b + 1) * Ld], _expand_kv(ks, Hq), _expand_kv(vs, Hq), mask, scale)
        ok &= np.allclose(o[b * Ld:(b + 1) * Ld], ref, atol=1e-12)
    return bool(ok)


def pin_verify_tree_mask(lib):
    """[SKV] can_handle: EAGLE trees (topk > 1) bring a custom draft mask while
    the prefix stays fully visible.  Checked against SDPA with the explicit
    mask; the lower-triangular mask reproduces the causal verify exactly."""
    q, kd, vd, kc, vc, indptr, Ld = _verify_case(seed=61, Ld=4)
    B, Hq, d = len(indptr) - 1, q.shape[1], q.shape[2]
    scale = 1 / math.sqrt(d)
    # a depth-2 tree per request: 0 -> {1, 2}, 1 -> 3 (each draft sees its ancestors and itself)
    tree = np.array([[1, 0, 0, 0], [1, 1, 0, 0], [1, 0, 1, 0], [1, 1, 0, 1]], dtype=np.uint8)
    dm = np.tile(tree, (B, 1))
    o, _ = oracle.verify_tree(q, kd, vd, kc, vc, indptr, dm, Ld, scale, lib=lib)
    ok = True
    for b in range(B):
        p0, p1 = int(indptr[b]), int(indptr[b + 1])
        ks = torch.cat([kc[p0:p1], kd[b * Ld:(b + 1) * Ld]])
        vs = torch.cat([vc[p0:p1], vd[b * Ld:(b + 1) * Ld]])
        L = p1 - p0
        mask = torch.ones((Ld, L + Ld), dtype=torch.bool)
        mask[:, L:] = torch.from_numpy(tree.astype(bool))
        ref = _sdpa(q[b * Ld:(b + 1) * Ld], _expand_kv(ks, Hq), _expand_kv(vs, Hq), mask, scale)
        ok &= np.allclose(o[b * Ld:(b + 1) * Ld], ref, atol=1e-12)
    causal = np.tile(np.tril(np.ones((Ld, Ld), dtype=np.uint8)), (B, 1))
    o1, l1 = oracle.verify_tree(q, kd, vd, kc, vc, indptr, causal, Ld, scale, lib=lib)
    o2, l2 = oracle.verify(q, kd, vd, kc, vc, indptr, Ld, scale, lib=lib)
    ok &= np.array_equal(o1, o2) and np.array_equal(l1, l2)
    return bool(ok)


def _random_tree(n, rng):
    """Ancestor mask of a random tree over n drafts in topological order."""
    parent = [-1] + [int(rng.integers(-1, j)) for j in range(1, n)]
    m = np.zeros((n, n), dtype=np.uint8)
    for j in range(n):
        a = j
        while a >= 0:
            m[j, a] = 1
            a = parent[a]
    return m


def pin_verify_extend_form(lib):
    """[SKV] the verify entry's signature (qo_indptr, kv_indptr, kv_indices,
    custom_mask, mask_indptr) and can_handle (ragged extend and custom masks
    left out of the split path): ragged draft counts, a prefix read through a
    token-granular page table, per-request tree masks.  Checked against SDPA
    on keys gathered with numpy fancy indexing; with a uniform draft count
    and the identity table it reproduces the contiguous verify exactly."""
    rng = np.random.default_rng(71)
    Hq, Hkv, d = 4, 2, 16
    scale = 1 / math.sqrt(d)
    Lds = [3, 0, 5, 1]
    lens = [29, 11, 0, 40]
    B = len(Lds)
    qo = np.concatenate([[0], np.cumsum(Lds)]).astype(np.int64)
    kvp = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    nslots = 120
    table = rng.permutation(nslots)[:int(kvp[-1])].astype(np.int32)
    NR = int(qo[-1])
    q = _rand((NR, Hq, d), 72)
    kd, vd = _rand((NR, Hkv, d), 73), _rand((NR, Hkv, d), 74)
    kc, vc = _rand((nslots, Hkv, d), 75), _rand((nslots, Hkv, d), 76)
    masks = [_random_tree(n, rng) for n in Lds]
    mi = np.concatenate([[0], np.cumsum([n * n for n in Lds])]).astype(np.int64)
    flat = np.concatenate([m.reshape(-1) for m in masks]).astype(np.uint8)
    ok = True
    for dm, mask_of in ((flat, lambda b: masks[b]), (None, lambda b: np.tril(np.ones((Lds[b],) * 2)))):
        o, lse = oracle.verify_extend(q, kd, vd, kc, vc, qo, kvp, scale, kv_indices=table,
                                      draft_mask=dm, mask_indptr=None if dm is None else mi,
                                      lib=lib)
        for b in range(B):
            if Lds[b] == 0:
                continue
            sl = slice(int(qo[b]), int(qo[b + 1]))
            slots = torch.from_numpy(table[kvp[b]:kvp[b + 1]].astype(np.int64))
            ks = torch.cat([kc[slots], kd[sl]])
            vs = torch.cat([vc[slots], vd[sl]])
            mask = torch.ones((Lds[b], lens[b] + Lds[b]), dtype=torch.bool)
            mask[:, lens[b]:] = torch.from_numpy(mask_of(b).astype(bool))
            ref = _sdpa(q[sl], _expand_kv(ks, Hq), _expand_kv(vs, Hq), mask, scale)
            ok &= np.allclose(o[sl], ref, atol=1e-12)
    # uniform draft count, identity table: the contiguous verify
    q2, kd2, vd2, kc2, vc2, indptr, Ld = _verify_case(seed=77)
    B2 = len(indptr) - 1
    qo2 = np.arange(B2 + 1, dtype=np.int64) * Ld
    o1, l1 = oracle.verify_extend(q2, kd2, vd2, kc2, vc2, qo2, indptr, 0.3,
                                  kv_indices=np.arange(int(indptr[-1]), dtype=np.int32), lib=lib)
    o2, l2 = oracle.verify(q2, kd2, vd2, kc2, vc2, indptr, Ld, 0.3, lib=lib)
    ok &= np.array_equal(o1, o2) and np.array_equal(l1, l2)
    return bool(ok)


def _split_combine(q, kd, vd, kc, vc, indptr, Ld, scale, nsplit):
    """Split-KV + LSE combine written out per [SKV] implementation item 1:
    stage 1 gives each prefix chunk a normalised partial O and its LSE
    (empty chunk: LSE = -inf); stage 2 merges the chunks and the causal
    draft block by their LSE weights."""
    BL, Hq, d = q.shape
    Hkv = kc.shape[1]
    G = Hq // Hkv
    o = np.zeros((BL, Hq, d))
    lse = np.zeros((BL, Hq))
    for r in range(BL):
        b, j = divmod(r, Ld)
        p0, p1 = int(indptr[b]), int(indptr[b + 1])
        chunk = -(-(p1 - p0) // nsplit) if p1 > p0 else 0
        for h in range(Hq):
            kvh = h // G
            qv = q[r, h].double().numpy()
            parts = []
            for s in range(nsplit):
                a, e = p0 + s * chunk, min(p0 + (s + 1) * chunk, p1)
                if e <= a:
                    parts.append((-np.inf, np.zeros(d)))
                    continue
                z = scale * (kc[a:e, kvh].double().numpy() @ qv)
                m = z.max()
                w = np.exp(z - m)
                parts.append((m + np.log(w.sum()), (w @ vc[a:e, kvh].double().numpy()) / w.sum()))
            zd = scale * (kd[b * Ld:b * Ld + j + 1, kvh].double().numpy() @ qv)
            for i, z in enumerate(zd):
                parts.append((z, vd[b * Ld + i, kvh].double().numpy()))
            M = max(p[0] for p in parts)
            wts = [math.exp(p[0] - M) if p[0] > -np.inf else 0.0 for p in parts]
            tot = sum(wts)
            o[r, h] = sum(w * p[1] for w, p in zip(wts, parts)) / tot
            lse[r, h] = M + math.log(tot)
    return o, lse


def pin_split_identity(lib):
    """[SKV] implementation item 1: split-KV partials plus an LSE combine
    equal the one-pass softmax, for any split count, empty splits included."""
    q, kd, vd, kc, vc, indptr, Ld = _verify_case()
    scale = 1 / math.sqrt(q.shape[2])
    o, lse = oracle.verify(q, kd, vd, kc, vc, indptr, Ld, scale, lib=lib)
    ok = True
    for nsplit in (1, 4, 7, 80):
        o2, lse2 = _split_combine(q, kd, vd, kc, vc, indptr, Ld, scale, nsplit)
        ok &= np.allclose(o, o2, atol=1e-12) and np.allclose(lse, lse2, atol=1e-12)
    return bool(ok)


def pin_sparse_latent(lib):
    """[MLA] environment: K = V = the shared latent; each query sees only its
    index list.  Rows t < topk list 0..t, so they equal dense causal MQA."""
    T, H, dl, topk = 40, 4, 32, 16
    wl = W.SparseLatentWorkload("t", T=T, H=H, dl=dl, topk=topk, seed=9)
    q, lat, idx = wl.make()
    q, lat = q.float(), lat.float()
    o, lse = oracle.sparse_latent(q, lat, idx, wl.scale, lib=lib)
    lat3 = lat[:, None, :].expand(T, H, dl)
    ok = np.allclose(o[:topk], _sdpa(q[:topk], lat3[:topk], lat3[:topk], "causal", wl.scale),
                     atol=1e-12)
    mask = torch.zeros((T, T), dtype=torch.bool)
    for t in range(T):
        sel = idx[t][idx[t] >= 0].long()
        mask[t, sel] = True
    ok &= np.allclose(o, _sdpa(q, lat3, lat3, mask, wl.scale), atol=1e-12)
    q0 = torch.zeros_like(q)
    _, lse0 = oracle.sparse_latent(q0, lat, idx, wl.scale, lib=lib)
    ok &= np.allclose(lse0, np.log(mask.sum(1).numpy())[:, None], atol=1e-12)
    return bool(ok)


def pin_verify_shared_prefix(lib):
    """One prefix shared by every request, stored once ([PS] design summary:
    the flat layout keeps the prefix K/V a single time) and seen by every
    draft row together with its own causal draft block ([SKV] implementation
    item 1).  Checked against torch SDPA with an explicit mask, and against
    the per-request verify on a cache that holds B physical copies of the
    prefix (the deduplication must not change the result)."""
    B, Ld, Hq, Hkv, d, L = 3, 4, 6, 2, 16, 45
    q = _rand((B * Ld, Hq, d), 51)
    kd, vd = _rand((B * Ld, Hkv, d), 52), _rand((B * Ld, Hkv, d), 53)
    kp, vp = _rand((L, Hkv, d), 54), _rand((L, Hkv, d), 55)
    scale = 1 / math.sqrt(d)
    o, lse = oracle.verify_shared(q, kd, vd, kp, vp, Ld, scale, lib=lib)
    ok = True
    for b in range(B):
        ks = torch.cat([kp, kd[b * Ld:(b + 1) * Ld]])
        vs = torch.cat([vp, vd[b * Ld:(b + 1) * Ld]])
        mask = torch.ones((Ld, L + Ld), dtype=torch.bool)
        mask[:, L:] = torch.tril(torch.ones((Ld, Ld), dtype=torch.bool))
        ref = _sdpa(q[b * Ld:(b + 1) * Ld], _expand_kv(ks, Hq), _expand_kv(vs, Hq), mask, scale)
        ok &= np.allclose(o[b * Ld:(b + 1) * Ld], ref, atol=1e-12)
    kc, vc = kp.repeat(B, 1, 1), vp.repeat(B, 1, 1)
    indptr = np.arange(B + 1, dtype=np.int64) * L
    o2, lse2 = oracle.verify(q, kd, vd, kc, vc, indptr, Ld, scale, lib=lib)
    ok &= np.array_equal(o, o2) and np.array_equal(lse, lse2)
    # with a draft tree per request ([SKV] can_handle: topk > 1): SDPA with the
    # tree over the drafts, and the per-request tree verify on the B copies
    rng = np.random.default_rng(56)
    trees = [_random_tree(Ld, rng) for _ in range(B)]
    dm = np.concatenate(trees).astype(np.uint8)
    o3, l3 = oracle.verify_shared(q, kd, vd, kp, vp, Ld, scale, lib=lib, draft_mask=dm)
    for b in range(B):
        ks = torch.cat([kp, kd[b * Ld:(b + 1) * Ld]])
        vs = torch.cat([vp, vd[b * Ld:(b + 1) * Ld]])
        mask = torch.ones((Ld, L + Ld), dtype=torch.bool)
        mask[:, L:] = torch.from_numpy(trees[b].astype(bool))
        ref = _sdpa(q[b * Ld:(b + 1) * Ld], _expand_kv(ks, Hq), _expand_kv(vs, Hq), mask, scale)
        ok &= np.allclose(o3[b * Ld:(b + 1) * Ld], ref, atol=1e-12)
    o4, l4 = oracle.verify_tree(q, kd, vd, kc, vc, indptr, dm, Ld, scale, lib=lib)
    ok &= np.array_equal(o3, o4) and np.array_equal(l3, l4)
    return bool(ok)


def pin_e4m3_decoder(lib):
    """The e4m3 decoder behind the fp8 verify (the split-KV verify page's fp8
    cache scaling) agrees with torch's float8_e4m3fn on all 256 codes."""
    codes = np.arange(256, dtype=np.uint8)
    mine = oracle.decode_e4m3(codes, lib=lib)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).double().numpy()
    nan = np.isnan(ref)
    return bool(np.array_equal(np.isnan(mine), nan) and np.array_equal(mine[~nan], ref[~nan]))


def pin_verify_fp8_cache(lib):
    """[SKV] implementation item 1 (stage 1 applies the fp8 scales): a cached
    key is k_scale * e4m3, a cached value v_scale * e4m3, drafts are not
    scaled.  Checked against torch SDPA fp64 on the decoded, scaled cache,
    and, with power-of-two scales, against the float verify on that cache."""
    q, kd, vd, kc, vc, indptr, Ld = _verify_case(seed=71)
    Hq, d = q.shape[1], q.shape[2]
    scale = 1 / math.sqrt(d)
    ok = True
    for ks, vs in ((0.37, 1.9), (0.25, 2.0)):
        kc8 = (kc / ks).to(torch.float8_e4m3fn)
        vc8 = (vc / vs).to(torch.float8_e4m3fn)
        o, lse = oracle.verify_fp8(q, kd, vd, kc8, vc8, ks, vs, indptr, Ld, scale, lib=lib)
        kr = torch.from_numpy(oracle.decode_e4m3(kc8, lib=lib) * ks)
        vr = torch.from_numpy(oracle.decode_e4m3(vc8, lib=lib) * vs)
        for b in range(len(indptr) - 1):
            p0, p1 = int(indptr[b]), int(indptr[b + 1])
            keys = torch.cat([kr[p0:p1], kd[b * Ld:(b + 1) * Ld].double()])
            vals = torch.cat([vr[p0:p1], vd[b * Ld:(b + 1) * Ld].double()])
            L = p1 - p0
            mask = torch.ones((Ld, L + Ld), dtype=torch.bool)
            mask[:, L:] = torch.tril(torch.ones((Ld, Ld), dtype=torch.bool))
            ref = _sdpa(q[b * Ld:(b + 1) * Ld], _expand_kv(keys, Hq), _expand_kv(vals, Hq),
                        mask, scale)
            ok &= np.allclose(o[b * Ld:(b + 1) * Ld], ref, atol=1e-12)
        if ks == 0.25:
            o2, lse2 = oracle.verify(q, kd, vd, kr.float(), vr.float(), indptr, Ld, scale,
                                     lib=lib)
            ok &= np.allclose(o, o2, atol=1e-12) and np.allclose(lse, lse2, atol=1e-12)
    # through a page table: the cache rows scattered over a larger pool
    # (numpy fancy indexing), the same result as the contiguous cache
    ntok = kc.shape[0]
    rng = np.random.default_rng(72)
    table = rng.permutation(2 * ntok)[:ntok].astype(np.int32)
    kc8 = (kc / 0.37).to(torch.float8_e4m3fn).view(torch.uint8)
    vc8 = (vc / 1.9).to(torch.float8_e4m3fn).view(torch.uint8)
    kpool = torch.zeros((2 * ntok,) + tuple(kc8.shape[1:]), dtype=torch.uint8)
    vpool = torch.zeros_like(kpool)
    kpool[torch.from_numpy(table.astype(np.int64))] = kc8
    vpool[torch.from_numpy(table.astype(np.int64))] = vc8
    o1, l1 = oracle.verify_fp8(q, kd, vd, kc8, vc8, 0.37, 1.9, indptr, Ld, scale, lib=lib)
    o2, l2 = oracle.verify_fp8(q, kd, vd, kpool, vpool, 0.37, 1.9, indptr, Ld, scale, lib=lib,
                               kv_indices=table)
    ok &= np.array_equal(o1, o2) and np.array_equal(l1, l2)
    return bool(ok)


def pin_backward_finite_differences(lib):
    """The backward is the derivative of the forward: central differences of
    L = sum(O * G) through the fp64 forward oracle, every input element of a
    small two-level tree (GQA 2:1), match dq, dk, dv."""
    segs = [(5, -1), (3, 0), (4, 0), (2, 1)]
    T, Hq, Hkv, d = 14, 2, 1, 3
    q, k, v = _rand((T, Hq, d), 81), _rand((T, Hkv, d), 82), _rand((T, Hkv, d), 83)
    G = _rand((T, Hq, d), 84).double().numpy()
    scale = 0.7
    dq, dk, dv = oracle.prefill_bwd(q, k, v, torch.from_numpy(G).float(), segs, scale, lib=lib)
    # G is rounded to fp32 by the call; use the same values for the loss
    G = torch.from_numpy(G).float().double().numpy()
    eps = 1e-2

    def loss(qq, kk, vv):
        o, _ = oracle.prefill(qq, kk, vv, segs, scale, lib=lib)
        return float((o * G).sum())

    ok = True
    for name, base, grad in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        flat = base.float().numpy().reshape(-1)
        for i in range(flat.size):
            up, dn = flat.copy(), flat.copy()
            up[i] += np.float32(eps)
            dn[i] -= np.float32(eps)
            args = {"q": q, "k": k, "v": v}
            args[name] = torch.from_numpy(up.reshape(base.shape))
            lu = loss(args["q"], args["k"], args["v"])
            args[name] = torch.from_numpy(dn.reshape(base.shape))
            ld = loss(args["q"], args["k"], args["v"])
            # divide by the step the fp32 inputs actually took
            fd = (lu - ld) / (float(up[i]) - float(dn[i]))
            ok &= abs(fd - grad.reshape(-1)[i]) < 1e-4 * max(1.0, abs(fd))
    return bool(ok)


def pin_backward_gradient_equivalence(lib):
    """[PS] test plan (gradient equivalence): the flat layout's gradients
    equal those of running each [prefix; s_i] on its own with ordinary causal
    attention (torch autograd in fp64), the prefix collecting the gradients of
    every suffix; each copy carries 1/N of the prefix rows' upstream
    gradient so that the summed losses equal the flat loss."""
    P, N, S, Hq, Hkv, d = 9, 3, 5, 4, 2, 8
    T = P + N * S
    q, k, v = _rand((T, Hq, d), 91), _rand((T, Hkv, d), 92), _rand((T, Hkv, d), 93)
    G = _rand((T, Hq, d), 94)
    scale = 1 / math.sqrt(d)
    dq, dk, dv = oracle.prefill_bwd(q, k, v, G, W.grpo_segments(P, N, S), scale, lib=lib)
    qd = q.double().requires_grad_(True)
    kd = k.double().requires_grad_(True)
    vd = v.double().requires_grad_(True)
    total = 0.0
    for i in range(N):
        sl = list(range(P)) + list(range(P + i * S, P + (i + 1) * S))
        qi, ki, vi = qd[sl], _expand_kv(kd[sl], Hq), _expand_kv(vd[sl], Hq)
        o = F.scaled_dot_product_attention(qi.permute(1, 0, 2)[None], ki.permute(1, 0, 2)[None],
                                           vi.permute(1, 0, 2)[None], is_causal=True,
                                           scale=scale)[0].permute(1, 0, 2)
        w = G.double()[sl].clone()
        w[:P] /= N
        total = total + (o * w).sum()
    total.backward()
    ok = (np.allclose(dq, qd.grad.numpy(), atol=1e-12) and
          np.allclose(dk, kd.grad.numpy(), atol=1e-12) and
          np.allclose(dv, vd.grad.numpy(), atol=1e-12))
    # the row-sampled dq agrees with the full backward
    rows = np.array([0, P - 1, P, T - 1, P + S + 2], dtype=np.int32)
    dqs = oracle.prefill_bwd_dq(q, k, v, G, W.grpo_segments(P, N, S), scale, rows, lib=lib)
    ok &= np.allclose(dqs, dq[rows], atol=1e-12)
    return bool(ok)


PINS = [pin_golden_masks, pin_golden_tiny_attention, pin_equivalence_route,
        pin_sdpa_random_trees, pin_closed_forms, pin_special_cases,
        pin_brute_force_python, pin_verify_against_sdpa, pin_split_identity,
        pin_verify_tree_mask, pin_verify_extend_form, pin_verify_shared_prefix, pin_e4m3_decoder, pin_verify_fp8_cache,
        pin_backward_finite_differences, pin_backward_gradient_equivalence, pin_sparse_latent]


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_oracle_pin(pin):
    assert pin(oracle.load())


# Planted mistakes (compile-time switches in oracle.c), each of which some
# pin above must catch: 1 drops the scale, 2 makes causality strict,
# 3 interleaves GQA heads, 4 hides the prefix from suffixes, 5 drops the
# row maximum from the LSE, 6 makes the draft block non-causal, 7 ignores
# the verify's page table, 8 drops D = rowsum(dO * O) from dS, 9 drops the
# scale from dk, 10 decodes e4m3 with exponent bias 8, 11 drops v_scale from
# the fp8 cache's values, 12 takes latent row 0 for a pad, 13 shortens the
# shared prefix by one token.
@pytest.mark.parametrize("mutant", list(range(1, 14)))
def test_planted_mistake_is_caught(mutant, tmp_path):
    path = oracle.build(mutant=mutant, out=str(tmp_path / f"liboracle_m{mutant}.so"))
    lib = oracle.load(path)
    results = {p.__name__: p(lib) for p in PINS}
    assert not all(results.values()), f"mutant {mutant} passed every pin"


def test_sparse_indices_are_valid():
    """The generator's index lists: sorted, distinct, in the causal past,
    dense for t < topk (input recipe reading of [MLA] environment)."""
    wl = W.SparseLatentWorkload("t", T=300, H=1, dl=8, topk=64, seed=3)
    _, _, idx = wl.make()
    for t in range(300):
        row = idx[t][idx[t] >= 0]
        assert len(row) == min(t + 1, 64)
        assert bool(torch.all(row[1:] > row[:-1]))
        assert int(row.max()) <= t
        if t < 64:
            assert torch.equal(row, torch.arange(t + 1, dtype=torch.int32))


def test_pair_counts_closed_form():
    """Visible pairs per head: the workload's closed form equals the count of
    the oracle's visibility matrix."""
    for P, N, S, groups in [(64, 4, 32, 1), (7, 3, 5, 2), (0, 3, 4, 1)]:
        wl = W.PrefillWorkload("t", P=P, N=N, S=S, Hq=1, Hkv=1, d=8, groups=groups)
        vis = oracle.visibility(wl.segments())
        assert int(vis.sum()) == wl.visible_pairs_per_head()
    assert W.GRPO.visible_pairs_per_head() == 11_537_408
    assert W.LARGE.visible_pairs_per_head() == 352_346_112
    assert W.SPARSE.pairs() == 31_458_304


def test_sparse_oracle_refuses_indices_outside_the_latent():
    """An index list entry must name a latent row or be the -1 pad: the
    checker refuses anything else instead of reading past its buffer."""
    wl = W.SparseLatentWorkload("t", T=20, H=2, dl=16, topk=8, seed=4)
    q, lat, idx = wl.make()
    oracle.sparse_latent(q, lat, idx, wl.scale)          # valid lists pass
    for bad_val in (lat.shape[0], 10_000, -2):
        bad = idx.clone()
        bad[13, 2] = bad_val
        with pytest.raises(ValueError):
            oracle.sparse_latent(q, lat, bad, wl.scale)
        # a row sample that skips the bad row is still served
        o, _ = oracle.sparse_latent(q, lat, bad, wl.scale, rows=[0, 12, 19])
        assert np.isfinite(o).all()
    with pytest.raises(ValueError):
        oracle.sparse_latent(q, lat, idx, wl.scale, rows=[20])
