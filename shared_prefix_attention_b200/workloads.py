"""Seeded synthetic inputs shaped like the workloads on the pages.

This module draws random numbers and lays out shapes; it holds none of the
attention arithmetic, so both the CUDA path and the fp64 oracle can consume
what it produces (the same bytes go to both sides).

Workloads (sizes as named; Q/K/V ~ N(0,1) * sigma, rounded once to the
storage dtype):

* ``tiny``   -- one prefix P=64 plus N=4 suffixes of S=32, 2 heads, d=64, fp32.
* ``grpo``   -- GRPO rollout group P=2048, N=8, S=512, 16/16 heads, d=128, bf16.
* ``large``  -- two packed groups of P=8192, N=16, S=1024, 32 query heads on
  8 KV heads, d=128, bf16.
* ``verify`` -- 32 requests, 16384-token cached prefix each, 4 draft tokens,
  32 query / 8 KV heads, d=128, 32 splits, bf16.
* ``verify-fp8`` -- the verify workload with the cached prefix stored as e4m3
  codes and per-tensor scales k_scale = 1/96, v_scale = 1/80.
* ``verify-shared`` -- the same 32 requests with 4 drafts each, all sharing
  one 16384-token cached prefix stored once, 32/8 heads, d=128, bf16.
* ``sparse`` -- 16384 queries, 64 heads on one 512-wide latent, 2048 indices
  per query drawn from its causal past, bf16.

The flat GRPO layout and the tree segments follow "KV-0 redundancy prefix
sharing attention mask design" (design summary; key changes section 2).
The verify shape follows "Split-KV flash-decode attention for EAGLE
target-verify" (motivation: 16k context; test shapes: 4 draft tokens).
The sparse shape follows "SM8x sparse-MLA prefill fallback re-reads the
shared MLA latent once per head" (environment: 16384 tokens, 64 heads,
index_topk 2048, kv_lora_rank 512, no rope part).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch


# --------------------------------------------------------------------------
# segment trees
# --------------------------------------------------------------------------

def grpo_segments(P: int, N: int, S: int, groups: int = 1) -> list[tuple[int, int]]:
    """(len, parent) per segment in flat order: for each group, the prefix
    (a root) followed by N suffixes whose parent is that prefix.  A group
    with P == 0 has no prefix segment: its N suffixes are roots."""
    segs: list[tuple[int, int]] = []
    for _ in range(groups):
        if P > 0:
            root = len(segs)
            segs.append((P, -1))
            segs.extend((S, root) for _ in range(N))
        else:
            segs.extend((S, -1) for _ in range(N))
    return segs


def chain_segments(lens: list[int]) -> list[tuple[int, int]]:
    """A chain: segment i's parent is segment i-1."""
    return [(n, i - 1) for i, n in enumerate(lens)]


def random_tree_segments(gen: torch.Generator, nseg: int, max_len: int,
                         groups: int = 1) -> list[tuple[int, int]]:
    """A random forest in flat order (parents precede children)."""
    segs: list[tuple[int, int]] = []
    for _ in range(groups):
        base = len(segs)
        for i in range(nseg):
            ln = int(torch.randint(1, max_len + 1, (1,), generator=gen))
            if i == 0:
                par = -1
            else:
                par = int(torch.randint(-1, i, (1,), generator=gen))
                par = -1 if par < 0 else base + par
            segs.append((ln, par))
    return segs


def group_indptr(segments, segs_per_group: list[int]) -> list[int]:
    out = [0]
    for n in segs_per_group:
        out.append(out[-1] + n)
    return out


# --------------------------------------------------------------------------
# workloads
# --------------------------------------------------------------------------

@dataclass
class PrefillWorkload:
    name: str
    P: int
    N: int
    S: int
    Hq: int
    Hkv: int
    d: int
    groups: int = 1
    dtype: torch.dtype = torch.bfloat16
    sigma: float = 0.5
    seed: int = 2

    @property
    def group_len(self) -> int:
        return self.P + self.N * self.S

    @property
    def T(self) -> int:
        return self.groups * self.group_len

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    def segments(self):
        return grpo_segments(self.P, self.N, self.S, self.groups)

    def seg_indptr(self) -> list[int]:
        per = (self.N + 1) if self.P > 0 else self.N
        return [g * per for g in range(self.groups + 1)]

    def cu_seqlens(self) -> list[int]:
        return [g * self.group_len for g in range(self.groups + 1)]

    def visible_pairs_per_head(self) -> int:
        """Exact visible (q, k) pairs per query head (closed form for the
        flat GRPO tree): causal prefix plus, per suffix, the whole prefix and
        its own causal triangle."""
        P, N, S = self.P, self.N, self.S
        per_group = P * (P + 1) // 2 + N * (S * P + S * (S + 1) // 2)
        return self.groups * per_group

    def flops(self) -> float:
        """4 * d * Hq * visible pairs (QK^T and PV, 2 flops per MAC)."""
        return 4.0 * self.d * self.Hq * self.visible_pairs_per_head()

    def make(self, device="cpu", seed: int | None = None):
        g = torch.Generator(device=device)
        g.manual_seed(self.seed if seed is None else seed)
        T = self.T

        def draw(shape):
            x = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
            return (x * self.sigma).to(self.dtype)

        q = draw((T, self.Hq, self.d))
        k = draw((T, self.Hkv, self.d))
        v = draw((T, self.Hkv, self.d))
        return q, k, v


@dataclass
class VerifyWorkload:
    name: str
    B: int
    L: int
    Ld: int
    Hq: int
    Hkv: int
    d: int
    nsplit: int
    dtype: torch.dtype = torch.bfloat16
    sigma: float = 0.5
    seed: int = 4
    prefix_lens: list[int] | None = None   # ragged prefixes (default: all L)

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    def lens(self) -> list[int]:
        return list(self.prefix_lens) if self.prefix_lens is not None else [self.L] * self.B

    def kv_indptr(self) -> list[int]:
        out = [0]
        for n in self.lens():
            out.append(out[-1] + n)
        return out

    def prefix_kv_bytes(self) -> int:
        """Prefix K and V bytes read once: sum(L_b) * Hkv * d * 2 tensors * elem."""
        elem = torch.tensor([], dtype=self.dtype).element_size()
        return sum(self.lens()) * self.Hkv * self.d * 2 * elem

    def make(self, device="cpu", seed: int | None = None):
        g = torch.Generator(device=device)
        g.manual_seed(self.seed if seed is None else seed)
        ntok = sum(self.lens())
        BL = self.B * self.Ld

        def draw(shape):
            x = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
            return (x * self.sigma).to(self.dtype)

        q = draw((BL, self.Hq, self.d))
        kd = draw((BL, self.Hkv, self.d))
        vd = draw((BL, self.Hkv, self.d))
        kc = draw((ntok, self.Hkv, self.d))
        vc = draw((ntok, self.Hkv, self.d))
        return q, kd, vd, kc, vc

    # per-tensor scales of the fp8 cache: stored codes are value / scale
    k_scale: float = 1.0 / 96
    v_scale: float = 1.0 / 80

    def make_fp8(self, device="cpu", seed: int | None = None):
        """As make(), with the cached prefix stored as e4m3 codes (uint8) of
        value / k_scale and value / v_scale (round to nearest)."""
        q, kd, vd, kc, vc = self.make(device, seed)
        kc8 = (kc.float() / self.k_scale).to(torch.float8_e4m3fn).view(torch.uint8)
        vc8 = (vc.float() / self.v_scale).to(torch.float8_e4m3fn).view(torch.uint8)
        return q, kd, vd, kc8, vc8

    def prefix_fp8_bytes(self) -> int:
        """Prefix K and V bytes of the e4m3 cache, read once."""
        return sum(self.lens()) * self.Hkv * self.d * 2


@dataclass
class SharedVerifyWorkload:
    """Speculative verify where all B requests share one cached prefix of L
    tokens (stored once) and each has Ld draft tokens."""
    name: str
    B: int
    L: int
    Ld: int
    Hq: int
    Hkv: int
    d: int
    nsplit: int = 0          # 0: the library's automatic choice
    dtype: torch.dtype = torch.bfloat16
    sigma: float = 0.5
    seed: int = 6

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    def flops(self) -> float:
        """4 d FLOP per (draft row, query head, visible key): the whole
        prefix plus drafts 0..j for draft j."""
        keys = self.B * (self.Ld * self.L + self.Ld * (self.Ld + 1) // 2)
        return 4.0 * self.d * self.Hq * keys

    def prefix_kv_bytes(self) -> int:
        """Prefix K and V bytes, read once for all requests."""
        elem = torch.tensor([], dtype=self.dtype).element_size()
        return self.L * self.Hkv * self.d * 2 * elem

    def make(self, device="cpu", seed: int | None = None):
        g = torch.Generator(device=device)
        g.manual_seed(self.seed if seed is None else seed)
        BL = self.B * self.Ld

        def draw(shape):
            x = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
            return (x * self.sigma).to(self.dtype)

        q = draw((BL, self.Hq, self.d))
        kd = draw((BL, self.Hkv, self.d))
        vd = draw((BL, self.Hkv, self.d))
        kp = draw((self.L, self.Hkv, self.d))
        vp = draw((self.L, self.Hkv, self.d))
        return q, kd, vd, kp, vp


@dataclass
class ExtendVerifyWorkload:
    """Speculative verify in the extend form: per-request draft counts, each
    request's prefix scattered over a token-granular KV pool through a page
    table (distinct random pool rows), and optionally a random draft tree per
    request (draft j's parent drawn uniformly from the prefix and drafts
    0..j-1; a draft sees its ancestors and itself)."""
    name: str
    draft_lens: list[int]
    prefix_lens: list[int]
    Hq: int
    Hkv: int
    d: int
    nsplit: int = 0
    tree: bool = True
    pool_slack: float = 1.25     # pool rows per prefix token
    dtype: torch.dtype = torch.bfloat16
    sigma: float = 0.5
    seed: int = 8

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    @property
    def B(self) -> int:
        return len(self.draft_lens)

    @property
    def n_rows(self) -> int:
        return sum(self.draft_lens)

    @property
    def max_draft_len(self) -> int:
        return max(self.draft_lens + [1])

    @property
    def max_prefix_len(self) -> int:
        return max(self.prefix_lens + [0])

    @staticmethod
    def _indptr(xs) -> list[int]:
        out = [0]
        for n in xs:
            out.append(out[-1] + n)
        return out

    def qo_indptr(self) -> list[int]:
        return self._indptr(self.draft_lens)

    def kv_indptr(self) -> list[int]:
        return self._indptr(self.prefix_lens)

    def mask_indptr(self) -> list[int]:
        return self._indptr([n * n for n in self.draft_lens])

    def pool_rows(self) -> int:
        return max(1, int(sum(self.prefix_lens) * self.pool_slack))

    def prefix_kv_bytes(self) -> int:
        elem = torch.tensor([], dtype=self.dtype).element_size()
        return sum(self.prefix_lens) * self.Hkv * self.d * 2 * elem

    def make(self, device="cpu", seed: int | None = None):
        """q, k_draft, v_draft [n_rows, H, d]; k_pool, v_pool [pool rows,
        Hkv, d]; kv_indices int32 [sum prefix]; draft mask uint8 (flat, the
        requests' Lb x Lb blocks in order) or None."""
        g = torch.Generator(device="cpu")
        g.manual_seed(self.seed if seed is None else seed)

        def draw(shape):
            x = torch.randn(shape, generator=g, dtype=torch.float32)
            return (x * self.sigma).to(self.dtype).to(device)

        NR = self.n_rows
        q = draw((NR, self.Hq, self.d))
        kd = draw((NR, self.Hkv, self.d))
        vd = draw((NR, self.Hkv, self.d))
        npool = self.pool_rows()
        kp = draw((npool, self.Hkv, self.d))
        vp = draw((npool, self.Hkv, self.d))
        idx = torch.randperm(npool, generator=g)[:sum(self.prefix_lens)].to(torch.int32)
        mask = None
        if self.tree:
            blocks = []
            for n in self.draft_lens:
                m = torch.zeros((n, n), dtype=torch.uint8)
                parent = []
                for j in range(n):
                    # -1 is the prefix (a root draft); else an earlier draft
                    parent.append(int(torch.randint(-1, j, (1,), generator=g)) if j else -1)
                    a = j
                    while a >= 0:
                        m[j, a] = 1
                        a = parent[a]
                blocks.append(m.reshape(-1))
            mask = torch.cat(blocks) if blocks else torch.zeros(0, dtype=torch.uint8)
            mask = mask.to(device)
        return q, kd, vd, kp, vp, idx.to(device), mask


@dataclass
class SparseLatentWorkload:
    name: str
    T: int
    H: int
    dl: int
    topk: int
    dtype: torch.dtype = torch.bfloat16
    sigma: float = 0.5
    seed: int = 5

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.dl)

    def pairs(self) -> int:
        return sum(min(t + 1, self.topk) for t in range(self.T))

    def flops(self) -> float:
        return 4.0 * self.dl * self.H * self.pairs()

    def make_indices(self, g: torch.Generator, device="cpu") -> torch.Tensor:
        """[T, topk] int32.  Row t < topk lists 0..t then -1 padding (dense
        causal); row t >= topk lists topk distinct positions drawn uniformly
        without replacement from [0, t], sorted ascending."""
        T, K = self.T, self.topk
        idx = torch.full((T, K), -1, dtype=torch.int32, device=device)
        dense = min(T, K)
        ar = torch.arange(K, device=device, dtype=torch.int32)
        tri = torch.where(ar[None, :] <= torch.arange(dense, device=device,
                                                       dtype=torch.int32)[:, None],
                          ar[None, :], torch.full_like(ar[None, :], -1))
        idx[:dense] = tri
        block = 256
        for r0 in range(K, T, block):
            r1 = min(T, r0 + block)
            width = r1  # positions 0 .. r1-1 cover every row's causal past
            u = torch.rand((r1 - r0, width), generator=g, device=device)
            pos = torch.arange(width, device=device)
            rows = torch.arange(r0, r1, device=device)
            u = torch.where(pos[None, :] <= rows[:, None], u, torch.full_like(u, -1.0))
            pick = torch.topk(u, K, dim=1).indices
            idx[r0:r1] = torch.sort(pick, dim=1).values.to(torch.int32)
        return idx

    def make(self, device="cpu", seed: int | None = None):
        g = torch.Generator(device=device)
        g.manual_seed(self.seed if seed is None else seed)

        def draw(shape):
            x = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
            return (x * self.sigma).to(self.dtype)

        q = draw((self.T, self.H, self.dl))
        lat = draw((self.T, self.dl))
        idx = self.make_indices(g, device)
        return q, lat, idx


TINY = PrefillWorkload("tiny P=64 N=4 S=32 H=2 d=64 fp32", P=64, N=4, S=32, Hq=2, Hkv=2,
                       d=64, dtype=torch.float32, sigma=1.0, seed=1)
GRPO = PrefillWorkload("grpo P=2048 N=8 S=512 H=16/16 d=128 bf16", P=2048, N=8, S=512,
                       Hq=16, Hkv=16, d=128, seed=2)
LARGE = PrefillWorkload("large 2x(P=8192 N=16 S=1024) H=32/8 d=128 bf16", P=8192, N=16,
                        S=1024, Hq=32, Hkv=8, d=128, groups=2, seed=3)
VERIFY = VerifyWorkload("verify B=32 L=16384 drafts=4 H=32/8 d=128 splits=32 bf16", B=32,
                        L=16384, Ld=4, Hq=32, Hkv=8, d=128, nsplit=32, seed=4)
VERIFY_FP8 = VerifyWorkload("verify-fp8 B=32 L=16384 drafts=4 H=32/8 d=128 splits=32 e4m3 cache",
                            B=32, L=16384, Ld=4, Hq=32, Hkv=8, d=128, nsplit=32, seed=7)
VERIFY_SHARED = SharedVerifyWorkload("verify-shared B=32 L=16384 drafts=4 H=32/8 d=128 bf16",
                                     B=32, L=16384, Ld=4, Hq=32, Hkv=8, d=128, seed=6)
SPARSE = SparseLatentWorkload("sparse T=16384 H=64 dl=512 topk=2048 bf16", T=16384, H=64,
                              dl=512, topk=2048, seed=5)
VERIFY_PAGED = ExtendVerifyWorkload(
    "verify-extend B=32 L=16384 drafts 1..8 trees, token-granular page table H=32/8 d=128 bf16",
    draft_lens=[1 + (5 * b) % 8 for b in range(32)], prefix_lens=[16384] * 32, Hq=32, Hkv=8,
    d=128, nsplit=32, seed=8)
