"""Benchmark of the shared-prefix attention hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                    [--impl psa|reference] [--no-extras]

One JSON line on rank 0.  The headline workload is the GRPO rollout group
(P=2048, N=8, S=512, 16/16 heads, d=128, bf16): metric = visible-block
attention TFLOP/s (exact visible-pair FLOPs, 4*d*Hq*pairs) over the flat
packed layout.  With extras on (default) the line also carries the
speculative-verify prefix-KV GB/s, the large two-group prefill and the
shared-latent sparse prefill, each device-timed the same way.

Timing: W untimed warm-up steps, then K steps, each bracketed by CUDA
events on the launching stream, with an L2 flush (a 256 MiB write) between
steps outside the events; barrier + synchronize around the whole region;
max over ranks.  N > 1 runs independent replicas (weak scaling): the path
has no exchange step.  ``--impl reference`` times the fp64 CPU oracle on the
host cores on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from shared_prefix_attention_b200 import workloads as W  # noqa: E402

METRIC = "visible-block attn TFLOP/s; verify prefix-KV GB/s; both as % of B200 roofline"
L2_FLUSH_BYTES = 256 << 20


# --------------------------------------------------------------------------- utils

def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained"), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


def kernel_source_hash(name: str) -> str:
    path = os.path.join(ROOT, "shared_prefix_attention_b200", "csrc", name)
    h = hashlib.sha256()
    for p in (path, os.path.join(ROOT, "shared_prefix_attention_b200", "csrc", "psa_device.cuh")):
        with open(p, "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def traffic_for(kernel_file: str, key: str):
    """DRAM bytes per launch from a committed ncu capture, or None when the
    capture is missing or the kernel source changed since it was taken."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f)
    e = d.get(key)
    if not e or e.get("source_hash") != kernel_source_hash(kernel_file):
        return None
    return e.get("dram_bytes_per_launch")


class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML while running."""

    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x2: "applications_clocks_setting"}

    def __init__(self, device_index: int, period_s: float = 0.001):
        self.samples = []
        self.max_mhz = None
        self._stop = threading.Event()
        self._period = period_s
        self._thread = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            vis = os.environ.get("CUDA_VISIBLE_DEVICES")
            idx = device_index
            if vis:
                ids = [x for x in vis.split(",") if x.strip()]
                if ids and ids[device_index].strip().isdigit():
                    idx = int(ids[device_index])
            self._h = pynvml.nvmlDeviceGetHandleByIndex(idx)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self._nv = None

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                mhz = nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM)
                rs = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                self.samples.append((mhz, rs))
            except Exception:
                pass
            time.sleep(self._period)

    def __enter__(self):
        if self._nv is not None:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._thread:
            self._thread.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [],
                    "samples": 0, "note": "NVML unavailable"}
        mhz = sorted(s[0] for s in self.samples)
        bits = 0
        for _, r in self.samples:
            bits |= int(r)
        reasons = [n for b, n in self.REASONS.items() if bits & b]
        return {"sm_mhz": mhz[len(mhz) // 2], "sm_max_mhz": self.max_mhz, "reasons": reasons,
                "samples": len(self.samples)}


def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


# --------------------------------------------------------------------------- workloads

class Runner:
    """One workload: inputs resident on the device, one step = one call of
    the public C-ABI entry point, algorithmic work per step."""
    name = ""
    unit = ""
    kernels_per_step = 1
    bound = "tensor"
    kernel_file = ""

    def work(self) -> float: ...
    def step(self): ...


class PrefillRunner(Runner):
    unit = "TFLOP/s"
    bound = "tensor"
    kernel_file = "psa_prefill.cu"

    def __init__(self, wl: W.PrefillWorkload, dev):
        import shared_prefix_attention_b200 as psa
        self.psa, self.wl, self.dev = psa, wl, dev
        self.name = wl.name
        self.q, self.k, self.v = wl.make(dev)
        self.sched = psa.plan_prefill(wl.segments(), wl.cu_seqlens(), wl.d, dev)
        self.o = torch.empty_like(self.q)
        self.lse = torch.empty((wl.T, wl.Hq), dtype=torch.float32, device=dev)
        n = psa.lib().psa_prefill_workspace_size(0 if wl.dtype == torch.bfloat16 else 1, wl.T,
                                                 wl.Hq, wl.Hkv, wl.d)
        self.ws = torch.empty(n, dtype=torch.uint8, device=dev)
        self.kernels_per_step = 1 if wl.dtype == torch.bfloat16 else 4

    def work(self):
        return self.wl.flops()

    def step(self):
        self.psa.prefill(self.q, self.k, self.v, self.sched, self.wl.scale, out=self.o,
                         lse=self.lse, workspace=self.ws)

    # end to end: host (pinned) inputs in, O and LSE back to the host
    def e2e_setup(self):
        self.hq, self.hk, self.hv = (t.cpu().pin_memory() for t in (self.q, self.k, self.v))
        self.ho = torch.empty(self.o.shape, dtype=self.o.dtype).pin_memory()
        self.hl = torch.empty(self.lse.shape, dtype=torch.float32).pin_memory()
        self.h2d = sum(t.numel() * t.element_size() for t in (self.hq, self.hk, self.hv))
        self.d2h = self.ho.numel() * self.ho.element_size() + self.hl.numel() * 4

    def e2e_step(self):
        self.q.copy_(self.hq, non_blocking=True)
        self.k.copy_(self.hk, non_blocking=True)
        self.v.copy_(self.hv, non_blocking=True)
        self.step()
        self.ho.copy_(self.o, non_blocking=True)
        self.hl.copy_(self.lse, non_blocking=True)

    def oracle_sample(self, budget_s: float):
        """(work done, seconds) of the oracle on a bounded row sample."""
        import oracle
        wl = self.wl
        q, k, v = (t.cpu() for t in (self.q, self.k, self.v))
        vis_per_row = None
        rows = []
        # rows spread over every segment, the last rows of each group first
        # (the longest ones), grown until the budget is used
        g = torch.Generator().manual_seed(0)
        perm = torch.randperm(wl.T, generator=g).tolist()
        t0 = time.perf_counter()
        done_flops = 0.0
        segs = wl.segments()
        start, lens, parent = oracle.segment_arrays(segs)
        seg_of = {}
        for s_i, (a, n) in enumerate(zip(start, lens)):
            for t in range(a, a + n):
                seg_of[t] = s_i
        chunk = 8
        i = 0
        while time.perf_counter() - t0 < budget_s and i < len(perm):
            rows = perm[i:i + chunk]
            i += chunk
            oracle.prefill(q, k, v, segs, wl.scale, rows=rows)
            for r in rows:
                s_i = seg_of[r]
                cnt = r - int(start[s_i]) + 1
                p = int(parent[s_i])
                while p >= 0:
                    cnt += int(lens[p])
                    p = int(parent[p])
                done_flops += 4.0 * wl.d * wl.Hq * cnt
        return done_flops, time.perf_counter() - t0, f"{i} random query rows x {wl.Hq} heads"


class VerifyRunner(Runner):
    unit = "GB/s"
    bound = "hbm"
    kernels_per_step = 2
    kernel_file = "psa_verify.cu"

    def __init__(self, wl: W.VerifyWorkload, dev):
        import shared_prefix_attention_b200 as psa
        self.psa, self.wl, self.dev = psa, wl, dev
        self.name = wl.name
        self.q, self.kd, self.vd, self.kc, self.vc = wl.make(dev)
        self.indptr = torch.tensor(wl.kv_indptr(), dtype=torch.int32, device=dev)
        self.o = torch.empty_like(self.q)
        self.lse = torch.empty(self.q.shape[:2], dtype=torch.float32, device=dev)
        n = psa.verify_workspace_size(wl.B, wl.Ld, wl.Hq, wl.d, wl.nsplit)
        self.ws = torch.empty(n, dtype=torch.uint8, device=dev)

    def work(self):
        return float(self.wl.prefix_kv_bytes())

    def step(self):
        wl = self.wl
        self.psa.verify(self.q, self.kd, self.vd, self.kc, self.vc, self.indptr, wl.L, wl.scale,
                        wl.Ld, nsplit=wl.nsplit, out=self.o, lse=self.lse, workspace=self.ws)

    def e2e_setup(self):
        ts = (self.q, self.kd, self.vd, self.kc, self.vc)
        self.hin = [t.cpu().pin_memory() for t in ts]
        self.ho = torch.empty(self.o.shape, dtype=self.o.dtype).pin_memory()
        self.hl = torch.empty(self.lse.shape, dtype=torch.float32).pin_memory()
        self.h2d = sum(t.numel() * t.element_size() for t in self.hin)
        self.d2h = self.ho.numel() * self.ho.element_size() + self.hl.numel() * 4

    def e2e_step(self):
        for d, h in zip((self.q, self.kd, self.vd, self.kc, self.vc), self.hin):
            d.copy_(h, non_blocking=True)
        self.step()
        self.ho.copy_(self.o, non_blocking=True)
        self.hl.copy_(self.lse, non_blocking=True)

    def oracle_sample(self, budget_s: float):
        import numpy as np
        import oracle
        wl = self.wl
        t0 = time.perf_counter()
        done, n = 0.0, 0
        per_row_bytes = wl.L * wl.Hkv * wl.d * 2 * 2 / wl.Ld  # prefix bytes per draft row
        b = 0
        while time.perf_counter() - t0 < budget_s and b < wl.B:
            p0, p1 = b * wl.L, (b + 1) * wl.L
            sl = slice(b * wl.Ld, (b + 1) * wl.Ld)
            oracle.verify(self.q[sl].cpu(), self.kd[sl].cpu(), self.vd[sl].cpu(),
                          self.kc[p0:p1].cpu(), self.vc[p0:p1].cpu(),
                          np.array([0, wl.L], dtype=np.int64), wl.Ld, wl.scale)
            done += per_row_bytes * wl.Ld
            n += 1
            b += 1
        return done, time.perf_counter() - t0, f"{n} whole requests ({n * wl.Ld} draft rows)"


class SparseRunner(Runner):
    unit = "TFLOP/s"
    bound = "tensor"
    kernel_file = "psa_sparse.cu"

    def __init__(self, wl: W.SparseLatentWorkload, dev):
        import shared_prefix_attention_b200 as psa
        self.psa, self.wl, self.dev = psa, wl, dev
        self.name = wl.name
        self.q, self.lat, self.idx = wl.make(dev)
        self.o = torch.empty_like(self.q)
        self.lse = torch.empty((wl.T, wl.H), dtype=torch.float32, device=dev)

    def work(self):
        return self.wl.flops()

    def step(self):
        self.psa.sparse_latent(self.q, self.lat, self.idx, self.wl.scale, out=self.o,
                               lse=self.lse)


class BackwardRunner(Runner):
    """Prefill backward (dq, dk, dv) of the GRPO group; the forward outputs
    are computed once outside the timed region."""
    unit = "TFLOP/s"
    bound = "tensor"
    kernels_per_step = 3
    kernel_file = "psa_backward.cu"

    def __init__(self, wl: W.PrefillWorkload, dev):
        import shared_prefix_attention_b200 as psa
        self.psa, self.wl, self.dev = psa, wl, dev
        self.name = wl.name.replace("grpo", "grpo-backward", 1)
        self.q, self.k, self.v = wl.make(dev)
        g = torch.Generator(device=dev)
        g.manual_seed(wl.seed + 100)
        self.dout = (torch.randn(self.q.shape, generator=g, device=dev) * wl.sigma).to(self.q.dtype)
        sched = psa.plan_prefill(wl.segments(), wl.cu_seqlens(), wl.d, dev)
        self.o, self.lse = psa.prefill(self.q, self.k, self.v, sched, wl.scale)
        self.scheds = psa.plan_prefill_bwd(wl.segments(), wl.cu_seqlens(), wl.d, dev)
        self.dq, self.dk, self.dv = (torch.empty_like(t) for t in (self.q, self.k, self.v))
        n = int(psa.lib().psa_prefill_bwd_workspace_size(wl.T, wl.Hq))
        self.ws = torch.empty(n, dtype=torch.uint8, device=dev)

    def work(self):
        # five products of the visible pairs (S, dP, dV, dQ, dK), 2 d FLOP each
        return self.wl.flops() * 10.0 / 4.0

    def step(self):
        self.psa.prefill_bwd(self.q, self.k, self.v, self.o, self.lse, self.dout, self.scheds,
                             self.wl.scale, dq=self.dq, dk=self.dk, dv=self.dv,
                             workspace=self.ws)


class VerifyFp8Runner(Runner):
    """Split-KV verify over an e4m3 prefix cache: HBM-bound on the cache bytes
    (one byte per element)."""
    unit = "GB/s"
    bound = "hbm"
    kernels_per_step = 2
    kernel_file = "psa_verify_fp8.cu"

    def __init__(self, wl: W.VerifyWorkload, dev):
        import shared_prefix_attention_b200 as psa
        self.psa, self.wl, self.dev = psa, wl, dev
        self.name = wl.name
        self.q, self.kd, self.vd, self.kc8, self.vc8 = wl.make_fp8(dev)
        self.indptr = torch.tensor(wl.kv_indptr(), dtype=torch.int32, device=dev)
        self.o = torch.empty_like(self.q)
        self.lse = torch.empty(self.q.shape[:2], dtype=torch.float32, device=dev)
        n = psa.verify_workspace_size(wl.B, wl.Ld, wl.Hq, wl.d, wl.nsplit)
        self.ws = torch.empty(n, dtype=torch.uint8, device=dev)

    def work(self):
        return float(self.wl.prefix_fp8_bytes())

    def step(self):
        wl = self.wl
        self.psa.verify_fp8(self.q, self.kd, self.vd, self.kc8, self.vc8, wl.k_scale, wl.v_scale,
                            self.indptr, wl.L, wl.scale, wl.Ld, nsplit=wl.nsplit, out=self.o,
                            lse=self.lse, workspace=self.ws)


class SharedVerifyRunner(Runner):
    """Verify against one prefix shared by all requests: tensor-bound (the
    stacked draft rows of a KV head multiply the prefix once)."""
    unit = "TFLOP/s"
    bound = "tensor"
    kernels_per_step = 2
    kernel_file = "psa_verify_shared.cu"

    def __init__(self, wl: W.SharedVerifyWorkload, dev):
        import shared_prefix_attention_b200 as psa
        self.psa, self.wl, self.dev = psa, wl, dev
        self.name = wl.name
        self.q, self.kd, self.vd, self.kp, self.vp = wl.make(dev)
        self.o = torch.empty_like(self.q)
        self.lse = torch.empty(self.q.shape[:2], dtype=torch.float32, device=dev)
        self.ns = wl.nsplit or psa.verify_shared_auto_splits(wl.B, wl.Ld, wl.Hq, wl.Hkv, wl.L)
        n = psa.verify_workspace_size(wl.B, wl.Ld, wl.Hq, wl.d, self.ns)
        self.ws = torch.empty(n, dtype=torch.uint8, device=dev)

    def work(self):
        return self.wl.flops()

    def step(self):
        wl = self.wl
        self.psa.verify_shared(self.q, self.kd, self.vd, self.kp, self.vp, wl.scale, wl.Ld,
                               nsplit=self.ns, out=self.o, lse=self.lse, workspace=self.ws)


class ExtendVerifyRunner(Runner):
    """Verify in the extend form: ragged drafts in trees, each prefix read
    through a token-granular page table (gathered with 16-byte copies)."""
    unit = "GB/s"
    bound = "hbm"
    kernels_per_step = 2
    kernel_file = "psa_verify.cu"

    def __init__(self, wl: W.ExtendVerifyWorkload, dev):
        import shared_prefix_attention_b200 as psa
        self.psa, self.wl, self.dev = psa, wl, dev
        self.name = wl.name
        q, kd, vd, kp, vp, idx, mask = wl.make("cpu")
        self.q, self.kd, self.vd, self.kp, self.vp, self.idx = (
            t.to(dev) for t in (q, kd, vd, kp, vp, idx))
        self.mask = None if mask is None else mask.to(dev)
        i32 = lambda xs: torch.tensor(xs, dtype=torch.int32, device=dev)  # noqa: E731
        self.qo, self.kvp, self.mi = i32(wl.qo_indptr()), i32(wl.kv_indptr()), i32(wl.mask_indptr())
        self.o = torch.empty_like(self.q)
        self.lse = torch.empty(self.q.shape[:2], dtype=torch.float32, device=dev)
        n = psa.verify_workspace_size(1, wl.n_rows, wl.Hq, wl.d, wl.nsplit)
        self.ws = torch.empty(n, dtype=torch.uint8, device=dev)

    def work(self):
        return float(self.wl.prefix_kv_bytes())

    def step(self):
        wl = self.wl
        self.psa.verify_extend(self.q, self.kd, self.vd, self.kp, self.vp, self.qo,
                               wl.max_draft_len, self.kvp, wl.max_prefix_len, wl.scale,
                               kv_indices=self.idx, draft_mask=self.mask,
                               mask_indptr=None if self.mask is None else self.mi,
                               nsplit=wl.nsplit, out=self.o, lse=self.lse, workspace=self.ws)

    def oracle_sample(self, budget_s: float):
        import numpy as np
        import oracle
        wl = self.wl
        qo, kvp = wl.qo_indptr(), wl.kv_indptr()
        host = [t.cpu() for t in (self.q, self.kd, self.vd, self.kp, self.vp, self.idx)]
        mask = None if self.mask is None else self.mask.cpu()
        t0 = time.perf_counter()
        done, n, b = 0.0, 0, 0
        per_tok = wl.Hkv * wl.d * 2 * 2  # prefix K and V bytes per token
        while time.perf_counter() - t0 < budget_s and b < wl.B:
            rows = np.arange(qo[b], qo[b + 1], dtype=np.int32)
            if len(rows):
                oracle.verify_extend(*host[:5], qo, kvp, wl.scale, kv_indices=host[5],
                                     draft_mask=mask,
                                     mask_indptr=None if mask is None else wl.mask_indptr(),
                                     rows=rows)
            done += per_tok * wl.prefix_lens[b]
            n += 1
            b += 1
        return done, time.perf_counter() - t0, f"{n} whole requests"


VERIFY_SMALL = W.VerifyWorkload("verify B=8 L=16384 drafts=4 H=32/8 d=128 splits=32 bf16", B=8,
                                L=16384, Ld=4, Hq=32, Hkv=8, d=128, nsplit=32, seed=4)
VERIFY_FP8_SMALL = W.VerifyWorkload(
    "verify-fp8 B=8 L=16384 drafts=4 H=32/8 d=128 splits=32 e4m3 cache", B=8, L=16384, Ld=4,
    Hq=32, Hkv=8, d=128, nsplit=32, seed=7)
VERIFY_PAGED_SMALL = W.ExtendVerifyWorkload(
    "verify-extend B=8 L=16384 drafts 1..8 trees, token-granular page table H=32/8 d=128 bf16",
    draft_lens=[1 + (5 * b) % 8 for b in range(8)], prefix_lens=[16384] * 8, Hq=32, Hkv=8, d=128,
    nsplit=32, seed=8)
SPARSE_SMALL = W.SparseLatentWorkload("sparse T=4096 H=64 dl=512 topk=2048 bf16", T=4096, H=64,
                                      dl=512, topk=2048, seed=5)


def make_runner(name: str, dev):
    return {"grpo": lambda: PrefillRunner(W.GRPO, dev),
            "verify8": lambda: VerifyRunner(VERIFY_SMALL, dev),
            "sparse4k": lambda: SparseRunner(SPARSE_SMALL, dev),
            "tiny": lambda: PrefillRunner(W.TINY, dev),
            "large": lambda: PrefillRunner(W.LARGE, dev),
            "verify": lambda: VerifyRunner(W.VERIFY, dev),
            "verify-shared": lambda: SharedVerifyRunner(W.VERIFY_SHARED, dev),
            "verify-fp8": lambda: VerifyFp8Runner(W.VERIFY_FP8, dev),
            "verify-fp8-8": lambda: VerifyFp8Runner(VERIFY_FP8_SMALL, dev),
            "verify-extend": lambda: ExtendVerifyRunner(W.VERIFY_PAGED, dev),
            "verify-extend8": lambda: ExtendVerifyRunner(VERIFY_PAGED_SMALL, dev),
            "grpo-backward": lambda: BackwardRunner(W.GRPO, dev),
            "sparse": lambda: SparseRunner(W.SPARSE, dev)}[name]()


# --------------------------------------------------------------------------- timing

def time_steps(fn, steps: int, warmup: int, flush: torch.Tensor, dist_on: bool):
    """Per-step CUDA-event times (ms) with an L2 flush between steps."""
    stream = torch.cuda.current_stream()
    for _ in range(warmup):
        flush.fill_(1)
        fn()
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    if dist_on:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    for i in range(steps):
        flush.fill_(i & 0xFF)
        starts[i].record(stream)
        fn()
        ends[i].record(stream)
    torch.cuda.synchronize()
    if dist_on:
        torch.distributed.barrier()
    return [s.elapsed_time(e) for s, e in zip(starts, ends)]


def max_over_ranks(x: float, dist_on: bool) -> float:
    """The slowest rank's time: every rank contributes its own and all get
    the maximum (NCCL on the GPUs; gloo keeps the tensor on the host)."""
    if not dist_on:
        return x
    on_gpu = torch.distributed.get_backend() == "nccl"
    t = torch.tensor([x], dtype=torch.float64, device="cuda" if on_gpu else "cpu")
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world: int, work_per_rank: float, ms_max: float, unit: str) -> float:
    """Weak scaling: every rank runs the same workload on its own GPU, so the
    job does world x work in the slowest rank's time."""
    scale = 1e12 if unit == "TFLOP/s" else 1e9
    return world * work_per_rank / (ms_max * 1e-3) / scale


def measure(runner, steps, warmup, flush, dist_on, world, peaks):
    per = time_steps(runner.step, steps, warmup, flush, dist_on)
    ms = max_over_ranks(sum(per) / len(per), dist_on)
    work = runner.work()
    value = job_throughput(world, work, ms, runner.unit)
    per_gpu = job_throughput(1, work, ms, runner.unit)
    if runner.bound == "tensor":
        peak = peaks["bf16_tflops"]
        unit = "TFLOP/s"
    else:
        peak = peaks["hbm_gbs"]
        unit = "GB/s"
    roof = {"bound": runner.bound, "achieved": round(per_gpu, 2), "peak": peak, "unit": unit,
            "frac": round(per_gpu / peak, 4),
            "peak_source": f"{peaks['source']} ({'bf16 burst' if runner.bound == 'tensor' else 'copy'})",
            "traffic": traffic_for(runner.kernel_file, runner.name),
            "work_per_launch": work,
            "timed_as": "whole library call per step (all of its kernels)"}
    if runner.bound == "hbm":
        roof["frac_vs_8TBs"] = round(per_gpu / 8000.0, 4)
    return value, ms, roof


# --------------------------------------------------------------------------- main

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="grpo",
                    choices=["grpo", "tiny", "large", "verify", "verify8", "verify-shared",
                             "verify-fp8", "verify-fp8-8", "verify-extend", "verify-extend8",
                             "grpo-backward",
                             "sparse",
                             "sparse4k"])
    ap.add_argument("--impl", default="psa", choices=["psa", "reference"])
    ap.add_argument("--no-extras", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=15.0,
                    help="seconds of oracle work for the CPU baseline")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        return run_reference(args, world, rank)

    dist_on = world > 1
    if dist_on:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    peaks = load_peaks()
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)

    runner = make_runner(args.workload, dev)
    with ClockSampler(local) as clk:
        value, ms, roof = measure(runner, args.steps, args.warmup, flush, dist_on, world, peaks)
    clocks = clk.summary()

    out = {"metric": METRIC, "value": round(value, 3), "unit": runner.unit, "n_gpus": world,
           "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 5),
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
           "dtype": "bf16" if args.workload != "tiny" else "f32",
           "data": "synthetic (seeded N(0,1)*sigma; no dataset)",
           "config": {"workload": runner.name, "l2": "flushed between steps (256 MiB write)",
                      "parallelism": f"replicas x{world}" if world > 1 else "single GPU"},
           "roofline": roof, "clocks": clocks,
           "gpu_launches": runner.kernels_per_step * args.steps}

    if not args.no_e2e and hasattr(runner, "e2e_setup"):
        runner.e2e_setup()
        per = time_steps(runner.e2e_step, max(3, min(args.steps, 10)), 2, flush, dist_on)
        ems = max_over_ranks(sum(per) / len(per), dist_on)
        out["e2e"] = {"value": round(job_throughput(world, runner.work(), ems, runner.unit), 3),
                      "unit": runner.unit, "ms_per_step": round(ems, 4),
                      "h2d_bytes_per_step": runner.h2d, "d2h_bytes_per_step": runner.d2h}

    if not args.no_extras and args.workload == "grpo":
        extras = {}
        for name in ("verify", "verify-fp8", "verify-extend", "verify-shared", "large",
                     "grpo-backward", "sparse"):
            try:
                r = make_runner(name, dev)
                v, m, rf = measure(r, max(3, min(args.steps, 10)), 3, flush, dist_on, world,
                                   peaks)
                extras[name] = {"workload": r.name, "value": round(v, 3), "unit": r.unit,
                                "ms_per_step": round(m, 4), "roofline": rf}
                del r
            except Exception as e:  # a kernel that is not built yet
                extras[name] = {"unavailable": f"{type(e).__name__}: {e}"[:200]}
            torch.cuda.empty_cache()
        out["extras"] = extras

    if rank == 0 and world == 1 and args.cpu_budget > 0:
        done, secs, sample = runner.oracle_sample(args.cpu_budget)
        scale = 1e12 if runner.unit == "TFLOP/s" else 1e9
        out["cpu_baseline"] = {"value": done / secs / scale, "unit": runner.unit,
                               "cores": host_cores(), "kind": "oracle",
                               "sample": f"{sample}, {secs:.1f} s"}
    if rank == 0:
        print(json.dumps(out), flush=True)
    if dist_on:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()


def run_reference(args, world, rank):
    """The oracle, as it stands, on the host cores: each step is a bounded
    sample of the same workload (rank 0 only)."""
    if rank != 0:
        return
    dev = torch.device("cuda", 0) if torch.cuda.is_available() else torch.device("cpu")
    runner = make_runner(args.workload, dev)
    per_step = max(2.0, 60.0 / max(1, args.steps + args.warmup))
    for _ in range(args.warmup):
        runner.oracle_sample(per_step / 4)
    done_t, secs_t, sample = 0.0, 0.0, ""
    for _ in range(args.steps):
        d, s, sample = runner.oracle_sample(per_step)
        done_t += d
        secs_t += s
    scale = 1e12 if runner.unit == "TFLOP/s" else 1e9
    value = done_t / secs_t / scale
    out = {"impl": "reference", "metric": METRIC, "value": value, "unit": runner.unit,
           "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
           "ms_per_step": 1e3 * secs_t / args.steps, "higher_is_better": True,
           "scaling": "weak", "vs_baseline": None, "dtype": "f64",
           "data": "synthetic (seeded N(0,1)*sigma; no dataset)",
           "config": {"workload": runner.name, "l2": "n/a (CPU)",
                      "parallelism": "host cores"},
           "cpu_baseline": {"value": value, "unit": runner.unit, "cores": host_cores(),
                            "kind": "oracle", "sample": f"per step: {sample}"},
           "e2e": {"value": value, "unit": runner.unit, "h2d_bytes_per_step": 0,
                   "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


if __name__ == "__main__":
    main()
