"""Benchmark of the shared-prefix attention hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                    [--impl psa|reference] [--no-extras]

One JSON line on rank 0.  The headline workload is the largest single-GPU
prefill: two packed rollout groups of P=8192, N=16, S=1024 (32 query heads
on 8 KV heads, d=128, bf16); metric = visible-block attention TFLOP/s
(exact visible-pair FLOPs, 4*d*Hq*pairs) over the flat packed layout.  With
extras on (default) the line also carries the GRPO group, the
speculative-verify prefix-KV GB/s (bf16, e4m3, paged extend form), the
shared-prefix verify, the GRPO backward and the shared-latent sparse
prefill, each timed with the headline's steps and warm-up, each with its own
end-to-end number and CPU-oracle baseline.

Timing: W untimed warm-up steps, then K steps, each bracketed by CUDA
events on the launching stream, with an L2 flush (a 256 MiB write) between
steps outside the events; barrier + synchronize around the whole region;
max over ranks.  N > 1 runs independent replicas (weak scaling): the path
has no exchange step.  ``--impl reference`` times the fp64 CPU oracle on the
host cores on a bounded sample of the same workload, on inputs built on the
host (the GPU and the CUDA library are not touched).
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
    """One workload on the GPU: inputs resident on the device, one step = one
    call of the public C-ABI entry point, algorithmic work per step.
    ``inputs`` are the tensors an end-to-end step copies in from pinned host
    memory, ``outputs`` the ones it reads back."""
    name = ""
    unit = ""
    kernels_per_step = 1
    bound = "tensor"
    kernel_file = ""
    inputs: list = []
    outputs: list = []

    def work(self) -> float: ...
    def step(self): ...

    # end to end: host (pinned) inputs in, outputs back to the host
    def e2e_setup(self):
        self.h_in = [t.cpu().pin_memory() for t in self.inputs]
        self.h_out = [torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in self.outputs]
        self.h2d = sum(t.numel() * t.element_size() for t in self.h_in)
        self.d2h = sum(t.numel() * t.element_size() for t in self.h_out)

    def e2e_step(self):
        for d, h in zip(self.inputs, self.h_in):
            d.copy_(h, non_blocking=True)
        self.step()
        for h, d in zip(self.h_out, self.outputs):
            h.copy_(d, non_blocking=True)

    def e2e_release(self):
        self.h_in, self.h_out = [], []


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
        self.inputs, self.outputs = [self.q, self.k, self.v], [self.o, self.lse]

    def work(self):
        return self.wl.flops()

    def step(self):
        self.psa.prefill(self.q, self.k, self.v, self.sched, self.wl.scale, out=self.o,
                         lse=self.lse, workspace=self.ws)


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
        self.inputs = [self.q, self.kd, self.vd, self.kc, self.vc]
        self.outputs = [self.o, self.lse]

    def work(self):
        return float(self.wl.prefix_kv_bytes())

    def step(self):
        wl = self.wl
        self.psa.verify(self.q, self.kd, self.vd, self.kc, self.vc, self.indptr, wl.L, wl.scale,
                        wl.Ld, nsplit=wl.nsplit, out=self.o, lse=self.lse, workspace=self.ws)


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
        self.inputs, self.outputs = [self.q, self.lat, self.idx], [self.o, self.lse]

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
        self.name = backward_name(wl)
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
        self.inputs = [self.q, self.k, self.v, self.o, self.lse, self.dout]
        self.outputs = [self.dq, self.dk, self.dv]

    def work(self):
        return backward_flops(self.wl)

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
        self.inputs = [self.q, self.kd, self.vd, self.kc8, self.vc8]
        self.outputs = [self.o, self.lse]

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
        self.inputs = [self.q, self.kd, self.vd, self.kp, self.vp]
        self.outputs = [self.o, self.lse]

    def work(self):
        return self.wl.flops()

    def step(self):
        wl = self.wl
        self.psa.verify_shared(self.q, self.kd, self.vd, self.kp, self.vp, wl.scale, wl.Ld,
                               nsplit=self.ns, out=self.o, lse=self.lse, workspace=self.ws)


class ExtendVerifyRunner(Runner):
    """Verify in the extend form: ragged drafts in trees, each prefix read
    through a token-granular page table (gathered with bulk copies)."""
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
        self.inputs = [self.q, self.kd, self.vd, self.kp, self.vp, self.idx] + (
            [] if self.mask is None else [self.mask])
        self.outputs = [self.o, self.lse]

    def work(self):
        return float(self.wl.prefix_kv_bytes())

    def step(self):
        wl = self.wl
        self.psa.verify_extend(self.q, self.kd, self.vd, self.kp, self.vp, self.qo,
                               wl.max_draft_len, self.kvp, wl.max_prefix_len, wl.scale,
                               kv_indices=self.idx, draft_mask=self.mask,
                               mask_indptr=None if self.mask is None else self.mi,
                               nsplit=wl.nsplit, out=self.o, lse=self.lse, workspace=self.ws)


def backward_name(wl: W.PrefillWorkload) -> str:
    return wl.name.replace("grpo", "grpo-backward", 1)


def backward_flops(wl: W.PrefillWorkload) -> float:
    """Five products of the visible pairs (S, dP, dV, dQ, dK), 2 d FLOP each."""
    return wl.flops() * 10.0 / 4.0


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
VERIFY_SHARED_SMALL = W.SharedVerifyWorkload(
    "verify-shared B=8 L=16384 drafts=4 H=32/8 d=128 bf16", B=8, L=16384, Ld=4, Hq=32, Hkv=8,
    d=128, seed=6)

# name -> (runner class, workload)
WORKLOADS = {
    "tiny": (PrefillRunner, W.TINY),
    "grpo": (PrefillRunner, W.GRPO),
    "large": (PrefillRunner, W.LARGE),
    "verify": (VerifyRunner, W.VERIFY),
    "verify8": (VerifyRunner, VERIFY_SMALL),
    "verify-shared": (SharedVerifyRunner, W.VERIFY_SHARED),
    "verify-shared8": (SharedVerifyRunner, VERIFY_SHARED_SMALL),
    "verify-fp8": (VerifyFp8Runner, W.VERIFY_FP8),
    "verify-fp8-8": (VerifyFp8Runner, VERIFY_FP8_SMALL),
    "verify-extend": (ExtendVerifyRunner, W.VERIFY_PAGED),
    "verify-extend8": (ExtendVerifyRunner, VERIFY_PAGED_SMALL),
    "grpo-backward": (BackwardRunner, W.GRPO),
    "sparse": (SparseRunner, W.SPARSE),
    "sparse4k": (SparseRunner, SPARSE_SMALL),
}

# the headline is the largest single-GPU prefill workload; every other
# workload of the metric rides along as an extra, timed the same way
HEADLINE = "large"
EXTRAS = ("grpo", "verify", "verify-fp8", "verify-extend", "verify-shared", "grpo-backward",
          "sparse")


def make_runner(name: str, dev):
    cls, wl = WORKLOADS[name]
    return cls(wl, dev)


# --------------------------------------------------------------------------- CPU oracle

class OracleSampler:
    """The fp64 oracle, as it stands, on a bounded sample of one workload.

    Inputs are built on the host from the workload's recipe (same shapes and
    distributions as the GPU's; nothing here touches the GPU or the CUDA
    library).  ``run(budget)`` returns (work done in the metric's unit
    numerator, seconds, description); ``full_work()`` is the whole
    workload's work, so the full-config CPU time is extrapolated as
    full_work / (work / seconds)."""
    unit = ""
    threads = 0      # host threads the oracle calls use (0: every core)

    def run(self, budget_s: float): ...
    def full_work(self) -> float: ...


def _visible_keys_per_row(segments) -> "np.ndarray":
    """Keys each flat row sees: its own segment up to itself plus every
    ancestor segment in full (the flat layout's visibility)."""
    import numpy as np
    lens = [n for n, _ in segments]
    start = np.cumsum([0] + lens[:-1])
    anc = []
    for i, (_, p) in enumerate(segments):
        a = 0
        while p >= 0:
            a += lens[p]
            p = segments[p][1]
        anc.append(a)
    out = np.zeros(sum(lens), dtype=np.int64)
    for s, (n, _) in enumerate(segments):
        out[start[s]:start[s] + n] = anc[s] + np.arange(1, n + 1)
    return out


class PrefillSampler(OracleSampler):
    unit = "TFLOP/s"

    def __init__(self, wl: W.PrefillWorkload):
        import numpy as np
        self.wl = wl
        q, k, v = wl.make("cpu")
        self.q, self.k, self.v = (np.ascontiguousarray(t.float().numpy()) for t in (q, k, v))
        self.vis = _visible_keys_per_row(wl.segments())
        self.perm = torch.randperm(wl.T, generator=torch.Generator().manual_seed(0)).numpy()
        self.pos = 0

    def full_work(self):
        return self.wl.flops()

    def run(self, budget_s):
        import numpy as np
        import oracle
        wl = self.wl
        chunk = 4 * oracle.default_threads()
        t0 = time.perf_counter()
        done, n = 0.0, 0
        while time.perf_counter() - t0 < budget_s:
            rows = self.perm[np.arange(self.pos, self.pos + chunk) % wl.T].astype(np.int32)
            self.pos += chunk
            oracle.prefill(self.q, self.k, self.v, wl.segments(), wl.scale, rows=rows)
            done += 4.0 * wl.d * wl.Hq * float(self.vis[rows].sum())
            n += chunk
        return done, time.perf_counter() - t0, f"{n} random query rows x {wl.Hq} heads"


class BackwardSampler(OracleSampler):
    """Whole heads of the backward: a KV head with its query heads over all
    T rows (the oracle's full backward on that head slice)."""
    unit = "TFLOP/s"

    def __init__(self, wl: W.PrefillWorkload):
        self.wl = wl
        q, k, v = wl.make("cpu")
        g = torch.Generator().manual_seed(wl.seed + 100)
        do = (torch.randn(q.shape, generator=g) * wl.sigma).to(q.dtype)
        self.t = (q, k, v, do)
        self.h = 0

    def full_work(self):
        return backward_flops(self.wl)

    def run(self, budget_s):
        import oracle
        wl = self.wl
        G = wl.Hq // wl.Hkv
        q, k, v, do = self.t
        t0 = time.perf_counter()
        done, n = 0.0, 0
        while n == 0 or time.perf_counter() - t0 < budget_s:
            h = self.h % wl.Hkv
            self.h += 1
            qs, dos = (x[:, h * G:(h + 1) * G].contiguous() for x in (q, do))
            ks, vs = (x[:, h:h + 1].contiguous() for x in (k, v))
            oracle.prefill_bwd(qs, ks, vs, dos, wl.segments(), wl.scale)
            done += backward_flops(wl) / wl.Hkv
            n += 1
        return done, time.perf_counter() - t0, (
            f"{n} whole KV head(s) ({G} query head(s) each) over all {wl.T} rows")


class VerifySampler(OracleSampler):
    """Whole requests: each sampled request's drafts against its own prefix,
    its inputs drawn on the host from the workload's recipe.  Enough
    requests go to one oracle call to give every host thread a draft row."""
    unit = "GB/s"

    def __init__(self, wl: W.VerifyWorkload, fp8: bool = False):
        import oracle
        self.wl, self.fp8 = wl, fp8
        self.b = 0
        self.per_call = max(1, oracle.default_threads() // wl.Ld)
        self.threads = min(oracle.default_threads(), self.per_call * wl.Ld)

    def _bytes(self, ntok):
        wl = self.wl
        return ntok * wl.Hkv * wl.d * 2 * (1 if self.fp8 else 2)

    def full_work(self):
        return float(self.wl.prefix_fp8_bytes() if self.fp8 else self.wl.prefix_kv_bytes())

    def run(self, budget_s):
        import numpy as np
        import oracle
        wl = self.wl
        t_wall = 0.0
        done, n = 0.0, 0
        while n == 0 or t_wall < budget_s:
            bs = [(self.b + i) % wl.B for i in range(self.per_call)]
            self.b += self.per_call
            lens = [wl.lens()[b] for b in bs]
            part = W.VerifyWorkload("part", B=len(bs), L=0, Ld=wl.Ld, Hq=wl.Hq, Hkv=wl.Hkv,
                                    d=wl.d, nsplit=1, prefix_lens=lens,
                                    seed=wl.seed * 1000 + bs[0])
            ind = np.array(part.kv_indptr(), dtype=np.int64)
            if self.fp8:
                q, kd, vd, kc, vc = part.make_fp8("cpu")
                t0 = time.perf_counter()
                oracle.verify_fp8(q, kd, vd, kc, vc, wl.k_scale, wl.v_scale, ind, wl.Ld,
                                  wl.scale)
            else:
                q, kd, vd, kc, vc = part.make("cpu")
                t0 = time.perf_counter()
                oracle.verify(q, kd, vd, kc, vc, ind, wl.Ld, wl.scale)
            t_wall += time.perf_counter() - t0
            done += self._bytes(sum(lens))
            n += len(bs)
        return done, t_wall, f"{n} whole requests ({n * wl.Ld} draft rows)"


class ExtendSampler(OracleSampler):
    """Whole requests of the extend form, batched per oracle call until every
    host thread has a draft row."""
    unit = "GB/s"

    def __init__(self, wl: W.ExtendVerifyWorkload):
        import oracle
        self.wl = wl
        self.b = 0
        self.threads = oracle.default_threads()

    def full_work(self):
        return float(self.wl.prefix_kv_bytes())

    def run(self, budget_s):
        import oracle
        wl = self.wl
        t_wall = 0.0
        done, n = 0.0, 0
        while n == 0 or t_wall < budget_s:
            bs = []
            while sum(wl.draft_lens[b] for b in bs) < self.threads and len(bs) < wl.B:
                bs.append(self.b % wl.B)
                self.b += 1
            part = W.ExtendVerifyWorkload(
                "part", draft_lens=[wl.draft_lens[b] for b in bs],
                prefix_lens=[wl.prefix_lens[b] for b in bs], Hq=wl.Hq, Hkv=wl.Hkv, d=wl.d,
                nsplit=1, tree=wl.tree, pool_slack=wl.pool_slack, seed=wl.seed * 1000 + bs[0])
            q, kd, vd, kp, vp, idx, mask = part.make("cpu")
            t0 = time.perf_counter()
            oracle.verify_extend(q, kd, vd, kp, vp, part.qo_indptr(), part.kv_indptr(), wl.scale,
                                 kv_indices=idx, draft_mask=mask,
                                 mask_indptr=None if mask is None else part.mask_indptr())
            t_wall += time.perf_counter() - t0
            done += float(part.prefix_kv_bytes())
            n += len(bs)
        return done, t_wall, f"{n} whole requests"


class SharedVerifySampler(OracleSampler):
    """Whole requests against the whole shared prefix, enough per oracle call
    to give every host thread a draft row."""
    unit = "TFLOP/s"

    def __init__(self, wl: W.SharedVerifyWorkload):
        import oracle
        self.wl = wl
        self.b = 0
        self.per_call = max(1, oracle.default_threads() // wl.Ld)
        self.threads = min(oracle.default_threads(), self.per_call * wl.Ld)

    def full_work(self):
        return self.wl.flops()

    def run(self, budget_s):
        import oracle
        wl = self.wl
        t_wall = 0.0
        done, n = 0.0, 0
        while n == 0 or t_wall < budget_s:
            part = W.SharedVerifyWorkload("part", B=self.per_call, L=wl.L, Ld=wl.Ld, Hq=wl.Hq,
                                          Hkv=wl.Hkv, d=wl.d, seed=wl.seed * 1000 + self.b)
            self.b += self.per_call
            q, kd, vd, kp, vp = part.make("cpu")
            t0 = time.perf_counter()
            oracle.verify_shared(q, kd, vd, kp, vp, wl.Ld, wl.scale)
            t_wall += time.perf_counter() - t0
            done += part.flops()
            n += self.per_call
        return done, t_wall, f"{n} whole requests ({n * wl.Ld} draft rows)"


class SparseSampler(OracleSampler):
    """Random query rows: the full latent, and for each sampled row its own
    Q and index list drawn on the host from the workload's recipe."""
    unit = "TFLOP/s"

    def __init__(self, wl: W.SparseLatentWorkload):
        self.wl = wl
        self.g = torch.Generator().manual_seed(wl.seed)
        self.lat = (torch.randn((wl.T, wl.dl), generator=self.g) * wl.sigma).to(wl.dtype)

    def full_work(self):
        return self.wl.flops()

    def _rows(self, rows):
        wl = self.wl
        idx = torch.full((len(rows), wl.topk), -1, dtype=torch.int32)
        for i, t in enumerate(rows):
            if t < wl.topk:
                idx[i, :t + 1] = torch.arange(t + 1, dtype=torch.int32)
            else:
                idx[i] = torch.sort(torch.randperm(t + 1, generator=self.g)[:wl.topk]).values
        q = (torch.randn((len(rows), wl.H, wl.dl), generator=self.g) * wl.sigma).to(wl.dtype)
        return q, idx

    def run(self, budget_s):
        import oracle
        wl = self.wl
        chunk = 2 * oracle.default_threads()
        t_wall = 0.0
        done, n = 0.0, 0
        while n == 0 or t_wall < budget_s:
            rows = torch.randint(0, wl.T, (chunk,), generator=self.g).tolist()
            q, idx = self._rows(rows)
            t0 = time.perf_counter()
            oracle.sparse_latent(q, self.lat, idx, wl.scale)
            t_wall += time.perf_counter() - t0
            done += 4.0 * wl.dl * wl.H * sum(min(t + 1, wl.topk) for t in rows)
            n += chunk
        return done, t_wall, f"{n} random query rows x {wl.H} heads"


def default_oracle_threads() -> int:
    import oracle
    return oracle.default_threads()


def make_sampler(name: str) -> OracleSampler:
    cls, wl = WORKLOADS[name]
    if cls is PrefillRunner:
        return PrefillSampler(wl)
    if cls is BackwardRunner:
        return BackwardSampler(wl)
    if cls is VerifyRunner:
        return VerifySampler(wl)
    if cls is VerifyFp8Runner:
        return VerifySampler(wl, fp8=True)
    if cls is ExtendVerifyRunner:
        return ExtendSampler(wl)
    if cls is SharedVerifyRunner:
        return SharedVerifySampler(wl)
    return SparseSampler(wl)


def workload_label(name: str) -> str:
    cls, wl = WORKLOADS[name]
    return backward_name(wl) if cls is BackwardRunner else wl.name


def cpu_baseline(name: str, budget_s: float) -> dict:
    """The oracle's rate on a bounded sample of ``name``, with the whole
    workload's CPU time extrapolated from it (labelled as such)."""
    sampler = make_sampler(name)
    done, secs, sample = sampler.run(budget_s)
    scale = 1e12 if sampler.unit == "TFLOP/s" else 1e9
    rate = done / secs
    return {"value": rate / scale, "unit": sampler.unit,
            "cores": sampler.threads or min(host_cores(), default_oracle_threads()),
            "kind": "oracle", "sample": f"{sample}, {secs:.1f} s",
            "full_config_s": round(sampler.full_work() / rate, 1),
            "full_config_s_is": "extrapolated (sampled rate x whole-workload work)"}


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

def e2e_measure(runner, steps, warmup, flush, dist_on, world):
    """The same call with the inputs copied in from pinned host memory and
    the outputs read back inside the timed region."""
    runner.e2e_setup()
    per = time_steps(runner.e2e_step, steps, warmup, flush, dist_on)
    ems = max_over_ranks(sum(per) / len(per), dist_on)
    out = {"value": round(job_throughput(world, runner.work(), ems, runner.unit), 3),
           "unit": runner.unit, "ms_per_step": round(ems, 4),
           "h2d_bytes_per_step": runner.h2d, "d2h_bytes_per_step": runner.d2h}
    runner.e2e_release()
    return out


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=HEADLINE, choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="psa", choices=["psa", "reference"])
    ap.add_argument("--no-extras", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=15.0,
                    help="seconds of oracle work for the headline's CPU baseline")
    ap.add_argument("--extra-cpu-budget", type=float, default=4.0,
                    help="seconds of oracle work for each extra's CPU baseline")
    ap.add_argument("--ref-step-s", type=float, default=0.0,
                    help="--impl reference: seconds of oracle work per step (0: spread "
                         "about a minute over warm-up and timed steps)")
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
    do_cpu = rank == 0 and world == 1

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

    if not args.no_e2e:
        out["e2e"] = e2e_measure(runner, args.steps, args.warmup, flush, dist_on, world)
    del runner
    torch.cuda.empty_cache()

    if not args.no_extras and args.workload == HEADLINE:
        extras = {}
        for name in EXTRAS:
            try:
                r = make_runner(name, dev)
                with ClockSampler(local) as eclk:
                    v, m, rf = measure(r, args.steps, args.warmup, flush, dist_on, world, peaks)
                ex = {"workload": r.name, "value": round(v, 3), "unit": r.unit,
                      "ms_per_step": round(m, 4), "steps": args.steps, "warmup": args.warmup,
                      "roofline": rf, "clocks": eclk.summary(),
                      "gpu_launches": r.kernels_per_step * args.steps}
                if not args.no_e2e:
                    ex["e2e"] = e2e_measure(r, args.steps, args.warmup, flush, dist_on, world)
                del r
            except Exception as e:  # a kernel that is not built yet
                ex = {"unavailable": f"{type(e).__name__}: {e}"[:200]}
            torch.cuda.empty_cache()
            extras[name] = ex
        if do_cpu and args.extra_cpu_budget > 0:
            for name, ex in extras.items():
                if "unavailable" not in ex:
                    ex["cpu_baseline"] = cpu_baseline(name, args.extra_cpu_budget)
        out["extras"] = extras

    if do_cpu and args.cpu_budget > 0:
        out["cpu_baseline"] = cpu_baseline(args.workload, args.cpu_budget)
    if rank == 0:
        print(json.dumps(out), flush=True)
    if dist_on:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()


def run_reference(args, world, rank):
    """The oracle, as it stands, on the host cores: each step is a bounded
    sample of the same workload (rank 0 only).  Inputs are built on the host;
    neither the GPU nor the CUDA library is touched."""
    if rank != 0:
        return
    sampler = make_sampler(args.workload)
    per_step = args.ref_step_s or max(2.0, 60.0 / max(1, args.steps + args.warmup))
    for _ in range(args.warmup):
        sampler.run(per_step / 4)
    done_t, secs_t, sample = 0.0, 0.0, ""
    for _ in range(args.steps):
        d, s, sample = sampler.run(per_step)
        done_t += d
        secs_t += s
    scale = 1e12 if sampler.unit == "TFLOP/s" else 1e9
    value = done_t / secs_t / scale
    cores = sampler.threads or min(host_cores(), default_oracle_threads())
    out = {"impl": "reference", "metric": METRIC, "value": value, "unit": sampler.unit,
           "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
           "ms_per_step": 1e3 * secs_t / args.steps, "higher_is_better": True,
           "scaling": "weak", "vs_baseline": None, "dtype": "f64",
           "data": "synthetic (seeded N(0,1)*sigma; no dataset)",
           "config": {"workload": workload_label(args.workload), "l2": "n/a (CPU)",
                      "parallelism": "host cores"},
           "cpu_baseline": {"value": value, "unit": sampler.unit, "cores": cores,
                            "kind": "oracle", "sample": f"per step: {sample}",
                            "full_config_s": round(sampler.full_work() / (done_t / secs_t), 1),
                            "full_config_s_is": "extrapolated (sampled rate x whole-workload "
                                                "work)"},
           "e2e": {"value": value, "unit": sampler.unit, "h2d_bytes_per_step": 0,
                   "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


if __name__ == "__main__":
    main()
