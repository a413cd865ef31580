"""Parity bar shared by the GPU tests: bf16 in, fp32 accumulate, bf16 out,
compared element by element with the fp64 oracle on the same input bytes.

  O:   max |gpu - oracle| <= 1e-2 and ||gpu - oracle||_F / ||oracle||_F <= 5e-3
  LSE: max |gpu - oracle| <= 1e-3 (natural log)
"""
import numpy as np
import torch

O_MAX_ABS = 1e-2
O_REL_FRO = 5e-3
LSE_MAX_ABS = 1e-3


def errors(o_gpu, lse_gpu, o_ref, lse_ref):
    o = o_gpu.detach().float().cpu().numpy().astype(np.float64) if torch.is_tensor(o_gpu) else o_gpu
    l = lse_gpu.detach().float().cpu().numpy().astype(np.float64) if torch.is_tensor(lse_gpu) else lse_gpu
    d = o - o_ref
    fro = float(np.linalg.norm(d) / max(np.linalg.norm(o_ref), 1e-30))
    return {
        "o_max_abs": float(np.abs(d).max()) if d.size else 0.0,
        "o_rel_fro": fro,
        "lse_max_abs": float(np.abs(l - lse_ref).max()) if l.size else 0.0,
    }


def assert_parity(o_gpu, lse_gpu, o_ref, lse_ref, what=""):
    e = errors(o_gpu, lse_gpu, o_ref, lse_ref)
    assert np.all(np.isfinite(o_gpu.float().cpu().numpy())), f"{what}: non-finite O"
    assert e["o_max_abs"] <= O_MAX_ABS, f"{what}: {e}"
    assert e["o_rel_fro"] <= O_REL_FRO, f"{what}: {e}"
    assert e["lse_max_abs"] <= LSE_MAX_ABS, f"{what}: {e}"
    return e
