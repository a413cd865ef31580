"""The bench's CPU arm (``--impl reference``): the fp64 oracle timed on the
host on inputs built on the host.  It must not touch the GPU or load the
CUDA library, and its line must carry the contract's keys."""
import json
import os
import subprocess
import sys

import pytest

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

_PROBE = """
import json, runpy, sys
sys.argv = ["bench.py", "--impl", "reference", "--workload", "tiny", "--steps", "2",
            "--warmup", "3", "--ref-step-s", "0.05"]
runpy.run_path("bench.py", run_name="__main__")
maps = open("/proc/self/maps").read()
print(json.dumps({"libpsa_loaded": "libpsa" in maps}))
"""


def test_reference_arm_runs_on_the_host_without_the_cuda_library():
    out = subprocess.run([sys.executable, "-c", _PROBE], cwd=ROOT, capture_output=True,
                         text=True, timeout=300, env={**os.environ, "CUDA_VISIBLE_DEVICES": ""})
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [json.loads(x) for x in out.stdout.splitlines() if x.startswith("{")]
    line, probe = lines[0], lines[-1]
    assert probe == {"libpsa_loaded": False}
    assert line["impl"] == "reference" and line["value"] > 0
    assert line["config"]["workload"] == bench.workload_label("tiny")
    for key in ("metric", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "cpu_baseline", "e2e"):
        assert key in line
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and "extrapolated" in cb[
        "full_config_s_is"]
    assert line["e2e"]["h2d_bytes_per_step"] == 0


@pytest.mark.parametrize("name", sorted(bench.WORKLOADS))
def test_every_bench_workload_has_a_host_sampler(name):
    s = bench.make_sampler(name)
    assert s.unit == bench.WORKLOADS[name][0].unit
    assert s.full_work() > 0


def test_headline_is_the_largest_prefill_and_extras_cover_every_kernel():
    assert bench.HEADLINE == "large"
    _, wl = bench.WORKLOADS["large"]
    assert wl.groups == 2 and wl.P == 8192 and wl.N == 16 and wl.S == 1024
    files = {bench.WORKLOADS[n][0].kernel_file for n in bench.EXTRAS + (bench.HEADLINE,)}
    assert files == {"psa_prefill.cu", "psa_verify.cu", "psa_verify_fp8.cu",
                     "psa_verify_shared.cu", "psa_backward.cu", "psa_sparse.cu"}
