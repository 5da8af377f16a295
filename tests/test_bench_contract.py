"""bench.py's output contract, on the CPU (no GPU needed).

The reference arm (`--impl reference`) times the fp64 oracle on the host's
cores and prints one JSON line with the keys the driver reads; the CUDA arm on
a machine without a GPU fails with a nonzero exit status instead of falling
back to anything.
"""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def run_bench(*args, timeout=240):
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], cwd=ROOT,
                          capture_output=True, text=True, timeout=timeout)


def json_lines(stdout):
    return [json.loads(l) for l in stdout.splitlines() if l.startswith("{")]


@pytest.mark.parametrize("workload", ["0", "4"])
def test_reference_arm_line(workload):
    r = run_bench("--impl", "reference", "--workload", workload, "--steps", "2", "--warmup", "3",
                  "--reference-seconds", "2")
    assert r.returncode == 0, r.stderr[-2000:]
    lines = json_lines(r.stdout)
    assert len(lines) == 1
    d = lines[0]
    assert d["impl"] == "reference"
    assert d["unit"] == "tokens/s" and d["higher_is_better"] is True
    assert d["value"] > 0 and d["steps"] == 2 and d["warmup"] == 3 and d["n_gpus"] == 1
    assert d["dtype"] == "f64" and d["data"] == "synthetic" and d["vs_baseline"] is None
    assert d["ms_per_step"] > 0
    assert d["config"]["workload"]
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"]
    assert cb["sample"]
    e2e = d["e2e"]
    assert e2e["value"] == d["value"] and e2e["unit"] == d["unit"]
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0


def test_cuda_arm_without_a_gpu_fails_loudly():
    import torch

    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    r = run_bench("--steps", "1", "--warmup", "3", "--no-cpu-baseline", "--no-e2e")
    assert r.returncode != 0
    assert not json_lines(r.stdout), "printed a result line without a GPU"
