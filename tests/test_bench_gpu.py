"""bench.py's JSON line on a GPU: the keys the measurement contract names and
their internal consistency, from a short run of the default workload (the
Mamba-2.8B layer forward)."""
import json
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_bench_line_contract(cuda_device):
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--steps", "3", "--warmup", "3",
                        "--no-cpu-baseline", "--no-bwd"],
                       capture_output=True, text=True, timeout=900, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-3000:]
    line = json.loads(r.stdout.strip().splitlines()[-1])
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
              "scaling", "vs_baseline", "dtype", "data", "config", "roofline", "e2e", "gpu_launches",
              "clocks"):
        assert k in line, k
    assert line["n_gpus"] == 1 and line["steps"] == 3 and line["warmup"] >= 3
    assert line["higher_is_better"] is True and line["scaling"] == "weak"
    assert line["data"] == "synthetic" and line["vs_baseline"] is None
    cfg = line["config"]
    assert cfg["workload"] == "mamba-2.8b-layer"
    # whole-job throughput: tokens x channels of one step over the step's device time
    bld = cfg["batch"] * cfg["seqlen"] * cfg["d_inner"]
    assert abs(line["value"] - bld / (line["ms_per_step"] * 1e-3)) <= 1e-6 * line["value"]
    rf = line["roofline"]
    assert rf["bound"] in ("alu", "hbm", "tensor")
    assert rf["unit"] in ("Tex2/s", "GB/s", "TFLOP/s")
    assert abs(rf["frac"] - rf["achieved"] / rf["peak"]) <= 1e-9 * rf["frac"]
    assert 0.0 < rf["frac"] < 1.5
    e2e = line["e2e"]
    assert e2e["unit"] == line["unit"]
    assert e2e["h2d_bytes_per_step"] > 0 and e2e["d2h_bytes_per_step"] > 0
    assert 0.0 < e2e["value"] < line["value"]  # the host copies of every step make it slower
    assert line["gpu_launches"] > 0
    if line["clocks"] is not None:  # sampled while the timed region runs
        assert line["clocks"]["sm_mhz"] > 0 and isinstance(line["clocks"]["reasons"], list)
