"""The special-function unit's exp2 rate, measured on the device.

The scan's roofline counts one ex2 per (batch, step, channel, state) element
against SMs x (ex2 per SM per cycle) x SM clock.  This test builds a small
probe (tests/probes/ex2_rate.cu: one CTA of 1024 threads per SM, 8
independent exp2 chains per thread, timed with the SM cycle counter) and
checks that the measured rate is the 16 per SM per cycle the roofline uses.
Method: ex2 count of a CTA / its clock64 cycles, median over the SMs.
"""
import ctypes
import os
import shutil
import subprocess

import numpy as np
import pytest

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))
EX2_PER_CLK_PER_SM = 16  # the value the benchmark's roofline uses


def _build(tmp_path):
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    so = str(tmp_path / "ex2_rate.so")
    subprocess.run([nvcc, "-O3", "-gencode", "arch=compute_100a,code=sm_100a", "-shared",
                    "-Xcompiler", "-fPIC", "-o", so, os.path.join(HERE, "probes", "ex2_rate.cu")],
                   check=True, capture_output=True)
    return so


def test_ex2_rate_per_sm_per_cycle(cuda_device, tmp_path):
    lib = ctypes.CDLL(_build(tmp_path))
    iters = 4096
    cyc = (ctypes.c_longlong * 1024)()
    sms = ctypes.c_int(0)
    rc = lib.ex2_rate_probe(iters, ctypes.byref(sms), cyc, 1024)
    assert rc == 0, rc
    n = sms.value
    cycles = np.array(cyc[:n], dtype=np.float64)
    per_cta = 1024 * 8 * iters
    rate = float(np.median(per_cta / cycles))
    print(f"ex2.approx.ftz.f32: {rate:.2f} per SM per cycle (median over {n} SMs; "
          f"min {np.min(per_cta / cycles):.2f}, max {np.max(per_cta / cycles):.2f})")
    assert 0.9 * EX2_PER_CLK_PER_SM <= rate <= 1.05 * EX2_PER_CLK_PER_SM
