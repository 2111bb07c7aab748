"""Builds libssmscan.so in-tree with nvcc for sm_100a only.

    python -m selective_state_space_54_b200.build [--force] [--ptxas-verbose]
"""
from __future__ import annotations

import argparse
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libssmscan.so")
SOURCES = ["ssm_api.cu", "ssm_fwd.cu", "ssm_bwd.cu", "ssm_bwd16.cu", "ssm_noalloc.cu", "ssm_step.cu", "ssm_conv.cu"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def sources() -> list[str]:
    return [os.path.join(CSRC, s) for s in SOURCES if os.path.exists(os.path.join(CSRC, s))]


def _stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    deps = sources() + [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith(".cuh")]
    deps.append(os.path.join(INCLUDE, "ssm_scan.h"))
    return any(os.path.getmtime(d) > t for d in deps)


def _compile(args):
    cmd, src = args
    r = subprocess.run(cmd, capture_output=True, text=True)
    return src, r.returncode, r.stdout + r.stderr


def build(force: bool = False, ptxas_verbose: bool = False, quiet: bool = True) -> str:
    """Compile every source to an object in parallel, then link the library."""
    if not force and not _stale():
        return LIB
    from concurrent.futures import ThreadPoolExecutor
    tmpdir = os.path.join(PKG, f"_build{os.getpid()}")
    os.makedirs(tmpdir, exist_ok=True)
    base = [nvcc(), "-O3", "-std=c++17", *ARCH, "-lineinfo", "-Xcompiler", "-fPIC",
            "-I", INCLUDE, "-I", CSRC, "-c"]
    if ptxas_verbose:
        base += ["-Xptxas", "-v"]
    jobs = []
    for src in sources():
        obj = os.path.join(tmpdir, os.path.basename(src) + ".o")
        jobs.append((base + ["-o", obj, src], src))
    try:
        with ThreadPoolExecutor(max_workers=min(len(jobs), os.cpu_count() or 1)) as ex:
            results = list(ex.map(_compile, jobs))
        log = "".join(out for _, _, out in results)
        if any(rc != 0 for _, rc, _ in results):
            sys.stderr.write(log)
            raise RuntimeError("nvcc failed building libssmscan.so")
        tmp = LIB + f".tmp{os.getpid()}"
        objs = [os.path.join(tmpdir, os.path.basename(src) + ".o") for src in sources()]
        r = subprocess.run([nvcc(), *ARCH, "-shared", "-o", tmp, *objs], capture_output=True, text=True)
        if r.returncode != 0:
            sys.stderr.write(r.stdout + r.stderr)
            raise RuntimeError("nvcc failed linking libssmscan.so")
        if ptxas_verbose or not quiet:
            sys.stderr.write(log)
        os.replace(tmp, LIB)
    finally:
        shutil.rmtree(tmpdir, ignore_errors=True)
    return LIB


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--ptxas-verbose", action="store_true")
    a = ap.parse_args()
    print(build(force=a.force, ptxas_verbose=a.ptxas_verbose, quiet=False))
