"""Host code under AddressSanitizer and UndefinedBehaviorSanitizer (no GPU).

The fp64 oracle's C code runs a set of small cases (every optional input on
and off, exact ZOH, an initial state, empty problems, several threads) built
with -fsanitize=address,undefined; the C caller of the library's ABI runs its
argument checks the same way.  Any out-of-bounds access, use after free, leak
or undefined operation in the instrumented code aborts the program with a
report, and the test fails.
"""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SAN = ["-O1", "-g", "-fsanitize=address,undefined", "-fno-sanitize-recover=all",
       "-fno-omit-frame-pointer"]


def _gcc():
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    return gcc


def _run(exe):
    env = dict(os.environ, ASAN_OPTIONS="detect_leaks=1:protect_shadow_gap=0",
               UBSAN_OPTIONS="print_stacktrace=1")
    r = subprocess.run([exe], capture_output=True, text=True, timeout=300, env=env)
    report = r.stdout + r.stderr
    assert r.returncode == 0, report
    assert "AddressSanitizer" not in report and "runtime error" not in report, report
    return report


def test_oracle_under_sanitizers(tmp_path):
    exe = str(tmp_path / "oracle_sanitize")
    subprocess.check_call([_gcc(), "-std=c99", "-Wall", "-Werror", *SAN,
                           os.path.join(ROOT, "tests", "c_abi", "oracle_sanitize.c"),
                           os.path.join(ROOT, "oracle", "ssm_oracle.c"), "-o", exe, "-lm", "-lpthread"])
    assert "ok" in _run(exe)


def test_abi_caller_under_sanitizers(tmp_path):
    from selective_state_space_54_b200.build import LIB, build
    build()
    exe = str(tmp_path / "abi_check_sanitize")
    libdir = os.path.dirname(LIB)
    subprocess.check_call([_gcc(), "-std=c99", "-Wall", "-Werror", *SAN, "-I", os.path.join(ROOT, "include"),
                           os.path.join(ROOT, "tests", "c_abi", "abi_check.c"), "-o", exe,
                           "-L", libdir, "-lssmscan", "-Wl,-rpath," + libdir])
    assert "passed" in _run(exe)
