"""ssm_scan_fwd_noalloc, the forward entry point for callers that cannot
allocate device memory (engine plugins whose host owns every allocation,
real-time loops that allocate nothing after start-up).  It must give the
same results as ssm_scan_fwd with a caller-provided workspace, call after
call, although its scratch is one static array shared by every call.

This file is collected last on purpose: it passes alone in a fresh process
and after every other test.
"""
import ctypes

import numpy as np
import pytest

import oracle
import synth
from gpu_util import assert_close, to_f64, upload

pytestmark = pytest.mark.gpu


def _noalloc(lib, shape, g, y, ls, stream):
    """The entry point itself, through ctypes: the caller passes inputs and
    outputs only, no workspace."""
    p = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())
    return lib.ssm_scan_fwd_noalloc(ctypes.byref(shape), p(g["u"]), p(g["delta"]), p(g["A"]),
                                    p(g["B"]), p(g["C"]), p(g["D"]), p(g["z"]),
                                    p(g["delta_bias"]), 1, None, p(y), p(ls), stream)


@pytest.mark.parametrize("dtype,batch,dim,L", [
    (synth.BF16, 8, 1536, 1024),   # enough channel groups that warps split groups
    (synth.F32, 2, 40, 1003),      # ragged groups and chunk tail
])
def test_noalloc_matches_workspace_entry_point(cuda_device, dtype, batch, dim, L):
    import torch
    import selective_state_space_54_b200 as ssm
    from selective_state_space_54_b200 import _lib
    lib = _lib.load()
    case = synth.make_case(batch, dim, L, 16, dtype, seed=77)
    g = upload(case, cuda_device)
    y_ref, ls_ref = ssm.scan_fwd(g["u"], g["delta"], g["A"], g["B"], g["C"], g["D"], g["z"],
                                 g["delta_bias"], return_last_state=True)
    torch.cuda.synchronize()
    ref_y, ref_ls = to_f64(y_ref), to_f64(ls_ref)
    shape = ssm.make_shape(batch, dim, L, 16, ssm.SSM_BF16 if dtype == synth.BF16 else ssm.SSM_F32)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for call in range(2):  # two calls in a row share the static scratch
        y = torch.full_like(g["u"], float("nan"))
        ls = torch.full((batch, dim, 16), float("nan"), dtype=torch.float32, device=cuda_device)
        assert _noalloc(lib, shape, g, y, ls, stream) == 0
        torch.cuda.synchronize()
        assert_close(to_f64(y), ref_y, dtype, f"y, call {call}")
        assert_close(to_f64(ls), ref_ls, dtype, f"last_state, call {call}", stored_bf16=False)


def test_noalloc_against_the_oracle(cuda_device):
    # directly against the fp64 oracle, on a shape where AUTO keeps the
    # warp-specialised look-back schedule
    import torch
    import selective_state_space_54_b200 as ssm
    from selective_state_space_54_b200 import _lib
    lib = _lib.load()
    batch, dim, L = 4, 5120, 512
    case = synth.make_case(batch, dim, L, 16, synth.BF16, seed=78)
    g = upload(case, cuda_device)
    shape = ssm.make_shape(batch, dim, L, 16, ssm.SSM_BF16)
    assert ssm.fwd_path(shape) == "lookback_ws"
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    y = torch.full_like(g["u"], float("nan"))
    ls = torch.full((batch, dim, 16), float("nan"), dtype=torch.float32, device=cuda_device)
    assert _noalloc(lib, shape, g, y, ls, stream) == 0
    torch.cuda.synchronize()
    ref = oracle.fwd(case)
    assert_close(to_f64(y), ref["y"], synth.BF16, "y")
    assert_close(to_f64(ls), ref["last_state"], synth.BF16, "last_state", stored_bf16=False)


def test_noalloc_token_major(cuda_device):
    # token-major activations through the entry point equal ssm_scan_fwd's, bit for bit
    import torch
    import selective_state_space_54_b200 as ssm
    from selective_state_space_54_b200 import _lib
    lib = _lib.load()
    batch, dim, L = 2, 1024, 1000
    case = synth.make_case(batch, dim, L, 16, synth.BF16, seed=79)
    g = upload(case, cuda_device)
    tm = dict(g)
    for k in ("u", "delta", "z"):
        tm[k] = g[k].transpose(1, 2).contiguous()
    y_ref, ls_ref = ssm.scan_fwd(tm["u"], tm["delta"], g["A"], g["B"], g["C"], g["D"], tm["z"],
                                 g["delta_bias"], return_last_state=True, token_major=True)
    shape = ssm.make_shape(batch, dim, L, 16, ssm.SSM_BF16, flags=ssm.SSM_FLAG_TOKEN_MAJOR)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for call in range(2):
        y = torch.full_like(tm["u"], float("nan"))
        ls = torch.full((batch, dim, 16), float("nan"), dtype=torch.float32, device=cuda_device)
        assert _noalloc(lib, shape, tm, y, ls, stream) == 0
        torch.cuda.synchronize()
        assert torch.equal(y, y_ref) and torch.equal(ls, ls_ref), f"call {call}"


def test_noalloc_rejects_shapes_beyond_the_static_scratch(cuda_device):
    # an explicit split-L schedule over a long, wide problem needs far more
    # scratch than the 16 MiB array: rejected before anything is launched
    import torch
    import selective_state_space_54_b200 as ssm
    from selective_state_space_54_b200 import _lib
    lib = _lib.load()
    shape = ssm.make_shape(64, 8192, 1 << 16, 64, ssm.SSM_BF16, ssm.SSM_PATH_SPLIT_L)
    assert ssm.fwd_workspace_bytes(shape) > (16 << 20)
    buf = torch.zeros(64, dtype=torch.float32, device=cuda_device)
    p = ctypes.c_void_p(buf.data_ptr())
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    rc = lib.ssm_scan_fwd_noalloc(ctypes.byref(shape), p, p, p, p, p, None, None, None, 1, None,
                                  p, None, stream)
    assert rc == _lib.SSM_ERR_UNSUPPORTED
    torch.cuda.synchronize()
    assert torch.count_nonzero(buf).item() == 0  # nothing was written


def test_noalloc_after_a_device_reset(cuda_device):
    # The scratch array's address is looked up on every call, so a device reset
    # between two calls is harmless: the library's self-test runs the entry point,
    # resets the device, reallocates and runs it again, and the two results must be
    # equal bit for bit.  It runs in a child process, because the reset ends the
    # primary context this process's tensors live in.
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    code = ("import sys; sys.path.insert(0, %r); "
            "from selective_state_space_54_b200 import _lib; "
            "print(_lib.load().ssm_scan_test_noalloc_reset_cycle())") % root
    r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout + r.stderr
    assert r.stdout.strip().splitlines()[-1] == "0", r.stdout + r.stderr
