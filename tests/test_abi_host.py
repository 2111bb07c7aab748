"""The C ABI without a GPU: the library loads, exports every declared symbol,
and rejects bad arguments with the documented status before any launch."""
import ctypes
import os
import re

import pytest

from selective_state_space_54_b200 import _lib
from selective_state_space_54_b200.build import INCLUDE, LIB, build

HEADER = os.path.join(INCLUDE, "ssm_scan.h")


@pytest.fixture(scope="module")
def lib():
    build()
    return _lib.load()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(ssm_[a-z0-9_]+)\s*\(", text)))


def test_header_and_binding_agree():
    assert sorted(_lib.EXPORTS) == declared_functions()


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_status_strings_and_version(lib):
    assert lib.ssm_status_string(0) == b"ok"
    assert b"timed out" in lib.ssm_status_string(_lib.SSM_ERR_DEVICE_TIMEOUT)
    assert lib.ssm_scan_version() >= 100


def _shape(**kw):
    d = dict(batch=2, dim=16, seqlen=64, dstate=16, io_dtype=_lib.SSM_BF16, path=0)
    d.update(kw)
    return _lib.ssm_shape(**d)


BAD_SHAPES = [
    (dict(batch=-1), _lib.SSM_ERR_INVALID_ARG),
    (dict(dim=-3), _lib.SSM_ERR_INVALID_ARG),
    (dict(seqlen=-1), _lib.SSM_ERR_INVALID_ARG),
    (dict(dstate=0), _lib.SSM_ERR_INVALID_ARG),
    (dict(dstate=65), _lib.SSM_ERR_UNSUPPORTED),
    (dict(io_dtype=7), _lib.SSM_ERR_UNSUPPORTED),
    (dict(path=9), _lib.SSM_ERR_UNSUPPORTED),
]


def _fwd(lib, shape, ptrs=None, ws=None, ws_bytes=0):
    p = dict(u=8, delta=8, A=16, B=8, C=8, D=None, z=None, bias=None, h0=None, y=8, ls=None)
    p.update(ptrs or {})
    v = lambda x: None if x is None else ctypes.c_void_p(x)
    return lib.ssm_scan_fwd(ctypes.byref(shape) if shape is not None else None, v(p["u"]),
                            v(p["delta"]), v(p["A"]), v(p["B"]), v(p["C"]), v(p["D"]), v(p["z"]),
                            v(p["bias"]), 1, v(p["h0"]), v(p["y"]), v(p["ls"]), v(ws), ws_bytes, None)


# argument checks passed: no workspace given (on a machine with a GPU) or no device
ACCEPTED = (_lib.SSM_ERR_WORKSPACE, _lib.SSM_ERR_CUDA)


def test_null_shape_rejected(lib):
    assert _fwd(lib, None) == _lib.SSM_ERR_INVALID_ARG
    assert lib.ssm_scan_fwd_workspace_bytes(None) == 0


@pytest.mark.parametrize("kw,code", BAD_SHAPES)
def test_bad_shapes_rejected(lib, kw, code):
    assert _fwd(lib, _shape(**kw)) == code
    assert lib.ssm_scan_fwd_workspace_bytes(ctypes.byref(_shape(**kw))) == 0
    assert lib.ssm_scan_bwd_workspace_bytes(ctypes.byref(_shape(**kw))) == 0


@pytest.mark.parametrize("missing", ["u", "delta", "A", "B", "C", "y"])
def test_null_required_pointer_rejected(lib, missing):
    assert _fwd(lib, _shape(), {missing: None}) == _lib.SSM_ERR_INVALID_ARG


@pytest.mark.parametrize("which,addr", [("u", 9), ("B", 3), ("A", 18), ("y", 1), ("z", 5),
                                         ("D", 2), ("ls", 6)])
def test_misaligned_pointer_rejected(lib, which, addr):
    assert _fwd(lib, _shape(), {which: addr}) == _lib.SSM_ERR_INVALID_ARG


def test_empty_problem_is_a_noop(lib):
    # batch*dim == 0: nothing to do, nothing touched, even with null pointers
    assert _fwd(lib, _shape(batch=0), {k: None for k in ("u", "delta", "A", "B", "C", "y")}) == 0
    assert _fwd(lib, _shape(dim=0), {k: None for k in ("u", "delta", "A", "B", "C", "y")}) == 0


def test_bwd_rejects_bad_shapes(lib):
    # shape, 8 input pointers, delta_softplus, initial_state, dout, fwd_workspace, 9 outputs,
    # ws, bytes, stream
    for kw, code in BAD_SHAPES:
        sh = _shape(**kw)
        assert lib.ssm_scan_bwd(ctypes.byref(sh), *[None] * 8, 1, *[None] * 12, None, 0, None) == code


def test_product_has_no_oracle_or_cpu_path():
    # the package never imports the oracle and carries no CPU implementation
    pkg = os.path.dirname(LIB)
    for root, _, files in os.walk(pkg):
        for f in files:
            if f.endswith(".py") or f.endswith(".cu") or f.endswith(".cuh"):
                text = open(os.path.join(root, f)).read()
                assert "import oracle" not in text and "from oracle" not in text, f
                assert "ssm_oracle" not in text, f


def _bwd(lib, shape, **over):
    # shape, u, delta, A, B, C, D, z, bias, softplus, h0, dout, fwd_ws,
    # du, ddelta, dA, dB, dC, dD, dz, dbias, dh0, ws, ws_bytes, stream
    p = dict(u=16, delta=16, A=16, B=16, C=16, D=None, z=None, bias=None, h0=None, dout=16, fws=None,
             du=16, ddelta=16, dA=16, dB=16, dC=16, dD=None, dz=None, dbias=None, dh0=None)
    p.update(over)
    v = lambda x: None if x is None else ctypes.c_void_p(x)
    return lib.ssm_scan_bwd(ctypes.byref(shape), v(p["u"]), v(p["delta"]), v(p["A"]), v(p["B"]),
                            v(p["C"]), v(p["D"]), v(p["z"]), v(p["bias"]), 1, v(p["h0"]),
                            v(p["dout"]), v(p["fws"]), v(p["du"]), v(p["ddelta"]), v(p["dA"]), v(p["dB"]),
                            v(p["dC"]), v(p["dD"]), v(p["dz"]), v(p["dbias"]), v(p["dh0"]),
                            None, 0, None)


@pytest.mark.parametrize("over", [dict(z=16), dict(dz=16), dict(D=16), dict(dD=16),
                                  dict(bias=16), dict(dbias=16)])
def test_bwd_gradient_pairs_must_match(lib, over):
    # dz exactly when z, dD exactly when D, ddelta_bias exactly when delta_bias
    assert _bwd(lib, _shape(), **over) == _lib.SSM_ERR_INVALID_ARG


@pytest.mark.parametrize("missing", ["u", "delta", "A", "B", "C", "dout", "du", "ddelta", "dA",
                                     "dB", "dC"])
def test_bwd_null_required_pointer_rejected(lib, missing):
    assert _bwd(lib, _shape(), **{missing: None}) == _lib.SSM_ERR_INVALID_ARG


def test_bwd_misaligned_rejected(lib):
    assert _bwd(lib, _shape(), du=17) == _lib.SSM_ERR_INVALID_ARG  # bf16 needs 2-byte
    assert _bwd(lib, _shape(), dA=6) == _lib.SSM_ERR_INVALID_ARG


def test_noalloc_rejects_bad_shapes_before_launch(lib):
    for kw, code in BAD_SHAPES:
        sh = _shape(**kw)
        rc = lib.ssm_scan_fwd_noalloc(ctypes.byref(sh), *[ctypes.c_void_p(16)] * 5, None, None,
                                      None, 1, None, ctypes.c_void_p(16), None, None)
        assert rc == code


def test_noalloc_flags_checked_before_launch(lib):
    # each flag on the allocation-free entry point, without a GPU: saved states
    # are refused (they would sit in the shared array, out of the backward's
    # reach); the other flags get ssm_scan_fwd's own checks
    def call(**kw):
        sh = _shape(**kw)
        return lib.ssm_scan_fwd_noalloc(ctypes.byref(sh), *[ctypes.c_void_p(16)] * 5, None, None,
                                        None, 1, None, ctypes.c_void_p(16), None, None)
    assert call(flags=_lib.SSM_FLAG_SAVE_STATES) == _lib.SSM_ERR_UNSUPPORTED
    assert call(flags=8) == _lib.SSM_ERR_INVALID_ARG
    assert call(flags=_lib.SSM_FLAG_ZOH_EXACT, path=_lib.SSM_PATH_SPLIT_L) == _lib.SSM_ERR_UNSUPPORTED
    assert call(flags=_lib.SSM_FLAG_TOKEN_MAJOR, io_dtype=_lib.SSM_F32) == _lib.SSM_ERR_UNSUPPORTED
    assert call(flags=_lib.SSM_FLAG_TOKEN_MAJOR, path=_lib.SSM_PATH_LOOKBACK) == \
        _lib.SSM_ERR_UNSUPPORTED


def _step(lib, shape, ptrs=None):
    p = dict(u=8, delta=8, A=16, B=8, C=8, D=None, z=None, bias=None, state=16, y=8)
    p.update(ptrs or {})
    v = lambda x: None if x is None else ctypes.c_void_p(x)
    return lib.ssm_scan_step(ctypes.byref(shape) if shape is not None else None, v(p["u"]),
                             v(p["delta"]), v(p["A"]), v(p["B"]), v(p["C"]), v(p["D"]), v(p["z"]),
                             v(p["bias"]), 1, v(p["state"]), v(p["y"]), None)


def test_step_rejects_bad_shapes_before_launch(lib):
    assert _step(lib, None) == _lib.SSM_ERR_INVALID_ARG
    for kw, code in BAD_SHAPES:
        kw = dict(kw)
        kw.setdefault("seqlen", 1)
        if kw["seqlen"] == -1:
            continue
        assert _step(lib, _shape(**kw)) == code, kw
    # a step is one token: any other seqlen is an error
    for L in (0, 2, 64):
        assert _step(lib, _shape(seqlen=L)) == _lib.SSM_ERR_INVALID_ARG


@pytest.mark.parametrize("missing", ["u", "delta", "A", "B", "C", "state", "y"])
def test_step_null_required_pointer_rejected(lib, missing):
    assert _step(lib, _shape(seqlen=1), {missing: None}) == _lib.SSM_ERR_INVALID_ARG


@pytest.mark.parametrize("which,addr", [("u", 9), ("B", 3), ("A", 18), ("y", 1), ("z", 5),
                                         ("D", 2), ("state", 6)])
def test_step_misaligned_pointer_rejected(lib, which, addr):
    assert _step(lib, _shape(seqlen=1), {which: addr}) == _lib.SSM_ERR_INVALID_ARG


def test_step_empty_problem_is_a_noop(lib):
    nulls = {k: None for k in ("u", "delta", "A", "B", "C", "state", "y")}
    assert _step(lib, _shape(seqlen=1, batch=0), nulls) == 0
    assert _step(lib, _shape(seqlen=1, dim=0), nulls) == 0


def _conv(lib, batch=2, dim=4, L=64, K=4, dtype=_lib.SSM_BF16, **ptrs):
    p = dict(x=16, w=16, bias=None, s0=None, out=16, s1=None)
    p.update(ptrs)
    v = lambda x: None if x is None else ctypes.c_void_p(x)
    return lib.ssm_causal_conv1d(batch, dim, L, K, dtype, v(p["x"]), v(p["w"]), v(p["bias"]),
                                 v(p["s0"]), 1, v(p["out"]), v(p["s1"]), None)


def test_conv_rejects_bad_arguments_before_launch(lib):
    assert _conv(lib, batch=-1) == _lib.SSM_ERR_INVALID_ARG
    assert _conv(lib, L=-1) == _lib.SSM_ERR_INVALID_ARG
    assert _conv(lib, K=0) == _lib.SSM_ERR_INVALID_ARG
    assert _conv(lib, K=9) == _lib.SSM_ERR_UNSUPPORTED
    assert _conv(lib, dtype=5) == _lib.SSM_ERR_UNSUPPORTED
    for k in ("x", "w", "out"):
        assert _conv(lib, **{k: None}) == _lib.SSM_ERR_INVALID_ARG, k
    assert _conv(lib, x=17) == _lib.SSM_ERR_INVALID_ARG
    assert _conv(lib, w=6) == _lib.SSM_ERR_INVALID_ARG
    assert _conv(lib, s1=2) == _lib.SSM_ERR_INVALID_ARG


def test_conv_empty_problem_is_a_noop(lib):
    assert _conv(lib, batch=0, x=None, w=None, out=None) == 0
    assert _conv(lib, dim=0, x=None, w=None, out=None) == 0


def test_flags_checked_before_launch(lib):
    assert _fwd(lib, _shape(flags=8)) == _lib.SSM_ERR_INVALID_ARG  # an unknown bit
    # exact ZOH runs on the two look-back paths; the others are refused
    for path in (_lib.SSM_PATH_LOOKBACK, _lib.SSM_PATH_LOOKBACK_WS):
        assert _fwd(lib, _shape(flags=_lib.SSM_FLAG_ZOH_EXACT, path=path)) in ACCEPTED
    for path in (_lib.SSM_PATH_SPLIT_L, _lib.SSM_PATH_PER_GROUP):
        assert _fwd(lib, _shape(flags=_lib.SSM_FLAG_ZOH_EXACT, path=path)) == \
            _lib.SSM_ERR_UNSUPPORTED
        assert lib.ssm_scan_fwd_workspace_bytes(
            ctypes.byref(_shape(flags=_lib.SSM_FLAG_ZOH_EXACT, path=path))) == 0
    # the backward takes both input terms: exact ZOH passes the argument checks
    # (and stops only at the missing workspace here)
    assert _bwd(lib, _shape(flags=_lib.SSM_FLAG_ZOH_EXACT)) == _lib.SSM_ERR_WORKSPACE


def test_warp_specialised_lanes_checked_before_launch(lib):
    # 4 lanes per channel in the warp-specialised kernel: 5..16 states,
    # channel-major, no saved states
    ws = _lib.SSM_PATH_LOOKBACK_WS
    for N in (1, 4, 17, 32, 64):
        assert _fwd(lib, _shape(path=ws, lanes=4, dstate=N)) == _lib.SSM_ERR_UNSUPPORTED, N
        assert lib.ssm_scan_fwd_workspace_bytes(ctypes.byref(_shape(path=ws, lanes=4, dstate=N))) == 0
    for N in (5, 8, 12, 16):
        assert _fwd(lib, _shape(path=ws, lanes=4, dstate=N)) in ACCEPTED, N
        assert _fwd(lib, _shape(path=ws, lanes=4, dstate=N, flags=_lib.SSM_FLAG_ZOH_EXACT)) in ACCEPTED, N
    assert _fwd(lib, _shape(path=ws, lanes=4, flags=_lib.SSM_FLAG_TOKEN_MAJOR)) == _lib.SSM_ERR_UNSUPPORTED
    assert _fwd(lib, _shape(path=ws, lanes=4, flags=_lib.SSM_FLAG_SAVE_STATES)) == _lib.SSM_ERR_UNSUPPORTED


def test_saved_states_flag_checked_before_launch(lib):
    save, zoh = _lib.SSM_FLAG_SAVE_STATES, _lib.SSM_FLAG_ZOH_EXACT
    # written by the warp-specialised kernel only: 2 lanes, AUTO or LOOKBACK_WS
    assert _fwd(lib, _shape(flags=save | zoh)) in ACCEPTED
    for path in (_lib.SSM_PATH_LOOKBACK, _lib.SSM_PATH_SPLIT_L, _lib.SSM_PATH_PER_GROUP):
        assert _fwd(lib, _shape(flags=save, path=path)) == _lib.SSM_ERR_UNSUPPORTED
    assert _fwd(lib, _shape(flags=save, lanes=4)) == _lib.SSM_ERR_UNSUPPORTED
    # a forward workspace for the backward needs the flag, and 256-byte alignment
    assert _bwd(lib, _shape(), fws=256) == _lib.SSM_ERR_INVALID_ARG
    assert _bwd(lib, _shape(flags=save), fws=272) == _lib.SSM_ERR_INVALID_ARG


def test_token_major_flag_checked_before_launch(lib):
    tok = _lib.SSM_FLAG_TOKEN_MAJOR
    assert _fwd(lib, _shape(flags=tok, io_dtype=_lib.SSM_F32)) == _lib.SSM_ERR_UNSUPPORTED
    assert _fwd(lib, _shape(flags=tok, dim=20)) == _lib.SSM_ERR_UNSUPPORTED
    assert _fwd(lib, _shape(flags=tok | _lib.SSM_FLAG_ZOH_EXACT)) == _lib.SSM_ERR_UNSUPPORTED
    assert _fwd(lib, _shape(flags=tok, path=_lib.SSM_PATH_LOOKBACK)) == _lib.SSM_ERR_UNSUPPORTED
    # the backward takes token-major activations on its d_state-16 kernel (dstate
    # 9..16), bf16, Euler, dim % 8 == 0
    assert _bwd(lib, _shape(flags=tok)) == _lib.SSM_ERR_WORKSPACE
    assert _bwd(lib, _shape(flags=tok, dstate=12)) == _lib.SSM_ERR_WORKSPACE
    assert _bwd(lib, _shape(flags=tok, dstate=32)) == _lib.SSM_ERR_UNSUPPORTED
    assert _bwd(lib, _shape(flags=tok, dstate=8)) == _lib.SSM_ERR_UNSUPPORTED
    assert _bwd(lib, _shape(flags=tok, io_dtype=_lib.SSM_F32)) == _lib.SSM_ERR_UNSUPPORTED
    assert _bwd(lib, _shape(flags=tok, dim=20)) == _lib.SSM_ERR_UNSUPPORTED
    assert _bwd(lib, _shape(flags=tok | _lib.SSM_FLAG_ZOH_EXACT)) == _lib.SSM_ERR_UNSUPPORTED


def test_c_program_against_the_header(lib, tmp_path):
    # the ABI from C: compile a small C caller against include/ssm_scan.h and link it
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    src = os.path.join(os.path.dirname(__file__), "c_abi", "abi_check.c")
    exe = str(tmp_path / "abi_check")
    libdir = os.path.dirname(LIB)
    subprocess.check_call([gcc, "-std=c99", "-Wall", "-Werror", "-I", INCLUDE, src, "-o", exe,
                           "-L", libdir, "-lssmscan", "-Wl,-rpath," + libdir])
    r = subprocess.run([exe], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, r.stderr


def test_conv_bwd_rejects_bad_arguments_before_launch(lib):
    v = lambda x: None if x is None else ctypes.c_void_p(x)

    def call(batch=2, dim=4, L=64, K=4, dtype=_lib.SSM_BF16, x=16, w=16, bias=None, dout=16, dx=16,
             dw=16, db=None):
        return lib.ssm_causal_conv1d_bwd(batch, dim, L, K, dtype, v(x), v(w), v(bias), None, 1,
                                         v(dout), v(dx), v(dw), v(db), None, None)
    assert call(batch=-1) == _lib.SSM_ERR_INVALID_ARG
    assert call(K=9) == _lib.SSM_ERR_UNSUPPORTED
    assert call(bias=16) == _lib.SSM_ERR_INVALID_ARG          # dbias missing
    assert call(dw=None) == _lib.SSM_ERR_INVALID_ARG
    assert call(w=6) == _lib.SSM_ERR_INVALID_ARG


@pytest.mark.parametrize("dstate,blk", [(16, 64), (8, 32), (4, 32)])
def test_bwd_workspace_holds_every_partial(lib, dstate, blk):
    # the backward's workspace must hold, besides the header and the saved
    # states, one dB/dC partial per channel block, batch element, step and
    # (padded) state, and the dA/dD/ddelta_bias partials of every batch
    # element: it grows with the batch (a missing factor here once sent the
    # partial sums past the end of the workspace)
    for batch, dim, L in ((1, 100, 50), (3, 100, 50), (2, 4096, 2048)):
        sh = _shape(batch=batch, dim=dim, seqlen=L, dstate=dstate)
        np_ = 16 if dstate > 8 else (8 if dstate > 4 else 4)
        ckpt = 4 * batch * (4 * -(-dim // 64)) * -(-L // 8) * 16 * np_
        parts = 4 * (-(-dim // blk) * batch * L * 2 * np_ + batch * dim * dstate + 2 * batch * dim)
        assert lib.ssm_scan_bwd_workspace_bytes(ctypes.byref(sh)) >= 256 + ckpt + parts


def test_injected_launch_failure_is_consumed_in_call_order(lib, capfd):
    # ssm_scan_test_fail_next: armed failures replace the first launch of the
    # next calls that pass their checks (nothing is launched); argument errors
    # come first and do not consume one.  Every call here is either rejected
    # by its checks or injected, so none launches.
    conv = lambda batch=2: lib.ssm_causal_conv1d(batch, 4, 64, 4, _lib.SSM_BF16, ctypes.c_void_p(16),
                                                 ctypes.c_void_p(16), None, None, 1,
                                                 ctypes.c_void_p(16), None, None)
    capfd.readouterr()
    lib.ssm_scan_test_fail_next(2)
    assert conv(batch=-1) == _lib.SSM_ERR_INVALID_ARG  # checks first: nothing consumed
    assert conv() == _lib.SSM_ERR_CUDA
    assert conv() == _lib.SSM_ERR_CUDA
    err = capfd.readouterr().err
    assert err.count("launch failure") == 2, err
    lib.ssm_scan_test_fail_next(1)
    lib.ssm_scan_test_fail_next(0)  # disarmed
    assert conv(batch=-1) == _lib.SSM_ERR_INVALID_ARG
    assert "launch failure" not in capfd.readouterr().err
