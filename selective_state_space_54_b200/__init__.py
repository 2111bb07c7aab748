"""B200 selective scan (S6): Python binding of libssmscan.so.

Argument marshalling only: torch tensors supply device pointers and the
current CUDA stream; every step of the scan runs in the library's CUDA
kernels (include/ssm_scan.h).  There is no CPU path.

    y, last_state = scan_fwd(u, delta, A, B, C, D, z, delta_bias,
                             delta_softplus=True, return_last_state=True)
    grads = scan_bwd(u, delta, A, B, C, D, z, delta_bias, dout)
    y_t = scan_step(u_t, delta_t, A, B_t, C_t, D, z_t, delta_bias, state=state)

Layouts: u, delta, z, y, dout (batch, dim, seqlen); B, C (batch, seqlen,
dstate); A (dim, dstate) fp32; D, delta_bias (dim,) fp32; states (batch, dim,
dstate) fp32.  io tensors are all bf16 or all fp32.
"""
from __future__ import annotations

import ctypes
import functools

from . import _lib
from ._lib import (PATH_NAMES, SSM_BF16, SSM_F32, SSM_FLAG_SAVE_STATES,  # noqa: F401
                   SSM_FLAG_TOKEN_MAJOR, SSM_FLAG_ZOH_EXACT, SSM_PATH_AUTO,
                   SSM_PATH_LOOKBACK, SSM_PATH_LOOKBACK_WS, SSM_PATH_PER_GROUP, SSM_PATH_SPLIT_L,
                   ssm_shape)

__all__ = ["scan_fwd", "scan_bwd", "scan_step", "causal_conv1d", "causal_conv1d_bwd", "fwd_workspace_bytes", "bwd_workspace_bytes",
           "fwd_path", "check", "ScanError", "make_shape"]


class ScanError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"{what}: {_lib.status_string(code)} ({code})")
        self.code = code


def _io_dtype(t) -> int:
    import torch
    if t.dtype == torch.bfloat16:
        return SSM_BF16
    if t.dtype == torch.float32:
        return SSM_F32
    raise TypeError(f"io tensors must be bfloat16 or float32, got {t.dtype}")


def make_shape(batch: int, dim: int, seqlen: int, dstate: int, io_dtype: int,
               path: int = SSM_PATH_AUTO, lanes: int = 0, flags: int = 0) -> ssm_shape:
    return ssm_shape(batch, dim, seqlen, dstate, io_dtype, path, lanes, flags)


def fwd_workspace_bytes(shape: ssm_shape) -> int:
    return int(_lib.load().ssm_scan_fwd_workspace_bytes(ctypes.byref(shape)))


def bwd_workspace_bytes(shape: ssm_shape) -> int:
    return int(_lib.load().ssm_scan_bwd_workspace_bytes(ctypes.byref(shape)))


def fwd_path(shape: ssm_shape) -> str:
    return PATH_NAMES[int(_lib.load().ssm_scan_fwd_path(ctypes.byref(shape)))]


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    import torch
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _check_io(name, t, shape, dtype, device):
    if t is None:
        return
    # one combined test on the common path; the message is built only on failure
    if t.is_cuda and t.device == device and t.shape == tuple(shape) and t.dtype == dtype and t.is_contiguous():
        return
    if not t.is_cuda or t.device != device:
        raise ValueError(f"{name} must be on {device}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    if t.dtype != dtype:
        raise TypeError(f"{name} has dtype {t.dtype}, expected {dtype}")
    raise ValueError(f"{name} must be contiguous")


def _workspace(nbytes, device, workspace):
    import torch
    if workspace is not None:
        if workspace.numel() * workspace.element_size() < nbytes:
            raise ValueError(f"workspace holds {workspace.nbytes} bytes, needs {nbytes}")
        return workspace
    return torch.empty(max(nbytes, 256), dtype=torch.uint8, device=device)


def scan_fwd(u, delta, A, B, C, D=None, z=None, delta_bias=None, *, delta_softplus=True,
             initial_state=None, y=None, last_state=None, return_last_state=False,
             workspace=None, path: int = SSM_PATH_AUTO, lanes: int = 0, zoh_exact=False,
             save_states=False, token_major=False, check_status=False, stream=None):
    """Forward selective scan; returns y, or (y, last_state).  zoh_exact selects the
    exact zero-order-hold input term instead of the Euler one (Delta * B).
    save_states also writes the state entering every 8-step chunk into
    ``workspace`` (which must then be given), for scan_bwd(fwd_workspace=...).
    token_major: u, delta, z and y are (batch, seqlen, dim) instead.
    The look-back schedules hand states between warps with a bounded wait that
    records a give-up in the workspace's error word instead of trapping:
    check_status=True synchronises after the launch and raises ScanError
    (SSM_ERR_DEVICE_TIMEOUT) if that happened; otherwise pass a workspace and
    call check(workspace) when convenient (an internal workspace is not kept)."""
    import torch
    if token_major:
        batch, seqlen, dim = u.shape
    else:
        batch, dim, seqlen = u.shape
    dstate = B.shape[-1]
    dt = u.dtype
    dev = u.device
    f32 = torch.float32
    act = (batch, seqlen, dim) if token_major else (batch, dim, seqlen)
    _check_io("u", u, act, dt, dev)
    _check_io("delta", delta, act, dt, dev)
    _check_io("z", z, act, dt, dev)
    _check_io("B", B, (batch, seqlen, dstate), dt, dev)
    _check_io("C", C, (batch, seqlen, dstate), dt, dev)
    _check_io("A", A, (dim, dstate), f32, dev)
    _check_io("D", D, (dim,), f32, dev)
    _check_io("delta_bias", delta_bias, (dim,), f32, dev)
    _check_io("initial_state", initial_state, (batch, dim, dstate), f32, dev)
    if y is None:
        y = torch.empty_like(u)
    _check_io("y", y, act, dt, dev)
    if last_state is None and return_last_state:
        last_state = torch.empty((batch, dim, dstate), dtype=f32, device=dev)
    _check_io("last_state", last_state, (batch, dim, dstate), f32, dev)
    flags = ((SSM_FLAG_ZOH_EXACT if zoh_exact else 0) | (SSM_FLAG_SAVE_STATES if save_states else 0)
             | (SSM_FLAG_TOKEN_MAJOR if token_major else 0))
    if save_states and workspace is None:
        raise ValueError("save_states writes into the workspace: pass workspace=")
    shape = make_shape(batch, dim, seqlen, dstate, _io_dtype(u), path, lanes, flags)
    nbytes = fwd_workspace_bytes(shape)
    if nbytes == 0 and batch * dim * seqlen > 0:
        raise ScanError(_lib.SSM_ERR_UNSUPPORTED, "ssm_scan_fwd_workspace_bytes")
    ws = _workspace(nbytes, dev, workspace)
    rc = _lib.load().ssm_scan_fwd(
        ctypes.byref(shape), _ptr(u), _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(z),
        _ptr(delta_bias), int(bool(delta_softplus)), _ptr(initial_state), _ptr(y),
        _ptr(last_state), _ptr(ws), ctypes.c_size_t(ws.numel()), _stream(stream))
    if rc != 0:
        raise ScanError(rc, "ssm_scan_fwd")
    if check_status:
        check(ws, stream)
    if return_last_state:
        return y, last_state
    return y


@functools.lru_cache(maxsize=64)
def _step_shape(batch, dim, dstate, io_dtype, flags):
    # read-only for the library (a const pointer): one struct per shape serves
    # every decode step of that shape
    return make_shape(batch, dim, 1, dstate, io_dtype, flags=flags)


def scan_step(u, delta, A, B, C, D=None, z=None, delta_bias=None, *, state,
              delta_softplus=True, zoh_exact=False, y=None, stream=None):
    """One recurrent step for every (batch, channel): updates `state` in place
    and returns y.  u, delta, z, y (batch, dim); B, C (batch, dstate); state
    (batch, dim, dstate) fp32."""
    import torch
    batch, dim = u.shape
    dstate = B.shape[-1]
    dt = u.dtype
    dev = u.device
    f32 = torch.float32
    _check_io("u", u, (batch, dim), dt, dev)
    _check_io("delta", delta, (batch, dim), dt, dev)
    _check_io("z", z, (batch, dim), dt, dev)
    _check_io("B", B, (batch, dstate), dt, dev)
    _check_io("C", C, (batch, dstate), dt, dev)
    _check_io("A", A, (dim, dstate), f32, dev)
    _check_io("D", D, (dim,), f32, dev)
    _check_io("delta_bias", delta_bias, (dim,), f32, dev)
    _check_io("state", state, (batch, dim, dstate), f32, dev)
    if y is None:
        y = torch.empty_like(u)
    _check_io("y", y, (batch, dim), dt, dev)
    shape = _step_shape(batch, dim, dstate, _io_dtype(u), SSM_FLAG_ZOH_EXACT if zoh_exact else 0)
    rc = _lib.load().ssm_scan_step(
        ctypes.byref(shape), _ptr(u), _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(z),
        _ptr(delta_bias), int(bool(delta_softplus)), _ptr(state), _ptr(y), _stream(stream))
    if rc != 0:
        raise ScanError(rc, "ssm_scan_step")
    return y


def causal_conv1d(x, weight, bias=None, *, initial_state=None, silu=True, out=None,
                  return_final_state=False, final_state=None, stream=None):
    """Causal depthwise conv1d along seqlen (+ SiLU); x, out (batch, dim, seqlen),
    weight (dim, width) fp32, states (batch, dim, width - 1) fp32."""
    import torch
    batch, dim, seqlen = x.shape
    width = weight.shape[-1]
    dev = x.device
    f32 = torch.float32
    _check_io("x", x, (batch, dim, seqlen), x.dtype, dev)
    _check_io("weight", weight, (dim, width), f32, dev)
    _check_io("bias", bias, (dim,), f32, dev)
    _check_io("initial_state", initial_state, (batch, dim, width - 1), f32, dev)
    if out is None:
        out = torch.empty_like(x)
    _check_io("out", out, (batch, dim, seqlen), x.dtype, dev)
    if final_state is None and return_final_state:
        final_state = torch.empty((batch, dim, width - 1), dtype=f32, device=dev)
    _check_io("final_state", final_state, (batch, dim, width - 1), f32, dev)
    rc = _lib.load().ssm_causal_conv1d(
        batch, dim, seqlen, width, _io_dtype(x), _ptr(x), _ptr(weight), _ptr(bias),
        _ptr(initial_state), int(bool(silu)), _ptr(out), _ptr(final_state), _stream(stream))
    if rc != 0:
        raise ScanError(rc, "ssm_causal_conv1d")
    if return_final_state:
        return out, final_state
    return out


def causal_conv1d_bwd(x, weight, bias, dout, *, initial_state=None, silu=True,
                      want_dinitial_state=False, stream=None):
    """Backward of causal_conv1d: returns dict(dx, dweight, dbias, dinitial_state)."""
    import torch
    batch, dim, seqlen = x.shape
    width = weight.shape[-1]
    dev, f32 = x.device, torch.float32
    _check_io("x", x, (batch, dim, seqlen), x.dtype, dev)
    _check_io("dout", dout, (batch, dim, seqlen), x.dtype, dev)
    _check_io("weight", weight, (dim, width), f32, dev)
    _check_io("bias", bias, (dim,), f32, dev)
    _check_io("initial_state", initial_state, (batch, dim, width - 1), f32, dev)
    g = {"dx": torch.empty_like(x), "dweight": torch.empty((dim, width), dtype=f32, device=dev),
         "dbias": torch.empty((dim,), dtype=f32, device=dev) if bias is not None else None,
         "dinitial_state": (torch.empty((batch, dim, width - 1), dtype=f32, device=dev)
                            if want_dinitial_state else None)}
    rc = _lib.load().ssm_causal_conv1d_bwd(
        batch, dim, seqlen, width, _io_dtype(x), _ptr(x), _ptr(weight), _ptr(bias),
        _ptr(initial_state), int(bool(silu)), _ptr(dout), _ptr(g["dx"]), _ptr(g["dweight"]),
        _ptr(g["dbias"]), _ptr(g["dinitial_state"]), _stream(stream))
    if rc != 0:
        raise ScanError(rc, "ssm_causal_conv1d_bwd")
    return g


def scan_bwd(u, delta, A, B, C, D, z, delta_bias, dout, *, delta_softplus=True,
             initial_state=None, want_dinitial_state=False, out=None, workspace=None,
             fwd_workspace=None, zoh_exact=False, token_major=False, stream=None):
    """Backward of scan_fwd by recomputation; returns a dict of gradients.
    fwd_workspace: the workspace of a scan_fwd(save_states=True) call on the same
    inputs, whose saved chunk states the backward then uses.  zoh_exact: the
    exact zero-order-hold input term.  token_major: u, delta, z, dout and the
    du, ddelta, dz gradients are (batch, seqlen, dim)."""
    import torch
    if token_major:
        batch, seqlen, dim = u.shape
    else:
        batch, dim, seqlen = u.shape
    dstate = B.shape[-1]
    dt, dev, f32 = u.dtype, u.device, torch.float32
    act = (batch, seqlen, dim) if token_major else (batch, dim, seqlen)
    for name, t, shp, ty in (("u", u, act, dt), ("delta", delta, act, dt),
                             ("z", z, act, dt), ("B", B, (batch, seqlen, dstate), dt),
                             ("C", C, (batch, seqlen, dstate), dt), ("A", A, (dim, dstate), f32),
                             ("D", D, (dim,), f32), ("delta_bias", delta_bias, (dim,), f32),
                             ("dout", dout, act, dt),
                             ("initial_state", initial_state, (batch, dim, dstate), f32)):
        _check_io(name, t, shp, ty, dev)
    g = dict(out or {})
    g.setdefault("du", torch.empty_like(u))
    g.setdefault("ddelta", torch.empty_like(u))
    g.setdefault("dA", torch.empty((dim, dstate), dtype=f32, device=dev))
    g.setdefault("dB", torch.empty_like(B))
    g.setdefault("dC", torch.empty_like(C))
    g.setdefault("dD", torch.empty((dim,), dtype=f32, device=dev) if D is not None else None)
    g.setdefault("dz", torch.empty_like(u) if z is not None else None)
    g.setdefault("ddelta_bias",
                 torch.empty((dim,), dtype=f32, device=dev) if delta_bias is not None else None)
    g.setdefault("dinitial_state",
                 torch.empty((batch, dim, dstate), dtype=f32, device=dev) if want_dinitial_state else None)
    flags = ((SSM_FLAG_SAVE_STATES if fwd_workspace is not None else 0)
             | (SSM_FLAG_ZOH_EXACT if zoh_exact else 0) | (SSM_FLAG_TOKEN_MAJOR if token_major else 0))
    shape = make_shape(batch, dim, seqlen, dstate, _io_dtype(u), flags=flags)
    nbytes = bwd_workspace_bytes(shape)
    ws = _workspace(nbytes, dev, workspace)
    rc = _lib.load().ssm_scan_bwd(
        ctypes.byref(shape), _ptr(u), _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(z),
        _ptr(delta_bias), int(bool(delta_softplus)), _ptr(initial_state), _ptr(dout),
        _ptr(fwd_workspace), _ptr(g["du"]), _ptr(g["ddelta"]), _ptr(g["dA"]), _ptr(g["dB"]), _ptr(g["dC"]),
        _ptr(g["dD"]), _ptr(g["dz"]), _ptr(g["ddelta_bias"]), _ptr(g["dinitial_state"]),
        _ptr(ws), ctypes.c_size_t(ws.numel()), _stream(stream))
    if rc != 0:
        raise ScanError(rc, "ssm_scan_bwd")
    return g


def check(workspace, stream=None) -> None:
    """Synchronise and raise ScanError if a device-side wait gave up."""
    rc = _lib.load().ssm_scan_check(_ptr(workspace), _stream(stream))
    if rc != 0:
        raise ScanError(rc, "ssm_scan_check")
