"""fp64 CPU oracle for the selective scan (S6): ctypes binding.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and
``bench.py`` (its CPU-baseline leg and its reference arm) may import this
package.  The product path (``selective_state_space_54_b200``) never does:
it has no CPU fallback.

The scan's arithmetic lives in ``ssm_oracle.c`` (a plain per-channel loop,
fp64, libm ``exp``/``log1p``/``expm1``); this module widens the stored inputs
to fp64 (exactly), calls it and returns numpy arrays.  See the header of
``ssm_oracle.c`` for the equations and the passages of the Mamba pages they
follow.  The causal convolution of the Mamba block (``conv1d``) is written
here directly in numpy, fp64, as its definition: a sum of shifted inputs.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

from synth import to_f64

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ssm_oracle.c")
_LIB = os.path.join(_HERE, "libssm_oracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile ssm_oracle.c into libssm_oracle.so (gcc, fp contraction off)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-ffp-contract=off", "-fPIC", "-shared",
                               "-o", tmp, _SRC, "-lm", "-lpthread"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        i64, pd, ci = ctypes.c_int64, ctypes.c_void_p, ctypes.c_int
        lib.oracle_fwd.argtypes = [i64] * 4 + [pd] * 9 + [ci, ci, pd, pd, ci]
        lib.oracle_fwd.restype = ci
        lib.oracle_bwd.argtypes = [i64] * 4 + [pd] * 9 + [ci, ci, pd] + [pd] * 9 + [ci]
        lib.oracle_bwd.restype = ci
        _lib = lib
    return _lib


def default_threads() -> int:
    return max(1, os.cpu_count() or 1)


def _f64(x, dtype=None):
    if x is None:
        return None
    if dtype is not None and x.dtype == np.uint16:
        return np.ascontiguousarray(to_f64(x, dtype))
    return np.ascontiguousarray(x, dtype=np.float64)


def _ptr(a):
    return None if a is None else a.ctypes.data


def _inputs(case):
    dt = case["dtype"]
    return dict(
        u=_f64(case["u"], dt), delta=_f64(case["delta"], dt),
        A=_f64(case["A"]), B=_f64(case["B"], dt), C=_f64(case["C"], dt),
        D=_f64(case.get("D")), z=_f64(case.get("z"), dt),
        delta_bias=_f64(case.get("delta_bias")),
    )


def fwd(case: dict, *, delta_softplus: bool = True, zoh_exact: bool = False,
        h0=None, want_last_state: bool = True, nthreads: int | None = None) -> dict:
    """Forward scan of ``case`` (a dict as made by ``synth.make_case``).

    Returns {"y": (batch, dim, seqlen) fp64, "last_state": (batch, dim, dstate)}.
    """
    lib = _load()
    bt, dm, L, N = case["batch"], case["dim"], case["seqlen"], case["dstate"]
    x = _inputs(case)
    h0 = _f64(h0)
    y = np.zeros((bt, dm, L), np.float64)
    ls = np.zeros((bt, dm, N), np.float64) if want_last_state else None
    rc = lib.oracle_fwd(bt, dm, L, N, _ptr(x["u"]), _ptr(x["delta"]), _ptr(x["A"]),
                        _ptr(x["B"]), _ptr(x["C"]), _ptr(x["D"]), _ptr(x["z"]),
                        _ptr(x["delta_bias"]), _ptr(h0), int(delta_softplus),
                        int(zoh_exact), _ptr(y), _ptr(ls), nthreads or default_threads())
    if rc != 0:
        raise RuntimeError(f"oracle_fwd failed: {rc}")
    return {"y": y, "last_state": ls}


def bwd(case: dict, dout, *, delta_softplus: bool = True, zoh_exact: bool = False, h0=None,
        want_dh0: bool = False, nthreads: int | None = None) -> dict:
    """Gradients of sum(dout * y) with respect to every input of ``case``
    (zoh_exact: for the exact zero-order-hold input term)."""
    lib = _load()
    bt, dm, L, N = case["batch"], case["dim"], case["seqlen"], case["dstate"]
    x = _inputs(case)
    dout = _f64(dout, case["dtype"])
    h0 = _f64(h0)
    g = {
        "du": np.zeros((bt, dm, L)), "ddelta": np.zeros((bt, dm, L)),
        "dA": np.zeros((dm, N)), "dB": np.zeros((bt, L, N)), "dC": np.zeros((bt, L, N)),
        "dD": np.zeros((dm,)), "dz": np.zeros((bt, dm, L)) if x["z"] is not None else None,
        "ddelta_bias": np.zeros((dm,)),
        "dh0": np.zeros((bt, dm, N)) if want_dh0 else None,
    }
    rc = lib.oracle_bwd(bt, dm, L, N, _ptr(x["u"]), _ptr(x["delta"]), _ptr(x["A"]),
                        _ptr(x["B"]), _ptr(x["C"]), _ptr(x["D"]), _ptr(x["z"]),
                        _ptr(x["delta_bias"]), _ptr(h0), int(delta_softplus), int(zoh_exact),
                        _ptr(dout),
                        _ptr(g["du"]), _ptr(g["ddelta"]), _ptr(g["dA"]), _ptr(g["dB"]),
                        _ptr(g["dC"]), _ptr(g["dD"]), _ptr(g["dz"]),
                        _ptr(g["ddelta_bias"]), _ptr(g["dh0"]),
                        nthreads or default_threads())
    if rc != 0:
        raise RuntimeError(f"oracle_bwd failed: {rc}")
    return g


def conv1d(x, weight, bias=None, *, dtype=None, initial_state=None, silu: bool = True):
    """Causal depthwise 1-D convolution along seqlen, then SiLU.

    The convolution layer the Mamba block applies to x_proj before the SSM,
    whose output passes through SiLU ("O que e um modelo Mamba?", ibm.com,
    the Mamba block walk-through).  Per channel d, width K:
        out_t = act(bias[d] + sum_k weight[d, k] * x_{t-K+1+k}),
    x_t for t < 0 taken from ``initial_state`` (batch, dim, K-1), zeros if None.
    Returns (out, final_state): out (batch, dim, L) fp64 and the last K-1
    inputs (batch, dim, K-1) fp64, oldest first.
    """
    xs = _f64(x, dtype)
    w = np.asarray(weight, np.float64)
    bt, dm, L = xs.shape
    K = w.shape[1]
    prev = np.zeros((bt, dm, K - 1)) if initial_state is None else \
        np.asarray(initial_state, np.float64).reshape(bt, dm, K - 1)
    xp = np.concatenate([prev, xs], axis=-1)  # x_{-(K-1)} .. x_{L-1}
    out = np.zeros((bt, dm, L))
    for k in range(K):
        out += w[None, :, k, None] * xp[:, :, k:k + L]
    if bias is not None:
        out += np.asarray(bias, np.float64)[None, :, None]
    if silu:
        out = out / (1.0 + np.exp(-out))
    return out, xp[:, :, L:L + K - 1].copy()


def conv1d_bwd(x, weight, bias, dout, *, dtype=None, initial_state=None, silu: bool = True):
    """Gradients of sum(dout * conv1d(x, weight, bias, initial_state, silu)).

    Written from the forward's definition (``conv1d`` above): with
    a_t = bias + sum_k w_k x_{t-K+1+k} and out_t = act(a_t),
        da_t    = dout_t * act'(a_t)           (SiLU'(a) = s (1 + a (1 - s)), s = sigmoid(a))
        dx_s    = sum_k w_k da_{s+K-1-k}       (terms with s+K-1-k < L)
        dw_k    = sum_{b,t} da_t x_{t-K+1+k}   (x_{<0} from the initial state)
        dbias   = sum_{b,t} da_t
    and the initial state's gradient is dx for the K-1 inputs before t = 0.
    Returns a dict of fp64 arrays: dx, dweight, dbias, dinitial_state.
    """
    xs = _f64(x, dtype)
    g = _f64(dout, dtype)
    w = np.asarray(weight, np.float64)
    bt, dm, L = xs.shape
    K = w.shape[1]
    prev = np.zeros((bt, dm, K - 1)) if initial_state is None else \
        np.asarray(initial_state, np.float64).reshape(bt, dm, K - 1)
    xp = np.concatenate([prev, xs], axis=-1)          # x_{-(K-1)} .. x_{L-1}
    a = np.zeros((bt, dm, L))
    for k in range(K):
        a += w[None, :, k, None] * xp[:, :, k:k + L]
    if bias is not None:
        a += np.asarray(bias, np.float64)[None, :, None]
    if silu:
        sg = 1.0 / (1.0 + np.exp(-a))
        da = g * sg * (1.0 + a * (1.0 - sg))
    else:
        da = g
    dxp = np.zeros((bt, dm, L + K - 1))              # gradient of every entry of xp
    for k in range(K):
        dxp[:, :, k:k + L] += w[None, :, k, None] * da
    dw = np.stack([(da * xp[:, :, k:k + L]).sum(axis=(0, 2)) for k in range(K)], axis=1)
    return {"dx": dxp[:, :, K - 1:], "dweight": dw, "dbias": da.sum(axis=(0, 2)),
            "dinitial_state": dxp[:, :, :K - 1].copy()}
