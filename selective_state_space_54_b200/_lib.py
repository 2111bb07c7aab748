"""ctypes view of libssmscan.so (the C ABI in include/ssm_scan.h).

The library is built in-tree by ``selective_state_space_54_b200.build``.
Loading fails loudly when it is missing: there is no fallback.
"""
from __future__ import annotations

import ctypes
import os

from .build import LIB

SSM_OK = 0
SSM_ERR_INVALID_ARG = -1
SSM_ERR_UNSUPPORTED = -2
SSM_ERR_WORKSPACE = -3
SSM_ERR_CUDA = -4
SSM_ERR_DEVICE_TIMEOUT = -5

SSM_F32 = 0
SSM_BF16 = 1

SSM_PATH_AUTO = 0
SSM_PATH_LOOKBACK = 1
SSM_PATH_SPLIT_L = 2
SSM_PATH_PER_GROUP = 3
SSM_PATH_LOOKBACK_WS = 4

SSM_FLAG_ZOH_EXACT = 1
SSM_FLAG_SAVE_STATES = 2
SSM_FLAG_TOKEN_MAJOR = 4

PATH_NAMES = {SSM_PATH_AUTO: "auto", SSM_PATH_LOOKBACK: "lookback",
              SSM_PATH_SPLIT_L: "split_l", SSM_PATH_PER_GROUP: "per_group",
              SSM_PATH_LOOKBACK_WS: "lookback_ws"}

# every symbol include/ssm_scan.h declares
EXPORTS = (
    "ssm_scan_fwd_workspace_bytes", "ssm_scan_bwd_workspace_bytes", "ssm_scan_fwd",
    "ssm_scan_bwd", "ssm_scan_check", "ssm_scan_test_wait_timeout", "ssm_scan_fwd_path",
    "ssm_status_string", "ssm_scan_version", "ssm_scan_fwd_noalloc", "ssm_scan_step",
    "ssm_causal_conv1d", "ssm_causal_conv1d_bwd", "ssm_scan_test_fail_next",
    "ssm_scan_test_noalloc_reset_cycle",
)


class ssm_shape(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int64), ("dim", ctypes.c_int64),
                ("seqlen", ctypes.c_int64), ("dstate", ctypes.c_int64),
                ("io_dtype", ctypes.c_int32), ("path", ctypes.c_int32),
                ("lanes", ctypes.c_int32), ("flags", ctypes.c_int32)]


_lib = None


def load(path: str | None = None):
    """Load libssmscan.so and declare the C signatures; raises if it is missing."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    p = path or LIB
    if not os.path.exists(p):
        raise RuntimeError(
            f"libssmscan.so not found at {p}; build it with "
            "`python -m selective_state_space_54_b200.build` (nvcc, sm_100a)")
    lib = ctypes.CDLL(p)
    vp, sz, ci, i64, i32 = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int, ctypes.c_int64, ctypes.c_int32
    shp = ctypes.POINTER(ssm_shape)
    lib.ssm_scan_fwd_workspace_bytes.argtypes = [shp]
    lib.ssm_scan_fwd_workspace_bytes.restype = sz
    lib.ssm_scan_bwd_workspace_bytes.argtypes = [shp]
    lib.ssm_scan_bwd_workspace_bytes.restype = sz
    lib.ssm_scan_fwd.argtypes = [shp, vp, vp, vp, vp, vp, vp, vp, vp, ci, vp, vp, vp, vp, sz, vp]
    lib.ssm_scan_fwd.restype = ci
    lib.ssm_scan_bwd.argtypes = ([shp, vp, vp, vp, vp, vp, vp, vp, vp, ci, vp, vp, vp]
                                 + [vp] * 9 + [vp, sz, vp])
    lib.ssm_scan_bwd.restype = ci
    lib.ssm_scan_fwd_noalloc.argtypes = [shp, vp, vp, vp, vp, vp, vp, vp, vp, ci, vp, vp, vp, vp]
    lib.ssm_scan_fwd_noalloc.restype = ci
    lib.ssm_scan_step.argtypes = [shp, vp, vp, vp, vp, vp, vp, vp, vp, ci, vp, vp, vp]
    lib.ssm_scan_step.restype = ci
    lib.ssm_causal_conv1d.argtypes = [i64, i64, i64, i32, i32, vp, vp, vp, vp, ci, vp, vp, vp]
    lib.ssm_causal_conv1d.restype = ci
    lib.ssm_causal_conv1d_bwd.argtypes = [i64, i64, i64, i32, i32, vp, vp, vp, vp, ci, vp, vp, vp, vp,
                                          vp, vp]
    lib.ssm_causal_conv1d_bwd.restype = ci
    lib.ssm_scan_check.argtypes = [vp, vp]
    lib.ssm_scan_check.restype = ci
    lib.ssm_scan_test_wait_timeout.argtypes = [vp, sz, i64, vp]
    lib.ssm_scan_test_wait_timeout.restype = ci
    lib.ssm_scan_test_fail_next.argtypes = [i32]
    lib.ssm_scan_test_fail_next.restype = None
    lib.ssm_scan_test_noalloc_reset_cycle.argtypes = []
    lib.ssm_scan_test_noalloc_reset_cycle.restype = i32
    lib.ssm_scan_fwd_path.argtypes = [shp]
    lib.ssm_scan_fwd_path.restype = i32
    lib.ssm_status_string.argtypes = [ci]
    lib.ssm_status_string.restype = ctypes.c_char_p
    lib.ssm_scan_version.argtypes = []
    lib.ssm_scan_version.restype = i32
    if path is None:
        _lib = lib
    return lib


def status_string(code: int) -> str:
    return load().ssm_status_string(code).decode()
