"""Helpers shared by the GPU tests: upload seeded cases, compare with the oracle."""
from __future__ import annotations

import numpy as np

import synth

# Tolerances of the selective-scan contract (all-fp32 path; bf16-input paths).
TOL_F32_REL_L2 = 1e-5
TOL_BF16_REL_L2 = 2e-3
TOL_BF16_MAXABS_FRAC = 1e-2


def to_torch(x, dtype: str, device):
    """numpy input (bf16 bits as uint16, or fp32) -> torch tensor on device."""
    import torch
    if x is None:
        return None
    if x.dtype == np.uint16:
        return torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).to(device).view(torch.bfloat16)
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(device)


def upload(case: dict, device) -> dict:
    dt = case["dtype"]
    out = {}
    for k in ("u", "delta", "z", "B", "C", "dy"):
        out[k] = to_torch(case.get(k), dt, device)
    for k in ("A", "D", "delta_bias"):
        v = case.get(k)
        out[k] = None if v is None else to_torch(np.asarray(v, np.float32), synth.F32, device)
    return out


def to_f64(t) -> np.ndarray:
    import torch
    return t.detach().to(torch.float64).cpu().numpy()


def rel_l2(got: np.ndarray, ref: np.ndarray) -> float:
    den = np.linalg.norm(ref.ravel())
    return float(np.linalg.norm((got - ref).ravel()) / (den if den > 0 else 1.0))


def assert_close(got: np.ndarray, ref: np.ndarray, dtype: str, what: str = "") -> dict:
    r = rel_l2(got, ref)
    mx = float(np.max(np.abs(got - ref))) if ref.size else 0.0
    scale = float(np.max(np.abs(ref))) if ref.size else 0.0
    assert np.all(np.isfinite(got)), f"{what}: non-finite values"
    if dtype == synth.F32:
        assert r <= TOL_F32_REL_L2, f"{what}: rel-L2 {r:.3e} > {TOL_F32_REL_L2}"
    else:
        assert r <= TOL_BF16_REL_L2, f"{what}: rel-L2 {r:.3e} > {TOL_BF16_REL_L2}"
        assert mx <= TOL_BF16_MAXABS_FRAC * scale, \
            f"{what}: max-abs {mx:.3e} > {TOL_BF16_MAXABS_FRAC} * {scale:.3e}"
    return {"rel_l2": r, "max_abs": mx, "max_ref": scale}
