"""Backward parity: ssm_scan_bwd through the C ABI against the fp64 oracle.

Every gradient the contract names (du, ddelta, dA, dB, dC, dD, dz,
ddelta_bias, and dinitial_state) is compared element by element with the
oracle's analytic backward, which the CPU tests pin to finite differences.
"""
import numpy as np
import pytest

import oracle
import synth
from gpu_util import assert_close, to_f64, upload

pytestmark = pytest.mark.gpu

GRADS = ("du", "ddelta", "dA", "dB", "dC", "dD", "dz", "ddelta_bias")
# gradients stored in the io dtype; the others are fp32 on every path
IO_GRADS = ("du", "ddelta", "dB", "dC", "dz")


def _bwd(case, device, softplus=True, h0=None, want_dh0=False):
    import torch
    import selective_state_space_54_b200 as ssm
    g = upload(case, device)
    h0_t = None if h0 is None else torch.from_numpy(np.asarray(h0, np.float32)).to(device)
    out = ssm.scan_bwd(g["u"], g["delta"], g["A"], g["B"], g["C"], g["D"], g["z"],
                       g["delta_bias"], g["dy"], delta_softplus=softplus, initial_state=h0_t,
                       want_dinitial_state=want_dh0)
    torch.cuda.synchronize()
    return {k: (None if v is None else to_f64(v)) for k, v in out.items()}


def _check(case, device, softplus=True, h0=None):
    ref = oracle.bwd(case, case["dy"], delta_softplus=softplus, h0=h0, want_dh0=h0 is not None)
    got = _bwd(case, device, softplus, h0, want_dh0=h0 is not None)
    stats = {}
    for k in GRADS:
        if ref.get(k) is None or (k == "dD" and case.get("D") is None) or \
                (k == "ddelta_bias" and case.get("delta_bias") is None) or \
                (k == "dz" and case.get("z") is None):
            continue
        # fp32 sums of bf16-path terms take the bf16-path tolerance
        stats[k] = assert_close(got[k], ref[k], case["dtype"], k, stored_bf16=k in IO_GRADS)
    if h0 is not None:
        stats["dh0"] = assert_close(got["dinitial_state"], ref["dh0"], case["dtype"], "dh0",
                                    stored_bf16=False)
    return stats


def _case(batch, dim, L, N, dtype, seed, **kw):
    c = synth.make_case(batch, dim, L, N, dtype, seed=seed, with_dy=True, **kw)
    return c


@pytest.mark.parametrize("dtype", [synth.F32, synth.BF16])
@pytest.mark.parametrize("N", [1, 4, 8, 16, 32])
def test_bwd_dstate_sizes(cuda_device, dtype, N):
    _check(_case(2, 40, 150, N, dtype, 200 + N), cuda_device)


@pytest.mark.parametrize("L", [1, 5, 16, 17, 63, 64, 333, 1024])
def test_bwd_ragged_lengths(cuda_device, L):
    _check(_case(2, 36, L, 16, synth.BF16, L), cuda_device)


@pytest.mark.parametrize("opt", ["no_z", "no_D", "no_bias", "no_softplus", "bare"])
def test_bwd_optional_terms(cuda_device, opt):
    kw = dict(with_z=opt not in ("no_z", "bare"), with_D=opt not in ("no_D", "bare"),
              with_bias=opt not in ("no_bias", "bare"))
    case = _case(2, 32, 200, 16, synth.F32, 5, **kw)
    softplus = opt != "no_softplus"
    if not softplus:
        case["delta"] = np.abs(case["delta"]) * 0.05 + 1e-3
        case["delta_bias"] = None
    _check(case, cuda_device, softplus=softplus)


def test_bwd_initial_state_gradient(cuda_device):
    case = _case(2, 32, 300, 16, synth.F32, 6)
    h0 = np.random.default_rng(2).standard_normal((2, 32, 16)).astype(np.float32)
    _check(case, cuda_device, h0=h0)


def test_bwd_deterministic_per_channel_outputs(cuda_device):
    # du, ddelta, dz involve no cross-channel sums: bitwise repeatable
    case = _case(2, 64, 512, 16, synth.BF16, 7)
    a = _bwd(case, cuda_device)
    b = _bwd(case, cuda_device)
    for k in ("du", "ddelta", "dz"):
        assert np.array_equal(a[k], b[k]), k


def test_bwd_full_mamba_1p4b_layer(cuda_device):
    # the training workload at full size, every gradient against the full oracle
    w = synth.WORKLOADS["mamba-1.4b-layer-train"]
    case = synth.make_workload(w)
    stats = _check(case, cuda_device)
    assert set(stats) >= {"du", "ddelta", "dA", "dB", "dC", "dD", "dz", "ddelta_bias"}


def test_bwd_single_step_and_single_channel(cuda_device):
    _check(_case(1, 1, 1, 16, synth.F32, 78), cuda_device)
    _check(_case(1, 3, 2, 4, synth.BF16, 79), cuda_device)


# ---- states saved by the forward (the chunk checkpoints of the training step) ----
def _bwd_saved(case, device, h0=None):
    import torch
    import selective_state_space_54_b200 as ssm
    g = upload(case, device)
    h0_t = None if h0 is None else torch.from_numpy(np.asarray(h0, np.float32)).to(device)
    shape = ssm.make_shape(case["batch"], case["dim"], case["seqlen"], case["dstate"],
                           ssm.SSM_BF16 if case["dtype"] == synth.BF16 else ssm.SSM_F32,
                           flags=ssm.SSM_FLAG_SAVE_STATES)
    ws = torch.empty(ssm.fwd_workspace_bytes(shape), dtype=torch.uint8, device=device)
    y = ssm.scan_fwd(g["u"], g["delta"], g["A"], g["B"], g["C"], g["D"], g["z"], g["delta_bias"],
                     initial_state=h0_t, workspace=ws, save_states=True)
    out = ssm.scan_bwd(g["u"], g["delta"], g["A"], g["B"], g["C"], g["D"], g["z"],
                       g["delta_bias"], g["dy"], initial_state=h0_t, fwd_workspace=ws,
                       want_dinitial_state=h0 is not None)
    torch.cuda.synchronize()
    return to_f64(y), {k: (None if v is None else to_f64(v)) for k, v in out.items()}


@pytest.mark.parametrize("dtype", [synth.F32, synth.BF16])
@pytest.mark.parametrize("N", [4, 16, 32])
def test_bwd_with_saved_states(cuda_device, dtype, N):
    # 40 channels: a partial 32-channel block; 333 steps: a partial 16-step chunk
    case = _case(2, 40, 333, N, dtype, 600 + N)
    h0 = np.random.default_rng(N).standard_normal((2, 40, N)).astype(np.float32)
    ref = oracle.bwd(case, case["dy"], h0=h0, want_dh0=True)
    y, got = _bwd_saved(case, cuda_device, h0)
    assert_close(y, oracle.fwd(case, h0=h0)["y"], dtype, "y")
    for k in GRADS:
        assert_close(got[k], ref[k], dtype, k, stored_bf16=k in IO_GRADS)
    assert_close(got["dinitial_state"], ref["dh0"], dtype, "dh0", stored_bf16=False)


def test_bwd_saved_states_agree_with_recomputed(cuda_device):
    case = _case(2, 64, 512, 16, synth.F32, 610)
    _, saved = _bwd_saved(case, cuda_device)
    recomputed = _bwd(case, cuda_device)
    for k in GRADS:
        assert_close(saved[k], recomputed[k], synth.F32, k)


def test_bwd_full_mamba_1p4b_layer_with_saved_states(cuda_device):
    w = synth.WORKLOADS["mamba-1.4b-layer-train"]
    case = synth.make_workload(w)
    ref = oracle.bwd(case, case["dy"])
    _, got = _bwd_saved(case, cuda_device)
    for k in GRADS:
        assert_close(got[k], ref[k], case["dtype"], k, stored_bf16=k in IO_GRADS)
