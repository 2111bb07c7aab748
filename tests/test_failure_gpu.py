"""Error paths through the real entry points on a GPU, with an injected launch
failure (ssm_scan_test_fail_next): the call returns SSM_ERR_CUDA, launches
nothing, leaves its outputs untouched, and the next call runs normally and
gives the same result as one that never saw a failure."""
import numpy as np
import pytest

import synth
from gpu_util import to_f64, upload

pytestmark = pytest.mark.gpu


def _arm(n):
    from selective_state_space_54_b200 import _lib
    _lib.load().ssm_scan_test_fail_next(n)


def test_injected_failure_forward_backward_step_conv(cuda_device):
    import torch
    import selective_state_space_54_b200 as ssm
    case = synth.make_case(2, 64, 300, 16, synth.BF16, seed=81, with_dy=True)
    g = upload(case, cuda_device)
    args = (g["u"], g["delta"], g["A"], g["B"], g["C"], g["D"], g["z"], g["delta_bias"])
    ref_y = to_f64(ssm.scan_fwd(*args))
    ref_g = {k: to_f64(v) for k, v in ssm.scan_bwd(*args, g["dy"]).items() if v is not None}

    y = torch.full_like(g["u"], 7.0)
    _arm(1)
    with pytest.raises(ssm.ScanError) as ei:
        ssm.scan_fwd(*args, y=y)
    assert ei.value.code == ssm._lib.SSM_ERR_CUDA
    torch.cuda.synchronize()
    assert torch.all(y == 7.0)  # nothing ran
    assert np.array_equal(to_f64(ssm.scan_fwd(*args, y=y)), ref_y)

    _arm(1)
    with pytest.raises(ssm.ScanError):
        ssm.scan_bwd(*args, g["dy"])
    got = ssm.scan_bwd(*args, g["dy"])
    for k, v in ref_g.items():
        assert np.array_equal(to_f64(got[k]), v), k

    state = torch.zeros((2, 64, 16), device=cuda_device)
    step_args = (g["u"][:, :, 0].contiguous(), g["delta"][:, :, 0].contiguous(), g["A"],
                 g["B"][:, 0, :].contiguous(), g["C"][:, 0, :].contiguous(), g["D"],
                 g["z"][:, :, 0].contiguous(), g["delta_bias"])
    _arm(1)
    with pytest.raises(ssm.ScanError):
        ssm.scan_step(*step_args, state=state)
    torch.cuda.synchronize()
    assert torch.all(state == 0)  # the state was not advanced
    ssm.scan_step(*step_args, state=state)
    assert torch.any(state != 0)

    w = torch.randn((64, 4), device=cuda_device)
    ref_c = to_f64(ssm.causal_conv1d(g["u"], w, g["D"]))
    _arm(1)
    with pytest.raises(ssm.ScanError):
        ssm.causal_conv1d(g["u"], w, g["D"])
    assert np.array_equal(to_f64(ssm.causal_conv1d(g["u"], w, g["D"])), ref_c)
    _arm(0)
