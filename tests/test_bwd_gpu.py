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


def _bwd(case, device, softplus=True, h0=None, want_dh0=False, zoh=False):
    import torch
    import selective_state_space_54_b200 as ssm
    g = upload(case, device)
    h0_t = None if h0 is None else torch.from_numpy(np.asarray(h0, np.float32)).to(device)
    out = ssm.scan_bwd(g["u"], g["delta"], g["A"], g["B"], g["C"], g["D"], g["z"],
                       g["delta_bias"], g["dy"], delta_softplus=softplus, initial_state=h0_t,
                       want_dinitial_state=want_dh0, zoh_exact=zoh)
    torch.cuda.synchronize()
    return {k: (None if v is None else to_f64(v)) for k, v in out.items()}


def _check(case, device, softplus=True, h0=None, zoh=False):
    ref = oracle.bwd(case, case["dy"], delta_softplus=softplus, h0=h0, want_dh0=h0 is not None,
                     zoh_exact=zoh)
    got = _bwd(case, device, softplus, h0, want_dh0=h0 is not None, zoh=zoh)
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
@pytest.mark.parametrize("N", [1, 4, 8, 12, 16, 32, 64])
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


@pytest.mark.parametrize("N", [4, 16])
def test_bwd_over_wide_softplus_and_gate_ranges(cuda_device, N):
    # the raw delta over s in [-30, 30] and z over [-100, 100] in every channel (rolled
    # differently per channel): the softplus derivative sigmoid(s) and the gate's
    # SiLU'(z) at saturation on both sides, every gradient against the oracle
    # (d_state 16 runs the d_state-16 kernel, 4 the general one)
    D, L = 16, 600
    case = _case(1, D, L, N, synth.F32, 71)
    s = np.linspace(-30.0, 30.0, L, dtype=np.float32)
    z = np.linspace(-100.0, 100.0, L, dtype=np.float32)
    case["delta"] = np.stack([np.roll(s, 37 * d) for d in range(D)])[None].astype(np.float32)
    case["z"] = np.stack([np.roll(z, 53 * d) for d in range(D)])[None].astype(np.float32)
    case["delta_bias"] = np.zeros(D, np.float32)  # s as written
    _check(case, cuda_device)


def test_bwd_initial_state_gradient(cuda_device):
    case = _case(2, 32, 300, 16, synth.F32, 6)
    h0 = np.random.default_rng(2).standard_normal((2, 32, 16)).astype(np.float32)
    _check(case, cuda_device, h0=h0)


@pytest.mark.parametrize("N,zoh", [(16, False), (8, False), (16, True), (8, True)])
def test_bwd_bitwise_repeatable(cuda_device, N, zoh):
    # every sum over channels, steps or the batch is formed in a fixed order
    # (per-block partials added by a separate pass, no atomics): two runs give
    # bitwise-equal gradients, the cross-channel ones included
    case = _case(3, 200, 777, N, synth.BF16, 7)
    h0 = np.random.default_rng(8).standard_normal((3, 200, N)).astype(np.float32)
    a = _bwd(case, cuda_device, h0=h0, want_dh0=True, zoh=zoh)
    b = _bwd(case, cuda_device, h0=h0, want_dh0=True, zoh=zoh)
    for k in GRADS + ("dinitial_state",):
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
def _bwd_saved(case, device, h0=None, zoh=False):
    import torch
    import selective_state_space_54_b200 as ssm
    g = upload(case, device)
    h0_t = None if h0 is None else torch.from_numpy(np.asarray(h0, np.float32)).to(device)
    shape = ssm.make_shape(case["batch"], case["dim"], case["seqlen"], case["dstate"],
                           ssm.SSM_BF16 if case["dtype"] == synth.BF16 else ssm.SSM_F32,
                           flags=ssm.SSM_FLAG_SAVE_STATES | (ssm.SSM_FLAG_ZOH_EXACT if zoh else 0))
    ws = torch.empty(ssm.fwd_workspace_bytes(shape), dtype=torch.uint8, device=device)
    y = ssm.scan_fwd(g["u"], g["delta"], g["A"], g["B"], g["C"], g["D"], g["z"], g["delta_bias"],
                     initial_state=h0_t, workspace=ws, save_states=True, zoh_exact=zoh)
    out = ssm.scan_bwd(g["u"], g["delta"], g["A"], g["B"], g["C"], g["D"], g["z"],
                       g["delta_bias"], g["dy"], initial_state=h0_t, fwd_workspace=ws,
                       want_dinitial_state=h0 is not None, zoh_exact=zoh)
    torch.cuda.synchronize()
    return to_f64(y), {k: (None if v is None else to_f64(v)) for k, v in out.items()}


@pytest.mark.parametrize("dtype", [synth.F32, synth.BF16])
@pytest.mark.parametrize("N", [4, 12, 16, 32])
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


# ---- the exact zero-order-hold input term (reading guide, "Metodo") ----------
@pytest.mark.parametrize("dtype", [synth.F32, synth.BF16])
@pytest.mark.parametrize("N", [1, 4, 12, 16, 32])
def test_bwd_zoh_exact(cuda_device, dtype, N):
    # 40 channels (a partial block), 333 steps (a partial chunk), an initial state
    case = _case(2, 40, 333, N, dtype, 650 + N)
    h0 = np.random.default_rng(N + 1).standard_normal((2, 40, N)).astype(np.float32)
    _check(case, cuda_device, h0=h0, zoh=True)


@pytest.mark.parametrize("N", [16, 8])
def test_bwd_zoh_exact_with_saved_states(cuda_device, N):
    # the exact-ZOH training step: the warp-specialised forward saves the chunk
    # states, the backward starts from them
    case = _case(2, 40, 333, N, synth.BF16, 670 + N)
    h0 = np.random.default_rng(N + 2).standard_normal((2, 40, N)).astype(np.float32)
    ref = oracle.bwd(case, case["dy"], h0=h0, want_dh0=True, zoh_exact=True)
    y, got = _bwd_saved(case, cuda_device, h0, zoh=True)
    assert_close(y, oracle.fwd(case, h0=h0, zoh_exact=True)["y"], synth.BF16, "y")
    for k in GRADS:
        assert_close(got[k], ref[k], synth.BF16, k, stored_bf16=k in IO_GRADS)
    assert_close(got["dinitial_state"], ref["dh0"], synth.BF16, "dh0", stored_bf16=False)


def test_bwd_zoh_exact_large_and_zero_steps(cuda_device):
    # Delta A on both sides of the series / closed-form switch, and A_n = 0
    case = _case(1, 32, 200, 16, synth.F32, 660)
    case["delta_bias"] = np.linspace(-6.0, 2.0, 32).astype(np.float32)
    case["A"] = case["A"].copy()
    case["A"][:, 3] = 0.0
    _check(case, cuda_device, zoh=True)


# ---- token-major activations (batch, seqlen, dim), as a projection writes them ----
@pytest.mark.parametrize("batch,dim,L", [(2, 64, 256), (1, 40, 333), (3, 8, 17), (2, 1024, 1000)])
def test_bwd_token_major(cuda_device, batch, dim, L):
    import torch
    import selective_state_space_54_b200 as ssm
    case = _case(batch, dim, L, 16, synth.BF16, 700 + dim)
    g = upload(case, cuda_device)
    cm = ssm.scan_bwd(g["u"], g["delta"], g["A"], g["B"], g["C"], g["D"], g["z"],
                      g["delta_bias"], g["dy"])
    tm = {k: g[k].transpose(1, 2).contiguous() for k in ("u", "delta", "z", "dy")}
    tk = ssm.scan_bwd(tm["u"], tm["delta"], g["A"], g["B"], g["C"], g["D"], tm["z"],
                      g["delta_bias"], tm["dy"], token_major=True)
    torch.cuda.synchronize()
    # the same arithmetic in the same order: only the loads and stores move
    for k in ("du", "ddelta", "dz"):
        assert torch.equal(tk[k].transpose(1, 2), cm[k]), k
    for k in ("dA", "dB", "dC", "dD", "ddelta_bias"):
        assert torch.equal(tk[k], cm[k]), k
    ref = oracle.bwd(case, case["dy"])
    for k in GRADS:
        got = tk[k].transpose(1, 2) if k in ("du", "ddelta", "dz") else tk[k]
        assert_close(to_f64(got), ref[k], synth.BF16, k, stored_bf16=k in IO_GRADS)


def test_bwd_token_major_with_saved_states(cuda_device):
    # the training step on projection-layout activations: the token-major
    # forward saves the chunk states, the token-major backward starts from them
    import torch
    import selective_state_space_54_b200 as ssm
    batch, dim, L = 2, 128, 500
    case = _case(batch, dim, L, 16, synth.BF16, 710)
    g = upload(case, cuda_device)
    tm = {k: g[k].transpose(1, 2).contiguous() for k in ("u", "delta", "z", "dy")}
    shape = ssm.make_shape(batch, dim, L, 16, ssm.SSM_BF16,
                           flags=ssm.SSM_FLAG_SAVE_STATES | ssm.SSM_FLAG_TOKEN_MAJOR)
    ws = torch.empty(ssm.fwd_workspace_bytes(shape), dtype=torch.uint8, device=cuda_device)
    ssm.scan_fwd(tm["u"], tm["delta"], g["A"], g["B"], g["C"], g["D"], tm["z"], g["delta_bias"],
                 workspace=ws, save_states=True, token_major=True)
    got = ssm.scan_bwd(tm["u"], tm["delta"], g["A"], g["B"], g["C"], g["D"], tm["z"],
                       g["delta_bias"], tm["dy"], fwd_workspace=ws, token_major=True)
    torch.cuda.synchronize()
    ref = oracle.bwd(case, case["dy"])
    for k in GRADS:
        v = got[k].transpose(1, 2) if k in ("du", "ddelta", "dz") else got[k]
        assert_close(to_f64(v), ref[k], synth.BF16, k, stored_bf16=k in IO_GRADS)


def test_bwd_writes_only_its_outputs_and_workspace(cuda_device):
    # outputs and the workspace sit inside larger buffers whose margins hold a
    # NaN pattern; the backward must touch none of them (a bounds check
    # without a sanitizer), on both kernels and with saved states
    import torch
    import selective_state_space_54_b200 as ssm
    pad = 4096
    for N, saved in ((16, False), (16, True), (8, False)):
        case = _case(3, 70, 301, N, synth.BF16, 720 + N)
        g = upload(case, cuda_device)
        shape = ssm.make_shape(3, 70, 301, N, ssm.SSM_BF16,
                               flags=ssm.SSM_FLAG_SAVE_STATES if saved else 0)
        fws = None
        if saved:
            fws = torch.empty(ssm.fwd_workspace_bytes(shape), dtype=torch.uint8, device=cuda_device)
            ssm.scan_fwd(g["u"], g["delta"], g["A"], g["B"], g["C"], g["D"], g["z"], g["delta_bias"],
                         workspace=fws, save_states=True)
        nws = ssm.bwd_workspace_bytes(shape)
        wbuf = torch.full((nws + 2 * pad,), 0x7F, dtype=torch.uint8, device=cuda_device)
        ws = wbuf[pad:pad + nws]
        bufs, out = {}, {}
        for k, like in (("du", g["u"]), ("ddelta", g["u"]), ("dz", g["u"]), ("dB", g["B"]), ("dC", g["C"])):
            bufs[k] = torch.full((like.numel() + 2 * pad,), float("nan"), dtype=like.dtype, device=cuda_device)
            out[k] = bufs[k][pad:pad + like.numel()].view(like.shape)
        for k, n in (("dA", 70 * N), ("dD", 70), ("ddelta_bias", 70)):
            bufs[k] = torch.full((n + 2 * pad,), float("nan"), dtype=torch.float32, device=cuda_device)
            out[k] = bufs[k][pad:pad + n].view((70, N) if k == "dA" else (70,))
        ssm.scan_bwd(g["u"], g["delta"], g["A"], g["B"], g["C"], g["D"], g["z"], g["delta_bias"],
                     g["dy"], out=out, workspace=ws, fwd_workspace=fws)
        torch.cuda.synchronize()
        assert (wbuf[:pad] == 0x7F).all() and (wbuf[pad + nws:] == 0x7F).all(), (N, saved, "workspace")
        for k, buf in bufs.items():
            n = out[k].numel()
            assert torch.isnan(buf[:pad].float()).all() and torch.isnan(buf[pad + n:].float()).all(), (N, saved, k)
        ref = oracle.bwd(case, case["dy"])
        for k in GRADS:
            assert_close(to_f64(out[k]), ref[k], synth.BF16, k, stored_bf16=k in IO_GRADS)
