"""Single-step (decode) parity: ssm_scan_step through the C ABI against the
fp64 oracle's scan of one token from a given state, and against the scan over
many tokens (the recurrence fed one token at a time)."""
import numpy as np
import pytest

import oracle
import synth
from gpu_util import assert_close, to_f64, upload

pytestmark = pytest.mark.gpu


def _state(batch, dim, N, seed):
    return np.random.default_rng(seed).standard_normal((batch, dim, N)).astype(np.float32)


def _step_inputs(g, t):
    """Token t of an uploaded case, in the step layouts."""
    return {k: (None if g[k] is None else g[k][:, :, t].contiguous()) for k in ("u", "delta", "z")} | \
           {k: g[k][:, t, :].contiguous() for k in ("B", "C")}


def _run_step(case, device, h0, softplus=True, t=0, state=None):
    import torch
    import selective_state_space_54_b200 as ssm
    g = upload(case, device)
    x = _step_inputs(g, t)
    st = state if state is not None else torch.from_numpy(h0).to(device)
    y = ssm.scan_step(x["u"], x["delta"], g["A"], x["B"], x["C"], g["D"], x["z"], g["delta_bias"],
                      state=st, delta_softplus=softplus)
    torch.cuda.synchronize()
    return to_f64(y), to_f64(st)


def _check(case, device, h0, softplus=True):
    ref = oracle.fwd(case, h0=h0, delta_softplus=softplus)
    y, st = _run_step(case, device, h0, softplus)
    assert_close(y, ref["y"][:, :, 0], case["dtype"], "y")
    # the state is fp32 arithmetic on exact inputs: fp32 tolerance on every path
    assert_close(st, ref["last_state"], synth.F32, "state")


@pytest.mark.parametrize("dtype", [synth.F32, synth.BF16])
@pytest.mark.parametrize("N", [1, 3, 4, 5, 8, 12, 16, 32, 33, 64])
def test_step_dstate_sizes(cuda_device, dtype, N):
    case = synth.make_case(3, 70, 1, N, dtype, seed=300 + N)
    _check(case, cuda_device, _state(3, 70, N, N))


@pytest.mark.parametrize("opt", ["no_z", "no_D", "no_bias", "no_softplus", "bare"])
def test_step_optional_terms(cuda_device, opt):
    kw = dict(with_z=opt not in ("no_z", "bare"), with_D=opt not in ("no_D", "bare"),
              with_bias=opt not in ("no_bias", "bare"))
    case = synth.make_case(2, 64, 1, 16, synth.F32, seed=31, **kw)
    softplus = opt != "no_softplus"
    if not softplus:
        case["delta"] = np.abs(case["delta"]) * 0.05 + 1e-3
        case["delta_bias"] = None
    _check(case, cuda_device, _state(2, 64, 16, 3), softplus=softplus)


@pytest.mark.parametrize("what", ["softplus", "gate"])
def test_step_over_wide_softplus_and_gate_ranges(cuda_device, what):
    # one token, one value per channel: with a zero state, Abar = 0, B = u = 1 and
    # C = 1/16 over 16 states, y = softplus(s) (no gate) over s in [-30, 30], or
    # y = SiLU(z) (Delta = 1 without softplus) over z in [-200, 200], element by element
    D, N = 1024, 16
    v = np.linspace(-30.0, 30.0, D) if what == "softplus" else np.linspace(-200.0, 200.0, D)
    v = v.astype(np.float32).reshape(1, D, 1)
    case = {"batch": 1, "dim": D, "seqlen": 1, "dstate": N, "dtype": synth.F32,
            "u": np.ones((1, D, 1), np.float32),
            "delta": v if what == "softplus" else np.ones((1, D, 1), np.float32),
            "A": np.full((D, N), -1e30, np.float32), "B": np.ones((1, 1, N), np.float32),
            "C": np.full((1, 1, N), 1.0 / N, np.float32), "D": None,
            "z": None if what == "softplus" else v, "delta_bias": None}
    softplus = what == "softplus"
    ref = oracle.fwd(case, delta_softplus=softplus)["y"][0, :, 0]
    y, _ = _run_step(case, cuda_device, np.zeros((1, D, N), np.float32), softplus=softplus)
    y = y[0]
    assert np.all(np.isfinite(y))
    if softplus:  # relative accuracy of the softplus, as for the scan
        bound = (1e-6 + 1e-7 * np.abs(v.ravel().astype(np.float64))) * ref
    else:         # SiLU; far on the negative side any value below 1e-15
        bound = 2e-6 * np.abs(ref) + 1e-15
    err = np.abs(y - ref)
    assert np.all(err <= bound), (what, float((err / bound).max()))


@pytest.mark.parametrize("batch,dim", [(1, 1), (1, 7), (5, 33), (2, 1000)])
def test_step_ragged_channel_counts(cuda_device, batch, dim):
    case = synth.make_case(batch, dim, 1, 16, synth.BF16, seed=batch * 1000 + dim)
    _check(case, cuda_device, _state(batch, dim, 16, dim))


# Blocks own a channel slice (128 channels at d_state 16) and walk the batch
# rows kb, kb + bps, ... with bps blocks per slice: one row per block, rows
# split unevenly between blocks (odd and even counts through the two row
# buffers), and more slices than the SMs hold (every block walks every row).
@pytest.mark.parametrize("dtype", [synth.BF16, synth.F32])
@pytest.mark.parametrize("batch,dim", [(7, 2000), (300, 130), (900, 130), (3, 100000)])
def test_step_rows_per_block(cuda_device, dtype, batch, dim):
    case = synth.make_case(batch, dim, 1, 16, dtype, seed=batch + dim)
    _check(case, cuda_device, _state(batch, dim, 16, batch))


def test_step_state_only_16_byte_aligned(cuda_device):
    # the state 16 bytes past a 32-byte boundary: two 16-byte accesses per
    # lane instead of one 32-byte access
    import torch
    batch, dim, N = 5, 300, 16
    case = synth.make_case(batch, dim, 1, N, synth.BF16, seed=17)
    h0 = _state(batch, dim, N, 11)
    buf = torch.zeros(h0.size + 8, dtype=torch.float32, device=cuda_device)
    assert buf.data_ptr() % 32 == 0
    st = buf[4:4 + h0.size].view(batch, dim, N)
    st.copy_(torch.from_numpy(h0))
    ref = oracle.fwd(case, h0=h0, delta_softplus=True)
    y, st = _run_step(case, cuda_device, h0, state=st)
    assert_close(y, ref["y"][:, :, 0], case["dtype"], "y")
    assert_close(st, ref["last_state"], synth.F32, "state")
    assert torch.all(buf[:4] == 0) and torch.all(buf[4 + h0.size:] == 0)


def test_step_zero_state_matches_scan_of_one_token(cuda_device):
    case = synth.make_case(2, 48, 1, 16, synth.BF16, seed=9)
    _check(case, cuda_device, np.zeros((2, 48, 16), np.float32))


def test_steps_equal_the_scan(cuda_device):
    # feeding L tokens one at a time reproduces the scan over the L tokens
    import torch
    import selective_state_space_54_b200 as ssm
    batch, dim, L, N = 2, 96, 64, 16
    case = synth.make_case(batch, dim, L, N, synth.F32, seed=12)
    h0 = _state(batch, dim, N, 4)
    ref = oracle.fwd(case, h0=h0)
    g = upload(case, cuda_device)
    st = torch.from_numpy(h0).to(cuda_device)
    ys = []
    for t in range(L):
        x = _step_inputs(g, t)
        ys.append(ssm.scan_step(x["u"], x["delta"], g["A"], x["B"], x["C"], g["D"], x["z"],
                                g["delta_bias"], state=st))
    y = torch.stack(ys, dim=-1)
    y_scan, ls_scan = ssm.scan_fwd(g["u"], g["delta"], g["A"], g["B"], g["C"], g["D"], g["z"],
                                   g["delta_bias"], initial_state=torch.from_numpy(h0).to(cuda_device),
                                   return_last_state=True)
    torch.cuda.synchronize()
    assert_close(to_f64(y), ref["y"], synth.F32, "stepped y")
    assert_close(to_f64(st), ref["last_state"], synth.F32, "stepped state")
    assert_close(to_f64(y), to_f64(y_scan), synth.F32, "stepped vs scan y")
    assert_close(to_f64(st), to_f64(ls_scan), synth.F32, "stepped vs scan state")


def test_step_reset_and_hold(cuda_device):
    # a huge Delta resets the state (exp underflows to 0); Delta = 0 holds it exactly
    import torch
    import selective_state_space_54_b200 as ssm
    case = synth.make_case(1, 32, 1, 16, synth.F32, seed=13, with_bias=False)
    h0 = _state(1, 32, 16, 5)
    g = upload(case, cuda_device)
    x = _step_inputs(g, 0)
    big = torch.full_like(x["delta"], 1e4)
    st = torch.from_numpy(h0).to(cuda_device)
    ssm.scan_step(x["u"], big, g["A"], x["B"], x["C"], g["D"], x["z"], None, state=st,
                  delta_softplus=False)
    expect = (1e4 * case["u"][0, :, 0, None].astype(np.float64) * case["B"][0, 0][None, :])
    torch.cuda.synchronize()
    np.testing.assert_allclose(to_f64(st)[0], expect, rtol=1e-6)
    st2 = torch.from_numpy(h0).to(cuda_device)
    zero = torch.zeros_like(x["delta"])
    ssm.scan_step(x["u"], zero, g["A"], x["B"], x["C"], g["D"], x["z"], None, state=st2,
                  delta_softplus=False)
    torch.cuda.synchronize()
    assert np.array_equal(to_f64(st2), h0.astype(np.float64))


def test_step_writes_only_its_outputs(cuda_device):
    import torch
    import selective_state_space_54_b200 as ssm
    batch, dim, N, pad = 3, 45, 12, 4096
    case = synth.make_case(batch, dim, 1, N, synth.BF16, seed=14)
    g = upload(case, cuda_device)
    x = _step_inputs(g, 0)
    h0 = _state(batch, dim, N, 6)
    sbuf = torch.full((pad + h0.size + pad,), 7.25, dtype=torch.float32, device=cuda_device)
    st = sbuf[pad:pad + h0.size].view(batch, dim, N)
    st.copy_(torch.from_numpy(h0))
    ybuf = torch.full((pad + batch * dim + pad,), 3.5, dtype=torch.bfloat16, device=cuda_device)
    y = ybuf[pad:pad + batch * dim].view(batch, dim)
    ssm.scan_step(x["u"], x["delta"], g["A"], x["B"], x["C"], g["D"], x["z"], g["delta_bias"],
                  state=st, y=y)
    torch.cuda.synchronize()
    assert torch.all(sbuf[:pad] == 7.25) and torch.all(sbuf[pad + h0.size:] == 7.25)
    assert torch.all(ybuf[:pad] == 3.5) and torch.all(ybuf[pad + batch * dim:] == 3.5)
    ref = oracle.fwd(case, h0=h0)
    assert_close(to_f64(st), ref["last_state"], synth.F32, "state")


def test_step_full_decode_workload(cuda_device):
    # the Mamba-2.8B decode shape at full size, every output against the oracle
    w = synth.WORKLOADS["mamba-2.8b-decode"]
    case = synth.make_workload(w)
    h0 = _state(w.batch, w.dim, w.dstate, 7)
    _check(case, cuda_device, h0)



@pytest.mark.parametrize("N", [4, 16, 12])
def test_step_zoh_exact_matches_oracle(cuda_device, N):
    import torch
    import selective_state_space_54_b200 as ssm
    case = synth.make_case(3, 64, 1, N, synth.F32, seed=500 + N)
    case["delta_bias"] = np.linspace(-4, 2, 64).astype(np.float32)  # both (e^x - 1)/x branches
    h0 = _state(3, 64, N, 9)
    ref = oracle.fwd(case, h0=h0, zoh_exact=True)
    g = upload(case, cuda_device)
    x = _step_inputs(g, 0)
    st = torch.from_numpy(h0).to(cuda_device)
    y = ssm.scan_step(x["u"], x["delta"], g["A"], x["B"], x["C"], g["D"], x["z"], g["delta_bias"],
                      state=st, zoh_exact=True)
    torch.cuda.synchronize()
    assert_close(to_f64(y), ref["y"][:, :, 0], synth.F32, "y")
    assert_close(to_f64(st), ref["last_state"], synth.F32, "state")


def test_step_batch_far_beyond_the_resident_blocks(cuda_device):
    # a batch far above the blocks that fit on the GPU (270000 rows of one
    # channel): each block walks several hundred rows
    batch, dim, N = 270000, 1, 16
    case = synth.make_case(batch, dim, 1, N, synth.BF16, seed=16)
    _check(case, cuda_device, _state(batch, dim, N, 10))


def test_step_rejects_bad_arguments(cuda_device):
    # the binding checks every tensor before the call: wrong device, shape,
    # dtype or layout raise, and nothing is launched (the state is untouched)
    import torch
    import selective_state_space_54_b200 as ssm
    batch, dim, N = 2, 40, 16
    case = synth.make_case(batch, dim, 1, N, synth.BF16, seed=18)
    g = upload(case, cuda_device)
    x = _step_inputs(g, 0)
    st = torch.from_numpy(_state(batch, dim, N, 12)).to(cuda_device)
    keep = st.clone()

    def call(**over):
        a = dict(u=x["u"], delta=x["delta"], A=g["A"], B=x["B"], C=x["C"], D=g["D"], z=x["z"],
                 delta_bias=g["delta_bias"])
        a.update(over)
        return ssm.scan_step(a["u"], a["delta"], a["A"], a["B"], a["C"], a["D"], a["z"], a["delta_bias"],
                             state=over.get("state", st))

    with pytest.raises(ValueError, match="must be on"):
        call(delta=x["delta"].cpu())
    with pytest.raises(ValueError, match="has shape"):
        call(z=x["z"][:, :-1].contiguous())
    with pytest.raises(TypeError, match="has dtype"):
        call(D=g["D"].double())
    with pytest.raises(ValueError, match="contiguous"):
        call(state=torch.empty((batch, N, dim), device=cuda_device).transpose(1, 2))
    torch.cuda.synchronize()
    assert torch.equal(st, keep)
    call()  # and the same arguments, corrected, run
    torch.cuda.synchronize()
    assert not torch.equal(st, keep)
