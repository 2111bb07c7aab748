"""Forward parity: the CUDA path through the C ABI against the fp64 oracle.

Small cases span several 32-step chunks, ragged chunk tails, ragged 8-channel
groups and every dstate padding; the named workloads run at their full sizes
in the launch configuration the benchmark uses and are checked on every
output element (the million-length workload on its 64 seeded channels over
the full length).  Every forward reads the workspace's device error word.
"""
import numpy as np
import pytest

import oracle
import synth
from gpu_util import assert_close, to_f64, upload

pytestmark = pytest.mark.gpu

PATHS = {"auto": 0, "lookback": 1, "split_l": 2, "per_group": 3, "lookback_ws": 4}
# every schedule with every lane split it supports
PATH_LANES = [("lookback", 2), ("lookback", 4), ("split_l", 2), ("split_l", 4),
              ("per_group", 2), ("per_group", 4), ("lookback_ws", 2), ("lookback_ws", 4)]


def _run(case, device, path="auto", softplus=True, h0=None, last=True, y_out=None, lanes=0,
         zoh=False):
    """One forward through the C ABI with an explicit workspace, whose device
    error word is read afterwards: a bounded look-back wait that gave up
    fails the test instead of passing silently."""
    import torch
    import selective_state_space_54_b200 as ssm
    g = upload(case, device)
    h0_t = None if h0 is None else torch.from_numpy(np.asarray(h0, np.float32)).to(device)
    shape = ssm.make_shape(case["batch"], case["dim"], case["seqlen"], case["dstate"],
                           ssm.SSM_BF16 if case["dtype"] == synth.BF16 else ssm.SSM_F32,
                           PATHS[path], lanes, ssm.SSM_FLAG_ZOH_EXACT if zoh else 0)
    ws = torch.empty(max(256, ssm.fwd_workspace_bytes(shape)), dtype=torch.uint8, device=device)
    y, ls = ssm.scan_fwd(g["u"], g["delta"], g["A"], g["B"], g["C"], g["D"], g["z"],
                         g["delta_bias"], delta_softplus=softplus, initial_state=h0_t,
                         return_last_state=True, path=PATHS[path], y=y_out, lanes=lanes,
                         zoh_exact=zoh, workspace=ws)
    ssm.check(ws)  # synchronises; raises on a device-side wait that gave up
    return to_f64(y), to_f64(ls)


def _check(case, device, path="auto", softplus=True, h0=None, lanes=0):
    ref = oracle.fwd(case, delta_softplus=softplus, h0=h0)
    y, ls = _run(case, device, path, softplus, h0, lanes=lanes)
    st = assert_close(y, ref["y"], case["dtype"], f"y[{path}]")
    # the state is fp32 on both io dtypes
    assert_close(ls, ref["last_state"], case["dtype"], f"last_state[{path}]", stored_bf16=False)
    return st


@pytest.mark.parametrize("path", ["auto", "lookback", "split_l", "per_group", "lookback_ws"])
def test_tiny_fp32_workload(cuda_device, path):
    case = synth.make_workload("tiny-fp32")
    _check(case, cuda_device, path)


@pytest.mark.parametrize("lanes", [2, 4])
@pytest.mark.parametrize("dtype", [synth.F32, synth.BF16])
@pytest.mark.parametrize("N", [1, 3, 4, 8, 12, 16, 32, 64])
def test_dstate_sizes(cuda_device, dtype, N, lanes):
    case = synth.make_case(2, 20, 200, N, dtype, seed=100 + N)
    _check(case, cuda_device, "per_group", lanes=lanes)


@pytest.mark.parametrize("path,lanes", PATH_LANES)
@pytest.mark.parametrize("L", [1, 7, 15, 16, 17, 31, 32, 33, 257, 1000, 1003])
def test_ragged_lengths_and_groups(cuda_device, path, L, lanes):
    # dim 44: ragged 16- and 8-channel groups; L odd -> scalar loads
    case = synth.make_case(3, 44, L, 16, synth.BF16, seed=L)
    _check(case, cuda_device, path, lanes=lanes)


@pytest.mark.parametrize("path,lanes", PATH_LANES)
def test_fp32_several_chunks(cuda_device, path, lanes):
    case = synth.make_case(2, 24, 777, 16, synth.F32, seed=7)
    _check(case, cuda_device, path, lanes=lanes)


@pytest.mark.parametrize("path", ["auto", "lookback_ws"])
@pytest.mark.parametrize("opt", ["no_z", "no_D", "no_bias", "no_softplus", "bare"])
def test_optional_terms(cuda_device, opt, path):
    kw = dict(with_z=opt not in ("no_z", "bare"), with_D=opt not in ("no_D", "bare"),
              with_bias=opt not in ("no_bias", "bare"))
    case = synth.make_case(2, 16, 300, 16, synth.F32, seed=3, **kw)
    softplus = opt != "no_softplus"
    if not softplus:
        # raw delta must stay positive without softplus (|Abar| <= 1)
        case["delta"] = np.abs(case["delta"]) * 0.05 + 1e-3
        case["delta_bias"] = None
    _check(case, cuda_device, path, softplus=softplus)


@pytest.mark.parametrize("path,lanes", PATH_LANES)
def test_initial_state(cuda_device, path, lanes):
    case = synth.make_case(2, 16, 500, 16, synth.F32, seed=9)
    h0 = np.random.default_rng(1).standard_normal((2, 16, 16)).astype(np.float32)
    _check(case, cuda_device, path, h0=h0, lanes=lanes)


def test_check_status_after_the_forward(cuda_device):
    # check_status=True synchronises and reads the error word of the (internal)
    # workspace: a healthy look-back forward returns normally and matches one without it
    import selective_state_space_54_b200 as ssm
    case = synth.make_case(8, 1536, 300, 16, synth.BF16, seed=71)
    g = upload(case, cuda_device)
    args = (g["u"], g["delta"], g["A"], g["B"], g["C"], g["D"], g["z"], g["delta_bias"])
    y0 = ssm.scan_fwd(*args)
    y1 = ssm.scan_fwd(*args, check_status=True)
    assert to_f64(y0).tobytes() == to_f64(y1).tobytes()


def test_continuation_matches_one_scan(cuda_device):
    # scan(L1) -> last_state -> scan(L2 from it) == scan(L1 + L2), on the GPU
    import torch
    import selective_state_space_54_b200 as ssm
    case = synth.make_case(2, 16, 640, 16, synth.F32, seed=21)
    g = upload(case, cuda_device)
    y_full, ls_full = ssm.scan_fwd(g["u"], g["delta"], g["A"], g["B"], g["C"], g["D"], g["z"],
                                   g["delta_bias"], return_last_state=True)
    cut = 320
    part = lambda t, lo, hi: t[..., lo:hi].contiguous()
    y1, ls1 = ssm.scan_fwd(part(g["u"], 0, cut), part(g["delta"], 0, cut), g["A"],
                           g["B"][:, :cut].contiguous(), g["C"][:, :cut].contiguous(), g["D"],
                           part(g["z"], 0, cut), g["delta_bias"], return_last_state=True)
    y2, ls2 = ssm.scan_fwd(part(g["u"], cut, 640), part(g["delta"], cut, 640), g["A"],
                           g["B"][:, cut:].contiguous(), g["C"][:, cut:].contiguous(), g["D"],
                           part(g["z"], cut, 640), g["delta_bias"], initial_state=ls1,
                           return_last_state=True)
    torch.cuda.synchronize()
    got = torch.cat([y1, y2], dim=-1)
    assert torch.allclose(got, y_full, rtol=1e-5, atol=1e-5)
    assert torch.allclose(ls2, ls_full, rtol=1e-5, atol=1e-5)


def test_large_delta_reset_bitwise(cuda_device):
    # Reading guide, "Perguntas": a large Delta resets the state.  exp2 of a
    # huge negative argument is exactly 0 in fp32 too, so outputs from t0 on
    # must not depend on anything before t0, bit for bit.
    case = synth.make_case(1, 16, 200, 16, synth.F32, seed=5, with_bias=False)
    t0 = 97
    case["delta"] = np.abs(case["delta"]) * 0.1 + 1e-3
    case["delta"][:, :, t0] = 1e4
    y0, ls0 = _run(case, cuda_device, "per_group", softplus=False)
    c2 = dict(case)
    rng = np.random.default_rng(3)
    c2["u"] = case["u"].copy()
    c2["u"][:, :, :t0] += rng.standard_normal((1, 16, t0)).astype(np.float32)
    c2["B"] = case["B"].copy()
    c2["B"][:, :t0] *= 3.0
    y1, ls1 = _run(c2, cuda_device, "per_group", softplus=False)
    assert np.array_equal(y0[..., t0:], y1[..., t0:])
    assert np.array_equal(ls0, ls1)


def test_paths_agree(cuda_device):
    case = synth.make_case(4, 64, 2048, 16, synth.BF16, seed=31)
    ref = oracle.fwd(case)["y"]
    outs = {(p, ln): _run(case, cuda_device, p, lanes=ln)[0] for p, ln in PATH_LANES}
    for k, y in outs.items():
        assert_close(y, ref, case["dtype"], str(k))
        d = np.max(np.abs(y - outs[("lookback", 2)]))
        assert d <= 2e-2 * np.max(np.abs(ref)), (k, d)


def test_softplus_accuracy_through_the_kernel(cuda_device):
    # N=1, B=1, C=1, u=1, no D, no gate, and A so negative that Abar = 0 at
    # every step: then h_t = Delta_t and y_t = Delta_t = softplus(s_t) exactly,
    # so the device softplus is checked against the oracle's log1p(exp(s))
    # over s in [-30, 30], element by element.
    L = 4096
    s = np.linspace(-30.0, 30.0, L).astype(np.float32)
    case = {"batch": 1, "dim": 1, "seqlen": L, "dstate": 1, "dtype": synth.F32,
            "u": np.ones((1, 1, L), np.float32), "delta": s.reshape(1, 1, L),
            "A": np.full((1, 1), -1e30, np.float32), "B": np.ones((1, L, 1), np.float32),
            "C": np.ones((1, L, 1), np.float32), "D": None, "z": None, "delta_bias": None}
    ref = oracle.fwd(case)["y"][0, 0]
    assert np.all(ref > 0)
    for lanes in (2, 4):
        y, _ = _run(case, cuda_device, "per_group", lanes=lanes)
        rel = np.abs(y[0, 0] - ref) / ref
        # exp(-|s|) is 2^(-|s| log2 e): the fp32 rounding of that argument
        # alone allows |s| * 6e-8 * ln 2 relative error
        bound = 1e-6 + 1e-7 * np.abs(s.astype(np.float64))
        assert np.all(rel <= bound), (lanes, float(rel.max()), float(s[np.argmax(rel / bound)]))


@pytest.mark.parametrize("path,lanes", PATH_LANES)
def test_softplus_accuracy_on_every_path(cuda_device, path, lanes):
    # the construction of the test above through every schedule (the warp-specialised
    # producer has its own packed softplus), with 8 equal states and C = 1/8 so that
    # every lane split runs: y_t = 8 (Delta_t / 8) = softplus(s_t) exactly
    L, N = 4096, 8
    s = np.linspace(-30.0, 30.0, L).astype(np.float32)
    case = {"batch": 1, "dim": 1, "seqlen": L, "dstate": N, "dtype": synth.F32,
            "u": np.ones((1, 1, L), np.float32), "delta": s.reshape(1, 1, L),
            "A": np.full((1, N), -1e30, np.float32), "B": np.ones((1, L, N), np.float32),
            "C": np.full((1, L, N), 1.0 / N, np.float32), "D": None, "z": None, "delta_bias": None}
    ref = oracle.fwd(case)["y"][0, 0]
    y, _ = _run(case, cuda_device, path, lanes=lanes)
    rel = np.abs(y[0, 0] - ref) / ref
    bound = 1e-6 + 1e-7 * np.abs(s.astype(np.float64))
    assert np.all(rel <= bound), (path, lanes, float(rel.max()), float(s[np.argmax(rel / bound)]))


@pytest.mark.parametrize("path,lanes", PATH_LANES)
def test_gate_over_a_wide_range(cuda_device, path, lanes):
    # y_t = yss_t * SiLU(z_t) with yss_t = 1 (Abar = 0, Delta = 1 without softplus,
    # B = u = 1 and C = 1/8 over 8 states): y is SiLU(z) itself, for z over [-200, 200].
    # Far on the negative side SiLU is below 1e-15 and e^-z overflows fp32: there the
    # kernels may return any value of that size (the warp-specialised gate clamps
    # 1 + e^-z at 2^64)
    L, N = 4096, 8
    z = np.linspace(-200.0, 200.0, L).astype(np.float32)
    case = {"batch": 1, "dim": 1, "seqlen": L, "dstate": N, "dtype": synth.F32,
            "u": np.ones((1, 1, L), np.float32), "delta": np.ones((1, 1, L), np.float32),
            "A": np.full((1, N), -1e30, np.float32), "B": np.ones((1, L, N), np.float32),
            "C": np.full((1, L, N), 1.0 / N, np.float32), "D": None, "z": z.reshape(1, 1, L),
            "delta_bias": None}
    ref = oracle.fwd(case, delta_softplus=False)["y"][0, 0]
    y, _ = _run(case, cuda_device, path, softplus=False, lanes=lanes)
    err = np.abs(y[0, 0] - ref)
    bound = 2e-6 * np.abs(ref) + 1e-15
    assert np.all(np.isfinite(y)), (path, lanes)
    assert np.all(err <= bound), (path, lanes, float((err / bound).max()), float(z[np.argmax(err / bound)]))


@pytest.mark.parametrize("path,lanes", [("lookback", 0), ("lookback_ws", 2), ("lookback_ws", 4)])
def test_deterministic(cuda_device, path, lanes):
    case = synth.make_case(2, 64, 1024, 16, synth.BF16, seed=41)
    a = _run(case, cuda_device, path, lanes=lanes)
    b = _run(case, cuda_device, path, lanes=lanes)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


def test_lookback_splits_groups_between_warps(cuda_device):
    # enough channel groups for several warps per SM sub-partition, with a
    # length whose chunk count does not divide evenly: warp shares start and
    # end inside groups, so the carried states are exercised on both paths
    case = synth.make_case(8, 1536, 1000, 16, synth.BF16, seed=61)
    ref = oracle.fwd(case)
    for path, lanes in (("lookback", 0), ("lookback_ws", 2), ("lookback_ws", 4)):
        y, ls = _run(case, cuda_device, path, lanes=lanes)
        assert_close(y, ref["y"], case["dtype"], f"{path}/{lanes}")
        assert_close(ls, ref["last_state"], case["dtype"], f"{path}/{lanes}", stored_bf16=False)


def test_guard_bands_untouched(cuda_device):
    # y is written into the middle of a larger buffer whose margins hold a
    # NaN pattern; the kernel must not touch them (bounds check without a sanitizer)
    import torch
    case = synth.make_case(2, 20, 333, 16, synth.BF16, seed=51)
    n = 2 * 20 * 333
    pad = 4096
    buf = torch.full((n + 2 * pad,), float("nan"), dtype=torch.bfloat16, device=cuda_device)
    y_view = buf[pad:pad + n].view(2, 20, 333)
    ref = oracle.fwd(case)
    y, _ = _run(case, cuda_device, "auto", y_out=y_view)
    assert_close(y, ref["y"], case["dtype"], "y")
    assert torch.isnan(buf[:pad].float()).all() and torch.isnan(buf[pad + n:].float()).all()


def test_wait_timeout_reports_status(cuda_device):
    # the bounded inter-warp wait gives up, records the error and the context stays usable
    import ctypes
    import torch
    import selective_state_space_54_b200 as ssm
    from selective_state_space_54_b200 import _lib
    lib = _lib.load()
    ws = torch.zeros(256, dtype=torch.uint8, device=cuda_device)
    s = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    assert lib.ssm_scan_test_wait_timeout(ctypes.c_void_p(ws.data_ptr()), 256, 20000, s) == 0
    assert lib.ssm_scan_check(ctypes.c_void_p(ws.data_ptr()), s) == _lib.SSM_ERR_DEVICE_TIMEOUT
    assert lib.ssm_scan_check(ctypes.c_void_p(ws.data_ptr()), s) == 0  # cleared
    _check(synth.make_workload("tiny-fp32"), cuda_device)  # still works
    del ssm


# ---- the named workloads at full size ---------------------------------------
def _forward_full_size(name, device):
    """Run the workload at full size in the benchmark's launch configuration
    (path AUTO, inputs resident on the device) and return the case and the
    device outputs as fp64 host arrays, after reading the error word."""
    import torch
    import selective_state_space_54_b200 as ssm
    w = synth.WORKLOADS[name]
    case = synth.make_workload(w)
    g = upload(case, device)
    shape = ssm.make_shape(w.batch, w.dim, w.seqlen, w.dstate,
                           ssm.SSM_BF16 if w.dtype == synth.BF16 else ssm.SSM_F32)
    ws = torch.empty(ssm.fwd_workspace_bytes(shape), dtype=torch.uint8, device=device)
    y, ls = ssm.scan_fwd(g["u"], g["delta"], g["A"], g["B"], g["C"], g["D"], g["z"],
                         g["delta_bias"], return_last_state=True, workspace=ws)
    ssm.check(ws)
    del g
    return w, case, to_f64(y), to_f64(ls)


def _every_element(name, device):
    """The whole y and last_state against the fp64 oracle, one batch element
    at a time (bounded host memory), with the contract's tolerances applied
    to the totals: rel-L2 <= 2e-3 and max-abs <= 1e-2 max|ref| on y (bf16),
    rel-L2 <= 2e-3 on the fp32 state."""
    w, case, y, ls = _forward_full_size(name, device)
    acc = {"y": [0.0, 0.0, 0.0, 0.0], "last_state": [0.0, 0.0, 0.0, 0.0]}  # err2, ref2, maxerr, maxref
    for b in range(w.batch):
        _, dims, sub = synth.subset_case(case, np.arange(b * w.dim, (b + 1) * w.dim))[0]
        ref = oracle.fwd(sub)
        for k, got in (("y", y[b:b + 1]), ("last_state", ls[b:b + 1])):
            r = ref[k]
            assert np.all(np.isfinite(got)), f"{name} {k} b={b}: non-finite"
            a = acc[k]
            a[0] += float(np.sum((got - r) ** 2))
            a[1] += float(np.sum(r ** 2))
            a[2] = max(a[2], float(np.max(np.abs(got - r))))
            a[3] = max(a[3], float(np.max(np.abs(r))))
        del ref, sub
    out = {}
    for k, (e2, r2, me, mr) in acc.items():
        rel = (e2 / r2) ** 0.5
        out[k] = rel
        print(f"{name} {k}: rel-L2 {rel:.3e} over every element, max-abs {me:.3e} (max|ref| {mr:.3e})")
        assert rel <= 2e-3, f"{name} {k}: rel-L2 {rel:.3e} > 2e-3"
        if k == "y":
            assert me <= 1e-2 * mr, f"{name} y: max-abs {me:.3e} > 1e-2 * {mr:.3e}"
    return out


def test_full_mamba_130m_layer(cuda_device):
    _every_element("mamba-130m-layer", cuda_device)


def test_full_mamba_2p8b_layer(cuda_device):
    _every_element("mamba-2.8b-layer", cuda_device)


def test_full_mamba_1p4b_layer_forward(cuda_device):
    _every_element("mamba-1.4b-layer-train", cuda_device)


def test_full_million_length(cuda_device):
    # the seeded 64 channels over the full 2^20 steps (the oracle is serial in t)
    w, case, y, ls = _forward_full_size("million-length", cuda_device)
    chans = synth.sample_channels(w)
    for b, dims, sub in synth.subset_case(case, chans):
        ref = oracle.fwd(sub)
        st = assert_close(y[b, dims][None], ref["y"], case["dtype"], f"million-length y b={b}")
        assert_close(ls[b, dims][None], ref["last_state"], case["dtype"],
                     f"million-length last_state b={b}", stored_bf16=False)
        print(f"million-length y: rel-L2 {st['rel_l2']:.3e} on {len(dims)} channels")


# ---- exact zero-order hold (the reading guide's "Metodo" discretisation) ----
def _run_zoh(case, device, path="auto", lanes=0, h0=None):
    return _run(case, device, path, lanes=lanes, h0=h0, zoh=True)


@pytest.mark.parametrize("lanes", [0, 2, 4])
@pytest.mark.parametrize("dtype", [synth.F32, synth.BF16])
@pytest.mark.parametrize("N", [1, 4, 16, 64])
def test_zoh_exact_matches_oracle(cuda_device, dtype, N, lanes):
    case = synth.make_case(2, 40, 333, N, dtype, seed=400 + N)
    ref = oracle.fwd(case, zoh_exact=True)
    y, ls = _run_zoh(case, cuda_device, "lookback" if lanes else "auto", lanes)
    assert_close(y, ref["y"], dtype, "y")
    assert_close(ls, ref["last_state"], dtype, "last_state", stored_bf16=False)


@pytest.mark.parametrize("dtype,N", [(synth.F32, 4), (synth.F32, 16), (synth.BF16, 4),
                                     (synth.BF16, 16), (synth.BF16, 64)])
def test_zoh_exact_warp_specialised(cuda_device, dtype, N):
    # the warp-specialised look-back kernel with the exact input term, on a
    # ragged shape (partial 16-channel group, partial chunk) with an initial state
    case = synth.make_case(2, 40, 333, N, dtype, seed=420 + N)
    h0 = np.random.default_rng(N).standard_normal((2, 40, N)).astype(np.float32)
    ref = oracle.fwd(case, zoh_exact=True, h0=h0)
    y, ls = _run_zoh(case, cuda_device, "lookback_ws", 2, h0=h0)
    assert_close(y, ref["y"], dtype, "y")
    assert_close(ls, ref["last_state"], dtype, "last_state", stored_bf16=False)


@pytest.mark.parametrize("dtype", [synth.F32, synth.BF16])
@pytest.mark.parametrize("N", [5, 8, 12, 16])
def test_warp_specialised_four_lanes(cuda_device, dtype, N):
    # 8-channel groups, 4 lanes per channel (2 or 4 states each): ragged
    # channel group (dim 44), ragged chunk, initial state; Euler and exact ZOH
    case = synth.make_case(2, 44, 333, N, dtype, seed=450 + N)
    h0 = np.random.default_rng(N).standard_normal((2, 44, N)).astype(np.float32)
    for zoh in (False, True):
        ref = oracle.fwd(case, zoh_exact=zoh, h0=h0)
        y, ls = _run(case, cuda_device, "lookback_ws", h0=h0, lanes=4, zoh=zoh)
        assert_close(y, ref["y"], dtype, f"y zoh={zoh}")
        assert_close(ls, ref["last_state"], dtype, f"last_state zoh={zoh}", stored_bf16=False)


def test_warp_specialised_four_lanes_limits(cuda_device):
    # 4 lanes per channel in the warp-specialised kernel: 5..16 states only,
    # and AUTO takes it where 16-channel groups are too few (the Mamba-130M layer)
    import selective_state_space_54_b200 as ssm
    for N, ok in ((4, False), (5, True), (16, True), (17, False), (64, False)):
        shape = ssm.make_shape(2, 64, 256, N, ssm.SSM_BF16, ssm.SSM_PATH_LOOKBACK_WS, 4)
        assert (ssm.fwd_workspace_bytes(shape) > 0) == ok, N
    assert ssm.fwd_path(ssm.make_shape(8, 1536, 2048, 16, ssm.SSM_BF16)) == "lookback_ws"


def test_auto_warp_specialised_with_fewer_groups_than_subpartitions(cuda_device):
    # batch 6 x d_inner 1536: 576 groups of 16 channels, at least 3/4 of the
    # SM sub-partitions of a B200 but fewer than all: AUTO takes the
    # warp-specialised kernel with one look-back worker per group
    import torch
    import selective_state_space_54_b200 as ssm
    sms = torch.cuda.get_device_properties(cuda_device).multi_processor_count
    groups = 6 * 1536 // 16
    if not (4 * groups >= 3 * 4 * sms and groups < 4 * sms):
        pytest.skip("shape chosen for a 148-SM device")
    assert ssm.fwd_path(ssm.make_shape(6, 1536, 300, 16, ssm.SSM_BF16)) == "lookback_ws"
    case = synth.make_case(6, 1536, 300, 16, synth.BF16, seed=470)
    ref = oracle.fwd(case)
    y, ls = _run(case, cuda_device)
    assert_close(y, ref["y"], synth.BF16, "y")
    assert_close(ls, ref["last_state"], synth.BF16, "last_state", stored_bf16=False)


def test_zoh_exact_auto_picks_warp_specialised(cuda_device):
    # a Mamba-layer-like shape: AUTO takes the warp-specialised kernel for ZOH too
    import selective_state_space_54_b200 as ssm
    case = synth.make_case(4, 5120, 160, 16, synth.BF16, seed=430)
    shape = ssm.make_shape(4, 5120, 160, 16, ssm.SSM_BF16, flags=ssm.SSM_FLAG_ZOH_EXACT)
    assert ssm.fwd_path(shape) == "lookback_ws"
    ref = oracle.fwd(case, zoh_exact=True)
    y, ls = _run_zoh(case, cuda_device)
    assert_close(y, ref["y"], synth.BF16, "y")
    assert_close(ls, ref["last_state"], synth.BF16, "last_state", stored_bf16=False)


def test_warp_specialised_capacity_fallback(cuda_device):
    # fp32 with 64 states does not fit the warp-specialised kernel's shared
    # memory: an explicit request is refused, AUTO takes the plain look-back
    # kernel on a shape where it would otherwise pick the specialised one
    import selective_state_space_54_b200 as ssm
    explicit = ssm.make_shape(4, 5120, 64, 64, ssm.SSM_F32, ssm.SSM_PATH_LOOKBACK_WS)
    assert ssm.fwd_workspace_bytes(explicit) == 0
    auto = ssm.make_shape(4, 5120, 64, 64, ssm.SSM_F32)
    assert ssm.fwd_path(auto) == "lookback"
    assert ssm.fwd_path(ssm.make_shape(4, 5120, 64, 64, ssm.SSM_BF16)) == "lookback_ws"
    case = synth.make_case(4, 5120, 64, 64, synth.F32, seed=440)
    ref = oracle.fwd(case)
    y, ls = _run(case, cuda_device)
    assert_close(y, ref["y"], synth.F32, "y")
    assert_close(ls, ref["last_state"], synth.F32, "last_state")


def test_zoh_exact_with_initial_state_and_large_steps(cuda_device):
    # Delta A spans both branches of (e^x - 1) / x (|x| < 1/2 and beyond)
    case = synth.make_case(1, 64, 200, 16, synth.F32, seed=410)
    case["delta_bias"] = np.full(64, 1.5, np.float32)
    h0 = np.random.default_rng(5).standard_normal((1, 64, 16)).astype(np.float32)
    ref = oracle.fwd(case, zoh_exact=True, h0=h0)
    y, ls = _run_zoh(case, cuda_device, h0=h0)
    assert_close(y, ref["y"], synth.F32, "y")
    assert_close(ls, ref["last_state"], synth.F32, "last_state")


def test_zoh_exact_gate_reduction(cuda_device):
    # N = 1, A = -1, B = 1, C = 1, no D, no z: exp(-softplus(s)) = sigmoid(-s), so
    # h_t = (1 - sigmoid(s_t)) h_{t-1} + sigmoid(s_t) u_t exactly (reading guide,
    # the question on Delta and recurrent gating)
    L = 500
    case = synth.make_case(1, 8, L, 1, synth.F32, seed=411, with_z=False, with_D=False)
    case["A"] = -np.ones((8, 1), np.float32)
    case["B"] = np.ones((1, L, 1), np.float32)
    case["C"] = np.ones((1, L, 1), np.float32)
    y, _ = _run_zoh(case, cuda_device)
    s = case["delta"].astype(np.float64) + case["delta_bias"].astype(np.float64)[None, :, None]
    sig = 1.0 / (1.0 + np.exp(-s))
    u = case["u"].astype(np.float64)
    h = np.zeros((1, 8))
    ref = np.zeros_like(u)
    for t in range(L):
        h = (1 - sig[:, :, t]) * h + sig[:, :, t] * u[:, :, t]
        ref[:, :, t] = h
    assert_close(y, ref, synth.F32, "gate recurrence")


def test_zoh_exact_is_not_euler(cuda_device):
    case = synth.make_case(1, 32, 128, 16, synth.F32, seed=412)
    case["delta_bias"] = np.full(32, 0.5, np.float32)
    y_zoh, _ = _run_zoh(case, cuda_device)
    y_eul, _ = _run(case, cuda_device)
    assert np.linalg.norm(y_zoh - y_eul) > 1e-2 * np.linalg.norm(y_eul)


# ---- degenerate sizes ----------------------------------------------------------
def test_zero_length_passes_the_state_through(cuda_device):
    import torch
    import selective_state_space_54_b200 as ssm
    dev = cuda_device
    u = torch.zeros((2, 8, 0), dtype=torch.bfloat16, device=dev)
    Bm = torch.zeros((2, 0, 16), dtype=torch.bfloat16, device=dev)
    A = torch.from_numpy(synth.s4d_real_A(8, 16)).to(dev)
    h0 = torch.randn((2, 8, 16), device=dev)
    y, ls = ssm.scan_fwd(u, u, A, Bm, Bm, initial_state=h0, return_last_state=True)
    y2, ls2 = ssm.scan_fwd(u, u, A, Bm, Bm, return_last_state=True)
    torch.cuda.synchronize()
    assert y.numel() == 0 and torch.equal(ls, h0) and not ls2.any()


def test_single_channel_single_step(cuda_device):
    for dtype in (synth.F32, synth.BF16):
        _check(synth.make_case(1, 1, 1, 16, dtype, seed=77), cuda_device)


# ---- token-major activations (batch, seqlen, dim), as a projection writes them ----
@pytest.mark.parametrize("batch,dim,L", [(2, 64, 256), (1, 40, 333), (3, 8, 17), (2, 1024, 1000)])
def test_token_major_equals_channel_major(cuda_device, batch, dim, L):
    import torch
    import selective_state_space_54_b200 as ssm
    case = synth.make_case(batch, dim, L, 16, synth.BF16, seed=700 + dim)
    g = upload(case, cuda_device)
    y_cm, ls_cm = ssm.scan_fwd(g["u"], g["delta"], g["A"], g["B"], g["C"], g["D"], g["z"],
                               g["delta_bias"], return_last_state=True, path=PATHS["lookback_ws"])
    tm = {k: g[k].transpose(1, 2).contiguous() for k in ("u", "delta", "z")}
    y_tm, ls_tm = ssm.scan_fwd(tm["u"], tm["delta"], g["A"], g["B"], g["C"], g["D"], tm["z"],
                               g["delta_bias"], return_last_state=True, token_major=True)
    torch.cuda.synchronize()
    # the same arithmetic in the same order: only the loads and stores move
    assert torch.equal(y_tm.transpose(1, 2), y_cm)
    assert torch.equal(ls_tm, ls_cm)
    ref = oracle.fwd(case)
    assert_close(to_f64(y_tm.transpose(1, 2)), ref["y"], synth.BF16, "y")
