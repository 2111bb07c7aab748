"""Seeded random small problems through every schedule against the fp64 oracle.

Each case draws batch, d_inner, L, d_state, io dtype, schedule, lanes per
channel, the exact-ZOH flag and an initial state from a fixed seed; shapes the
library refuses for that schedule must be refused by the workspace query,
every other one must match the oracle (forward always, backward on a subset).
"""
import numpy as np
import pytest

import oracle
import synth
from gpu_util import assert_close, to_f64, to_torch, upload

pytestmark = pytest.mark.gpu

PATHS = {"auto": 0, "lookback": 1, "split_l": 2, "per_group": 3, "lookback_ws": 4}
GRADS = ("du", "ddelta", "dA", "dB", "dC", "dD", "dz", "ddelta_bias")


def _supported(path, lanes, N, dtype, zoh):
    """The library's documented rules (include/ssm_scan.h)."""
    if zoh and path in ("split_l", "per_group"):
        return False
    if path == "lookback_ws":
        if lanes == 4 and not (5 <= N <= 16):
            return False
        if dtype == synth.F32 and N > 32:
            return False  # the warp-specialised kernel's shared memory does not fit
    return True


@pytest.mark.parametrize("i", range(120))
def test_random_case_against_the_oracle(cuda_device, i):
    import torch
    import selective_state_space_54_b200 as ssm
    rng = np.random.default_rng(9000 + i)
    batch = int(rng.integers(1, 4))
    dim = int(rng.choice([1, 7, 16, 33, 64, 100, 200]))
    L = int(rng.choice([1, 5, 16, 31, 64, 129, 300, 777]))
    N = int(rng.choice([1, 3, 4, 5, 8, 12, 16, 20, 32, 64]))
    dtype = synth.BF16 if rng.random() < 0.6 else synth.F32
    path = str(rng.choice(list(PATHS)))
    lanes = 0 if path == "auto" else int(rng.choice([2, 4]))
    zoh = bool(rng.random() < 0.3)
    with_h0 = bool(rng.random() < 0.5)
    case = synth.make_case(batch, dim, L, N, dtype, seed=9100 + i, with_dy=True)
    h0 = rng.standard_normal((batch, dim, N)).astype(np.float32) if with_h0 else None
    flags = ssm.SSM_FLAG_ZOH_EXACT if zoh else 0
    shape = ssm.make_shape(batch, dim, L, N, ssm.SSM_BF16 if dtype == synth.BF16 else ssm.SSM_F32,
                           PATHS[path], lanes, flags)
    need = ssm.fwd_workspace_bytes(shape)
    if not _supported(path, lanes, N, dtype, zoh):
        assert need == 0, (path, lanes, N, dtype, zoh)
        return
    assert need > 0, (path, lanes, N, dtype, zoh)
    g = upload(case, cuda_device)
    h0_t = None if h0 is None else torch.from_numpy(h0).to(cuda_device)
    ws = torch.empty(need, dtype=torch.uint8, device=cuda_device)
    args = (g["u"], g["delta"], g["A"], g["B"], g["C"], g["D"], g["z"], g["delta_bias"])
    y, ls = ssm.scan_fwd(*args, initial_state=h0_t, return_last_state=True, path=PATHS[path],
                         lanes=lanes, zoh_exact=zoh, workspace=ws)
    ssm.check(ws)
    ref = oracle.fwd(case, h0=h0, zoh_exact=zoh)
    what = f"case {i}: {batch}x{dim}x{L} N={N} {dtype} {path}/{lanes} zoh={zoh} h0={with_h0}"
    assert_close(to_f64(y), ref["y"], dtype, "y " + what)
    assert_close(to_f64(ls), ref["last_state"], dtype, "last_state " + what, stored_bf16=False)
    if i % 3 == 0:  # the backward on a third of the cases
        got = ssm.scan_bwd(*args, g["dy"], initial_state=h0_t, want_dinitial_state=with_h0,
                           zoh_exact=zoh)
        refb = oracle.bwd(case, case["dy"], h0=h0, want_dh0=with_h0, zoh_exact=zoh)
        for k in GRADS:
            assert_close(to_f64(got[k]), refb[k], dtype, f"{k} {what}",
                         stored_bf16=k in ("du", "ddelta", "dB", "dC", "dz"))
        if with_h0:
            assert_close(to_f64(got["dinitial_state"]), refb["dh0"], dtype, "dh0 " + what,
                         stored_bf16=False)


@pytest.mark.parametrize("i", range(60))
def test_random_conv1d_case_against_the_oracle(cuda_device, i):
    # causal conv1d + SiLU forward and backward: random widths, lengths around the
    # backward's 512-step segments and the forward's 2048-step warps, row counts that
    # make the backward's warp ranges start and end inside rows or hold several
    # segments of one, dtypes, and every optional term
    import torch
    import selective_state_space_54_b200 as ssm
    rng = np.random.default_rng(7000 + i)
    batch = int(rng.integers(1, 4))
    dim = int(rng.choice([1, 3, 16, 40, 129]))
    L = int(rng.choice([1, 2, 7, 8, 100, 511, 512, 513, 1024, 1500, 2049, 5000, 20000]))
    K = int(rng.integers(1, 9))
    dtype = synth.BF16 if rng.random() < 0.6 else synth.F32
    silu = bool(rng.random() < 0.8)
    with_bias = bool(rng.random() < 0.7)
    with_state = bool(rng.random() < 0.6)
    x = synth.normal((batch, dim, L), 7100 + i, "u", dtype)
    dout = synth.normal((batch, dim, L), 7100 + i, "dy", dtype)
    w = (rng.standard_normal((dim, K)) / np.sqrt(K)).astype(np.float32)
    b = rng.standard_normal(dim).astype(np.float32) if with_bias else None
    s0 = rng.standard_normal((batch, dim, K - 1)).astype(np.float32) if with_state else None

    ref, ref_s = oracle.conv1d(x, w, b, dtype=dtype, initial_state=s0, silu=silu)
    refb = oracle.conv1d_bwd(x, w, b, dout, dtype=dtype, initial_state=s0, silu=silu)
    f = lambda a: None if a is None else torch.from_numpy(a).to(cuda_device)
    xt, gt = to_torch(x, dtype, cuda_device), to_torch(dout, dtype, cuda_device)
    out, fs = ssm.causal_conv1d(xt, f(w), f(b), initial_state=f(s0), silu=silu,
                                return_final_state=True)
    grads = ssm.causal_conv1d_bwd(xt, f(w), f(b), gt, initial_state=f(s0), silu=silu,
                                  want_dinitial_state=True)
    torch.cuda.synchronize()
    tag = f"case {i}: batch {batch} dim {dim} L {L} K {K} {dtype} silu {silu}"
    assert_close(to_f64(out), ref, dtype, f"{tag} out")
    if K > 1:
        assert np.array_equal(to_f64(fs), ref_s), tag
    assert_close(to_f64(grads["dx"]), refb["dx"], dtype, f"{tag} dx")
    assert_close(to_f64(grads["dweight"]), refb["dweight"], dtype, f"{tag} dweight", stored_bf16=False)
    if with_bias:
        assert_close(to_f64(grads["dbias"]), refb["dbias"], dtype, f"{tag} dbias", stored_bf16=False)
    if K > 1:
        assert_close(to_f64(grads["dinitial_state"]), refb["dinitial_state"], dtype,
                     f"{tag} dinitial_state", stored_bf16=False)
