"""Causal depthwise conv1d (+ SiLU) parity: ssm_causal_conv1d through the C ABI
against the fp64 oracle, on seeded inputs of the Mamba block's shapes."""
import numpy as np
import pytest

import oracle
import synth
from gpu_util import assert_close, to_f64, to_torch

pytestmark = pytest.mark.gpu


def _inputs(batch, dim, L, K, dtype, seed):
    x = synth.normal((batch, dim, L), seed, "u", dtype)
    g = np.random.default_rng(seed)
    w = (g.standard_normal((dim, K)) / np.sqrt(K)).astype(np.float32)
    b = g.standard_normal(dim).astype(np.float32)
    s0 = g.standard_normal((batch, dim, K - 1)).astype(np.float32)
    return x, w, b, s0


def _run(x, w, b, s0, dtype, device, silu=True):
    import torch
    import selective_state_space_54_b200 as ssm
    xt = to_torch(x, dtype, device)
    f = lambda a: None if a is None else torch.from_numpy(a).to(device)
    out, fs = ssm.causal_conv1d(xt, f(w), f(b), initial_state=f(s0), silu=silu,
                                return_final_state=True)
    torch.cuda.synchronize()
    return to_f64(out), to_f64(fs)


def _check(batch, dim, L, K, dtype, seed, device, with_bias=True, with_state=True, silu=True):
    x, w, b, s0 = _inputs(batch, dim, L, K, dtype, seed)
    b = b if with_bias else None
    s0 = s0 if with_state else None
    ref, ref_s = oracle.conv1d(x, w, b, dtype=dtype, initial_state=s0, silu=silu)
    out, fs = _run(x, w, b, s0, dtype, device, silu)
    assert_close(out, ref, dtype, "out")
    if K > 1:
        # the state is a copy of inputs: exact
        assert np.array_equal(fs, ref_s)


@pytest.mark.parametrize("dtype", [synth.F32, synth.BF16])
@pytest.mark.parametrize("K", [1, 2, 3, 4, 5, 8])
def test_conv_widths(cuda_device, dtype, K):
    _check(2, 24, 700, K, dtype, 50 + K, cuda_device)


@pytest.mark.parametrize("L", [1, 2, 3, 7, 8, 9, 255, 256, 257, 1000])
def test_conv_ragged_lengths(cuda_device, L):
    _check(2, 5, L, 4, synth.BF16, L, cuda_device)


@pytest.mark.parametrize("opt", ["no_bias", "no_state", "no_silu"])
def test_conv_optional_terms(cuda_device, opt):
    _check(1, 16, 300, 4, synth.F32, 7, cuda_device, with_bias=opt != "no_bias",
           with_state=opt != "no_state", silu=opt != "no_silu")


def test_conv_streaming_in_pieces(cuda_device):
    # two calls chained through the state equal one call over the whole sequence
    import torch
    import selective_state_space_54_b200 as ssm
    x, w, b, s0 = _inputs(2, 40, 1000, 4, synth.F32, 9)
    dev = cuda_device
    xt = torch.from_numpy(x).to(dev)
    wt, bt, st = (torch.from_numpy(a).to(dev) for a in (w, b, s0))
    full, fs = ssm.causal_conv1d(xt, wt, bt, initial_state=st, return_final_state=True)
    a, sa = ssm.causal_conv1d(xt[:, :, :333].contiguous(), wt, bt, initial_state=st,
                              return_final_state=True)
    c, sc = ssm.causal_conv1d(xt[:, :, 333:].contiguous(), wt, bt, initial_state=sa,
                              return_final_state=True)
    torch.cuda.synchronize()
    assert torch.equal(torch.cat([a, c], dim=-1), full)
    assert torch.equal(sc, fs)


def test_conv_unaligned_rows_take_the_scalar_path(cuda_device):
    # L * 2 bytes not a multiple of 16: no vector access, same results
    _check(3, 7, 77, 4, synth.BF16, 11, cuda_device)


def test_conv_sixteen_byte_aligned_buffers(cuda_device):
    # x 16 bytes into its allocation: rows of 1024 steps take 16-byte accesses instead
    # of 32-byte ones; same results
    import torch
    import selective_state_space_54_b200 as ssm
    x, w, b, s0 = _inputs(2, 8, 1024, 4, synth.BF16, 61)
    ref, ref_s = oracle.conv1d(x, w, b, dtype=synth.BF16, initial_state=s0, silu=True)
    dense = to_torch(x, synth.BF16, cuda_device)
    flat = torch.empty(dense.numel() + 8, dtype=dense.dtype, device=cuda_device)
    xv = flat[8:].view(dense.shape)
    xv.copy_(dense)
    assert xv.data_ptr() % 32 == 16
    f = lambda a: torch.from_numpy(a).to(cuda_device)
    out, fs = ssm.causal_conv1d(xv, f(w), f(b), initial_state=f(s0), silu=True, return_final_state=True)
    torch.cuda.synchronize()
    assert_close(to_f64(out), ref, synth.BF16, "out")
    assert np.array_equal(to_f64(fs), ref_s)


def test_conv_full_mamba_2p8b_layer(cuda_device):
    # the Mamba-2.8B layer's x_proj shape (batch 4, d_inner 5120, L 8192), sampled rows
    import torch
    import selective_state_space_54_b200 as ssm
    w_ = synth.WORKLOADS["mamba-2.8b-layer"]
    x, w, b, _ = _inputs(w_.batch, w_.dim, w_.seqlen, 4, synth.BF16, 21)
    out, fs = _run(x, w, b, None, synth.BF16, cuda_device)
    rows = np.random.default_rng(3).choice(w_.batch * w_.dim, 64, replace=False)
    for r in rows:
        bi, d = divmod(int(r), w_.dim)
        ref, ref_s = oracle.conv1d(x[bi:bi + 1, d:d + 1], w[d:d + 1], b[d:d + 1], dtype=synth.BF16)
        assert_close(out[bi:bi + 1, d:d + 1], ref, synth.BF16, f"row {r}")
        assert np.array_equal(fs[bi:bi + 1, d:d + 1], ref_s)


def test_conv_zero_length_passes_the_state_through(cuda_device):
    import torch
    import selective_state_space_54_b200 as ssm
    dev = cuda_device
    x = torch.zeros((2, 6, 0), dtype=torch.bfloat16, device=dev)
    w = torch.randn((6, 4), device=dev)
    s0 = torch.randn((2, 6, 3), device=dev)
    out, fs = ssm.causal_conv1d(x, w, initial_state=s0, return_final_state=True)
    out2, fs2 = ssm.causal_conv1d(x, w, return_final_state=True)
    torch.cuda.synchronize()
    assert out.numel() == 0 and torch.equal(fs, s0) and not fs2.any()


# ---- backward --------------------------------------------------------------------
def _run_bwd(x, w, b, s0, dout, dtype, device, silu=True):
    import torch
    import selective_state_space_54_b200 as ssm
    f = lambda a: None if a is None else torch.from_numpy(a).to(device)
    g = ssm.causal_conv1d_bwd(to_torch(x, dtype, device), f(w), f(b), to_torch(dout, dtype, device),
                              initial_state=f(s0), silu=silu, want_dinitial_state=True)
    torch.cuda.synchronize()
    return {k: (None if v is None else to_f64(v)) for k, v in g.items()}


def _check_bwd(batch, dim, L, K, dtype, seed, device, with_bias=True, with_state=True, silu=True):
    x, w, b, s0 = _inputs(batch, dim, L, K, dtype, seed)
    dout = synth.normal((batch, dim, L), seed, "dy", dtype)
    b = b if with_bias else None
    s0 = s0 if with_state else None
    ref = oracle.conv1d_bwd(x, w, b, dout, dtype=dtype, initial_state=s0, silu=silu)
    got = _run_bwd(x, w, b, s0, dout, dtype, device, silu)
    assert_close(got["dx"], ref["dx"], dtype, "dx")
    # parameter sums are fp32 sums of bf16-input terms: the bf16 path's tolerance
    assert_close(got["dweight"], ref["dweight"], dtype, "dweight", stored_bf16=False)
    if with_bias:
        assert_close(got["dbias"], ref["dbias"], dtype, "dbias", stored_bf16=False)
    if K > 1:
        assert_close(got["dinitial_state"], ref["dinitial_state"], dtype, "dinitial_state",
                     stored_bf16=False)


@pytest.mark.parametrize("dtype", [synth.F32, synth.BF16])
@pytest.mark.parametrize("K", [1, 2, 4, 8])
def test_conv_bwd_widths(cuda_device, dtype, K):
    _check_bwd(2, 24, 1500, K, dtype, 80 + K, cuda_device)


@pytest.mark.parametrize("L", [1, 2, 3, 7, 8, 9, 255, 256, 257, 1023, 1024, 1025, 3000])
def test_conv_bwd_ragged_lengths(cuda_device, L):
    _check_bwd(2, 5, L, 4, synth.F32, 90 + L, cuda_device)


@pytest.mark.parametrize("opt", ["no_bias", "no_state", "no_silu"])
def test_conv_bwd_optional_terms(cuda_device, opt):
    _check_bwd(1, 16, 700, 4, synth.F32, 13, cuda_device, with_bias=opt != "no_bias",
               with_state=opt != "no_state", silu=opt != "no_silu")


@pytest.mark.parametrize("L", [1, 9, 511, 512, 513, 1537, 4096])
def test_conv_bwd_ragged_lengths_bf16(cuda_device, L):
    # rows of L * 2 bytes a multiple of 16 (512, 4096) reach shared memory by cp.async,
    # the others by element loads; 512-step segments, the last one ragged
    _check_bwd(2, 5, L, 4, synth.BF16, 190 + L, cuda_device)


def test_conv_bwd_unaligned_rows_take_the_element_path(cuda_device):
    _check_bwd(3, 7, 1077, 4, synth.BF16, 12, cuda_device)


@pytest.mark.parametrize("dtype,K", [(synth.BF16, 4), (synth.BF16, 7), (synth.F32, 8)])
def test_conv_bwd_rows_across_warp_ranges(cuda_device, dtype, K):
    # the backward's warps walk contiguous ranges of 512-step segments: over 16 rows of
    # 640,024 steps the ranges start and end inside rows (the first inputs before a range
    # and the da after it come from memory) and hold several segments of one row (lane
    # 31's second dx half waits for the next segment's first da values)
    _check_bwd(2, 8, 512 * 1250 + 24, K, dtype, 31 + K, cuda_device)


def test_conv_bwd_dx_is_bitwise_repeatable(cuda_device):
    # dx and the initial state's gradient take no atomics: equal bits on every call
    # (dweight and dbias are summed with atomics, equal only to rounding)
    x, w, b, s0 = _inputs(2, 24, 5000, 4, synth.BF16, 44)
    dout = synth.normal((2, 24, 5000), 44, "dy", synth.BF16)
    g1 = _run_bwd(x, w, b, s0, dout, synth.BF16, cuda_device)
    g2 = _run_bwd(x, w, b, s0, dout, synth.BF16, cuda_device)
    assert np.array_equal(g1["dx"], g2["dx"])
    assert np.array_equal(g1["dinitial_state"], g2["dinitial_state"])
    np.testing.assert_allclose(g1["dweight"], g2["dweight"], rtol=1e-5, atol=1e-6)


@pytest.mark.parametrize("dtype", [synth.F32, synth.BF16])
def test_conv_saturated_silu(cuda_device, dtype):
    # pre-activations in the hundreds: e^-a overflows to infinity on the negative side,
    # where SiLU and its derivative must come out as (signed) zeros, not NaN
    x, w, b, s0 = _inputs(2, 16, 3000, 4, dtype, 55)
    xs = (synth.bf16_bits_to_f32(x) * 100.0).astype(np.float32) if dtype == synth.BF16 else x * 100.0
    if dtype == synth.BF16:
        xs = synth.f32_to_bf16_bits(xs)
    dout = synth.normal((2, 16, 3000), 55, "dy", dtype)
    with np.errstate(over="ignore"):
        ref, ref_s = oracle.conv1d(xs, w, b, dtype=dtype, initial_state=s0, silu=True)
        refb = oracle.conv1d_bwd(xs, w, b, dout, dtype=dtype, initial_state=s0, silu=True)
    out, fs = _run(xs, w, b, s0, dtype, cuda_device)
    got = _run_bwd(xs, w, b, s0, dout, dtype, cuda_device)
    assert np.all(np.isfinite(out)) and np.all(np.isfinite(got["dx"]))
    assert_close(out, ref, dtype, "out")
    assert_close(got["dx"], refb["dx"], dtype, "dx")
    assert_close(got["dweight"], refb["dweight"], dtype, "dweight", stored_bf16=False)
    assert_close(got["dbias"], refb["dbias"], dtype, "dbias", stored_bf16=False)


def test_conv_bwd_full_mamba_2p8b_layer(cuda_device):
    # the x_proj shape at full size; dx on sampled rows, parameter sums in full
    w_ = synth.WORKLOADS["mamba-2.8b-layer"]
    x, w, b, _ = _inputs(w_.batch, w_.dim, w_.seqlen, 4, synth.BF16, 22)
    dout = synth.normal((w_.batch, w_.dim, w_.seqlen), 22, "dy", synth.BF16)
    got = _run_bwd(x, w, b, None, dout, synth.BF16, cuda_device)
    ref = oracle.conv1d_bwd(x, w, b, dout, dtype=synth.BF16)
    assert_close(got["dx"], ref["dx"], synth.BF16, "dx")
    assert_close(got["dweight"], ref["dweight"], synth.BF16, "dweight", stored_bf16=False)
    assert_close(got["dbias"], ref["dbias"], synth.BF16, "dbias", stored_bf16=False)

