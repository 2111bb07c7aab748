"""Pins of the fp64 oracle to facts that do not come from the oracle itself.

Each test checks the oracle against something the Mamba pages or plain
mathematics fix independently of its code: the time-invariant limit (a
convolution), a brute-force unrolled sum, the reset/preserve behaviour of
Delta, the gating identity for N=1, linearity, special values of the gate and
of softplus, and finite differences for the backward.  A dropped term, a wrong
sign, a shifted time index or a transposed operand in the oracle fails at
least one of them.
"""
import math

import numpy as np
import pytest

import oracle
import synth


def _case(batch, dim, L, N, seed, *, softplus=True, z=True, D=True, bias=True):
    rng = np.random.default_rng(seed)
    c = {
        "batch": batch, "dim": dim, "seqlen": L, "dstate": N, "dtype": synth.F32,
        "u": rng.standard_normal((batch, dim, L)),
        "delta": rng.standard_normal((batch, dim, L)) * 0.5,
        # A varies over both d and n (d != n shapes catch a transposed A)
        "A": -np.exp(rng.uniform(-1.0, 1.5, size=(dim, N))),
        "B": rng.standard_normal((batch, L, N)),
        "C": rng.standard_normal((batch, L, N)),
        "D": rng.standard_normal(dim) if D else None,
        "z": rng.standard_normal((batch, dim, L)) if z else None,
        "delta_bias": rng.uniform(-3, 0, size=dim) if bias else None,
    }
    if not softplus:
        # without softplus keep Delta = raw + bias > 0, so that |Abar| <= 1
        c["delta"] = np.abs(c["delta"]) + 0.05
        if bias:
            c["delta_bias"] = rng.uniform(0.0, 0.3, size=dim)
    return c


def _rel(a, b):
    return np.linalg.norm((a - b).ravel()) / max(np.linalg.norm(b.ravel()), 1e-300)


# -- P1: time-invariant limit == explicit convolution ------------------------
# "Mamba: Linear-Time Sequence Modeling..." reading guide, "Perguntas" (LTI
# systems admit a global convolution); "O que e um modelo Mamba?" (the S4
# convolution kernel).  With Delta, B, C constant in t the recurrence is the
# causal convolution y_t = sum_k K_k u_{t-k} + D u_t, K_k = sum_n C_n Abar_n^k Bbar_n.
@pytest.mark.parametrize("zoh", [False, True])
def test_lti_limit_is_convolution(zoh):
    rng = np.random.default_rng(11)
    batch, dim, L, N = 2, 3, 40, 5
    c = _case(batch, dim, L, N, 1, softplus=False, z=False, bias=False)
    dl = rng.uniform(0.05, 0.6, size=dim)
    c["delta"] = np.broadcast_to(dl[None, :, None], (batch, dim, L)).copy()
    Bn = rng.standard_normal((batch, N))
    Cn = rng.standard_normal((batch, N))
    c["B"] = np.broadcast_to(Bn[:, None, :], (batch, L, N)).copy()
    c["C"] = np.broadcast_to(Cn[:, None, :], (batch, L, N)).copy()
    y = oracle.fwd(c, delta_softplus=False, zoh_exact=zoh)["y"]
    ref = np.zeros_like(y)
    for b in range(batch):
        for d in range(dim):
            A = c["A"][d]
            bbar = (np.expm1(dl[d] * A) / A if zoh else dl[d]) * Bn[b]
            K = np.array([np.sum(Cn[b] * np.exp(k * dl[d] * A) * bbar) for k in range(L)])
            u = c["u"][b, d]
            ref[b, d] = np.convolve(u, K)[:L] + c["D"][d] * u
    assert _rel(y, ref) < 1e-12


# -- P2: brute-force unrolled sum on tiny inputs -----------------------------
# Associativity of the linear recurrence (reading guide "Termos-chave",
# Parallel Associative Scan): h_t = sum_{s<=t} (prod_{r=s+1..t} Abar_r) Bbar_s u_s.
def test_bruteforce_unrolled_sum():
    batch, dim, L, N = 2, 3, 13, 4
    c = _case(batch, dim, L, N, 2)
    y = oracle.fwd(c)["y"]
    ref = np.zeros_like(y)
    for b in range(batch):
        for d in range(dim):
            s = c["delta"][b, d] + c["delta_bias"][d]
            dl = np.logaddexp(0.0, s)          # softplus, an independent routine
            cum = np.concatenate([[0.0], np.cumsum(dl)])
            for t in range(L):
                h = np.zeros(N)
                for s_ in range(t + 1):
                    decay = np.exp(c["A"][d] * (cum[t + 1] - cum[s_ + 1]))
                    h += decay * dl[s_] * c["B"][b, s_] * c["u"][b, d, s_]
                yss = np.dot(c["C"][b, t], h) + c["D"][d] * c["u"][b, d, t]
                zt = c["z"][b, d, t]
                ref[b, d, t] = yss * zt / (1.0 + math.exp(-zt))
    assert _rel(y, ref) < 1e-12


# -- P3: a large Delta resets the state (A < 0) ------------------------------
# Reading guide "Perguntas": a large Delta makes the model focus on the current
# input and reset the state.  exp(1e4 * A) underflows to exactly 0 in fp64.
def test_large_delta_resets_state_bitwise():
    batch, dim, L, N, t0 = 1, 4, 30, 6, 17
    c = _case(batch, dim, L, N, 3, softplus=False, bias=False)
    c["delta"][:, :, t0] = 1e4
    y0 = oracle.fwd(c, delta_softplus=False)
    rng = np.random.default_rng(5)
    c2 = {k: (v.copy() if isinstance(v, np.ndarray) else v) for k, v in c.items()}
    c2["u"][:, :, :t0] += rng.standard_normal((batch, dim, t0))
    c2["B"][:, :t0] += rng.standard_normal((batch, t0, N))
    c2["delta"][:, :, :t0] *= rng.uniform(0.5, 2.0, size=(batch, dim, t0))
    y1 = oracle.fwd(c2, delta_softplus=False)
    assert np.array_equal(y0["y"][..., t0:], y1["y"][..., t0:])
    assert np.array_equal(y0["last_state"], y1["last_state"])
    assert not np.array_equal(y0["y"][..., :t0], y1["y"][..., :t0])


# -- P3': a zero Delta preserves the state and ignores the input ------------
# Reading guide "Perguntas": a small Delta keeps the state and ignores the input.
def test_zero_delta_preserves_state_bitwise():
    batch, dim, L, N, t1 = 2, 3, 20, 4, 9
    c = _case(batch, dim, L, N, 4, softplus=False, bias=False, z=False, D=False)
    c["delta"][:, :, t1] = 0.0
    y0 = oracle.fwd(c, delta_softplus=False)
    c2 = {k: (v.copy() if isinstance(v, np.ndarray) else v) for k, v in c.items()}
    c2["u"][:, :, t1] += 3.0
    c2["B"][:, t1] += 2.0
    y1 = oracle.fwd(c2, delta_softplus=False)
    assert np.array_equal(y0["y"], y1["y"])
    assert np.array_equal(y0["last_state"], y1["last_state"])
    # with C_{t1} = C_{t1-1} the output repeats: h_{t1} == h_{t1-1} exactly
    c3 = {k: (v.copy() if isinstance(v, np.ndarray) else v) for k, v in c.items()}
    c3["C"][:, t1] = c3["C"][:, t1 - 1]
    y3 = oracle.fwd(c3, delta_softplus=False)["y"]
    assert np.array_equal(y3[..., t1], y3[..., t1 - 1])


# -- P4: the N=1, A=-1, B=1 gating reduction ---------------------------------
# Reading guide, "O Mecanismo de Selecao (S6)": with N=1, A=-1, B=1 the
# recurrence is the gated update h_t = (1 - g_t) h_{t-1} + g_t x_t with
# g_t = sigmoid(.), exactly for the ZOH input term because exp(-softplus(s)) = sigmoid(-s).
def _gate_case(L, seed):
    rng = np.random.default_rng(seed)
    c = {
        "batch": 1, "dim": 1, "seqlen": L, "dstate": 1, "dtype": synth.F32,
        "u": rng.standard_normal((1, 1, L)), "delta": rng.standard_normal((1, 1, L)) * 2,
        "A": np.array([[-1.0]]), "B": np.ones((1, L, 1)), "C": np.ones((1, L, 1)),
        "D": None, "z": None, "delta_bias": None,
    }
    return c


def _sig(x):
    return 0.5 * (1.0 + np.tanh(0.5 * x))


def test_gate_reduction_zoh_exact():
    L = 50
    c = _gate_case(L, 7)
    y = oracle.fwd(c, zoh_exact=True)["y"][0, 0]
    s, u = c["delta"][0, 0], c["u"][0, 0]
    h, ref = 0.0, np.zeros(L)
    for t in range(L):
        g = _sig(s[t])
        h = (1.0 - g) * h + g * u[t]
        ref[t] = h
    assert _rel(y, ref) < 1e-13


def test_gate_reduction_euler():
    # the Euler input term of the contract gives h_t = sigmoid(-s) h + softplus(s) u
    L = 50
    c = _gate_case(L, 8)
    y = oracle.fwd(c, zoh_exact=False)["y"][0, 0]
    s, u = c["delta"][0, 0], c["u"][0, 0]
    h, ref = 0.0, np.zeros(L)
    for t in range(L):
        h = _sig(-s[t]) * h + np.logaddexp(0.0, s[t]) * u[t]
        ref[t] = h
    assert _rel(y, ref) < 1e-13


# -- special values: softplus(0) = ln 2, bias placement, SiLU(ln 3) = 0.75 ln 3
def test_special_values_softplus_bias_and_gate():
    base = {
        "batch": 1, "dim": 1, "seqlen": 1, "dstate": 1, "dtype": synth.F32,
        "u": np.ones((1, 1, 1)), "delta": np.zeros((1, 1, 1)), "A": np.zeros((1, 1)),
        "B": np.ones((1, 1, 1)), "C": np.ones((1, 1, 1)), "D": None, "z": None,
        "delta_bias": None,
    }
    assert oracle.fwd(base)["y"][0, 0, 0] == pytest.approx(math.log(2.0), rel=1e-15)
    # Parameter + s_Delta(x): the bias is added before softplus
    c = dict(base, delta=np.full((1, 1, 1), 0.3),
             delta_bias=np.array([math.log(math.expm1(1.0)) - 0.3]))
    assert oracle.fwd(c)["y"][0, 0, 0] == pytest.approx(1.0, rel=1e-14)
    # without softplus the bias is still added
    assert oracle.fwd(c, delta_softplus=False)["y"][0, 0, 0] == pytest.approx(
        math.log(math.expm1(1.0)), rel=1e-14)
    # gate: y = yss * SiLU(z); C = 0, D = 1, u = 1 gives y = SiLU(z)
    g = dict(base, C=np.zeros((1, 1, 1)), D=np.ones(1))
    for zv, want in [(math.log(3.0), 0.75 * math.log(3.0)), (0.0, 0.0),
                     (-math.log(3.0), -0.25 * math.log(3.0))]:
        out = oracle.fwd(dict(g, z=np.full((1, 1, 1), zv)))["y"][0, 0, 0]
        assert out == pytest.approx(want, rel=1e-15, abs=1e-300)


# -- P5: linearity in u with the gate off ------------------------------------
def test_linearity_in_u():
    c = _case(2, 3, 25, 4, 9, z=False)
    rng = np.random.default_rng(10)
    u1, u2 = rng.standard_normal(c["u"].shape), rng.standard_normal(c["u"].shape)
    y1 = oracle.fwd(dict(c, u=u1))["y"]
    y2 = oracle.fwd(dict(c, u=u2))["y"]
    y12 = oracle.fwd(dict(c, u=2.5 * u1 - 0.75 * u2))["y"]
    assert _rel(y12, 2.5 * y1 - 0.75 * y2) < 1e-12


def test_initial_state_continuation():
    # scan(L1) -> last_state -> scan(L2 from it) == scan(L1 + L2)
    c = _case(2, 3, 30, 4, 12)
    full = oracle.fwd(c)
    cut = 13
    head = {k: (v[..., :cut] if k in ("u", "delta", "z") else v) for k, v in c.items()}
    head = dict(head, B=c["B"][:, :cut], C=c["C"][:, :cut], seqlen=cut)
    tail = {k: (v[..., cut:] if k in ("u", "delta", "z") else v) for k, v in c.items()}
    tail = dict(tail, B=c["B"][:, cut:], C=c["C"][:, cut:], seqlen=30 - cut)
    h = oracle.fwd(head)
    t = oracle.fwd(tail, h0=h["last_state"])
    assert np.array_equal(np.concatenate([h["y"], t["y"]], axis=-1), full["y"])
    assert np.array_equal(t["last_state"], full["last_state"])


def test_thread_count_does_not_change_forward():
    c = _case(3, 5, 17, 3, 13)
    a = oracle.fwd(c, nthreads=1)
    b = oracle.fwd(c, nthreads=4)
    assert np.array_equal(a["y"], b["y"]) and np.array_equal(a["last_state"], b["last_state"])


# -- P6: backward against central finite differences -------------------------
_GRAD_OF = {"u": "du", "delta": "ddelta", "A": "dA", "B": "dB", "C": "dC",
            "D": "dD", "z": "dz", "delta_bias": "ddelta_bias"}


def _objective(c, dout, softplus, h0=None, zoh=False):
    return float(np.sum(dout * oracle.fwd(c, delta_softplus=softplus, h0=h0, zoh_exact=zoh)["y"]))


@pytest.mark.parametrize("zoh", [False, True])
@pytest.mark.parametrize("softplus", [True, False])
def test_backward_matches_finite_differences(softplus, zoh):
    # zoh: the exact zero-order-hold input term of the reading guide's "Metodo"
    # (Bbar = (Delta A)^-1 (exp(Delta A) - I) Delta B); one A entry per channel
    # is 0 there, so the A -> 0 limit of its derivative is checked too, and
    # Delta A spans both sides of the oracle's series/closed-form switch
    c = _case(2, 3, 11, 3, 21, softplus=softplus)
    if zoh:
        c["A"] = c["A"].copy()
        c["A"][:, 1] = 0.0
    rng = np.random.default_rng(22)
    dout = rng.standard_normal(c["u"].shape)
    h0 = rng.standard_normal((2, 3, 3)) * 0.5
    g = oracle.bwd(c, dout, delta_softplus=softplus, zoh_exact=zoh, h0=h0, want_dh0=True)
    for name, gname in _GRAD_OF.items():
        x = c[name]
        flat_idx = rng.choice(x.size, size=min(6, x.size), replace=False)
        for fi in flat_idx:
            idx = np.unravel_index(fi, x.shape)
            eps = 1e-6 * max(1.0, abs(x[idx]))
            xp, xm = x.copy(), x.copy()
            xp[idx] += eps
            xm[idx] -= eps
            fd = (_objective(dict(c, **{name: xp}), dout, softplus, h0, zoh)
                  - _objective(dict(c, **{name: xm}), dout, softplus, h0, zoh)) / (2 * eps)
            an = g[gname][idx]
            assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), (name, idx, fd, an)
    # gradient with respect to the initial state
    for fi in rng.choice(h0.size, size=4, replace=False):
        idx = np.unravel_index(fi, h0.shape)
        hp, hm = h0.copy(), h0.copy()
        hp[idx] += 1e-6
        hm[idx] -= 1e-6
        fd = (_objective(c, dout, softplus, hp, zoh) - _objective(c, dout, softplus, hm, zoh)) / 2e-6
        assert abs(fd - g["dh0"][idx]) <= 1e-6 * max(1.0, abs(fd))
    if zoh:  # every dA entry, the A = 0 column included
        for idx in np.ndindex(*c["A"].shape):
            eps = 1e-6
            xp, xm = c["A"].copy(), c["A"].copy()
            xp[idx] += eps
            xm[idx] -= eps
            fd = (_objective(dict(c, A=xp), dout, softplus, h0, True)
                  - _objective(dict(c, A=xm), dout, softplus, h0, True)) / (2 * eps)
            assert abs(fd - g["dA"][idx]) <= 1e-6 * max(1.0, abs(fd)), (idx, fd, g["dA"][idx])


@pytest.mark.parametrize("zoh", [False, True])
def test_backward_adjoint_dot_product(zoh):
    # <J^T dout, v> == d/de f(x + e v) for a random direction over all inputs
    c = _case(2, 4, 9, 3, 31)
    rng = np.random.default_rng(32)
    dout = rng.standard_normal(c["u"].shape)
    g = oracle.bwd(c, dout, zoh_exact=zoh)
    v = {k: rng.standard_normal(c[k].shape) for k in _GRAD_OF}
    eps = 1e-6
    cp = dict(c, **{k: c[k] + eps * v[k] for k in v})
    cm = dict(c, **{k: c[k] - eps * v[k] for k in v})
    fd = (_objective(cp, dout, True, zoh=zoh) - _objective(cm, dout, True, zoh=zoh)) / (2 * eps)
    an = sum(float(np.sum(g[_GRAD_OF[k]] * v[k])) for k in v)
    assert abs(fd - an) <= 1e-6 * max(1.0, abs(an))


def test_backward_thread_count_invariance():
    c = _case(2, 6, 15, 4, 41)
    dout = np.random.default_rng(42).standard_normal(c["u"].shape)
    a = oracle.bwd(c, dout, nthreads=1)
    b = oracle.bwd(c, dout, nthreads=3)
    for k in ("du", "ddelta", "dz"):
        assert np.array_equal(a[k], b[k])
    for k in ("dA", "dB", "dC", "dD", "ddelta_bias"):
        assert np.allclose(a[k], b[k], rtol=1e-13, atol=1e-13)


# -- the input generator: the stored recipe, not the method -----------------
def test_synth_recipe():
    w = synth.WORKLOADS["tiny-fp32"]
    c = synth.make_workload(w)
    assert c["u"].dtype == np.float32 and c["u"].shape == (1, 16, 64)
    assert c["B"].shape == (1, 64, 4)
    assert np.array_equal(c["A"][3], -np.arange(1, 5, dtype=np.float32))
    dt = np.log1p(np.exp(c["delta_bias"].astype(np.float64)))
    assert np.all(dt > 0.999e-3) and np.all(dt < 1.001e-1)
    c1 = synth.make_case(2, 3, 100, 4, synth.BF16, seed=5, threads=1)
    c2 = synth.make_case(2, 3, 100, 4, synth.BF16, seed=5, threads=4)
    assert np.array_equal(c1["u"], c2["u"]) and c1["u"].dtype == np.uint16
    x = np.array([1.0, 1.00390625, 1.005859375, -2.5, 3.0e-3], np.float32)
    back = synth.bf16_bits_to_f32(synth.f32_to_bf16_bits(x))
    # RNE: 1+2^-8 is a tie between 1 and 1+2^-7 -> even (1.0)
    assert back[0] == 1.0 and back[1] == 1.0 and back[2] == np.float32(1.0078125)
    assert back[3] == -2.5


# -- the causal convolution of the Mamba block (ibm.com walk-through) --------
def _conv_inputs(seed, bt=2, dm=3, L=40, K=4):
    g = np.random.default_rng(seed)
    return (g.standard_normal((bt, dm, L)), g.standard_normal((dm, K)), g.standard_normal(dm),
            g.standard_normal((bt, dm, K - 1)))


def test_conv_matches_numpy_convolve():
    # a library routine: np.convolve(x, w reversed)[:L] is the causal filter
    x, w, b, _ = _conv_inputs(1)
    out, _ = oracle.conv1d(x, w, b, silu=False)
    for i in range(x.shape[0]):
        for d in range(x.shape[1]):
            ref = np.convolve(x[i, d], w[d][::-1])[:x.shape[2]] + b[d]
            np.testing.assert_allclose(out[i, d], ref, rtol=1e-13, atol=1e-13)


def test_conv_identity_and_shift_kernels():
    x, _, _, _ = _conv_inputs(2)
    ident = np.zeros((3, 4)); ident[:, 3] = 1.0   # weight on the current token
    out, st = oracle.conv1d(x, ident, silu=False)
    assert np.array_equal(out, x)
    assert np.array_equal(st, x[:, :, -3:])
    shift = np.zeros((3, 4)); shift[:, 0] = 1.0   # weight on the token 3 steps back
    out, _ = oracle.conv1d(x, shift, silu=False)
    assert np.array_equal(out[:, :, 3:], x[:, :, :-3]) and not out[:, :, :3].any()


def test_conv_silu_closed_form():
    x, w, b, _ = _conv_inputs(3)
    lin, _ = oracle.conv1d(x, w, b, silu=False)
    act, _ = oracle.conv1d(x, w, b, silu=True)
    np.testing.assert_allclose(act, lin * (1.0 / (1.0 + np.exp(-lin))), rtol=1e-15)


def test_conv_streaming_in_pieces():
    # convolving [x1 | x2] equals convolving x1, then x2 from x1's final state
    x, w, b, s0 = _conv_inputs(4, L=50)
    full, fs = oracle.conv1d(x, w, b, initial_state=s0)
    a, sa = oracle.conv1d(x[:, :, :17], w, b, initial_state=s0)
    c, sc = oracle.conv1d(x[:, :, 17:], w, b, initial_state=sa)
    np.testing.assert_allclose(np.concatenate([a, c], axis=-1), full, rtol=1e-14, atol=1e-14)
    assert np.array_equal(sc, fs)
    # shorter than the window: the state shifts through
    e, se = oracle.conv1d(x[:, :, :2], w, b, initial_state=s0)
    assert np.array_equal(se, np.concatenate([s0[:, :, 2:], x[:, :, :2]], axis=-1))


def test_conv_backward_matches_finite_differences():
    # central differences of L = sum(dout * conv1d(...)) in fp64, every input
    x, w, b, s0 = _conv_inputs(5, bt=1, dm=2, L=12, K=4)
    dout = np.random.default_rng(6).standard_normal(x.shape)
    g = oracle.conv1d_bwd(x, w, b, dout, initial_state=s0)
    loss = lambda xx, ww, bb, ss: float((dout * oracle.conv1d(xx, ww, bb, initial_state=ss)[0]).sum())
    eps = 1e-6
    for name, arr, key in (("x", x, "dx"), ("w", w, "dweight"), ("b", b, "dbias"),
                           ("s0", s0, "dinitial_state")):
        num = np.zeros_like(arr)
        it = np.nditer(arr, flags=["multi_index"])
        for _ in it:
            i = it.multi_index
            args = {"x": x.copy(), "w": w.copy(), "b": b.copy(), "s0": s0.copy()}
            args[name][i] += eps
            hi = loss(args["x"], args["w"], args["b"], args["s0"])
            args[name][i] -= 2 * eps
            lo = loss(args["x"], args["w"], args["b"], args["s0"])
            num[i] = (hi - lo) / (2 * eps)
        np.testing.assert_allclose(g[key], num, rtol=1e-6, atol=1e-7, err_msg=name)


def test_conv_backward_without_activation_is_the_adjoint():
    # linear case: <dout, conv(x)> = <conv^T(dout), x> for the x part (bias and state zero)
    x, w, _, _ = _conv_inputs(7, bt=2, dm=3, L=30, K=3)
    dout = np.random.default_rng(8).standard_normal(x.shape)
    out, _ = oracle.conv1d(x, w, silu=False)
    g = oracle.conv1d_bwd(x, w, None, dout, silu=False)
    np.testing.assert_allclose((dout * out).sum(), (g["dx"] * x).sum(), rtol=1e-12)
    np.testing.assert_allclose(g["dbias"], dout.sum(axis=(0, 2)), rtol=1e-12)
