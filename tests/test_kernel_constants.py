"""CPU pins of the constants the kernels carry.

The forward's softplus evaluates log1p(x) for x = exp(-|s|) in (0, 1] as
x * p(x), with p the degree-8 polynomial that interpolates log1p(x)/x at the
9 Chebyshev nodes of [0, 1].  This test re-derives p by that method (numpy
polynomial interpolation at the nodes), checks that every coefficient in the
source is the fp32 rounding of the derived one, and that the fp32 Horner
evaluation stays within the stated 2.3e-7 relative error of log1p on (0, 1].
"""
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "selective_state_space_54_b200", "csrc")
FLOAT = r"(-?\d\.\d+e[-+]\d+)f"


def _chebyshev_interpolant():
    k = np.arange(9)
    x = 0.5 + 0.5 * np.cos((2 * k + 1) * np.pi / 18)  # Chebyshev nodes of [0, 1]
    return np.polyfit(x, np.log1p(x) / x, 8)          # highest degree first


def _source_coefficients(path, func):
    src = open(path).read()
    body = src[src.index(func):]
    body = body[:body.index("\n}\n")]
    return [float(v) for v in re.findall(FLOAT, body)]


def test_softplus_polynomial_is_the_chebyshev_interpolant():
    ref = _chebyshev_interpolant()
    ref32 = ref.astype(np.float32)
    for path, func in ((os.path.join(CSRC, "ssm_common.cuh"), "float softplus_fast("),
                       (os.path.join(CSRC, "ssm_fwd.cu"), "f2 softplus2(")):
        got = _source_coefficients(path, func)
        # the log2(e) factor of the exp argument comes first in softplus_fast
        got = [g for g in got if abs(g - 1.4426950408889634) > 1e-6]
        assert len(got) == 9, (path, got)
        got = np.array(got)
        # each printed coefficient is the derived one to fp32 precision
        assert np.all(np.abs(got - ref) <= 2 ** -23 * np.abs(ref) + 1e-12), (path, got - ref)
        assert np.array_equal(got.astype(np.float32), ref32) or \
            np.max(np.abs(got.astype(np.float32) - ref32) / np.abs(ref32)) <= 2 ** -23


def test_softplus_polynomial_error_bound():
    coef = np.array(_source_coefficients(os.path.join(CSRC, "ssm_common.cuh"),
                                         "float softplus_fast("))
    coef = coef[np.abs(coef - 1.4426950408889634) > 1e-6].astype(np.float32)
    x = np.concatenate([np.geomspace(1e-30, 1e-3, 2000), np.linspace(1e-3, 1.0, 400001)])
    x = x.astype(np.float32)
    # Horner with fused multiply-adds, as the kernel evaluates it (fmaf): the
    # product of two fp32 values is exact in fp64, so one rounding to fp32
    # after the fp64 sum stands for the FMA's single rounding
    x64 = x.astype(np.float64)
    p = np.full_like(x64, coef[0])
    for c in coef[1:]:
        p = (p * x64 + np.float64(c)).astype(np.float32).astype(np.float64)
    got = (x64 * p).astype(np.float32).astype(np.float64)
    ref = np.log1p(x.astype(np.float64))
    rel = np.abs(got - ref) / ref
    assert rel.max() <= 2.3e-7, rel.max()


def test_reciprocal_seed_and_newton_steps():
    # SiLU's 1/(1 + e^-z) runs on the FMA pipe: seed bits(y0) = K - bits(d),
    # then three Newton-Raphson steps.  K is the constant that minimises the
    # seed's maximum relative error over a binade (a direct search gives
    # 5.05 %), and three steps bring any d in [1, 2^64] to fp32 accuracy.
    src = open(os.path.join(CSRC, "ssm_fwd.cu")).read()
    K = int(re.search(r"kRcpSeed = (0x[0-9A-Fa-f]+);", src).group(1), 16)
    x = np.linspace(1.0, 2.0, 100001, dtype=np.float32)
    bits = x.view(np.int32).astype(np.int64)

    def seed_err(k):
        y = (np.int64(k) - bits).astype(np.int32).view(np.float32).astype(np.float64)
        return float(np.max(np.abs(y * x - 1.0)))
    e = seed_err(K)
    assert e <= 0.0506
    assert all(seed_err(K + dk) >= e - 1e-9 for dk in (-0x800, -0x40, 0x40, 0x800))
    d = np.concatenate([np.linspace(1.0, 4.0, 5001), np.geomspace(4.0, 1.8e19, 5001)]).astype(np.float32)
    y = (np.int64(K) - d.view(np.int32).astype(np.int64)).astype(np.int32).view(np.float32)
    for _ in range(3):  # y + y (1 - d y), each product-sum rounded once like an FMA
        e1 = (1.0 - d.astype(np.float64) * y.astype(np.float64)).astype(np.float32)
        y = (y.astype(np.float64) + y.astype(np.float64) * e1.astype(np.float64)).astype(np.float32)
    rel = np.abs(y.astype(np.float64) * d.astype(np.float64) - 1.0)
    assert rel.max() <= 3e-7, rel.max()


def _zoh_constants():
    src = open(os.path.join(CSRC, "ssm_common.cuh")).read()
    got = {}
    for name in ([f"kZohW{k}" for k in range(1, 6)] + [f"kZohP{m}" for m in range(8)]
                 + ["kZohWSmall", "kZohPSmall"]):
        m = re.search(r"\b" + name + r" = " + FLOAT, src)
        assert m, name
        got[name] = float(m.group(1))
    return got


def test_zoh_series_coefficients():
    # (e^x - 1)/x = sum_k x^k / (k+1)!, evaluated in y = x / ln 2 (the ex2
    # argument): term k carries ln2^k / (k+1)!; the switch to (e^x - 1)/A is at
    # |x| = 1/4, i.e. |y| = 0.25 / ln 2
    import math
    c = _zoh_constants()
    for k in range(1, 6):
        ref = math.log(2) ** k / math.factorial(k + 1)
        assert abs(c[f"kZohW{k}"] - ref) <= 2 ** -23 * ref, (k, c[f"kZohW{k}"], ref)
    assert abs(c["kZohWSmall"] - 0.25 / math.log(2)) <= 2 ** -23


def test_zoh_two_branch_error_bound():
    # The consumer's Delta (e^x - 1)/x: the series to x^5 below |x| = 1/4, else
    # (a - 1)/A with a = 2^(x/ln 2) from the special-function unit.  Emulated in
    # fp32 with a perturbed by the ex2 unit's error (up to 2 ulp, either sign),
    # relative to the exact value: below 1e-6 everywhere.
    c = _zoh_constants()
    T = [np.float32(c[f"kZohW{k}"]) for k in range(5, 0, -1)]
    x = np.concatenate([-np.geomspace(1e-8, 60.0, 40001), np.geomspace(1e-8, 10.0, 20001)])
    y = (x / np.log(2)).astype(np.float32)
    exact = np.expm1(x) / x
    # series branch, fused Horner in fp32 (one rounding per step)
    q = np.full_like(y, T[0], dtype=np.float32)
    for t in T[1:] + [np.float32(1.0)]:
        q = (q.astype(np.float64) * y.astype(np.float64) + np.float64(t)).astype(np.float32)
    worst = 0.0
    for ulps in (-2, 0, 2):
        a = (np.exp2(y.astype(np.float64)) * (1 + ulps * 2.0 ** -24)).astype(np.float32)
        # Delta = 1, A = x: (a - 1) * (1/A) against the series
        big = ((a - np.float32(1)).astype(np.float32) * (np.float32(1) / x.astype(np.float32))).astype(np.float32)
        got = np.where(np.abs(y) < np.float32(c["kZohWSmall"]), q, big).astype(np.float64)
        worst = max(worst, float(np.max(np.abs(got / exact - 1))))
    assert worst < 1e-6, worst


def test_psi_series_coefficients():
    # the backward's A derivative Delta^2 psi(x), psi(x) = (x e^x - (e^x - 1)) / x^2:
    # its series terms ln2^m (m+1)/(m+2)! in y = x / ln 2 (switch at |x| = 1/2),
    # and the series against the closed form where that is accurate
    import math
    c = _zoh_constants()
    ln2 = math.log(2)
    for m in range(8):
        ref = ln2 ** m * (m + 1) / math.factorial(m + 2)
        assert abs(c[f"kZohP{m}"] - ref) <= 2 ** -23 * ref, m
    assert abs(c["kZohPSmall"] - 0.5 / ln2) <= 2 ** -22
    x = np.linspace(-0.5, 0.5, 2001)
    x = x[np.abs(x) > 1e-3]
    y = x / ln2
    q = np.zeros_like(y)
    for m in range(7, -1, -1):
        q = q * y + c[f"kZohP{m}"]
    exact = (x * np.exp(x) - np.expm1(x)) / x ** 2
    assert np.max(np.abs(q / exact - 1)) < 1e-7
