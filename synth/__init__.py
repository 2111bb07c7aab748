"""Seeded synthetic inputs for the selective scan (S6).

This module is the only code shared by the fp64 oracle (``oracle/``) and the
CUDA path (``selective_state_space_54_b200``).  It draws random tensors and
lays them out; it holds none of the scan's arithmetic.

Workloads follow the layer shapes the Mamba pages discuss ("Mamba: Linear-Time
Sequence Modeling with Selective State Spaces", reading guide, section
"O Mecanismo de Seleção": B_t, C_t are Linear_N(x_t) projections shared by all
D channels, Delta_t = softplus(Parameter + s_Delta(x_t))):

* u, delta (raw, before bias and softplus), z, B, C, dy ~ N(0, 1), drawn in
  fp32 and rounded to nearest-even bf16 when the io dtype is bf16;
* A[d, n] = -(n + 1) (S4D-real), fp32;
* D ~ N(0, 1), fp32;
* delta_bias[d] = log(expm1(dt_d)) (the inverse of softplus) with dt_d
  log-uniform in [1e-3, 1e-1], fp32.

Layouts (row-major, last index contiguous):
  u, delta, z, dy : (batch, dim, seqlen)
  B, C            : (batch, seqlen, dstate)
  A               : (dim, dstate)
  D, delta_bias   : (dim,)

bf16 tensors are returned as ``uint16`` arrays holding the raw bf16 bits.

Random streams: tensor ``k`` of a case with seed ``s`` is drawn in fixed
chunks of 2**22 elements, chunk ``j`` from PCG64(SeedSequence([s, k, j])), so
the values do not depend on the number of generator threads.
"""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field

import numpy as np

F32 = "f32"
BF16 = "bf16"

_CHUNK = 1 << 22
# stream ids, fixed forever so stored seeds keep meaning the same values
_STREAM = {"u": 0, "delta": 1, "z": 2, "B": 3, "C": 4, "D": 5, "dt": 6, "dy": 7,
           "perm": 8}


@dataclass(frozen=True)
class Workload:
    """One synthetic workload: a layer shape, an io dtype and a seed."""
    name: str
    batch: int
    seqlen: int
    dim: int
    dstate: int
    dtype: str
    seed: int
    last_state: bool = False
    backward: bool = False
    sample_channels: int = 0  # >0: the oracle checks this many seeded channels
    notes: str = ""
    extra: dict = field(default_factory=dict)

    @property
    def bld(self) -> int:
        return self.batch * self.seqlen * self.dim

    @property
    def bldn(self) -> int:
        return self.bld * self.dstate


# The five workloads of the selective-scan benchmark, by what they are.
WORKLOADS = {
    "tiny-fp32": Workload("tiny-fp32", 1, 64, 16, 4, F32, 0,
                          notes="tiny fp32 forward, z-gating on"),
    "mamba-130m-layer": Workload("mamba-130m-layer", 8, 2048, 1536, 16, BF16, 1,
                                 notes="Mamba-130M layer forward"),
    "mamba-2.8b-layer": Workload("mamba-2.8b-layer", 4, 8192, 5120, 16, BF16, 2,
                                 last_state=True,
                                 notes="Mamba-2.8B layer forward + last_state"),
    "million-length": Workload("million-length", 1, 1 << 20, 1024, 16, BF16, 3,
                               sample_channels=64,
                               notes="1M-length forward, split-L path"),
    "mamba-1.4b-layer-train": Workload("mamba-1.4b-layer-train", 8, 2048, 4096, 16,
                                       BF16, 4, backward=True,
                                       notes="Mamba-1.4B layer forward+backward"),
    "mamba-2.8b-decode": Workload("mamba-2.8b-decode", 128, 1, 5120, 16, BF16, 5,
                                  last_state=True, extra={"decode": True},
                                  notes="Mamba-2.8B layer single-token step, fp32 state "
                                        "(batch, d_inner, d_state) updated in place"),
}
WORKLOAD_ORDER = list(WORKLOADS)


def _threads(threads: int | None) -> int:
    if threads:
        return threads
    return max(1, min(32, os.cpu_count() or 1))


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 to bf16 (round to nearest, ties to even); returns uint16 bits."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    v = x.view(np.uint32).copy()
    lsb = (v >> np.uint32(16)) & np.uint32(1)
    v += np.uint32(0x7FFF)
    v += lsb
    return (v >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bits to fp32."""
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def to_f64(x: np.ndarray, dtype: str) -> np.ndarray:
    """Exact widening of a stored io tensor (bf16 bits or fp32) to fp64."""
    if dtype == BF16:
        return bf16_bits_to_f32(x).astype(np.float64)
    return np.asarray(x, dtype=np.float32).astype(np.float64)


def _normal_into(out: np.ndarray, seed: int, stream: int, dtype: str, threads: int) -> None:
    flat = out.reshape(-1)
    n = flat.size
    nchunks = (n + _CHUNK - 1) // _CHUNK

    def one(j: int) -> None:
        lo, hi = j * _CHUNK, min(n, (j + 1) * _CHUNK)
        g = np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, stream, j])))
        x = g.standard_normal(hi - lo, dtype=np.float32)
        if dtype == BF16:
            v = x.view(np.uint32)
            lsb = (v >> np.uint32(16)) & np.uint32(1)
            v += np.uint32(0x7FFF)
            v += lsb
            flat[lo:hi] = (v >> np.uint32(16)).astype(np.uint16)
        else:
            flat[lo:hi] = x

    if nchunks == 1:
        one(0)
    else:
        with ThreadPoolExecutor(min(threads, nchunks)) as ex:
            list(ex.map(one, range(nchunks)))


def normal(shape, seed: int, stream: str | int, dtype: str = F32, threads: int | None = None):
    """N(0,1) tensor of ``shape``; bf16 as uint16 bits, f32 as float32."""
    sid = _STREAM[stream] if isinstance(stream, str) else int(stream)
    out = np.empty(shape, dtype=np.uint16 if dtype == BF16 else np.float32)
    _normal_into(out, seed, sid, dtype, _threads(threads))
    return out


def s4d_real_A(dim: int, dstate: int) -> np.ndarray:
    """A[d, n] = -(n + 1), the S4D-real initialisation, fp32."""
    return np.broadcast_to(-(np.arange(dstate, dtype=np.float32) + 1.0), (dim, dstate)).copy()


def delta_bias_loguniform(dim: int, seed: int, lo: float = 1e-3, hi: float = 1e-1) -> np.ndarray:
    """delta_bias = log(expm1(dt)), dt log-uniform in [lo, hi], fp32."""
    g = np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, _STREAM["dt"], 0])))
    dt = np.exp(g.uniform(np.log(lo), np.log(hi), size=dim))
    return np.log(np.expm1(dt)).astype(np.float32)


def make_case(batch: int, dim: int, seqlen: int, dstate: int, dtype: str = BF16,
              seed: int = 0, *, with_z: bool = True, with_D: bool = True,
              with_bias: bool = True, with_dy: bool = False,
              threads: int | None = None) -> dict:
    """All inputs of one scan problem, laid out as the module docstring says."""
    th = _threads(threads)
    case = {
        "batch": batch, "dim": dim, "seqlen": seqlen, "dstate": dstate,
        "dtype": dtype, "seed": seed,
        "u": normal((batch, dim, seqlen), seed, "u", dtype, th),
        "delta": normal((batch, dim, seqlen), seed, "delta", dtype, th),
        "B": normal((batch, seqlen, dstate), seed, "B", dtype, th),
        "C": normal((batch, seqlen, dstate), seed, "C", dtype, th),
        "A": s4d_real_A(dim, dstate),
        "z": normal((batch, dim, seqlen), seed, "z", dtype, th) if with_z else None,
        "D": normal((dim,), seed, "D", F32, th) if with_D else None,
        "delta_bias": delta_bias_loguniform(dim, seed) if with_bias else None,
        "dy": normal((batch, dim, seqlen), seed, "dy", dtype, th) if with_dy else None,
    }
    return case


def make_workload(w: Workload | str, threads: int | None = None) -> dict:
    """Inputs of a named workload (delta_softplus on, z-gating on)."""
    if isinstance(w, str):
        w = WORKLOADS[w]
    return make_case(w.batch, w.dim, w.seqlen, w.dstate, w.dtype, w.seed,
                     with_dy=w.backward, threads=threads)


def sample_channels(w: Workload | str, count: int | None = None) -> np.ndarray:
    """Seeded choice (without replacement) of flat channel ids b*dim + d."""
    if isinstance(w, str):
        w = WORKLOADS[w]
    k = count or w.sample_channels or 64
    g = np.random.Generator(np.random.PCG64(np.random.SeedSequence([w.seed, _STREAM["perm"], 0])))
    return np.sort(g.permutation(w.batch * w.dim)[:k])


def subset_case(case: dict, channels) -> list:
    """Split a case into per-batch sub-cases holding only ``channels``.

    Returns a list of (b, dims, subcase) where subcase is a batch-1 problem
    with the selected channels of batch b; used to check long problems one
    channel at a time against the oracle.
    """
    dim = case["dim"]
    channels = np.asarray(channels)
    out = []
    for b in np.unique(channels // dim):
        dims = np.sort(channels[channels // dim == b] % dim)
        sub = dict(case)
        sub["batch"] = 1
        sub["dim"] = len(dims)
        for k in ("u", "delta", "z", "dy"):
            if case.get(k) is not None:
                sub[k] = np.ascontiguousarray(case[k][b:b + 1, dims, :])
        for k in ("B", "C"):
            sub[k] = np.ascontiguousarray(case[k][b:b + 1])
        sub["A"] = np.ascontiguousarray(case["A"][dims])
        for k in ("D", "delta_bias"):
            if case.get(k) is not None:
                sub[k] = np.ascontiguousarray(case[k][dims])
        out.append((int(b), dims, sub))
    return out
