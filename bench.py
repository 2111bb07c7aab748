#!/usr/bin/env python3
"""Benchmark of the B200 selective scan (S6) forward.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME]

A step is one forward scan (softplus, discretisation, recurrence, C
contraction, D skip, SiLU gate, last_state) over one batch of the workload,
inputs resident in HBM.  The default workload is the Mamba-2.8B layer shape
(batch 4, L 8192, d_inner 5120, d_state 16, bf16 io, fp32 state).  Multi-GPU
runs (torchrun, one rank per GPU) process one independent replica per rank:
the scan's (batch, channel) rows are independent, so there is no collective
(weak scaling).  Rank 0 prints one JSON line.

--impl reference times the fp64 CPU oracle on the host cores (bounded samples
of the same workload), the only reference implementation there is.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "selective-scan fwd/bwd tokens·channels/s and % of HBM/SFU roofline, 1 B200"
UNIT = "tokens·channels/s"
MUFU_EX2_PER_CLK_PER_SM = 16  # special-function unit ex2 rate per SM and clock


def _csrc(*names):
    return [os.path.join(ROOT, "selective_state_space_54_b200", "csrc", f) for f in names]


# committed ncu summary of each timed kernel and the sources it was captured from
PROFILE_TRAFFIC = {
    "lookback": (os.path.join(ROOT, "profiles", "fwd_lookback_mamba-2.8b-layer.md"),
                 _csrc("ssm_fwd.cu", "ssm_common.cuh")),
    "lookback_ws": (os.path.join(ROOT, "profiles", "fwd_ws_mamba-2.8b-layer.md"),
                    _csrc("ssm_fwd.cu", "ssm_common.cuh")),
    "decode": (os.path.join(ROOT, "profiles", "step_mamba-2.8b-decode.md"),
               _csrc("ssm_step.cu", "ssm_common.cuh")),
    "conv1d": (os.path.join(ROOT, "profiles", "conv1d_mamba-2.8b-layer.md"),
               _csrc("ssm_conv.cu", "ssm_common.cuh")),
    "bwd16": (os.path.join(ROOT, "profiles", "bwd16_mamba-1.4b-layer-train.md"),
              _csrc("ssm_bwd16.cu", "ssm_common.cuh")),
}
KERNEL_SOURCES = _csrc("ssm_fwd.cu", "ssm_common.cuh")


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="mamba-2.8b-layer", choices=list(synth.WORKLOADS))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-bwd", action="store_true",
                    help="skip the training-workload forward+backward measurement")
    ap.add_argument("--lanes", type=int, default=0, choices=[0, 2, 4],
                    help="lanes per channel (0: the library's choice)")
    ap.add_argument("--path", default="auto",
                    choices=["auto", "lookback", "split_l", "per_group", "lookback_ws"])
    ap.add_argument("--batch", type=int, default=0,
                    help="override the workload's batch (smaller cases for profiling only)")
    ap.add_argument("--seqlen", type=int, default=0,
                    help="override the workload's sequence length (smaller cases for profiling only)")
    return ap.parse_args()


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": d.get("hbm_gbs", 6650.0), "sm_max_mhz": d.get("sm_max_mhz", 1965.0),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "sm_max_mhz": 1965.0, "source": "fallback"}


def alg_bytes(w: synth.Workload) -> int:
    """Bytes every input and output must cross HBM once."""
    es = 2 if w.dtype == synth.BF16 else 4
    bld = w.bld
    b = 4 * bld * es                                   # u, delta, z in; y out
    b += 2 * w.batch * w.seqlen * w.dstate * es        # B, C
    b += w.dim * w.dstate * 4 + 2 * w.dim * 4          # A, D, delta_bias
    if w.last_state:
        b += w.batch * w.dim * w.dstate * 4
    return b


def source_sha(sources=None) -> str:
    h = hashlib.sha256()
    for p in sources or KERNEL_SOURCES:
        with open(p, "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def profiled_traffic(path: str):
    """dram bytes per launch from the committed ncu summary, if the kernel is unchanged."""
    f, sources = PROFILE_TRAFFIC.get(path, (None, None))
    if not f or not os.path.exists(f):
        return None
    vals = {}
    for line in open(f):
        if ":" in line and line.strip().startswith("- "):
            k, v = line.strip()[2:].split(":", 1)
            vals[k.strip()] = v.strip().strip("`")
    if vals.get("kernel_source_sha256_16") != source_sha(sources):
        return None
    try:
        return float(vals["dram_bytes_per_launch_full_size"])
    except (KeyError, ValueError):
        return None


class ClockSampler:
    """nvidia-smi clock / throttle sampling during the timed region."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = os.path.join("/tmp", f"ssm_clocks_{os.getpid()}.csv")

    def __enter__(self):
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=self.f, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            time.sleep(0.15)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.f.close()

    def summary(self):
        if self.proc is None or not os.path.exists(self.path):
            return None
        rows = []
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append({"sm": float(parts[1]), "max": float(parts[2]),
                             "power": float(parts[3]) if parts[3] not in ("[N/A]", "") else None,
                             "active": parts[4], "hw": parts[5], "hw_thermal": parts[6],
                             "sw_thermal": parts[7], "sw_power": parts[8]})
            except ValueError:
                continue
        if not rows:
            return None
        loaded = [r for r in rows if r["power"] is None or r["power"] > 250] or rows
        reasons = set()
        for r in loaded:
            for k, name in (("hw", "hw_slowdown"), ("hw_thermal", "hw_thermal_slowdown"),
                            ("sw_thermal", "sw_thermal_slowdown"), ("sw_power", "sw_power_cap")):
                if r[k].lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(r["sm"] for r in loaded),
                "sm_max_mhz": max(r["max"] for r in rows), "samples": len(loaded),
                "reasons": sorted(reasons)}


def dist_max(x: float, world: int, device) -> float:
    """Max of a per-rank time over all ranks (every rank calls it, same order)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_value(world: int, units_per_rank: float, seconds_max: float) -> float:
    """Whole-job throughput: every rank processes its own replica (weak scaling)."""
    return world * units_per_rank / seconds_max


def init_dist(args):
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import torch.distributed as dist
        from datetime import timedelta
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    return world, rank, local


def cpu_baseline(w: synth.Workload, case: dict, target_s: float = 12.0, y_gpu=None, ls_gpu=None):
    """The fp64 oracle as it stands, timed on the host cores on a bounded sample.
    With the GPU's y and last_state of the timed run (host tensors), also their
    agreement with the oracle on the rows of the final sample (untimed):
    returns (baseline, parity)."""
    import oracle
    threads = oracle.default_threads()
    nch = w.batch * w.dim
    k = min(nch, max(threads, 16))
    t_first = None
    while True:
        chans = synth.sample_channels(w, k)
        subs = synth.subset_case(case, chans)
        dt = 0.0
        acc = {"y": [0.0, 0.0, 0.0, 0.0], "last_state": [0.0, 0.0, 0.0, 0.0]}  # err2, ref2, max err, max ref
        for b, dims, sub in subs:
            t0 = time.perf_counter()
            ref = oracle.fwd(sub, nthreads=threads)
            dt += time.perf_counter() - t0
            if y_gpu is not None:
                for key, got_t in (("y", y_gpu), ("last_state", ls_gpu)):
                    got = got_t[b, dims].double().numpy()
                    r = ref[key][0]
                    a = acc[key]
                    a[0] += float(np.sum((got - r) ** 2))
                    a[1] += float(np.sum(r ** 2))
                    a[2] = max(a[2], float(np.max(np.abs(got - r))))
                    a[3] = max(a[3], float(np.max(np.abs(r))))
        t_first = t_first or dt
        if dt >= target_s * 0.5 or k >= nch:
            break
        k = min(nch, int(k * max(2.0, target_s / max(dt, 1e-3))))
    base = {"value": k * w.seqlen / dt, "unit": UNIT, "cores": threads, "kind": "oracle",
            "sample": f"{k} of {nch} (batch, channel) rows over the full L={w.seqlen}, "
                      f"fp64, {dt:.1f} s"}
    parity = None
    if y_gpu is not None:
        parity = {"against": "the fp64 oracle on the same inputs", "rows": f"{k} of {nch}",
                  "tolerance": ("rel-L2 <= 2e-3 and max-abs <= 1e-2 max|ref|" if w.dtype == synth.BF16
                                else "rel-L2 <= 1e-5")}
        for key, (e2, r2, me, mr) in acc.items():
            parity[key] = {"rel_l2": (e2 / r2) ** 0.5 if r2 > 0 else 0.0, "max_abs": me, "max_ref": mr}
    return base, parity


def run_reference(args, w):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    case = synth.make_workload(w)
    threads = oracle.default_threads()
    nch = w.batch * w.dim
    # size one step to about 3 s of host work
    k = min(nch, max(threads, 8))
    chans = synth.sample_channels(w, k)
    subs = synth.subset_case(case, chans)
    t0 = time.perf_counter()
    for _, _, sub in subs:
        oracle.fwd(sub, nthreads=threads)
    dt = time.perf_counter() - t0
    k = min(nch, max(1, int(k * 3.0 / max(dt, 1e-3))))
    chans = synth.sample_channels(w, k)
    subs = synth.subset_case(case, chans)
    for _ in range(args.warmup):
        for _, _, sub in subs:
            oracle.fwd(sub, nthreads=threads)
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        for _, _, sub in subs:
            oracle.fwd(sub, nthreads=threads)
        times.append(time.perf_counter() - t0)
    per_step = sum(times) / len(times)
    value = k * w.seqlen / per_step
    sample = f"{k} of {nch} (batch, channel) rows over the full L={w.seqlen} per step, fp64"
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": per_step * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_of(w, "oracle"),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def to_torch(x, device):
    """numpy input (bf16 bits as uint16, or fp32) -> torch tensor on device."""
    import torch
    if x.dtype == np.uint16:
        return torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).to(device).view(torch.bfloat16)
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(device)


def config_of(w, path):
    return {"workload": w.name, "batch": w.batch, "seqlen": w.seqlen, "d_inner": w.dim,
            "d_state": w.dstate, "io_dtype": w.dtype, "state_dtype": "f32",
            "delta_softplus": True, "z_gate": True, "last_state": w.last_state, "path": path,
            "l2": "inputs larger than L2 (no flush)" if alg_bytes(w) > 126e6 else "L2 resident",
            "seed": w.seed}


def time_fwd_bwd(torch, dev, stream, fwd, bwd, steps):
    """Device time of `steps` forward + backward steps queued back to back,
    with events between the two halves of each step and one synchronise on
    each side of the whole sequence, so the host's launch work overlaps the
    device's instead of being timed.  Returns the summed forward and backward
    milliseconds."""
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
    torch.cuda.synchronize(dev)
    for e in evs:
        e[0].record(stream)
        fwd()
        e[1].record(stream)
        bwd()
        e[2].record(stream)
    torch.cuda.synchronize(dev)
    return (sum(e[0].elapsed_time(e[1]) for e in evs), sum(e[1].elapsed_time(e[2]) for e in evs))


def measure_training(ssm, torch, dev, args, world, barrier, max_over_ranks, w=None):
    """Forward + recomputation backward on the Mamba-1.4B layer training shape."""
    w = w or synth.WORKLOADS["mamba-1.4b-layer-train"]
    case = synth.make_workload(w)
    g = {k: to_torch(case[k], dev) for k in ("u", "delta", "z", "B", "C", "dy")}
    for k in ("A", "D", "delta_bias"):
        g[k] = torch.from_numpy(np.asarray(case[k], np.float32)).to(dev)
    del case
    y = torch.empty_like(g["u"])
    # the training step: the forward saves the state entering every 8-step
    # chunk in its workspace, and the backward starts from those
    shape = ssm.make_shape(w.batch, w.dim, w.seqlen, w.dstate,
                           ssm.SSM_BF16 if w.dtype == synth.BF16 else ssm.SSM_F32,
                           flags=ssm.SSM_FLAG_SAVE_STATES)
    ws_f = torch.empty(ssm.fwd_workspace_bytes(shape), dtype=torch.uint8, device=dev)
    ws_b = torch.empty(ssm.bwd_workspace_bytes(shape), dtype=torch.uint8, device=dev)
    out = {"du": torch.empty_like(g["u"]), "ddelta": torch.empty_like(g["u"]),
           "dz": torch.empty_like(g["u"]), "dB": torch.empty_like(g["B"]),
           "dC": torch.empty_like(g["C"]),
           "dA": torch.empty((w.dim, w.dstate), dtype=torch.float32, device=dev),
           "dD": torch.empty((w.dim,), dtype=torch.float32, device=dev),
           "ddelta_bias": torch.empty((w.dim,), dtype=torch.float32, device=dev)}
    stream = torch.cuda.current_stream(dev)

    def fwd():
        ssm.scan_fwd(g["u"], g["delta"], g["A"], g["B"], g["C"], g["D"], g["z"], g["delta_bias"],
                     y=y, workspace=ws_f, save_states=True)

    def bwd():
        ssm.scan_bwd(g["u"], g["delta"], g["A"], g["B"], g["C"], g["D"], g["z"], g["delta_bias"],
                     g["dy"], out=out, workspace=ws_b, fwd_workspace=ws_f)

    for _ in range(max(3, args.warmup)):
        fwd()
        bwd()
    torch.cuda.synchronize(dev)
    steps = max(3, min(args.steps, 10))
    barrier()
    t_f, t_b = time_fwd_bwd(torch, dev, stream, fwd, bwd, steps)
    barrier()
    ms_f = max_over_ranks(t_f / steps)
    ms_b = max_over_ranks(t_b / steps)
    # The roofline counts the method's own special-function work: one exp2
    # per (b, t, d, n) element (the decay exp(Delta A) the backward must
    # recompute).  The kernel's own count is reported beside it: the d_state-16
    # backward exponentiates 6 of every 8 steps to rebuild the 2-step group
    # entry states of a chunk, then every step again for the group whose
    # decays the reverse pass uses (1.75 per element).
    ex2_per_element = 1
    kernel_ex2 = 1.75
    pk = peaks()
    sm_count = torch.cuda.get_device_properties(dev).multi_processor_count
    ex2_peak = sm_count * MUFU_EX2_PER_CLK_PER_SM * pk["sm_max_mhz"] * 1e6
    bwd_achieved = ex2_per_element * w.bldn / (ms_b * 1e-3)
    bwd_roofline = {"bound": "alu", "achieved": bwd_achieved / 1e12, "peak": ex2_peak / 1e12,
                    "unit": "Tex2/s", "frac": bwd_achieved / ex2_peak,
                    # the committed capture is of this workload's Euler, channel-major launch
                    "traffic": profiled_traffic("bwd16") if w.name == "mamba-1.4b-layer-train" else None,
                    "kernel": "k_bwd16", "ex2_per_element": ex2_per_element,
                    "kernel_ex2_per_element": kernel_ex2,
                    "kernel_mufu_frac": kernel_ex2 * w.bldn / (ms_b * 1e-3) / ex2_peak,
                    # the FP32-pipe view: the gradient formulas need 11 fp32 operations
                    # per (b, t, d, n) element (a fused multiply-add counted once): the
                    # state recomputation x = Delta A, Delta u B, a h + b (3); the reverse
                    # recurrence dy C + (a g) (2); dC, dB, sum_n g B, g a h_{t-1}, dA and
                    # dDelta's A term (6); peak = SMs x 128 fp32 lanes x clock
                    "fp32_pipe": {"ops_per_element": 11,
                                  "peak_tops": sm_count * 128 * pk["sm_max_mhz"] * 1e6 / 1e12,
                                  "frac": 11 * w.bldn / (ms_b * 1e-3) / (sm_count * 128 * pk["sm_max_mhz"] * 1e6)},
                    "peak_basis": f"{sm_count} SMs x {MUFU_EX2_PER_CLK_PER_SM} ex2/clk x "
                                  f"{pk['sm_max_mhz']:.0f} MHz (sm_max_mhz, {pk['source']})"}
    variants = measure_training_variants(ssm, torch, dev, g, y, out, w, steps, barrier, max_over_ranks)
    return {"workload": w.name, "batch": w.batch, "seqlen": w.seqlen, "d_inner": w.dim,
            "d_state": w.dstate, "io_dtype": w.dtype, "steps": steps,
            "fwd_path": ssm.fwd_path(shape), "saved_states": True, "fwd_ms": ms_f, "bwd_ms": ms_b,
            **variants,
            "bwd_roofline": bwd_roofline,
            "value": aggregate_value(world, w.bld, (ms_f + ms_b) * 1e-3), "unit": UNIT + " (fwd+bwd)",
            "bwd_value": aggregate_value(world, w.bld, ms_b * 1e-3),
            "bwd_ex2_per_element": ex2_per_element, "bwd_kernel_ex2_per_element": kernel_ex2,
            "bwd_kernels_per_step": 2}


def measure_training_variants(ssm, torch, dev, g, y, out, w, steps, barrier, max_over_ranks):
    """The same training step (forward saving chunk states, backward from them)
    with the exact zero-order-hold input term (the general backward kernel)
    and with token-major activations ([batch][seqlen][d_inner] u, delta, z,
    dout and their gradients; the d_state-16 kernel)."""
    stream = torch.cuda.current_stream(dev)
    res = {}
    tm = None
    if w.dtype == synth.BF16 and w.dim % 8 == 0:
        tm = {k: g[k].transpose(1, 2).contiguous() for k in ("u", "delta", "z", "dy")}
        tm_out = dict(out, du=torch.empty_like(tm["u"]), ddelta=torch.empty_like(tm["u"]),
                      dz=torch.empty_like(tm["u"]))
        y_tm = torch.empty_like(tm["u"])
    for name, flags in (("zoh_exact", ssm.SSM_FLAG_ZOH_EXACT), ("token_major", ssm.SSM_FLAG_TOKEN_MAJOR)):
        tok = name == "token_major"
        if tok and tm is None:
            continue
        shape = ssm.make_shape(w.batch, w.dim, w.seqlen, w.dstate,
                               ssm.SSM_BF16 if w.dtype == synth.BF16 else ssm.SSM_F32,
                               flags=ssm.SSM_FLAG_SAVE_STATES | flags)
        ws_f = torch.empty(ssm.fwd_workspace_bytes(shape), dtype=torch.uint8, device=dev)
        ws_b = torch.empty(ssm.bwd_workspace_bytes(shape), dtype=torch.uint8, device=dev)
        a = tm if tok else g
        o = tm_out if tok else out
        yy = y_tm if tok else y

        def fwd():
            ssm.scan_fwd(a["u"], a["delta"], g["A"], g["B"], g["C"], g["D"], a["z"], g["delta_bias"],
                         y=yy, workspace=ws_f, save_states=True, zoh_exact=not tok, token_major=tok)

        def bwd():
            ssm.scan_bwd(a["u"], a["delta"], g["A"], g["B"], g["C"], g["D"], a["z"], g["delta_bias"],
                         a["dy"], out=o, workspace=ws_b, fwd_workspace=ws_f, zoh_exact=not tok,
                         token_major=tok)

        for _ in range(3):
            fwd()
            bwd()
        torch.cuda.synchronize(dev)
        ssm.check(ws_f)
        barrier()
        t_f, t_b = time_fwd_bwd(torch, dev, stream, fwd, bwd, steps)
        barrier()
        ssm.check(ws_f)
        res[name] = {"fwd_ms": max_over_ranks(t_f / steps), "bwd_ms": max_over_ranks(t_b / steps),
                     "fwd_path": ssm.fwd_path(shape),
                     "bwd_kernel": "k_bwd16 (exact ZOH)" if not tok else "k_bwd16 (token-major)"}
        del ws_f, ws_b
    return res


def measure_forward(ssm, torch, dev, args, world, barrier, max_over_ranks, name):
    """The forward alone on another workload (path AUTO, inputs resident in
    HBM), with its special-function roofline.  The roofline counts the
    method's one exp2 per (b, t, d, n) element; the split-L schedule's own
    count (each element exponentiated in both passes) is reported beside it."""
    w = synth.WORKLOADS[name]
    case = synth.make_workload(w)
    g = {k: to_torch(case[k], dev) for k in ("u", "delta", "z", "B", "C")}
    for k in ("A", "D", "delta_bias"):
        g[k] = torch.from_numpy(np.asarray(case[k], np.float32)).to(dev)
    del case
    y = torch.empty_like(g["u"])
    ls = torch.empty((w.batch, w.dim, w.dstate), dtype=torch.float32, device=dev)
    shape = ssm.make_shape(w.batch, w.dim, w.seqlen, w.dstate,
                           ssm.SSM_BF16 if w.dtype == synth.BF16 else ssm.SSM_F32)
    path = ssm.fwd_path(shape)
    ws = torch.empty(ssm.fwd_workspace_bytes(shape), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        ssm.scan_fwd(g["u"], g["delta"], g["A"], g["B"], g["C"], g["D"], g["z"], g["delta_bias"],
                     y=y, last_state=ls, return_last_state=True, workspace=ws)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize(dev)
    ssm.check(ws)
    k = max(3, min(args.steps, 10 if w.bld > 5e8 else 20))
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize(dev)
    ev0.record(stream)
    for _ in range(k):
        step()
    ev1.record(stream)
    torch.cuda.synchronize(dev)
    ssm.check(ws)
    ms = max_over_ranks(ev0.elapsed_time(ev1) / k)
    pk = peaks()
    sm_count = torch.cuda.get_device_properties(dev).multi_processor_count
    ex2_peak = sm_count * MUFU_EX2_PER_CLK_PER_SM * pk["sm_max_mhz"] * 1e6
    kernel_ex2 = 2 if path == "split_l" else 1
    achieved = w.bldn / (ms * 1e-3)
    nbytes = alg_bytes(w)
    del g, y, ls, ws
    return {"workload": w.name, "batch": w.batch, "seqlen": w.seqlen, "d_inner": w.dim,
            "d_state": w.dstate, "io_dtype": w.dtype, "path": path, "steps": k,
            "l2": "inputs larger than L2 (no flush)" if nbytes > 126e6 else "L2 resident",
            "ms_per_step": ms, "value": aggregate_value(world, w.bld, ms * 1e-3), "unit": UNIT,
            "roofline": {"bound": "alu", "achieved": achieved / 1e12, "peak": ex2_peak / 1e12,
                         "unit": "Tex2/s", "frac": achieved / ex2_peak, "traffic": None,
                         "ex2_per_element": 1, "kernel_ex2_per_element": kernel_ex2,
                         "kernel_mufu_frac": kernel_ex2 * achieved / ex2_peak,
                         "algorithmic_bytes": nbytes,
                         "hbm_achieved_gbs": nbytes / (ms * 1e-3) / 1e9,
                         "hbm_frac": nbytes / (ms * 1e-3) / 1e9 / pk["hbm_gbs"],
                         "peak_basis": f"{sm_count} SMs x {MUFU_EX2_PER_CLK_PER_SM} ex2/clk x "
                                       f"{pk['sm_max_mhz']:.0f} MHz (sm_max_mhz, {pk['source']})"},
            "gpu_launches": k * {"split_l": 3, "lookback_ws": 2}.get(path, 1)}


def decode_bytes(w: synth.Workload) -> int:
    """Bytes one decode step must move: the fp32 state read and written, the
    per-channel token inputs and output, B/C, and A/D/bias once."""
    es = 2 if w.dtype == synth.BF16 else 4
    bd = w.batch * w.dim
    return (8 * bd * w.dstate + 4 * es * bd + 2 * es * w.batch * w.dstate
            + 4 * w.dim * w.dstate + 8 * w.dim)


def copy_same_bytes(torch, dev, stream, nbytes, slots, k, graph, barrier, max_over_ranks):
    """A plain device-to-device copy moving the same bytes as one step (nbytes/2
    read, nbytes/2 written), over `slots` buffer pairs cycled like the step's
    inputs and timed the same way (CUDA graph replay or eager launches).  It is
    torch's copy_ of contiguous same-dtype buffers (a device-to-device memcpy),
    not this library's work: the bandwidth a plain copy reaches at this size,
    beside the large-copy peak the roofline divides by."""
    half = (nbytes // 2 + 255) // 256 * 256
    src = [torch.empty(half, dtype=torch.uint8, device=dev).fill_(i + 1) for i in range(slots)]
    dst = [torch.empty(half, dtype=torch.uint8, device=dev) for _ in range(slots)]

    def run():
        for i in range(k):
            dst[i % slots].copy_(src[i % slots])

    for _ in range(3):
        run()
    torch.cuda.synchronize(dev)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if graph:
        g = torch.cuda.CUDAGraph()
        cap = torch.cuda.Stream(dev)
        cap.wait_stream(stream)
        with torch.cuda.stream(cap):
            with torch.cuda.graph(g, stream=cap):
                run()
        torch.cuda.synchronize(dev)
        g.replay()
    torch.cuda.synchronize(dev)
    barrier()
    torch.cuda.synchronize(dev)
    ev0.record(stream)
    if graph:
        g.replay()
    else:
        run()
    ev1.record(stream)
    torch.cuda.synchronize(dev)
    ms = max_over_ranks(ev0.elapsed_time(ev1) / k)
    if graph:
        del g
    del src, dst
    return {"us_per_copy": ms * 1e3, "bytes": 2 * half, "gbs": 2 * half / (ms * 1e-3) / 1e9,
            "timing": "CUDA graph replay" if graph else "eager launches", "slots": slots}


def measure_decode(ssm, torch, dev, args, world, barrier, max_over_ranks, w=None):
    """Single-token steps on the decode workload, replayed from a CUDA graph.

    Four independent (state, token) slots are cycled so that every step reads
    and writes a state that is not in L2 (4 states > 126 MB of L2)."""
    w = w or synth.WORKLOADS["mamba-2.8b-decode"]
    slots = 4
    case = synth.make_workload(w)
    A = torch.from_numpy(np.asarray(case["A"], np.float32)).to(dev)
    D = torch.from_numpy(np.asarray(case["D"], np.float32)).to(dev)
    bias = torch.from_numpy(np.asarray(case["delta_bias"], np.float32)).to(dev)
    tok = {k: to_torch(case[k], dev) for k in ("u", "delta", "z", "B", "C")}
    xs, states, ys = [], [], []
    gen = torch.Generator(device=dev)
    gen.manual_seed(w.seed)
    for i in range(slots):
        x = {k: tok[k][:, :, 0].contiguous() for k in ("u", "delta", "z")}
        x.update({k: tok[k][:, 0, :].contiguous() for k in ("B", "C")})
        if i:  # other tokens: the same values rolled along the channels
            x = {k: torch.roll(v, i, dims=-1).contiguous() for k, v in x.items()}
        xs.append(x)
        states.append(torch.randn((w.batch, w.dim, w.dstate), generator=gen, device=dev,
                                  dtype=torch.float32))
        ys.append(torch.empty_like(x["u"]))

    def step(i):
        x = xs[i % slots]
        ssm.scan_step(x["u"], x["delta"], A, x["B"], x["C"], D, x["z"], bias,
                      state=states[i % slots], y=ys[i % slots])

    stream = torch.cuda.current_stream(dev)
    k = max(args.steps, 8) // slots * slots
    for i in range(max(3, args.warmup) * slots):
        step(i)
    torch.cuda.synchronize(dev)
    # eager: one library call per step from Python
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
    barrier()
    torch.cuda.synchronize(dev)
    ev[0].record(stream)
    for i in range(k):
        step(i)
    ev[1].record(stream)
    torch.cuda.synchronize(dev)
    ms_eager = max_over_ranks(ev[0].elapsed_time(ev[1]) / k)
    # the same k steps captured once in a CUDA graph and replayed
    g = torch.cuda.CUDAGraph()
    cap = torch.cuda.Stream(dev)
    cap.wait_stream(stream)
    with torch.cuda.stream(cap):
        step(0)  # warm the capture stream
        torch.cuda.synchronize(dev)
        with torch.cuda.graph(g, stream=cap):
            for i in range(k):
                step(i)
    torch.cuda.synchronize(dev)
    g.replay()
    torch.cuda.synchronize(dev)
    barrier()
    torch.cuda.synchronize(dev)
    ev[2].record(stream)
    g.replay()
    ev[3].record(stream)
    torch.cuda.synchronize(dev)
    ms = max_over_ranks(ev[2].elapsed_time(ev[3]) / k)
    del g
    nbytes = decode_bytes(w)
    pk = peaks()
    achieved = nbytes / (ms * 1e-3) / 1e9
    cp = copy_same_bytes(torch, dev, stream, nbytes, slots, k, True, barrier, max_over_ranks)
    cp["step_frac_of_copy"] = achieved / cp["gbs"]
    return {"workload": w.name, "batch": w.batch, "d_inner": w.dim, "d_state": w.dstate,
            "io_dtype": w.dtype, "state_dtype": "f32", "steps": k, "state_slots": slots,
            "l2": f"{slots} state slots of {8 * w.batch * w.dim * w.dstate // 2 / 1e6:.0f} MB cycled",
            "us_per_step": ms * 1e3, "us_per_step_eager": ms_eager * 1e3,
            "value": aggregate_value(world, w.batch * w.dim, ms * 1e-3),
            "unit": "tokens·channels/s (single-token steps, CUDA graph replay)",
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": pk["hbm_gbs"],
                         "unit": "GB/s", "frac": achieved / pk["hbm_gbs"],
                         "traffic": profiled_traffic("decode"),
                         "kernel": "k_step_rows", "algorithmic_bytes": nbytes,
                         "peak_basis": f"measured copy bandwidth ({pk['source']})"},
            "copy_same_bytes": cp,
            "gpu_launches": k}


def measure_conv(ssm, torch, dev, args, world, barrier, max_over_ranks, w=None, width=4):
    """Causal depthwise conv1d + SiLU over the layer's x_proj shape (batch, d_inner, L)."""
    w = w or synth.WORKLOADS["mamba-2.8b-layer"]
    x = to_torch(synth.normal((w.batch, w.dim, w.seqlen), w.seed, "u", w.dtype), dev)
    g = np.random.default_rng(w.seed)
    wt = torch.from_numpy((g.standard_normal((w.dim, width)) / 2).astype(np.float32)).to(dev)
    bt = torch.from_numpy(g.standard_normal(w.dim).astype(np.float32)).to(dev)
    out = torch.empty_like(x)
    fs = torch.empty((w.batch, w.dim, width - 1), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        ssm.causal_conv1d(x, wt, bt, out=out, final_state=fs)

    for _ in range(max(3, args.warmup)):
        step()
    k = max(3, min(args.steps, 20))
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize(dev)
    ev0.record(stream)
    for _ in range(k):
        step()
    ev1.record(stream)
    torch.cuda.synchronize(dev)
    ms = max_over_ranks(ev0.elapsed_time(ev1) / k)
    # the backward on the same shape: x and dout read, dx written
    dout = torch.empty_like(x).normal_()

    def step_bwd():
        ssm.causal_conv1d_bwd(x, wt, bt, dout)

    for _ in range(max(3, args.warmup)):
        step_bwd()
    barrier()
    torch.cuda.synchronize(dev)
    ev0.record(stream)
    for _ in range(k):
        step_bwd()
    ev1.record(stream)
    torch.cuda.synchronize(dev)
    ms_b = max_over_ranks(ev0.elapsed_time(ev1) / k)
    es = x.element_size()
    nbytes = 2 * es * w.bld + 4 * w.batch * w.dim * (width - 1) + 4 * w.dim * (width + 1)
    nbytes_b = 3 * es * w.bld + 4 * w.dim * (2 * width + 2)
    pk = peaks()
    achieved = nbytes / (ms * 1e-3) / 1e9
    cp = copy_same_bytes(torch, dev, stream, nbytes, 1, k, False, barrier, max_over_ranks)
    cp["conv_frac_of_copy"] = achieved / cp["gbs"]
    return {"workload": w.name, "batch": w.batch, "seqlen": w.seqlen, "d_inner": w.dim,
            "width": width, "io_dtype": w.dtype, "silu": True, "steps": k,
            "l2": "inputs larger than L2 (no flush)", "ms_per_step": ms,
            "value": aggregate_value(world, w.bld, ms * 1e-3), "unit": UNIT,
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": pk["hbm_gbs"], "unit": "GB/s",
                         "frac": achieved / pk["hbm_gbs"], "traffic": profiled_traffic("conv1d"),
                         "kernel": "k_conv",
                         "algorithmic_bytes": nbytes,
                         "peak_basis": f"measured copy bandwidth ({pk['source']})"},
            "bwd": {"ms_per_step": ms_b, "algorithmic_bytes": nbytes_b,
                    "achieved_gbs": nbytes_b / (ms_b * 1e-3) / 1e9,
                    "frac": nbytes_b / (ms_b * 1e-3) / 1e9 / pk["hbm_gbs"], "kernel": "k_conv_bwd"},
            "copy_same_bytes": cp,
            "gpu_launches": k}


def main():
    args = parse()
    w = synth.WORKLOADS[args.workload]
    if args.batch:
        import dataclasses
        w = dataclasses.replace(w, batch=args.batch, name=f"{w.name}[batch={args.batch}]")
    if args.seqlen:
        import dataclasses
        w = dataclasses.replace(w, seqlen=args.seqlen, name=f"{w.name}[seqlen={args.seqlen}]")
    args.reduced = bool(args.batch or args.seqlen)  # a profiling case: no sub-records
    if args.impl == "reference":
        return run_reference(args, w)

    import torch
    import selective_state_space_54_b200 as ssm
    from selective_state_space_54_b200 import _lib

    world, rank, local = init_dist(args)
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)

    def barrier0():
        if world > 1:
            import torch.distributed as dist
            dist.barrier()

    if w.extra.get("decode"):
        dec = measure_decode(ssm, torch, dev, args, world, barrier0,
                             lambda x: dist_max(x, world, dev), w)
        line = {"metric": METRIC, "value": dec["value"], "unit": UNIT, "n_gpus": world,
                "steps": dec["steps"], "warmup": max(3, args.warmup),
                "ms_per_step": dec["us_per_step"] * 1e-3, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
                "config": {"workload": w.name, "batch": w.batch, "d_inner": w.dim,
                           "d_state": w.dstate, "io_dtype": w.dtype, "step": "decode",
                           "l2": dec["l2"], "seed": w.seed},
                "roofline": dec["roofline"], "decode": dec, "gpu_launches": dec["gpu_launches"]}
        if rank == 0:
            print(json.dumps(line), flush=True)
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
        return
    if w.backward:
        # the training step itself: forward + recomputation backward
        def max0(x):
            return dist_max(x, world, dev)
        tr = measure_training(ssm, torch, dev, args, world, barrier0, max0, w)
        line = {"metric": METRIC, "value": tr["value"], "unit": UNIT, "n_gpus": world,
                "steps": tr["steps"], "warmup": max(3, args.warmup),
                "ms_per_step": tr["fwd_ms"] + tr["bwd_ms"], "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
                "config": dict(config_of(w, tr["fwd_path"]), step="fwd+bwd"), "bwd": tr,
                "roofline": tr["bwd_roofline"], "gpu_launches": 4 * tr["steps"]}
        if rank == 0:
            print(json.dumps(line), flush=True)
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
        return

    case = synth.make_workload(w)
    g = {k: to_torch(case[k], dev) for k in ("u", "delta", "z", "B", "C")}
    for k in ("A", "D", "delta_bias"):
        g[k] = torch.from_numpy(np.asarray(case[k], np.float32)).to(dev)
    y = torch.empty_like(g["u"])
    ls = torch.empty((w.batch, w.dim, w.dstate), dtype=torch.float32, device=dev)
    path_id = {"auto": 0, "lookback": 1, "split_l": 2, "per_group": 3, "lookback_ws": 4}[args.path]
    shape = ssm.make_shape(w.batch, w.dim, w.seqlen, w.dstate,
                           ssm.SSM_BF16 if w.dtype == synth.BF16 else ssm.SSM_F32,
                           path_id, args.lanes)
    path = ssm.fwd_path(shape)
    ws = torch.empty(ssm.fwd_workspace_bytes(shape), dtype=torch.uint8, device=dev)
    # our kernels per forward: the warp-specialised schedule widens B and C first
    launches_per_step = {"lookback": 1, "per_group": 1, "split_l": 3, "lookback_ws": 2}[path]
    stream = torch.cuda.current_stream(dev)

    def step():
        ssm.scan_fwd(g["u"], g["delta"], g["A"], g["B"], g["C"], g["D"], g["z"], g["delta_bias"],
                     y=y, last_state=ls, return_last_state=True, workspace=ws, path=path_id,
                     lanes=args.lanes)

    def barrier():
        if world > 1:
            import torch.distributed as dist
            dist.barrier()

    def max_over_ranks(x: float) -> float:
        return dist_max(x, world, dev)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize(dev)
    ssm.check(ws)

    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(dev.index if world == 1 else local) as clk:
        barrier()
        torch.cuda.synchronize(dev)
        ev0.record(stream)
        for _ in range(args.steps):
            step()
        ev1.record(stream)
        torch.cuda.synchronize(dev)
        barrier()
    ssm.check(ws)
    ms = max_over_ranks(ev0.elapsed_time(ev1) / args.steps)
    clocks = clk.summary()
    # the timed run's outputs, for the parity check beside the CPU baseline
    y_keep = ls_keep = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        y_keep, ls_keep = y.cpu(), ls.cpu()

    # the same forward on token-major activations (batch, seqlen, d_inner)
    tok = None
    if not args.no_bwd and not args.reduced and w.dtype == synth.BF16 and w.dim % 8 == 0:
        tm = {k: g[k].transpose(1, 2).contiguous() for k in ("u", "delta", "z")}
        y_tm = torch.empty_like(tm["u"])

        def step_tm():
            ssm.scan_fwd(tm["u"], tm["delta"], g["A"], g["B"], g["C"], g["D"], tm["z"],
                         g["delta_bias"], y=y_tm, last_state=ls, return_last_state=True,
                         workspace=ws, token_major=True)

        for _ in range(max(3, args.warmup)):
            step_tm()
        torch.cuda.synchronize(dev)
        barrier()
        torch.cuda.synchronize(dev)
        ev0.record(stream)
        for _ in range(args.steps):
            step_tm()
        ev1.record(stream)
        torch.cuda.synchronize(dev)
        ms_tm = max_over_ranks(ev0.elapsed_time(ev1) / args.steps)
        tok = {"layout": "[batch][seqlen][d_inner] u, delta, z, y", "ms_per_step": ms_tm,
               "value": aggregate_value(world, w.bld, ms_tm * 1e-3), "unit": UNIT}
        del tm, y_tm

    # the same forward with the exact zero-order-hold input term, Delta u (e^x - 1)/x B
    zoh = None
    if not args.no_bwd and not args.reduced:
        def step_zoh():
            ssm.scan_fwd(g["u"], g["delta"], g["A"], g["B"], g["C"], g["D"], g["z"],
                         g["delta_bias"], y=y, last_state=ls, return_last_state=True,
                         workspace=ws, zoh_exact=True)

        for _ in range(max(3, args.warmup)):
            step_zoh()
        torch.cuda.synchronize(dev)
        barrier()
        torch.cuda.synchronize(dev)
        ev0.record(stream)
        for _ in range(args.steps):
            step_zoh()
        ev1.record(stream)
        torch.cuda.synchronize(dev)
        ssm.check(ws)
        ms_z = max_over_ranks(ev0.elapsed_time(ev1) / args.steps)
        zshape = ssm.make_shape(w.batch, w.dim, w.seqlen, w.dstate,
                                ssm.SSM_BF16 if w.dtype == synth.BF16 else ssm.SSM_F32,
                                flags=ssm.SSM_FLAG_ZOH_EXACT)
        zoh = {"path": ssm.fwd_path(zshape), "ms_per_step": ms_z,
               "value": aggregate_value(world, w.bld, ms_z * 1e-3), "unit": UNIT}

    # end to end through the public API: pinned host inputs in, result out, every
    # step.  Steps are pipelined two deep on three streams, as a serving loop
    # would run them: step k+1's inputs cross PCIe host-to-device while step k
    # scans and step k-1's y and last_state cross device-to-host (the two
    # copy directions use separate engines).  Every step copies all of its
    # inputs in and its results out; the timed region spans all of it.
    e2e = None
    if not args.no_e2e:
        host = {k: g[k].cpu().pin_memory() for k in ("u", "delta", "z", "B", "C", "A", "D", "delta_bias")}
        y_host = torch.empty(y.shape, dtype=y.dtype).pin_memory()
        ls_host = torch.empty(ls.shape, dtype=ls.dtype).pin_memory()
        dbuf = [{k: torch.empty_like(g[k]) for k in host} for _ in range(2)]
        ybuf = [y, torch.empty_like(y)]
        lsbuf = [ls, torch.empty_like(ls)]
        h2d = sum(t.numel() * t.element_size() for t in host.values())
        d2h = y_host.numel() * y_host.element_size() + ls_host.numel() * ls_host.element_size()
        s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        ev_in = [torch.cuda.Event() for _ in range(2)]
        ev_done = [torch.cuda.Event() for _ in range(2)]
        ev_out = [torch.cuda.Event() for _ in range(2)]

        def e2e_step(i):
            b = i % 2
            s_in.wait_event(ev_done[b])         # the scan of step i-2 has read dbuf[b]
            with torch.cuda.stream(s_in):
                for k in host:
                    dbuf[b][k].copy_(host[k], non_blocking=True)
            ev_in[b].record(s_in)
            stream.wait_event(ev_in[b])
            stream.wait_event(ev_out[b])        # step i-2's results have left ybuf[b]
            d = dbuf[b]
            ssm.scan_fwd(d["u"], d["delta"], d["A"], d["B"], d["C"], d["D"], d["z"], d["delta_bias"],
                         y=ybuf[b], last_state=lsbuf[b], return_last_state=True, workspace=ws,
                         path=path_id, lanes=args.lanes, stream=stream)
            ev_done[b].record(stream)
            s_out.wait_event(ev_done[b])
            with torch.cuda.stream(s_out):
                y_host.copy_(ybuf[b], non_blocking=True)
                ls_host.copy_(lsbuf[b], non_blocking=True)
            ev_out[b].record(s_out)

        for i in range(2):
            e2e_step(i)
        torch.cuda.synchronize(dev)
        k_e2e = max(3, args.steps)  # the run's K steps, as the device-timed leg
        barrier()
        torch.cuda.synchronize(dev)
        ev0.record(stream)
        s_in.wait_event(ev0)
        s_out.wait_event(ev0)
        for i in range(k_e2e):
            e2e_step(i)
        stream.wait_event(ev_out[(k_e2e - 1) % 2])
        ev1.record(stream)
        torch.cuda.synchronize(dev)
        barrier()
        ssm.check(ws)
        ms_e2e = max_over_ranks(ev0.elapsed_time(ev1) / k_e2e)
        e2e = {"value": aggregate_value(world, w.bld, ms_e2e * 1e-3), "unit": UNIT,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": ms_e2e,
               "pipeline": "2 steps in flight: host-to-device copies of step k+1 and "
                           "device-to-host copies of step k-1 overlap the scan of step k "
                           "(three streams)"}
        del host, dbuf

    bwd = dec = conv = m130 = mlen = None
    if not args.no_bwd and not args.reduced:
        m130 = measure_forward(ssm, torch, dev, args, world, barrier, max_over_ranks,
                               "mamba-130m-layer")
        mlen = measure_forward(ssm, torch, dev, args, world, barrier, max_over_ranks,
                               "million-length")
        bwd = measure_training(ssm, torch, dev, args, world, barrier, max_over_ranks)
        dec = measure_decode(ssm, torch, dev, args, world, barrier, max_over_ranks)
        conv = measure_conv(ssm, torch, dev, args, world, barrier, max_over_ranks)

    pk = peaks()
    sm_count = torch.cuda.get_device_properties(dev).multi_processor_count
    sec = ms * 1e-3
    ex2_peak = sm_count * MUFU_EX2_PER_CLK_PER_SM * pk["sm_max_mhz"] * 1e6
    achieved = w.bldn / sec
    roofline = {"bound": "alu", "achieved": achieved / 1e12, "peak": ex2_peak / 1e12,
                "unit": "Tex2/s", "frac": achieved / ex2_peak,
                "traffic": profiled_traffic(path),
                "kernel": {"lookback": "k_fwd_lookback", "lookback_ws": "k_fwd_ws"}.get(
                    path, f"k_fwd_segment ({path})"),
                "peak_basis": f"{sm_count} SMs x {MUFU_EX2_PER_CLK_PER_SM} ex2/clk x "
                              f"{pk['sm_max_mhz']:.0f} MHz (sm_max_mhz, {pk['source']})",
                "algorithmic_bytes": alg_bytes(w),
                "hbm_achieved_gbs": alg_bytes(w) / sec / 1e9, "hbm_peak_gbs": pk["hbm_gbs"],
                "hbm_frac": alg_bytes(w) / sec / 1e9 / pk["hbm_gbs"],
                # against the nominal HBM3e bandwidth too (8 TB/s), for context
                "hbm_frac_of_nominal_8tbs": alg_bytes(w) / sec / 1e9 / 8000.0}
    if clocks and clocks.get("sm_mhz"):
        at_clock = sm_count * MUFU_EX2_PER_CLK_PER_SM * clocks["sm_mhz"] * 1e6
        roofline["frac_at_measured_clock"] = achieved / at_clock

    line = {"metric": METRIC, "value": aggregate_value(world, w.bld, sec), "unit": UNIT,
            "n_gpus": world,
            "steps": args.steps, "warmup": max(3, args.warmup), "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic", "config": dict(config_of(w, path), parallelism=f"replicas x{world}"),
            "roofline": roofline, "clocks": clocks, "e2e": e2e, "bwd": bwd, "decode": dec, "conv1d": conv, "token_major": tok,
            "zoh_exact": zoh,
            "mamba_130m_layer": m130, "million_length": mlen,
            "gpu_launches": launches_per_step * args.steps}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"], line["parity"] = cpu_baseline(w, case, y_gpu=y_keep, ls_gpu=ls_keep)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    _ = _lib


if __name__ == "__main__":
    main()
