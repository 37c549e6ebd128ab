#!/usr/bin/env python
"""Benchmark of the selective-scan forward (S6) on B200.

Default workload: the Mamba-2.8B-like layer scan -- batch 4, d_inner 5120,
d_state 16, L 4096, bf16 u/delta/z/B/C, fp32 A/D/state, softplus on delta,
D skip and silu(z) gate.  A "step" is one selscan_fwd call over that batch
(the whole hot path: softplus, discretisation, scan, output contraction,
gate, final state).  Throughput is elements (batch * d_inner * L) per second.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config 2]
    python bench.py --impl reference ...   # the fp64 CPU oracle, timed

For N > 1 (launched with torch.distributed.run) each rank scans its own
independent shard of the same shape (the path has no exchange step), so the
scaling is weak; the step time is the max over ranks.
"""
from __future__ import annotations

import argparse
import contextlib
import gc
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synthetic  # noqa: E402

BASE_CONFIGS = {k: dict(v) for k, v in synthetic.CONFIGS.items()}

METRIC = "selective-scan Gelem/s (B·D·L) and % of B200 HBM roofline, 1 GPU"

# DRAM bytes per launch (dram__bytes_read.sum + dram__bytes_write.sum) from the
# ncu captures summarised in profiles/, keyed by config and the kernel they
# were taken on; reported as roofline.traffic only for that kernel.
NCU_TRAFFIC = {
    # config 2 captured at L = 2048, scaled by tokens to L = 4096
    2: ("scan_diag_bf16_kernel lane-per-channel v6", 640.3e6),
    # config 3 (two-pass form, both kernels of one call) captured at
    # L = 32768, scaled by tokens to L = 131072
    3: ("scan_diag_bf16_kernel lane-per-channel two-pass v7", 2484.5e6),
    4: ("ssd_scalarA_kernel v6", 108.1e6),
}
KERNEL_TAG = {2: "scan_diag_bf16_kernel lane-per-channel v6",
              1: "scan_diag_bf16_kernel lane-per-channel v6",
              3: "scan_diag_bf16_kernel lane-per-channel two-pass v7",
              0: "scan_diag_kernel fp32 v3", 4: "ssd_scalarA_kernel v6"}
HBM_FALLBACK_GBS = 6650.0
NOMINAL_HBM_GBS = 8000.0  # the HGX/DGX nominal figure, reported beside the measured peak


def measured_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return json.load(f), "measured"
    except Exception:
        return {"hbm_gbs": HBM_FALLBACK_GBS, "bf16_tflops": 1590.0}, "fallback"


# ------------------------------------------------------------ byte counts
def algorithmic_bytes(cfg: dict) -> int:
    """Bytes one call must move at minimum: every input read once, every
    output written once (the expanded state is never stored)."""
    es = 2 if cfg["dtype"] == "bf16" else 4
    b, L = cfg["batch"], cfg["L"]
    if cfg["kind"] == "diag":
        dim, N = cfg["dim"], cfg["N"]
        stream = (3 if cfg["gate"] else 2) * es + es           # u, delta, (z) + y
        total = b * dim * L * stream
        total += 2 * b * N * L * es                             # B, C
        total += dim * N * 4 + dim * 4 * (2 if cfg["D"] else 1)  # A, bias, D
        total += b * dim * N * 4                                 # last_state
        return total
    H, P, N, G = cfg["nheads"], cfg["headdim"], cfg["N"], cfg["ngroups"]
    dim = H * P
    total = b * dim * L * es * (3 if cfg["gate"] else 2)        # x, (z), y
    total += b * H * L * 4                                       # dt
    total += 2 * b * G * N * L * es                              # B, C
    total += H * 4 * 3                                           # A, D, bias
    total += b * H * P * N * 4                                   # last_state
    return total


def ssd_flops(cfg: dict, Q: int = 128) -> float:
    """Tensor-core FLOPs of the chunked SSD form per call at chunk length Q
    (the kernel's Q = 128): C.B^T once per batch and chunk since heads share
    B/C; per head the intra-chunk product, the chunk state and the
    carried-in term."""
    b, L = cfg["batch"], cfg["L"]
    H, P, N = cfg["nheads"], cfg["headdim"], cfg["N"]
    nch = (L + Q - 1) // Q
    per_chunk = 2 * Q * Q * N + H * (2 * Q * Q * P + 2 * N * Q * P + 2 * Q * N * P)
    return float(b * nch * per_chunk)


def ssd_bwd_flops(cfg: dict, Q: int = 32) -> float:
    """Tensor-core FLOPs of the chunked scalar-A backward per call at chunk
    length Q (the kernels' Q = 32), counting each product once (the extra
    products of split operands are not counted): C.B^T once per batch, group
    and chunk; per head and chunk dout.x^T, the two products of y~ and of u,
    the two of dC and of dB, the dh recurrence and the forward state
    recurrence."""
    b, L = cfg["batch"], cfg["L"]
    H, P, N, G = cfg["nheads"], cfg["headdim"], cfg["N"], cfg["ngroups"]
    nch = (L + Q - 1) // Q
    per_head = 6 * Q * Q * P + 4 * Q * Q * N + 12 * Q * P * N
    return float(b * nch * (G * 2 * Q * Q * N + H * per_head))


# nominal dense tensor throughput of tf32 relative to bf16 on B200 (1.1 / 2.25 PFLOP/s)
TF32_PER_BF16 = 1.1 / 2.25


# ------------------------------------------------------------ ranks
@contextlib.contextmanager
def gc_paused(collect: bool = True):
    """Keep Python's garbage collector off for a timed region (after a full
    collection unless the caller just made one).  With torch loaded a full
    collection pauses the host for tens to hundreds of milliseconds; inside
    a timed loop of asynchronous calls that pause drains the GPU's queue
    and is counted as device time."""
    if collect:
        gc.collect()
    was_on = gc.isenabled()
    gc.disable()
    try:
        yield
    finally:
        if was_on:
            gc.enable()


def max_over_ranks(values, device="cuda"):
    """Element-wise max of a list of floats over all ranks of the default
    process group (identity without one).  Every rank must call it with the
    same number of values, in the same order."""
    import torch
    import torch.distributed as tdist
    if not (tdist.is_available() and tdist.is_initialized()) or tdist.get_world_size() == 1:
        return [float(v) for v in values]
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    tdist.all_reduce(t, op=tdist.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


def aggregate_rate(world: int, units_per_rank: float, ms_per_step: float) -> float:
    """Whole-job throughput: every rank processes its own shard of the same
    size each step, and the step takes the slowest rank's time."""
    return world * units_per_rank / (ms_per_step * 1e-3)


def shard_seed(cfg: dict, rank: int) -> int:
    """Seed of a rank's independent shard (rank 0 keeps the config's seed)."""
    return int(cfg["seed"]) + 7919 * rank


# ------------------------------------------------------------ clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None
        self.lines = []
        self.t = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-i", str(self.dev), "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        self.t = threading.Thread(target=self._pump, daemon=True)
        self.t.start()
        time.sleep(0.3)  # let nvidia-smi start reporting

    def _pump(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    def stop(self, t0: float, t1: float) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.1)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = [l for (ts, l) in self.lines if t0 <= ts <= t1] or [l for (_, l) in self.lines]
        sm, smax, power, reasons = [], [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            parts = [p.strip() for p in r.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
                power.append(float(parts[3]))
            except ValueError:
                continue
            for nm, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "power_w_max": max(power) if power else None,
                "samples": len(sm), "reasons": sorted(reasons)}


def physical_gpu_index(local: int) -> int:
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    if vis:
        ids = [v.strip() for v in vis.split(",") if v.strip()]
        if local < len(ids) and ids[local].isdigit():
            return int(ids[local])
    return local


# ------------------------------------------------------------ CPU oracle
def oracle_sample(cfg_idx: int, inp: dict, seconds: float = 10.0):
    """Time the fp64 oracle on a bounded sample of the workload: whole
    channels (all tokens, all batches) of the first d_inner rows, grown
    until about `seconds` of single-threaded CPU work."""
    import oracle
    cfg = synthetic.CONFIGS[cfg_idx]
    L, b = cfg["L"], cfg["batch"]
    n = 1
    spent = 0.0
    done_elems = 0
    while True:
        t0 = time.perf_counter()
        if cfg["kind"] == "diag":
            oracle.selscan(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], D=inp["D"],
                           z=inp["z"], delta_bias=inp["delta_bias"],
                           delta_softplus=inp["softplus"], channels=(0, n))
            elems = b * n * L
            unit = f"{n} channel(s)"
        else:
            P = cfg["headdim"]
            h = max(1, n // P)
            oracle.selscan_scalarA(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], P,
                                   D=inp["D"], z=inp["z"], heads=(0, h))
            elems = b * h * P * L
            unit = f"{h} head(s)"
        dt = time.perf_counter() - t0
        spent, done_elems = dt, elems
        if dt >= seconds * 0.5 or n >= (cfg.get("dim") or cfg["nheads"] * cfg["headdim"]):
            break
        grow = max(2.0, min(16.0, seconds / max(dt, 1e-3)))
        n = int(min(n * grow, cfg.get("dim") or cfg["nheads"] * cfg["headdim"]))
    out = {"value": done_elems / spent / 1e9, "unit": "Gelem/s", "cores": 1,
           "kind": "oracle",
           "sample": f"{unit} x batch {b} x L {L} = {done_elems} elements, "
                     f"{spent:.1f} s single-threaded fp64",
           "host": host_cpu()}
    out["all_cores"] = oracle_all_cores(cfg, inp, n, seconds)
    return out


def host_cpu() -> dict:
    """Host cores and CPU model of the machine the baseline ran on."""
    model = None
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return {"nproc": os.cpu_count(), "cpu_model": model}


def oracle_all_cores(cfg: dict, inp: dict, n: int, seconds: float) -> dict:
    """The same unchanged single-threaded oracle, run over channel (or
    head) ranges on every host core at once: one call per core, side by
    side (the oracle's C loop runs without the interpreter lock).  The sample
    is `n` channels per core, capped at the workload's d_inner."""
    import oracle
    from concurrent.futures import ThreadPoolExecutor
    cores = os.cpu_count() or 1
    L, b = cfg["L"], cfg["batch"]
    if cfg["kind"] == "diag":
        total = min(cfg["dim"], n * cores)
        edges = np.linspace(0, total, min(cores, total) + 1).astype(int)

        def one(r):
            oracle.selscan(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], D=inp["D"],
                           z=inp["z"], delta_bias=inp["delta_bias"],
                           delta_softplus=inp["softplus"], channels=r)
        per = 1
        what = "channels"
    else:
        P = cfg["headdim"]
        total = min(cfg["nheads"], max(1, n // P) * cores)
        edges = np.linspace(0, total, min(cores, total) + 1).astype(int)

        def one(r):
            oracle.selscan_scalarA(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], P,
                                   D=inp["D"], z=inp["z"], heads=r)
        per = P
        what = "heads"
    ranges = [(int(a), int(c)) for a, c in zip(edges[:-1], edges[1:]) if c > a]
    t0 = time.perf_counter()
    with ThreadPoolExecutor(len(ranges)) as ex:
        list(ex.map(one, ranges))
    dt = time.perf_counter() - t0
    elems = b * total * per * L
    return {"value": elems / dt / 1e9, "unit": "Gelem/s", "cores": len(ranges),
            "sample": f"{total} {what} x batch {b} x L {L} = {elems} elements over "
                      f"{len(ranges)} threads, {dt:.1f} s"}


def scan_config(cfg: dict, world: int) -> dict:
    """The ``config`` object of a forward-scan line (both arms)."""
    return {"workload": cfg["name"], "batch": cfg["batch"],
            "d_inner": cfg.get("dim") or cfg["nheads"] * cfg["headdim"],
            "d_state": cfg["N"], "seq_len": cfg["L"], "seed": cfg["seed"],
            "global_batch": cfg["batch"] * world,
            "l2": "inputs larger than L2 (no flush)" if algorithmic_bytes(cfg) > 126e6 else
                  "inputs smaller than L2",
            "parallelism": f"dp{world} (independent shards, no collective)"}


def step_config(cfg: dict, world: int) -> dict:
    """The ``config`` object of a decode-step line (both arms); ``cfg`` is
    the step workload (``step_workload``)."""
    dim = cfg.get("dim") or cfg["nheads"] * cfg["headdim"]
    return {"workload": step_name(cfg), "batch": cfg["batch"], "d_inner": dim,
            "d_state": cfg["N"], "global_batch": cfg["batch"] * world,
            "l2": "state larger than L2 (no flush)" if step_bytes(cfg) > 126e6 else
                  "state smaller than L2",
            "parallelism": f"dp{world} (independent shards, no collective)"}


def cfg_dim(cfg: dict) -> int:
    """d_inner of a config (channels; heads x headdim for scalar A)."""
    return cfg["dim"] if cfg["kind"] == "diag" else cfg["nheads"] * cfg["headdim"]


def bwd_config(cfg: dict, world: int) -> dict:
    """The ``config`` object of a backward line (both arms)."""
    return {"workload": "backward of " + cfg["name"], "batch": cfg["batch"],
            "d_inner": cfg_dim(cfg), "d_state": cfg["N"], "seq_len": cfg["L"],
            "global_batch": cfg["batch"] * world,
            "l2": "inputs larger than L2 (no flush)" if bwd_bytes(cfg) > 126e6 else
                  "inputs smaller than L2",
            "parallelism": f"dp{world} (independent shards, no collective)"}


def run_reference(args, rank: int, world: int):
    """Reference arm: the fp64 oracle on the host cores (rank 0 only)."""
    if rank != 0:
        return
    if args.op == "step":
        run_reference_step(args, world)
        return
    if args.op == "bwd":
        run_reference_bwd(args, world)
        return
    cfg = synthetic.CONFIGS[args.config]
    inp = synthetic.make_config(args.config)
    import oracle
    # one step = one whole channel (all batches, all tokens) of the workload;
    # grow to several channels if that is too fast to time
    per_step_channels = 1
    L, b = cfg["L"], cfg["batch"]

    def step(i):
        if cfg["kind"] == "diag":
            c0 = (i * per_step_channels) % cfg["dim"]
            oracle.selscan(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], D=inp["D"],
                           z=inp["z"], delta_bias=inp["delta_bias"],
                           delta_softplus=inp["softplus"], channels=(c0, c0 + per_step_channels))
            return b * per_step_channels * L
        P = cfg["headdim"]
        h = i % cfg["nheads"]
        oracle.selscan_scalarA(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], P,
                               D=inp["D"], z=inp["z"], heads=(h, h + 1))
        return b * P * L

    budget = 150.0  # keep the whole reference run within a few minutes
    for i in range(args.warmup):
        step(i)
    t0 = time.perf_counter()
    elems = 0
    steps_done = 0
    for i in range(args.steps):
        elems += step(i)
        steps_done += 1
        if time.perf_counter() - t0 > budget:
            break
    dt = time.perf_counter() - t0
    val = elems / dt / 1e9
    line = {
        "impl": "reference", "metric": METRIC, "value": val, "unit": "Gelem/s",
        "n_gpus": world, "steps": steps_done, "warmup": args.warmup,
        "ms_per_step": dt / steps_done * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": dict(scan_config(cfg, world),
                       sample_per_step="one channel (all batches, all tokens)"
                       if cfg["kind"] == "diag" else "one head"),
        "cpu_baseline": {"value": val, "unit": "Gelem/s", "cores": 1, "kind": "oracle",
                         "sample": f"{steps_done} steps x {elems // max(steps_done, 1)} elements"},
        "e2e": {"value": val, "unit": "Gelem/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def run_reference_step(args, world: int):
    """Reference arm of ``--op step``: the oracle's decode step, each timed
    step a bounded sample of batch rows of the same workload."""
    base = synthetic.CONFIGS[args.config]
    batch = args.batch or STEP_BATCH[base["kind"]]
    cfg = step_workload(base, batch)
    rows = min(batch, 8)  # rows per timed step
    if cfg["kind"] == "diag":
        inp = synthetic.make_diag(rows, cfg["dim"], cfg["N"], 1, dtype=cfg["dtype"],
                                  seed=cfg["seed"], gate=cfg["gate"], D=cfg["D"])
        shape = (rows, cfg["dim"], cfg["N"])
    else:
        inp = synthetic.make_scalarA(rows, cfg["nheads"], cfg["headdim"], cfg["N"], 1,
                                     ngroups=cfg["ngroups"], dtype=cfg["dtype"],
                                     seed=cfg["seed"], gate=cfg["gate"])
        shape = (rows, cfg["nheads"], cfg["headdim"], cfg["N"])
    state = np.random.default_rng(cfg["seed"] + 1000).standard_normal(shape, dtype=np.float32)
    one = lambda: oracle_step_sample(dict(cfg, batch=rows), inp, state, seconds=0.0)
    for _ in range(args.warmup):
        one()
    t0 = time.perf_counter()
    done = 0
    for _ in range(args.steps):
        one()
        done += 1
        if time.perf_counter() - t0 > 150.0:
            break
    dt = time.perf_counter() - t0
    val = done * rows / dt
    print(json.dumps({
        "impl": "reference",
        "metric": "selective-scan decode step, tokens/s (one token per batch row) and % of "
                  "B200 HBM roofline, 1 GPU",
        "value": val, "unit": "tokens/s", "n_gpus": world, "steps": done,
        "warmup": args.warmup, "ms_per_step": dt / done * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": dict(step_config(cfg, world), sample_per_step=f"{rows} batch rows"),
        "cpu_baseline": {"value": val, "unit": "tokens/s", "cores": 1, "kind": "oracle",
                         "sample": f"{done} steps x {rows} batch rows"},
        "e2e": {"value": val, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }), flush=True)


def run_reference_bwd(args, world: int):
    """Reference arm of ``--op bwd``: the oracle's backward, each timed step
    one whole channel (all batches, all tokens) of the workload."""
    cfg = synthetic.CONFIGS[args.config]
    inp = synthetic.make_config(args.config)
    scalar = cfg["kind"] == "scalarA"
    dy = np.random.default_rng(cfg["seed"] + 500).standard_normal(
        inp["x" if scalar else "u"].shape, dtype=np.float32)
    import oracle

    def one(i):
        if scalar:
            # one head (its P channels, all batches, all tokens) per step
            P, hh = cfg["headdim"], i % cfg["nheads"]
            g = hh // (cfg["nheads"] // cfg["ngroups"])
            ch = lambda x: None if x is None else x[:, hh * P:(hh + 1) * P]
            hv = lambda x: None if x is None else x[hh:hh + 1]
            oracle.selscan_scalarA_bwd(ch(inp["x"]), inp["dt"][:, hh:hh + 1], hv(inp["A"]),
                                       inp["B"][:, g:g + 1], inp["C"][:, g:g + 1], P,
                                       ch(dy), D=hv(inp["D"]), z=ch(inp["z"]))
            return
        c = i % cfg["dim"]
        sl = lambda x: None if x is None else x[:, c:c + 1]
        vec = lambda x: None if x is None else x[c:c + 1]
        oracle.selscan_bwd(sl(inp["u"]), sl(inp["delta"]), inp["A"][c:c + 1], inp["B"],
                           inp["C"], dy[:, c:c + 1], D=vec(inp["D"]), z=sl(inp["z"]),
                           delta_bias=vec(inp["delta_bias"]))

    for i in range(args.warmup):
        one(i)
    t0 = time.perf_counter()
    done = 0
    for i in range(args.steps):
        one(i)
        done += 1
        if time.perf_counter() - t0 > 150.0:
            break
    dt = time.perf_counter() - t0
    per_step = cfg["headdim"] if scalar else 1  # channels per step
    val = done * per_step * cfg["batch"] * cfg["L"] / dt / 1e9
    print(json.dumps({
        "impl": "reference",
        "metric": "selective-scan backward Gelem/s (B·D·L) and % of B200 HBM roofline, 1 GPU",
        "value": val, "unit": "Gelem/s", "n_gpus": world, "steps": done,
        "warmup": args.warmup, "ms_per_step": dt / done * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": dict(bwd_config(cfg, world),
                       sample_per_step=("one head" if scalar else "one channel") +
                       " (all batches, all tokens)"),
        "cpu_baseline": {"value": val, "unit": "Gelem/s", "cores": 1, "kind": "oracle",
                         "sample": f"{done} steps x one " + ("head" if scalar else "channel")},
        "e2e": {"value": val, "unit": "Gelem/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }), flush=True)


# ------------------------------------------------------------ GPU arm
def to_dev(a, dtype, torch):
    if a is None:
        return None
    t = torch.from_numpy(np.ascontiguousarray(a))
    return (t.to(torch.bfloat16) if dtype == "bf16" else t.float()).cuda()


def pipelined_e2e(torch, stream, steps, pinned, dev_sets, compute, host_outs):
    """End-to-end steps through the public API, pipelined as a loader drives
    the call: every step copies its inputs from pinned host memory (``pinned``,
    name -> tensor) into one of two device buffer sets (``dev_sets``), runs
    ``compute(j)`` on set j on ``stream`` (it returns the device tensors of
    the step's results) and copies those results into pinned host memory
    (``host_outs[j]``, in the same order).  The copies in, the compute and the
    copies out run on three streams, so step i + 1's inputs go in while step
    i computes and step i - 1's results come out (PCIe carries both
    directions at once); events keep a buffer set from being refilled before
    the step that used it has computed and copied its results out.  Returns
    the milliseconds per step, from the first copy in to the last copy out,
    after two untimed steps."""
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    ev_in, ev_comp, ev_out = ([torch.cuda.Event() for _ in range(2)] for _ in range(3))

    def run(n):
        for i in range(n):
            j = i & 1
            with torch.cuda.stream(s_in):
                s_in.wait_event(ev_comp[j])  # the step that last read set j has computed
                for k, t in pinned.items():
                    dev_sets[j][k].copy_(t, non_blocking=True)
                ev_in[j].record(s_in)
            stream.wait_event(ev_in[j])
            stream.wait_event(ev_out[j])     # set j's previous results are out
            res = compute(j)
            ev_comp[j].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_comp[j])
                for src, dst in zip(res, host_outs[j]):
                    dst.copy_(src, non_blocking=True)
                    src.record_stream(s_out)  # keep pooled memory until the copy is done
                ev_out[j].record(s_out)

    run(2)
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    with gc_paused():
        e0.record(s_in)
        run(steps)
        stream.wait_event(ev_out[(steps - 1) & 1])
        e1.record(stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / steps


def second_set(torch, dev, keys):
    """A second device buffer set for the keys copied in every step."""
    return {k: (torch.empty_like(v) if (k in keys and v is not None) else v)
            for k, v in dev.items()}


def run_gpu(args, rank: int, world: int, local: int):
    import torch
    import selective_state_space_selscan_b200 as ss
    torch.cuda.set_device(local)
    cfg = synthetic.CONFIGS[args.config]
    inp = synthetic.make_config(args.config, seed=shard_seed(cfg, rank))
    dt = cfg["dtype"]
    stream = torch.cuda.current_stream()
    if cfg["kind"] == "diag":
        dev = {k: to_dev(inp[k], dt, torch) for k in ("u", "delta", "B", "C", "z")}
        dev.update({k: to_dev(inp[k], "f32", torch) for k in ("A", "D", "delta_bias")})
        y = torch.empty_like(dev["u"])
        hs = torch.empty((cfg["batch"], cfg["dim"], cfg["N"]), dtype=torch.float32,
                         device="cuda")

        def call_on(d, yy, hh):
            ss.selscan_fwd(d["u"], d["delta"], d["A"], d["B"], d["C"], D=d["D"],
                           z=d["z"], delta_bias=d["delta_bias"], delta_softplus=True,
                           out=yy, last_state=hh)
        host_in = ("u", "delta", "B", "C", "z", "A", "D", "delta_bias")
    else:
        dev = {k: to_dev(inp[k], dt, torch) for k in ("x", "B", "C", "z")}
        dev.update({k: to_dev(inp[k], "f32", torch) for k in ("dt", "A", "D")})
        y = torch.empty_like(dev["x"])
        hs = torch.empty((cfg["batch"], cfg["nheads"], cfg["headdim"], cfg["N"]),
                         dtype=torch.float32, device="cuda")

        def call_on(d, yy, hh):
            ss.selscan_fwd_scalarA(d["x"], d["dt"], d["A"], d["B"], d["C"],
                                   cfg["headdim"], D=d["D"], z=d["z"], out=yy,
                                   last_state=hh)
        host_in = ("x", "dt", "B", "C", "z", "A", "D")

    def call():
        call_on(dev, y, hs)

    elems = synthetic.elements(args.config)
    dist = world > 1
    if dist:
        import torch.distributed as tdist

    def barrier():
        if dist:
            tdist.barrier()

    # collect garbage and start the clock sampler first, so that the warm-up
    # keeps the GPU busy (and its clocks up) until the timed region starts
    gc.collect()
    clocks = ClockSampler(physical_gpu_index(local)) if rank == 0 else None
    if clocks:
        clocks.start()
    for _ in range(max(3, args.warmup)):
        call()
    ss.check()
    barrier()
    torch.cuda.synchronize()

    # timed region: K steps, per-launch events on the launching stream
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    barrier()
    torch.cuda.synchronize()
    t_wall0 = time.time()
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    n_launch0 = ss.launch_count()
    with gc_paused(collect=False):
        start.record(stream)
        for i in range(args.steps):
            ev[i][0].record(stream)
            call()
            ev[i][1].record(stream)
        end.record(stream)
    torch.cuda.synchronize()
    barrier()
    t_wall1 = time.time()
    n_launch = ss.launch_count() - n_launch0
    ss.check()
    total_ms = start.elapsed_time(end)
    launch_ms = [a.elapsed_time(b) for a, b in ev]
    clock_info = clocks.stop(t_wall0, t_wall1) if clocks else None
    total_ms, avg_launch_ms = max_over_ranks([total_ms, statistics.mean(launch_ms)])
    ms_per_step = total_ms / args.steps
    value = aggregate_rate(world, elems, ms_per_step) / 1e9

    # end to end through the public API, every step: inputs from pinned host
    # memory in, the scan, y and the final state out (pipelined_e2e)
    pinned = {k: torch.from_numpy(np.ascontiguousarray(inp[k])).to(
        torch.bfloat16 if (dt == "bf16" and k not in ("A", "D", "delta_bias", "dt")) else
        torch.float32).pin_memory() for k in host_in if inp.get(k) is not None}
    sets = [(dev, y, hs), (second_set(torch, dev, pinned), torch.empty_like(y),
                           torch.empty_like(hs))]
    host_out = [(torch.empty(y.shape, dtype=y.dtype).pin_memory(),
                 torch.empty(hs.shape, dtype=hs.dtype).pin_memory()) for _ in range(2)]
    h2d = sum(t.numel() * t.element_size() for t in pinned.values())
    d2h = sum(t.numel() * t.element_size() for t in host_out[0])
    e2e_steps = max(2, min(args.steps, 10))

    def compute(j):
        d, yy, hh = sets[j]
        call_on(d, yy, hh)
        return (yy, hh)

    barrier()
    e2e_ms = pipelined_e2e(torch, stream, e2e_steps, pinned, [st[0] for st in sets], compute,
                           host_out)
    e2e_ms = max_over_ranks([e2e_ms])[0]
    barrier()
    if rank != 0:
        return

    peaks, peaks_src = measured_peaks()
    nbytes = algorithmic_bytes(cfg)
    achieved = nbytes / (avg_launch_ms * 1e-3) / 1e9
    traffic = args.traffic
    if traffic is None and args.config in NCU_TRAFFIC and \
            NCU_TRAFFIC[args.config][0] == KERNEL_TAG.get(args.config) and \
            synthetic.CONFIGS[args.config] == BASE_CONFIGS[args.config]:
        traffic = NCU_TRAFFIC[args.config][1]
    roof = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
            "frac": achieved / peaks["hbm_gbs"], "frac_nominal": achieved / NOMINAL_HBM_GBS,
            "traffic": traffic,
            "peak_source": f"{peaks_src} HBM copy bandwidth",
            "bytes_per_launch": nbytes, "avg_launch_ms": avg_launch_ms,
            "kernels_per_call": n_launch / args.steps}
    if n_launch != args.steps:
        roof["note"] = ("the call runs the two-pass form (aggregate pass, then output pass); "
                        "achieved is over the whole call")
    if cfg["kind"] == "scalarA":
        fl = ssd_flops(cfg)
        roof["tensor"] = {"flops_per_launch": fl,
                          "achieved_tflops": fl / (avg_launch_ms * 1e-3) / 1e12,
                          "peak_tflops": peaks.get("bf16_tflops"),
                          "frac": fl / (avg_launch_ms * 1e-3) / 1e12 / peaks.get("bf16_tflops", 1590.0)}
    line = {
        "metric": METRIC, "value": value, "unit": "Gelem/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": dt, "data": "synthetic",
        "config": scan_config(cfg, world),
        "roofline": roof,
        "e2e": {"value": aggregate_rate(world, elems, e2e_ms) / 1e9, "unit": "Gelem/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "steps": e2e_steps},
        "gpu_launches": n_launch,
        "clocks": clock_info,
    }
    if not args.no_cpu_baseline and world == 1:  # the oracle baseline: rank 0 at N = 1
        line["cpu_baseline"] = oracle_sample(args.config, inp, seconds=args.cpu_seconds)
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------ decode step
STEP_BATCH = {"diag": 1024, "scalarA": 512}  # state 336 / 537 MB, far above L2
# DRAM bytes per launch of the decode step at the default batch (ncu capture
# summarised in profiles/step_kernel_decode.md), keyed by config
STEP_NCU_TRAFFIC = {2: ("step_kernel v2", 660.0e6), 4: ("step_kernel v2", 1019.7e6)}
STEP_KERNEL_TAG = "step_kernel v2"


def step_workload(cfg: dict, batch: int) -> dict:
    """The decode step of a config's layer: one token for ``batch`` rows."""
    return dict(cfg, batch=batch, L=1)


def step_name(cfg: dict) -> str:
    if cfg["kind"] == "diag":
        shape = f"D{cfg['dim']} N{cfg['N']}"
    else:
        shape = f"H{cfg['nheads']} P{cfg['headdim']} N{cfg['N']} G{cfg['ngroups']}"
    extra = (", gate" if cfg["gate"] else "") + (", D skip" if cfg.get("D") else "")
    return f"{cfg['kind']} decode step ({shape}, {cfg['dtype']}{extra}), batch {cfg['batch']}"


def step_bytes(cfg: dict) -> int:
    """Bytes one decode step must move: the fp32 state read and written, the
    token's inputs and y, B and C, and the per-channel parameters."""
    es = 2 if cfg["dtype"] == "bf16" else 4
    b = cfg["batch"]
    if cfg["kind"] == "diag":
        dim, N, units = cfg["dim"], cfg["N"], cfg["dim"]
        tok = b * dim * es * (4 if cfg["gate"] else 3)           # u, delta, (z), y
        params = dim * N * 4 + units * 4 * (2 if cfg["D"] else 1)
        bc = 2 * b * N * es
    else:
        units, P, N = cfg["nheads"], cfg["headdim"], cfg["N"]
        dim = units * P
        tok = b * dim * es * (3 if cfg["gate"] else 2) + b * units * 4  # x, (z), y, dt
        params = units * 4 * 2
        bc = 2 * b * cfg["ngroups"] * N * es
    return b * dim * N * 4 * 2 + tok + bc + params


def run_step(args, rank: int, world: int, local: int):
    """Decode-step arm (``--op step``): selscan_step / selscan_step_scalarA
    on the config's layer with ``--batch`` rows (default 512 diagonal, 256
    scalar), the state resident on the device and updated in place."""
    import torch
    import selective_state_space_selscan_b200 as ss
    torch.cuda.set_device(local)
    base = synthetic.CONFIGS[args.config]
    batch = args.batch or STEP_BATCH[base["kind"]]
    cfg = step_workload(base, batch)
    dt = cfg["dtype"]
    stream = torch.cuda.current_stream()
    rng = np.random.default_rng(cfg["seed"] + 1000 + rank)
    if cfg["kind"] == "diag":
        inp = synthetic.make_diag(batch, cfg["dim"], cfg["N"], 1, dtype=dt, seed=shard_seed(cfg, rank),
                                  gate=cfg["gate"], D=cfg["D"])
        state_shape = (batch, cfg["dim"], cfg["N"])
        tok_keys = ("u", "delta", "z", "B", "C")
    else:
        inp = synthetic.make_scalarA(batch, cfg["nheads"], cfg["headdim"], cfg["N"], 1,
                                     ngroups=cfg["ngroups"], dtype=dt, seed=shard_seed(cfg, rank),
                                     gate=cfg["gate"])
        state_shape = (batch, cfg["nheads"], cfg["headdim"], cfg["N"])
        tok_keys = ("x", "dt", "z", "B", "C")
    host = {k: inp[k][..., 0] for k in tok_keys if inp.get(k) is not None}
    dev = {k: to_dev(v, "f32" if k == "dt" else dt, torch) for k, v in host.items()}
    par = {k: to_dev(inp[k], "f32", torch) for k in ("A", "D", "delta_bias")
           if inp.get(k) is not None}
    state = torch.from_numpy(rng.standard_normal(state_shape, dtype=np.float32)).cuda()
    first = dev["u"] if "u" in dev else dev["x"]
    y = torch.empty(first.shape, dtype=first.dtype, device="cuda")

    if cfg["kind"] == "diag":
        def call_on(d, yy):
            ss.selscan_step(state, d["u"], d["delta"], par["A"], d["B"], d["C"],
                            D=par.get("D"), z=d.get("z"), delta_bias=par.get("delta_bias"),
                            out=yy)
    else:
        def call_on(d, yy):
            ss.selscan_step_scalarA(state, d["x"], d["dt"], par["A"], d["B"], d["C"],
                                    cfg["headdim"], D=par.get("D"), z=d.get("z"), out=yy)

    def call():
        call_on(dev, y)

    dist = world > 1
    if dist:
        import torch.distributed as tdist

    def barrier():
        if dist:
            tdist.barrier()

    # collect garbage and start the clock sampler first, so that the warm-up
    # keeps the GPU busy (and its clocks up) until the timed region starts
    gc.collect()
    clocks = ClockSampler(physical_gpu_index(local)) if rank == 0 else None
    if clocks:
        clocks.start()
    for _ in range(max(3, args.warmup)):
        call()
    ss.check()
    barrier()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    barrier()
    torch.cuda.synchronize()
    t_wall0 = time.time()
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    n_launch0 = ss.launch_count()
    with gc_paused(collect=False):
        start.record(stream)
        for i in range(args.steps):
            ev[i][0].record(stream)
            call()
            ev[i][1].record(stream)
        end.record(stream)
    torch.cuda.synchronize()
    barrier()
    t_wall1 = time.time()
    n_launch = ss.launch_count() - n_launch0
    ss.check()
    total_ms = start.elapsed_time(end)
    avg_launch_ms = statistics.mean(a.elapsed_time(b) for a, b in ev)
    clock_info = clocks.stop(t_wall0, t_wall1) if clocks else None
    total_ms, avg_launch_ms = max_over_ranks([total_ms, avg_launch_ms])
    ms_per_step = total_ms / args.steps
    value = aggregate_rate(world, batch, ms_per_step)

    # end to end: the token's inputs from pinned host memory, y back, every
    # step (pipelined_e2e); the state stays resident on the device, as a
    # decoding server keeps it, and is updated in place step after step
    pinned = {k: torch.from_numpy(np.ascontiguousarray(v)).to(
        torch.float32 if (k == "dt" or dt == "f32") else torch.bfloat16).pin_memory()
        for k, v in host.items()}
    sets = [dev, second_set(torch, dev, pinned)]
    ys = [y, torch.empty_like(y)]
    host_out = [(torch.empty(y.shape, dtype=y.dtype).pin_memory(),) for _ in range(2)]
    h2d = sum(t.numel() * t.element_size() for t in pinned.values())
    d2h = host_out[0][0].numel() * host_out[0][0].element_size()
    e2e_steps = max(2, min(args.steps, 100))

    def compute(j):
        call_on(sets[j], ys[j])
        return (ys[j],)

    barrier()
    e2e_ms = pipelined_e2e(torch, stream, e2e_steps, pinned, sets, compute, host_out)
    e2e_ms = max_over_ranks([e2e_ms])[0]
    barrier()
    if rank != 0:
        return
    peaks, peaks_src = measured_peaks()
    nbytes = step_bytes(cfg)
    traffic = args.traffic
    if traffic is None and args.config in STEP_NCU_TRAFFIC and \
            STEP_NCU_TRAFFIC[args.config][0] == STEP_KERNEL_TAG and \
            batch == STEP_BATCH[cfg["kind"]] and base == BASE_CONFIGS[args.config]:
        traffic = STEP_NCU_TRAFFIC[args.config][1]
    achieved = nbytes / (avg_launch_ms * 1e-3) / 1e9
    dim = cfg.get("dim") or cfg["nheads"] * cfg["headdim"]
    line = {
        "metric": "selective-scan decode step, tokens/s (one token per batch row) and % of "
                  "B200 HBM roofline, 1 GPU",
        "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": dt, "data": "synthetic",
        "config": step_config(cfg, world),
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"],
                     "unit": "GB/s", "frac": achieved / peaks["hbm_gbs"],
                     "frac_nominal": achieved / NOMINAL_HBM_GBS,
                     "traffic": traffic, "peak_source": f"{peaks_src} HBM copy bandwidth",
                     "bytes_per_launch": nbytes, "avg_launch_ms": avg_launch_ms},
        "e2e": {"value": aggregate_rate(world, batch, e2e_ms), "unit": "tokens/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": e2e_steps},
        "gpu_launches": n_launch,
        "clocks": clock_info,
    }
    if not args.no_cpu_baseline and world == 1:  # the oracle baseline: rank 0 at N = 1
        line["cpu_baseline"] = oracle_step_sample(cfg, inp, state.cpu().numpy(),
                                                  seconds=args.cpu_seconds)
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------ backward
def bwd_bytes(cfg: dict) -> int:
    """Bytes one backward call must move: u, delta, z, dy read and du,
    ddelta, dz written once, B and C read and dB, dC (fp32) written once,
    the per-channel parameters and their gradients.  Scalar A: x, z, dy read
    and dx, dz written (bf16), dt read and ddt written (fp32, per head), B
    and C read (bf16) and dB, dC written (fp32) per group."""
    if cfg["kind"] == "scalarA":
        b, H, P, N, L = cfg["batch"], cfg["nheads"], cfg["headdim"], cfg["N"], cfg["L"]
        G = cfg["ngroups"]
        total = b * H * P * L * 2 * ((2 if cfg["gate"] else 1) * 2 + 1)   # x, z in+grad; dy
        total += b * H * L * 8                                             # dt in, ddt out
        total += 2 * b * G * N * L * (2 + 4)                               # B, C in; dB, dC out
        total += 4 * H * 4                                                 # A, dA, D, dD
        return total
    es = 2 if cfg["dtype"] == "bf16" else 4
    b, dim, N, L = cfg["batch"], cfg["dim"], cfg["N"], cfg["L"]
    per_elem = es * (3 if cfg["gate"] else 2) * 2 + es           # (u, delta, z) in+grad, dy
    total = b * dim * L * per_elem
    total += 2 * b * N * L * (es + 4)                               # B, C in; dB, dC out
    total += 2 * dim * N * 4 + 4 * dim * 4                          # A, dA; D, dD, bias, dbias
    return total


# DRAM bytes per launch of the backward's dominant kernel (ncu): captured at
# L = 1024 and scaled by tokens to L = 4096 (profiles/selscan_bwd_config2.md,
# profiles/ssd_bwd_scalarA_config4.md)
BWD_NCU_TRAFFIC = {2: ("selscan_bwd_kernel v5", 4 * 687.2e6),
                   4: ("ssd_bwd_kernel v9", 4 * 185.6e6)}
BWD_KERNEL_TAG = {2: "selscan_bwd_kernel v5", 4: "ssd_bwd_kernel v9"}


def bwd_traffic(args, cfg):
    if args.traffic is not None:
        return args.traffic
    ent = BWD_NCU_TRAFFIC.get(args.config)
    if ent and ent[0] == BWD_KERNEL_TAG.get(args.config) and cfg == BASE_CONFIGS[args.config]:
        return ent[1]
    return None


def run_bwd(args, rank: int, world: int, local: int):
    """Backward arm (``--op bwd``): selscan_bwd on the config's diagonal
    workload with a seeded upstream gradient dy."""
    import torch
    import selective_state_space_selscan_b200 as ss
    torch.cuda.set_device(local)
    cfg = synthetic.CONFIGS[args.config]
    scalar = cfg["kind"] == "scalarA"
    inp = synthetic.make_config(args.config, seed=shard_seed(cfg, rank))
    dt = cfg["dtype"]
    stream = torch.cuda.current_stream()
    rng = np.random.default_rng(shard_seed(cfg, rank) + 500)
    xk = "x" if scalar else "u"
    dy_host = rng.standard_normal(inp[xk].shape, dtype=np.float32)
    if scalar:
        dev = {k: to_dev(inp[k], dt, torch) for k in ("x", "B", "C", "z")}
        dev["dt"] = to_dev(inp["dt"], "f32", torch)
        par = {k: to_dev(inp[k], "f32", torch) for k in ("A", "D")}
    else:
        dev = {k: to_dev(inp[k], dt, torch) for k in ("u", "delta", "B", "C", "z")}
        par = {k: to_dev(inp[k], "f32", torch) for k in ("A", "D", "delta_bias")}
    dev["dy"] = to_dev(dy_host, dt, torch)

    def call_on(d):
        if scalar:
            return ss.selscan_bwd_scalarA(d["x"], d["dt"], par["A"], d["B"], d["C"],
                                          inp["headdim"], d["dy"], D=par["D"], z=d["z"])
        return ss.selscan_bwd(d["u"], d["delta"], par["A"], d["B"], d["C"], d["dy"],
                              D=par["D"], z=d["z"], delta_bias=par["delta_bias"])

    def call():
        return call_on(dev)

    dist = world > 1
    if dist:
        import torch.distributed as tdist

    def barrier():
        if dist:
            tdist.barrier()

    # collect garbage and start the clock sampler first, so that the warm-up
    # keeps the GPU busy (and its clocks up) until the timed region starts
    gc.collect()
    clocks = ClockSampler(physical_gpu_index(local)) if rank == 0 else None
    if clocks:
        clocks.start()
    for _ in range(max(3, args.warmup)):
        call()
    ss.check()
    barrier()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    barrier()
    torch.cuda.synchronize()
    t_wall0 = time.time()
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    n_launch0 = ss.launch_count()
    with gc_paused(collect=False):
        start.record(stream)
        for i in range(args.steps):
            ev[i][0].record(stream)
            grads = call()
            ev[i][1].record(stream)
        end.record(stream)
    torch.cuda.synchronize()
    barrier()
    t_wall1 = time.time()
    n_launch = ss.launch_count() - n_launch0
    ss.check()
    total_ms = start.elapsed_time(end)
    avg_launch_ms = statistics.mean(a.elapsed_time(b) for a, b in ev)
    clock_info = clocks.stop(t_wall0, t_wall1) if clocks else None
    total_ms, avg_launch_ms = max_over_ranks([total_ms, avg_launch_ms])
    ms_per_step = total_ms / args.steps
    elems = cfg["batch"] * cfg_dim(cfg) * cfg["L"]
    value = aggregate_rate(world, elems, ms_per_step) / 1e9

    # end to end: inputs and dy from pinned host memory in, every gradient out,
    # every step (pipelined_e2e)
    host_keys = ("x", "dt", "B", "C", "z", "dy") if scalar else ("u", "delta", "B", "C", "z", "dy")
    src = dict(inp, dy=dy_host)
    pinned = {k: torch.from_numpy(np.ascontiguousarray(src[k])).to(
        torch.bfloat16 if (dt == "bf16" and k != "dt") else torch.float32).pin_memory()
        for k in host_keys if src.get(k) is not None}
    out_keys = [k for k, v in grads.items() if v is not None]
    host_out = [tuple(torch.empty(grads[k].shape, dtype=grads[k].dtype).pin_memory()
                      for k in out_keys) for _ in range(2)]
    sets = [dev, second_set(torch, dev, pinned)]
    h2d = sum(t.numel() * t.element_size() for t in pinned.values())
    d2h = sum(t.numel() * t.element_size() for t in host_out[0])
    e2e_steps = max(2, min(args.steps, 10))

    def compute(j):
        g = call_on(sets[j])
        return tuple(g[k] for k in out_keys)

    barrier()
    e2e_ms = pipelined_e2e(torch, stream, e2e_steps, pinned, sets, compute, host_out)
    e2e_ms = max_over_ranks([e2e_ms])[0]
    barrier()
    if rank != 0:
        return
    peaks, peaks_src = measured_peaks()
    nbytes = bwd_bytes(cfg)
    achieved = nbytes / (avg_launch_ms * 1e-3) / 1e9
    line = {
        "metric": "selective-scan backward Gelem/s (B·D·L) and % of B200 HBM roofline, 1 GPU",
        "value": value, "unit": "Gelem/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": dt, "data": "synthetic",
        "config": bwd_config(cfg, world),
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"],
                     "unit": "GB/s", "frac": achieved / peaks["hbm_gbs"],
                     "frac_nominal": achieved / NOMINAL_HBM_GBS,
                     "traffic": bwd_traffic(args, cfg), "peak_source": f"{peaks_src} HBM copy bandwidth",
                     "bytes_per_launch": nbytes, "avg_launch_ms": avg_launch_ms,
                     "kernels_per_call": n_launch / args.steps},
        "e2e": {"value": aggregate_rate(world, elems, e2e_ms) / 1e9, "unit": "Gelem/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": e2e_steps},
        "gpu_launches": n_launch,
        "clocks": clock_info,
    }
    if scalar:
        fl = ssd_bwd_flops(cfg)
        peak = peaks.get("bf16_tflops", 1590.0) * TF32_PER_BF16
        line["roofline"]["tensor"] = {
            "flops_per_launch": fl, "dtype": "tf32",
            "achieved_tflops": fl / (avg_launch_ms * 1e-3) / 1e12, "peak_tflops": peak,
            "peak_source": f"{peaks_src} bf16 GEMM x nominal tf32/bf16 ratio {TF32_PER_BF16:.3f}",
            "frac": fl / (avg_launch_ms * 1e-3) / 1e12 / peak}
    if not args.no_cpu_baseline and world == 1:  # the oracle baseline: rank 0 at N = 1
        line["cpu_baseline"] = oracle_bwd_sample(cfg, inp, dy_host, seconds=args.cpu_seconds)
    print(json.dumps(line), flush=True)


def oracle_bwd_sample(cfg: dict, inp: dict, dy: np.ndarray, seconds: float = 10.0):
    """The fp64 oracle's backward on whole channels of the workload (all
    batches, all tokens; whole heads for scalar A), grown until about
    `seconds` of work; Gelem/s."""
    import oracle
    n, spent = 1, 0.0
    b, L = cfg["batch"], cfg["L"]
    if cfg["kind"] == "scalarA":
        P, per = cfg["headdim"], cfg["nheads"] // cfg["ngroups"]
        while True:
            ch = lambda x: None if x is None else x[:, :n * P]
            hv = lambda x: None if x is None else x[:n]
            t0 = time.perf_counter()
            oracle.selscan_scalarA_bwd(ch(inp["x"]), inp["dt"][:, :n], inp["A"][:n],
                                       inp["B"][:, :1], inp["C"][:, :1], P, dy[:, :n * P],
                                       D=hv(inp["D"]), z=ch(inp["z"]))
            spent = time.perf_counter() - t0
            if spent >= seconds * 0.5 or n >= per:
                break
            n = int(min(per, n * max(2.0, min(16.0, seconds / max(spent, 1e-3)))))
        return {"value": b * n * P * L / spent / 1e9, "unit": "Gelem/s", "cores": 1,
                "kind": "oracle",
                "sample": f"{n} head(s) x {P} channels x batch {b} x L {L}, {spent:.1f} s "
                          "single-threaded fp64"}
    while True:
        sl = lambda x: None if x is None else x[:, :n]
        vec = lambda x: None if x is None else x[:n]
        t0 = time.perf_counter()
        oracle.selscan_bwd(sl(inp["u"]), sl(inp["delta"]), inp["A"][:n], inp["B"], inp["C"],
                           dy[:, :n], D=vec(inp["D"]), z=sl(inp["z"]),
                           delta_bias=vec(inp["delta_bias"]))
        spent = time.perf_counter() - t0
        if spent >= seconds * 0.5 or n >= cfg["dim"]:
            break
        n = int(min(cfg["dim"], n * max(2.0, min(16.0, seconds / max(spent, 1e-3)))))
    return {"value": b * n * L / spent / 1e9, "unit": "Gelem/s", "cores": 1, "kind": "oracle",
            "sample": f"{n} channel(s) x batch {b} x L {L}, {spent:.1f} s single-threaded fp64"}


def oracle_step_sample(cfg: dict, inp: dict, state: np.ndarray, seconds: float = 10.0):
    """The fp64 oracle's decode step on the first rows of the batch, grown
    until about `seconds` of single-threaded work; tokens/s."""
    import oracle
    rows, spent = 1, 0.0
    while True:
        t0 = time.perf_counter()
        if cfg["kind"] == "diag":
            oracle.selscan_step(state[:rows], inp["u"][:rows, :, 0], inp["delta"][:rows, :, 0],
                                inp["A"], inp["B"][:rows, :, 0], inp["C"][:rows, :, 0],
                                D=inp["D"], z=None if inp["z"] is None else inp["z"][:rows, :, 0],
                                delta_bias=inp["delta_bias"])
        else:
            sl = lambda a: None if a is None else a[:rows]
            oracle.selscan_scalarA(sl(inp["x"]), sl(inp["dt"]), inp["A"], sl(inp["B"]),
                                   sl(inp["C"]), cfg["headdim"], D=inp["D"], z=sl(inp["z"]),
                                   h0=state[:rows])
        spent = time.perf_counter() - t0
        if spent >= seconds * 0.5 or rows >= cfg["batch"]:
            break
        rows = int(min(cfg["batch"], rows * max(2.0, min(16.0, seconds / max(spent, 1e-3)))))
    return {"value": rows / spent, "unit": "tokens/s", "cores": 1, "kind": "oracle",
            "sample": f"{rows} batch row(s) of one decode step, {spent:.2f} s "
                      "single-threaded fp64"}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--config", type=int, default=2)
    ap.add_argument("--batch", type=int, default=None,
                    help="override the config's batch (smaller profiling cases)")
    ap.add_argument("--seqlen", type=int, default=None,
                    help="override the config's L (smaller profiling cases)")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--op", default="scan", choices=["scan", "step", "bwd"],
                    help="scan: the forward over the config's sequence (default); "
                         "step: one decode step of the config's layer; "
                         "bwd: the backward pass of the config's scan")
    ap.add_argument("--traffic", type=float, default=None,
                    help="DRAM bytes per launch from an ncu capture of this kernel")
    args = ap.parse_args()

    if args.batch is not None and args.op != "step":
        synthetic.CONFIGS[args.config] = dict(synthetic.CONFIGS[args.config], batch=args.batch)
    if args.seqlen is not None:
        synthetic.CONFIGS[args.config] = dict(synthetic.CONFIGS[args.config], L=args.seqlen)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    if world > 1:
        import datetime
        import torch
        import torch.distributed as tdist
        torch.cuda.set_device(local)
        tdist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                 device_id=torch.device("cuda", local))
    try:
        {"step": run_step, "bwd": run_bwd}.get(args.op, run_gpu)(args, rank, world, local)
    finally:
        if world > 1:
            import torch.distributed as tdist
            tdist.destroy_process_group()


if __name__ == "__main__":
    main()
