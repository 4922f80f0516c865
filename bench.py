#!/usr/bin/env python
"""Throughput benchmark of patch-restricted attention on B200.

One step = one forward call of the library (NPA or PCPP, per the workload)
over the whole synthetic workload, inputs resident in HBM. Prints one JSON
line (rank 0) with the useful TFLOP/s of all ranks, the roofline of the
kernel, an end-to-end figure through host buffers, the CPU oracle timed on a
bounded sample, and the SM clocks seen during the timed region.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
    python bench.py --impl reference ...   # the CPU oracle, as it stands

Multi-GPU (torchrun, one process per GPU): every rank runs the full workload
as an independent replica (the attention of different images, heads or
patches needs no exchange), so per-GPU work is fixed and scaling is weak.
"""
from __future__ import annotations

import argparse
import glob
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

from workloads import ASG_WORKLOADS, COMPARATORS, PRESETS, AsgWorkload, Workload, make_asg_inputs, make_inputs, \
    preset  # noqa: E402

DEFAULT_WORKLOAD = "npa_sdxl_4096"
L2_BYTES = 126 * 1024 * 1024
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
DATASHEET_BF16_DENSE_TFLOPS = 2250.0
KERNEL_NAME = "npa_fwd_kernel"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=60)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD,
                    choices=sorted(PRESETS) + sorted(COMPARATORS) + sorted(ASG_WORKLOADS))
    ap.add_argument("--cpu-seconds", type=float, default=15.0,
                    help="approximate CPU time of the oracle baseline sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-per-config", action="store_true",
                    help="skip timing the other target workloads (per_config) after the headline one")
    ap.add_argument("--flush-l2", action="store_true",
                    help="write 256 MB between launches even when the inputs exceed L2 (cold-cache variant)")
    return ap.parse_args()


def describe(w: Workload) -> dict:
    cfg = {"workload": w.name, "B": w.B, "heads": w.heads, "grid": f"{w.H}x{w.W}", "d": w.d}
    if w.geometry in ("npa", "md"):
        cfg.update({"geometry": w.geometry, "patch": w.patch, "margin": w.margin})
        if w.geometry == "md":
            cfg["comparator"] = "overlapping NPA windows, each attending within itself, outputs averaged"
    elif w.geometry == "gq":
        cfg.update({"geometry": "gq", "queries": "the global tokens, over all image and global keys"})
    else:
        cfg.update({"geometry": "pcpp", "n_strips": w.n_strips, "p": w.p})
    cfg["global_tokens"] = w.G
    if w.smooth_k:
        cfg["k"] = "3x3 box-filtered"
    return cfg


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in ("hbm_gbs", "bf16_tflops", "bf16_tflops_sustained")}, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def _strip_comments(src: str) -> str:
    """C/C++ source without comments, trailing spaces or blank lines (string
    literals are kept as they are)."""
    import re
    pattern = re.compile(r'//[^\n]*|/\*.*?\*/|"(?:\\.|[^"\\])*"', re.S)
    src = pattern.sub(lambda m: m.group(0) if m.group(0).startswith('"') else "", src)
    return "\n".join(line.rstrip() for line in src.splitlines() if line.strip())


def kernel_source_hash() -> str:
    """Hash of the kernel sources (csrc/), comments and layout excluded: the
    recorded ncu counters apply while the code itself is unchanged."""
    h = hashlib.sha256()
    for f in sorted(glob.glob(os.path.join(ROOT, "patch_res_diffusion_b200", "csrc", "*"))):
        with open(f, encoding="utf-8") as fh:
            h.update(os.path.basename(f).encode())
            h.update(_strip_comments(fh.read()).encode())
    return h.hexdigest()[:16]


def recorded_traffic(workload: str):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on
    the current kernel source (else None)."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        rec = json.load(f)
    ent = rec.get(workload)
    if not ent or ent.get("kernel_source_hash") != kernel_source_hash():
        return None
    return ent.get("dram_bytes_per_launch")


def useful_flops(w: Workload) -> float:
    import patch_res_diffusion_b200 as npa
    if w.geometry == "npa":
        return npa.npa_useful_flops(w.B, w.heads, w.H, w.W, w.d, w.patch, w.margin, w.G)
    if w.geometry == "md":
        return npa.npa_multidiffusion_useful_flops(w.B, w.heads, w.H, w.W, w.d, w.patch, w.margin, w.G)
    if w.geometry == "gq":
        return 4.0 * w.d * w.B * w.heads * w.G * (w.H * w.W + w.G)
    return npa.pcpp_useful_flops(w.B, w.heads, w.H, w.W, w.d, w.n_strips, w.p, w.G)


def max_over_ranks(ms: float, world: int, device) -> float:
    """The slowest rank's timed region (every rank takes part; world 1 returns
    ms). ``device``: where the reduction tensor lives (cuda under NCCL, cpu
    under gloo)."""
    if world <= 1:
        return ms
    import torch
    import torch.distributed as dist
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(world: int, units_per_rank_step: float, steps: int, slowest_ms: float) -> float:
    """Units per second of the whole job: every rank processed
    ``units_per_rank_step`` per step (replicas: weak scaling), over the
    slowest rank's time."""
    return world * units_per_rank_step * steps / (slowest_ms * 1e-3)


# ---------------------------------------------------------------------------
# CPU oracle baseline (bounded sample of the same workload)
# ---------------------------------------------------------------------------

def oracle_rate(w: Workload, inp: dict, seconds: float) -> dict:
    """Times the float64 oracle on a growing random query sample until about
    ``seconds`` of wall time; returns useful TFLOP/s and what was sampled."""
    import oracle
    rng = np.random.default_rng(123)
    N = w.H * w.W
    geom = dict(patch=w.patch, margin=w.margin) if w.geometry in ("npa", "md") else \
        dict(n_strips=w.n_strips, p=w.p)
    fn = {"npa": oracle.npa_attention, "md": oracle.multidiffusion_attention}.get(w.geometry,
                                                                                  oracle.pcpp_attention)
    if w.geometry == "pcpp_stale":
        fn = lambda q, k, v, **kw: oracle.pcpp_attention_stale(q, k, v, inp["ks"], inp["vs"], **kw)
    if w.geometry == "gq":
        N_img = N
        N = w.G  # the queries are the global tokens
        fn = lambda q, k, v, gk, gv, G, queries, **kw: oracle.global_query_attention(
            inp["gq"], k, v, gk, gv, G=G, queries=queries, **{a: kw[a] for a in ("B", "heads", "H", "W", "d")})
        geom = {}
    if w.geometry == "gq":
        key_count = lambda t: N_img
    elif w.geometry == "npa":
        key_count = lambda t: len(oracle.npa_key_set(w.H, w.W, w.patch, w.margin, t))
    elif w.geometry == "md":
        key_count = lambda t: md_query_pairs(w, t) - w.G * md_cover(w, t)
    else:
        key_count = lambda t: len(oracle.pcpp_key_set(w.H, w.W, w.n_strips, w.p, t))
    n, total_q, total_pairs, total_t = 64, 0, 0, 0.0
    while total_t < seconds:
        qs = np.stack([rng.integers(w.B, size=n), rng.integers(w.heads, size=n), rng.integers(N, size=n)],
                      axis=1).astype(np.int32)
        pairs = sum(key_count(int(t)) + w.G * (md_cover(w, int(t)) if w.geometry == "md" else 1)
                    for t in qs[:, 2])
        t0 = time.perf_counter()
        out = fn(inp["q"], inp["k"], inp["v"], gk=inp.get("gk"), gv=inp.get("gv"), G=w.G, B=w.B, heads=w.heads,
                 H=w.H, W=w.W, d=w.d, queries=qs, **geom)
        dt = time.perf_counter() - t0
        last_sample = (qs, out)
        total_q += n
        total_pairs += pairs
        total_t += dt
        n = min(n * 2, 1 << 16)
    flops = 4.0 * w.d * total_pairs
    return {
        "value": flops / total_t / 1e12,
        "unit": "TFLOP/s",
        "cores": oracle.num_threads(),
        "kind": "oracle",
        "sample": f"{total_q} uniformly drawn (b, h, query) rows of {w.name}, float64, {total_t:.1f} s",
        "seconds": total_t,
        "last_sample": last_sample,
    }


def _md_axis(L: int, P: int, m: int, x: int):
    """Extents of the windows containing coordinate x along one axis."""
    out = []
    for i in range((L + P - 1) // P):
        lo, hi = max(0, i * P - m), min(L, (i + 1) * P + m)
        if lo <= x < hi:
            out.append(hi - lo)
    return out


def md_cover(w: Workload, t: int) -> int:
    """Windows containing token t (overlapping-window comparator)."""
    return len(_md_axis(w.H, w.patch, w.margin, t // w.W)) * len(_md_axis(w.W, w.patch, w.margin, t % w.W))


def md_query_pairs(w: Workload, t: int) -> int:
    """(query, key) pairs the comparator evaluates for token t: its window's
    keys (plus the global keys) in every window containing it."""
    rows, cols = _md_axis(w.H, w.patch, w.margin, t // w.W), _md_axis(w.W, w.patch, w.margin, t % w.W)
    return sum(rows) * sum(cols) + w.G * len(rows) * len(cols)


def run_reference(args, w: Workload, rank: int) -> None:
    if rank != 0:
        return
    inp = make_inputs(w)
    steps = []
    budget = max(0.5, min(2.0 * args.cpu_seconds, 30.0) / max(1, args.steps + args.warmup))
    for i in range(args.warmup + args.steps):
        r = oracle_rate(w, inp, budget)
        if i >= args.warmup:
            steps.append(r)
    value = statistics.median(r["value"] for r in steps)
    flops_step = useful_flops_host(w)
    line = {
        "impl": "reference",
        "metric": "patch-attention useful TFLOP/s (bf16) and % of B200 dense BF16 peak",
        "value": value,
        "unit": "TFLOP/s",
        "n_gpus": args.gpus,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": flops_step / (value * 1e12) * 1e3,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f64",
        "data": "synthetic",
        "config": describe(w),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": steps[0]["cores"], "kind": "oracle",
                         "sample": "each step: " + steps[-1]["sample"]},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "note": "ms_per_step is projected from the sampled rate to the full workload",
    }
    print(json.dumps(line), flush=True)


def useful_flops_host(w: Workload) -> float:
    import oracle
    if w.geometry == "gq":
        return 4.0 * w.d * w.B * w.heads * w.G * (w.H * w.W + w.G)
    if w.geometry == "md":
        return 4.0 * w.d * w.B * w.heads * oracle.md_pair_count(w.H, w.W, w.patch, w.margin, w.G)
    pairs = oracle.pair_count("pcpp" if w.geometry == "pcpp_stale" else w.geometry, w.H, w.W, patch=w.patch,
                              margin=w.margin, n_strips=w.n_strips, p=w.p, G=w.G)
    return 4.0 * w.d * w.B * w.heads * pairs


# ---------------------------------------------------------------------------
# Clock sampling during the timed region
# ---------------------------------------------------------------------------

class ClockSampler:
    """Samples SM clocks, power and throttle reasons with nvidia-smi every
    20 ms; ``stop()`` keeps the samples stamped inside the window between
    ``mark_begin()`` and ``mark_end()`` (host wall clock; the timed region),
    or the nearest sample when none falls inside."""
    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None
        self.path = os.path.join("/tmp", f"npa_clocks_{os.getpid()}_{device_index}.csv")
        self.t0 = self.t1 = None

    def start(self):
        try:
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.dev), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "20"],
                                         stdout=self.fh, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def mark_begin(self):
        self.t0 = time.time()

    def mark_end(self):
        self.t1 = time.time()

    @staticmethod
    def _stamp(text: str):
        import datetime
        for fmt in ("%Y/%m/%d %H:%M:%S.%f", "%Y/%m/%d %H:%M:%S"):
            try:
                return datetime.datetime.strptime(text, fmt).timestamp()
            except ValueError:
                continue
        return None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.fh.close()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 10:
                    continue
                try:
                    rows.append({"t": self._stamp(parts[0]), "sm": float(parts[2]), "max": float(parts[3]),
                                 "power": float(parts[4]), "hw": parts[6], "hw_thermal": parts[7],
                                 "sw_thermal": parts[8], "sw_power": parts[9]})
                except ValueError:
                    continue
        os.unlink(self.path)
        if not rows:
            return None
        inside = [r for r in rows if r["t"] is not None and self.t0 is not None and self.t1 is not None
                  and self.t0 <= r["t"] <= self.t1]
        basis = "samples stamped inside the timed region"
        if not inside:
            mid = 0.5 * (self.t0 + self.t1) if self.t0 is not None and self.t1 is not None else None
            stamped = [r for r in rows if r["t"] is not None]
            if mid is not None and stamped:
                inside = [min(stamped, key=lambda r: abs(r["t"] - mid))]
                basis = "no sample inside the timed region; the nearest one"
            else:
                inside = rows
                basis = "no timestamps; every sample"
        reasons = set()
        for r in inside:
            for key, name in (("hw", "hw_slowdown"), ("hw_thermal", "hw_thermal_slowdown"),
                              ("sw_thermal", "sw_thermal_slowdown"), ("sw_power", "sw_power_cap")):
                if r[key].lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(r["sm"] for r in inside), "sm_max_mhz": max(r["max"] for r in rows),
                "reasons": sorted(reasons), "samples": len(inside), "basis": basis,
                "power_w_max": max(r["power"] for r in inside),
                "region_s": (self.t1 - self.t0) if self.t0 is not None and self.t1 is not None else None}


# ---------------------------------------------------------------------------
# The GPU arm
# ---------------------------------------------------------------------------

def prepare(w: Workload, dev, flush_l2: bool, inp: dict = None):
    """Device tensors, workspaces and the library call of one workload step.
    Returns a namespace with ``call()`` (one step on the current stream),
    the tensors, the useful flops, the minimum HBM bytes and the L2 flush
    buffer (allocated when the inputs fit in twice the L2 or when asked)."""
    import types
    import torch
    import patch_res_diffusion_b200 as npa

    inp = make_inputs(w) if inp is None else inp

    def dev_bf16(a):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).to(dev).view(torch.bfloat16)

    q, k, v = dev_bf16(inp["q"]), dev_bf16(inp["k"]), dev_bf16(inp["v"])
    gk = dev_bf16(inp["gk"]) if w.G else None
    gv = dev_bf16(inp["gv"]) if w.G else None
    ks = dev_bf16(inp["ks"]) if w.geometry == "pcpp_stale" else None
    vs = dev_bf16(inp["vs"]) if w.geometry == "pcpp_stale" else None
    gq = dev_bf16(inp["gq"]) if w.geometry == "gq" else None
    o = torch.empty_like(gq if gq is not None else q)
    stream = torch.cuda.current_stream(dev)
    # minimum HBM bytes of one call: every input read once, the output written once
    bytes_io = (q.numel() * 4 + (2 * gk.numel() if w.G else 0)) * 2  # q, k, v, o (+ global k, v)
    if w.geometry == "gq":  # global queries and output, global k, v, image k, v
        bytes_io = (4 * gq.numel() + 2 * k.numel()) * 2
    elif w.geometry == "pcpp_stale":  # + the borrowed rows of the previous step's k, v
        r = npa.pcpp_neighbor_rows(w.H // w.n_strips, w.p)
        bytes_io += 2 * (2 * r * (w.n_strips - 1)) * w.W * w.d * 2 * w.B * w.heads
    needs_flush = bytes_io < 2 * L2_BYTES or flush_l2
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev) if needs_flush else None

    md_bytes = npa.npa_multidiffusion_workspace_size(w.B, w.heads, w.H, w.W, w.d, w.patch, w.margin) \
        if w.geometry == "md" else 0
    md_ws = [torch.empty(md_bytes, dtype=torch.uint8, device=dev) for _ in range(2)] if md_bytes else None
    gq_bytes = npa.npa_global_query_workspace_size(w.B, w.heads, w.H, w.W, w.d, w.G) if gq is not None else 0
    gq_ws = torch.empty(max(gq_bytes, 16), dtype=torch.uint8, device=dev) if gq is not None else None

    def call():
        if w.geometry == "npa":
            npa.npa_attention_fwd(q, k, v, o, w.B, w.heads, w.H, w.W, w.d, w.patch, w.margin, gk, gv, w.G, stream)
        elif w.geometry == "md":
            npa.npa_multidiffusion_attention_fwd(q, k, v, o, w.B, w.heads, w.H, w.W, w.d, w.patch, w.margin,
                                                 md_ws[0], md_bytes, gk, gv, w.G, stream)
        elif w.geometry == "pcpp_stale":
            npa.pcpp_attention_fwd_stale(q, k, v, ks, vs, o, w.B, w.heads, w.H, w.W, w.d, w.n_strips, w.p, 0,
                                         w.n_strips, gk, gv, w.G, stream)
        elif w.geometry == "gq":
            npa.npa_global_query_attention_fwd(gq, k, v, gk, gv, o, w.B, w.heads, w.H, w.W, w.d, w.G, gq_ws,
                                               gq_bytes, stream)
        else:
            npa.pcpp_attention_fwd(q, k, v, o, w.B, w.heads, w.H, w.W, w.d, w.n_strips, w.p, gk, gv, w.G, stream)

    launches = 2 if w.geometry == "md" or gq_bytes > 0 else 1
    return types.SimpleNamespace(w=w, inp=inp, q=q, k=k, v=v, gk=gk, gv=gv, gq=gq, o=o, stream=stream,
                                 flops=useful_flops(w), bytes_io=bytes_io, flush=flush, md_ws=md_ws,
                                 md_bytes=md_bytes, call=call, launches=launches)


def timed_steps(prep, steps: int, warmup: int, dev, world: int, local_rank: int) -> dict:
    """``warmup`` untimed steps, then exactly ``steps`` timed ones bracketed by
    a synchronize (and a barrier when world > 1) on both sides, with CUDA
    events around every step and around the region on the launching stream.
    With a flush buffer, 256 MB are written before every step (outside the
    per-step events) and the region's time is the sum of the per-step
    times. Clocks are sampled during the region."""
    import torch
    import torch.distributed as dist
    import patch_res_diffusion_b200 as npa

    stream, flush, call = prep.stream, prep.flush, prep.call
    for _ in range(warmup):
        if flush is not None:
            flush.fill_(1)
        call()
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    t_begin = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local_rank)
    clocks.start()
    time.sleep(0.3)
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    clocks.mark_begin()
    t_begin.record(stream)
    for i in range(steps):
        if flush is not None:
            flush.fill_(1)
        starts[i].record(stream)
        call()
        ends[i].record(stream)
    t_end.record(stream)
    torch.cuda.synchronize(dev)
    clocks.mark_end()
    if world > 1:
        dist.barrier()
    time.sleep(0.1)
    clk = clocks.stop()
    status = npa.npa_device_status(stream)
    if status != npa.NPA_OK:
        raise RuntimeError(f"device status {npa.npa_status_string(status)}")
    kernel_ms = [a.elapsed_time(b) for a, b in zip(starts, ends)]
    elapsed_ms = t_begin.elapsed_time(t_end)
    return {"kernel_ms": kernel_ms, "timed_ms": sum(kernel_ms) if flush is not None else elapsed_ms,
            "clocks": clk}


def per_config_entry(prep, res: dict, pk: dict) -> dict:
    """One workload's figures for the ``per_config`` object of the line."""
    km = res["kernel_ms"]
    avg = sum(km) / len(km)
    tf = prep.flops / (avg * 1e-3) / 1e12
    return {
        "config": describe(prep.w),
        "ms": {"median": statistics.median(km), "best": min(km), "mean": avg},
        "useful_tflops": tf,
        "frac_of_burst": tf / pk["bf16_tflops"],
        "frac_of_sustained": tf / pk["bf16_tflops_sustained"],
        "useful_flops_per_call": prep.flops,
        "l2": "flushed (256 MB write) before every launch" if prep.flush is not None else "inputs larger than L2",
        "launches_per_call": prep.launches,
        "steps": len(km),
        "clocks": res["clocks"],
    }


def sample_parity(w: Workload, o, qs: np.ndarray, ref: np.ndarray) -> dict:
    """The timed call's output against the float64 oracle on the rows the CPU
    baseline computed (the same seeded inputs): max and mean absolute
    difference and relative L2, with the gates the tests use."""
    import torch
    rows = w.G if w.geometry == "gq" else w.H * w.W
    flat = o.reshape(-1, w.d)
    idx = torch.from_numpy((qs[:, 0].astype(np.int64) * w.heads + qs[:, 1]) * rows + qs[:, 2]).to(o.device)
    got = flat.index_select(0, idx).float().cpu().numpy().astype(np.float64)
    diff = np.abs(got - ref)
    m = {"rows": int(len(qs)), "max_abs": float(diff.max()), "mean_abs": float(diff.mean()),
         "rel_l2": float(np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-300))}
    m["within_gates"] = bool(np.isfinite(got).all() and m["max_abs"] <= 2e-2 and m["mean_abs"] <= 2e-3
                             and m["rel_l2"] <= 1e-2)
    m["gates"] = "max |d| <= 2e-2, mean |d| <= 2e-3, relative L2 <= 1e-2 against the float64 oracle"
    return m


# The other target workloads reported beside the headline one.
PER_CONFIG = ["tiny_npa", "pcpp_4x32_p0.3", "pcpp_8x16_p0.8", "npa_sdxl_2048", "npa_flux_4096"]


def run_ours(args, w: Workload, rank: int, world: int, local_rank: int) -> None:
    import torch
    import torch.distributed as dist
    import patch_res_diffusion_b200 as npa

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    prep = prepare(w, dev, args.flush_l2)
    inp, q, k, v, gk, gv, o, stream = prep.inp, prep.q, prep.k, prep.v, prep.gk, prep.gv, prep.o, prep.stream
    flops, bytes_io, flush, md_ws, md_bytes = prep.flops, prep.bytes_io, prep.flush, prep.md_ws, prep.md_bytes
    res = timed_steps(prep, args.steps, args.warmup, dev, world, local_rank)
    kernel_ms, clk = res["kernel_ms"], res["clocks"]
    kernel_ms_sum = sum(kernel_ms)
    timed_ms = max_over_ranks(res["timed_ms"], world, dev)
    value = whole_job_rate(world, flops, args.steps, timed_ms) / 1e12
    avg_kernel_ms = kernel_ms_sum / args.steps

    # End to end through host buffers: every step copies its inputs from pinned
    # host memory, runs the call and reads the output back. Steps are pipelined
    # over three streams with double-buffered device tensors, so step i+1's
    # upload overlaps step i's kernel and step i-1's download.
    e2e = None
    if not args.no_e2e and w.geometry in ("npa", "pcpp", "md"):
        hq, hk, hv = (x.to("cpu").pin_memory() for x in (q, k, v))
        hg = [x.to("cpu").pin_memory() for x in (gk, gv)] if w.G else []
        hos = [torch.empty(o.shape, dtype=o.dtype, pin_memory=True) for _ in range(2)]
        bufs = [(q, k, v, gk, gv, o)]
        bufs.append(tuple(torch.empty_like(x) if x is not None else None for x in (q, k, v, gk, gv, o)))
        h2d = sum(x.numel() * 2 for x in [hq, hk, hv] + hg)
        d2h = o.numel() * 2
        s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        ev_in = [torch.cuda.Event() for _ in range(2)]
        ev_k = [torch.cuda.Event() for _ in range(2)]
        ev_out = [torch.cuda.Event() for _ in range(2)]

        def e2e_steps(n):
            for i in range(n):
                b = i % 2
                bq, bk, bv, bgk, bgv, bo = bufs[b]
                with torch.cuda.stream(s_in):
                    if i >= 2:
                        s_in.wait_event(ev_k[b])
                    bq.copy_(hq, non_blocking=True)
                    bk.copy_(hk, non_blocking=True)
                    bv.copy_(hv, non_blocking=True)
                    if w.G:
                        bgk.copy_(hg[0], non_blocking=True)
                        bgv.copy_(hg[1], non_blocking=True)
                    ev_in[b].record(s_in)
                stream.wait_event(ev_in[b])
                if i >= 2:
                    stream.wait_event(ev_out[b])
                if w.geometry == "npa":
                    npa.npa_attention_fwd(bq, bk, bv, bo, w.B, w.heads, w.H, w.W, w.d, w.patch, w.margin, bgk, bgv,
                                          w.G, stream)
                elif w.geometry == "md":
                    npa.npa_multidiffusion_attention_fwd(bq, bk, bv, bo, w.B, w.heads, w.H, w.W, w.d, w.patch,
                                                         w.margin, md_ws[b], md_bytes, bgk, bgv, w.G, stream)
                else:
                    npa.pcpp_attention_fwd(bq, bk, bv, bo, w.B, w.heads, w.H, w.W, w.d, w.n_strips, w.p, bgk,
                                           bgv, w.G, stream)
                ev_k[b].record(stream)
                with torch.cuda.stream(s_out):
                    s_out.wait_event(ev_k[b])
                    hos[b].copy_(bo, non_blocking=True)
                    ev_out[b].record(s_out)

        e2e_steps(max(2, args.warmup))
        torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(s_in)
        e2e_steps(args.steps)
        s_out.wait_stream(stream)
        s_out.wait_stream(s_in)
        e1.record(s_out)
        torch.cuda.synchronize(dev)
        e_ms = e0.elapsed_time(e1)
        e_ms = max_over_ranks(e_ms, world, dev)
        e2e = {"value": whole_job_rate(world, flops, args.steps, e_ms) / 1e12, "unit": "TFLOP/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e_ms / args.steps,
               "pipelined": "upload / kernel / download on three streams, double-buffered"}
        status = npa.npa_device_status(stream)
        if status != npa.NPA_OK:
            raise RuntimeError(f"device status {npa.npa_status_string(status)}")

    # The other target workloads, timed the same way on this GPU (one process,
    # N = 1 only; the headline line stays on the requested workload).
    per_config = None
    if world == 1 and not args.no_per_config and w.name == DEFAULT_WORKLOAD:
        pk, _ = peaks()
        per_config = {}
        for name in PER_CONFIG:
            other = prepare(PRESETS[name], dev, args.flush_l2)
            per_config[name] = per_config_entry(other, timed_steps(other, args.steps, args.warmup, dev, 1,
                                                                   local_rank), pk)
            del other
            torch.cuda.empty_cache()

    if rank != 0:
        return
    pk, pk_kind = peaks()
    achieved = flops / (avg_kernel_ms * 1e-3) / 1e12
    roofline = {
        "bound": "tensor", "achieved": achieved, "peak": pk["bf16_tflops"], "unit": "TFLOP/s",
        "frac": achieved / pk["bf16_tflops"], "traffic": recorded_traffic(w.name),
        "peak_kind": f"{pk_kind} bf16 burst",
        "frac_of_sustained": achieved / pk["bf16_tflops_sustained"],
        "frac_of_datasheet_dense": achieved / DATASHEET_BF16_DENSE_TFLOPS,
        "kernel": {"md": KERNEL_NAME + " + md_combine_kernel (timed together: one call)",
                   "gq": KERNEL_NAME + " + gq_combine_kernel (timed together: one call)"}.get(w.geometry, KERNEL_NAME),
        "useful_flops_per_launch": flops,
        "avg_launch_ms": avg_kernel_ms,
        "hbm_min_bytes_per_launch": bytes_io,
    }
    cpu = None
    parity = None
    if not args.no_cpu_baseline and world == 1:
        cpu = oracle_rate(w, inp, args.cpu_seconds)
        cpu.pop("seconds", None)
        qs, ref = cpu.pop("last_sample")
        parity = sample_parity(w, o, qs, ref)
    cfg = describe(w)
    cfg["parallelism"] = f"replicas x{world}" if world > 1 else "single GPU"
    cfg["l2"] = ("flushed (256 MB write) between launches; value from per-launch events" if flush is not None
                 else f"inputs larger than L2 ({bytes_io / 2**20:.0f} MiB touched per launch)")
    line = {
        "metric": "patch-attention useful TFLOP/s (bf16) and % of B200 dense BF16 peak",
        "value": value,
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": timed_ms / args.steps,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic",
        "config": cfg,
        "roofline": roofline,
        "cpu_baseline": cpu,
        "e2e": e2e,
        "clocks": clk,
        "gpu_launches": args.steps * prep.launches,
        "kernel_ms": {"median": statistics.median(kernel_ms), "best": min(kernel_ms)},
    }
    if parity is not None:
        line["parity"] = parity
    if per_config is not None:
        line["per_config"] = per_config
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# ASG guidance combine (HBM-bound elementwise pass)
# ---------------------------------------------------------------------------
ASG_METRIC = "ASG guidance combine: algorithmic HBM bytes per second"


def asg_describe(w: AsgWorkload) -> dict:
    return {"workload": w.name, "n_patches": w.n_patches, "B": w.B, "C": w.C, "pixels_per_patch": w.S,
            "w_t": w.w_t, "algorithmic_bytes": w.algorithmic_bytes()}


def asg_oracle_rate(w: AsgWorkload, inp: dict, seconds: float) -> dict:
    """Times the float64 oracle on growing leading slices of the patches."""
    import oracle
    n, total_b, total_t = 1, 0, 0.0
    while total_t < seconds:
        k = min(n, w.n_patches)
        t0 = time.perf_counter()
        oracle.asg_guidance_combine(inp["eps"][:k], inp["ref"], inp["mask"][:k], w.w_t)
        total_t += time.perf_counter() - t0
        total_b += 2 * (2 * k * w.B * w.C * w.S + k * w.B * w.S + w.B * w.C * w.S)
        n *= 2
    return {"value": total_b / total_t / 1e9, "unit": "GB/s", "cores": 1, "kind": "oracle",
            "sample": f"leading patch slices of {w.name}, float64 NumPy, {total_t:.1f} s"}


def run_asg(args, w: AsgWorkload, rank: int, world: int, local_rank: int) -> None:
    import torch
    import torch.distributed as dist
    import patch_res_diffusion_b200 as npa

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    inp = make_asg_inputs(w)
    as_dev = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).to(dev).view(torch.bfloat16)
    eps, ref, mask = as_dev(inp["eps"]), as_dev(inp["ref"]), as_dev(inp["mask"])
    out = torch.empty_like(eps)
    stream = torch.cuda.current_stream(dev)
    nbytes = w.algorithmic_bytes()
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev) if nbytes < 2 * L2_BYTES else None

    def call(e=eps, r=ref, m=mask, o=out):
        npa.asg_guidance_combine(e, r, m, o, w.n_patches, w.B, w.C, w.S, w.w_t, stream)

    for _ in range(args.warmup):
        if flush is not None:
            flush.fill_(1)
        call()
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    clocks = ClockSampler(local_rank)
    clocks.start()
    time.sleep(0.3)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    t0.record(stream)
    for i in range(args.steps):
        if flush is not None:
            flush.fill_(1)
        starts[i].record(stream)
        call()
        ends[i].record(stream)
    t1.record(stream)
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    clk = clocks.stop()
    kernel_ms = [a.elapsed_time(b) for a, b in zip(starts, ends)]
    timed_ms = sum(kernel_ms) if flush is not None else t0.elapsed_time(t1)
    timed_ms = max_over_ranks(timed_ms, world, dev)
    value = whole_job_rate(world, nbytes, args.steps, timed_ms) / 1e9
    avg_ms = sum(kernel_ms) / args.steps

    e2e = None
    if not args.no_e2e:
        h_in = [x.to("cpu").pin_memory() for x in (eps, ref, mask)]
        h_out = torch.empty(out.shape, dtype=out.dtype, pin_memory=True)
        h2d = sum(x.numel() * 2 for x in h_in)
        d2h = out.numel() * 2

        def e2e_step():
            for hd, dv in zip(h_in, (eps, ref, mask)):
                dv.copy_(hd, non_blocking=True)
            call()
            h_out.copy_(out, non_blocking=True)

        for _ in range(2):
            e2e_step()
        torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(args.steps):
            e2e_step()
        b.record(stream)
        torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()
        e_ms = max_over_ranks(a.elapsed_time(b), world, dev)
        e2e = {"value": whole_job_rate(world, nbytes, args.steps, e_ms) / 1e9, "unit": "GB/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e_ms / args.steps}
    if rank != 0:
        return
    pk, pk_kind = peaks()
    achieved = nbytes / (avg_ms * 1e-3) / 1e9
    cfg = asg_describe(w)
    cfg["parallelism"] = f"replicas x{world}" if world > 1 else "single GPU"
    cfg["l2"] = ("flushed (256 MB write) between launches; value from per-launch events" if flush is not None
                 else f"inputs larger than L2 ({nbytes / 2**20:.0f} MiB per launch)")
    line = {
        "metric": ASG_METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": timed_ms / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16 in, f32 arithmetic", "data": "synthetic", "config": cfg,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": pk["hbm_gbs"], "unit": "GB/s",
                     "frac": achieved / pk["hbm_gbs"], "traffic": None, "peak_kind": f"{pk_kind} HBM copy",
                     "kernel": "asg_combine_kernel", "bytes_per_launch": nbytes, "avg_launch_ms": avg_ms},
        "cpu_baseline": None if args.no_cpu_baseline or world > 1 else asg_oracle_rate(w, inp, args.cpu_seconds),
        "e2e": e2e, "clocks": clk, "gpu_launches": args.steps,
        "kernel_ms": {"median": statistics.median(kernel_ms), "best": min(kernel_ms)},
    }
    print(json.dumps(line), flush=True)


def run_asg_reference(args, w: AsgWorkload, rank: int) -> None:
    if rank != 0:
        return
    inp = make_asg_inputs(w)
    budget = max(0.5, min(2.0 * args.cpu_seconds, 30.0) / max(1, args.steps + args.warmup))
    steps = [asg_oracle_rate(w, inp, budget) for _ in range(args.warmup + args.steps)][args.warmup:]
    value = statistics.median(r["value"] for r in steps)
    print(json.dumps({
        "impl": "reference", "metric": ASG_METRIC, "value": value, "unit": "GB/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": w.algorithmic_bytes() / (value * 1e9) * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": asg_describe(w),
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": 1, "kind": "oracle", "sample": steps[-1]["sample"]},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


def main():
    args = parse()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.workload in ASG_WORKLOADS:
        w = ASG_WORKLOADS[args.workload]
        if args.impl == "reference":
            run_asg_reference(args, w, rank)
            return
        run = run_asg
    else:
        w = preset(args.workload)
        if args.impl == "reference":
            run_reference(args, w, rank)
            return
        run = run_ours
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    try:
        run(args, w, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
