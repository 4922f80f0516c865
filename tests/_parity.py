"""Helpers shared by the GPU parity tests: device transfer, the comparison
gates and the query sets used at full workload sizes."""
from __future__ import annotations

import numpy as np

import oracle
from workloads import Workload

# Parity gates on bf16 outputs against the float64 oracle. The first two are
# the stated acceptance bounds; the relative L2 gate is tighter because with
# N(0,1) inputs the outputs themselves are only ~1e-2 in size at 128x128
# windows, so the absolute bounds alone would not catch a shifted window.
MAX_ABS = 2e-2
MEAN_ABS = 2e-3
REL_L2 = 1e-2


def to_device(bits: np.ndarray, device="cuda"):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16))
    return t.to(device).view(torch.bfloat16)


def to_f64(t) -> np.ndarray:
    import torch
    return t.detach().to("cpu").contiguous().view(torch.int16).numpy().view(np.uint16).astype(np.uint32) \
        .__lshift__(16).view(np.float32).astype(np.float64)


def run_gpu(w: Workload, inp: dict, *, margin=None, p=None, stream=None):
    """Runs the library on a workload's inputs; returns the output tensor (bf16, device)."""
    import torch
    import patch_res_diffusion_b200 as npa
    q, k, v = (to_device(inp[n]) for n in ("q", "k", "v"))
    gk = to_device(inp["gk"]) if w.G else None
    gv = to_device(inp["gv"]) if w.G else None
    o = torch.full_like(q, float("nan"))
    if w.geometry == "npa":
        npa.npa_attention(q, k, v, w.H, w.W, w.patch, w.margin if margin is None else margin, gk, gv, out=o,
                          stream=stream)
    else:
        npa.pcpp_attention(q, k, v, w.H, w.W, w.n_strips, w.p if p is None else p, gk, gv, out=o, stream=stream)
    return o


def run_oracle(w: Workload, inp: dict, queries=None, **override):
    geom = dict(patch=w.patch, margin=w.margin) if w.geometry == "npa" else dict(n_strips=w.n_strips, p=w.p)
    geom.update(override)
    fn = oracle.npa_attention if w.geometry == "npa" else oracle.pcpp_attention
    return fn(inp["q"], inp["k"], inp["v"], gk=inp.get("gk"), gv=inp.get("gv"), G=w.G, B=w.B, heads=w.heads,
              H=w.H, W=w.W, d=w.d, queries=queries, **geom)


def compare(got: np.ndarray, ref: np.ndarray) -> dict:
    diff = np.abs(got - ref)
    return {
        "max_abs": float(diff.max()),
        "mean_abs": float(diff.mean()),
        "rel_l2": float(np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-300)),
        "finite": bool(np.isfinite(got).all()),
    }


def log_metrics(name: str, m: dict) -> None:
    """Appends the comparison to the file named by NPA_PARITY_LOG, if set."""
    import json
    import os
    path = os.environ.get("NPA_PARITY_LOG")
    if path:
        with open(path, "a") as f:
            f.write(json.dumps({"case": name, **m}) + "\n")


def passes(m: dict) -> bool:
    return m["finite"] and m["max_abs"] <= MAX_ABS and m["mean_abs"] <= MEAN_ABS and m["rel_l2"] <= REL_L2


def sample_queries(w: Workload, n_random: int = 512, seed: int = 0, max_bh: int = None) -> np.ndarray:
    """Deterministic query sample: for every (b, h) (or the first ``max_bh``),
    the four corner tokens of every patch or strip, plus ``n_random`` uniform
    (b, h, t) triples."""
    rng = np.random.default_rng(seed)
    if w.geometry == "npa":
        r_starts = list(range(0, w.H, w.patch))
        c_starts = list(range(0, w.W, w.patch))
        spans = [(r0, min(w.H, r0 + w.patch), c0, min(w.W, c0 + w.patch)) for r0 in r_starts for c0 in c_starts]
    else:
        s = w.H // w.n_strips
        spans = [(i * s, (i + 1) * s, 0, w.W) for i in range(w.n_strips)]
    bhs = [(b, h) for b in range(w.B) for h in range(w.heads)]
    if max_bh is not None:
        bhs = bhs[:max_bh]
    out = []
    for b, h in bhs:
        for r0, r1, c0, c1 in spans:
            for r, c in ((r0, c0), (r0, c1 - 1), (r1 - 1, c0), (r1 - 1, c1 - 1)):
                out.append((b, h, r * w.W + c))
    N = w.H * w.W
    for _ in range(n_random):
        out.append((int(rng.integers(w.B)), int(rng.integers(w.heads)), int(rng.integers(N))))
    return np.array(out, dtype=np.int32)


def patch_edge_queries(w: Workload, random_frac: float = 0.01, seed: int = 0) -> np.ndarray:
    """Query set for the workloads too large for a full oracle run: for every
    (b, h) and every patch, the patch's first 128 and last 128 queries in
    row-major order within the patch (its first and last query tile), plus
    ``random_frac`` of all (b, h, t) rows drawn uniformly without
    replacement. Returns an (n, 3) int32 array of (b, h, t), unique rows."""
    rng = np.random.default_rng(seed)
    N = w.H * w.W
    per_patch = []
    for r0 in range(0, w.H, w.patch):
        for c0 in range(0, w.W, w.patch):
            rows = np.arange(r0, min(w.H, r0 + w.patch))
            cols = np.arange(c0, min(w.W, c0 + w.patch))
            toks = (rows[:, None] * w.W + cols[None, :]).ravel()   # row-major within the patch
            per_patch.append(np.unique(np.concatenate([toks[:128], toks[-128:]])))
    toks = np.concatenate(per_patch)
    bh = np.arange(w.B * w.heads)
    flat = (bh[:, None].astype(np.int64) * N + toks[None, :]).ravel()
    n_rand = int(np.ceil(random_frac * w.B * w.heads * N))
    flat = np.unique(np.concatenate([flat, rng.choice(w.B * w.heads * N, size=n_rand, replace=False)]))
    return np.stack([flat // (w.heads * N), (flat // N) % w.heads, flat % N], axis=1).astype(np.int32)


def gather_rows(o, w: Workload, qs: np.ndarray) -> np.ndarray:
    """Rows (b, h, t) of a device output [B, heads, N, d], as float64."""
    import torch
    flat = o.reshape(w.B * w.heads * w.H * w.W, w.d)
    idx = torch.from_numpy((qs[:, 0].astype(np.int64) * w.heads + qs[:, 1]) * (w.H * w.W) + qs[:, 2])
    return to_f64(flat.index_select(0, idx.to(o.device)))
