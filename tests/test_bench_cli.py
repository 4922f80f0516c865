"""bench.py's launcher contract on the CPU: the reference arm (the oracle on
the host cores) under torchrun with two ranks prints exactly one JSON line
from rank 0 and every rank exits 0; the replicas' timing reduction (slowest
rank, whole-job rate) agrees on every rank under gloo."""
import json
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_reference_arm_under_torchrun_two_ranks():
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(_port()), "bench.py", "--impl", "reference",
           "--gpus", "2", "--steps", "2", "--warmup", "1", "--workload", "tiny_npa", "--cpu-seconds", "1"]
    res = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert res.returncode == 0, res.stderr[-2000:]
    lines = [l for l in res.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "TFLOP/s" and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["e2e"]["h2d_bytes_per_step"] == 0
    assert d["config"]["workload"] == "tiny_npa" and d["n_gpus"] == 2


def _rank_timing(rank, world, port, out):
    import torch.distributed as dist
    import bench
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    try:
        ms = [12.5, 20.0, 7.25][rank]
        slowest = bench.max_over_ranks(ms, world, "cpu")
        with open(f"{out}.{rank}", "w") as f:
            f.write(repr((slowest, bench.whole_job_rate(world, 1e12, 10, slowest))))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_max_over_ranks_and_whole_job_rate_gloo(tmp_path, world):
    """The multi-GPU bench (one replica per rank) reports the slowest rank's
    time and the whole job's units over it; every rank must agree."""
    import torch.multiprocessing as mp
    out = str(tmp_path / "r")
    mp.start_processes(_rank_timing, args=(world, _port(), out), nprocs=world, start_method="spawn")
    import ast
    results = [ast.literal_eval(open(f"{out}.{r}").read()) for r in range(world)]
    slowest = max([12.5, 20.0, 7.25][:world])
    for got_ms, rate in results:
        assert got_ms == slowest
        assert rate == world * 1e12 * 10 / (slowest * 1e-3)


def test_sample_parity_indexes_the_sampled_rows():
    """bench.sample_parity gathers output rows (b, h, t) of a [B, heads, N, d]
    tensor and compares them with oracle rows; checked on the CPU with the
    oracle's own full output rounded to bf16 (within the gates) and with one
    sampled row planted wrong (outside them)."""
    import numpy as np
    import torch
    import bench
    import oracle
    from workloads import Workload, make_inputs
    w = Workload("cpu_tiny", "npa", B=2, heads=3, H=8, W=6, d=64, patch=4, margin=2)
    inp = make_inputs(w)
    full = oracle.npa_attention(inp["q"], inp["k"], inp["v"], B=w.B, heads=w.heads, H=w.H, W=w.W, d=w.d,
                                patch=w.patch, margin=w.margin)
    o = torch.from_numpy(full).to(torch.bfloat16)
    rng = np.random.default_rng(0)
    qs = np.stack([rng.integers(w.B, size=40), rng.integers(w.heads, size=40), rng.integers(w.H * w.W, size=40)],
                  1).astype(np.int32)
    ref = np.stack([full[b, h, t] for b, h, t in qs])
    m = bench.sample_parity(w, o, qs, ref)
    assert m["rows"] == 40 and m["within_gates"] and m["rel_l2"] < 1e-2
    b, h, t = qs[7]
    o[b, h, t] += 0.5
    assert not bench.sample_parity(w, o, qs, ref)["within_gates"]
