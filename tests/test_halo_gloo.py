"""Multi-rank PCPP on the CPU (gloo, world size 2 to 4, even and uneven
strip shares): each rank owns a range of strips, exchanges its boundary rows
with its neighbours, and runs the two-source oracle for its strips.
Exchanging the current step's rows and using them at once is the synchronous
limit, so the ranks' outputs must equal the single-process single-source PCPP
oracle exactly."""
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import oracle
from patch_res_diffusion_b200 import halo
from workloads import Workload, make_inputs


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, w, out_path):
    import torch.distributed as dist
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    try:
        inp = make_inputs(w)
        s = w.H // w.n_strips
        begin, count = halo.strip_range(w.n_strips, rank, world)
        as_t = lambda a: torch.from_numpy(a.view(np.int16).copy())
        k, v = as_t(inp["k"]), as_t(inp["v"])
        # this rank only holds its own strips' rows; the rest is garbage
        own = np.zeros(w.H * w.W, dtype=bool)
        own[begin * s * w.W:(begin + count) * s * w.W] = True
        for t in (k, v):
            t[:, :, torch.from_numpy(~own)] = 12345
        k_stale = torch.full_like(k, -777)
        v_stale = torch.full_like(v, -777)
        halo.exchange_borrowed_rows(k, v, k_stale, v_stale, w.H, w.W, w.n_strips, w.p, rank, world)
        to_np = lambda t: t.numpy().view(np.uint16)
        rows = np.arange(w.H * w.W)[own]
        qs = np.array([(b, h, t) for b in range(w.B) for h in range(w.heads) for t in rows], dtype=np.int32)
        got = oracle.pcpp_attention_stale(inp["q"], to_np(k), to_np(v), to_np(k_stale), to_np(v_stale),
                                          B=w.B, heads=w.heads, H=w.H, W=w.W, d=w.d, n_strips=w.n_strips,
                                          p=w.p, queries=qs)
        np.save(f"{out_path}.{rank}.npy", got)
        np.save(f"{out_path}.{rank}.q.npy", qs)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,w", [
    (2, Workload("halo_2", "pcpp", B=1, heads=2, H=16, W=6, d=16, n_strips=4, p=0.5)),
    (3, Workload("halo_3", "pcpp", B=2, heads=1, H=18, W=5, d=16, n_strips=6, p=0.4)),
    (2, Workload("halo_p1", "pcpp", B=1, heads=1, H=12, W=4, d=16, n_strips=2, p=1.0)),
    # uneven share: 6 strips over 4 ranks hold 2, 2, 1, 1 strips
    (4, Workload("halo_uneven", "pcpp", B=1, heads=2, H=24, W=4, d=16, n_strips=6, p=0.5)),
], ids=lambda x: x if isinstance(x, int) else x.name)
def test_exchange_then_attend_equals_synchronous_pcpp(tmp_path, world, w):
    oracle.lib()  # build before the workers start
    out = str(tmp_path / "o")
    mp.start_processes(_worker, args=(world, _free_port(), w, out), nprocs=world, start_method="spawn")
    inp = make_inputs(w)
    ref = oracle.pcpp_attention(inp["q"], inp["k"], inp["v"], B=w.B, heads=w.heads, H=w.H, W=w.W, d=w.d,
                                n_strips=w.n_strips, p=w.p)
    covered = 0
    for rank in range(world):
        got = np.load(f"{out}.{rank}.npy")
        qs = np.load(f"{out}.{rank}.q.npy")
        np.testing.assert_array_equal(got, ref[qs[:, 0], qs[:, 1], qs[:, 2]])
        covered += len(qs)
    assert covered == w.B * w.heads * w.H * w.W


def test_strip_ranges_partition():
    for n, world in [(4, 2), (6, 4), (8, 8), (5, 2)]:
        ranges = [halo.strip_range(n, r, world) for r in range(world)]
        assert ranges[0][0] == 0 and sum(c for _, c in ranges) == n
        for (b0, c0), (b1, _) in zip(ranges, ranges[1:]):
            assert b0 + c0 == b1
    with pytest.raises(ValueError):
        halo.strip_range(2, 0, 3)


def test_exchange_volume_vs_allgather():
    """Borrowed-row exchange moves far less than an all-gather of K and V:
    SDXL 2048^2 attention shape, 4 strips at p = 0.3 (10 rows)."""
    ex = halo.exchange_bytes(2, 10, 128, 128, 64, 4, 0.3, 4)
    ag = halo.allgather_bytes(2, 10, 128, 128, 64, 4)
    assert ex == 2 * 3 * 2 * 10 * 128 * 2 * 10 * 64 * 2
    assert ex / ag < 0.2
