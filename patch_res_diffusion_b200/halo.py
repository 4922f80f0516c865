"""Neighbour exchange of PCPP's borrowed rows between devices.

Partially Conditioned Patch Parallelism (pith.science review), "Core claim"
and "What carries the argument": patch parallelism normally all-gathers the
previous step's activations; PCPP instead sends each device's boundary rows
to its two adjacent devices only, and a strip attends to its own rows plus
the p-fraction of each neighbour strip next to it, taken from the previous
step.

Layout used here (one process per GPU): every rank keeps full-size bf16
K and V buffers ``[B, heads, H*W, d]`` for the current step, of which it
computes only its own strips ``[begin, begin + count)``, and full-size
``k_stale`` / ``v_stale`` buffers. ``exchange_borrowed_rows`` sends the top
``r`` rows of the rank's first strip to the rank above and the bottom ``r``
rows of its last strip to the rank below, and writes what it receives into
``k_stale`` / ``v_stale`` at the same token positions. The next step's
attention for the rank's strips then reads those rows through
``pcpp_attention_fwd_stale`` (the own strips from the current buffers).

This module is host plumbing (``torch.distributed`` point-to-point
operations: NCCL over NVLink on GPUs, gloo on CPUs); it moves data and does no
attention arithmetic.
"""
from __future__ import annotations

from typing import List, Tuple

__all__ = ["strip_range", "neighbor_rows", "exchange_borrowed_rows", "exchange_bytes", "allgather_bytes"]


def neighbor_rows(strip_rows: int, p: float) -> int:
    """r = ceil(p * s) with a 1e-9 allowance, limited to [0, s] (same reading
    as the C library's pcpp_neighbor_rows)."""
    import math
    if strip_rows < 1 or not (0.0 <= p <= 1.0):
        raise ValueError("bad strip size or partial value")
    return max(0, min(strip_rows, int(math.ceil(p * strip_rows - 1e-9))))


def strip_range(n_strips: int, rank: int, world: int) -> Tuple[int, int]:
    """Contiguous share of the strips for ``rank``: (begin, count)."""
    if world < 1 or not 0 <= rank < world or n_strips < world:
        raise ValueError("need at least one strip per rank")
    base, extra = divmod(n_strips, world)
    begin = rank * base + min(rank, extra)
    return begin, base + (1 if rank < extra else 0)


def _rows(t, row0: int, nrows: int, W: int):
    """View of token rows [row0, row0 + nrows) of a [B, heads, H*W, d] tensor."""
    return t[:, :, row0 * W:(row0 + nrows) * W, :]


def exchange_borrowed_rows(k, v, k_stale, v_stale, H: int, W: int, n_strips: int, p: float, rank: int,
                           world: int, group=None) -> None:
    """Send this rank's boundary rows of k/v to its neighbours and receive
    theirs into k_stale / v_stale (blocking). Rows that one of the rank's
    strips borrows from another of its own strips are copied locally, so
    every borrowed row the next attention reads is the latest one available
    on this rank."""
    import torch
    import torch.distributed as dist

    s = H // n_strips
    r = neighbor_rows(s, p)
    if r == 0:
        return
    begin, count = strip_range(n_strips, rank, world)
    top, bottom = begin * s, (begin + count) * s          # this rank's first / one-past-last row
    for i in range(1, count):                             # boundaries between this rank's strips
        row = top + i * s
        for src, dst_stale in ((k, k_stale), (v, v_stale)):
            _rows(dst_stale, row - r, 2 * r, W).copy_(_rows(src, row - r, 2 * r, W))
    if world == 1:
        return
    ops: List[dist.P2POp] = []
    recv: List[Tuple[torch.Tensor, torch.Tensor]] = []
    for src, dst_stale in ((k, k_stale), (v, v_stale)):
        if rank > 0:   # exchange with the rank above
            send = _rows(src, top, r, W).contiguous()
            buf = torch.empty_like(send)
            ops.append(dist.P2POp(dist.isend, send, rank - 1, group))
            ops.append(dist.P2POp(dist.irecv, buf, rank - 1, group))
            recv.append((buf, _rows(dst_stale, top - r, r, W)))
        if rank < world - 1:  # exchange with the rank below
            send = _rows(src, bottom - r, r, W).contiguous()
            buf = torch.empty_like(send)
            ops.append(dist.P2POp(dist.isend, send, rank + 1, group))
            ops.append(dist.P2POp(dist.irecv, buf, rank + 1, group))
            recv.append((buf, _rows(dst_stale, bottom, r, W)))
    for work in dist.batch_isend_irecv(ops):
        work.wait()
    for buf, dst in recv:
        dst.copy_(buf)


def exchange_bytes(B: int, heads: int, H: int, W: int, d: int, n_strips: int, p: float, world: int,
                   elem_bytes: int = 2) -> int:
    """Bytes all ranks send per exchange: K and V, r rows to each neighbour."""
    r = neighbor_rows(H // n_strips, p)
    return 2 * (world - 1) * 2 * r * W * B * heads * d * elem_bytes


def allgather_bytes(B: int, heads: int, H: int, W: int, d: int, world: int, elem_bytes: int = 2) -> int:
    """Bytes all ranks receive when every rank all-gathers the full K and V
    (the patch-parallel baseline PCPP replaces): each receives the other
    ranks' shares."""
    full = B * heads * H * W * d * elem_bytes
    return 2 * world * (full * (world - 1) // world)
