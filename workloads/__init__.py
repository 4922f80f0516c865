"""Seeded synthetic inputs and the named workload presets.

This module is shared by the tests, the benchmark and the oracle harness. It
draws random numbers and rounds them to bfloat16; it holds none of the
attention method's arithmetic (no windows, no softmax, no flop counts).

Recipe (the same bits go to the CPU oracle and to the GPU):
  * generator: NumPy PCG64, ``default_rng(seed + tensor_index)`` with tensor
    index q=0, k=1, v=2, global k=3, global v=4;
  * draws: float64 standard normal N(0, 1);
  * optional spatial smoothing of k (the "NPA SDXL 2048^2" workload): a 3x3
    box filter over the token grid, per (batch, head, channel), taking the
    mean over the in-bounds neighbours, in float64, before rounding;
  * rounding: float64 -> bfloat16, round to nearest, ties to even, done in
    one step on the float64 bits (no float32 intermediate, so no double
    rounding).

Tensors are returned as ``uint16`` arrays holding bfloat16 bit patterns in the
layout ``[B, heads, H*W, d]`` (token index ``t = row*W + col``) and, for the
global tokens, ``[B, heads, G, d]``.
"""
from __future__ import annotations

import dataclasses
from typing import Dict, Optional

import numpy as np

__all__ = [
    "Workload", "PRESETS", "COMPARATORS", "preset", "AsgWorkload", "ASG_WORKLOADS", "make_asg_inputs", "f64_to_bf16_bits", "bf16_bits_to_f64",
    "make_inputs", "box_filter_3x3",
]


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic attention workload.

    ``geometry`` is ``"npa"`` (square query patches of side ``patch`` with a
    K/V window grown by ``margin`` and clipped to the grid), ``"pcpp"``
    (``n_strips`` row strips, each also seeing the nearest rows of its
    adjacent strips, the count set by the partial value ``p``), ``"md"`` (the
    overlapping-window comparator: every NPA window attends within itself,
    outputs averaged over the windows containing a token), ``"pcpp_stale"``
    (PCPP with the borrowed rows read from a second, previous-step K/V) or
    ``"gq"`` (the G global tokens as queries over all image and global keys).
    """

    name: str
    geometry: str
    B: int
    heads: int
    H: int
    W: int
    d: int
    patch: int = 0
    margin: int = 0
    n_strips: int = 0
    p: float = 0.0
    G: int = 0
    smooth_k: bool = False
    seed: int = 0

    @property
    def n_tokens(self) -> int:
        return self.H * self.W

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


# The five workloads the throughput and parity targets are stated on, plus the
# strip/partial-value pairings the PCPP review page implies once classifier-free
# guidance halves the device count (p=0.3 with 2 strips, p=0.8 with 4 strips).
PRESETS: Dict[str, Workload] = {
    w.name: w
    for w in [
        Workload("tiny_npa", "npa", B=1, heads=2, H=16, W=16, d=64, patch=8, margin=4),
        Workload("pcpp_4x32_p0.3", "pcpp", B=2, heads=10, H=128, W=128, d=64, n_strips=4, p=0.3),
        Workload("pcpp_8x16_p0.8", "pcpp", B=2, heads=10, H=128, W=128, d=64, n_strips=8, p=0.8),
        Workload("npa_sdxl_2048", "npa", B=2, heads=10, H=128, W=128, d=64, patch=64, margin=32,
                 smooth_k=True),
        Workload("npa_sdxl_4096", "npa", B=2, heads=10, H=256, W=256, d=64, patch=64, margin=32),
        Workload("npa_flux_4096", "npa", B=1, heads=24, H=256, W=256, d=128, patch=64, margin=32,
                 G=512),
        # pages' pairing of the partial value with the strip count
        Workload("pcpp_2x64_p0.3", "pcpp", B=2, heads=10, H=128, W=128, d=64, n_strips=2, p=0.3),
        Workload("pcpp_4x32_p0.8", "pcpp", B=2, heads=10, H=128, W=128, d=64, n_strips=4, p=0.8),
    ]
}


# Workloads of the later rows (not the throughput targets): the
# overlapping-window comparator on the SDXL 4096^2 attention shape, PCPP with
# stale neighbour rows on the PCPP 4x32 shape, and the text-query half of FLUX
# 4096^2 joint attention.
COMPARATORS: Dict[str, Workload] = {
    w.name: w
    for w in [
        Workload("md_sdxl_4096", "md", B=2, heads=10, H=256, W=256, d=64, patch=64, margin=32),
        Workload("pcpp_stale_4x32_p0.3", "pcpp_stale", B=2, heads=10, H=128, W=128, d=64, n_strips=4, p=0.3),
        Workload("gq_flux_4096", "gq", B=1, heads=24, H=256, W=256, d=128, G=512),
    ]
}


def preset(name: str) -> Workload:
    return PRESETS[name] if name in PRESETS else COMPARATORS[name]


def f64_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float64 values to bfloat16 (nearest, ties to even) in one step.

    Works on the float64 bit pattern: the 52-bit mantissa is rounded to the 7
    bits bfloat16 keeps, then the (exactly representable) result is narrowed
    to float32, whose top half is the bfloat16 pattern. Valid for finite values
    whose magnitude lies in the float32 normal range or is zero; that is every
    draw this module makes (|x| below 2^-126 has probability ~1e-38).
    """
    x = np.ascontiguousarray(x, dtype=np.float64)
    if not np.all(np.isfinite(x)):
        raise ValueError("non-finite input")
    ax = np.abs(x)
    if np.any((ax != 0) & ((ax < 2.0 ** -126) | (ax >= 2.0 ** 127))):
        raise ValueError("value outside the bfloat16 normal range")
    u = x.view(np.uint64)
    drop = np.uint64(45)  # 52 mantissa bits - 7 kept
    lsb = (u >> drop) & np.uint64(1)
    u = (u + (np.uint64(1) << np.uint64(44)) - np.uint64(1) + lsb) & ~((np.uint64(1) << drop) - np.uint64(1))
    f32 = u.view(np.float64).astype(np.float32)  # exact: 8 significant bits
    return (f32.view(np.uint32) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f64(b: np.ndarray) -> np.ndarray:
    """Exact widening of bfloat16 bit patterns to float64."""
    b = np.ascontiguousarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def box_filter_3x3(x: np.ndarray, H: int, W: int) -> np.ndarray:
    """Mean over the in-bounds 3x3 neighbourhood of every token, per channel.

    ``x`` is float64 ``[..., H*W, d]``; the result has the same shape.
    """
    lead = x.shape[:-2]
    d = x.shape[-1]
    g = x.reshape(lead + (H, W, d))
    acc = np.zeros_like(g)
    cnt = np.zeros((H, W), dtype=np.float64)
    for dr in (-1, 0, 1):
        for dc in (-1, 0, 1):
            r0, r1 = max(0, -dr), min(H, H - dr)
            c0, c1 = max(0, -dc), min(W, W - dc)
            acc[..., r0:r1, c0:c1, :] += g[..., r0 + dr:r1 + dr, c0 + dc:c1 + dc, :]
            cnt[r0:r1, c0:c1] += 1.0
    return (acc / cnt[:, :, None]).reshape(x.shape)


def _normal(seed: int, shape) -> np.ndarray:
    return np.random.default_rng(seed).standard_normal(shape, dtype=np.float64)


def make_inputs(w: Workload, seed: Optional[int] = None) -> Dict[str, np.ndarray]:
    """Draw the q, k, v (and global gk, gv) tensors of a workload as bf16
    bits; stale-row PCPP adds ks, vs and the global-query form adds gq."""
    s = w.seed if seed is None else seed
    shape = (w.B, w.heads, w.n_tokens, w.d)
    out: Dict[str, np.ndarray] = {}
    out["q"] = f64_to_bf16_bits(_normal(s + 0, shape))
    kf = _normal(s + 1, shape)
    if w.smooth_k:
        kf = box_filter_3x3(kf, w.H, w.W)
    out["k"] = f64_to_bf16_bits(kf)
    del kf
    out["v"] = f64_to_bf16_bits(_normal(s + 2, shape))
    if w.G > 0:
        gshape = (w.B, w.heads, w.G, w.d)
        out["gk"] = f64_to_bf16_bits(_normal(s + 3, gshape))
        out["gv"] = f64_to_bf16_bits(_normal(s + 4, gshape))
    if w.geometry == "pcpp_stale":  # the previous step's keys / values
        out["ks"] = f64_to_bf16_bits(_normal(s + 5, shape))
        out["vs"] = f64_to_bf16_bits(_normal(s + 6, shape))
    if w.geometry == "gq":  # the global tokens' own queries
        out["gq"] = f64_to_bf16_bits(_normal(s + 7, (w.B, w.heads, w.G, w.d)))
    return out


@dataclasses.dataclass(frozen=True)
class AsgWorkload:
    """One synthetic ASG guidance-combine workload: ``n_patches`` latent
    patches of ``S`` pixels and ``C`` channels for ``B`` batch elements, one
    reference patch, one mask per patch, weight ``w_t``."""

    name: str
    n_patches: int
    B: int
    C: int
    S: int
    w_t: float = 0.8
    seed: int = 0

    @property
    def elements(self) -> int:
        return self.n_patches * self.B * self.C * self.S

    def algorithmic_bytes(self) -> int:
        """eps read and out written once, the mask read once, the reference once."""
        return 2 * (2 * self.elements + self.n_patches * self.B * self.S + self.B * self.C * self.S)


# SDXL at 4096^2: a 512^2 x 4 latent cut into 16 patches of the model's
# native 128^2 latent size, classifier-free guidance batch 2. The bulk case
# streams ~1.2 GB through the same kernel to measure its bandwidth.
ASG_WORKLOADS: Dict[str, AsgWorkload] = {
    w.name: w
    for w in [
        AsgWorkload("asg_sdxl_4096", n_patches=16, B=2, C=4, S=128 * 128),
        AsgWorkload("asg_bulk", n_patches=16, B=8, C=16, S=256 * 256),
    ]
}


def make_asg_inputs(w: AsgWorkload) -> Dict[str, np.ndarray]:
    """eps and the reference ~ N(0, 1), the mask ~ U[0, 1), as bf16 bits (seeds
    seed + 0, 1, 2)."""
    eps = f64_to_bf16_bits(_normal(w.seed, (w.n_patches, w.B, w.C, w.S)))
    ref = f64_to_bf16_bits(_normal(w.seed + 1, (w.B, w.C, w.S)))
    mask = f64_to_bf16_bits(np.random.default_rng(w.seed + 2).uniform(0.0, 1.0, (w.n_patches, w.B, w.S)))
    return {"eps": eps, "ref": ref, "mask": mask}
