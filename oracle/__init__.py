"""CPU oracle for patch-restricted self-attention (float64).

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, by ``__graft_entry__.smoke``
and by the benchmark's CPU-baseline leg. The library's compute path never
imports it, and it shares no code with the CUDA sources.

Two independent formulations of the same definition:

* :func:`npa_attention` / :func:`pcpp_attention` call the C gather oracle
  (``npa_oracle.c``): per query, build the key set from the definition, gather,
  softmax in double. OpenMP over queries only.
* :func:`dense_attention` builds the full ``[N, N+G]`` membership mask from a
  coordinate predicate and applies a masked softmax with NumPy, float64. It is
  only meant for small grids (up to ~64x64 tokens).

Definitions followed (see ``npa_oracle.c`` for the readings taken where the
pages are silent):
  * NPA: ScaleDiff (atlas.scime.ai summary), "Approach": non-overlapping query
    patches, each attending to an overlapping K/V neighbourhood (patch grown by
    a margin, clipped to the grid).
  * PCPP: Partially Conditioned Patch Parallelism (pith.science review), "What
    carries the argument" / "Core claim": a strip attends to itself plus the
    p-fraction of each adjacent strip's height next to it.
"""
from __future__ import annotations

import ctypes
from typing import Optional, Sequence

import numpy as np

from . import build as _build

__all__ = [
    "lib", "npa_key_set", "pcpp_key_set", "pcpp_neighbor_rows", "npa_attention",
    "pcpp_attention", "pcpp_attention_stale", "pair_count", "num_threads", "dense_mask",
    "dense_attention", "dense_pcpp_stale", "global_query_attention", "bf16_to_f64",
    "multidiffusion_attention", "md_window_keys", "md_window_count", "md_pair_count",
    "asg_guidance_combine",
]

_LIB = None


def lib() -> ctypes.CDLL:
    global _LIB
    if _LIB is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        i32p = ctypes.POINTER(ctypes.c_int32)
        u16p = ctypes.c_void_p
        L.oracle_npa_key_set.argtypes = [ctypes.c_int] * 5 + [i32p]
        L.oracle_npa_key_set.restype = ctypes.c_int
        L.oracle_pcpp_key_set.argtypes = [ctypes.c_int] * 3 + [ctypes.c_double, ctypes.c_int, i32p]
        L.oracle_pcpp_key_set.restype = ctypes.c_int
        L.oracle_pcpp_neighbor_rows.argtypes = [ctypes.c_int, ctypes.c_double]
        L.oracle_pcpp_neighbor_rows.restype = ctypes.c_int
        common = [u16p] * 5 + [ctypes.c_void_p] + [ctypes.c_int] * 5
        L.oracle_npa_attention.argtypes = common + [ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                                    ctypes.c_void_p, ctypes.c_long]
        L.oracle_npa_attention.restype = ctypes.c_int
        L.oracle_pcpp_attention.argtypes = common + [ctypes.c_int, ctypes.c_double, ctypes.c_int,
                                                     ctypes.c_void_p, ctypes.c_long]
        L.oracle_pcpp_attention.restype = ctypes.c_int
        L.oracle_pcpp_attention_stale.argtypes = [u16p] * 7 + [ctypes.c_void_p] + [ctypes.c_int] * 5 + [
            ctypes.c_int, ctypes.c_double, ctypes.c_int, ctypes.c_void_p, ctypes.c_long]
        L.oracle_pcpp_attention_stale.restype = ctypes.c_int
        L.oracle_global_query_attention.argtypes = [u16p] * 5 + [ctypes.c_void_p] + [ctypes.c_int] * 6 + [
            ctypes.c_void_p, ctypes.c_long]
        L.oracle_global_query_attention.restype = ctypes.c_int
        L.oracle_multidiffusion_attention.argtypes = common + [ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                                               ctypes.c_void_p, ctypes.c_long]
        L.oracle_multidiffusion_attention.restype = ctypes.c_int
        L.oracle_md_window_keys.argtypes = [ctypes.c_int] * 6 + [i32p]
        L.oracle_md_window_keys.restype = ctypes.c_int
        L.oracle_md_window_count.argtypes = [ctypes.c_int] * 5
        L.oracle_md_window_count.restype = ctypes.c_int
        L.oracle_md_pair_count.argtypes = [ctypes.c_int] * 5
        L.oracle_md_pair_count.restype = ctypes.c_longlong
        L.oracle_pair_count.argtypes = [ctypes.c_int] * 5 + [ctypes.c_double, ctypes.c_int]
        L.oracle_pair_count.restype = ctypes.c_longlong
        L.oracle_num_threads.argtypes = []
        L.oracle_num_threads.restype = ctypes.c_int
        _LIB = L
    return _LIB


def num_threads() -> int:
    return int(lib().oracle_num_threads())


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bfloat16 bit patterns to float64."""
    b = np.ascontiguousarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def npa_key_set(H: int, W: int, P: int, m: int, t: int) -> np.ndarray:
    buf = np.empty(H * W, dtype=np.int32)
    n = lib().oracle_npa_key_set(H, W, P, m, t, buf.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)))
    if n < 0:
        raise ValueError("bad NPA key-set arguments")
    return buf[:n].copy()


def pcpp_key_set(H: int, W: int, n_strips: int, p: float, t: int) -> np.ndarray:
    buf = np.empty(H * W, dtype=np.int32)
    n = lib().oracle_pcpp_key_set(H, W, n_strips, float(p), t,
                                  buf.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)))
    if n < 0:
        raise ValueError("bad PCPP key-set arguments")
    return buf[:n].copy()


def pcpp_neighbor_rows(strip_rows: int, p: float) -> int:
    return int(lib().oracle_pcpp_neighbor_rows(strip_rows, float(p)))


def pair_count(geometry: str, H: int, W: int, *, patch: int = 0, margin: int = 0,
               n_strips: int = 0, p: float = 0.0, G: int = 0) -> int:
    """Sum over all queries of one (b, h) of the key-set size (image + global)."""
    g = 0 if geometry == "npa" else 1
    a = patch if g == 0 else n_strips
    b = margin if g == 0 else 0
    n = lib().oracle_pair_count(g, H, W, a, b, float(p), G)
    if n < 0:
        raise ValueError("bad geometry")
    return int(n)


def _u16(x: Optional[np.ndarray]):
    if x is None:
        return None, None
    a = np.ascontiguousarray(x, dtype=np.uint16)
    return a, a.ctypes.data_as(ctypes.c_void_p)


def _call(fn, geometry_args, q, k, v, gk, gv, B, heads, H, W, d, G, queries):
    q, qp = _u16(q)
    k, kp = _u16(k)
    v, vp = _u16(v)
    gk, gkp = _u16(gk)
    gv, gvp = _u16(gv)
    if queries is None:
        out = np.empty((B, heads, H * W, d), dtype=np.float64)
        qs_p, nq = None, 0
    else:
        qs = np.ascontiguousarray(np.asarray(queries, dtype=np.int32).reshape(-1, 3))
        out = np.empty((qs.shape[0], d), dtype=np.float64)
        qs_p, nq = qs.ctypes.data_as(ctypes.c_void_p), qs.shape[0]
    rc = fn(qp, kp, vp, gkp, gvp, out.ctypes.data_as(ctypes.c_void_p), B, heads, H, W, d,
            *geometry_args, G, qs_p, nq)
    if rc != 0:
        raise RuntimeError(f"oracle failed with code {rc}")
    return out


def npa_attention(q, k, v, *, B, heads, H, W, d, patch, margin, gk=None, gv=None, G=0,
                  queries: Optional[Sequence] = None) -> np.ndarray:
    """NPA attention in float64. ``queries``: optional (n, 3) array of (b, h, t)."""
    return _call(lib().oracle_npa_attention, (patch, margin), q, k, v, gk, gv, B, heads, H, W, d,
                 G, queries)


def pcpp_attention(q, k, v, *, B, heads, H, W, d, n_strips, p, gk=None, gv=None, G=0,
                   queries: Optional[Sequence] = None) -> np.ndarray:
    """PCPP attention in float64. ``queries``: optional (n, 3) array of (b, h, t)."""
    return _call(lib().oracle_pcpp_attention, (n_strips, float(p)), q, k, v, gk, gv, B, heads, H,
                 W, d, G, queries)


def multidiffusion_attention(q, k, v, *, B, heads, H, W, d, patch, margin, gk=None, gv=None, G=0,
                             queries: Optional[Sequence] = None) -> np.ndarray:
    """Overlapping-window (MultiDiffusion-style) attention in float64: every
    NPA window attends within itself; a token's output is the mean over the
    windows that contain it. ``queries``: optional (n, 3) array of (b, h, t)."""
    return _call(lib().oracle_multidiffusion_attention, (patch, margin), q, k, v, gk, gv, B, heads, H, W, d,
                 G, queries)


def md_window_keys(H: int, W: int, patch: int, margin: int, pi: int, pj: int) -> np.ndarray:
    """Token ids of window (pi, pj), ascending."""
    out = np.empty(H * W, dtype=np.int32)
    n = lib().oracle_md_window_keys(H, W, patch, margin, pi, pj,
                                    out.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)))
    if n < 0:
        raise ValueError("bad window arguments")
    return out[:n].copy()


def md_window_count(H: int, W: int, patch: int, margin: int, t: int) -> int:
    """Number of windows containing token t."""
    n = lib().oracle_md_window_count(H, W, patch, margin, t)
    if n < 0:
        raise ValueError("bad arguments")
    return int(n)


def md_pair_count(H: int, W: int, patch: int, margin: int, G: int = 0) -> int:
    """(query, key) pairs of one (b, h) under overlapping-window attention."""
    n = lib().oracle_md_pair_count(H, W, patch, margin, G)
    if n < 0:
        raise ValueError("bad arguments")
    return int(n)


def pcpp_attention_stale(q, k, v, ks, vs, *, B, heads, H, W, d, n_strips, p, gk=None, gv=None, G=0,
                         queries: Optional[Sequence] = None) -> np.ndarray:
    """PCPP attention with stale neighbour rows, float64: the keys of a query's
    own strip come from k/v, the borrowed neighbour rows from ks/vs (the
    previous step's keys/values, same layout)."""
    q, qp = _u16(q)
    k, kp = _u16(k)
    v, vp = _u16(v)
    ks, ksp = _u16(ks)
    vs, vsp = _u16(vs)
    gk, gkp = _u16(gk)
    gv, gvp = _u16(gv)
    if queries is None:
        out = np.empty((B, heads, H * W, d), dtype=np.float64)
        qs_p, nq = None, 0
    else:
        qs = np.ascontiguousarray(np.asarray(queries, dtype=np.int32).reshape(-1, 3))
        out = np.empty((qs.shape[0], d), dtype=np.float64)
        qs_p, nq = qs.ctypes.data_as(ctypes.c_void_p), qs.shape[0]
    rc = lib().oracle_pcpp_attention_stale(qp, kp, vp, ksp, vsp, gkp, gvp, out.ctypes.data_as(ctypes.c_void_p),
                                           B, heads, H, W, d, n_strips, float(p), G, qs_p, nq)
    if rc != 0:
        raise RuntimeError(f"oracle failed with code {rc}")
    return out


def global_query_attention(gq, k, v, gk, gv, *, B, heads, H, W, d, G,
                           queries: Optional[Sequence] = None) -> np.ndarray:
    """Text-query half of joint attention, float64: each global token attends
    to all H*W image tokens and all G global tokens. ``queries``: optional
    (n, 3) array of (b, h, g); otherwise the full [B, heads, G, d] result."""
    gq, gqp = _u16(gq)
    k, kp = _u16(k)
    v, vp = _u16(v)
    gk, gkp = _u16(gk)
    gv, gvp = _u16(gv)
    if queries is None:
        out = np.empty((B, heads, G, d), dtype=np.float64)
        qs_p, nq = None, 0
    else:
        qs = np.ascontiguousarray(np.asarray(queries, dtype=np.int32).reshape(-1, 3))
        out = np.empty((qs.shape[0], d), dtype=np.float64)
        qs_p, nq = qs.ctypes.data_as(ctypes.c_void_p), qs.shape[0]
    rc = lib().oracle_global_query_attention(gqp, kp, vp, gkp, gvp, out.ctypes.data_as(ctypes.c_void_p), B, heads,
                                             H, W, d, G, qs_p, nq)
    if rc != 0:
        raise RuntimeError(f"oracle failed with code {rc}")
    return out


# ---------------------------------------------------------------------------
# Dense formulation: a membership predicate over coordinates, then a masked
# softmax over the full key axis.
# ---------------------------------------------------------------------------

def dense_mask(geometry: str, H: int, W: int, *, patch: int = 0, margin: int = 0,
               n_strips: int = 0, p: float = 0.0, G: int = 0) -> np.ndarray:
    """Boolean ``[N, N+G]``: entry (t, j) is True when query t may attend key j.

    NPA: key (r', c') is visible to query (r, c) when r' lies within ``margin``
    rows of the query's patch row span and c' within ``margin`` columns of its
    column span (the grid bounds clip automatically). PCPP: key row r' is
    visible to a query in strip i when it lies in strip i, or in strip i-1 at
    most ``r`` rows above strip i's first row, or in strip i+1 at most ``r``
    rows below its last row.
    """
    N = H * W
    rows = np.arange(N) // W
    cols = np.arange(N) % W
    if geometry == "npa":
        P, m = patch, margin
        pr0 = (rows // P) * P
        pr1 = np.minimum(pr0 + P, H)
        pc0 = (cols // P) * P
        pc1 = np.minimum(pc0 + P, W)
        ok_r = (rows[None, :] >= (pr0 - m)[:, None]) & (rows[None, :] < (pr1 + m)[:, None])
        ok_c = (cols[None, :] >= (pc0 - m)[:, None]) & (cols[None, :] < (pc1 + m)[:, None])
        img = ok_r & ok_c
    elif geometry == "pcpp":
        s = H // n_strips
        r = pcpp_neighbor_rows(s, p)
        qi = rows // s
        ki = rows // s
        dist_above = (qi[:, None] * s) - rows[None, :]            # >0: key above strip start
        dist_below = rows[None, :] - ((qi[:, None] + 1) * s - 1)  # >0: key below strip end
        same = ki[None, :] == qi[:, None]
        above = (ki[None, :] == qi[:, None] - 1) & (dist_above <= r)
        below = (ki[None, :] == qi[:, None] + 1) & (dist_below <= r)
        img = same | above | below
    else:
        raise ValueError(geometry)
    if G:
        img = np.concatenate([img, np.ones((N, G), dtype=bool)], axis=1)
    return img


def dense_attention(q, k, v, *, geometry: str, B, heads, H, W, d, gk=None, gv=None, G=0,
                    **geom) -> np.ndarray:
    """Masked-softmax attention over all keys, float64, ``[B, heads, N, d]``."""
    mask = dense_mask(geometry, H, W, G=G, **geom)
    Q = bf16_to_f64(q).reshape(B, heads, H * W, d)
    K = bf16_to_f64(k).reshape(B, heads, H * W, d)
    V = bf16_to_f64(v).reshape(B, heads, H * W, d)
    if G:
        K = np.concatenate([K, bf16_to_f64(gk).reshape(B, heads, G, d)], axis=2)
        V = np.concatenate([V, bf16_to_f64(gv).reshape(B, heads, G, d)], axis=2)
    logits = np.einsum("bhtc,bhjc->bhtj", Q, K) / np.sqrt(d)
    logits = np.where(mask[None, None], logits, -np.inf)
    logits -= logits.max(axis=-1, keepdims=True)
    w = np.exp(logits)
    w /= w.sum(axis=-1, keepdims=True)
    return np.einsum("bhtj,bhjc->bhtc", w, V)


def dense_pcpp_stale(q, k, v, ks, vs, *, B, heads, H, W, d, n_strips, p, gk=None, gv=None, G=0) -> np.ndarray:
    """Dense form of the two-source PCPP: logits against the current keys where
    the key row shares the query's strip and against the stale keys elsewhere,
    one masked softmax over all keys, values picked the same way."""
    N = H * W
    mask = dense_mask("pcpp", H, W, n_strips=n_strips, p=p, G=G)
    strip = (np.arange(N) // W) // (H // n_strips)
    own = strip[:, None] == strip[None, :]                      # [N, N] same strip
    Q = bf16_to_f64(q).reshape(B, heads, N, d)
    Kf = bf16_to_f64(k).reshape(B, heads, N, d)
    Vf = bf16_to_f64(v).reshape(B, heads, N, d)
    Ks = bf16_to_f64(ks).reshape(B, heads, N, d)
    Vs = bf16_to_f64(vs).reshape(B, heads, N, d)
    lf = np.einsum("bhtc,bhjc->bhtj", Q, Kf)
    ls = np.einsum("bhtc,bhjc->bhtj", Q, Ks)
    logits = np.where(own[None, None], lf, ls)
    if G:
        lg = np.einsum("bhtc,bhjc->bhtj", Q, bf16_to_f64(gk).reshape(B, heads, G, d))
        logits = np.concatenate([logits, lg], axis=-1)
    logits = logits / np.sqrt(d)
    logits = np.where(mask[None, None], logits, -np.inf)
    logits -= logits.max(axis=-1, keepdims=True)
    w = np.exp(logits)
    w /= w.sum(axis=-1, keepdims=True)
    wi = w[..., :N]
    out = np.einsum("bhtj,bhjc->bhtc", np.where(own[None, None], wi, 0.0), Vf)
    out += np.einsum("bhtj,bhjc->bhtc", np.where(own[None, None], 0.0, wi), Vs)
    if G:
        out += np.einsum("bhtj,bhjc->bhtc", w[..., N:], bf16_to_f64(gv).reshape(B, heads, G, d))
    return out


# ---------------------------------------------------------------------------
# Asynchronous structure guidance (ASG) combine
# ---------------------------------------------------------------------------

def asg_guidance_combine(eps, eps_ref, mask, w_t: float) -> np.ndarray:
    """ASGDiffusion (pith.science review), "core_discovery" and
    "key_machinery": the corrected noise of patch i is its own prediction plus
    the guidance G_t = w_t * M * (eps_ref - eps_i), where eps_ref is the
    reference patch's prediction from the previous step (the asynchronous
    substitution) and M the normalised mask. Reading taken here: M is one
    spatial map per patch and batch element, broadcast over the channels.

    eps: bf16 bits [n_patches, B, C, S]; eps_ref: [B, C, S]; mask: [n_patches,
    B, S]. Returns float64 [n_patches, B, C, S], exact up to float64 rounding.
    """
    e = bf16_to_f64(np.asarray(eps, dtype=np.uint16))
    r = bf16_to_f64(np.asarray(eps_ref, dtype=np.uint16))
    m = bf16_to_f64(np.asarray(mask, dtype=np.uint16))
    if e.ndim != 4 or r.shape != e.shape[1:] or m.shape != (e.shape[0], e.shape[1], e.shape[3]):
        raise ValueError("shapes: eps [n, B, C, S], eps_ref [B, C, S], mask [n, B, S]")
    return e + float(w_t) * m[:, :, None, :] * (r[None] - e)
