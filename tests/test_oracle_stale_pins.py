"""Pins for the two-source PCPP oracle: keys of a query's own strip come from
the current keys/values, the borrowed neighbour rows from the previous step's
(PCPP review, "Core claim")."""
import json
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from workloads import bf16_bits_to_f64, f64_to_bf16_bits

GOLDEN = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "index_sets.json")))


def rnd(rng, shape):
    return f64_to_bf16_bits(rng.standard_normal(shape))


def sdpa(qb, kb, vb):
    t = [torch.from_numpy(bf16_bits_to_f64(x)) for x in (qb, kb, vb)]
    return F.scaled_dot_product_attention(*t).numpy()


@pytest.mark.parametrize("case", GOLDEN["pcpp"], ids=lambda c: f"pcpp{c['H']}x{c['W']}n{c['n']}p{c['p']}t{c['t']}")
def test_probe_exposes_key_sources(case):
    """q = 0; current values = identity, stale values = 3 x identity: output
    row t is 1/|S| on the own-strip keys, 3/|S| on the borrowed rows, 0 elsewhere."""
    H, W = case["H"], case["W"]
    N = H * W
    d = N
    q = np.zeros((1, 1, N, d), dtype=np.uint16)
    rng = np.random.default_rng(1)
    k, ks = rnd(rng, (1, 1, N, d)), rnd(rng, (1, 1, N, d))
    v = f64_to_bf16_bits(np.eye(N).reshape(1, 1, N, d))
    vs = f64_to_bf16_bits(3 * np.eye(N).reshape(1, 1, N, d))
    o = oracle.pcpp_attention_stale(q, k, v, ks, vs, B=1, heads=1, H=H, W=W, d=d, n_strips=case["n"], p=case["p"])
    row = o[0, 0, case["t"]]
    expect = np.zeros(N)
    n = len(case["keys"])
    for j in case["keys"]:
        expect[j] = (3.0 if j in case["stale"] else 1.0) / n
    np.testing.assert_allclose(row, expect, rtol=0, atol=1e-15)


def test_probe_negative_control_sources_swapped():
    case = GOLDEN["pcpp"][0]
    H, W = case["H"], case["W"]
    N = H * W
    q = np.zeros((1, 1, N, N), dtype=np.uint16)
    k = rnd(np.random.default_rng(2), (1, 1, N, N))
    v = f64_to_bf16_bits(np.eye(N).reshape(1, 1, N, N))
    vs = f64_to_bf16_bits(3 * np.eye(N).reshape(1, 1, N, N))
    # fresh and stale swapped: the probe must no longer match the golden sources
    o = oracle.pcpp_attention_stale(q, k, vs, k, v, B=1, heads=1, H=H, W=W, d=N, n_strips=case["n"], p=case["p"])
    n = len(case["keys"])
    expect = np.zeros(N)
    for j in case["keys"]:
        expect[j] = (3.0 if j in case["stale"] else 1.0) / n
    assert np.abs(o[0, 0, case["t"]] - expect).max() > 0.1


def test_equal_sources_reduce_to_single_source():
    rng = np.random.default_rng(3)
    H, W, d = 12, 7, 16
    q, k, v = (rnd(rng, (2, 2, H * W, d)) for _ in range(3))
    a = oracle.pcpp_attention_stale(q, k, v, k, v, B=2, heads=2, H=H, W=W, d=d, n_strips=4, p=0.5)
    b = oracle.pcpp_attention(q, k, v, B=2, heads=2, H=H, W=W, d=d, n_strips=4, p=0.5)
    np.testing.assert_array_equal(a, b)


def test_zero_p_never_reads_the_stale_buffers():
    rng = np.random.default_rng(4)
    H, W, d, n = 9, 4, 8, 3
    q, k, v, ks, vs = (rnd(rng, (1, 2, H * W, d)) for _ in range(5))
    got = oracle.pcpp_attention_stale(q, k, v, ks, vs, B=1, heads=2, H=H, W=W, d=d, n_strips=n, p=0.0)
    s = H // n
    expect = np.empty_like(got)
    for i in range(n):
        toks = list(range(i * s * W, (i + 1) * s * W))
        expect[:, :, toks] = sdpa(q[:, :, toks], k[:, :, toks], v[:, :, toks])
    np.testing.assert_allclose(got, expect, rtol=0, atol=1e-12)


def test_two_strips_full_neighbour_is_sdpa_over_mixed_keys():
    """n = 2, p = 1: strip 0 sees its own rows (current) and all of strip 1
    (stale); a library attention over the concatenated keys gives the same."""
    rng = np.random.default_rng(5)
    H, W, d = 6, 5, 16
    q, k, v, ks, vs = (rnd(rng, (1, 2, H * W, d)) for _ in range(5))
    got = oracle.pcpp_attention_stale(q, k, v, ks, vs, B=1, heads=2, H=H, W=W, d=d, n_strips=2, p=1.0)
    half = H // 2 * W
    top = sdpa(q[:, :, :half], np.concatenate([k[:, :, :half], ks[:, :, half:]], 2),
               np.concatenate([v[:, :, :half], vs[:, :, half:]], 2))
    bot = sdpa(q[:, :, half:], np.concatenate([ks[:, :, :half], k[:, :, half:]], 2),
               np.concatenate([vs[:, :, :half], v[:, :, half:]], 2))
    np.testing.assert_allclose(got[:, :, :half], top, rtol=0, atol=1e-12)
    np.testing.assert_allclose(got[:, :, half:], bot, rtol=0, atol=1e-12)


@pytest.mark.parametrize("H,W,n,p,G", [(16, 8, 4, 0.3, 0), (24, 5, 3, 0.8, 9), (16, 7, 8, 0.5, 0), (12, 4, 2, 1.0, 3)])
def test_gather_equals_dense(H, W, n, p, G):
    rng = np.random.default_rng(H * W + G)
    B, heads, d = 1, 2, 16
    q, k, v, ks, vs = (rnd(rng, (B, heads, H * W, d)) for _ in range(5))
    gk = rnd(rng, (B, heads, G, d)) if G else None
    gv = rnd(rng, (B, heads, G, d)) if G else None
    a = oracle.pcpp_attention_stale(q, k, v, ks, vs, gk=gk, gv=gv, G=G, B=B, heads=heads, H=H, W=W, d=d,
                                    n_strips=n, p=p)
    b = oracle.dense_pcpp_stale(q, k, v, ks, vs, gk=gk, gv=gv, G=G, B=B, heads=heads, H=H, W=W, d=d,
                                n_strips=n, p=p)
    np.testing.assert_allclose(a, b, rtol=0, atol=1e-12)
