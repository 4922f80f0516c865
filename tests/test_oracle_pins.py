"""Pins the CPU oracle to facts that do not come from the oracle itself.

* hand-enumerated key sets and row counts (``tests/golden/index_sets.json``),
  checked both on the key-set builder and, through probe inputs, on the
  attention routine end to end;
* special cases that reduce to full attention, per-patch attention or
  per-strip attention, computed by a library routine
  (``torch.nn.functional.scaled_dot_product_attention`` in float64 on CPU);
* closed forms (a one-key set returns its value row; constant values are
  returned unchanged because the weights sum to one);
* agreement of the two independent formulations (gather vs dense mask);
* invariance under a permutation of the global tokens;
* a cross-check between the geometries (PCPP with n strips equals NPA with
  patch side s and margin r once the grid is no wider than s).
Negative controls plant an off-by-one margin or neighbour-row count in the
oracle's arguments and check that the pins reject it.
"""
import json
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from workloads import PRESETS, f64_to_bf16_bits, bf16_bits_to_f64

GOLDEN = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "index_sets.json")))


def rand_bf16(rng, shape, scale=1.0):
    return f64_to_bf16_bits(rng.standard_normal(shape) * scale)


def sdpa(qb, kb, vb):
    q = torch.from_numpy(bf16_bits_to_f64(qb))
    k = torch.from_numpy(bf16_bits_to_f64(kb))
    v = torch.from_numpy(bf16_bits_to_f64(vb))
    return F.scaled_dot_product_attention(q, k, v).numpy()


# --------------------------------------------------------------------------
# Hand-enumerated key sets
# --------------------------------------------------------------------------

@pytest.mark.parametrize("case", GOLDEN["npa"], ids=lambda c: f"npa{c['H']}x{c['W']}P{c['P']}m{c['m']}t{c['t']}")
def test_npa_key_set_hand_enumerated(case):
    got = oracle.npa_key_set(case["H"], case["W"], case["P"], case["m"], case["t"])
    assert got.tolist() == case["keys"]


@pytest.mark.parametrize("case", GOLDEN["pcpp"], ids=lambda c: f"pcpp{c['H']}x{c['W']}n{c['n']}p{c['p']}t{c['t']}")
def test_pcpp_key_set_hand_enumerated(case):
    got = oracle.pcpp_key_set(case["H"], case["W"], case["n"], case["p"], case["t"])
    assert sorted(got.tolist()) == case["keys"]


@pytest.mark.parametrize("case", GOLDEN["pcpp_neighbor_rows"], ids=lambda c: f"s{c['s']}p{c['p']}")
def test_pcpp_neighbor_rows_golden(case):
    assert oracle.pcpp_neighbor_rows(case["s"], case["p"]) == case["r"]


@pytest.mark.parametrize("case", GOLDEN["pcpp_kv_rows"], ids=lambda c: f"n{c['n']}p{c['p']}")
def test_pcpp_kv_rows_golden(case):
    H, n, W = case["H"], case["n"], 3
    s = H // n
    rows = [len(oracle.pcpp_key_set(H, W, n, case["p"], (i * s) * W)) // W for i in range(n)]
    assert rows == case["rows"]


@pytest.mark.parametrize("case", GOLDEN["npa_window_sides"], ids=lambda c: f"L{c['L']}")
def test_npa_window_sides_golden(case):
    L, P, m = case["L"], case["P"], case["m"]
    sides = [len(oracle.npa_key_set(L, 1, P, m, pi * P)) for pi in range((L + P - 1) // P)]
    assert sides == case["sides"]


@pytest.mark.parametrize("case", GOLDEN["pair_counts_per_head"], ids=lambda c: c["workload"])
def test_pair_counts_golden(case):
    w = PRESETS[case["workload"]]
    got = oracle.pair_count(w.geometry, w.H, w.W, patch=w.patch, margin=w.margin,
                            n_strips=w.n_strips, p=w.p, G=w.G)
    assert got == case["pairs"]


def test_negative_control_margin_off_by_one():
    """A margin one too large or too small must break the hand-enumerated sets."""
    for case in GOLDEN["npa"]:
        if case["m"] == 0:
            continue
        for dm in (-1, 1):
            got = oracle.npa_key_set(case["H"], case["W"], case["P"], case["m"] + dm, case["t"])
            assert got.tolist() != case["keys"]


def test_negative_control_neighbor_rows_off_by_one():
    for case in GOLDEN["pcpp_kv_rows"]:
        H, n = case["H"], case["n"]
        s = H // n
        # a p that yields one row fewer must change the row counts
        r = oracle.pcpp_neighbor_rows(s, case["p"])
        p_less = (r - 1) / s
        rows = [len(oracle.pcpp_key_set(H, 1, n, p_less, i * s)) for i in range(n)]
        assert rows != case["rows"]


# --------------------------------------------------------------------------
# Probe inputs: q = 0 makes every logit equal, so the softmax is uniform over
# the key set; with V = identity the output row t is the indicator of S(t)
# divided by |S(t)|, which exposes the key set through the attention routine.
# --------------------------------------------------------------------------

def _probe(geometry, H, W, **geom):
    N = H * W
    d = N
    q = np.zeros((1, 1, N, d), dtype=np.uint16)
    k = rand_bf16(np.random.default_rng(5), (1, 1, N, d))
    v = f64_to_bf16_bits(np.eye(N).reshape(1, 1, N, d))
    if geometry == "npa":
        return oracle.npa_attention(q, k, v, B=1, heads=1, H=H, W=W, d=d, **geom)[0, 0]
    return oracle.pcpp_attention(q, k, v, B=1, heads=1, H=H, W=W, d=d, **geom)[0, 0]


@pytest.mark.parametrize("case", GOLDEN["npa"], ids=lambda c: f"npa{c['H']}x{c['W']}P{c['P']}m{c['m']}t{c['t']}")
def test_probe_exposes_npa_key_set(case):
    o = _probe("npa", case["H"], case["W"], patch=case["P"], margin=case["m"])
    row = o[case["t"]]
    keys = case["keys"]
    expect = np.zeros_like(row)
    expect[keys] = 1.0 / len(keys)
    np.testing.assert_allclose(row, expect, rtol=0, atol=1e-15)


@pytest.mark.parametrize("case", GOLDEN["pcpp"], ids=lambda c: f"pcpp{c['H']}x{c['W']}n{c['n']}p{c['p']}t{c['t']}")
def test_probe_exposes_pcpp_key_set(case):
    o = _probe("pcpp", case["H"], case["W"], n_strips=case["n"], p=case["p"])
    row = o[case["t"]]
    keys = case["keys"]
    expect = np.zeros_like(row)
    expect[keys] = 1.0 / len(keys)
    np.testing.assert_allclose(row, expect, rtol=0, atol=1e-15)


def test_probe_negative_control():
    case = GOLDEN["npa"][0]
    o = _probe("npa", case["H"], case["W"], patch=case["P"], margin=case["m"] + 1)
    expect = np.zeros(case["H"] * case["W"])
    expect[case["keys"]] = 1.0 / len(case["keys"])
    assert np.abs(o[case["t"]] - expect).max() > 1e-3


# --------------------------------------------------------------------------
# Special cases against a library routine
# --------------------------------------------------------------------------

def _inputs(rng, B, heads, N, d, G):
    q = rand_bf16(rng, (B, heads, N, d))
    k = rand_bf16(rng, (B, heads, N, d))
    v = rand_bf16(rng, (B, heads, N, d))
    gk = rand_bf16(rng, (B, heads, G, d)) if G else None
    gv = rand_bf16(rng, (B, heads, G, d)) if G else None
    return q, k, v, gk, gv


def _full(q, k, v, gk, gv):
    if gk is not None:
        k = np.concatenate([k, gk], axis=2)
        v = np.concatenate([v, gv], axis=2)
    return sdpa(q, k, v)


@pytest.mark.parametrize("H,W,P,m,G", [(9, 7, 3, 9, 0), (9, 7, 3, 9, 5), (6, 10, 10, 0, 0),
                                         (5, 5, 8, 2, 3), (12, 4, 5, 12, 0)])
def test_npa_window_covering_grid_is_full_attention(H, W, P, m, G):
    rng = np.random.default_rng(H * 100 + W)
    B, heads, d = 2, 2, 16
    q, k, v, gk, gv = _inputs(rng, B, heads, H * W, d, G)
    got = oracle.npa_attention(q, k, v, gk=gk, gv=gv, G=G, B=B, heads=heads, H=H, W=W, d=d, patch=P, margin=m)
    np.testing.assert_allclose(got, _full(q, k, v, gk, gv), rtol=0, atol=1e-12)


@pytest.mark.parametrize("H,W,n,p,G", [(8, 5, 1, 0.0, 0), (8, 5, 1, 0.6, 4), (8, 5, 2, 1.0, 0),
                                         (6, 3, 2, 1.0, 2)])
def test_pcpp_full_context_is_full_attention(H, W, n, p, G):
    rng = np.random.default_rng(H * 10 + n)
    B, heads, d = 1, 3, 16
    q, k, v, gk, gv = _inputs(rng, B, heads, H * W, d, G)
    got = oracle.pcpp_attention(q, k, v, gk=gk, gv=gv, G=G, B=B, heads=heads, H=H, W=W, d=d, n_strips=n, p=p)
    np.testing.assert_allclose(got, _full(q, k, v, gk, gv), rtol=0, atol=1e-12)


def test_pcpp_three_strips_p1_is_not_full_attention():
    """With n >= 3 strips even p = 1 leaves non-adjacent strips out."""
    rng = np.random.default_rng(11)
    H, W, n, d = 6, 2, 3, 8
    q, k, v, _, _ = _inputs(rng, 1, 1, H * W, d, 0)
    got = oracle.pcpp_attention(q, k, v, B=1, heads=1, H=H, W=W, d=d, n_strips=n, p=1.0)
    assert np.abs(got - _full(q, k, v, None, None)).max() > 1e-3


@pytest.mark.parametrize("H,W,P", [(8, 8, 4), (7, 9, 3), (5, 6, 5)])
def test_npa_zero_margin_is_per_patch_attention(H, W, P):
    rng = np.random.default_rng(P)
    B, heads, d = 1, 2, 8
    q, k, v, _, _ = _inputs(rng, B, heads, H * W, d, 0)
    got = oracle.npa_attention(q, k, v, B=B, heads=heads, H=H, W=W, d=d, patch=P, margin=0)
    expect = np.empty_like(got)
    for r0 in range(0, H, P):
        for c0 in range(0, W, P):
            toks = [r * W + c for r in range(r0, min(H, r0 + P)) for c in range(c0, min(W, c0 + P))]
            expect[:, :, toks] = sdpa(q[:, :, toks], k[:, :, toks], v[:, :, toks])
    np.testing.assert_allclose(got, expect, rtol=0, atol=1e-12)


@pytest.mark.parametrize("H,W,n", [(8, 3, 4), (9, 2, 3)])
def test_pcpp_zero_p_is_per_strip_attention(H, W, n):
    rng = np.random.default_rng(n)
    B, heads, d = 1, 2, 8
    q, k, v, _, _ = _inputs(rng, B, heads, H * W, d, 0)
    got = oracle.pcpp_attention(q, k, v, B=B, heads=heads, H=H, W=W, d=d, n_strips=n, p=0.0)
    s = H // n
    expect = np.empty_like(got)
    for i in range(n):
        toks = list(range(i * s * W, (i + 1) * s * W))
        expect[:, :, toks] = sdpa(q[:, :, toks], k[:, :, toks], v[:, :, toks])
    np.testing.assert_allclose(got, expect, rtol=0, atol=1e-12)


# --------------------------------------------------------------------------
# Closed forms
# --------------------------------------------------------------------------

def test_single_key_returns_its_value():
    rng = np.random.default_rng(3)
    H, W, d = 5, 4, 16
    q, k, v, _, _ = _inputs(rng, 1, 2, H * W, d, 0)
    got = oracle.npa_attention(q, k, v, B=1, heads=2, H=H, W=W, d=d, patch=1, margin=0)
    np.testing.assert_array_equal(got, bf16_bits_to_f64(v))
    got = oracle.pcpp_attention(q, k, v, B=1, heads=2, H=H, W=1 * W, d=d, n_strips=H, p=0.0)
    # strips of one row: each query sees its own row of W keys; W=4 so not a single key,
    # but with W=1 the set is the token itself
    q1, k1, v1 = q[:, :, :H], k[:, :, :H], v[:, :, :H]
    got1 = oracle.pcpp_attention(q1, k1, v1, B=1, heads=2, H=H, W=1, d=d, n_strips=H, p=0.0)
    np.testing.assert_array_equal(got1, bf16_bits_to_f64(v1))
    assert got.shape == (1, 2, H * W, d)


@pytest.mark.parametrize("geometry", ["npa", "pcpp"])
def test_constant_values_are_preserved(geometry):
    """Weights sum to one: V = 1 everywhere gives O = 1 everywhere."""
    rng = np.random.default_rng(8)
    H, W, d, G = 12, 10, 32, 7
    q, k, _, gk, _ = _inputs(rng, 1, 2, H * W, d, G)
    ones = f64_to_bf16_bits(np.ones((1, 2, H * W, d)))
    gones = f64_to_bf16_bits(np.ones((1, 2, G, d)))
    geom = dict(patch=4, margin=2) if geometry == "npa" else dict(n_strips=3, p=0.5)
    fn = oracle.npa_attention if geometry == "npa" else oracle.pcpp_attention
    got = fn(q, k, ones, gk=gk, gv=gones, G=G, B=1, heads=2, H=H, W=W, d=d, **geom)
    np.testing.assert_allclose(got, 1.0, rtol=0, atol=1e-13)


# --------------------------------------------------------------------------
# Two formulations, global-token permutation, cross-geometry
# --------------------------------------------------------------------------

@pytest.mark.parametrize("geometry,H,W,geom,G", [
    ("npa", 16, 16, dict(patch=8, margin=4), 0),
    ("npa", 13, 11, dict(patch=4, margin=3), 6),
    ("npa", 20, 9, dict(patch=6, margin=1), 0),
    ("pcpp", 16, 8, dict(n_strips=4, p=0.3), 0),
    ("pcpp", 24, 5, dict(n_strips=3, p=0.8), 9),
    ("pcpp", 16, 7, dict(n_strips=8, p=0.5), 0),
])
def test_gather_equals_dense(geometry, H, W, geom, G):
    rng = np.random.default_rng(H * W + G)
    B, heads, d = 1, 2, 16
    q, k, v, gk, gv = _inputs(rng, B, heads, H * W, d, G)
    fn = oracle.npa_attention if geometry == "npa" else oracle.pcpp_attention
    got = fn(q, k, v, gk=gk, gv=gv, G=G, B=B, heads=heads, H=H, W=W, d=d, **geom)
    dense = oracle.dense_attention(q, k, v, gk=gk, gv=gv, G=G, geometry=geometry, B=B, heads=heads,
                                   H=H, W=W, d=d, **geom)
    np.testing.assert_allclose(got, dense, rtol=0, atol=1e-12)


def test_dense_mask_matches_golden_sets():
    for case in GOLDEN["npa"]:
        mask = oracle.dense_mask("npa", case["H"], case["W"], patch=case["P"], margin=case["m"])
        assert np.flatnonzero(mask[case["t"]]).tolist() == case["keys"]
    for case in GOLDEN["pcpp"]:
        mask = oracle.dense_mask("pcpp", case["H"], case["W"], n_strips=case["n"], p=case["p"])
        assert np.flatnonzero(mask[case["t"]]).tolist() == case["keys"]


def test_global_token_permutation_invariance():
    rng = np.random.default_rng(21)
    H, W, d, G = 10, 10, 16, 11
    q, k, v, gk, gv = _inputs(rng, 1, 2, H * W, d, G)
    a = oracle.npa_attention(q, k, v, gk=gk, gv=gv, G=G, B=1, heads=2, H=H, W=W, d=d, patch=4, margin=2)
    perm = rng.permutation(G)
    b = oracle.npa_attention(q, k, v, gk=gk[:, :, perm], gv=gv[:, :, perm], G=G, B=1, heads=2, H=H,
                             W=W, d=d, patch=4, margin=2)
    np.testing.assert_allclose(a, b, rtol=0, atol=1e-13)


@pytest.mark.parametrize("H,W,n,p", [(12, 3, 3, 0.5), (16, 4, 4, 0.3), (15, 2, 3, 0.8)])
def test_pcpp_equals_npa_when_grid_narrower_than_strip(H, W, n, p):
    s = H // n
    assert W <= s
    r = oracle.pcpp_neighbor_rows(s, p)
    rng = np.random.default_rng(H + W)
    q, k, v, _, _ = _inputs(rng, 1, 2, H * W, 16, 0)
    a = oracle.pcpp_attention(q, k, v, B=1, heads=2, H=H, W=W, d=16, n_strips=n, p=p)
    b = oracle.npa_attention(q, k, v, B=1, heads=2, H=H, W=W, d=16, patch=s, margin=r)
    np.testing.assert_allclose(a, b, rtol=0, atol=1e-13)


def test_query_subset_matches_full_run():
    rng = np.random.default_rng(4)
    B, heads, H, W, d, G = 2, 2, 9, 9, 16, 3
    q, k, v, gk, gv = _inputs(rng, B, heads, H * W, d, G)
    full = oracle.npa_attention(q, k, v, gk=gk, gv=gv, G=G, B=B, heads=heads, H=H, W=W, d=d, patch=4, margin=1)
    qs = np.array([[1, 0, 80], [0, 1, 0], [1, 1, 40], [0, 0, 17]], dtype=np.int32)
    sub = oracle.npa_attention(q, k, v, gk=gk, gv=gv, G=G, B=B, heads=heads, H=H, W=W, d=d, patch=4,
                               margin=1, queries=qs)
    for i, (b, h, t) in enumerate(qs):
        np.testing.assert_array_equal(sub[i], full[b, h, t])


def test_bad_arguments_raise():
    with pytest.raises(ValueError):
        oracle.npa_key_set(4, 4, 0, 1, 0)
    with pytest.raises(ValueError):
        oracle.pcpp_key_set(5, 4, 2, 0.5, 0)  # 5 rows do not split into 2 strips
    assert oracle.pcpp_neighbor_rows(4, 1.5) == -1
