"""Pins for the overlapping-window (MultiDiffusion-style) attention oracle,
the comparator for NPA (ScaleDiff summary, "Problem" and "Approach":
MultiDiffusion processes overlapping patches and averages them; NPA keeps the
query patches disjoint). Reading: the overlapping patches are the NPA windows;
inside a window every token attends to the whole window (and the global
tokens); a token's output is the mean over the windows containing it.

Each pin checks the oracle against something other than itself: hand
enumeration, a closed form from per-axis window sizes, library attention
(torch, float64) where the method reduces to it, a dense masked formulation,
and a probe whose answer is known in closed form."""
import json
import os

import numpy as np
import pytest
import torch

import oracle
from workloads import bf16_bits_to_f64, f64_to_bf16_bits

GOLDEN = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "md_windows.json")))


def _rand(rng, *shape):
    return f64_to_bf16_bits(rng.standard_normal(shape))


def _t(bits):
    return torch.from_numpy(bf16_bits_to_f64(bits))


def _sdpa(q, k, v):
    """Library attention, float64, over the last two axes."""
    return torch.nn.functional.scaled_dot_product_attention(q, k, v).numpy()


@pytest.mark.parametrize("case", GOLDEN["cases"], ids=lambda c: f"{c['H']}x{c['W']}")
def test_hand_enumerated_windows_and_counts(case):
    H, W, P, m = case["H"], case["W"], case["patch"], case["margin"]
    for key, toks in case["windows"].items():
        pi, pj = map(int, key.split(","))
        assert oracle.md_window_keys(H, W, P, m, pi, pj).tolist() == toks
    for t, c in case["counts"].items():
        assert oracle.md_window_count(H, W, P, m, int(t)) == c
    cover = case["axis_cover"]
    for t in range(H * W):
        assert oracle.md_window_count(H, W, P, m, t) == cover[t // W] * cover[t % W]
    assert oracle.md_pair_count(H, W, P, m, 0) == case["pairs_G0"]
    assert oracle.md_pair_count(H, W, P, m, 2) == case["pairs_G2"]


def _axis_sizes(L, P, m):
    return [min(L, (i + 1) * P + m) - max(0, i * P - m) for i in range((L + P - 1) // P)]


@pytest.mark.parametrize("H,W,P,m,G", [(256, 256, 64, 32, 0), (128, 128, 64, 32, 0), (40, 37, 16, 5, 7),
                                       (100, 100, 9, 3, 0), (64, 64, 16, 0, 3)])
def test_pair_count_closed_form(H, W, P, m, G):
    """Windows form a grid, so sum |W|^2 = (sum of row sizes^2)(sum of column
    sizes^2) and sum |W| = (sum of row sizes)(sum of column sizes)."""
    r, c = _axis_sizes(H, P, m), _axis_sizes(W, P, m)
    expect = sum(x * x for x in r) * sum(x * x for x in c) + G * sum(r) * sum(c)
    assert oracle.md_pair_count(H, W, P, m, G) == expect
    if (H, W, P, m, G) == (256, 256, 64, 32, 0):
        s = GOLDEN["sdxl_4096"]
        assert r == s["axis_window_sizes"] and expect == s["pairs_per_head"]
        assert oracle.pair_count("npa", H, W, patch=P, margin=m) == s["npa_pairs_per_head"]


@pytest.mark.parametrize("P,m", [(20, 0), (5, 30)])
def test_single_window_is_full_attention(P, m):
    """One window over the whole grid (patch covers the grid, or the margin
    reaches every border from every patch): plain full attention."""
    rng = np.random.default_rng(1)
    B, h, H, W, d = 1, 2, 8, 9, 16
    q, k, v = (_rand(rng, B, h, H * W, d) for _ in range(3))
    got = oracle.multidiffusion_attention(q, k, v, B=B, heads=h, H=H, W=W, d=d, patch=P, margin=m)
    np.testing.assert_allclose(got, _sdpa(_t(q), _t(k), _t(v)), rtol=0, atol=1e-12)


def test_zero_margin_is_per_patch_attention():
    """m = 0: the windows are the disjoint patches, every token lies in one,
    and the result is attention within each patch - also NPA with m = 0."""
    rng = np.random.default_rng(2)
    B, h, H, W, d, P = 1, 2, 8, 8, 16, 4
    q, k, v = (_rand(rng, B, h, H * W, d) for _ in range(3))
    got = oracle.multidiffusion_attention(q, k, v, B=B, heads=h, H=H, W=W, d=d, patch=P, margin=0)
    npa = oracle.npa_attention(q, k, v, B=B, heads=h, H=H, W=W, d=d, patch=P, margin=0)
    np.testing.assert_allclose(got, npa, rtol=0, atol=1e-12)
    expect = np.empty_like(got)
    for pi in range(H // P):
        for pj in range(W // P):
            ids = torch.from_numpy(oracle.md_window_keys(H, W, P, 0, pi, pj).astype(np.int64))
            Q, K, V = (_t(x)[:, :, ids] for x in (q, k, v))
            expect[:, :, ids.numpy()] = _sdpa(Q, K, V)
    np.testing.assert_allclose(got, expect, rtol=0, atol=1e-12)


def test_dense_form_with_global_tokens():
    """Independent dense formulation: per window, a membership mask over the
    full key axis (window tokens + global tokens), masked softmax by the
    library, averaged with coverage counts."""
    rng = np.random.default_rng(3)
    B, h, H, W, d, P, m, G = 2, 1, 11, 10, 16, 4, 2, 3
    q, k, v = (_rand(rng, B, h, H * W, d) for _ in range(3))
    gk, gv = _rand(rng, B, h, G, d), _rand(rng, B, h, G, d)
    got = oracle.multidiffusion_attention(q, k, v, B=B, heads=h, H=H, W=W, d=d, patch=P, margin=m,
                                          gk=gk, gv=gv, G=G)
    Q = _t(q)
    K = torch.cat([_t(k), _t(gk)], dim=2)
    V = torch.cat([_t(v), _t(gv)], dim=2)
    rows = torch.arange(H * W) // W
    cols = torch.arange(H * W) % W
    acc = torch.zeros(B, h, H * W, d, dtype=torch.float64)
    cnt = torch.zeros(H * W, dtype=torch.float64)
    for pi in range((H + P - 1) // P):
        for pj in range((W + P - 1) // P):
            r0, r1 = max(0, pi * P - m), min(H, (pi + 1) * P + m)
            c0, c1 = max(0, pj * P - m), min(W, (pj + 1) * P + m)
            inside = (rows >= r0) & (rows < r1) & (cols >= c0) & (cols < c1)
            mask = torch.cat([inside, torch.ones(G, dtype=torch.bool)])[None, :].expand(H * W, -1)
            o = torch.nn.functional.scaled_dot_product_attention(Q, K, V, attn_mask=mask)
            acc += o * inside[None, None, :, None]
            cnt += inside
    np.testing.assert_allclose(got, (acc / cnt[None, None, :, None]).numpy(), rtol=0, atol=1e-12)


def test_probe_closed_form():
    """q = 0 makes every window's softmax uniform. With v one-hot on key j in
    channel 0 and v = 1 in channel 1: o(t)[0] = mean over windows W containing
    t of [j in W] / |W|, and o(t)[1] = 1."""
    B, h, H, W, d, P, m = 1, 1, 9, 7, 16, 3, 2
    N = H * W
    zero = np.zeros((B, h, N, d), dtype=np.uint16)
    for j in (0, 31, N - 1):
        v = np.zeros((B, h, N, d))
        v[0, 0, j, 0] = 1.0
        v[0, 0, :, 1] = 1.0
        got = oracle.multidiffusion_attention(zero, zero, f64_to_bf16_bits(v), B=B, heads=h, H=H, W=W, d=d,
                                              patch=P, margin=m)
        nph, npw = (H + P - 1) // P, (W + P - 1) // P
        wins = [set(oracle.md_window_keys(H, W, P, m, a, b).tolist()) for a in range(nph) for b in range(npw)]
        for t in range(N):
            mine = [w for w in wins if t in w]
            expect = sum((j in w) / len(w) for w in mine) / len(mine)
            assert abs(got[0, 0, t, 0] - expect) < 1e-12
            assert abs(got[0, 0, t, 1] - 1.0) < 1e-12


def test_query_subset_matches_full():
    rng = np.random.default_rng(4)
    B, h, H, W, d, P, m = 2, 2, 12, 12, 16, 4, 3
    q, k, v = (_rand(rng, B, h, H * W, d) for _ in range(3))
    full = oracle.multidiffusion_attention(q, k, v, B=B, heads=h, H=H, W=W, d=d, patch=P, margin=m)
    qs = np.array([(1, 0, 0), (0, 1, 77), (1, 1, H * W - 1)], dtype=np.int32)
    sub = oracle.multidiffusion_attention(q, k, v, B=B, heads=h, H=H, W=W, d=d, patch=P, margin=m, queries=qs)
    np.testing.assert_array_equal(sub, full[qs[:, 0], qs[:, 1], qs[:, 2]])


@pytest.mark.parametrize("dm", [-1, 1])
def test_negative_control_margin_off_by_one(dm):
    """A mistake planted in the oracle's arguments (margin off by one) must
    break the hand-enumerated windows, the coverage counts and the pair
    count, so the pins above would catch it."""
    case = GOLDEN["cases"][0]
    H, W, P, m = case["H"], case["W"], case["patch"], case["margin"] + dm
    windows_ok = all(oracle.md_window_keys(H, W, P, m, *map(int, key.split(","))).tolist() == toks
                     for key, toks in case["windows"].items())
    counts_ok = all(oracle.md_window_count(H, W, P, m, int(t)) == c for t, c in case["counts"].items())
    assert not windows_ok and not counts_ok
    assert oracle.md_pair_count(H, W, P, m, 0) != case["pairs_G0"]


def test_negative_control_patch_off_by_one():
    case = GOLDEN["cases"][1]
    H, W, P, m = case["H"], case["W"], case["patch"] + 1, case["margin"]
    assert oracle.md_pair_count(H, W, P, m, 0) != case["pairs_G0"]
    assert any(oracle.md_window_count(H, W, P, m, int(t)) != c for t, c in case["counts"].items())
