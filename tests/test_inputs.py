"""The seeded input generator: single-step bfloat16 rounding and the recipe."""
import numpy as np
import torch

from workloads import PRESETS, Workload, bf16_bits_to_f64, box_filter_3x3, f64_to_bf16_bits, make_inputs


def test_bf16_rounding_known_values():
    one = 1.0
    cases = {
        one: 0x3F80,
        -2.0: 0xC000,
        one + 2.0 ** -8: 0x3F80,                      # tie -> even (mantissa 0)
        one + 3 * 2.0 ** -8: 0x3F82,                  # tie -> even (mantissa 2)
        one + 2.0 ** -8 + 2.0 ** -40: 0x3F81,         # above the tie: a float32 detour would lose this
        one + 2.0 ** -7 - 2.0 ** -30: 0x3F81,
        0.0: 0x0000,
        3.140625: 0x4049,
    }
    x = np.array(list(cases.keys()))
    got = f64_to_bf16_bits(x)
    assert got.tolist() == list(cases.values())


def test_bf16_rounding_matches_torch_away_from_ties():
    rng = np.random.default_rng(0)
    x = rng.standard_normal(200_000)
    ours = f64_to_bf16_bits(x)
    theirs = torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    # float64 -> float32 -> bfloat16 differs from one-step rounding only when the
    # float32 value is an exact bfloat16 tie, which has probability ~2^-16 per draw
    assert (ours != theirs).mean() < 1e-4
    back = bf16_bits_to_f64(ours)
    assert np.all(np.abs(back - x) <= np.abs(x) * 2.0 ** -8)


def test_box_filter_mean_of_inbounds_neighbours():
    H, W = 3, 4
    x = np.arange(H * W, dtype=np.float64).reshape(1, H * W, 1)
    y = box_filter_3x3(x, H, W).reshape(H, W)
    g = np.arange(H * W, dtype=np.float64).reshape(H, W)
    assert y[0, 0] == np.mean(g[0:2, 0:2])
    assert y[1, 1] == np.mean(g[0:3, 0:3])
    assert y[2, 3] == np.mean(g[1:3, 2:4])


def test_make_inputs_is_seeded_and_shaped():
    w = Workload("t", "npa", B=1, heads=2, H=6, W=5, d=16, patch=3, margin=1, G=4)
    a = make_inputs(w)
    b = make_inputs(w)
    for key in ("q", "k", "v", "gk", "gv"):
        np.testing.assert_array_equal(a[key], b[key])
    assert a["q"].shape == (1, 2, 30, 16) and a["gk"].shape == (1, 2, 4, 16)
    # tensor index offsets the seed: q and k differ
    assert not np.array_equal(a["q"], a["k"])
    ref = f64_to_bf16_bits(np.random.default_rng(2).standard_normal((1, 2, 30, 16)))
    np.testing.assert_array_equal(a["v"], ref)


def test_smoothed_k_has_smaller_spread():
    w = PRESETS["npa_sdxl_2048"].replace(B=1, heads=1, H=32, W=32)
    k = bf16_bits_to_f64(make_inputs(w)["k"])
    assert 0.25 < k.std() < 0.45


def test_later_row_inputs_follow_the_seed_recipe():
    """Stale-row PCPP adds the previous step's k, v (seeds +5, +6); the
    global-query form adds the global tokens' queries (seed +7). Each is an
    independent N(0, 1) draw rounded to bf16, like q, k and v."""
    from workloads import COMPARATORS
    w = COMPARATORS["pcpp_stale_4x32_p0.3"].replace(B=1, heads=1, H=8, W=8, n_strips=2)
    inp = make_inputs(w)
    shape = (1, 1, 64, w.d)
    for name, off in (("ks", 5), ("vs", 6)):
        expect = f64_to_bf16_bits(np.random.default_rng(w.seed + off).standard_normal(shape))
        np.testing.assert_array_equal(inp[name], expect)
    assert not np.array_equal(inp["ks"], inp["k"])
    g = COMPARATORS["gq_flux_4096"].replace(heads=2, H=4, W=4, G=10)
    ginp = make_inputs(g)
    expect = f64_to_bf16_bits(np.random.default_rng(g.seed + 7).standard_normal((1, 2, 10, g.d)))
    np.testing.assert_array_equal(ginp["gq"], expect)
    assert set(ginp) == {"q", "k", "v", "gk", "gv", "gq"}
