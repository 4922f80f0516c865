"""Pins for the ASG guidance-combine oracle (ASGDiffusion review,
"core_discovery": corrected noise = eps_i + w_t * M * (eps_ref - eps_i)):
a hand-worked example, the special cases the formula reduces to, and the
broadcast structure (M shared across channels, the reference shared across
patches)."""
import json
import os

import numpy as np
import pytest

import oracle
from workloads import bf16_bits_to_f64, f64_to_bf16_bits

GOLDEN = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "asg_combine.json")))


def _rand(rng, *shape):
    return f64_to_bf16_bits(rng.standard_normal(shape))


def test_hand_worked_example():
    g = GOLDEN
    eps, ref, m = (f64_to_bf16_bits(np.array(g[k], dtype=np.float64)) for k in ("eps", "eps_ref", "mask"))
    np.testing.assert_array_equal(oracle.asg_guidance_combine(eps, ref, m, g["w_t"]), np.array(g["out"]))


@pytest.fixture
def tensors():
    rng = np.random.default_rng(5)
    n, B, C, S = 3, 2, 4, 37
    return _rand(rng, n, B, C, S), _rand(rng, B, C, S), f64_to_bf16_bits(rng.uniform(0, 1, (n, B, S))), (n, B, C, S)


def test_special_cases(tensors):
    eps, ref, m, (n, B, C, S) = tensors
    e = bf16_bits_to_f64(eps)
    np.testing.assert_array_equal(oracle.asg_guidance_combine(eps, ref, m, 0.0), e)             # no guidance
    zero = np.zeros_like(m)
    np.testing.assert_array_equal(oracle.asg_guidance_combine(eps, ref, zero, 3.0), e)          # mask off
    one = f64_to_bf16_bits(np.ones((n, B, S)))
    np.testing.assert_array_equal(oracle.asg_guidance_combine(eps, ref, one, 1.0),              # full pull
                                  np.broadcast_to(bf16_bits_to_f64(ref)[None], e.shape))
    half = oracle.asg_guidance_combine(eps, ref, one, 0.5)
    np.testing.assert_allclose(half, 0.5 * (e + bf16_bits_to_f64(ref)[None]), rtol=0, atol=1e-15)


def test_broadcast_structure(tensors):
    eps, ref, m, (n, B, C, S) = tensors
    out = oracle.asg_guidance_combine(eps, ref, m, 0.7)
    perm_c = np.array([2, 0, 3, 1])
    np.testing.assert_array_equal(oracle.asg_guidance_combine(eps[:, :, perm_c], ref[:, perm_c], m, 0.7),
                                  out[:, :, perm_c])                       # the mask does not depend on C
    perm_p = np.array([1, 2, 0])
    np.testing.assert_array_equal(oracle.asg_guidance_combine(eps[perm_p], ref, m[perm_p], 0.7),
                                  out[perm_p])                             # one reference for every patch


def test_shapes_checked(tensors):
    eps, ref, m, _ = tensors
    with pytest.raises(ValueError):
        oracle.asg_guidance_combine(eps, ref[:, :, :-1], m, 1.0)
    with pytest.raises(ValueError):
        oracle.asg_guidance_combine(eps, ref, m[:, :, :-1], 1.0)


def test_negative_controls_break_the_worked_example():
    """Mistakes planted through the oracle's arguments - a sign error
    (negated weight) or a complemented mask - must fail the hand-worked
    example, so the pin catches them."""
    g = GOLDEN
    eps, ref, m = (f64_to_bf16_bits(np.array(g[k], dtype=np.float64)) for k in ("eps", "eps_ref", "mask"))
    want = np.array(g["out"])
    assert not np.array_equal(oracle.asg_guidance_combine(eps, ref, m, -g["w_t"]), want)
    one_minus = f64_to_bf16_bits(1.0 - np.array(g["mask"], dtype=np.float64))
    assert not np.array_equal(oracle.asg_guidance_combine(eps, ref, one_minus, g["w_t"]), want)
