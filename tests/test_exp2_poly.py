"""The FMA-pipe exponential (Cody-Waite reduction + minimax polynomial) the
kernel can use for part of its exponentials: its error bound, its handling of
masked (-inf) arguments, and that the kernel source carries the fitted
coefficients."""
import os
import re

import numpy as np

from patch_res_diffusion_b200 import fit_exp2_poly as fit

KERNEL = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                      "patch_res_diffusion_b200", "csrc", "npa_fwd_kernel.cuh")


def test_minimax_error_bound():
    c, e = fit.remez()
    assert e < 1e-4  # far below the bf16 rounding of P (2^-9)
    # equioscillation: the error reaches +-e at degree+2 points
    grid = np.linspace(fit.LO, fit.HI, 100001)
    err = np.polyval(c[::-1], grid) / np.exp2(grid) - 1.0
    assert abs(err.max() - e) < 1e-7 and abs(-err.min() - e) < 1e-7


def test_float32_sequence_matches_exp2():
    c = fit.coefficients_f32()
    x = np.linspace(-120.0, 8.0, 1_000_001, dtype=np.float32)
    got = fit.emulate_exp2_f32(x, c).astype(np.float64)
    rel = np.abs(got / np.exp2(x.astype(np.float64)) - 1.0)
    assert rel.max() < 1e-4
    # integers are reproduced closely and the result is monotone on a fine grid
    xi = np.arange(-100, 9, dtype=np.float32)
    assert np.allclose(fit.emulate_exp2_f32(xi, c), np.exp2(xi.astype(np.float64)), rtol=1e-4, atol=0)


def test_masked_arguments_give_exact_zero():
    c = fit.coefficients_f32()
    x = np.array([-np.inf, -1e30, -125.5, -200.0], dtype=np.float32)
    assert np.all(fit.emulate_exp2_f32(x, c) == 0.0)
    assert fit.emulate_exp2_f32(np.array([-125.0], dtype=np.float32), c)[0] > 0.0


def test_kernel_carries_fitted_coefficients():
    src = open(KERNEL).read()
    body = src[src.index("exp2_poly_x2"):]
    c = fit.coefficients_f32()
    for v in c.tolist():
        assert re.search(re.escape(repr(v)) + "f", body), v
