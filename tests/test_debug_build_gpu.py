"""The bounds-checking build (``libnpa_b200_debug.so``, NPA_DEBUG_BOUNDS) on
the GPU: device-side checks of every TMA box origin against its tensor's
extent and of every output row against the output's row count, reported in
the status word (NPA_ERR_DEVICE_BOUNDS) without trapping. It stands in for a
memory checker, which this test setup does not run.

* the small, ragged and degenerate parity cases run under it with status OK
  and still match the float64 oracle;
* the attention kernel's abort path: a launch whose first CTA withholds one
  arrival runs its bounded waits out (1 ms), records NPA_ERR_DEVICE_TIMEOUT,
  drains what it issued and frees its tensor memory; the next call on the
  same context is correct.
"""
import numpy as np
import pytest

from workloads import Workload, make_inputs
from _parity import compare, log_metrics, passes, run_gpu, run_oracle, to_device, to_f64
from test_parity_gpu import EDGE, SMALL

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def npa():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from patch_res_diffusion_b200 import build
    build.build()
    import patch_res_diffusion_b200 as m
    m.use_bounds_checking(True)
    assert m.npa_device_status() == m.NPA_OK
    yield m
    assert m.npa_device_status() == m.NPA_OK
    m.use_bounds_checking(False)


@pytest.mark.parametrize("w", SMALL + EDGE, ids=lambda w: w.name)
def test_checked_build_parity_and_no_bounds_error(npa, w):
    inp = make_inputs(w)
    got = to_f64(run_gpu(w, inp))
    assert npa.npa_device_status() == npa.NPA_OK
    m = compare(got, run_oracle(w, inp))
    log_metrics("bounds-checked " + w.name, m)
    assert passes(m), m


def test_checked_build_other_entry_points(npa):
    """Stale-row PCPP on a strip range, the split text-query attention and the
    overlapping-window comparator also run clean under the checks."""
    import oracle
    rng = np.random.default_rng(4)
    from workloads import f64_to_bf16_bits
    r = lambda shape: f64_to_bf16_bits(rng.standard_normal(shape))
    H, W = 24, 40
    q, k, v, ks, vs = (r((1, 2, H * W, 64)) for _ in range(5))
    o = npa.pcpp_attention_stale(*(to_device(x) for x in (q, k, v, ks, vs)), H, W, 3, 0.5, strips=(1, 2))
    assert npa.npa_device_status() == npa.NPA_OK
    ref = oracle.pcpp_attention_stale(q, k, v, ks, vs, B=1, heads=2, H=H, W=W, d=64, n_strips=3, p=0.5)
    sel = slice(8 * W, H * W)
    assert passes(compare(to_f64(o)[:, :, sel], ref[:, :, sel]))
    G = 130
    gq, gk, gv = r((1, 2, G, 128)), r((1, 2, G, 128)), r((1, 2, G, 128))
    k2, v2 = r((1, 2, H * W, 128)), r((1, 2, H * W, 128))
    o = npa.global_query_attention(*(to_device(x) for x in (gq, k2, v2, gk, gv)), H, W, split=True)
    assert npa.npa_device_status() == npa.NPA_OK
    ref = oracle.global_query_attention(gq, k2, v2, gk, gv, B=1, heads=2, H=H, W=W, d=128, G=G)
    assert passes(compare(to_f64(o), ref))
    o = npa.multidiffusion_attention(*(to_device(x) for x in (q, k, v)), H, W, 8, 3)
    assert npa.npa_device_status() == npa.NPA_OK
    ref = oracle.multidiffusion_attention(q, k, v, B=1, heads=2, H=H, W=W, d=64, patch=8, margin=3)
    assert passes(compare(to_f64(o), ref))


ABORT_CASES = [
    Workload("abort_npa_d64", "npa", B=1, heads=2, H=64, W=64, d=64, patch=32, margin=16),
    Workload("abort_npa_d128_global", "npa", B=1, heads=2, H=48, W=48, d=128, patch=16, margin=8, G=70),
    Workload("abort_pcpp_d64", "pcpp", B=1, heads=2, H=64, W=64, d=64, n_strips=4, p=0.3),
]


@pytest.mark.parametrize("w", ABORT_CASES, ids=lambda w: w.name)
def test_abort_path_drains_and_the_next_call_is_correct(npa, w):
    inp = make_inputs(w)
    npa.npa_debug_withhold_arrival_once(1000)          # 1 ms waits, one arrival withheld
    run_gpu(w, inp)
    assert npa.npa_device_status() == npa.NPA_ERR_DEVICE_TIMEOUT
    assert npa.npa_device_status() == npa.NPA_OK       # the read cleared it
    got = to_f64(run_gpu(w, inp))                      # same context, normal call
    assert npa.npa_device_status() == npa.NPA_OK
    m = compare(got, run_oracle(w, inp))
    log_metrics("after abort " + w.name, m)
    assert passes(m), m
