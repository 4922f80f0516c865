"""GPU parity of the overlapping-window (MultiDiffusion-style) comparator
against the float64 oracle: every NPA window attends within itself and a
token's output is the mean over the windows containing it. Small grids are
compared in full; the SDXL attention shapes on sampled queries."""
import pytest

import oracle
from workloads import Workload, make_inputs
from _parity import compare, log_metrics, passes, sample_queries, to_device, to_f64

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from patch_res_diffusion_b200 import build
    build.build()
    import patch_res_diffusion_b200 as npa
    npa.lib()
    yield
    assert npa.npa_device_status() == npa.NPA_OK


def gpu(w: Workload, inp, margin=None):
    import patch_res_diffusion_b200 as npa
    q, k, v = (to_device(inp[n]) for n in ("q", "k", "v"))
    gk = to_device(inp["gk"]) if w.G else None
    gv = to_device(inp["gv"]) if w.G else None
    o = torch.full_like(q, float("nan"))
    npa.multidiffusion_attention(q, k, v, w.H, w.W, w.patch, w.margin if margin is None else margin, gk, gv, out=o)
    return o


def ref(w: Workload, inp, queries=None, margin=None):
    return oracle.multidiffusion_attention(inp["q"], inp["k"], inp["v"], gk=inp.get("gk"), gv=inp.get("gv"), G=w.G,
                                           B=w.B, heads=w.heads, H=w.H, W=w.W, d=w.d, patch=w.patch,
                                           margin=w.margin if margin is None else margin, queries=queries)


SMALL = [
    Workload("md_24", "npa", B=1, heads=2, H=24, W=24, d=64, patch=8, margin=4),
    Workload("md_ragged_g", "npa", B=1, heads=2, H=40, W=37, d=64, patch=16, margin=5, G=7),
    Workload("md_d128_g", "npa", B=2, heads=1, H=32, W=32, d=128, patch=8, margin=3, G=5),
    Workload("md_wide_margin", "npa", B=1, heads=1, H=20, W=20, d=64, patch=4, margin=6),
    Workload("md_single_window", "npa", B=1, heads=2, H=16, W=16, d=64, patch=16, margin=0),
    Workload("md_96x128", "npa", B=1, heads=1, H=64, W=64, d=64, patch=32, margin=16, seed=3),
]


@pytest.mark.parametrize("w", SMALL, ids=lambda w: w.name)
def test_small_full_parity(w):
    inp = make_inputs(w)
    got = to_f64(gpu(w, inp))
    m = compare(got, ref(w, inp))
    log_metrics(f"multidiffusion {w.name}", m)
    assert passes(m), m


def test_zero_margin_equals_npa_bit_for_bit():
    """With margin 0 the windows are the disjoint patches: the comparator must
    reproduce NPA's output exactly (same tiles, one window per token)."""
    import patch_res_diffusion_b200 as npa
    w = Workload("md_m0", "npa", B=2, heads=2, H=32, W=48, d=64, patch=16, margin=0)
    inp = make_inputs(w)
    q, k, v = (to_device(inp[n]) for n in ("q", "k", "v"))
    a = npa.multidiffusion_attention(q, k, v, w.H, w.W, w.patch, 0)
    b = npa.npa_attention(q, k, v, w.H, w.W, w.patch, 0)
    torch.cuda.synchronize()
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_deterministic():
    w = SMALL[1]
    inp = make_inputs(w)
    a, b = gpu(w, inp), gpu(w, inp)
    torch.cuda.synchronize()
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


@pytest.mark.parametrize("shape", ["sdxl_2048", "sdxl_4096_2heads"])
def test_sdxl_shapes_sampled(shape):
    """SDXL attention shapes (64-token patches, 32-token margin): 2048^2 at
    B2 h10 (128^2 tokens), 4096^2 at B1 h2 (256^2 tokens), on sampled queries
    including every patch corner."""
    w = (Workload("md_2048", "npa", B=2, heads=10, H=128, W=128, d=64, patch=64, margin=32)
         if shape == "sdxl_2048" else
         Workload("md_4096", "npa", B=1, heads=2, H=256, W=256, d=64, patch=64, margin=32))
    inp = make_inputs(w)
    qs = sample_queries(w, n_random=384, max_bh=2)
    got = to_f64(gpu(w, inp))[qs[:, 0], qs[:, 1], qs[:, 2]]
    m = compare(got, ref(w, inp, queries=qs))
    log_metrics(f"multidiffusion {shape} sampled", m)
    assert passes(m), m


def _random_md(n, seed=55):
    import numpy as np
    rng = np.random.default_rng(seed)
    out = []
    for i in range(n):
        H, W = int(rng.integers(2, 48)), int(rng.integers(2, 48))
        patch = int(rng.integers(1, max(2, min(H, W) + 1)))
        out.append(Workload(f"rand_md_{i}", "npa", B=int(rng.integers(1, 3)), heads=int(rng.integers(1, 3)), H=H, W=W,
                            d=int(rng.choice([64, 128])), patch=patch, margin=int(rng.integers(0, patch + 4)),
                            G=int(rng.choice([0, int(rng.integers(1, 40))])), seed=i))
    return out


@pytest.mark.parametrize("w", _random_md(10), ids=lambda w: w.name)
def test_random_geometries_full_parity(w):
    """Seeded random small geometries of the comparator, every row against the oracle."""
    inp = make_inputs(w)
    m = compare(to_f64(gpu(w, inp)), ref(w, inp))
    log_metrics(f"random multidiffusion {w.name}", m)
    assert passes(m), (w, m)
