"""GPU parity of the text-query half of joint attention (global tokens as
queries over all image and global keys) against the float64 oracle, with
and without the key-range split workspace."""
import numpy as np
import pytest

import oracle
from workloads import f64_to_bf16_bits
from _parity import compare, log_metrics, passes, to_device, to_f64

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


def make(B, heads, H, W, d, G, seed):
    rng = np.random.default_rng(seed)
    r = lambda shape: f64_to_bf16_bits(rng.standard_normal(shape))
    return {"gq": r((B, heads, G, d)), "k": r((B, heads, H * W, d)), "v": r((B, heads, H * W, d)),
            "gk": r((B, heads, G, d)), "gv": r((B, heads, G, d))}


def gpu(inp, H, W, split):
    import patch_res_diffusion_b200 as npa
    t = {n: to_device(a) for n, a in inp.items()}
    o = torch.full_like(t["gq"], float("nan"))
    npa.global_query_attention(t["gq"], t["k"], t["v"], t["gk"], t["gv"], H, W, out=o, split=split)
    return o


@pytest.mark.parametrize("B,heads,H,W,d,G", [(1, 2, 16, 16, 64, 100), (1, 3, 32, 48, 128, 300),
                                               (2, 1, 40, 64, 64, 1), (1, 2, 20, 36, 128, 129)])
@pytest.mark.parametrize("split", [False, True])
def test_global_query_full_parity(B, heads, H, W, d, G, split):
    inp = make(B, heads, H, W, d, G, G + d)
    got = to_f64(gpu(inp, H, W, split))
    ref = oracle.global_query_attention(inp["gq"], inp["k"], inp["v"], inp["gk"], inp["gv"], B=B, heads=heads,
                                        H=H, W=W, d=d, G=G)
    m = compare(got, ref)
    log_metrics(f"global query {B}x{heads} {H}x{W} d{d} G{G} split={split}", m)
    assert passes(m), m


_FLUX_REF = {}


@pytest.mark.parametrize("split", [False, True])
def test_global_query_flux_shape_every_row(split):
    """FLUX-like 4096^2 joint attention, text half: 512 text queries x
    (65,536 image + 512 text) keys, 24 heads, d = 128, every output row."""
    import patch_res_diffusion_b200 as npa
    B, heads, H, W, d, G = 1, 24, 256, 256, 128, 512
    inp = make(B, heads, H, W, d, G, 5)
    if split:
        assert npa.npa_global_query_workspace_size(B, heads, H, W, d, G) > 0
    got = to_f64(gpu(inp, H, W, split))
    if "ref" not in _FLUX_REF:
        _FLUX_REF["ref"] = oracle.global_query_attention(inp["gq"], inp["k"], inp["v"], inp["gk"], inp["gv"], B=B,
                                                         heads=heads, H=H, W=W, d=d, G=G)
    m = compare(got, _FLUX_REF["ref"])
    log_metrics(f"global query FLUX split={split} (every row)", m)
    assert passes(m), m


@pytest.mark.parametrize("i", range(8))
def test_random_global_query_shapes(i):
    """Seeded random text-query shapes, split and unsplit, against the oracle."""
    rng = np.random.default_rng(300 + i)
    B, heads = int(rng.integers(1, 3)), int(rng.integers(1, 6))
    H, W, d, G = int(rng.integers(1, 48)), int(rng.integers(1, 48)), int(rng.choice([64, 128])), int(rng.integers(1, 400))
    inp = make(B, heads, H, W, d, G, 400 + i)
    ref = oracle.global_query_attention(inp["gq"], inp["k"], inp["v"], inp["gk"], inp["gv"], B=B, heads=heads, H=H,
                                        W=W, d=d, G=G)
    for split in (False, True):
        m = compare(to_f64(gpu(inp, H, W, split)), ref)
        log_metrics(f"random global query {B}x{heads} {H}x{W} d{d} G{G} split={split}", m)
        assert passes(m), (B, heads, H, W, d, G, split, m)
