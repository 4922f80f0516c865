"""The allocation-free variant of the text-query attention.

Some callers cannot give the library device memory - a plugin whose host
framework owns every allocation, or a service that forbids cudaMalloc after
start-up because it can synchronise the device. For them
npa_global_query_attention_fwd_noalloc keeps the key-range split partials in
a fixed array inside the library. These tests call it through the C ABI and
check it, on two calls in a row with different inputs (the array keeps the
previous call's contents), against the entry point that takes a caller
workspace and against the float64 oracle; at the FLUX text shape the array
holds fewer partials than the split plan asks for, so the capped split count
is exercised too. Problems too large for the array are refused. This file is
collected last."""
import numpy as np
import pytest

import oracle
from workloads import f64_to_bf16_bits
from _parity import compare, log_metrics, passes, to_device, to_f64

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def npa():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from patch_res_diffusion_b200 import build
    build.build()
    import patch_res_diffusion_b200 as m
    m.lib()
    return m


def _inputs(B, heads, H, W, d, G, seed):
    rng = np.random.default_rng(seed)
    r = lambda shape: f64_to_bf16_bits(rng.standard_normal(shape))
    return {"gq": r((B, heads, G, d)), "k": r((B, heads, H * W, d)), "v": r((B, heads, H * W, d)),
            "gk": r((B, heads, G, d)), "gv": r((B, heads, G, d))}


def _both_calls(npa, B, heads, H, W, d, G, inp):
    """One call of the workspace entry point and one of the no-alloc entry
    point on the same inputs; returns both outputs (bf16, device)."""
    L = npa.lib()
    t = {n: to_device(a) for n, a in inp.items()}
    ws_bytes = npa.npa_global_query_workspace_size(B, heads, H, W, d, G)
    ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    ref = torch.full_like(t["gq"], float("nan"))
    got = torch.full_like(t["gq"], float("nan"))
    ptrs = [t[n].data_ptr() for n in ("gq", "k", "v", "gk", "gv")]
    rc = L.npa_global_query_attention_fwd(*ptrs, ref.data_ptr(), B, heads, H, W, d, G, ws.data_ptr(), ws_bytes,
                                          stream)
    assert rc == npa.NPA_OK
    rc = L.npa_global_query_attention_fwd_noalloc(*ptrs, got.data_ptr(), B, heads, H, W, d, G, stream)
    assert rc == npa.NPA_OK
    torch.cuda.synchronize()
    return got, ref


@pytest.mark.parametrize("shape", [
    # B, heads, H, W, d, G: split across the GPU, the array holds every planned partial
    (1, 8, 128, 128, 128, 256),
    # the FLUX text shape (24 heads, 512 text tokens, d = 128) on a small grid:
    # 6.4 MB per partial, so the 16 MiB array caps the split count at 2
    (1, 24, 32, 32, 128, 512),
], ids=["split_fits", "flux_text_capped"])
def test_noalloc_matches_workspace_entry_point_and_oracle_on_two_calls(npa, shape):
    B, heads, H, W, d, G = shape
    assert npa.npa_global_query_workspace_size(B, heads, H, W, d, G) > 0  # the plan splits the key range
    for call in range(2):
        inp = _inputs(B, heads, H, W, d, G, seed=10 + call)
        got, ref = _both_calls(npa, B, heads, H, W, d, G, inp)
        m = compare(to_f64(got), to_f64(ref))
        assert passes(m), (call, m)
        expect = oracle.global_query_attention(inp["gq"], inp["k"], inp["v"], inp["gk"], inp["gv"], B=B,
                                               heads=heads, H=H, W=W, d=d, G=G)
        m = compare(to_f64(got), expect)
        log_metrics(f"noalloc {B}x{heads} G{G} d{d} call {call}", m)
        assert passes(m), (call, m)
    assert npa.npa_device_status() == npa.NPA_OK


def test_noalloc_refuses_problems_larger_than_its_array(npa):
    # 64 heads x 2048 global tokens x (128 + 2) x 4 bytes = 68 MB per partial > 16 MiB
    B, heads, H, W, d, G = 1, 64, 16, 16, 128, 2048
    t = {n: to_device(a) for n, a in _inputs(B, heads, H, W, d, G, seed=3).items()}
    go = torch.zeros_like(t["gq"])
    rc = npa.lib().npa_global_query_attention_fwd_noalloc(
        *[t[n].data_ptr() for n in ("gq", "k", "v", "gk", "gv")], go.data_ptr(), B, heads, H, W, d, G,
        torch.cuda.current_stream().cuda_stream)
    assert rc == npa.NPA_ERR_UNSUPPORTED
    torch.cuda.synchronize()
    assert int(go.abs().max()) == 0  # nothing was launched
