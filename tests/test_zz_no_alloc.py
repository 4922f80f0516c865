"""The allocation-free variant of the text-query attention.

Some callers cannot give the library device memory - a plugin whose host
framework owns every allocation, or a service that forbids cudaMalloc after
start-up because it can synchronise the device. For them
npa_global_query_attention_fwd_noalloc keeps the key-range split partials in
a fixed array inside the library. These tests call it through the C ABI and
check it against the entry point that takes a caller workspace, on two
calls in a row (the array keeps the previous call's contents), and that
problems too large for the array are refused. This file is collected last."""
import numpy as np
import pytest

from workloads import f64_to_bf16_bits
from _parity import compare, passes, to_device, to_f64

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
    r = lambda shape: to_device(f64_to_bf16_bits(rng.standard_normal(shape)))
    return r((B, heads, G, d)), r((B, heads, H * W, d)), r((B, heads, H * W, d)), r((B, heads, G, d)), \
        r((B, heads, G, d))


def test_noalloc_matches_workspace_entry_point_on_two_calls(npa):
    B, heads, H, W, d, G = 1, 8, 128, 128, 128, 256
    L = npa.lib()
    ws_bytes = npa.npa_global_query_workspace_size(B, heads, H, W, d, G)
    assert ws_bytes > 0  # this shape is split across the GPU, so the fixed array is used
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    for call in range(2):
        gq, k, v, gk, gv = _inputs(B, heads, H, W, d, G, seed=10 + call)
        ref = torch.full_like(gq, float("nan"))
        got = torch.full_like(gq, float("nan"))
        rc = L.npa_global_query_attention_fwd(gq.data_ptr(), k.data_ptr(), v.data_ptr(), gk.data_ptr(),
                                              gv.data_ptr(), ref.data_ptr(), B, heads, H, W, d, G, ws.data_ptr(),
                                              ws_bytes, stream)
        assert rc == npa.NPA_OK
        rc = L.npa_global_query_attention_fwd_noalloc(gq.data_ptr(), k.data_ptr(), v.data_ptr(), gk.data_ptr(),
                                                      gv.data_ptr(), got.data_ptr(), B, heads, H, W, d, G, stream)
        assert rc == npa.NPA_OK
        torch.cuda.synchronize()
        m = compare(to_f64(got), to_f64(ref))
        assert passes(m), (call, m)
    assert npa.npa_device_status() == npa.NPA_OK


def test_noalloc_refuses_problems_larger_than_its_array(npa):
    # 64 heads x 2048 global tokens x (128 + 2) x 4 bytes = 68 MB per partial > 16 MiB
    B, heads, H, W, d, G = 1, 64, 16, 16, 128, 2048
    gq, k, v, gk, gv = _inputs(B, heads, H, W, d, G, seed=3)
    go = torch.zeros_like(gq)
    rc = npa.lib().npa_global_query_attention_fwd_noalloc(gq.data_ptr(), k.data_ptr(), v.data_ptr(), gk.data_ptr(),
                                                          gv.data_ptr(), go.data_ptr(), B, heads, H, W, d, G,
                                                          torch.cuda.current_stream().cuda_stream)
    assert rc == npa.NPA_ERR_UNSUPPORTED
    torch.cuda.synchronize()
    assert int(go.abs().max()) == 0  # nothing was launched
