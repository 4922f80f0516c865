"""The C-ABI library on the host: it loads, exports every symbol the header
declares, validates arguments before touching a GPU, and its geometry helpers
agree with the oracle's brute-force counts. No compute call is made here."""
import ctypes
import os
import re
import subprocess

import numpy as np
import pytest

import oracle
import patch_res_diffusion_b200 as npa
from workloads import PRESETS

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "npa.h")


def header_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\*?\s*([a-z_][a-z0-9_]*)\s*\(",
                                 src, flags=re.M)))


@pytest.fixture(scope="module")
def L():
    from patch_res_diffusion_b200 import build
    build.build()
    return npa.lib()


def test_header_declares_the_bound_symbols():
    assert header_functions() == sorted(npa.EXPORTED_SYMBOLS + npa.DEBUG_ONLY_SYMBOLS)


def _exported(path):
    out = subprocess.run(["nm", "-D", "--defined-only", path], capture_output=True, text=True, check=True).stdout
    return {line.split()[-1] for line in out.splitlines() if " T " in line}


def test_library_exports_every_header_symbol(L):
    exported = _exported(npa.LIB_PATH)
    for name in npa.EXPORTED_SYMBOLS:
        assert name in exported, name
        assert getattr(L, name) is not None
    for name in npa.DEBUG_ONLY_SYMBOLS:   # the bounds-checking build's own entry points
        assert name not in exported, name


def test_bounds_checking_library_exports_every_header_symbol(L):
    exported = _exported(npa.DEBUG_LIB_PATH)
    for name in header_functions():
        assert name in exported, name


def test_status_strings(L):
    for code, name in [(0, "NPA_OK"), (1, "NPA_ERR_INVALID_ARG"), (2, "NPA_ERR_UNSUPPORTED"),
                       (3, "NPA_ERR_MISALIGNED"), (4, "NPA_ERR_CUDA"), (5, "NPA_ERR_DEVICE_TIMEOUT"),
                       (6, "NPA_ERR_DEVICE_BOUNDS")]:
        assert npa.npa_status_string(code) == name
    assert npa.npa_status_string(99) == "NPA_ERR_UNKNOWN"


# fake, never dereferenced addresses: validation rejects these calls before any CUDA call
A, B_, C_, O_ = 0x10000, 0x20000000, 0x40000000, 0x60000000


def _npa(L, q=A, k=B_, v=C_, o=O_, B=1, h=1, H=8, W=8, d=64, P=4, m=1, g=None):
    return L.npa_attention_fwd(q, k, v, o, B, h, H, W, d, P, m, g, None)


def _pcpp(L, q=A, k=B_, v=C_, o=O_, B=1, h=1, H=8, W=8, d=64, n=2, p=0.5, g=None):
    return L.pcpp_attention_fwd(q, k, v, o, B, h, H, W, d, n, p, g, None)


def test_null_and_size_arguments_rejected(L):
    assert _npa(L, q=None) == npa.NPA_ERR_INVALID_ARG
    assert _npa(L, o=None) == npa.NPA_ERR_INVALID_ARG
    assert _npa(L, B=0) == npa.NPA_ERR_INVALID_ARG
    assert _npa(L, H=0) == npa.NPA_ERR_INVALID_ARG
    assert _npa(L, P=0) == npa.NPA_ERR_INVALID_ARG
    assert _npa(L, m=-1) == npa.NPA_ERR_INVALID_ARG
    assert _pcpp(L, n=0) == npa.NPA_ERR_INVALID_ARG


def test_sizes_past_the_tensor_map_limits_rejected(L):
    # a 2^20 x 2^20 grid at d = 64 needs 2^47-byte row strides: refused before any CUDA call
    assert _npa(L, H=1 << 20, W=1 << 20) == npa.NPA_ERR_UNSUPPORTED
    assert _pcpp(L, H=1 << 20, W=1 << 20, n=1) == npa.NPA_ERR_UNSUPPORTED


def test_unsupported_head_dim(L):
    for d in (16, 32, 96, 256):
        assert _npa(L, d=d) == npa.NPA_ERR_UNSUPPORTED
        assert _pcpp(L, d=d) == npa.NPA_ERR_UNSUPPORTED


def test_misaligned_pointers(L):
    assert _npa(L, q=A + 8) == npa.NPA_ERR_MISALIGNED
    assert _npa(L, o=O_ + 2) == npa.NPA_ERR_MISALIGNED
    g = ctypes.byref(npa._GlobalKV(0x70000008, 0x78000000, 5))
    assert _npa(L, g=g) == npa.NPA_ERR_MISALIGNED


def test_overlapping_output_rejected(L):
    assert _npa(L, o=A + 64) == npa.NPA_ERR_INVALID_ARG
    assert _pcpp(L, o=C_) == npa.NPA_ERR_INVALID_ARG
    g = ctypes.byref(npa._GlobalKV(O_ + 16, 0x78000000, 5))
    assert _npa(L, g=g) == npa.NPA_ERR_INVALID_ARG


def test_global_token_arguments(L):
    assert _npa(L, g=ctypes.byref(npa._GlobalKV(None, 0x78000000, 5))) == npa.NPA_ERR_INVALID_ARG
    assert _npa(L, g=ctypes.byref(npa._GlobalKV(0x70000000, 0x78000000, -1))) == npa.NPA_ERR_INVALID_ARG


def test_pcpp_argument_domain(L):
    assert _pcpp(L, H=9, n=2) == npa.NPA_ERR_INVALID_ARG          # strips must divide H
    assert _pcpp(L, p=1.5) == npa.NPA_ERR_INVALID_ARG
    assert _pcpp(L, p=-0.1) == npa.NPA_ERR_INVALID_ARG
    assert _pcpp(L, p=float("nan")) == npa.NPA_ERR_INVALID_ARG


@pytest.mark.parametrize("s", list(range(1, 70)))
def test_neighbor_rows_agree_with_oracle(s):
    for p in np.round(np.linspace(0, 1, 41), 6).tolist() + [0.3, 0.7, 0.8, 1 / 3, 2 / 3]:
        assert npa.pcpp_neighbor_rows(s, p) == oracle.pcpp_neighbor_rows(s, p), (s, p)
    assert npa.pcpp_neighbor_rows(s, 1.01) == -1


@pytest.mark.parametrize("name", list(PRESETS))
def test_useful_flops_match_oracle_pair_count(name):
    w = PRESETS[name]
    pairs = oracle.pair_count(w.geometry, w.H, w.W, patch=w.patch, margin=w.margin, n_strips=w.n_strips,
                              p=w.p, G=w.G)
    expect = 4.0 * w.d * w.B * w.heads * pairs
    if w.geometry == "npa":
        got = npa.npa_useful_flops(w.B, w.heads, w.H, w.W, w.d, w.patch, w.margin, w.G)
    else:
        got = npa.pcpp_useful_flops(w.B, w.heads, w.H, w.W, w.d, w.n_strips, w.p, w.G)
    assert got == expect


@pytest.mark.parametrize("H,W,P,m,G", [(17, 23, 5, 3, 0), (9, 31, 8, 0, 7), (40, 13, 64, 2, 1), (30, 30, 7, 30, 0)])
def test_useful_flops_ragged_npa(H, W, P, m, G):
    pairs = oracle.pair_count("npa", H, W, patch=P, margin=m, G=G)
    assert npa.npa_useful_flops(2, 3, H, W, 128, P, m, G) == 4.0 * 128 * 6 * pairs


@pytest.mark.parametrize("H,W,n,p,G", [(30, 7, 5, 0.45, 0), (24, 9, 8, 1.0, 3), (12, 5, 1, 0.5, 0)])
def test_useful_flops_pcpp(H, W, n, p, G):
    pairs = oracle.pair_count("pcpp", H, W, n_strips=n, p=p, G=G)
    assert npa.pcpp_useful_flops(1, 2, H, W, 64, n, p, G) == 4.0 * 64 * 2 * pairs


def test_flops_helper_rejects_bad_geometry():
    assert npa.npa_useful_flops(1, 1, 8, 8, 64, 0, 1) < 0
    assert npa.pcpp_useful_flops(1, 1, 9, 8, 64, 2, 0.5) < 0
    assert npa.pcpp_useful_flops(1, 1, 8, 8, 64, 2, 1.5) < 0


def _stale(L, q=A, k=B_, v=C_, ks=0x30000000, vs=0x50000000, o=O_, H=8, n=2, p=0.5, b=0, c=1, d=64):
    return L.pcpp_attention_fwd_stale(q, k, v, ks, vs, o, 1, 1, H, 8, d, n, p, b, c, None, None)


def test_stale_entry_point_validation(L):
    assert _stale(L, ks=None) == npa.NPA_ERR_INVALID_ARG
    assert _stale(L, vs=None) == npa.NPA_ERR_INVALID_ARG
    assert _stale(L, ks=0x30000008) == npa.NPA_ERR_MISALIGNED
    assert _stale(L, o=0x30000000) == npa.NPA_ERR_INVALID_ARG       # output overlaps k_stale
    assert _stale(L, b=-1) == npa.NPA_ERR_INVALID_ARG
    assert _stale(L, c=0) == npa.NPA_ERR_INVALID_ARG
    assert _stale(L, b=1, c=2) == npa.NPA_ERR_INVALID_ARG            # past the last strip
    assert _stale(L, H=9) == npa.NPA_ERR_INVALID_ARG
    assert _stale(L, p=2.0) == npa.NPA_ERR_INVALID_ARG
    assert _stale(L, d=96) == npa.NPA_ERR_UNSUPPORTED


def test_global_query_validation(L):
    f = lambda gq=A, k=B_, v=C_, gk=0x30000000, gv=0x50000000, go=O_, G=5, d=64, ws=None: \
        L.npa_global_query_attention_fwd(gq, k, v, gk, gv, go, 1, 1, 8, 8, d, G, ws, 0, None)
    assert f(gq=None) == npa.NPA_ERR_INVALID_ARG
    assert f(gk=None) == npa.NPA_ERR_INVALID_ARG
    assert f(G=0) == npa.NPA_ERR_INVALID_ARG
    assert f(d=96) == npa.NPA_ERR_UNSUPPORTED
    assert f(go=O_ + 4) == npa.NPA_ERR_MISALIGNED
    assert f(go=A) == npa.NPA_ERR_INVALID_ARG          # output overlaps the queries
    assert f(ws=0x70000008) == npa.NPA_ERR_MISALIGNED
    assert L.npa_global_query_workspace_size(1, 1, 8, 8, 96, 5) == 0
    assert L.npa_global_query_workspace_size(1, 1, 8, 8, 64, 0) == 0


def test_multidiffusion_validation(L):
    ws_ok = L.npa_multidiffusion_workspace_size(1, 1, 8, 8, 64, 4, 2)
    f = lambda q=A, o=O_, ws=0x70000000, nb=ws_ok, patch=4, margin=2, d=64, H=8: \
        L.npa_multidiffusion_attention_fwd(q, B_, C_, o, 1, 1, H, 8, d, patch, margin, None, ws, nb, None)
    assert f(ws=None) == npa.NPA_ERR_INVALID_ARG
    assert f(ws=0x70000008) == npa.NPA_ERR_MISALIGNED
    assert f(nb=ws_ok - 1) == npa.NPA_ERR_INVALID_ARG                 # workspace too small
    assert f(ws=A) == npa.NPA_ERR_INVALID_ARG                         # workspace overlaps q
    assert f(ws=O_) == npa.NPA_ERR_INVALID_ARG                        # workspace overlaps o
    assert f(patch=0) == npa.NPA_ERR_INVALID_ARG
    assert f(margin=-1) == npa.NPA_ERR_INVALID_ARG
    assert f(d=96) == npa.NPA_ERR_UNSUPPORTED
    assert f(q=None) == npa.NPA_ERR_INVALID_ARG
    assert f(H=300, patch=1, margin=0, nb=1 << 40) == npa.NPA_ERR_UNSUPPORTED   # 300 patch rows > 256
    assert L.npa_multidiffusion_workspace_size(1, 1, 8, 8, 96, 4, 2) == 0
    assert L.npa_multidiffusion_workspace_size(1, 1, 8, 8, 64, 0, 2) == 0


@pytest.mark.parametrize("H,W,P,m,G", [(256, 256, 64, 32, 0), (40, 37, 16, 5, 7), (9, 7, 3, 2, 0),
                                       (64, 64, 16, 0, 3)])
def test_multidiffusion_flops_and_workspace_match_oracle_windows(H, W, P, m, G):
    d, B, h = 64, 2, 3
    assert npa.npa_multidiffusion_useful_flops(B, h, H, W, d, P, m, G) == \
        4.0 * d * B * h * oracle.md_pair_count(H, W, P, m, G)
    nph, npw = (H + P - 1) // P, (W + P - 1) // P
    # the windows of column 0 (width min(W, P + m)) and of row 0 (height
    # min(H, P + m)) give the per-axis extents
    hs = [len(oracle.md_window_keys(H, W, P, m, i, 0)) // min(W, P + m) for i in range(nph)]
    ws = [len(oracle.md_window_keys(H, W, P, m, 0, j)) // min(H, P + m) for j in range(npw)]
    assert npa.npa_multidiffusion_workspace_size(B, h, H, W, d, P, m) == 4 * d * B * h * sum(hs) * sum(ws)


def test_asg_validation(L):
    f = lambda eps=A, ref=B_, m=C_, out=O_, n=2, B=1, C=4, S=64, w=1.5: \
        L.asg_guidance_combine(eps, ref, m, out, n, B, C, S, w, None)
    assert f(eps=None) == npa.NPA_ERR_INVALID_ARG
    assert f(out=None) == npa.NPA_ERR_INVALID_ARG
    assert f(n=0) == npa.NPA_ERR_INVALID_ARG
    assert f(S=0) == npa.NPA_ERR_INVALID_ARG
    assert f(w=float("nan")) == npa.NPA_ERR_INVALID_ARG
    assert f(w=float("inf")) == npa.NPA_ERR_INVALID_ARG
    assert f(m=C_ + 2) == npa.NPA_ERR_MISALIGNED
    assert f(out=A + 16) == npa.NPA_ERR_INVALID_ARG        # partly overlaps eps (only exact in-place is allowed)
    assert f(out=B_) == npa.NPA_ERR_INVALID_ARG            # overlaps the reference
    assert f(out=C_) == npa.NPA_ERR_INVALID_ARG            # overlaps the mask
