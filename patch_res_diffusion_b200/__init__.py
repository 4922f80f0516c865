"""B200 (sm_100a) patch-restricted self-attention: Python binding.

A thin ctypes layer over the C ABI in ``include/npa.h`` (``libnpa_b200.so``,
built in-tree by ``patch_res_diffusion_b200.build``). The functions below carry
the C names and only marshal arguments; every step of the computation runs in
the library's CUDA kernels. There is no fallback: if the library is missing or
a call fails, an exception is raised.

* ``npa_attention_fwd`` - Neighborhood Patch Attention (ScaleDiff summary,
  "Approach"): non-overlapping query patches, each attending to its patch
  grown by a margin and clipped to the grid.
* ``pcpp_attention_fwd`` - partially conditioned attention (PCPP review, "What
  carries the argument"): row strips attending to themselves plus the nearest
  ceil(p * rows) rows of each adjacent strip.
* ``pcpp_attention_fwd_stale`` - PCPP as it runs across devices (PCPP review,
  "Core claim"): the strip's own keys from the current step, the borrowed
  neighbour rows from the previous step's keys/values.
* ``npa_global_query_attention_fwd`` (and ``..._noalloc``) - the text-query
  half of joint attention: global tokens as queries over all keys.
* ``npa_multidiffusion_attention_fwd`` - the overlapping-window comparator
  (ScaleDiff summary, "Approach": MultiDiffusion averages overlapping
  patches): each NPA window attends within itself and a token's output is the
  mean over the windows that contain it.
* ``asg_guidance_combine`` - asynchronous structure guidance (ASGDiffusion
  review, "core_discovery"): eps + w_t * M * (eps_ref - eps) per patch.

The lower-case helpers (``npa_attention``, ``pcpp_attention``,
``pcpp_attention_stale``, ``global_query_attention``,
``multidiffusion_attention``, ``asg_combine``) take torch CUDA tensors and
allocate outputs and workspaces; the computation is the same C call.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

__all__ = [
    "NpaError", "lib", "LIB_PATH", "NPA_OK", "NPA_ERR_INVALID_ARG", "NPA_ERR_UNSUPPORTED",
    "NPA_ERR_MISALIGNED", "NPA_ERR_CUDA", "NPA_ERR_DEVICE_TIMEOUT", "npa_attention_fwd",
    "pcpp_attention_fwd", "pcpp_neighbor_rows", "npa_useful_flops", "pcpp_useful_flops",
    "npa_device_status", "npa_selftest_wait_timeout", "npa_status_string", "npa_attention",
    "pcpp_attention", "pcpp_attention_fwd_stale", "pcpp_attention_stale", "npa_global_query_attention_fwd",
    "npa_global_query_workspace_size", "npa_global_query_attention_fwd_noalloc", "global_query_attention",
    "npa_multidiffusion_attention_fwd", "npa_multidiffusion_workspace_size", "npa_multidiffusion_useful_flops",
    "multidiffusion_attention", "asg_guidance_combine", "asg_combine", "EXPORTED_SYMBOLS", "DEBUG_LIB_PATH",
    "DEBUG_ONLY_SYMBOLS", "NPA_ERR_DEVICE_BOUNDS", "use_bounds_checking", "npa_debug_withhold_arrival_once",
]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libnpa_b200.so")
DEBUG_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libnpa_b200_debug.so")

NPA_OK = 0
NPA_ERR_INVALID_ARG = 1
NPA_ERR_UNSUPPORTED = 2
NPA_ERR_MISALIGNED = 3
NPA_ERR_CUDA = 4
NPA_ERR_DEVICE_TIMEOUT = 5
NPA_ERR_DEVICE_BOUNDS = 6

EXPORTED_SYMBOLS = (
    "npa_attention_fwd", "pcpp_attention_fwd", "pcpp_attention_fwd_stale", "pcpp_neighbor_rows", "npa_useful_flops",
    "pcpp_useful_flops", "npa_device_status", "npa_selftest_wait_timeout", "npa_status_string",
    "npa_global_query_attention_fwd", "npa_global_query_workspace_size",
    "npa_global_query_attention_fwd_noalloc", "npa_multidiffusion_attention_fwd",
    "npa_multidiffusion_workspace_size", "npa_multidiffusion_useful_flops", "asg_guidance_combine",
)
# exported by the bounds-checking build only
DEBUG_ONLY_SYMBOLS = ("npa_debug_withhold_arrival_once",)


class NpaError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"{what}: {npa_status_string(code)} ({code})")
        self.code = code


class _GlobalKV(ctypes.Structure):
    _fields_ = [("k", ctypes.c_void_p), ("v", ctypes.c_void_p), ("n_tokens", ctypes.c_int)]


_LIB: Optional[ctypes.CDLL] = None
_LOADED = {}


def lib() -> ctypes.CDLL:
    """The C library in use (the normal build unless use_bounds_checking(True)
    switched to the bounds-checking one). Raises if it has not been built."""
    global _LIB
    if _LIB is None:
        _LIB = _load(LIB_PATH)
    return _LIB


def use_bounds_checking(on: bool) -> None:
    """Routes every call of this module to the bounds-checking build
    (``libnpa_b200_debug.so``: device-side checks of every TMA box origin and
    output row, NPA_ERR_DEVICE_BOUNDS on a failure) or back to the normal one.
    Each library keeps its own device status word."""
    global _LIB
    _LIB = _load(DEBUG_LIB_PATH if on else LIB_PATH)


def _load(path: str) -> ctypes.CDLL:
    if path not in _LOADED:
        if not os.path.exists(path):
            raise ImportError(f"{path} is missing: build it with `python -m patch_res_diffusion_b200.build`")
        L = ctypes.CDLL(path)
        vp, i, d = ctypes.c_void_p, ctypes.c_int, ctypes.c_double
        gkv = ctypes.POINTER(_GlobalKV)
        L.npa_attention_fwd.argtypes = [vp, vp, vp, vp, i, i, i, i, i, i, i, gkv, vp]
        L.npa_attention_fwd.restype = i
        L.pcpp_attention_fwd.argtypes = [vp, vp, vp, vp, i, i, i, i, i, i, d, gkv, vp]
        L.pcpp_attention_fwd.restype = i
        L.pcpp_attention_fwd_stale.argtypes = [vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, d, i, i, gkv, vp]
        L.pcpp_attention_fwd_stale.restype = i
        L.npa_global_query_attention_fwd.argtypes = [vp] * 6 + [i] * 6 + [vp, ctypes.c_size_t, vp]
        L.npa_global_query_attention_fwd.restype = i
        L.npa_global_query_attention_fwd_noalloc.argtypes = [vp] * 6 + [i] * 6 + [vp]
        L.npa_global_query_attention_fwd_noalloc.restype = i
        L.npa_multidiffusion_attention_fwd.argtypes = [vp, vp, vp, vp, i, i, i, i, i, i, i, gkv, vp,
                                                       ctypes.c_size_t, vp]
        L.npa_multidiffusion_attention_fwd.restype = i
        L.npa_multidiffusion_workspace_size.argtypes = [i] * 7
        L.npa_multidiffusion_workspace_size.restype = ctypes.c_size_t
        L.npa_multidiffusion_useful_flops.argtypes = [i] * 8
        L.npa_multidiffusion_useful_flops.restype = d
        L.asg_guidance_combine.argtypes = [vp] * 4 + [i] * 4 + [ctypes.c_float, vp]
        L.asg_guidance_combine.restype = i
        L.npa_global_query_workspace_size.argtypes = [i] * 6
        L.npa_global_query_workspace_size.restype = ctypes.c_size_t
        L.pcpp_neighbor_rows.argtypes = [i, d]
        L.pcpp_neighbor_rows.restype = i
        L.npa_useful_flops.argtypes = [i, i, i, i, i, i, i, i]
        L.npa_useful_flops.restype = d
        L.pcpp_useful_flops.argtypes = [i, i, i, i, i, i, d, i]
        L.pcpp_useful_flops.restype = d
        L.npa_device_status.argtypes = [vp]
        L.npa_device_status.restype = i
        L.npa_selftest_wait_timeout.argtypes = [ctypes.c_uint32, vp]
        L.npa_selftest_wait_timeout.restype = i
        L.npa_status_string.argtypes = [i]
        L.npa_status_string.restype = ctypes.c_char_p
        if path == DEBUG_LIB_PATH:
            L.npa_debug_withhold_arrival_once.argtypes = [ctypes.c_uint32]
            L.npa_debug_withhold_arrival_once.restype = i
        _LOADED[path] = L
    return _LOADED[path]


def _ptr(x) -> Optional[int]:
    """Device address of a tensor (``data_ptr``) or a raw integer address."""
    if x is None:
        return None
    if hasattr(x, "data_ptr"):
        return int(x.data_ptr())
    return int(x)


def _stream(stream) -> Optional[int]:
    if stream is None:
        try:
            import torch
            if torch.cuda.is_available():
                return int(torch.cuda.current_stream().cuda_stream)
        except ImportError:
            pass
        return None
    if hasattr(stream, "cuda_stream"):
        return int(stream.cuda_stream)
    return int(stream)


def _gkv(global_k, global_v, n_tokens: int):
    if not n_tokens:
        return None
    return ctypes.byref(_GlobalKV(_ptr(global_k), _ptr(global_v), int(n_tokens)))


def _check(code: int, what: str) -> None:
    if code != NPA_OK:
        raise NpaError(code, what)


def npa_attention_fwd(q, k, v, o, B: int, heads: int, H: int, W: int, d: int, patch: int, margin: int,
                      global_k=None, global_v=None, n_global: int = 0, stream=None) -> None:
    """C ``npa_attention_fwd``: bf16 [B, heads, H*W, d] device buffers."""
    _check(lib().npa_attention_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), B, heads, H, W, d, patch, margin,
                                   _gkv(global_k, global_v, n_global), _stream(stream)),
           "npa_attention_fwd")


def pcpp_attention_fwd(q, k, v, o, B: int, heads: int, H: int, W: int, d: int, n_strips: int, p: float,
                       global_k=None, global_v=None, n_global: int = 0, stream=None) -> None:
    """C ``pcpp_attention_fwd``: bf16 [B, heads, H*W, d] device buffers."""
    _check(lib().pcpp_attention_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), B, heads, H, W, d, n_strips,
                                    float(p), _gkv(global_k, global_v, n_global), _stream(stream)),
           "pcpp_attention_fwd")


def pcpp_attention_fwd_stale(q, k, v, k_stale, v_stale, o, B: int, heads: int, H: int, W: int, d: int,
                             n_strips: int, p: float, strip_begin: int, strip_count: int, global_k=None,
                             global_v=None, n_global: int = 0, stream=None) -> None:
    """C ``pcpp_attention_fwd_stale``: own-strip keys from k/v, borrowed rows from k_stale/v_stale."""
    _check(lib().pcpp_attention_fwd_stale(_ptr(q), _ptr(k), _ptr(v), _ptr(k_stale), _ptr(v_stale), _ptr(o), B,
                                          heads, H, W, d, n_strips, float(p), strip_begin, strip_count,
                                          _gkv(global_k, global_v, n_global), _stream(stream)),
           "pcpp_attention_fwd_stale")


def npa_global_query_attention_fwd(gq, k, v, gk, gv, go, B: int, heads: int, H: int, W: int, d: int, G: int,
                                   workspace=None, workspace_bytes: int = 0, stream=None) -> None:
    """C ``npa_global_query_attention_fwd``: global-token queries over all keys."""
    _check(lib().npa_global_query_attention_fwd(_ptr(gq), _ptr(k), _ptr(v), _ptr(gk), _ptr(gv), _ptr(go), B, heads,
                                                H, W, d, G, _ptr(workspace), int(workspace_bytes),
                                                _stream(stream)),
           "npa_global_query_attention_fwd")


def npa_global_query_attention_fwd_noalloc(gq, k, v, gk, gv, go, B: int, heads: int, H: int, W: int, d: int,
                                           G: int, stream=None) -> None:
    """C ``npa_global_query_attention_fwd_noalloc``: the same computation with
    the split partials in the library's fixed device array (no caller memory)."""
    _check(lib().npa_global_query_attention_fwd_noalloc(_ptr(gq), _ptr(k), _ptr(v), _ptr(gk), _ptr(gv), _ptr(go),
                                                        B, heads, H, W, d, G, _stream(stream)),
           "npa_global_query_attention_fwd_noalloc")


def npa_multidiffusion_attention_fwd(q, k, v, o, B: int, heads: int, H: int, W: int, d: int, patch: int,
                                     margin: int, workspace, workspace_bytes: int, global_k=None, global_v=None,
                                     n_global: int = 0, stream=None) -> None:
    """C ``npa_multidiffusion_attention_fwd``: overlapping-window attention;
    ``workspace`` holds npa_multidiffusion_workspace_size() bytes."""
    _check(lib().npa_multidiffusion_attention_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), B, heads, H, W, d, patch,
                                                  margin, _gkv(global_k, global_v, n_global), _ptr(workspace),
                                                  int(workspace_bytes), _stream(stream)),
           "npa_multidiffusion_attention_fwd")


def npa_multidiffusion_workspace_size(B, heads, H, W, d, patch, margin) -> int:
    return int(lib().npa_multidiffusion_workspace_size(B, heads, H, W, d, patch, margin))


def npa_multidiffusion_useful_flops(B, heads, H, W, d, patch, margin, G=0) -> float:
    return float(lib().npa_multidiffusion_useful_flops(B, heads, H, W, d, patch, margin, G))


def asg_guidance_combine(eps, eps_ref, mask, out, n_patches: int, B: int, C: int, S: int, w_t: float,
                         stream=None) -> None:
    """C ``asg_guidance_combine``: out = eps + w_t * mask * (eps_ref - eps)."""
    _check(lib().asg_guidance_combine(_ptr(eps), _ptr(eps_ref), _ptr(mask), _ptr(out), n_patches, B, C, S,
                                      float(w_t), _stream(stream)),
           "asg_guidance_combine")


def npa_global_query_workspace_size(B, heads, H, W, d, G) -> int:
    return int(lib().npa_global_query_workspace_size(B, heads, H, W, d, G))


def pcpp_neighbor_rows(strip_rows: int, p: float) -> int:
    return int(lib().pcpp_neighbor_rows(strip_rows, float(p)))


def npa_useful_flops(B, heads, H, W, d, patch, margin, G=0) -> float:
    return float(lib().npa_useful_flops(B, heads, H, W, d, patch, margin, G))


def pcpp_useful_flops(B, heads, H, W, d, n_strips, p, G=0) -> float:
    return float(lib().pcpp_useful_flops(B, heads, H, W, d, n_strips, float(p), G))


def npa_device_status(stream=None) -> int:
    return int(lib().npa_device_status(_stream(stream)))


def npa_selftest_wait_timeout(limit_us: int, stream=None) -> None:
    _check(lib().npa_selftest_wait_timeout(int(limit_us), _stream(stream)), "npa_selftest_wait_timeout")


def npa_debug_withhold_arrival_once(wait_limit_us: int) -> None:
    """C ``npa_debug_withhold_arrival_once`` (bounds-checking build only):
    the next attention launch's first CTA withholds one arrival and its
    bounded waits of ``wait_limit_us`` run out (the abort path)."""
    L = lib()
    if not hasattr(L, "npa_debug_withhold_arrival_once"):
        raise NpaError(NPA_ERR_UNSUPPORTED, "npa_debug_withhold_arrival_once needs use_bounds_checking(True)")
    _check(L.npa_debug_withhold_arrival_once(int(wait_limit_us)), "npa_debug_withhold_arrival_once")


def npa_status_string(code: int) -> str:
    try:
        return lib().npa_status_string(int(code)).decode()
    except ImportError:
        return f"status {code}"


# ---------------------------------------------------------------------------
# torch conveniences (allocation of the output only; the call is the C one)
# ---------------------------------------------------------------------------

def _shape(q, H, W):
    if q.dim() != 4 or q.shape[2] != H * W:
        raise ValueError(f"expected [B, heads, H*W={H * W}, d], got {tuple(q.shape)}")
    return int(q.shape[0]), int(q.shape[1]), int(q.shape[3])


def npa_attention(q, k, v, H: int, W: int, patch: int, margin: int, global_k=None, global_v=None,
                  out=None, stream=None):
    """NPA forward on torch bf16 CUDA tensors [B, heads, H*W, d]; returns ``out``."""
    B, heads, d = _shape(q, H, W)
    if out is None:
        out = q.new_empty(q.shape)
    G = 0 if global_k is None else int(global_k.shape[2])
    npa_attention_fwd(q, k, v, out, B, heads, H, W, d, patch, margin, global_k, global_v, G, stream)
    return out


def pcpp_attention(q, k, v, H: int, W: int, n_strips: int, p: float, global_k=None, global_v=None,
                   out=None, stream=None):
    """PCPP forward on torch bf16 CUDA tensors [B, heads, H*W, d]; returns ``out``."""
    B, heads, d = _shape(q, H, W)
    if out is None:
        out = q.new_empty(q.shape)
    G = 0 if global_k is None else int(global_k.shape[2])
    pcpp_attention_fwd(q, k, v, out, B, heads, H, W, d, n_strips, p, global_k, global_v, G, stream)
    return out


def pcpp_attention_stale(q, k, v, k_stale, v_stale, H: int, W: int, n_strips: int, p: float, strips=None,
                         global_k=None, global_v=None, out=None, stream=None):
    """Two-source PCPP forward on torch bf16 CUDA tensors; ``strips`` is an
    optional (begin, count) range of strips to compute (default: all)."""
    B, heads, d = _shape(q, H, W)
    if out is None:
        out = q.new_empty(q.shape)
    begin, count = (0, n_strips) if strips is None else strips
    G = 0 if global_k is None else int(global_k.shape[2])
    pcpp_attention_fwd_stale(q, k, v, k_stale, v_stale, out, B, heads, H, W, d, n_strips, p, begin, count,
                             global_k, global_v, G, stream)
    return out


def global_query_attention(gq, k, v, gk, gv, H: int, W: int, out=None, split: bool = True, stream=None):
    """Global-token queries [B, heads, G, d] over all image and global keys
    (torch bf16 CUDA tensors); with ``split`` a workspace is allocated so the
    key range can be split across the GPU."""
    import torch
    B, heads, G, d = (int(x) for x in gq.shape)
    if out is None:
        out = gq.new_empty(gq.shape)
    ws, nbytes = None, 0
    if split:
        nbytes = npa_global_query_workspace_size(B, heads, H, W, d, G)
        if nbytes:
            ws = torch.empty(nbytes, dtype=torch.uint8, device=gq.device)
    npa_global_query_attention_fwd(gq, k, v, gk, gv, out, B, heads, H, W, d, G, ws, nbytes, stream)
    return out


def multidiffusion_attention(q, k, v, H: int, W: int, patch: int, margin: int, global_k=None, global_v=None,
                             out=None, workspace=None, stream=None):
    """Overlapping-window attention on torch bf16 CUDA tensors [B, heads,
    H*W, d]; allocates the float32 window workspace unless one is given."""
    import torch
    B, heads, d = _shape(q, H, W)
    if out is None:
        out = q.new_empty(q.shape)
    nbytes = npa_multidiffusion_workspace_size(B, heads, H, W, d, patch, margin)
    if workspace is None:
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=q.device)
    G = 0 if global_k is None else int(global_k.shape[2])
    npa_multidiffusion_attention_fwd(q, k, v, out, B, heads, H, W, d, patch, margin, workspace,
                                     workspace.numel() * workspace.element_size(), global_k, global_v, G, stream)
    return out


def asg_combine(eps, eps_ref, mask, w_t: float, out=None, stream=None):
    """ASG combine on torch bf16 CUDA tensors: eps [n, B, C, S], eps_ref
    [B, C, S], mask [n, B, S]; ``out=eps`` works in place."""
    n, B, C, S = (int(x) for x in eps.shape)
    if out is None:
        out = eps.new_empty(eps.shape)
    asg_guidance_combine(eps, eps_ref, mask, out, n, B, C, S, w_t, stream)
    return out
