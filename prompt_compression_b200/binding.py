"""ctypes binding of include/speckv.h: argument marshalling only.

Each function takes torch tensors that already live on the GPU, checks dtype,
device and contiguity, and passes raw pointers, sizes and the current CUDA
stream to the C entry point of the same name.  Output tensors are the
caller's; a workspace is allocated with torch only when none is given.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_PKG, "libspeckv.so")
_lib = None

SPK_OK, SPK_ERR_ARG, SPK_ERR_UNSUPPORTED, SPK_ERR_WORKSPACE, SPK_ERR_CUDA, SPK_ERR_TIMEOUT = range(6)
_STATUS = {0: "SPK_OK", 1: "SPK_ERR_ARG", 2: "SPK_ERR_UNSUPPORTED", 3: "SPK_ERR_WORKSPACE",
           4: "SPK_ERR_CUDA", 5: "SPK_ERR_TIMEOUT"}


class SpeckvError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{_STATUS.get(status, status)}: {message}")
        self.status = status


class SpeckvShape(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int), ("layers", ctypes.c_int), ("hq", ctypes.c_int),
                ("hkv", ctypes.c_int), ("head_dim", ctypes.c_int), ("n_in", ctypes.c_int),
                ("n_window", ctypes.c_int), ("n_lookahead", ctypes.c_int), ("scale", ctypes.c_float)]


class SpecpcShape(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int), ("layers", ctypes.c_int), ("l_skip", ctypes.c_int),
                ("hq", ctypes.c_int), ("hkv", ctypes.c_int), ("head_dim", ctypes.c_int),
                ("n_in", ctypes.c_int), ("n_rows", ctypes.c_int), ("n_lookahead", ctypes.c_int),
                ("scale", ctypes.c_float)]


def library_path() -> str:
    return _LIB_PATH


def load_library():
    """Load libspeckv.so; raises if it is missing (there is no fallback)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(_LIB_PATH):
        raise ImportError(f"{_LIB_PATH} is missing: build it with `python -m prompt_compression_b200.build`")
    lib = ctypes.CDLL(_LIB_PATH)
    vp, sz, I, F = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int, ctypes.c_float
    sk = ctypes.POINTER(SpeckvShape)
    sp = ctypes.POINTER(SpecpcShape)
    sig = {
        "speckv_workspace_size": (sz, [sk]),
        "speckv_score": (I, [sk, vp, vp, vp, vp, vp, sz, vp]),
        "speckv_row_lse": (I, [sk, vp, vp, vp, vp]),
        "specpc_workspace_size": (sz, [sp]),
        "specpc_score": (I, [sp, vp, vp, vp, vp, vp, sz, vp]),
        "topk_workspace_size": (sz, [I, I]),
        "topk_select": (I, [vp, I, I, I, I, I, vp, vp, vp, sz, vp]),
        "kv_compact": (I, [vp, vp, I, I, I, I, vp, I, I, vp, vp, vp]),
        "spk_last_error": (ctypes.c_char_p, []),
        "spk_device_error": (I, [ctypes.POINTER(I), ctypes.POINTER(I), I]),
        "spk_selftest_wait_timeout": (I, [ctypes.c_longlong, vp]),
        "spk_exp2_fma": (I, [vp, vp, I, vp]),
        "spk_mapped_host_pointer": (I, [vp, ctypes.POINTER(vp)]),
        "decode_attention": (I, [I, I, I, I, I, I, F, vp, vp, vp, vp, vp]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def _check(status: int):
    if status != SPK_OK:
        msg = load_library().spk_last_error().decode(errors="replace")
        raise SpeckvError(status, msg)


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _dev(t: Optional[torch.Tensor], name: str, dtype=None) -> Optional[int]:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr()


def mapped_host_pointer(t: torch.Tensor) -> int:
    """Device address of a page-locked host tensor (spk_mapped_host_pointer)."""
    if t.is_cuda or not t.is_pinned():
        raise ValueError("expected a page-locked (pinned) host tensor")
    dev = ctypes.c_void_p()
    _check(load_library().spk_mapped_host_pointer(ctypes.c_void_p(t.data_ptr()), ctypes.byref(dev)))
    return int(dev.value)


def _src(t: Optional[torch.Tensor], name: str) -> Optional[int]:
    """A gather source: a CUDA tensor, or a pinned host tensor read in place."""
    if t is None or t.is_cuda:
        return _dev(t, name)
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return mapped_host_pointer(t)


def _workspace(ws: Optional[torch.Tensor], nbytes: int, device) -> torch.Tensor:
    if ws is None:
        return torch.empty(max(nbytes, 256), dtype=torch.uint8, device=device)
    return ws


# --------------------------------------------------------------------- SpecKV
def speckv_shape(q: torch.Tensor, k: torch.Tensor, n_window: int, scale: float = 1.0) -> SpeckvShape:
    if q.dim() != 5 or k.dim() != 5:
        raise ValueError("q is [B, L, Hq, R, d] and k is [B, L, Hkv, n_in, d]")
    B, L, hq, R, d = q.shape
    Bk, Lk, hkv, n_in, dk = k.shape
    if (B, L, d) != (Bk, Lk, dk):
        raise ValueError("q and k disagree on batch, layers or head_dim")
    return SpeckvShape(B, L, hq, hkv, d, n_in, n_window, R - n_window, float(scale))


def speckv_workspace_size(shape: SpeckvShape) -> int:
    return int(load_library().speckv_workspace_size(ctypes.byref(shape)))


def speckv_score(q, k, n_window: int, scores, window_mass=None, workspace=None, scale: float = 1.0,
                 stream=None):
    """scores[u][j] (and window_mass[u][j]) for every unit u = (b, layer, KV head)."""
    lib = load_library()
    shape = speckv_shape(q, k, n_window, scale)
    need = speckv_workspace_size(shape)
    ws = _workspace(workspace, need, q.device)
    _check(lib.speckv_score(ctypes.byref(shape), _dev(q, "q", torch.bfloat16), _dev(k, "k", torch.bfloat16),
                            _dev(scores, "scores", torch.float32),
                            _dev(window_mass, "window_mass", torch.float32),
                            _dev(ws, "workspace"), ws.numel() * ws.element_size(), _stream(stream)))
    return scores


def speckv_row_lse(q, k, n_window: int, lse2, scale: float = 1.0, stream=None):
    lib = load_library()
    shape = speckv_shape(q, k, n_window, scale)
    _check(lib.speckv_row_lse(ctypes.byref(shape), _dev(q, "q", torch.bfloat16), _dev(k, "k", torch.bfloat16),
                              _dev(lse2, "lse2", torch.float32), _stream(stream)))
    return lse2


# --------------------------------------------------------------------- SpecPC
def specpc_shape(q, k, l_skip: int, n_lookahead: int, scale: float = 1.0) -> SpecpcShape:
    if q.dim() != 5 or k.dim() != 5:
        raise ValueError("q is [B, L, Hq, W, d] and k is [B, L, Hkv, n_in, d]")
    B, L, hq, W, d = q.shape
    _, _, hkv, n_in, _ = k.shape
    return SpecpcShape(B, L, l_skip, hq, hkv, d, n_in, W, n_lookahead, float(scale))


def specpc_workspace_size(shape: SpecpcShape) -> int:
    return int(load_library().specpc_workspace_size(ctypes.byref(shape)))


def specpc_score(q, k, row_weights, scores, l_skip: int, n_lookahead: int = 1, workspace=None,
                 scale: float = 1.0, stream=None):
    lib = load_library()
    shape = specpc_shape(q, k, l_skip, n_lookahead, scale)
    ws = _workspace(workspace, specpc_workspace_size(shape), q.device)
    _check(lib.specpc_score(ctypes.byref(shape), _dev(q, "q", torch.bfloat16), _dev(k, "k", torch.bfloat16),
                            _dev(row_weights, "row_weights", torch.float32),
                            _dev(scores, "scores", torch.float32), _dev(ws, "workspace"),
                            ws.numel() * ws.element_size(), _stream(stream)))
    return scores


# --------------------------------------------------------------------- selection
def topk_workspace_size(units: int, n_cand: int) -> int:
    return int(load_library().topk_workspace_size(units, n_cand))


def topk_select(scores, k: int, n_tail: int, idx, pool_kernel: int = 7, pooled=None, workspace=None,
                stream=None):
    """scores [units, n_cand] fp32 -> idx [units, min(k, n_cand) + n_tail] int32."""
    lib = load_library()
    units, n_cand = scores.shape
    ws = _workspace(workspace, topk_workspace_size(units, n_cand), scores.device)
    _check(lib.topk_select(_dev(scores, "scores", torch.float32), units, n_cand, pool_kernel, k, n_tail,
                           _dev(idx, "idx", torch.int32), _dev(pooled, "pooled", torch.float32),
                           _dev(ws, "workspace"), ws.numel() * ws.element_size(), _stream(stream)))
    return idx


def kv_compact(k, v, idx, k_out, v_out, units_per_idx: int = 1, stream=None):
    """k, v [units, n_src, d] (any 2-byte or 4-byte dtype); idx [units/units_per_idx, n_idx].
    k and v may be CUDA tensors or pinned host tensors (gathered in place)."""
    lib = load_library()
    n_src, d = k.shape[-2], k.shape[-1]
    units = k.numel() // (n_src * d) if n_src * d else 0
    n_idx = idx.shape[-1]
    _check(lib.kv_compact(_src(k, "k"), _src(v, "v"), units, n_src, d, k.element_size(),
                          _dev(idx, "idx", torch.int32), n_idx, units_per_idx, _dev(k_out, "k_out"),
                          _dev(v_out, "v_out"), _stream(stream)))
    return k_out, v_out


def decode_attention(q, k, v, out=None, scale: float = 1.0, stream=None):
    """Decode attention over a compacted cache: q [B, L, Hq, d], k/v [B, L, Hkv, n_kv, d]
    (bf16, CUDA) -> out fp32 [B, L, Hq, d]."""
    lib = load_library()
    Bsz, L, hq, d = q.shape
    hkv, n_kv = k.shape[2], k.shape[3]
    if out is None:
        out = torch.empty((Bsz, L, hq, d), dtype=torch.float32, device=q.device)
    _check(lib.decode_attention(Bsz, L, hq, hkv, d, n_kv, float(scale), _dev(q, "q", torch.bfloat16),
                                _dev(k, "k", torch.bfloat16), _dev(v, "v", torch.bfloat16),
                                _dev(out, "out", torch.float32), _stream(stream)))
    return out


# --------------------------------------------------------------------- errors
def spk_device_error(clear: bool = True):
    """(status, site) of the first error a kernel recorded (synchronises the device)."""
    lib = load_library()
    st, site = ctypes.c_int(0), ctypes.c_int(0)
    _check(lib.spk_device_error(ctypes.byref(st), ctypes.byref(site), 1 if clear else 0))
    return st.value, site.value


def spk_selftest_wait_timeout(limit_ns: int, stream=None):
    _check(load_library().spk_selftest_wait_timeout(int(limit_ns), _stream(stream)))


def spk_exp2_fma(t, y, stream=None):
    """y = 2^t through the scoring epilogues' FMA-pipe exponential (diagnostic)."""
    _check(load_library().spk_exp2_fma(_dev(t, "t", torch.float32), _dev(y, "y", torch.float32), t.numel(),
                                       _stream(stream)))
    return y
