"""ctypes binding of include/speckv.h: argument marshalling only.

Each function takes torch tensors that already live on the GPU, checks their
sizes, dtype, device and contiguity, and passes raw pointers, sizes and the
CUDA stream to the C entry point of the same name.  The C ABI cannot see how
large a buffer is, so every output's element count is checked here against
the shape the entry point will write (ValueError on a mismatch) before the
call.  Output tensors are the caller's; a workspace is allocated with torch
only when none is given, and then on the stream the kernels run on.
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


class VsShape(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int), ("layers", ctypes.c_int), ("hq", ctypes.c_int),
                ("hkv", ctypes.c_int), ("head_dim", ctypes.c_int), ("n", ctypes.c_int), ("n_q", ctypes.c_int),
                ("n_vertical", ctypes.c_int), ("n_slash", ctypes.c_int), ("scale", ctypes.c_float)]


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
    vsp = ctypes.POINTER(VsShape)
    sig = {
        "speckv_workspace_size": (sz, [sk]),
        "speckv_score": (I, [sk, vp, vp, vp, vp, vp, sz, vp]),
        "speckv_row_lse": (I, [sk, vp, vp, vp, vp]),
        "speckv_row_offsets": (I, [sk, vp, vp, vp, sz, vp]),
        "speckv_colsum": (I, [sk, vp, vp, vp, vp, vp, sz, vp]),
        "speckv_prefill_attention": (I, [sk, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]),
        "specpc_workspace_size": (sz, [sp]),
        "specpc_score": (I, [sp, vp, vp, vp, vp, vp, sz, vp]),
        "specpc_row_offsets": (I, [sp, vp, vp, vp, vp, sz, vp]),
        "specpc_colsum": (I, [sp, vp, vp, vp, vp, sz, vp]),
        "topk_workspace_size": (sz, [I, I]),
        "topk_select": (I, [vp, I, I, I, I, I, vp, vp, vp, sz, vp]),
        "topk_select_pool": (I, [vp, I, I, I, I, I, I, vp, vp, vp, sz, vp]),
        "kv_compact": (I, [vp, vp, I, I, I, I, vp, I, I, vp, vp, vp]),
        "spk_last_error": (ctypes.c_char_p, []),
        "spk_device_error": (I, [ctypes.POINTER(I), ctypes.POINTER(I), I]),
        "spk_selftest_wait_timeout": (I, [ctypes.c_longlong, vp]),
        "spk_exp2_fma": (I, [vp, vp, I, vp]),
        "spk_mapped_host_pointer": (I, [vp, ctypes.POINTER(vp)]),
        "decode_attention": (I, [I, I, I, I, I, I, F, vp, vp, vp, vp, vp]),
        "vs_workspace_size": (sz, [vsp]),
        "vs_sparse_attention": (I, [vsp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]),
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


SPK_POOL_MAX, SPK_POOL_AVG = 0, 1


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _stream_object(stream, device):
    """The torch stream the kernels will run on (a raw handle is wrapped)."""
    if stream is None:
        return torch.cuda.current_stream(device)
    if isinstance(stream, torch.cuda.Stream):
        return stream
    return torch.cuda.ExternalStream(int(stream), device=device)


def _numel(t: Optional[torch.Tensor], name: str, expected: int, required: bool = True):
    """An output (or input) must hold exactly the elements the kernel touches."""
    if t is None:
        if required:
            raise ValueError(f"{name} is required")
        return
    if t.numel() != expected:
        raise ValueError(f"{name} has {t.numel()} elements, the call needs {expected}")


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


def _workspace(ws: Optional[torch.Tensor], nbytes: int, device, stream=None) -> torch.Tensor:
    """The caller's workspace, or a temporary one.  A temporary is allocated
    on the stream the kernels are enqueued on: the caching allocator then
    hands its memory to later allocations of that stream only, which run
    after the kernels, although the tensor is released when the call returns."""
    if ws is not None:
        return ws
    with torch.cuda.stream(_stream_object(stream, device)):
        return torch.empty(max(nbytes, 256), dtype=torch.uint8, device=device)


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
    units = shape.batch * shape.layers * shape.hkv
    _numel(scores, "scores", units * (shape.n_in - n_window), required=shape.n_in > n_window)
    _numel(window_mass, "window_mass", units * n_window, required=False)
    need = speckv_workspace_size(shape)
    ws = _workspace(workspace, need, q.device, stream)
    _check(lib.speckv_score(ctypes.byref(shape), _dev(q, "q", torch.bfloat16), _dev(k, "k", torch.bfloat16),
                            _dev(scores, "scores", torch.float32),
                            _dev(window_mass, "window_mass", torch.float32),
                            _dev(ws, "workspace"), ws.numel() * ws.element_size(), _stream(stream)))
    return scores


def speckv_row_offsets(q, k, n_window: int, workspace, scale: float = 1.0, stream=None):
    """Pass 1 of speckv_score: the row offsets, written into `workspace`."""
    lib = load_library()
    shape = speckv_shape(q, k, n_window, scale)
    if workspace is None:
        raise ValueError("workspace is required (speckv_workspace_size bytes)")
    _check(lib.speckv_row_offsets(ctypes.byref(shape), _dev(q, "q", torch.bfloat16), _dev(k, "k", torch.bfloat16),
                                  _dev(workspace, "workspace"), workspace.numel() * workspace.element_size(),
                                  _stream(stream)))
    return workspace


def speckv_colsum(q, k, n_window: int, scores, workspace, window_mass=None, scale: float = 1.0, stream=None):
    """Pass 2 of speckv_score, from a workspace speckv_row_offsets filled."""
    lib = load_library()
    shape = speckv_shape(q, k, n_window, scale)
    units = shape.batch * shape.layers * shape.hkv
    _numel(scores, "scores", units * (shape.n_in - n_window), required=shape.n_in > n_window)
    _numel(window_mass, "window_mass", units * n_window, required=False)
    if workspace is None:
        raise ValueError("workspace is required (the one speckv_row_offsets filled)")
    _check(lib.speckv_colsum(ctypes.byref(shape), _dev(q, "q", torch.bfloat16), _dev(k, "k", torch.bfloat16),
                             _dev(scores, "scores", torch.float32), _dev(window_mass, "window_mass", torch.float32),
                             _dev(workspace, "workspace"), workspace.numel() * workspace.element_size(),
                             _stream(stream)))
    return scores


def speckv_prefill_attention(q, k, v, k_look, v_look, n_window: int, out=None, lse2=None, workspace=None,
                             scale: float = 1.0, stream=None):
    """Prefill attention of the window and lookahead rows: q [B, L, Hq, R, d];
    k, v [B, L, Hkv, n_in, d] (input tokens); k_look, v_look [B, L, Hkv,
    n_lookahead, d] or None.  Returns out bf16 [B, L, Hq, R, d]; fills lse2
    (fp32 [units, g*R]) and the column pass's workspace when given."""
    lib = load_library()
    shape = speckv_shape(q, k, n_window, scale)
    units = shape.batch * shape.layers * shape.hkv
    rows = shape.hq // shape.hkv * (shape.n_window + shape.n_lookahead)
    if tuple(v.shape) != tuple(k.shape):
        raise ValueError("v must have k's shape")
    look = (shape.batch, shape.layers, shape.hkv, shape.n_lookahead, shape.head_dim)
    if shape.n_lookahead > 0:
        if k_look is None or v_look is None or tuple(k_look.shape) != look or tuple(v_look.shape) != look:
            raise ValueError(f"k_look and v_look must be {list(look)}")
    else:
        k_look = v_look = None
    if out is None:
        out = torch.empty(q.shape, dtype=torch.bfloat16, device=q.device)
    _numel(out, "out", q.numel())
    _numel(lse2, "lse2", units * rows, required=False)
    ws_bytes = 0
    if workspace is not None:
        ws_bytes = workspace.numel() * workspace.element_size()
    _check(lib.speckv_prefill_attention(ctypes.byref(shape), _dev(q, "q", torch.bfloat16),
                                        _dev(k, "k", torch.bfloat16), _dev(v, "v", torch.bfloat16),
                                        _dev(k_look, "k_look", torch.bfloat16), _dev(v_look, "v_look", torch.bfloat16),
                                        _dev(out, "out", torch.bfloat16), _dev(lse2, "lse2", torch.float32),
                                        _dev(workspace, "workspace"), ws_bytes, _stream(stream)))
    return out


def speckv_row_lse(q, k, n_window: int, lse2, scale: float = 1.0, stream=None):
    lib = load_library()
    shape = speckv_shape(q, k, n_window, scale)
    _numel(lse2, "lse2", shape.batch * shape.layers * shape.hq * (shape.n_window + shape.n_lookahead))
    _check(lib.speckv_row_lse(ctypes.byref(shape), _dev(q, "q", torch.bfloat16), _dev(k, "k", torch.bfloat16),
                              _dev(lse2, "lse2", torch.float32), _stream(stream)))
    return lse2


# --------------------------------------------------------------------- SpecPC
def specpc_shape(q, k, l_skip: int, n_lookahead: int, scale: float = 1.0) -> SpecpcShape:
    if q.dim() != 5 or k.dim() != 5:
        raise ValueError("q is [B, L, Hq, W, d] and k is [B, L, Hkv, n_in, d]")
    B, L, hq, W, d = q.shape
    Bk, Lk, hkv, n_in, dk = k.shape
    if (B, L, d) != (Bk, Lk, dk):
        raise ValueError("q and k disagree on batch, layers or head_dim")
    return SpecpcShape(B, L, l_skip, hq, hkv, d, n_in, W, n_lookahead, float(scale))


def specpc_workspace_size(shape: SpecpcShape) -> int:
    return int(load_library().specpc_workspace_size(ctypes.byref(shape)))


def specpc_score(q, k, row_weights, scores, l_skip: int, n_lookahead: int = 1, workspace=None,
                 scale: float = 1.0, stream=None):
    lib = load_library()
    shape = specpc_shape(q, k, l_skip, n_lookahead, scale)
    _numel(row_weights, "row_weights", shape.n_rows)
    _numel(scores, "scores", shape.batch * shape.n_in)
    ws = _workspace(workspace, specpc_workspace_size(shape), q.device, stream)
    _check(lib.specpc_score(ctypes.byref(shape), _dev(q, "q", torch.bfloat16), _dev(k, "k", torch.bfloat16),
                            _dev(row_weights, "row_weights", torch.float32),
                            _dev(scores, "scores", torch.float32), _dev(ws, "workspace"),
                            ws.numel() * ws.element_size(), _stream(stream)))
    return scores


def specpc_row_offsets(q, k, row_weights, workspace, l_skip: int, n_lookahead: int = 1, scale: float = 1.0,
                       stream=None):
    """Pass 1 of specpc_score into `workspace`."""
    lib = load_library()
    shape = specpc_shape(q, k, l_skip, n_lookahead, scale)
    _numel(row_weights, "row_weights", shape.n_rows)
    if workspace is None:
        raise ValueError("workspace is required (specpc_workspace_size bytes)")
    _check(lib.specpc_row_offsets(ctypes.byref(shape), _dev(q, "q", torch.bfloat16), _dev(k, "k", torch.bfloat16),
                                  _dev(row_weights, "row_weights", torch.float32), _dev(workspace, "workspace"),
                                  workspace.numel() * workspace.element_size(), _stream(stream)))
    return workspace


def specpc_colsum(q, k, scores, workspace, l_skip: int, n_lookahead: int = 1, scale: float = 1.0, stream=None):
    """Pass 2 of specpc_score from a workspace specpc_row_offsets filled."""
    lib = load_library()
    shape = specpc_shape(q, k, l_skip, n_lookahead, scale)
    _numel(scores, "scores", shape.batch * shape.n_in)
    if workspace is None:
        raise ValueError("workspace is required (the one specpc_row_offsets filled)")
    _check(lib.specpc_colsum(ctypes.byref(shape), _dev(q, "q", torch.bfloat16), _dev(k, "k", torch.bfloat16),
                             _dev(scores, "scores", torch.float32), _dev(workspace, "workspace"),
                             workspace.numel() * workspace.element_size(), _stream(stream)))
    return scores


# --------------------------------------------------------------------- selection
def topk_workspace_size(units: int, n_cand: int) -> int:
    return int(load_library().topk_workspace_size(units, n_cand))


def topk_select(scores, k: int, n_tail: int, idx, pool_kernel: int = 7, pooled=None, workspace=None,
                stream=None, pool_mode: int = SPK_POOL_MAX):
    """scores [units, n_cand] fp32 -> idx [units, min(k, n_cand) + n_tail] int32.
    pool_mode SPK_POOL_MAX (topk_select) or SPK_POOL_AVG (topk_select_pool)."""
    lib = load_library()
    if scores.dim() != 2:
        raise ValueError("scores is [units, n_cand]")
    units, n_cand = scores.shape
    if k < 0 or n_tail < 0:
        raise ValueError("k and n_tail must be >= 0")
    _numel(idx, "idx", units * (min(k, n_cand) + n_tail), required=units * (min(k, n_cand) + n_tail) > 0)
    _numel(pooled, "pooled", units * n_cand, required=False)
    ws = _workspace(workspace, topk_workspace_size(units, n_cand), scores.device, stream)
    args = (_dev(scores, "scores", torch.float32), units, n_cand)
    tail = (pool_kernel, k, n_tail, _dev(idx, "idx", torch.int32), _dev(pooled, "pooled", torch.float32),
            _dev(ws, "workspace"), ws.numel() * ws.element_size(), _stream(stream))
    if pool_mode == SPK_POOL_MAX:
        _check(lib.topk_select(*args, *tail))
    else:
        _check(lib.topk_select_pool(*args, int(pool_mode), *tail))
    return idx


def kv_compact(k, v, idx, k_out, v_out, units_per_idx: int = 1, stream=None):
    """k, v [units, n_src, d] (any 2-byte or 4-byte dtype); idx [units/units_per_idx, n_idx].
    k and v may be CUDA tensors or pinned host tensors (gathered in place)."""
    lib = load_library()
    if k.dim() < 2:
        raise ValueError("k is [..., n_src, head_dim]")
    n_src, d = k.shape[-2], k.shape[-1]
    units = k.numel() // (n_src * d) if n_src * d else 0
    if units_per_idx < 1 or units % units_per_idx:
        raise ValueError(f"units ({units}) must be a multiple of units_per_idx ({units_per_idx})")
    n_idx = idx.shape[-1]
    _numel(idx, "idx", units // units_per_idx * n_idx)
    _numel(k_out, "k_out", units * n_idx * d)
    if k_out.element_size() != k.element_size():
        raise ValueError("k_out must have k's element size")
    if (v is None) != (v_out is None):
        raise ValueError("v and v_out are given together or not at all")
    if v is not None:
        if tuple(v.shape) != tuple(k.shape) or v.element_size() != k.element_size():
            raise ValueError("v must have k's shape and element size")
        _numel(v_out, "v_out", units * n_idx * d)
        if v_out.element_size() != k.element_size():
            raise ValueError("v_out must have k's element size")
    _check(lib.kv_compact(_src(k, "k"), _src(v, "v"), units, n_src, d, k.element_size(),
                          _dev(idx, "idx", torch.int32), n_idx, units_per_idx, _dev(k_out, "k_out"),
                          _dev(v_out, "v_out"), _stream(stream)))
    return k_out, v_out


def decode_attention(q, k, v, out=None, scale: float = 1.0, stream=None):
    """Decode attention over a compacted cache: q [B, L, Hq, d], k/v [B, L, Hkv, n_kv, d]
    (bf16, CUDA) -> out fp32 [B, L, Hq, d]."""
    lib = load_library()
    if q.dim() != 4 or k.dim() != 5 or v.dim() != 5:
        raise ValueError("q is [B, L, Hq, d]; k and v are [B, L, Hkv, n_kv, d]")
    Bsz, L, hq, d = q.shape
    hkv, n_kv = k.shape[2], k.shape[3]
    if tuple(k.shape) != (Bsz, L, hkv, n_kv, d) or tuple(v.shape) != tuple(k.shape):
        raise ValueError("k and v must be [B, L, Hkv, n_kv, d] with q's B, L and d")
    if out is None:
        out = torch.empty((Bsz, L, hq, d), dtype=torch.float32, device=q.device)
    _numel(out, "out", Bsz * L * hq * d)
    _check(lib.decode_attention(Bsz, L, hq, hkv, d, n_kv, float(scale), _dev(q, "q", torch.bfloat16),
                                _dev(k, "k", torch.bfloat16), _dev(v, "v", torch.bfloat16),
                                _dev(out, "out", torch.float32), _stream(stream)))
    return out


# --------------------------------------------------------------------- Vertical-Slash sparse prefill
def vs_shape(q, k, n_vertical: int, n_slash: int, scale: float = 1.0) -> VsShape:
    if q.dim() != 5 or k.dim() != 5:
        raise ValueError("q is [B, L, Hq, n_q, d] and k is [B, L, Hkv, n, d]")
    B, L, hq, n_q, d = q.shape
    Bk, Lk, hkv, n, dk = k.shape
    if (B, L, d) != (Bk, Lk, dk):
        raise ValueError("q and k disagree on batch, layers or head_dim")
    return VsShape(B, L, hq, hkv, d, n, n_q, n_vertical, n_slash, float(scale))


def vs_workspace_size(shape: VsShape) -> int:
    return int(load_library().vs_workspace_size(ctypes.byref(shape)))


def vs_sparse_attention(q, k, v, vertical, slash, out=None, lse2=None, workspace=None, scale: float = 1.0,
                        stream=None):
    """Vertical-Slash sparse attention: q [B, L, Hq, n_q, d] (the last n_q
    positions), k, v [B, L, Hkv, n, d]; vertical int32 [units, n_v] and slash
    int32 [units, n_s] (ascending) per unit = (b, layer, KV head).  Returns
    out bf16 [B, L, Hq, n_q, d]; fills lse2 (fp32 [B*L*Hq, n_q]) when given."""
    lib = load_library()
    if vertical is None or slash is None or vertical.dim() < 1 or slash.dim() < 1:
        raise ValueError("vertical and slash are int32 [units, count] tensors")
    n_v, n_s = vertical.shape[-1], slash.shape[-1]
    shape = vs_shape(q, k, n_v, n_s, scale)
    units = shape.batch * shape.layers * shape.hkv
    if tuple(v.shape) != tuple(k.shape):
        raise ValueError("v must have k's shape")
    _numel(vertical, "vertical", units * n_v)
    _numel(slash, "slash", units * n_s)
    if out is None:
        out = torch.empty(q.shape, dtype=torch.bfloat16, device=q.device)
    _numel(out, "out", q.numel())
    _numel(lse2, "lse2", shape.batch * shape.layers * shape.hq * shape.n_q, required=False)
    ws = None
    if n_v > 0:
        ws = _workspace(workspace, vs_workspace_size(shape), q.device, stream)
    _check(lib.vs_sparse_attention(ctypes.byref(shape), _dev(q, "q", torch.bfloat16), _dev(k, "k", torch.bfloat16),
                                   _dev(v, "v", torch.bfloat16), _dev(vertical, "vertical", torch.int32),
                                   _dev(slash, "slash", torch.int32), _dev(out, "out", torch.bfloat16),
                                   _dev(lse2, "lse2", torch.float32), _dev(ws, "workspace"),
                                   ws.numel() * ws.element_size() if ws is not None else 0, _stream(stream)))
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
