"""fp64 CPU oracle for lookahead importance scoring -- TEST INFRASTRUCTURE.

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path (the CUDA library
and its Python binding in ``prompt_compression_b200``) never does, and this
package imports nothing from it.

The arithmetic lives in ``oracle.c`` (plain single-threaded C, double
precision); this module only builds it with gcc and marshals numpy arrays.
Definitions follow "Draft-based Approximate Inference for LLMs" (paper
notes), section "关键设计" (SpecKV, SpecPC, SpecKV-PC) and section
"损失函数 / 训练策略" (local pooling).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None

_dp = ctypes.POINTER(ctypes.c_double)
_u16p = ctypes.POINTER(ctypes.c_uint16)
_i32p = ctypes.POINTER(ctypes.c_int32)
_u8p = ctypes.POINTER(ctypes.c_uint8)


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so (gcc, -O2, strict IEEE)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-fno-fast-math",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        I, D = ctypes.c_int, ctypes.c_double
        lib.oracle_speckv_unit.argtypes = [_u16p, _u16p, I, I, I, I, I, D, _dp, _dp, _dp]
        lib.oracle_speckv_unit_f64.argtypes = [_dp, _dp, I, I, I, I, I, D, _dp, _dp, _dp]
        lib.oracle_specpc_batch.argtypes = [_u16p, _u16p, _dp, I, I, I, I, I, I, I, I, D, _dp]
        lib.oracle_specpc_batch_f64.argtypes = [_dp, _dp, _dp, I, I, I, I, I, I, I, I, D, _dp]
        lib.oracle_maxpool.argtypes = [_dp, I, I, _dp]
        lib.oracle_avgpool.argtypes = [_dp, I, I, _dp]
        lib.oracle_topk_with_tail.argtypes = [_dp, I, I, I, _i32p]
        lib.oracle_gather_rows.argtypes = [_u8p, I, I, _i32p, I, _u8p]
        lib.oracle_decode_row.argtypes = [_u16p, _u16p, _u16p, I, I, D, _dp]
        lib.oracle_prefill_row.argtypes = [_u16p, _u16p, _u16p, I, I, I, D, _dp, _dp]
        lib.oracle_vs_row.argtypes = [_u16p, _u16p, _u16p, _u8p, _u8p, I, I, I, D, _dp, _dp]
        for f in (lib.oracle_speckv_unit, lib.oracle_speckv_unit_f64, lib.oracle_specpc_batch,
                  lib.oracle_specpc_batch_f64, lib.oracle_maxpool, lib.oracle_avgpool, lib.oracle_topk_with_tail,
                  lib.oracle_gather_rows, lib.oracle_decode_row, lib.oracle_prefill_row, lib.oracle_vs_row):
            f.restype = ctypes.c_int
        _lib = lib
    return _lib


def _ptr(a, t):
    return a.ctypes.data_as(t)


def _check(rc):
    if rc < 0:
        raise ValueError("oracle rejected its arguments")
    return rc


def speckv_unit(q, k, n_window: int, n_lookahead: int, scale: float = 1.0, with_lse=False):
    """SpecKV scores of one unit.

    q: [g, R, d] and k: [n_in, d], either uint16 bf16 bit patterns or floats
    (floats run the same definition in fp64 without rounding).
    Returns (scores [n_pre], window_mass [n_window]) or, with with_lse,
    (scores, window_mass, lse [g*R], natural log).
    """
    lib = _load()
    q = np.ascontiguousarray(q)
    k = np.ascontiguousarray(k)
    g, R, d = q.shape
    n_in = k.shape[0]
    assert R == n_window + n_lookahead and k.shape[1] == d
    scores = np.zeros(n_in - n_window, np.float64)
    wm = np.zeros(max(n_window, 1), np.float64)
    lse = np.zeros(max(g * R, 1), np.float64)
    if q.dtype == np.uint16:
        rc = lib.oracle_speckv_unit(_ptr(q, _u16p), _ptr(k, _u16p), g, n_window, n_lookahead,
                                    n_in, d, scale, _ptr(scores, _dp), _ptr(wm, _dp),
                                    _ptr(lse, _dp))
    else:
        qd = np.ascontiguousarray(q, np.float64)
        kd = np.ascontiguousarray(k, np.float64)
        rc = lib.oracle_speckv_unit_f64(_ptr(qd, _dp), _ptr(kd, _dp), g, n_window, n_lookahead,
                                        n_in, d, scale, _ptr(scores, _dp), _ptr(wm, _dp),
                                        _ptr(lse, _dp))
    _check(rc)
    wm = wm[:n_window]
    return (scores, wm, lse[:g * R]) if with_lse else (scores, wm)


def specpc_batch(q, k, weights, l_skip: int, n_lookahead: int, scale: float = 1.0):
    """SpecPC scores of one batch element: q [L,Hq,W,d], k [L,Hkv,n_in,d]."""
    lib = _load()
    q = np.ascontiguousarray(q)
    k = np.ascontiguousarray(k)
    L, hq, W, d = q.shape
    _, hkv, n_in, _ = k.shape
    w = np.ascontiguousarray(weights, np.float64)
    assert w.shape == (W,)
    out = np.zeros(n_in, np.float64)
    if q.dtype == np.uint16:
        rc = lib.oracle_specpc_batch(_ptr(q, _u16p), _ptr(k, _u16p), _ptr(w, _dp), L, l_skip, hq,
                                     hkv, W, n_lookahead, n_in, d, scale, _ptr(out, _dp))
    else:
        qd = np.ascontiguousarray(q, np.float64)
        kd = np.ascontiguousarray(k, np.float64)
        rc = lib.oracle_specpc_batch_f64(_ptr(qd, _dp), _ptr(kd, _dp), _ptr(w, _dp), L, l_skip,
                                         hq, hkv, W, n_lookahead, n_in, d, scale, _ptr(out, _dp))
    _check(rc)
    return out


def maxpool(s, kernel: int = 7):
    lib = _load()
    s = np.ascontiguousarray(s, np.float64)
    out = np.zeros_like(s)
    _check(lib.oracle_maxpool(_ptr(s, _dp), s.size, kernel, _ptr(out, _dp)))
    return out


def avgpool(s, kernel: int = 7):
    """Mean over the window [j - r, j + r] clipped to the row, r = kernel // 2."""
    lib = _load()
    s = np.ascontiguousarray(s, np.float64)
    out = np.zeros_like(s)
    _check(lib.oracle_avgpool(_ptr(s, _dp), s.size, kernel, _ptr(out, _dp)))
    return out


def pool(s, kernel: int = 7, mode: str = "max"):
    """Local pooling of one row of scores: mode "max" or "avg"."""
    return maxpool(s, kernel) if mode == "max" else avgpool(s, kernel)


def topk_with_tail(pooled, k: int, n_tail: int):
    lib = _load()
    p = np.ascontiguousarray(pooled, np.float64)
    n = p.size
    out = np.zeros(max(min(k, n) + n_tail, 1), np.int32)
    m = _check(lib.oracle_topk_with_tail(_ptr(p, _dp), n, k, n_tail, _ptr(out, _i32p)))
    return out[:m]


def gather_rows(src, idx):
    """dst[t] = src[idx[t]] row by row, bytes copied as they are."""
    lib = _load()
    src = np.ascontiguousarray(src)
    idx = np.ascontiguousarray(idx, np.int32)
    n_src = src.shape[0]
    row_bytes = src[0].nbytes if n_src else 0
    dst = np.zeros((idx.size,) + src.shape[1:], src.dtype)
    _check(lib.oracle_gather_rows(_ptr(src.view(np.uint8), _u8p), n_src, row_bytes,
                                  _ptr(idx, _i32p), idx.size, _ptr(dst.view(np.uint8), _u8p)))
    return dst


def decode_attention(q, k, v, scale: float = 1.0):
    """Decode attention over a compacted cache, every (batch, layer, query head):
    q [B][L][Hq][d], k/v [B][L][Hkv][n_kv][d] (bf16 bit patterns) -> out
    [B][L][Hq][d] in float64; query head qh reads KV head qh // (Hq // Hkv)."""
    lib = _load()
    q = np.ascontiguousarray(q, np.uint16)
    k = np.ascontiguousarray(k, np.uint16)
    v = np.ascontiguousarray(v, np.uint16)
    B, L, hq, d = q.shape
    hkv, n_kv = k.shape[2], k.shape[3]
    g = hq // hkv
    out = np.zeros((B, L, hq, d), np.float64)
    for b in range(B):
        for l in range(L):
            for qh in range(hq):
                row = np.zeros(d, np.float64)
                _check(lib.oracle_decode_row(_ptr(q[b, l, qh], _u16p), _ptr(k[b, l, qh // g], _u16p),
                                             _ptr(v[b, l, qh // g], _u16p), n_kv, d, scale, _ptr(row, _dp)))
                out[b, l, qh] = row
    return out


def prefill_unit(q, k, v, n_window: int, n_lookahead: int, n_in: int, scale: float = 1.0, rows=None):
    """Prefill attention of one unit's window and lookahead rows.

    q [g, R, d] (R = n_window + n_lookahead), k/v [n_in + n_lookahead, d]
    (input tokens, then the lookahead tokens) as bf16 bit patterns.  Window
    row i sits at position n_in - n_window + i, lookahead row i at
    n_in + (i - n_window); each attends to the keys up to its position.
    Returns (out [g, R, d] float64, lse_in [g * R], natural log over the
    input keys only).  With rows = [(h, i), ...] only those rows are
    evaluated and the result is (out [len(rows), d], lse_in [len(rows)])."""
    lib = _load()
    q = np.ascontiguousarray(q, np.uint16)
    k = np.ascontiguousarray(k, np.uint16)
    v = np.ascontiguousarray(v, np.uint16)
    g, R, d = q.shape
    assert R == n_window + n_lookahead and k.shape == v.shape and k.shape[0] >= n_in + n_lookahead
    pairs = [(h, i) for h in range(g) for i in range(R)] if rows is None else [(int(h), int(i)) for h, i in rows]
    out = np.zeros((len(pairs), d), np.float64)
    lse = np.zeros(len(pairs), np.float64)
    for j, (h, i) in enumerate(pairs):
        assert 0 <= h < g and 0 <= i < R
        pos = n_in - n_window + i if i < n_window else n_in + (i - n_window)
        l = ctypes.c_double(0.0)
        _check(lib.oracle_prefill_row(_ptr(q[h, i], _u16p), _ptr(k, _u16p), _ptr(v, _u16p), pos + 1, n_in, d,
                                      scale, _ptr(out[j], _dp), ctypes.byref(l)))
        lse[j] = l.value
    if rows is None:
        return out.reshape(g, R, d), lse
    return out, lse


def vs_attention_unit(q, k, v, vertical, slash, scale: float = 1.0, rows=None):
    """Vertical-Slash sparse attention of one unit's query heads.

    q [g, n_q, d]: the last n_q positions of the sequence (row i at
    n - n_q + i); k, v [n, d]; vertical: key indices every row sees; slash:
    offsets o = p - j every row sees (bf16 bit patterns for q, k, v).
    Returns (out [g, n_q, d] float64, lse [g * n_q], natural log).  With
    rows = [(h, i), ...] only those rows are evaluated and the result is
    (out [len(rows), d], lse [len(rows)])."""
    lib = _load()
    q = np.ascontiguousarray(q, np.uint16)
    k = np.ascontiguousarray(k, np.uint16)
    v = np.ascontiguousarray(v, np.uint16)
    g, n_q, d = q.shape
    n = k.shape[0]
    vm = np.zeros(n, np.uint8)
    sm = np.zeros(n, np.uint8)
    vm[np.asarray(vertical, np.int64)] = 1
    sm[np.asarray(slash, np.int64)] = 1
    pairs = [(h, i) for h in range(g) for i in range(n_q)] if rows is None else [(int(h), int(i)) for h, i in rows]
    out = np.zeros((len(pairs), d), np.float64)
    lse = np.zeros(len(pairs), np.float64)
    for j, (h, i) in enumerate(pairs):
        assert 0 <= h < g and 0 <= i < n_q
        l = ctypes.c_double(0.0)
        _check(lib.oracle_vs_row(_ptr(q[h, i], _u16p), _ptr(k, _u16p), _ptr(v, _u16p), _ptr(vm, _u8p),
                                 _ptr(sm, _u8p), n, n - n_q + i, d, scale, _ptr(out[j], _dp), ctypes.byref(l)))
        lse[j] = l.value
    if rows is None:
        return out.reshape(g, n_q, d), lse
    return out, lse


def speckv_select_unit(q, k, n_window, n_lookahead, c_max, pool=7, scale=1.0):
    """Scores -> pooled -> top-C_max + window indices for one unit."""
    s, wm = speckv_unit(q, k, n_window, n_lookahead, scale)
    p = maxpool(s, pool)
    return s, p, topk_with_tail(p, c_max, n_window)
