"""The C-ABI library loads and exports every symbol include/speckv.h declares,
and argument errors are reported before anything touches a GPU (no GPU needed)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "speckv.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b([a-z_][a-z0-9_]*)\s*\(", text)) - {"if", "sizeof"})


@pytest.fixture(scope="module")
def lib():
    from prompt_compression_b200 import build
    build.build_library()
    from prompt_compression_b200 import binding
    return binding.load_library()


def test_header_declares_the_boundary():
    names = declared_functions()
    for f in ("speckv_score", "specpc_score", "topk_select", "topk_select_pool", "kv_compact", "spk_last_error",
              "speckv_workspace_size", "specpc_workspace_size", "topk_workspace_size"):
        assert f in names


def test_every_declared_symbol_is_exported(lib):
    for name in declared_functions():
        assert hasattr(lib, name), f"{name} declared in speckv.h but not exported"


def test_workspace_sizes(lib):
    from prompt_compression_b200 import binding as B
    s = B.SpeckvShape(1, 64, 40, 8, 128, 65536, 64, 128, 1.0)
    assert B.speckv_workspace_size(s) == 512 * 1024 * 32    # 32 B per row, rows padded to 128
    s = B.SpecpcShape(1, 24, 4, 14, 2, 64, 32768, 256, 1, 1.0)
    # row offsets (40 units x 1792 rows x 32 B) + on 148 SMs the 128 key blocks
    # are split into 8 segment groups: 128 x 8 x 14 heads x 1 KB of partial sums
    assert B.specpc_workspace_size(s) == 40 * 1792 * 32 + 128 * 8 * 14 * 1024
    s = B.SpecpcShape(2, 24, 4, 14, 2, 64, 131072, 256, 1, 1.0)
    assert B.specpc_workspace_size(s) == 80 * 1792 * 32      # 1024 blocks fill 148 SMs: no split
    assert B.topk_workspace_size(512, 65472) == 512 * 65472 * 4


@pytest.mark.parametrize("fields,status,needle", [
    ((1, 1, 4, 2, 96, 64, 8, 8, 1.0), 2, "head_dim"),
    ((1, 1, 4, 3, 64, 64, 8, 8, 1.0), 1, "multiple"),
    ((1, 1, 4, 2, 64, 64, 80, 8, 1.0), 1, "n_window"),
    ((1, 1, 4, 2, 64, 64, 8, 8, -1.0), 1, "scale"),
    ((1, 1, 64, 2, 64, 64, 64, 8, 1.0), 2, "exceeds"),
    ((1, 1, 4, 2, 64, 64, 0, 0, 1.0), 1, ">= 1"),
])
def test_speckv_argument_errors(lib, fields, status, needle):
    from prompt_compression_b200 import binding as B
    s = B.SpeckvShape(*fields)
    rc = lib.speckv_score(ctypes.byref(s), 16, 16, 16, None, 16, 1 << 20, None)
    assert rc == status
    assert needle in lib.spk_last_error().decode()
    assert lib.speckv_workspace_size(ctypes.byref(s)) == 0


def test_speckv_workspace_and_pointer_errors(lib):
    from prompt_compression_b200 import binding as B
    s = B.SpeckvShape(1, 1, 4, 2, 64, 64, 8, 8, 1.0)
    assert lib.speckv_score(ctypes.byref(s), 16, 16, 16, None, 16, 8, None) == B.SPK_ERR_WORKSPACE
    assert lib.speckv_score(ctypes.byref(s), 16, 16, None, None, 16, 1 << 20, None) == B.SPK_ERR_ARG
    assert lib.speckv_score(ctypes.byref(s), 18, 16, 16, None, 16, 1 << 20, None) == B.SPK_ERR_ARG


def test_specpc_argument_errors(lib):
    from prompt_compression_b200 import binding as B
    bad = [((1, 4, 4, 4, 2, 64, 100, 16, 1, 1.0), 1),      # l_skip == layers
           ((1, 4, 1, 4, 2, 96, 100, 16, 1, 1.0), 2),      # head_dim 96 unsupported
           ((1, 4, 1, 4, 2, 64, 100, 101, 1, 1.0), 1),     # window longer than the input
           ((1, 4, 1, 34, 2, 64, 100, 16, 1, 1.0), 2),     # group of 17 query heads
           ((1, 4, 1, 4, 2, 64, 100, 16, 0, 1.0), 1)]      # no lookahead token
    for fields, status in bad:
        s = B.SpecpcShape(*fields)
        assert lib.specpc_score(ctypes.byref(s), 16, 16, 16, 16, 16, 1 << 30, None) == status, fields


def test_topk_and_compact_argument_errors(lib):
    from prompt_compression_b200 import binding as B
    assert lib.topk_select(16, 4, 100, 4, 10, 0, 16, None, 16, 1 << 20, None) == B.SPK_ERR_ARG  # even pool
    assert lib.topk_select(16, 4, 100, 7, 10, 0, 16, None, 16, 8, None) == B.SPK_ERR_WORKSPACE
    assert lib.topk_select(16, 4, 100, 7, -1, 0, 16, None, 16, 1 << 20, None) == B.SPK_ERR_ARG
    assert lib.topk_select_pool(16, 4, 100, 2, 7, 10, 0, 16, None, 16, 1 << 20, None) == B.SPK_ERR_ARG   # mode
    assert "pool_mode" in lib.spk_last_error().decode()
    assert lib.topk_select_pool(16, 4, 100, 1, 6, 10, 0, 16, None, 16, 1 << 20, None) == B.SPK_ERR_ARG   # even
    assert lib.kv_compact(16, 16, 4, 10, 60, 2, 16, 3, 1, 16, 16, None) == B.SPK_ERR_UNSUPPORTED
    assert lib.kv_compact(16, 16, 5, 10, 64, 2, 16, 3, 2, 16, 16, None) == B.SPK_ERR_ARG
    assert lib.kv_compact(16, None, 4, 10, 64, 2, 16, 3, 1, 16, 16, None) == B.SPK_ERR_ARG
    assert lib.kv_compact(24, 16, 4, 10, 64, 2, 16, 3, 1, 16, 16, None) == B.SPK_ERR_ARG


def test_mapped_host_pointer_rejects_unmapped_memory(lib):
    # ordinary (pageable) host memory is not mapped into any device: the call
    # reports an error and leaves the output alone (here, or on a GPU machine)
    import numpy as np
    buf = np.zeros(64, dtype=np.uint8)
    out = ctypes.c_void_p(12345)
    rc = lib.spk_mapped_host_pointer(ctypes.c_void_p(buf.ctypes.data), ctypes.byref(out))
    assert rc != 0
    assert out.value == 12345
    assert lib.spk_mapped_host_pointer(None, ctypes.byref(out)) == 1   # SPK_ERR_ARG


@pytest.mark.parametrize("args,status,needle", [
    ((1, 1, 4, 3, 128, 10, 1.0), 1, "multiple"),
    ((1, 1, 36, 2, 128, 10, 1.0), 2, "exceeds 8"),
    ((1, 1, 4, 2, 96, 10, 1.0), 2, "head_dim"),
    ((1, 1, 4, 2, 128, 0, 1.0), 1, ">= 1"),
    ((1, 1, 4, 2, 128, 10, -1.0), 1, "scale"),
    ((1, 1, 4, 2, 128, 10, 1.0), 1, "non-NULL"),
])
def test_decode_argument_errors(lib, args, status, needle):
    B, L, hq, hkv, d, n_kv, scale = args
    rc = lib.decode_attention(B, L, hq, hkv, d, n_kv, ctypes.c_float(scale), None, None, None, None, None)
    assert rc == status
    assert needle in lib.spk_last_error().decode()


def _prototypes():
    """name -> number of parameters, from the header's declarations."""
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    protos = {}
    for m in re.finditer(r"\b([a-z_][a-z0-9_]*)\s*\(([^;{}]*?)\)\s*;", text, flags=re.S):
        name, params = m.group(1), m.group(2).strip()
        protos[name] = 0 if params in ("", "void") else params.count(",") + 1
    return protos


def test_binding_signatures_match_the_header(lib):
    # every function the Python binding declares takes as many arguments as
    # its prototype in include/speckv.h (the boundary cannot drift silently)
    protos = _prototypes()
    checked = 0
    for name, n in protos.items():
        fn = getattr(lib, name)
        if fn.argtypes is None:
            continue
        assert len(fn.argtypes) == n, f"{name}: header has {n} parameters, binding {len(fn.argtypes)}"
        checked += 1
    assert checked >= 10
