"""Host-side checks of the Python binding (no GPU needed).

The C ABI receives raw pointers and cannot tell how large a buffer is, so the
binding rejects every output (and index) tensor whose element count differs
from what the entry point will touch -- before anything reaches the library.
A workspace the binding allocates itself is allocated on the stream the
kernels run on, so that the caching allocator cannot give its memory to
other work while those kernels still use it.
"""
import contextlib

import pytest
import torch

from prompt_compression_b200 import binding as B


def _bf16(*shape):
    return torch.zeros(shape, dtype=torch.bfloat16)


def _f32(*shape):
    return torch.zeros(shape, dtype=torch.float32)


def _i32(*shape):
    return torch.zeros(shape, dtype=torch.int32)


@pytest.fixture(scope="module", autouse=True)
def lib():
    from prompt_compression_b200 import build
    build.build_library()
    return B.load_library()


def test_speckv_score_rejects_wrong_output_sizes():
    q, k = _bf16(1, 2, 4, 24, 64), _bf16(1, 2, 2, 300, 64)      # 4 units, n_window 8 -> n_pre 292
    with pytest.raises(ValueError, match="scores has"):
        B.speckv_score(q, k, 8, _f32(4, 291))
    with pytest.raises(ValueError, match="window_mass has"):
        B.speckv_score(q, k, 8, _f32(4, 292), window_mass=_f32(4, 7))
    with pytest.raises(ValueError, match="lse2 has"):
        B.speckv_row_lse(q, k, 8, _f32(4, 2 * 24 - 1))
    # the right sizes get as far as the device checks
    with pytest.raises(ValueError, match="CUDA"):
        B.speckv_score(q, k, 8, _f32(4, 292), workspace=torch.zeros(1 << 20, dtype=torch.uint8))
    with pytest.raises(ValueError, match="disagree"):
        B.speckv_score(q, _bf16(1, 3, 2, 300, 64), 8, _f32(4, 292))


def test_specpc_score_rejects_wrong_sizes():
    q, k = _bf16(2, 3, 4, 16, 64), _bf16(2, 3, 2, 100, 64)
    with pytest.raises(ValueError, match="row_weights has"):
        B.specpc_score(q, k, _f32(15), _f32(2, 100), 1)
    with pytest.raises(ValueError, match="scores has"):
        B.specpc_score(q, k, _f32(16), _f32(2, 99), 1)
    with pytest.raises(ValueError, match="disagree"):
        B.specpc_score(q, _bf16(2, 3, 2, 100, 128), _f32(16), _f32(2, 100), 1)


def test_topk_select_rejects_wrong_sizes():
    s = _f32(3, 500)
    with pytest.raises(ValueError, match="idx has"):
        B.topk_select(s, 40, 8, _i32(3, 47))
    with pytest.raises(ValueError, match="idx has"):
        B.topk_select(s, 900, 0, _i32(3, 900))                   # k > n_cand keeps n_cand
    with pytest.raises(ValueError, match="pooled has"):
        B.topk_select(s, 40, 8, _i32(3, 48), pooled=_f32(3, 499))
    with pytest.raises(ValueError, match="units, n_cand"):
        B.topk_select(_f32(1500), 40, 8, _i32(3, 48))
    with pytest.raises(ValueError, match="CUDA"):
        B.topk_select(s, 900, 0, _i32(3, 500), workspace=torch.zeros(1 << 16, dtype=torch.uint8))


def test_kv_compact_rejects_wrong_sizes():
    k, v = _bf16(6, 300, 64), _bf16(6, 300, 64)
    idx = _i32(2, 40)                                            # shared by 3 units each
    ok_out = _bf16(6, 40, 64)
    with pytest.raises(ValueError, match="idx has"):
        B.kv_compact(k, v, idx, ok_out, ok_out.clone(), units_per_idx=1)
    with pytest.raises(ValueError, match="k_out has"):
        B.kv_compact(k, v, idx, _bf16(6, 39, 64), ok_out.clone(), units_per_idx=3)
    with pytest.raises(ValueError, match="v_out has"):
        B.kv_compact(k, v, idx, ok_out, _bf16(5, 40, 64), units_per_idx=3)
    with pytest.raises(ValueError, match="multiple"):
        B.kv_compact(k, v, _i32(1, 40), ok_out, ok_out.clone(), units_per_idx=4)
    with pytest.raises(ValueError, match="element size"):
        B.kv_compact(k, v, idx, torch.zeros((6, 40, 64), dtype=torch.float32), ok_out.clone(), units_per_idx=3)
    with pytest.raises(ValueError, match="together"):
        B.kv_compact(k, v, idx, ok_out, None, units_per_idx=3)
    with pytest.raises(ValueError, match="shape"):
        B.kv_compact(k, _bf16(6, 301, 64), idx, ok_out, ok_out.clone(), units_per_idx=3)


def test_decode_attention_rejects_wrong_sizes():
    q, k = _bf16(1, 2, 8, 128), _bf16(1, 2, 2, 50, 128)
    with pytest.raises(ValueError, match="out has"):
        B.decode_attention(q, k, k.clone(), out=_f32(1, 2, 8, 127))
    with pytest.raises(ValueError, match="must be"):
        B.decode_attention(q, k, _bf16(1, 2, 2, 51, 128), out=_f32(1, 2, 8, 128))


def test_temporary_workspace_is_allocated_on_the_launch_stream(monkeypatch):
    # A workspace the binding creates is released when the call returns while
    # the kernels may still be running on `stream`; allocating it under that
    # stream ties its memory to that stream's later work only.
    entered = []
    allocated_under = []

    @contextlib.contextmanager
    def fake_stream_ctx(s):
        entered.append(s)
        try:
            yield
        finally:
            entered.pop()

    def fake_empty(*args, **kwargs):
        allocated_under.append(entered[-1] if entered else None)
        return torch.zeros(4, dtype=torch.uint8)

    sentinel = object()
    monkeypatch.setattr(B, "_stream_object", lambda stream, device: sentinel if stream == 1234 else None)
    monkeypatch.setattr(B.torch.cuda, "stream", fake_stream_ctx)
    monkeypatch.setattr(B.torch, "empty", fake_empty)
    B._workspace(None, 4096, "cpu", 1234)
    assert allocated_under == [sentinel]
    given = torch.zeros(8, dtype=torch.uint8)
    assert B._workspace(given, 4096, "cpu", 1234) is given      # the caller's workspace is used as is
    assert allocated_under == [sentinel]
