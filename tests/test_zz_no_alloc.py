"""speckv_score_static_ws: the scoring entry point for callers that cannot
allocate device memory (engines that own all of HBM through their own pool,
plugin hosts without access to the CUDA allocator).  It keeps its scratch in
a fixed array inside the library, so it must give the same scores as the
workspace entry point, call after call, even though every call reuses (and
never clears) that array.  This file is collected last on purpose."""
import ctypes

import numpy as np
import pytest

from tests.gpu_helpers import assert_scores_close

pytestmark = pytest.mark.gpu


def _lib():
    from prompt_compression_b200 import build
    build.build_library()
    from prompt_compression_b200 import binding as B
    lib = B.load_library()
    fn = lib.speckv_score_static_ws
    fn.restype = ctypes.c_int
    fn.argtypes = [ctypes.POINTER(B.SpeckvShape), ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                   ctypes.c_void_p, ctypes.c_void_p]
    return lib, B


@pytest.mark.parametrize("shape", [
    # B, L, hq, hkv, d, n_in, n_window, n_lookahead
    (1, 1, 4, 2, 64, 512, 16, 16),
    (1, 4, 8, 2, 128, 3000, 64, 64),
    (1, 2, 10, 2, 128, 1111, 64, 128),      # 960 rows per unit, ragged keys
])
def test_static_scratch_matches_workspace_entry(shape):
    import torch
    lib, B = _lib()
    Bsz, L, hq, hkv, d, n_in, nw, nl = shape
    gen = torch.Generator(device="cuda").manual_seed(sum(shape))
    q = (torch.randn((Bsz, L, hq, nw + nl, d), generator=gen, device="cuda") / d ** 0.5).to(torch.bfloat16)
    k = torch.randn((Bsz, L, hkv, n_in, d), generator=gen, device="cuda").to(torch.bfloat16)
    units = Bsz * L * hkv
    ref = torch.empty((units, n_in - nw), dtype=torch.float32, device="cuda")
    ref_wm = torch.empty((units, nw), dtype=torch.float32, device="cuda")
    B.speckv_score(q, k, nw, ref, ref_wm)
    sh = B.speckv_shape(q, k, nw)
    stream = torch.cuda.current_stream().cuda_stream
    for call in range(2):                     # the second call reuses the array as the first left it
        out = torch.full((units, n_in - nw), float("nan"), dtype=torch.float32, device="cuda")
        wm = torch.full((units, nw), float("nan"), dtype=torch.float32, device="cuda")
        rc = lib.speckv_score_static_ws(ctypes.byref(sh), q.data_ptr(), k.data_ptr(), out.data_ptr(),
                                        wm.data_ptr(), stream)
        assert rc == 0, lib.spk_last_error().decode()
        torch.cuda.synchronize()
        assert_scores_close(out.cpu().numpy(), ref.cpu().numpy(), f"call {call} scores")
        assert_scores_close(wm.cpu().numpy(), ref_wm.cpu().numpy(), f"call {call} window mass")
    from prompt_compression_b200 import spk_device_error
    assert spk_device_error() == (0, 0)


def test_static_scratch_rejects_oversized_shapes():
    lib, B = _lib()
    # 64 layers x 8 KV heads x 1024 padded rows x 32 B = 16 MiB fits; 4 batch elements do not
    ok = B.SpeckvShape(1, 64, 40, 8, 128, 65536, 64, 128, 1.0)
    big = B.SpeckvShape(4, 64, 40, 8, 128, 65536, 64, 128, 1.0)
    rc = lib.speckv_score_static_ws(ctypes.byref(big), 256, 256, 256, None, None)
    assert rc == B.SPK_ERR_UNSUPPORTED
    assert "static scratch" in lib.spk_last_error().decode()
    assert lib.speckv_workspace_size(ctypes.byref(ok)) <= 1 << 24
