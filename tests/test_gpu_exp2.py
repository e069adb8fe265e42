"""The FMA-pipe exponential used by the scoring epilogues, against exp2 in
fp64 (numpy) and against CUDA's exp2f, over its argument range."""
import numpy as np
import pytest

pytestmark = pytest.mark.gpu


def test_exp2_fma_relative_error():
    import torch
    from prompt_compression_b200 import build
    build.build_library()
    import prompt_compression_b200 as P
    t = torch.cat([torch.linspace(-126.0, 0.5, 2_000_001), torch.linspace(-1.0, 1.0, 100_001),
                   torch.tensor([0.0, -0.5, 0.5, -125.5, -1e-7, 3.0, 20.0])]).float().cuda()
    y = torch.empty_like(t)
    P.spk_exp2_fma(t, y)
    ref_cuda = torch.exp2(t)                         # CUDA's exp2f
    torch.cuda.synchronize()
    tt = t.cpu().numpy().astype(np.float64)
    got = y.cpu().numpy().astype(np.float64)
    exact = np.exp2(tt)
    normal = tt >= -125.0                            # results in the normal fp32 range
    rel = np.abs(got[normal] / exact[normal] - 1.0)
    assert rel.max() <= 3e-6, rel.max()
    rel_cuda = np.abs(got[normal] / ref_cuda.cpu().numpy().astype(np.float64)[normal] - 1.0)
    assert rel_cuda.max() <= 3.3e-6, rel_cuda.max()
    # below the normal range the value is tiny and never negative
    assert (got >= 0).all() and got[tt < -125].max(initial=0) < 2.4e-38
    # exact at the integers
    ints = np.arange(-120, 4, dtype=np.float32)
    ti = torch.from_numpy(ints).cuda()
    yi = torch.empty_like(ti)
    P.spk_exp2_fma(ti, yi)
    torch.cuda.synchronize()
    np.testing.assert_allclose(yi.cpu().numpy(), np.exp2(ints.astype(np.float64)), rtol=3e-6)


def test_exp2_fma_clamps_minus_infinity():
    import torch
    import prompt_compression_b200 as P
    t = torch.tensor([-float("inf"), -1e30, -200.0, -126.0], device="cuda")
    y = torch.empty_like(t)
    P.spk_exp2_fma(t, y)
    torch.cuda.synchronize()
    v = y.cpu().numpy()
    assert np.all(v >= 0) and np.all(v < 2.4e-38)
