"""The library's FMA-pipe 2^x (a Cody-Waite split and a degree-5 polynomial fitted to 2^f on
[-1/2, 1/2]; used for part of the summaries' weights) against 2^x in fp64: within 3e-7
relative for x in [-120, 0] (the MUFU ex2.approx path has an error of the same order), and at
most 2^-119 below (a weight that small is negligible next to the maximum's 1)."""
import ctypes

import numpy as np
import pytest

pytestmark = pytest.mark.gpu


def test_exp2_polynomial_accuracy():
    import torch
    import linear_attention_rnn_wkv_b200 as wkv
    L = wkv.lib()
    f = L.wkv_testhook_exp2_fma
    f.argtypes = [ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
    f.restype = ctypes.c_int
    rng = np.random.default_rng(11)
    x = np.concatenate([np.linspace(-120.0, 0.0, 1_000_001), rng.uniform(-120.0, 0.0, 1_000_000),
                        -np.arange(121, dtype=np.float64), np.arange(-125.0, 0.0, 0.5) + 0.25,
                        [-130.0, -1e4, -1e38, -0.0]]).astype(np.float32)
    xg = torch.from_numpy(x).cuda()
    yg = torch.empty_like(xg)
    assert f(x.size, xg.data_ptr(), yg.data_ptr(), torch.cuda.current_stream().cuda_stream) == 0
    torch.cuda.synchronize()
    y = yg.cpu().numpy().astype(np.float64)
    exact = np.exp2(x.astype(np.float64))
    inside = x >= -120.0
    rel = np.abs(y[inside] / exact[inside] - 1.0)
    assert rel.max() <= 3e-7, rel.max()
    assert np.all(np.isfinite(y)) and np.all(y >= 0.0)
    assert np.all(y[~inside] <= 2.0 ** -119)
    assert y[x == 0.0].min() == pytest.approx(1.0, rel=3e-7)
