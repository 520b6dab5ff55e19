"""GPU: the FMA-pipe exponential (schnet_test_exp2) against float64 exp2 and
against CUDA's own exp2f (torch.exp2 on the device), over the arguments the
softplus gives it (x <= 0; below -30 the argument is taken as -30)."""
import ctypes as C

import numpy as np
import pytest
import torch

from schnet_gnn_molecular_b200 import _native as nat

pytestmark = pytest.mark.gpu


def _run(x: np.ndarray) -> np.ndarray:
    lib = nat.load()
    xd = torch.as_tensor(x.astype(np.float32), device="cuda")
    yd = torch.empty_like(xd)
    st = lib.schnet_test_exp2(C.c_void_p(xd.data_ptr()), C.c_void_p(yd.data_ptr()), xd.numel(),
                              C.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0
    torch.cuda.synchronize()
    return yd.cpu().numpy()


def test_against_float64_and_exp2f():
    rng = np.random.default_rng(3)
    x = np.concatenate([np.linspace(-30.0, 0.0, 1_000_001), -rng.exponential(3.0, 200_001),
                        [0.0, -0.5, -1.0, -1.5, -29.5, -30.0]]).astype(np.float32)
    x = np.maximum(x, -30.0).astype(np.float32)
    y = _run(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    assert np.max(np.abs(y / ref - 1)) <= 2.5e-7
    cuda = torch.exp2(torch.as_tensor(x, device="cuda")).cpu().numpy().astype(np.float64)
    assert np.max(np.abs(y / cuda - 1)) <= 4e-7


def test_clamp_and_odd_length():
    x = np.array([-31.0, -100.0, -1e30, -0.25, -7.0], dtype=np.float32)
    y = _run(x)
    assert y[0] == y[1] == y[2] and abs(y[0] / 2 ** -30 - 1) <= 2.5e-7
    assert abs(y[3] / 2 ** -0.25 - 1) <= 2.5e-7 and abs(y[4] / 2 ** -7 - 1) <= 2.5e-7
