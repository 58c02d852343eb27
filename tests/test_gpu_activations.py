"""Accuracy of the kernels' own sigmoid and tanh, read through the public API.

A diagonal-GRU call with T = 1, no recurrent weights and h0 = 0 returns
h_0 = z c = sigma(p_z) tanh(p_c) per channel (one Newton step from the warm
start is exact for a one-step sequence).  With p_z = 40, sigma(p_z) rounds to
1.0 in float32, so H is tanh(p_c) as the kernels evaluate it; with p_c = 40,
tanh(p_c) rounds to 1.0 and H is sigma(p_z).  Both are compared over a dense
grid with the fp64 values and with CUDA's own float32 tanhf/expf (through
torch on the device).  The update gate shares its reciprocal with the reset
gate, with exponents capped at 2^62, so below 2^-62 sigma is that floor.
"""
import numpy as np
import pytest
import torch

from nonlinear_rnn_iteration_b200 import binding

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _grid():
    # dense around 0 and the series/definition switch at |x| = 1/16, then out
    # to saturation; both signs
    pos = np.concatenate([np.geomspace(1e-30, 1e-3, 200), np.linspace(1e-3, 0.2, 4000),
                          np.linspace(0.0625 - 1e-4, 0.0625 + 1e-4, 401), np.linspace(0.2, 20.0, 4000),
                          np.array([30.0, 50.0, 90.0, 1e4, 3e38])])
    x = np.concatenate([-pos[::-1], [0.0], pos]).astype(np.float32)
    n = (len(x) + 7) // 8 * 8  # D a multiple of 8: the vectorised path
    return np.pad(x, (0, n - len(x)))


def _gru_t1(pz, pc):
    D = len(pz)
    px = np.stack([pz, np.zeros_like(pz), pc])[None, None].astype(np.float32)  # (1,1,3,D)
    H = binding.newton_forward(binding.DIAG_GRU, torch.from_numpy(px).to(DEV), None, None, K=1)
    return H.reshape(D).cpu().numpy().astype(np.float64)


def test_tanh_matches_fp64_and_cuda(cuda_device):
    x = _grid()
    got = _gru_t1(np.full_like(x, 40.0), x)
    exact = np.tanh(x.astype(np.float64))
    cuda = torch.tanh(torch.from_numpy(x).to(DEV)).cpu().numpy().astype(np.float64)
    # relative error against fp64, with an absolute floor at the float32 spacing of 1
    err = np.abs(got - exact) / np.maximum(np.abs(exact), 2.0 ** -24)
    assert err.max() <= 4e-6, (x[err.argmax()], got[err.argmax()], exact[err.argmax()])
    assert np.abs(got - cuda).max() <= 4e-6
    assert (np.sign(got) == np.sign(exact)).all()
    assert np.abs(got).max() <= 1.0


def test_sigmoid_matches_fp64_and_cuda(cuda_device):
    x = _grid()
    x = x[np.abs(x) < 80]  # sigma saturates to 0 / 1 well before
    x = np.pad(x, (0, (-len(x)) % 8))
    got = _gru_t1(x, np.full_like(x, 40.0))
    exact = 1.0 / (1.0 + np.exp(-x.astype(np.float64)))
    cuda = torch.sigmoid(torch.from_numpy(x).to(DEV)).cpu().numpy().astype(np.float64)
    # the GRU's update and reset gates share one reciprocal, whose exponents
    # are capped at 2^62: below that sigma is returned as 2^-62
    capped = -x.astype(np.float64) * np.log2(np.e) > 61.9
    err = np.abs(got - exact) / np.maximum(exact, 1e-30)
    err[capped] = 0.0
    assert err.max() <= 4e-6, (x[err.argmax()], got[err.argmax()], exact[err.argmax()])
    assert np.abs(got - exact)[capped].max() <= 2.0 ** -61
    assert np.abs(got - cuda).max() <= 2e-6
    assert got.min() > 0.0 and got.max() <= 1.0
