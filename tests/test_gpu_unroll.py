"""The sequential unroll of the diagonal cells on the GPU (pararnn_unroll)
against the fp64 oracle's unroll, through the C ABI: every cell, f32 and
bf16 pre-activations, an initial state, ragged sizes and slow memory, and the
Newton forward at K = T reaching the same sequence."""
import numpy as np
import pytest
import torch

import oracle
import slow_inputs
from gpu_util import rel_err, to_np
from nonlinear_rnn_iteration_b200 import binding

pytestmark = pytest.mark.gpu
TOL_H = 1e-4
DEV = "cuda:0"


def _inputs(cell, B, T, D, seed, h0=False, bf16=False):
    rng = np.random.default_rng(seed)
    G, S = oracle.NUM_GATES[cell], oracle.STATE_WIDTH[cell]
    px = rng.standard_normal((B, T, G, D)).astype(np.float32)
    if cell == oracle.LINEAR:
        px[:, :, 0, :] = 1.0 / (1.0 + np.exp(-px[:, :, 0, :]))
        w = None
    else:
        w = rng.uniform(-0.5, 0.5, (G, D)).astype(np.float32)
    hz = (0.5 * rng.standard_normal((B, S, D))).astype(np.float32) if h0 else None
    t = lambda a: None if a is None else torch.from_numpy(np.ascontiguousarray(a)).to(DEV)
    pxt = t(px).to(torch.bfloat16) if bf16 else t(px)
    px_used = pxt.float().cpu().numpy() if bf16 else px
    return px_used, w, hz, pxt, t(w), t(hz)


@pytest.mark.parametrize("cell", [oracle.LINEAR, oracle.DIAG_GRU, oracle.DIAG_LSTM])
@pytest.mark.parametrize("case", [(2, 300, 136), (1, 97, 37), (3, 5, 130), (1, 1, 1)], ids=lambda c: "B%dT%dD%d" % c)
@pytest.mark.parametrize("h0", [False, True])
def test_unroll_matches_oracle(cell, case, h0, cuda_device):
    B, T, D = case
    px, w, hz, pxt, wt, hzt = _inputs(cell, B, T, D, seed=T + D + cell, h0=h0)
    H = binding.unroll(cell, pxt, wt, hzt)
    assert rel_err(to_np(H), oracle.unroll(cell, px, w, hz)) <= TOL_H


@pytest.mark.parametrize("cell", [oracle.LINEAR, oracle.DIAG_GRU, oracle.DIAG_LSTM])
def test_unroll_bf16_slow_memory_and_newton(cell, cuda_device):
    px, w, hz, pxt, wt, hzt = _inputs(cell, 2, 400, 64, seed=3, bf16=True)
    H = binding.unroll(cell, pxt, wt, hzt)
    assert rel_err(to_np(H), oracle.unroll(cell, px, w, hz)) <= TOL_H
    spx, sw, shz, _ = slow_inputs.diag_host(cell, 2, 700, 72, 19)
    t = lambda a: None if a is None else torch.from_numpy(np.ascontiguousarray(a)).to(DEV)
    H = binding.unroll(cell, t(spx), t(sw), t(shz))
    assert rel_err(to_np(H), oracle.unroll(cell, spx, sw, shz)) <= TOL_H
    # the Newton forward at K = T is the same sequence
    px, w, hz, pxt, wt, hzt = _inputs(cell, 1, 12, 40, seed=5, h0=True)
    Hn = binding.newton_forward(cell, pxt, wt, hzt, K=12)
    assert rel_err(to_np(Hn), to_np(binding.unroll(cell, pxt, wt, hzt))) <= TOL_H


def test_unroll_arguments_and_status(cuda_device):
    px = torch.zeros((1, 8, 3, 16), device=DEV)
    H = torch.empty((1, 8, 1, 16), device=DEV)
    ws = torch.empty(256, dtype=torch.uint8, device=DEV)
    s = torch.cuda.current_stream()
    assert binding.pararnn_unroll(9, 1, 8, 16, binding.F32, px, None, None, H, ws, 256, s) == binding.EINVAL
    assert binding.pararnn_unroll(binding.DIAG_GRU, 1, 8, 16, binding.F32, px, None, None, H, ws, 8, s) == binding.EINVAL
    assert binding.pararnn_unroll(binding.DIAG_GRU, 1, 8, 16, binding.F32, px.cpu(), None, None, H, ws, 256,
                                  s) == binding.EINVAL
    bad = torch.full((1, 8, 3, 16), float("nan"), device=DEV)
    assert binding.pararnn_unroll(binding.DIAG_GRU, 1, 8, 16, binding.F32, bad, None, None, H, ws, 256, s) == binding.OK
    assert binding.pararnn_status_sync(ws, s) == binding.ENONFINITE
