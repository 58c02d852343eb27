"""The slow-memory parity inputs really make tile and chunk products matter
(CPU, oracle only): with them, a unit gradient at the last step still
reaches 80 steps back (the longest diagonal tile), and a 128-step chunk
product of head-wise Jacobians keeps a norm above 0.1.  With the standard
inputs both are 1e-13 .. 1e-28."""
import numpy as np
import pytest

import oracle
import slow_inputs
from nonlinear_rnn_iteration_b200 import workloads


def _reach(cell, px, w, hz):
    H = oracle.unroll(cell, px, w, hz)
    T = px.shape[1]
    g = np.zeros((1, T, oracle.STATE_WIDTH[cell], px.shape[3]))
    g[0, -1, -1, :] = 1.0  # dL/dh at the last step only
    dpx, _, _ = oracle.adjoint(cell, px, w, hz, H, g)
    return np.abs(dpx[0, T - 81]).max()


@pytest.mark.parametrize("cell", [oracle.LINEAR, oracle.DIAG_GRU, oracle.DIAG_LSTM])
def test_diag_tile_reach(cell):
    px, w, hz, _ = slow_inputs.diag_host(cell, 1, 400, 8, seed=5)
    assert _reach(cell, px, w, hz) > 1e-3
    # the standard recipe: the same gradient has vanished 80 steps back
    rng = np.random.default_rng(5)
    G, S = oracle.NUM_GATES[cell], oracle.STATE_WIDTH[cell]
    px = rng.standard_normal((1, 400, G, 8)).astype(np.float32)
    if cell == oracle.LINEAR:
        px[:, :, 0, :] = 1.0 / (1.0 + np.exp(-px[:, :, 0, :]))
    w = None if cell == oracle.LINEAR else rng.uniform(-0.5, 0.5, (G, 8)).astype(np.float32)
    hz = (0.5 * rng.standard_normal((1, S, 8))).astype(np.float32)
    assert _reach(cell, px, w, hz) < 1e-9


def _chunk_product_norm(px, U):
    H = oracle.head_gru_unroll(px, U)
    Q = np.eye(U.shape[-1])
    for t in range(128, 256):
        Q = oracle.head_gru_jacobian(px[0, t], U[:, 0], H[0, t - 1]) @ Q
    return np.linalg.norm(Q, 2)


def test_head_chunk_product_norm():
    px, U = slow_inputs.head_host(1, 300, 64, 1, seed=364)
    assert _chunk_product_norm(px, U) > 0.1
    x = workloads.head_host_inputs(1, 300, 64, 1, 364)
    assert _chunk_product_norm(x["px"], x["U"]) < 1e-20
