"""Picard sweeps before the Newton iterations (pararnn_newton_forward_picard)
and the measured Newton budget K = 0 selects, on the GPU through the C ABI,
against the fp64 oracle.

Tolerances as in test_gpu_parity: H <= 1e-4 (relative error with a 1e-2 * max
floor); residual histories to float32 rounding of the O(1) residuals.
"""
import numpy as np
import pytest
import torch

import oracle
import slow_inputs
from gpu_util import rel_err, to_np
from nonlinear_rnn_iteration_b200 import binding, workloads

pytestmark = pytest.mark.gpu
TOL_H = 1e-4
DEV = "cuda:0"


def _inputs(cell, B, T, D, seed, h0=False, bf16=False):
    rng = np.random.default_rng(seed)
    G, S = oracle.NUM_GATES[cell], oracle.STATE_WIDTH[cell]
    px = rng.standard_normal((B, T, G, D)).astype(np.float32)
    w = rng.uniform(-0.5, 0.5, (G, D)).astype(np.float32)
    hz = (0.5 * rng.standard_normal((B, S, D))).astype(np.float32) if h0 else None
    px_used = workloads.round_bf16(px) if bf16 else px
    t = lambda a: None if a is None else torch.from_numpy(np.ascontiguousarray(a)).to(DEV)
    pxt = t(px).to(torch.bfloat16) if bf16 else t(px)
    return dict(px=px_used, w=w, h0=hz, pxt=pxt, wt=t(w), h0t=t(hz))


# several tiles along T and D, ragged tails, the TMA path (D % 4 == 0) and the
# element-wise path (odd D), sequences shorter than the Picard reach
CASES = [
    (oracle.DIAG_GRU, 2, 300, 136),
    (oracle.DIAG_GRU, 1, 131, 37),
    (oracle.DIAG_GRU, 1, 3, 8),
    (oracle.DIAG_LSTM, 2, 250, 72),
    (oracle.DIAG_LSTM, 1, 77, 13),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "cell%d_B%dT%dD%d" % c)
@pytest.mark.parametrize("P", [1, 2, 4])
@pytest.mark.parametrize("h0", [False, True])
def test_picard_forward(case, P, h0, cuda_device):
    cell, B, T, D = case
    K = 2
    x = _inputs(cell, B, T, D, seed=T + D + P, h0=h0)
    resid = torch.zeros(K + 1, device=DEV)
    H = binding.newton_forward(cell, x["pxt"], x["wt"], x["h0t"], K=K, resid_hist=resid, picard_iters=P)
    Ho, ro = oracle.newton_picard(cell, x["px"], x["w"], x["h0"], P=P, K=K)
    assert rel_err(to_np(H), Ho) <= TOL_H
    r = to_np(resid)
    assert np.all(np.abs(r - ro) <= 1e-4 * max(1.0, ro[0]) + 1e-5 * ro), (r, ro)


@pytest.mark.parametrize("cell", [oracle.DIAG_GRU, oracle.DIAG_LSTM])
def test_picard_bf16_and_slow_memory(cell, cuda_device):
    x = _inputs(cell, 2, 400, 64, seed=3, bf16=True)
    H = binding.newton_forward(cell, x["pxt"], x["wt"], None, K=3, picard_iters=2)
    Ho, _ = oracle.newton_picard(cell, x["px"], x["w"], None, P=2, K=3)
    assert rel_err(to_np(H), Ho) <= TOL_H
    # slow memory: carries between tiles that do not vanish
    px, w, hz, _ = slow_inputs.diag_host(cell, 2, 700, 72, 17)
    t = lambda a: None if a is None else torch.from_numpy(np.ascontiguousarray(a)).to(DEV)
    H = binding.newton_forward(cell, t(px), t(w), t(hz), K=3, picard_iters=3)
    Ho, _ = oracle.newton_picard(cell, px, w, hz, P=3, K=3)
    assert rel_err(to_np(H), Ho) <= TOL_H


def test_picard_zero_is_the_plain_forward(cuda_device):
    for cell in (oracle.LINEAR, oracle.DIAG_GRU, oracle.DIAG_LSTM):
        x = _inputs(cell, 2, 500, 96, seed=8)
        if cell == oracle.LINEAR:
            x["pxt"][:, :, 0, :] = torch.sigmoid(x["pxt"][:, :, 0, :])
            x["wt"] = None
        H0 = binding.newton_forward(cell, x["pxt"], x["wt"], None, K=2)
        S = oracle.STATE_WIDTH[cell]
        H1 = torch.empty_like(H0)
        ws = binding.workspace_for(cell, 2, 500, 96, 2, DEV)
        st = binding.pararnn_newton_forward_picard(cell, 2, 500, 96, binding.F32, x["pxt"], x["wt"], None, 0, 2, H1,
                                                   ws, ws.numel(), None, torch.cuda.current_stream())
        assert st == binding.OK
        torch.cuda.synchronize()
        assert torch.equal(H0, H1)
        if cell == oracle.LINEAR:
            # the linear cell is exact in one scan and ignores the sweeps
            H2 = binding.newton_forward(cell, x["pxt"], None, None, K=2, picard_iters=3)
            assert torch.equal(H0, H2)
        assert H0.shape[2] == S


def test_picard_sweeps_make_rows_exact(cuda_device):
    # with h0 = 0, P sweeps and K Newton steps fix the first P + K + 1 rows;
    # P = T - 1 sweeps and one Newton step reproduce the whole unroll
    for cell in (oracle.DIAG_GRU, oracle.DIAG_LSTM):
        x = _inputs(cell, 1, 5, 40, seed=12)
        U = oracle.unroll(cell, x["px"], x["w"])
        H = binding.newton_forward(cell, x["pxt"], x["wt"], None, K=1, picard_iters=4)
        assert rel_err(to_np(H), U) <= TOL_H


@pytest.mark.parametrize("cell", [oracle.DIAG_GRU, oracle.DIAG_LSTM])
@pytest.mark.parametrize("T", [300, 5000])
def test_k_zero_takes_the_measured_kstar(cell, T, cuda_device):
    B, D = 2, 64
    x = _inputs(cell, B, T, D, seed=T)
    ks = binding.pararnn_kstar(cell, T)
    assert 1 <= ks <= 8
    resid = torch.zeros(ks + 1, device=DEV)
    H0 = binding.newton_forward(cell, x["pxt"], x["wt"], None, K=0, resid_hist=resid)
    Hk = binding.newton_forward(cell, x["pxt"], x["wt"], None, K=ks)
    assert torch.equal(H0, Hk)
    Ho, ro = oracle.newton(cell, x["px"], x["w"], None, K=ks)
    assert rel_err(to_np(H0), Ho) <= TOL_H
    r = to_np(resid)
    assert np.all(np.abs(r - ro) <= 1e-4 * max(1.0, ro[0]) + 1e-5 * ro), (r, ro)
    # the budget it chose reaches the sequential unroll within the table's 1e-4
    U = oracle.unroll(cell, x["px"], x["w"])
    assert rel_err(to_np(H0), U) <= 1e-4
