"""Closed-form special cases, derived by hand, and the oracle regression fixture.

The pages print no worked example with numbers, so the hand-derived cases
below are the ones the mathematics fixes:

* linear cell, a = 1/2, b = 1 (News section of the pararnn-torch page: an
  affine recurrence is one exact scan): h_t = sum_{s<=t} 2^{-(t-s)}
  = 2 - 2^{-t} from h_{-1} = 0, and h = 2 is a fixed point.
* GRU with z = r = 1 (pre-activations +40 saturate the sigmoid to 1.0 in
  double precision) and a_c = 1, p_c = 0: f(h) = tanh(h), so the unroll is the
  iterated tanh, one Newton step from the zero warm start gives
  (tanh(h0), tanh(h0)) on T = 2, and the second step gives the unroll.
* LSTM with zero weights, i = 0, f = 1, o = 1/2 (pre-activations -40, +40, 0):
  c stays at c0 and h_t = tanh(c0) / 2.
"""
import json
import math
import os

import numpy as np

import oracle
from nonlinear_rnn_iteration_b200 import workloads

HERE = os.path.dirname(os.path.abspath(__file__))


def test_linear_closed_form():
    T = 6
    px = np.zeros((1, T, 2, 1))
    px[0, :, 0, 0] = 0.5
    px[0, :, 1, 0] = 1.0
    H = oracle.unroll(oracle.LINEAR, px)
    assert np.allclose(H[0, :, 0, 0], [2.0 - 2.0 ** (-t) for t in range(T)], rtol=0, atol=1e-15)
    Hf = oracle.unroll(oracle.LINEAR, px, None, np.full((1, 1, 1), 2.0))
    assert np.all(Hf == 2.0)


def test_gru_iterated_tanh():
    T, h0 = 5, 1.0
    px = np.zeros((1, T, 3, 1))
    px[0, :, 0, 0] = 40.0  # z = 1
    px[0, :, 1, 0] = 40.0  # r = 1
    w = np.array([[0.0], [0.0], [1.0]])
    H = oracle.unroll(oracle.DIAG_GRU, px, w, np.full((1, 1, 1), h0))
    ref, s = [], h0
    for _ in range(T):
        s = math.tanh(s)
        ref.append(s)
    assert np.allclose(H[0, :, 0, 0], ref, rtol=0, atol=1e-15)
    H1, _ = oracle.newton(oracle.DIAG_GRU, px[:, :2], w, np.full((1, 1, 1), h0), K=1)
    assert np.allclose(H1[0, :, 0, 0], [math.tanh(h0), math.tanh(h0)], rtol=0, atol=1e-15)
    H2, _ = oracle.newton(oracle.DIAG_GRU, px[:, :2], w, np.full((1, 1, 1), h0), K=2)
    assert np.allclose(H2[0, :, 0, 0], ref[:2], rtol=0, atol=1e-15)


def test_lstm_frozen_cell():
    T, c0 = 4, 1.0
    px = np.zeros((1, T, 4, 1))
    px[0, :, 0, 0] = -40.0  # i = 0
    px[0, :, 1, 0] = 40.0   # f = 1
    w = np.zeros((4, 1))
    h0 = np.array([[[c0], [0.0]]])
    H = oracle.unroll(oracle.DIAG_LSTM, px, w, h0)
    assert np.allclose(H[0, :, 0, 0], c0, rtol=0, atol=1e-15)
    assert np.allclose(H[0, :, 1, 0], 0.5 * math.tanh(c0), rtol=0, atol=1e-15)


def test_oracle_regression_fixture():
    with open(os.path.join(HERE, "golden", "oracle_small.json")) as f:
        fx = json.load(f)
    for c in fx["cases"]:
        w = workloads.WORKLOADS[c["shaped_after"]].with_shape(B=c["B"], T=c["T"], D=c["D"], K=c["K"])
        x = workloads.host_inputs(w, seed=c["seed"], with_grad=True)
        H, resid = oracle.newton(w.cell_id, x["px"], x["a"], None, K=c["K"], nthreads=2)
        dpx, da, dh0 = oracle.adjoint(w.cell_id, x["px"], x["a"], None, H, x["dLdH"], nthreads=2)
        for got, key in ((H, "H"), (resid, "resid"), (dpx, "dLdpx"), (da, "dLda"), (dh0, "dLdh0")):
            np.testing.assert_allclose(np.ravel(got), c[key], rtol=1e-12, atol=1e-14, err_msg=key)
