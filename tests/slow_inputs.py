"""Slow-memory inputs for the parity tests (numpy only, no GPU).

With the standard input recipe a step's Jacobian is about 0.5 in size, so
the product over a tile or chunk of 32-128 steps is 1e-10 .. 1e-28 and a
wrong product there would not show in any output.  These inputs shift one
gate so that each step's Jacobian stays near 1:
  linear cell   a_t = sig(N(0,1) + 5)
  GRU           p_z - 5  (the update gate almost closed)
  LSTM          p_f + 2  (a larger shift makes the first Newton iterates
                          from the zero guess overflow-sized)
  head-wise GRU p_z - 5
"""
import numpy as np

import oracle
from nonlinear_rnn_iteration_b200 import workloads

# (gate index, shift) per diagonal cell
DIAG_SHIFT = {oracle.LINEAR: (0, 5.0), oracle.DIAG_GRU: (0, -5.0), oracle.DIAG_LSTM: (1, 2.0)}
HEAD_SHIFT = -5.0  # added to p_z of the head-wise GRU


def diag_host(cell, B, T, D, seed):
    """px (B,T,G,D), w (G,D) or None, h0 (B,S,D), dL/dH (B,T,S,D), float32."""
    rng = np.random.default_rng(seed)
    G, S = oracle.NUM_GATES[cell], oracle.STATE_WIDTH[cell]
    px = rng.standard_normal((B, T, G, D)).astype(np.float32)
    gate, shift = DIAG_SHIFT[cell]
    px[:, :, gate, :] += shift
    if cell == oracle.LINEAR:
        px[:, :, 0, :] = 1.0 / (1.0 + np.exp(-px[:, :, 0, :]))
        w = None
    else:
        w = rng.uniform(-0.5, 0.5, (G, D)).astype(np.float32)
    hz = (0.5 * rng.standard_normal((B, S, D))).astype(np.float32)
    g = rng.standard_normal((B, T, S, D)).astype(np.float32)
    return px, w, hz, g


def head_host(B, T, D, nh, seed):
    """The head-wise recipe (workloads.head_host_inputs) with p_z shifted: px, U."""
    x = workloads.head_host_inputs(B, T, D, nh, seed)
    px = x["px"].copy()
    px[:, :, 0, :] += HEAD_SHIFT
    return px, x["U"]
