"""fp64 CPU oracle for the ParaRNN hot path -- TEST INFRASTRUCTURE ONLY.

Only the test suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product library never calls it and
shares no code with it: the arithmetic lives in ``pararnn_oracle.c`` (plain C,
double precision, one channel at a time, sequential in time), and this module
only marshals numpy arrays into it.

Functions and what they follow:

* :func:`unroll` -- the sequential recurrence s_t = f(s_{t-1}, x_t)
  (pararnn-torch PyPI page, API overview: ``sequential_apply``).
* :func:`newton` -- K Newton iterations on F(H)_t = h_t - f(h_{t-1}, x_t) = 0
  from the warm start h^(0)_t = f(0, x_t) (pararnn-torch PyPI page, Method
  section; ParaRNN thread, tweet [3/8]); each step's linear system is solved
  by plain forward substitution.
* :func:`newton_picard` -- the same after P Picard (fixed-point) sweeps
  h^(p+1)_t = f(h^(p)_{t-1}, x_t) from the warm start (API overview,
  "Solver": ``picard_iters``; Method section: zero-hidden start + Picard).
* :func:`residual` -- max |F(H)| of a given trajectory.
* :func:`adjoint` -- reverse recursion lambda_t = g_t + A_{t+1}^T lambda_{t+1}
  at a given trajectory and the gradients w.r.t. pre-activations, diagonal
  weights and the initial state (Method section, backward pass).
* :func:`cell_step`, :func:`cell_jacobian`, :func:`cell_param_grads` -- one
  cell application and its closed-form derivatives, exposed for the pins.
* :func:`head_gru_unroll`, :func:`head_gru_newton`, :func:`head_gru_adjoint`,
  :func:`head_gru_step`, :func:`head_gru_jacobian` -- the same for the head-wise GRU
  (``ParaGRU(mix='head', n_heads)`` on the pararnn-torch page: block-diagonal
  recurrent weights, one dense d x d block per head, d = D / n_heads).

Cells: ``LINEAR`` (S=1, gates a,b), ``DIAG_GRU`` (S=1, gates z,r,c),
``DIAG_LSTM`` (S=2 state (c,h), gates i,f,o,c).  Layouts are row-major with
channels fastest: px (B,T,G,D), w (G,D), h0 (B,S,D), H (B,T,S,D).  The
head-wise GRU: px (B,T,3,D), U (3, n_heads, d, d), h0 (B,D), H (B,T,D).

Every function here is pinned by ``tests/test_oracle_pins.py`` against
library routines (torch.nn.GRU / LSTMCell, autograd, dense linear solves),
closed forms and brute force; none is "parity unpinned".
"""
from __future__ import annotations

import contextlib
import ctypes
import os
import subprocess

import numpy as np

LINEAR, DIAG_GRU, DIAG_LSTM = 0, 1, 2
NUM_GATES = {LINEAR: 2, DIAG_GRU: 3, DIAG_LSTM: 4}
STATE_WIDTH = {LINEAR: 1, DIAG_GRU: 1, DIAG_LSTM: 2}

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "pararnn_oracle.c")
_SO = os.path.join(_HERE, "liboracle.so")
_lib = None


def compile_source(src: str, so: str) -> str:
    """gcc -O2, IEEE double arithmetic: no fast-math, no FMA contraction."""
    tmp = so + ".tmp%d" % os.getpid()
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off",
                           "-fno-fast-math", "-o", tmp, src, "-lm", "-lpthread"])
    os.replace(tmp, so)
    return so


def build(force: bool = False) -> str:
    """Compile the oracle next to its source if it is missing or stale."""
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
        compile_source(_SRC, _SO)
    return _SO


@contextlib.contextmanager
def use_library(so_path: str):
    """Temporarily route every call to another build of the oracle source
    (the tests use this to check that a planted mistake fails a pin)."""
    global _lib
    saved = _lib
    _lib = _bind(so_path)
    try:
        yield
    finally:
        _lib = saved


def _load():
    global _lib
    if _lib is None:
        _lib = _bind(build())
    return _lib


def _bind(so_path):
    lib = ctypes.CDLL(so_path)
    P = ctypes.c_void_p
    i64 = ctypes.c_int64
    ci = ctypes.c_int
    for name in ("oracle_cell_step", "oracle_cell_jacobian"):
        getattr(lib, name).argtypes = [ci, P, P, P, P]
        getattr(lib, name).restype = None
    lib.oracle_cell_param_grads.argtypes = [ci, P, P, P, P, P]
    lib.oracle_cell_param_grads.restype = None
    lib.oracle_unroll.argtypes = [ci, i64, i64, i64, P, P, P, P, ci]
    lib.oracle_unroll.restype = ci
    lib.oracle_newton.argtypes = [ci, i64, i64, i64, P, P, P, ci, P, P, ci]
    lib.oracle_newton.restype = ci
    lib.oracle_newton_picard.argtypes = [ci, i64, i64, i64, P, P, P, ci, ci, P, P, ci]
    lib.oracle_newton_picard.restype = ci
    lib.oracle_residual.argtypes = [ci, i64, i64, i64, P, P, P, P, ci]
    lib.oracle_residual.restype = ctypes.c_double
    lib.oracle_adjoint.argtypes = [ci, i64, i64, i64, P, P, P, P, P, P, P, P, ci]
    lib.oracle_adjoint.restype = ci
    for name in ("oracle_head_gru_step", "oracle_head_gru_jacobian"):
        getattr(lib, name).argtypes = [ci, P, P, P, P]
        getattr(lib, name).restype = None
    lib.oracle_head_gru_unroll.argtypes = [i64, i64, i64, ci, P, P, P, P, ci]
    lib.oracle_head_gru_unroll.restype = ci
    lib.oracle_head_gru_newton.argtypes = [i64, i64, i64, ci, P, P, P, ci, P, P, ci]
    lib.oracle_head_gru_newton.restype = ci
    lib.oracle_head_gru_adjoint.argtypes = [i64, i64, i64, ci, P, P, P, P, P, P, P, P, ci]
    lib.oracle_head_gru_adjoint.restype = ci
    return lib


def _f64(x):
    if x is None:
        return None
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _threads(n):
    return max(1, int(n if n else (os.cpu_count() or 1)))


def _shape(cell, px):
    G = NUM_GATES[cell]
    if px.ndim != 4 or px.shape[2] != G:
        raise ValueError("px must be (B,T,%d,D), got %s" % (G, px.shape))
    B, T, _, D = px.shape
    return B, T, D


def cell_step(cell, p, w, s):
    lib = _load()
    p, w, s = _f64(p), _f64(w if w is not None else np.zeros(NUM_GATES[cell])), _f64(s)
    out = np.zeros(STATE_WIDTH[cell])
    lib.oracle_cell_step(cell, _ptr(p), _ptr(w), _ptr(s), _ptr(out))
    return out


def cell_jacobian(cell, p, w, s):
    lib = _load()
    S = STATE_WIDTH[cell]
    p, w, s = _f64(p), _f64(w if w is not None else np.zeros(NUM_GATES[cell])), _f64(s)
    A = np.zeros(S * S)
    lib.oracle_cell_jacobian(cell, _ptr(p), _ptr(w), _ptr(s), _ptr(A))
    return A.reshape(S, S)


def cell_param_grads(cell, p, w, s):
    lib = _load()
    S, G = STATE_WIDTH[cell], NUM_GATES[cell]
    p, w, s = _f64(p), _f64(w if w is not None else np.zeros(G)), _f64(s)
    dp, da = np.zeros(S * G), np.zeros(S * G)
    lib.oracle_cell_param_grads(cell, _ptr(p), _ptr(w), _ptr(s), _ptr(dp), _ptr(da))
    return dp.reshape(S, G), da.reshape(S, G)


def unroll(cell, px, w=None, h0=None, nthreads=None):
    lib = _load()
    px, w, h0 = _f64(px), _f64(w), _f64(h0)
    B, T, D = _shape(cell, px)
    H = np.zeros((B, T, STATE_WIDTH[cell], D))
    rc = lib.oracle_unroll(cell, B, T, D, _ptr(px), _ptr(w), _ptr(h0), _ptr(H), _threads(nthreads))
    if rc:
        raise ValueError("oracle_unroll rejected its arguments (%d)" % rc)
    return H


def newton(cell, px, w=None, h0=None, K=1, nthreads=None):
    """Returns (H^(K), resid) with resid[k] = max |F(H^(k))| for k = 0..K."""
    lib = _load()
    px, w, h0 = _f64(px), _f64(w), _f64(h0)
    B, T, D = _shape(cell, px)
    H = np.zeros((B, T, STATE_WIDTH[cell], D))
    resid = np.zeros(K + 1)
    rc = lib.oracle_newton(cell, B, T, D, _ptr(px), _ptr(w), _ptr(h0), int(K), _ptr(H), _ptr(resid),
                           _threads(nthreads))
    if rc:
        raise ValueError("oracle_newton rejected its arguments (%d)" % rc)
    return H, resid


def newton_picard(cell, px, w=None, h0=None, P=0, K=1, nthreads=None):
    """P Picard sweeps h^(p+1)_t = f(h^(p)_{t-1}, x_t) from the warm start,
    then K Newton iterations; returns (H^(K), resid) with resid[k] = max
    |F(H^(k))| for k = 0..K, H^(0) being the guess after the sweeps."""
    lib = _load()
    px, w, h0 = _f64(px), _f64(w), _f64(h0)
    B, T, D = _shape(cell, px)
    H = np.zeros((B, T, STATE_WIDTH[cell], D))
    resid = np.zeros(K + 1)
    rc = lib.oracle_newton_picard(cell, B, T, D, _ptr(px), _ptr(w), _ptr(h0), int(P), int(K), _ptr(H), _ptr(resid),
                                  _threads(nthreads))
    if rc:
        raise ValueError("oracle_newton_picard rejected its arguments (%d)" % rc)
    return H, resid


def residual(cell, px, w, h0, H, nthreads=None):
    """max |F(H)|_t = max |H_t - f(H_{t-1}, x_t)| over the whole batch, for a
    given trajectory H (B,T,S,D); H_{-1} = h0."""
    lib = _load()
    px, w, h0, H = _f64(px), _f64(w), _f64(h0), _f64(H)
    B, T, D = _shape(cell, px)
    if H.shape != (B, T, STATE_WIDTH[cell], D):
        raise ValueError("H must be (B,T,S,D) = %s, got %s" % ((B, T, STATE_WIDTH[cell], D), H.shape))
    r = float(lib.oracle_residual(cell, B, T, D, _ptr(px), _ptr(w), _ptr(h0), _ptr(H), _threads(nthreads)))
    if r < 0:
        raise ValueError("oracle_residual rejected its arguments (%g)" % r)
    return r


def adjoint(cell, px, w, h0, H, dLdH, nthreads=None):
    """Returns (dL_dpx (B,T,G,D), dL_da (G,D), dL_dh0 (B,S,D)) at trajectory H."""
    lib = _load()
    px, w, h0, H, dLdH = _f64(px), _f64(w), _f64(h0), _f64(H), _f64(dLdH)
    B, T, D = _shape(cell, px)
    G, S = NUM_GATES[cell], STATE_WIDTH[cell]
    if H.shape != (B, T, S, D) or dLdH.shape != (B, T, S, D):
        raise ValueError("H and dL_dH must be (B,T,S,D)")
    dpx = np.zeros((B, T, G, D))
    da = np.zeros((G, D))
    dh0 = np.zeros((B, S, D))
    rc = lib.oracle_adjoint(cell, B, T, D, _ptr(px), _ptr(w), _ptr(h0), _ptr(H), _ptr(dLdH), _ptr(dpx),
                            _ptr(da), _ptr(dh0), _threads(nthreads))
    if rc:
        raise ValueError("oracle_adjoint rejected its arguments (%d)" % rc)
    return dpx, da, dh0


# ---- head-wise GRU ---------------------------------------------------------

def _head_shape(px, U):
    if px.ndim != 4 or px.shape[2] != 3:
        raise ValueError("px must be (B,T,3,D), got %s" % (px.shape,))
    B, T, _, D = px.shape
    if U.ndim != 4 or U.shape[0] != 3 or U.shape[2] != U.shape[3] or U.shape[1] * U.shape[2] != D:
        raise ValueError("U must be (3, n_heads, d, d) with n_heads * d = D, got %s" % (U.shape,))
    return B, T, D, U.shape[1]


def head_gru_step(p, U, s):
    """One head: p (3, d) = (p_z, p_r, p_c), U (3, d, d), s (d,) -> f (d,)."""
    lib = _load()
    p, U, s = _f64(p), _f64(U), _f64(s)
    d = s.shape[0]
    out = np.zeros(d)
    lib.oracle_head_gru_step(d, _ptr(p), _ptr(U), _ptr(s), _ptr(out))
    return out


def head_gru_jacobian(p, U, s):
    """One head: d f / d s, (d, d)."""
    lib = _load()
    p, U, s = _f64(p), _f64(U), _f64(s)
    d = s.shape[0]
    A = np.zeros((d, d))
    lib.oracle_head_gru_jacobian(d, _ptr(p), _ptr(U), _ptr(s), _ptr(A))
    return A


def head_gru_unroll(px, U, h0=None, nthreads=None):
    lib = _load()
    px, U, h0 = _f64(px), _f64(U), _f64(h0)
    B, T, D, nh = _head_shape(px, U)
    H = np.zeros((B, T, D))
    rc = lib.oracle_head_gru_unroll(B, T, D, nh, _ptr(px), _ptr(U), _ptr(h0), _ptr(H), _threads(nthreads))
    if rc:
        raise ValueError("oracle_head_gru_unroll: bad arguments")
    return H


def head_gru_newton(px, U, h0=None, K=1, nthreads=None):
    """Returns (H^(K), resid) with resid[k] = max |F(H^(k))| for k = 0..K."""
    lib = _load()
    px, U, h0 = _f64(px), _f64(U), _f64(h0)
    B, T, D, nh = _head_shape(px, U)
    H = np.zeros((B, T, D))
    resid = np.zeros(K + 1)
    rc = lib.oracle_head_gru_newton(B, T, D, nh, _ptr(px), _ptr(U), _ptr(h0), K, _ptr(H), _ptr(resid),
                                    _threads(nthreads))
    if rc:
        raise ValueError("oracle_head_gru_newton: bad arguments")
    return H, resid


def head_gru_adjoint(px, U, H, dLdH, h0=None, nthreads=None):
    """Adjoint at trajectory H: returns (dL/dpx (B,T,3,D), dL/dU (3,n_heads,d,d), dL/dh0 (B,D))."""
    lib = _load()
    px, U, h0, H, g = _f64(px), _f64(U), _f64(h0), _f64(H), _f64(dLdH)
    B, T, D, nh = _head_shape(px, U)
    dpx = np.zeros((B, T, 3, D))
    dU = np.zeros(U.shape)
    dh0 = np.zeros((B, D))
    rc = lib.oracle_head_gru_adjoint(B, T, D, nh, _ptr(px), _ptr(U), _ptr(h0), _ptr(H), _ptr(g), _ptr(dpx), _ptr(dU),
                                     _ptr(dh0), _threads(nthreads))
    if rc:
        raise ValueError("oracle_head_gru_adjoint: bad arguments")
    return dpx, dU, dh0
