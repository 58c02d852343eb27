"""Pins for the fp64 oracle: checks against something other than itself.

Each ``pin_*`` function raises AssertionError on failure.  They are run by
``test_oracle_pins.py`` and, against mutated builds of the oracle source, by
``test_oracle_mutations.py``.

What pins what:

* cell step      -- torch.nn.GRUCell / LSTMCell configured as one channel of
                    the diagonal cell (library routine); linear: by hand.
* Jacobian       -- torch autograd of those torch cells w.r.t. the state.
* param grads    -- torch autograd w.r.t. the input (= pre-activations) and
                    the recurrent weights (= diagonal weights).
* unroll         -- torch cells stepped in a loop; linear: the explicit
                    closed-form sum h_t = sum_s (prod_{s<r<=t} a_r) b_s.
* Newton         -- a dense Newton step on the whole trajectory: torch
                    autograd Jacobian of F(H) and torch.linalg.solve, from the
                    warm start; plus the theorems that an affine cell is solved
                    exactly by one step (pararnn-torch PyPI page, News: the
                    RWKV-7 cell "needs 0", an exact scan) and that the
                    lower-bidiagonal system makes each step fix one more
                    prefix row; plus LSTM with zero weights exact in 2 steps.
* adjoint        -- dense implicit-function gradient (solve J^T lambda = g,
                    then -lambda^T dF/dtheta by autograd) at an unconverged
                    iterate; BPTT by torch autograd at the unroll; central
                    finite differences of <g, unroll(theta)>.
* Picard sweeps -- a plain loop over torch's cells from the warm start, a
                    dense Newton step from the swept guess, and the prefix
                    theorem (each sweep fixes one more leading row; T sweeps
                    give the unroll).
* residual       -- strictly decreasing over Newton steps on seeded cells of
                    every workload's cell (an empirical property, not a
                    theorem); max |F(H)| of an arbitrary trajectory against
                    the torch residual of the dense Newton pin, and zero at
                    the unroll.
"""
import numpy as np
import torch

import oracle
from nonlinear_rnn_iteration_b200 import workloads
from torch_cells import step_fn, step_fn_weights, unroll_channel

CELLS = (oracle.LINEAR, oracle.DIAG_GRU, oracle.DIAG_LSTM)


def _rng(seed):
    return np.random.default_rng(seed)


def _rand_inputs(cell, B, T, D, seed, h0=False, weights=True):
    rng = _rng(seed)
    G, S = oracle.NUM_GATES[cell], oracle.STATE_WIDTH[cell]
    px = rng.standard_normal((B, T, G, D))
    if cell == oracle.LINEAR:
        px[:, :, 0, :] = 1.0 / (1.0 + np.exp(-px[:, :, 0, :]))
        w = None
    else:
        w = rng.uniform(-0.5, 0.5, (G, D)) if weights else np.zeros((G, D))
    hz = rng.standard_normal((B, S, D)) * 0.5 if h0 else None
    return px, w, hz


def _close(a, b, tol, what):
    a, b = np.asarray(a, dtype=np.float64), np.asarray(b, dtype=np.float64)
    scale = max(1.0, float(np.max(np.abs(b))) if b.size else 1.0)
    err = float(np.max(np.abs(a - b))) if a.size else 0.0
    assert np.all(np.isfinite(a)), "%s: non-finite values" % what
    assert err <= tol * scale, "%s: max abs err %.3e > %.1e (scale %.3g)" % (what, err, tol, scale)


def _wcol(w, d, G):
    return np.zeros(G) if w is None else w[:, d]


def _h0col(h0, b, d, S):
    return np.zeros(S) if h0 is None else h0[b, :, d]


# --------------------------------------------------------------------------


def pin_cell_step():
    rng = _rng(1)
    for cell in CELLS:
        G, S = oracle.NUM_GATES[cell], oracle.STATE_WIDTH[cell]
        for _ in range(25):
            p = rng.standard_normal(G) * 2.0
            a = rng.uniform(-1.0, 1.0, G) if cell else np.zeros(G)
            s = rng.standard_normal(S)
            ref = step_fn(cell, a)(torch.tensor(s), torch.tensor(p)).detach().numpy()
            _close(oracle.cell_step(cell, p, a, s), ref, 1e-14, "cell %d step" % cell)


def pin_jacobian():
    rng = _rng(2)
    for cell in CELLS:
        G, S = oracle.NUM_GATES[cell], oracle.STATE_WIDTH[cell]
        for _ in range(25):
            p = rng.standard_normal(G) * 2.0
            a = rng.uniform(-1.0, 1.0, G) if cell else np.zeros(G)
            s = rng.standard_normal(S)
            f = step_fn(cell, a)
            J = torch.autograd.functional.jacobian(lambda x: f(x, torch.tensor(p)), torch.tensor(s))
            _close(oracle.cell_jacobian(cell, p, a, s), J.numpy().reshape(S, S), 1e-12,
                   "cell %d Jacobian" % cell)


def pin_param_grads():
    rng = _rng(3)
    for cell in CELLS:
        G, S = oracle.NUM_GATES[cell], oracle.STATE_WIDTH[cell]
        fw = step_fn_weights(cell)
        for _ in range(25):
            p = rng.standard_normal(G) * 2.0
            a = rng.uniform(-1.0, 1.0, G) if cell else np.zeros(G)
            s = rng.standard_normal(S)
            Jp, Ja = torch.autograd.functional.jacobian(
                lambda pp, aa: fw(torch.tensor(s), pp, aa), (torch.tensor(p), torch.tensor(a)))
            dp, da = oracle.cell_param_grads(cell, p, a, s)
            _close(dp, Jp.numpy().reshape(S, G), 1e-12, "cell %d d/dp" % cell)
            _close(da, Ja.numpy().reshape(S, G), 1e-12, "cell %d d/da" % cell)


def pin_unroll():
    for cell in CELLS:
        B, T, D = 2, 40, 3
        px, w, h0 = _rand_inputs(cell, B, T, D, seed=10 + cell, h0=True)
        H = oracle.unroll(cell, px, w, h0, nthreads=3)
        S, G = oracle.STATE_WIDTH[cell], oracle.NUM_GATES[cell]
        for b in range(B):
            for d in range(D):
                ref = unroll_channel(cell, px[b, :, :, d], _wcol(w, d, G), _h0col(h0, b, d, S))
                _close(H[b, :, :, d], ref, 1e-13, "cell %d unroll" % cell)
    # linear: explicit closed form, no recurrence
    px, _, h0 = _rand_inputs(oracle.LINEAR, 1, 30, 2, seed=19, h0=True)
    H = oracle.unroll(oracle.LINEAR, px, None, h0)
    for d in range(2):
        a, bb = px[0, :, 0, d], px[0, :, 1, d]
        for t in range(30):
            ref = np.prod(a[: t + 1]) * h0[0, 0, d]
            for s in range(t + 1):
                ref += np.prod(a[s + 1: t + 1]) * bb[s]
            _close(H[0, t, 0, d], ref, 1e-13, "linear closed form")


def _dense_F(cell, p, a, h0):
    """F(H) = H_t - f(H_{t-1}, x_t) of one channel, with torch cells."""
    T, _ = p.shape
    S = oracle.STATE_WIDTH[cell]
    fw = step_fn_weights(cell)

    def F(Hflat, pp, aa, hh0):
        Hm = Hflat.reshape(T, S)
        prev, outs = hh0, []
        for t in range(T):
            outs.append(Hm[t] - fw(prev, pp[t], aa))
            prev = Hm[t]
        return torch.cat(outs)
    return F


def pin_newton_dense():
    for cell in CELLS:
        T, G, S = 12, oracle.NUM_GATES[cell], oracle.STATE_WIDTH[cell]
        for h0flag in (False, True):
            px, w, h0 = _rand_inputs(cell, 1, T, 1, seed=30 + cell + 5 * h0flag, h0=h0flag)
            p = torch.tensor(px[0, :, :, 0])
            a = torch.tensor(_wcol(w, 0, G))
            hh0 = torch.tensor(_h0col(h0, 0, 0, S))
            F = _dense_F(cell, p, a, hh0)
            f0 = step_fn_weights(cell)
            H = torch.stack([f0(torch.zeros(S, dtype=torch.float64), p[t], a) for t in range(T)]).reshape(-1)
            res = [float(F(H, p, a, hh0).abs().max())]
            for k in range(1, 4):
                J = torch.autograd.functional.jacobian(lambda x: F(x, p, a, hh0), H)
                H = H + torch.linalg.solve(J, -F(H, p, a, hh0))
                res.append(float(F(H, p, a, hh0).abs().max()))
                Ho, ro = oracle.newton(cell, px, w, h0, K=k)
                _close(Ho[0, :, :, 0], H.detach().numpy().reshape(T, S), 1e-12,
                       "cell %d Newton k=%d vs dense" % (cell, k))
                _close(ro, res, 1e-12, "cell %d residual history k=%d" % (cell, k))


def pin_residual_function():
    # max |F(H)| of an arbitrary trajectory (not a Newton iterate) against the
    # torch residual F(H)_t = H_t - f(H_{t-1}, x_t) built from torch's cells;
    # several channels and batch rows, so a max over the wrong axis fails too
    for cell in CELLS:
        B, T, D, G, S = 2, 9, 3, oracle.NUM_GATES[cell], oracle.STATE_WIDTH[cell]
        for h0flag in (False, True):
            px, w, h0 = _rand_inputs(cell, B, T, D, seed=60 + cell + 3 * h0flag, h0=h0flag)
            H = _rng(70 + cell).standard_normal((B, T, S, D)) * 0.7
            ref = 0.0
            for b in range(B):
                for d in range(D):
                    p = torch.tensor(px[b, :, :, d])
                    a = torch.tensor(_wcol(w, d, G))
                    hh0 = torch.tensor(_h0col(h0, b, d, S))
                    F = _dense_F(cell, p, a, hh0)
                    ref = max(ref, float(F(torch.tensor(H[b, :, :, d]).reshape(-1), p, a, hh0).abs().max()))
            _close(oracle.residual(cell, px, w, h0, H, nthreads=2), ref, 1e-13, "cell %d residual of H" % cell)
        # the unroll solves F(H) = 0
        U = oracle.unroll(cell, px, w, h0)
        assert oracle.residual(cell, px, w, h0, U) < 1e-14, "cell %d residual of the unroll" % cell


def pin_affine_one_step():
    # linear cell, any K >= 1
    px, _, h0 = _rand_inputs(oracle.LINEAR, 2, 64, 3, seed=40, h0=True)
    U = oracle.unroll(oracle.LINEAR, px, None, h0)
    for K in (1, 2):
        Hn, _ = oracle.newton(oracle.LINEAR, px, None, h0, K=K)
        _close(Hn, U, 1e-13, "linear Newton K=%d" % K)
    # GRU with zero recurrent weights: h' = (1-z) h + z c is affine in h
    px, w, h0 = _rand_inputs(oracle.DIAG_GRU, 2, 64, 3, seed=41, h0=True, weights=False)
    U = oracle.unroll(oracle.DIAG_GRU, px, w, h0)
    Hn, res = oracle.newton(oracle.DIAG_GRU, px, w, h0, K=1)
    _close(Hn, U, 1e-13, "GRU a=0 Newton K=1")
    assert res[1] < 1e-13 and res[0] > 1e-3, "GRU a=0 residuals %s" % res


def pin_prefix_exact():
    for cell in CELLS:
        T = 8
        for h0flag in (False, True):
            px, w, h0 = _rand_inputs(cell, 1, T, 2, seed=50 + cell + 7 * h0flag, h0=h0flag)
            U = oracle.unroll(cell, px, w, h0)
            for k in range(0, T + 1):
                Hn, _ = oracle.newton(cell, px, w, h0, K=k)
                exact_rows = k + 1 if not h0flag else k  # warm start is exact at t=0 when h0 = 0
                n = min(exact_rows, T)
                if n:
                    _close(Hn[:, :n], U[:, :n], 1e-12, "cell %d prefix after %d steps" % (cell, k))
                if k >= T:
                    _close(Hn, U, 1e-12, "cell %d after T steps" % cell)


def pin_picard_torch_loop():
    # P Picard sweeps from the warm start written as a plain loop over torch's
    # cells, then one dense Newton step (autograd Jacobian, linear solve) from
    # there: the oracle's sweeps and its Newton step from the swept guess
    for cell in CELLS:
        T, G, S = 10, oracle.NUM_GATES[cell], oracle.STATE_WIDTH[cell]
        for h0flag in (False, True):
            px, w, h0 = _rand_inputs(cell, 2, T, 2, seed=80 + cell + 5 * h0flag, h0=h0flag)
            for P in (1, 2, 3):
                Hp, _ = oracle.newton_picard(cell, px, w, h0, P=P, K=0)
                H1, r1 = oracle.newton_picard(cell, px, w, h0, P=P, K=1)
                for b in range(2):
                    for d in range(2):
                        p = torch.tensor(px[b, :, :, d])
                        a = torch.tensor(_wcol(w, d, G))
                        hh0 = torch.tensor(_h0col(h0, b, d, S))
                        f = step_fn_weights(cell)
                        X = [f(torch.zeros(S, dtype=torch.float64), p[t], a) for t in range(T)]
                        for _ in range(P):
                            X = [f(hh0 if t == 0 else X[t - 1], p[t], a) for t in range(T)]
                        Xs = torch.stack(X)
                        _close(Hp[b, :, :, d], Xs.numpy(), 1e-13, "cell %d Picard P=%d" % (cell, P))
                        F = _dense_F(cell, p, a, hh0)
                        Hf = Xs.reshape(-1)
                        J = torch.autograd.functional.jacobian(lambda x: F(x, p, a, hh0), Hf)
                        Hn = Hf + torch.linalg.solve(J, -F(Hf, p, a, hh0))
                        _close(H1[b, :, :, d], Hn.detach().numpy().reshape(T, S), 1e-12,
                               "cell %d Picard P=%d + Newton" % (cell, P))


def pin_picard_prefix_exact():
    # sweep p makes one more leading row exact: with h0 = 0 the warm start is
    # already exact at t = 0, so P sweeps fix rows 0..P, and K Newton steps
    # after them rows 0..P+K; P >= T sweeps alone give the unroll
    for cell in CELLS:
        T = 8
        for h0flag in (False, True):
            px, w, h0 = _rand_inputs(cell, 1, T, 2, seed=90 + cell + 7 * h0flag, h0=h0flag)
            U = oracle.unroll(cell, px, w, h0)
            for P in range(0, T + 1):
                for K in (0, 1, 2):
                    Hn, _ = oracle.newton_picard(cell, px, w, h0, P=P, K=K)
                    n = min(T, P + K + (0 if h0flag else 1))
                    if n:
                        _close(Hn[:, :n], U[:, :n], 1e-12, "cell %d P=%d K=%d prefix" % (cell, P, K))
                    if cell != oracle.LINEAR and n < T and K == 0:
                        # the next row is not exact yet (a missing sweep would pass the check above)
                        assert np.max(np.abs(Hn[:, n] - U[:, n])) > 1e-9, "cell %d P=%d row %d" % (cell, P, n)
                if P >= T:
                    _close(oracle.newton_picard(cell, px, w, h0, P=P, K=0)[0], U, 1e-12, "cell %d P=T" % cell)


def pin_lstm_zero_weights():
    px, w, h0 = _rand_inputs(oracle.DIAG_LSTM, 2, 48, 3, seed=60, h0=True, weights=False)
    U = oracle.unroll(oracle.DIAG_LSTM, px, w, h0)
    H1, _ = oracle.newton(oracle.DIAG_LSTM, px, w, h0, K=1)
    H2, _ = oracle.newton(oracle.DIAG_LSTM, px, w, h0, K=2)
    _close(H1[:, :, 0], U[:, :, 0], 1e-13, "LSTM a=0: c exact after 1 step")
    assert np.max(np.abs(H1[:, :, 1] - U[:, :, 1])) > 1e-6, "LSTM a=0: h should not be exact after 1 step"
    _close(H2, U, 1e-13, "LSTM a=0: exact after 2 steps")


def pin_adjoint_dense():
    for cell in CELLS:
        T, G, S = 10, oracle.NUM_GATES[cell], oracle.STATE_WIDTH[cell]
        px, w, h0 = _rand_inputs(cell, 1, T, 1, seed=70 + cell, h0=True)
        g = _rng(71 + cell).standard_normal((1, T, S, 1))
        H, _ = oracle.newton(cell, px, w, h0, K=1)  # unconverged iterate
        p = torch.tensor(px[0, :, :, 0], requires_grad=True)
        a = torch.tensor(_wcol(w, 0, G), requires_grad=True)
        hh0 = torch.tensor(_h0col(h0, 0, 0, S), requires_grad=True)
        F = _dense_F(cell, p, a, hh0)
        Hf = torch.tensor(H[0, :, :, 0].reshape(-1))
        J = torch.autograd.functional.jacobian(lambda x: F(x, p.detach(), a.detach(), hh0.detach()), Hf)
        lam = torch.linalg.solve(J.T, torch.tensor(g[0, :, :, 0].reshape(-1)))
        Fv = F(Hf, p, a, hh0)
        gp, ga, gh = torch.autograd.grad(Fv, (p, a, hh0), grad_outputs=-lam, allow_unused=True)
        dpx, da, dh0 = oracle.adjoint(cell, px, w, h0, H, g)
        _close(dpx[0, :, :, 0], gp.numpy(), 1e-11, "cell %d adjoint dL/dpx (dense)" % cell)
        if cell != oracle.LINEAR:
            _close(da[:, 0], ga.numpy(), 1e-11, "cell %d adjoint dL/da (dense)" % cell)
        _close(dh0[0, :, 0], gh.numpy(), 1e-11, "cell %d adjoint dL/dh0 (dense)" % cell)


def pin_adjoint_bptt():
    for cell in CELLS:
        T, G, S = 16, oracle.NUM_GATES[cell], oracle.STATE_WIDTH[cell]
        px, w, h0 = _rand_inputs(cell, 1, T, 1, seed=80 + cell, h0=True)
        g = _rng(81 + cell).standard_normal((1, T, S, 1))
        p = torch.tensor(px[0, :, :, 0], requires_grad=True)
        a = torch.tensor(_wcol(w, 0, G), requires_grad=True)
        s = torch.tensor(_h0col(h0, 0, 0, S), requires_grad=True)
        fw = step_fn_weights(cell)
        L, st = 0.0, s
        for t in range(T):
            st = fw(st, p[t], a)
            L = L + (st * torch.tensor(g[0, t, :, 0])).sum()
        gp, ga, gh = torch.autograd.grad(L, (p, a, s), allow_unused=True)
        U = oracle.unroll(cell, px, w, h0)
        dpx, da, dh0 = oracle.adjoint(cell, px, w, h0, U, g)
        _close(dpx[0, :, :, 0], gp.numpy(), 1e-11, "cell %d BPTT dL/dpx" % cell)
        if cell != oracle.LINEAR:
            _close(da[:, 0], ga.numpy(), 1e-11, "cell %d BPTT dL/da" % cell)
        _close(dh0[0, :, 0], gh.numpy(), 1e-11, "cell %d BPTT dL/dh0" % cell)


def pin_adjoint_fd():
    eps = 1e-6
    for cell in CELLS:
        B, T, D = 1, 6, 2
        px, w, h0 = _rand_inputs(cell, B, T, D, seed=90 + cell, h0=True)
        S = oracle.STATE_WIDTH[cell]
        g = _rng(91 + cell).standard_normal((B, T, S, D))

        def L(px_, w_, h0_):
            return float(np.sum(g * oracle.unroll(cell, px_, w_, h0_)))
        U = oracle.unroll(cell, px, w, h0)
        dpx, da, dh0 = oracle.adjoint(cell, px, w, h0, U, g)
        for idx in np.ndindex(px.shape):
            pp, pm = px.copy(), px.copy()
            pp[idx] += eps
            pm[idx] -= eps
            fd = (L(pp, w, h0) - L(pm, w, h0)) / (2 * eps)
            assert abs(fd - dpx[idx]) < 1e-7 * max(1.0, abs(fd)), "cell %d FD dL/dpx%s" % (cell, idx)
        if w is not None:
            for idx in np.ndindex(w.shape):
                wp, wm = w.copy(), w.copy()
                wp[idx] += eps
                wm[idx] -= eps
                fd = (L(px, wp, h0) - L(px, wm, h0)) / (2 * eps)
                assert abs(fd - da[idx]) < 1e-7 * max(1.0, abs(fd)), "cell %d FD dL/da%s" % (cell, idx)
        for idx in np.ndindex(h0.shape):
            hp, hm = h0.copy(), h0.copy()
            hp[idx] += eps
            hm[idx] -= eps
            fd = (L(px, w, hp) - L(px, w, hm)) / (2 * eps)
            assert abs(fd - dh0[idx]) < 1e-7 * max(1.0, abs(fd)), "cell %d FD dL/dh0%s" % (cell, idx)


def pin_residual_monotone():
    # every nonlinear workload's cell and Newton budget, at a shape the oracle runs in well under a second
    for name in ("gru_1x1024x64_k3", "gru_8x4096x2048_k3", "lstm_4x32768x1024_k4", "gru_1x131072x4096_k2_bf16"):
        w = workloads.WORKLOADS[name]
        small = w.with_shape(B=1, T=min(w.T, 2048), D=16)
        x = workloads.host_inputs(small)
        _, res = oracle.newton(small.cell_id, x["px"], x["a"], None, K=w.K)
        assert all(res[k + 1] < res[k] for k in range(w.K)), "%s residuals not decreasing: %s" % (name, res)


# ---- head-wise GRU (block-diagonal recurrent weights) ----------------------
# One head of width d is torch.nn.GRUCell(3d, d) with
#   x = (p_z, p_r, p_c), all biases 0,
#   weight_ih row blocks (r | z | n) = ([0 I 0] | [-I 0 0] | [0 0 I]),
#   weight_hh row blocks (r | z | n) = (U_r | -U_z | U_c):
# negating the z pre-activation turns torch's kept-state weight into our
# (1 - z), and torch's candidate tanh(W_in x + r * (W_hn h)) is our
# c = tanh(p_c + r * (U_c h)).


def _torch_head_cell(U):
    d = U.shape[-1]
    cell = torch.nn.GRUCell(3 * d, d, bias=True).double()
    I, Z = np.eye(d), np.zeros((d, d))
    w_ih = np.block([[Z, I, Z], [-I, Z, Z], [Z, Z, I]])
    w_hh = np.concatenate([U[1], -U[0], U[2]], axis=0)
    with torch.no_grad():
        cell.weight_ih.copy_(torch.tensor(w_ih))
        cell.weight_hh.copy_(torch.tensor(w_hh))
        cell.bias_ih.zero_()
        cell.bias_hh.zero_()
    return cell


def _head_inputs(B, T, nh, d, seed, h0=False):
    rng = _rng(seed)
    D = nh * d
    px = rng.standard_normal((B, T, 3, D))
    U = rng.uniform(-1.0, 1.0, (3, nh, d, d)) / np.sqrt(d)
    hz = rng.standard_normal((B, D)) * 0.5 if h0 else None
    return px, U, hz


def _torch_head_unroll(px, U, h0):
    B, T, _, D = px.shape
    nh, d = U.shape[1], U.shape[2]
    out = np.zeros((B, T, D))
    for h in range(nh):
        cell = _torch_head_cell(U[:, h])
        sl = slice(h * d, (h + 1) * d)
        s = torch.zeros(B, d, dtype=torch.float64) if h0 is None else torch.tensor(h0[:, sl])
        for t in range(T):
            x = torch.tensor(px[:, t, :, sl].reshape(B, 3 * d))
            s = cell(x, s)
            out[:, t, sl] = s.detach().numpy()
    return out


def pin_head_step_and_jacobian():
    rng = _rng(31)
    for d in (1, 3, 8):
        for _ in range(10):
            p = rng.standard_normal((3, d)) * 2.0
            U = rng.uniform(-1.0, 1.0, (3, d, d))
            s = rng.standard_normal(d)
            cell = _torch_head_cell(U)
            f = lambda x: cell(torch.tensor(p.reshape(1, 3 * d)), x.reshape(1, d)).reshape(d)
            _close(oracle.head_gru_step(p, U, s), f(torch.tensor(s)).detach().numpy(), 1e-14, "head step d=%d" % d)
            J = torch.autograd.functional.jacobian(f, torch.tensor(s)).numpy()
            _close(oracle.head_gru_jacobian(p, U, s), J, 1e-12, "head Jacobian d=%d" % d)


def pin_head_unroll():
    for h0 in (False, True):
        px, U, hz = _head_inputs(2, 9, 3, 4, seed=32, h0=h0)
        _close(oracle.head_gru_unroll(px, U, hz), _torch_head_unroll(px, U, hz), 1e-13, "head unroll h0=%s" % h0)


def pin_head_newton_dense():
    # dense Newton on the whole trajectory: F(X)_t = X_t - f(X_{t-1}, x_t),
    # Jacobian by autograd, each step by torch.linalg.solve; heads at once
    B, T, nh, d = 1, 5, 2, 3
    D = nh * d
    for h0 in (False, True):
        px, U, hz = _head_inputs(B, T, nh, d, seed=33, h0=h0)
        cells = [_torch_head_cell(U[:, h]) for h in range(nh)]
        s0 = torch.zeros(D, dtype=torch.float64) if hz is None else torch.tensor(hz[0])

        def f_all(prev, t):
            outs = []
            for h in range(nh):
                sl = slice(h * d, (h + 1) * d)
                x = torch.tensor(px[0, t, :, sl].reshape(1, 3 * d))
                outs.append(cells[h](x, prev[sl].reshape(1, d)).reshape(d))
            return torch.cat(outs)

        def F(Xflat):
            X = Xflat.reshape(T, D)
            rows, prev = [], s0
            for t in range(T):
                rows.append(X[t] - f_all(prev, t))
                prev = X[t]
            return torch.cat(rows)

        X = torch.cat([f_all(torch.zeros(D, dtype=torch.float64), t) for t in range(T)])  # warm start
        for k in range(1, 4):
            J = torch.autograd.functional.jacobian(F, X)
            X = X - torch.linalg.solve(J, F(X))
            H, resid = oracle.head_gru_newton(px, U, hz, K=k)
            _close(H[0], X.detach().numpy().reshape(T, D), 1e-11, "head Newton k=%d h0=%s" % (k, h0))
            _close(resid[k], float(torch.max(torch.abs(F(X)))), 1e-11, "head residual k=%d" % k)


def pin_head_prefix_exact_and_diagonal():
    # Newton on the lower block-bidiagonal system makes the first k rows exact
    # after k steps and everything exact after T steps
    px, U, hz = _head_inputs(1, 8, 2, 3, seed=34, h0=True)
    ref = _torch_head_unroll(px, U, hz)
    for k in (1, 3, 5):
        H, _ = oracle.head_gru_newton(px, U, hz, K=k)
        _close(H[:, :k], ref[:, :k], 1e-12, "head prefix exact k=%d" % k)
        if k == 1:  # not vacuous: one step leaves the later rows inexact
            assert np.max(np.abs(H[:, k:] - ref[:, k:])) > 1e-6, "head Newton exact everywhere after one step"
    H, _ = oracle.head_gru_newton(px, U, hz, K=8)
    _close(H, ref, 1e-12, "head exact after T steps")
    # diagonal blocks: the diagonal GRU, computed by its own code path
    rng = _rng(35)
    B, T, nh, d = 2, 20, 2, 3
    D = nh * d
    px = rng.standard_normal((B, T, 3, D))
    a = rng.uniform(-0.5, 0.5, (3, D))
    U = np.zeros((3, nh, d, d))
    for g in range(3):
        for h in range(nh):
            U[g, h] = np.diag(a[g, h * d:(h + 1) * d])
    Hh, rh = oracle.head_gru_newton(px, U, K=3)
    Hd, rd = oracle.newton(oracle.DIAG_GRU, px, a, K=3)
    _close(Hh, Hd[:, :, 0, :], 1e-13, "head with diagonal blocks vs the diagonal GRU")
    _close(rh, rd, 1e-13, "head vs diagonal residual history")


def _torch_head_unroll_t(px_t, U_t, h0_t, d):
    """The head-wise unroll on torch tensors (differentiable in px, U, h0)."""
    B, T, _, D = px_t.shape
    nh = U_t.shape[1]
    outs = []
    for h in range(nh):
        sl = slice(h * d, (h + 1) * d)
        I, Z = torch.eye(d, dtype=torch.float64), torch.zeros((d, d), dtype=torch.float64)
        w_ih = torch.cat([torch.cat([Z, I, Z], 1), torch.cat([-I, Z, Z], 1), torch.cat([Z, Z, I], 1)], 0)
        w_hh = torch.cat([U_t[1, h], -U_t[0, h], U_t[2, h]], 0)
        zb = torch.zeros(3 * d, dtype=torch.float64)
        s = h0_t[:, sl]
        seq = []
        for t in range(T):
            s = torch._VF.gru_cell(px_t[:, t, :, sl].reshape(B, 3 * d), s, w_ih, w_hh, zb, zb)
            seq.append(s)
        outs.append(torch.stack(seq, 1))
    return torch.cat(outs, 2)


def pin_head_adjoint_bptt():
    # at the unroll the adjoint is back-propagation through time
    B, T, nh, d = 2, 7, 2, 3
    px, U, hz = _head_inputs(B, T, nh, d, seed=36, h0=True)
    g = _rng(37).standard_normal((B, T, nh * d))
    px_t, U_t, h0_t = (torch.tensor(a, requires_grad=True) for a in (px, U, hz))
    Ht = _torch_head_unroll_t(px_t, U_t, h0_t, d)
    (Ht * torch.tensor(g)).sum().backward()
    dpx, dU, dh0 = oracle.head_gru_adjoint(px, U, Ht.detach().numpy(), g, hz)
    _close(dpx, px_t.grad.numpy(), 1e-12, "head adjoint dL/dpx vs BPTT")
    _close(dU, U_t.grad.numpy(), 1e-12, "head adjoint dL/dU vs BPTT")
    _close(dh0, h0_t.grad.numpy(), 1e-12, "head adjoint dL/dh0 vs BPTT")


def pin_head_adjoint_dense():
    # at an unconverged iterate: the implicit gradient of F(H) = 0, solved
    # densely -- lambda = J^T \ g, dL/dtheta = -(dF/dtheta)^T lambda
    B, T, nh, d = 1, 5, 2, 2
    D = nh * d
    px, U, hz = _head_inputs(B, T, nh, d, seed=38, h0=True)
    H, _ = oracle.head_gru_newton(px, U, hz, K=1)
    g = _rng(39).standard_normal((B, T, D))

    def F(Hf, pxf, Uf, h0f):
        Hm = Hf.reshape(B, T, D)
        prev = torch.cat([h0f.reshape(B, 1, D), Hm[:, :-1]], 1)
        rows = []
        for t in range(T):
            f_t = _torch_head_unroll_t(pxf[:, t:t + 1], Uf, prev[:, t], d)[:, 0]
            rows.append(Hm[:, t] - f_t)
        return torch.stack(rows, 1).reshape(-1)

    args = tuple(torch.tensor(a) for a in (H, px, U, hz))
    J = torch.autograd.functional.jacobian(F, args)
    lam = torch.linalg.solve(J[0].reshape(B * T * D, B * T * D).T, torch.tensor(g).reshape(-1))
    grads = [-(Jk.reshape(B * T * D, -1).T @ lam).reshape(a.shape) for Jk, a in zip(J[1:], args[1:])]
    dpx, dU, dh0 = oracle.head_gru_adjoint(px, U, H, g, hz)
    _close(dpx, grads[0].numpy(), 1e-11, "head adjoint dL/dpx vs implicit gradient")
    _close(dU, grads[1].numpy(), 1e-11, "head adjoint dL/dU vs implicit gradient")
    _close(dh0, grads[2].numpy(), 1e-11, "head adjoint dL/dh0 vs implicit gradient")


def pin_head_adjoint_diagonal():
    # diagonal blocks: the diagonal GRU's adjoint (its own code path); dL/dU's
    # diagonal is the diagonal cell's dL/da
    rng = _rng(40)
    B, T, nh, d = 2, 15, 2, 3
    D = nh * d
    px = rng.standard_normal((B, T, 3, D))
    a = rng.uniform(-0.5, 0.5, (3, D))
    U = np.zeros((3, nh, d, d))
    for gi in range(3):
        for h in range(nh):
            U[gi, h] = np.diag(a[gi, h * d:(h + 1) * d])
    H, _ = oracle.newton(oracle.DIAG_GRU, px, a, K=2)
    g = rng.standard_normal((B, T, 1, D))
    dpx_d, da_d, dh0_d = oracle.adjoint(oracle.DIAG_GRU, px, a, None, H, g)
    dpx, dU, dh0 = oracle.head_gru_adjoint(px, U, H[:, :, 0, :], g[:, :, 0, :])
    _close(dpx, dpx_d, 1e-13, "head adjoint vs diagonal dL/dpx")
    diag = np.stack([np.concatenate([np.diag(dU[gi, h]) for h in range(nh)]) for gi in range(3)])
    _close(diag, da_d, 1e-13, "head adjoint dL/dU diagonal vs diagonal dL/da")
    _close(dh0, dh0_d[:, 0, :], 1e-13, "head adjoint vs diagonal dL/dh0")


ALL_PINS = [pin_cell_step, pin_jacobian, pin_param_grads, pin_unroll, pin_newton_dense, pin_affine_one_step,
            pin_prefix_exact, pin_picard_torch_loop, pin_picard_prefix_exact, pin_lstm_zero_weights, pin_adjoint_dense, pin_adjoint_bptt, pin_adjoint_fd,
            pin_residual_monotone, pin_residual_function, pin_head_step_and_jacobian, pin_head_unroll, pin_head_newton_dense,
            pin_head_prefix_exact_and_diagonal, pin_head_adjoint_bptt, pin_head_adjoint_dense,
            pin_head_adjoint_diagonal]
