"""How many Newton iterations the GPU forward needs: K* against the unroll.

The pages' practical knob is the number of Newton iterations (``max_iters``):
the solve is exact after T iterations (the system is lower bidiagonal, so
each iteration makes at least one more step exact), and in practice far
fewer suffice.  Here K* is the smallest K for which the GPU forward matches
the fp64 sequential unroll (the oracle) within 1e-4, on the synthetic
diagonal GRU and LSTM cells (pre-activations ~ N(0,1), recurrent weights
~ U(-0.5, 0.5), h0 = 0), for sequence lengths from 16 to 4096.  The test
checks that K* exists well below T, that the error at K* + 1 is no larger,
that K = T gives the unroll for a short sequence, and that the residual
history the kernel reports falls with K.  Run with -s to print the table.
"""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import rel_err, to_np
from nonlinear_rnn_iteration_b200 import binding

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
TAU = 1e-4
K_MAX = 24


def _draw(cell, T, D, seed):
    rng = np.random.default_rng(seed)
    G = oracle.NUM_GATES[cell]
    px = rng.standard_normal((1, T, G, D)).astype(np.float32)
    w = rng.uniform(-0.5, 0.5, (G, D)).astype(np.float32)
    return px, w


def _errors(cell, px, w, ks):
    ref = oracle.unroll(cell, px, w)
    pxt, wt = torch.from_numpy(px).to(DEV), torch.from_numpy(w).to(DEV)
    return {k: rel_err(to_np(binding.newton_forward(cell, pxt, wt, None, K=k)), ref) for k in ks}


@pytest.mark.parametrize("cell", [oracle.DIAG_GRU, oracle.DIAG_LSTM], ids=["gru", "lstm"])
def test_kstar_against_unroll(cell, cuda_device):
    rows = []
    for T in (16, 64, 256, 1024, 4096):
        px, w = _draw(cell, T, 64, seed=100 + T)
        err = _errors(cell, px, w, range(1, K_MAX + 1))
        kstar = next((k for k in range(1, K_MAX + 1) if err[k] <= TAU), None)
        rows.append((T, kstar, err))
        assert kstar is not None, "no K <= %d reaches %g at T=%d: %s" % (K_MAX, TAU, T, err)
        assert kstar < T or T <= 16
        if kstar < K_MAX:
            assert err[kstar + 1] <= TAU
    name = "GRU" if cell == oracle.DIAG_GRU else "LSTM"
    print("\nK* (rel. error vs the fp64 unroll <= %g), %s, B=1, D=64" % (TAU, name))
    for T, kstar, err in rows:
        print("  T=%5d  K*=%2d   error at K=1,2,3,4: %s" % (T, kstar, ", ".join("%.1e" % err[k] for k in (1, 2, 3, 4))))
    # K* does not grow faster than the sequence length
    ks = [r[1] for r in rows]
    assert ks == sorted(ks) or max(ks) - min(ks) <= 4


KSTAR_GRID = (16, 64, 256, 1024, 4096, 16384, 65536, 131072, 262144)


@pytest.mark.parametrize("cell", [oracle.DIAG_GRU, oracle.DIAG_LSTM], ids=["gru", "lstm"])
def test_library_kstar_table_reaches_the_unroll(cell, cuda_device):
    """The table K = 0 reads (pararnn_kstar): on its own grid, with the draws
    it was measured on (256 channels, two seeds per length), the forward at
    K*(cell, T) matches the fp64 unroll within 1e-4, and K = 0 gives exactly
    that forward."""
    name = "GRU" if cell == oracle.DIAG_GRU else "LSTM"
    print("\nlibrary K*, %s, B=1, D=256: error at K*-1 and K*" % name)
    for T in KSTAR_GRID:
        ks = binding.pararnn_kstar(cell, T)
        for seed in (100 + T, 7 + T):
            px, w = _draw(cell, T, 256, seed)
            ref = oracle.unroll(cell, px, w)
            pxt, wt = torch.from_numpy(px).to(DEV), torch.from_numpy(w).to(DEV)
            H = binding.newton_forward(cell, pxt, wt, None, K=ks)
            assert torch.equal(H, binding.newton_forward(cell, pxt, wt, None, K=0))
            err = rel_err(to_np(H), ref)
            below = rel_err(to_np(binding.newton_forward(cell, pxt, wt, None, K=ks - 1)), ref)
            print("  T=%6d seed=%6d K*=%d  error %.1e at K*-1, %.1e at K*" % (T, seed, ks, below, err))
            assert err <= TAU, (T, seed, ks, err)


@pytest.mark.parametrize("cell", [oracle.DIAG_GRU, oracle.DIAG_LSTM], ids=["gru", "lstm"])
def test_k_equal_t_is_the_unroll(cell, cuda_device):
    T = 12
    px, w = _draw(cell, T, 40, seed=7)
    err = _errors(cell, px, w, [T])
    # exact up to float32 rounding (the error floor past K* is ~1e-5 on the
    # element-wise metric)
    assert err[T] <= 5e-5


@pytest.mark.parametrize("cell", [oracle.DIAG_GRU, oracle.DIAG_LSTM], ids=["gru", "lstm"])
def test_residual_history_falls(cell, cuda_device):
    px, w = _draw(cell, 2048, 64, seed=11)
    K = 8
    resid = torch.zeros(K + 1, device=DEV)
    binding.newton_forward(cell, torch.from_numpy(px).to(DEV), torch.from_numpy(w).to(DEV), None, K=K,
                           resid_hist=resid)
    r = resid.cpu().numpy()
    assert np.isfinite(r).all()
    # the residual of the warm start is O(1); Newton drives it down to rounding
    assert r[0] > 1e-2 and r[-1] < 1e-5 * r[0]
    for k in range(1, K + 1):
        assert r[k] <= r[k - 1] * 1.01 + 1e-6


def test_kstar_head_wise(cuda_device):
    """The same measurement for the head-wise GRU (dense 64 x 64 Jacobian
    blocks, the chunk products on tcgen05), with the workload's draw:
    pre-activations ~ N(0,1), U ~ U(-1,1)/sqrt(d), h0 = 0, two heads."""
    from nonlinear_rnn_iteration_b200 import workloads

    rows = []
    for T in (16, 64, 256, 1024):
        x = workloads.head_host_inputs(1, T, 128, 2, 200 + T)
        ref = oracle.head_gru_unroll(x["px"], x["U"], None)
        pxt, Ut = torch.from_numpy(x["px"]).to(DEV), torch.from_numpy(x["U"]).to(DEV)
        err = {k: rel_err(to_np(binding.head_gru_forward(pxt, Ut, None, K=k)), ref) for k in range(1, K_MAX + 1)}
        kstar = next((k for k in range(1, K_MAX + 1) if err[k] <= TAU), None)
        rows.append((T, kstar, err))
        assert kstar is not None, "no K <= %d reaches %g at T=%d: %s" % (K_MAX, TAU, T, err)
        assert kstar < T or T <= 16
        if kstar < K_MAX:
            assert err[kstar + 1] <= TAU
    print("\nK* (rel. error vs the fp64 unroll <= %g), head-wise GRU, B=1, D=128, 2 heads of 64" % TAU)
    for T, kstar, err in rows:
        print("  T=%5d  K*=%2d   error at K=1,2,3,4: %s" % (T, kstar, ", ".join("%.1e" % err[k] for k in (1, 2, 3, 4))))
