"""The forward's small-problem path: a channel group's tiles along T in one
thread-block cluster, carries passed through distributed shared memory, one
kernel launch per call.  Through the C ABI on the GPU:

* its results are bit-identical to the look-back path's on the same inputs
  (the hook PARARNN_HOOK_NO_CLUSTER forces the look-back path), and match the
  fp64 oracle;
* its status word, tagged with the call number, reports a non-finite output,
  and a later call of either path reports its own status only.
"""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import rel_err, to_np
from nonlinear_rnn_iteration_b200 import binding

pytestmark = pytest.mark.gpu
TOL_H = 1e-4
DEV = "cuda:0"
NO_CLUSTER = 2


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
    return dict(px=px_used, w=w, h0=hz, pxt=pxt, wt=t(w), h0t=t(hz))


def _both_paths(cell, x, K, resid=False, picard=0):
    outs = []
    for flags in (0, NO_CLUSTER):
        assert binding.pararnn_debug_hooks(0, flags) == binding.OK
        try:
            r = torch.zeros(K + 1, device=DEV) if resid else None
            H = binding.newton_forward(cell, x["pxt"], x["wt"], x["h0t"], K=K, resid_hist=r, picard_iters=picard)
            outs.append((H, r))
        finally:
            binding.pararnn_debug_hooks(0, 0)
    return outs


# (cell, B, T, D): T within 8 tiles along T (one cluster per channel group),
# several channel groups and batch rows, ragged T and D, one-tile clusters
CASES = [
    (oracle.DIAG_GRU, 1, 1024, 64),
    (oracle.DIAG_GRU, 3, 700, 100),
    (oracle.DIAG_GRU, 2, 37, 37),
    (oracle.DIAG_LSTM, 2, 560, 72),
    (oracle.DIAG_LSTM, 1, 200, 13),
    (oracle.LINEAR, 2, 1000, 136),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "cell%d_B%dT%dD%d" % c)
@pytest.mark.parametrize("h0", [False, True])
def test_cluster_path_matches_lookback_bitwise(case, h0, cuda_device):
    cell, B, T, D = case
    K = 3
    x = _inputs(cell, B, T, D, seed=T + D, h0=h0)
    (Hc, rc), (Hl, rl) = _both_paths(cell, x, K, resid=True)
    assert torch.equal(Hc, Hl)
    assert torch.equal(rc, rl)
    Ho, ro = oracle.newton(cell, x["px"], x["w"], x["h0"], K=K)
    assert rel_err(to_np(Hc), Ho) <= TOL_H
    r = to_np(rc)
    assert np.all(np.abs(r - ro) <= 1e-4 * max(1.0, ro[0]) + 1e-5 * ro), (r, ro)


@pytest.mark.parametrize("cell", [oracle.DIAG_GRU, oracle.DIAG_LSTM])
def test_cluster_path_bf16_and_picard(cell, cuda_device):
    x = _inputs(cell, 2, 500, 64, seed=5, bf16=True)
    (Hc, _), (Hl, _) = _both_paths(cell, x, 2)
    assert torch.equal(Hc, Hl)
    Ho, _ = oracle.newton(cell, x["px"], x["w"], None, K=2)
    assert rel_err(to_np(Hc), Ho) <= TOL_H
    x = _inputs(cell, 1, 400, 40, seed=6, h0=True)
    (Hc, _), (Hl, _) = _both_paths(cell, x, 2, picard=2)
    assert torch.equal(Hc, Hl)
    Ho, _ = oracle.newton_picard(cell, x["px"], x["w"], x["h0"], P=2, K=2)
    assert rel_err(to_np(Hc), Ho) <= TOL_H


def test_cluster_status_is_tagged_per_call(cuda_device):
    cell, B, T, D, K = oracle.DIAG_GRU, 1, 300, 64, 2
    x = _inputs(cell, B, T, D, seed=9)
    bad = x["pxt"].clone()
    bad[0, 17, 2, 5] = float("nan")
    ws = binding.workspace_for(cell, B, T, D, K, DEV)
    stream = torch.cuda.current_stream()
    H = torch.empty((B, T, 1, D), device=DEV)

    def run(px, flags):
        assert binding.pararnn_debug_hooks(0, flags) == binding.OK
        try:
            st = binding.pararnn_newton_forward(cell, B, T, D, binding.F32, px, x["wt"], None, K, H, ws, ws.numel(),
                                                None, stream)
            assert st == binding.OK, binding.pararnn_last_error()
            return binding.pararnn_status_sync(ws, stream)
        finally:
            binding.pararnn_debug_hooks(0, 0)

    assert run(bad, 0) == binding.ENONFINITE           # cluster path, NaN
    assert run(x["pxt"], 0) == binding.OK              # cluster path: the older flag is not this call's
    assert run(bad, NO_CLUSTER) == binding.ENONFINITE  # look-back path, NaN
    assert run(x["pxt"], 0) == binding.OK              # cluster path after a look-back call
    assert run(bad, 0) == binding.ENONFINITE
    assert run(x["pxt"], NO_CLUSTER) == binding.OK     # look-back path clears the header


def test_back_to_back_calls_read_the_previous_calls_output():
    # The cluster kernel is launched with programmatic dependent launch: a
    # call may be launched while the previous one runs, and must still see
    # everything it wrote.  Chain two calls with no host synchronisation,
    # the second reading the first's output as its pre-activations (H of the
    # first is written over the start of the second's px buffer), and
    # compare with the same calls separated by a synchronisation.
    cell, B, T, D, K = oracle.DIAG_GRU, 1, 1024, 64, 3
    x = _inputs(cell, B, T, D, seed=41)
    s = torch.cuda.current_stream()
    px2_ref = torch.from_numpy(_inputs(cell, B, T, D, seed=42)["px"]).to(DEV)
    H1 = binding.newton_forward(cell, x["pxt"], x["wt"], None, K=K)
    torch.cuda.synchronize()
    px2_ref.view(-1)[: B * T * D].copy_(H1.view(-1))
    torch.cuda.synchronize()
    ref = binding.newton_forward(cell, px2_ref, x["wt"], None, K=K)
    torch.cuda.synchronize()
    for rep in range(5):
        px2 = torch.from_numpy(_inputs(cell, B, T, D, seed=42)["px"]).to(DEV)
        torch.cuda.synchronize()
        H1_into_px2 = px2.view(-1)[: B * T * D].view(B, T, 1, D)
        # the first call writes straight into px2; the second reads px2
        binding.newton_forward(cell, x["pxt"], x["wt"], None, K=K, out=H1_into_px2, sync_status=False)
        H2 = binding.newton_forward(cell, px2, x["wt"], None, K=K, sync_status=False)
        torch.cuda.synchronize()
        assert torch.equal(px2, px2_ref), rep
        assert torch.equal(H2, ref), rep
