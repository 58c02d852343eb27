"""The workspace contract and the bounded waits, on the GPU, through the C ABI.

* Every call clears, on its stream, the look-back words it reads, so a
  workspace holding words left by another call -- even words tagged with the
  very number the next call will use -- gives the oracle's answer.
* The time-out path of the real look-back: with the stall hook the first tile
  of the scan never publishes its carry, the next tile's bounded wait runs out
  after a 20 ms limit, the call reports PARARNN_ETIMEOUT and returns quickly,
  and an ordinary call on the same workspace afterwards is correct again.
"""
import time

import numpy as np
import pytest
import torch

import oracle
from gpu_util import rel_err, to_np
from nonlinear_rnn_iteration_b200 import binding

pytestmark = pytest.mark.gpu
TOL_H, TOL_G = 1e-4, 1e-3
DEV = "cuda:0"
HEADER_WORDS = 256 // 8  # the first tile's status word follows the 256-byte header
NO_CLUSTER = 2           # PARARNN_HOOK_NO_CLUSTER


def _inputs(cell, B, T, D, seed):
    rng = np.random.default_rng(seed)
    G, S = oracle.NUM_GATES[cell], oracle.STATE_WIDTH[cell]
    px = rng.standard_normal((B, T, G, D)).astype(np.float32)
    if cell == oracle.LINEAR:
        px[:, :, 0, :] = 1.0 / (1.0 + np.exp(-px[:, :, 0, :]))
        w = None
    else:
        w = rng.uniform(-0.5, 0.5, (G, D)).astype(np.float32)
    g = rng.standard_normal((B, T, S, D)).astype(np.float32)
    t = lambda a: None if a is None else torch.from_numpy(np.ascontiguousarray(a)).to(DEV)
    return dict(px=px, w=w, g=g, pxt=t(px), wt=t(w), gt=t(g))


def _tag(words, i):
    return int(words[i].item()) >> 32


def _retag(ws, old, new):
    """Rewrite every 64-bit word tagged `old` so that it carries `new`: the
    words of one call made to look like the next call's own."""
    words = ws.view(torch.int64)
    hit = ((words >> 32) & 0xFFFFFFFF) == old
    low = words & 0xFFFFFFFF
    words.copy_(torch.where(hit, low | (new << 32), words))
    return int(hit.sum().item())


@pytest.fixture
def lookback_path():
    # these tests plant look-back words, so the forward must take the
    # look-back path even where the problem would fit the cluster path
    assert binding.pararnn_debug_hooks(0, NO_CLUSTER) == binding.OK
    yield
    binding.pararnn_debug_hooks(0, 0)


@pytest.mark.parametrize("cell", [oracle.LINEAR, oracle.DIAG_GRU, oracle.DIAG_LSTM])
def test_stale_lookback_words_with_live_tags(cell, cuda_device, lookback_path):
    # one workspace, large enough for both shapes, never zero-filled
    shapes = [(2, 1500, 160, 3), (1, 2300, 96, 2)]
    n = max(binding.pararnn_workspace_bytes(cell, B, T, D, K) for B, T, D, K in shapes)
    ws = torch.empty(n, dtype=torch.uint8, device=DEV)
    ws.fill_(0xA5)
    words = ws.view(torch.int64)
    # call A fills the look-back words of its shape
    B, T, D, K = shapes[0]
    xa = _inputs(cell, B, T, D, seed=1)
    binding.newton_forward(cell, xa["pxt"], xa["wt"], None, K=K, workspace=ws)
    ea = _tag(words, HEADER_WORDS)
    assert ea != 0
    # make A's words look like call B's (the next call on this thread takes
    # the next number), then run B of another shape over them
    assert _retag(ws, ea, ea + 1) > 100
    B, T, D, K = shapes[1]
    xb = _inputs(cell, B, T, D, seed=2)
    H = binding.newton_forward(cell, xb["pxt"], xb["wt"], None, K=K, workspace=ws)
    assert _tag(words, HEADER_WORDS) == ea + 1  # B did run under the planted tag
    Ho, _ = oracle.newton(cell, xb["px"], xb["w"], None, K=K)
    assert rel_err(to_np(H), Ho) <= TOL_H
    # the backward over the forward's retagged words
    assert _retag(ws, ea + 1, ea + 2) > 100
    dpx, da, _ = binding.newton_backward(cell, xb["pxt"], H, xb["gt"], xb["wt"], workspace=ws)
    assert _tag(words, HEADER_WORDS) == ea + 2
    dpxo, dao, _ = oracle.adjoint(cell, xb["px"], xb["w"], None, Ho, xb["g"])
    assert rel_err(to_np(dpx), dpxo) <= TOL_G
    if da is not None:
        assert rel_err(to_np(da), dao) <= TOL_G


def test_uniform_fill_that_reads_as_published_carries(cuda_device, lookback_path):
    # every word of the workspace says "inclusive state published" under the
    # tag the next call will use, with a payload of float bits 2 (a carry of
    # about 3e-45): a call that trusted it would start each tile from zero
    cell, B, T, D, K = oracle.DIAG_GRU, 2, 1200, 96, 3
    x = _inputs(cell, B, T, D, seed=3)
    ws = binding.workspace_for(cell, B, T, D, K, DEV)
    binding.newton_forward(cell, x["pxt"], x["wt"], None, K=K, workspace=ws)
    words = ws.view(torch.int64)
    e = _tag(words, HEADER_WORDS)
    words.fill_(((e + 1) << 32) | 2)
    H = binding.newton_forward(cell, x["pxt"], x["wt"], None, K=K, workspace=ws)
    assert _tag(words, HEADER_WORDS) == e + 1
    Ho, _ = oracle.newton(cell, x["px"], x["w"], None, K=K)
    assert rel_err(to_np(H), Ho) <= TOL_H


@pytest.mark.parametrize("cell", [oracle.LINEAR, oracle.DIAG_GRU, oracle.DIAG_LSTM])
def test_lookback_timeout_then_recovery(cell, cuda_device):
    # several tiles along T (one channel group), so tile 1 waits on tile 0
    B, T, D, K = 1, 1000, 32, 2
    x = _inputs(cell, B, T, D, seed=4)
    ws = binding.workspace_for(cell, B, T, D, K, DEV)
    stream = torch.cuda.current_stream()
    H = torch.empty((B, T, oracle.STATE_WIDTH[cell], D), device=DEV)
    G = oracle.NUM_GATES[cell]
    dpx = torch.empty((B, T, G, D), device=DEV)
    assert binding.pararnn_debug_hooks(20_000_000, 1) == binding.OK  # 20 ms, stall the first tile
    try:
        # (the stall hook also keeps the forward on the look-back path)
        for direction in ("forward", "backward"):
            torch.cuda.synchronize()
            t0 = time.perf_counter()
            if direction == "forward":
                st = binding.pararnn_newton_forward(cell, B, T, D, binding.F32, x["pxt"], x["wt"], None, K, H, ws,
                                                    ws.numel(), None, stream)
            else:
                st = binding.pararnn_newton_backward(cell, B, T, D, binding.F32, x["pxt"], x["wt"], None, H,
                                                     x["gt"], dpx, None, None, ws, ws.numel(), stream)
            assert st == binding.OK, binding.pararnn_last_error()
            assert binding.pararnn_status_sync(ws, stream) == binding.ETIMEOUT, direction
            elapsed = time.perf_counter() - t0
            assert elapsed < 1.0, (direction, elapsed)
    finally:
        assert binding.pararnn_debug_hooks(0, 0) == binding.OK
    # the context is usable and the same workspace gives the right answer
    Hn = binding.newton_forward(cell, x["pxt"], x["wt"], None, K=K, workspace=ws)
    Ho, _ = oracle.newton(cell, x["px"], x["w"], None, K=K)
    assert rel_err(to_np(Hn), Ho) <= TOL_H
    dpxn, _, _ = binding.newton_backward(cell, x["pxt"], Hn, x["gt"], x["wt"], workspace=ws)
    dpxo, _, _ = oracle.adjoint(cell, x["px"], x["w"], None, Ho, x["g"])
    assert rel_err(to_np(dpxn), dpxo) <= TOL_G

