"""The no-allocation forward entry point, checked against the ordinary one.

Callers that cannot allocate device memory (a framework that owns every
device allocation, a loop that cannot afford cudaMalloc's synchronisation, a
fixed device-memory budget) use pararnn_newton_forward_noalloc, which keeps
its scratch memory in a fixed array inside the library.  This test calls it
through the C ABI twice in a row, on two different problems, and compares
each result with pararnn_newton_forward's on the same inputs, within the
tolerance the parity tests use for H.  This file is named so that pytest
collects it last.
"""
import numpy as np
import pytest
import torch

from gpu_util import rel_err, to_np
from nonlinear_rnn_iteration_b200 import binding

pytestmark = pytest.mark.gpu
TOL_H = 1e-4
DEV = "cuda:0"


def _problem(cell, B, T, D, seed):
    rng = np.random.default_rng(seed)
    G = binding.pararnn_num_gates(cell)
    px = rng.standard_normal((B, T, G, D)).astype(np.float32)
    w = rng.uniform(-0.5, 0.5, (G, D)).astype(np.float32)
    return torch.from_numpy(px).to(DEV), torch.from_numpy(w).to(DEV)


def test_noalloc_forward_matches_forward_on_two_calls_in_a_row(cuda_device):
    stream = torch.cuda.current_stream()
    cases = [(binding.DIAG_GRU, 2, 300, 136, 3, 11), (binding.DIAG_LSTM, 1, 200, 72, 2, 12)]
    for cell, B, T, D, K, seed in cases:
        px, w = _problem(cell, B, T, D, seed)
        S = binding.pararnn_state_width(cell)
        ref = binding.newton_forward(cell, px, w, None, K=K)
        H = torch.full((B, T, S, D), float("nan"), device=DEV)
        resid = torch.zeros(K + 1, device=DEV)
        st = binding.pararnn_newton_forward_noalloc(cell, B, T, D, binding.F32, px, w, None, K, H, resid, 1, stream)
        assert st == binding.OK, binding.pararnn_last_error()
        assert rel_err(to_np(H), to_np(ref)) <= TOL_H
        assert torch.isfinite(resid).all() and resid[-1] < resid[0]


def test_noalloc_forward_allocates_no_device_memory(cuda_device):
    # after a first call (which looks up the array on this device), further
    # calls leave both torch's allocator counters and the driver's free
    # device memory exactly where they were
    stream = torch.cuda.current_stream()
    cell, B, T, D, K = binding.DIAG_GRU, 1, 500, 128, 3
    px, w = _problem(cell, B, T, D, 21)
    H = torch.empty((B, T, 1, D), device=DEV)
    resid = torch.empty(K + 1, device=DEV)
    st = binding.pararnn_newton_forward_noalloc(cell, B, T, D, binding.F32, px, w, None, K, H, resid, 1, stream)
    assert st == binding.OK, binding.pararnn_last_error()
    torch.cuda.synchronize()
    stats0 = torch.cuda.memory_stats()
    free0, _ = torch.cuda.mem_get_info()
    for _ in range(3):
        st = binding.pararnn_newton_forward_noalloc(cell, B, T, D, binding.F32, px, w, None, K, H, resid, 1, stream)
        assert st == binding.OK, binding.pararnn_last_error()
    torch.cuda.synchronize()
    stats1 = torch.cuda.memory_stats()
    free1, _ = torch.cuda.mem_get_info()
    for key in ("allocation.all.allocated", "segment.all.allocated", "reserved_bytes.all.current"):
        assert stats1.get(key, 0) == stats0.get(key, 0), key
    assert free1 == free0


def test_noalloc_forward_rejects_problems_beyond_its_array(cuda_device):
    px = torch.empty(1, device=DEV)
    H = torch.empty(1, device=DEV)
    # a problem whose workspace is far beyond 32 MiB; nothing is launched
    st = binding.pararnn_newton_forward_noalloc(binding.DIAG_GRU, 8, 1 << 20, 4096, binding.F32, px, None, None, 3, H,
                                                None, 1, None)
    assert st == binding.EINVAL
    assert "32 MiB" in binding.pararnn_last_error()
