"""Error paths on the GPU, none of which faults or hangs the device:
argument errors caught on the host, a non-finite input reported through the
workspace status, and the bounded inter-block wait running out on a flag that
nothing sets (the kernel records the time-out and returns)."""
import numpy as np
import pytest
import torch

from nonlinear_rnn_iteration_b200 import binding

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def test_nonfinite_input_is_reported(cuda_device):
    px = torch.randn(1, 256, 3, 64, device=DEV)
    px[0, 100, 1, 7] = float("nan")
    with pytest.raises(binding.PararnnError) as e:
        binding.newton_forward(binding.DIAG_GRU, px, None, None, K=2)
    assert e.value.status == binding.ENONFINITE
    # the library and the context stay usable
    H = binding.newton_forward(binding.DIAG_GRU, torch.randn(1, 256, 3, 64, device=DEV), None, None, K=2)
    assert torch.isfinite(H).all()


def test_nonfinite_residual_is_visible(cuda_device):
    px = torch.randn(1, 64, 2, 8, device=DEV)
    px[0, 10, 1, 3] = float("inf")
    resid = torch.zeros(2, device=DEV)
    with pytest.raises(binding.PararnnError):
        binding.newton_forward(binding.LINEAR, px, None, None, K=1, resid_hist=resid)
    assert not torch.isfinite(resid).all()


def test_wait_time_out_ends_cleanly(cuda_device):
    n = binding.pararnn_workspace_bytes(binding.LINEAR, 1, 1, 1, 1)
    ws = torch.zeros(n, dtype=torch.uint8, device=DEV)
    st = torch.cuda.current_stream()
    assert binding.pararnn_probe_wait_timeout(ws, n, 20_000_000, st) == binding.OK  # 20 ms
    assert binding.pararnn_status_sync(ws, st) == binding.ETIMEOUT
    # a normal call afterwards on the same workspace reports OK
    px = torch.randn(1, 1, 2, 1, device=DEV)
    H = torch.empty(1, 1, 1, 1, device=DEV)
    assert binding.pararnn_newton_forward(0, 1, 1, 1, 0, px, None, None, 1, H, ws, n, None, st) == binding.OK
    assert binding.pararnn_status_sync(ws, st) == binding.OK


def test_host_memory_is_rejected(cuda_device):
    host = np.zeros((1, 8, 3, 8), dtype=np.float32)
    H = torch.empty(1, 8, 1, 8, device=DEV)
    n = binding.pararnn_workspace_bytes(1, 1, 8, 8, 2)
    ws = torch.zeros(n, dtype=torch.uint8, device=DEV)
    st = binding.pararnn_newton_forward(1, 1, 8, 8, 0, host.ctypes.data, None, None, 2, H, ws, n, None, None)
    assert st == binding.EINVAL
    assert "device-accessible" in binding.pararnn_last_error()


def test_misaligned_pointer_is_rejected(cuda_device):
    buf = torch.zeros(1 + 8 * 3 * 8, device=DEV)
    H = torch.empty(1, 8, 1, 8, device=DEV)
    n = binding.pararnn_workspace_bytes(1, 1, 8, 8, 2)
    ws = torch.zeros(n, dtype=torch.uint8, device=DEV)
    st = binding.pararnn_newton_forward(1, 1, 8, 8, 0, buf.data_ptr() + 2, None, None, 2, H, ws, n, None, None)
    assert st == binding.EINVAL
