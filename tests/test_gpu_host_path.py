"""The forward on host buffers (pararnn_newton_forward_host): slices of batch
rows (and of channels) pipelined through three device slots must give,
value for value, exactly the bits pararnn_newton_forward gives for the whole
batch on the device."""
import numpy as np
import pytest
import torch

from nonlinear_rnn_iteration_b200 import binding

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _inputs(cell, B, T, D, seed, bf16=False):
    g = torch.Generator().manual_seed(seed)
    G = binding.pararnn_num_gates(cell)
    px = torch.randn((B, T, G, D), generator=g)
    if cell == binding.LINEAR:
        px[:, :, 0] = torch.sigmoid(px[:, :, 0])
        w = None
    else:
        w = (torch.rand((G, D), generator=g) - 0.5).to(DEV)
    if bf16:
        px = px.to(torch.bfloat16)
    return px, w


@pytest.mark.parametrize("cell,K,bf16", [(binding.LINEAR, 1, False), (binding.DIAG_GRU, 3, False),
                                         (binding.DIAG_GRU, 2, True), (binding.DIAG_LSTM, 3, False)])
@pytest.mark.parametrize("rows", [1, 2, 5, 9])
def test_host_path_matches_device_path(cell, K, bf16, rows, cuda_device):
    B, T, D = 5, 300, 136
    px, w = _inputs(cell, B, T, D, seed=cell * 10 + rows, bf16=bf16)
    ref = binding.newton_forward(cell, px.to(DEV), w, None, K=K).cpu()
    H = binding.newton_forward_host(cell, px.pin_memory(), w, None, K=K, rows_per_slice=rows)
    assert torch.equal(H, ref)


def test_host_path_pageable_memory_and_h0(cuda_device):
    B, T, D = 4, 200, 64
    px, w = _inputs(binding.DIAG_GRU, B, T, D, seed=3)
    h0 = torch.randn((B, 1, D), device=DEV)
    ref = binding.newton_forward(binding.DIAG_GRU, px.to(DEV), w, h0, K=3).cpu()
    H = binding.newton_forward_host(binding.DIAG_GRU, px, w, h0, K=3, rows_per_slice=1)
    assert torch.equal(H, ref)


def test_host_path_reports_nonfinite_and_bad_arguments(cuda_device):
    B, T, D = 6, 100, 64
    px, w = _inputs(binding.DIAG_GRU, B, T, D, seed=4)
    px[4, 50, 1, 7] = float("nan")  # in the fifth slice
    with pytest.raises(binding.PararnnError) as e:
        binding.newton_forward_host(binding.DIAG_GRU, px.pin_memory(), w, None, K=2, rows_per_slice=1)
    assert e.value.status == binding.ENONFINITE
    assert binding.pararnn_newton_forward_host_workspace_bytes(binding.DIAG_GRU, B, T, D, 2, binding.F32, 0) == 0
    n = binding.pararnn_newton_forward_host_workspace_bytes(binding.DIAG_GRU, B, T, D, 2, binding.F32, 2)
    ws = torch.zeros(n, dtype=torch.uint8, device=DEV)
    H = torch.empty((B, T, 1, D))
    assert binding.pararnn_newton_forward_host(binding.DIAG_GRU, B, T, D, binding.F32, px, w, None, 2, H, ws, n - 256,
                                               2, 0, None) == binding.EINVAL
    # channel slices: a multiple of 8, of a D that is a multiple of 8
    assert binding.pararnn_newton_forward_host(binding.DIAG_GRU, B, T, D, binding.F32, px, w, None, 2, H, ws, n,
                                               2, 12, None) == binding.EINVAL


@pytest.mark.parametrize("cell,K,bf16", [(binding.LINEAR, 1, False), (binding.DIAG_GRU, 3, False),
                                         (binding.DIAG_GRU, 2, True), (binding.DIAG_LSTM, 3, False)])
@pytest.mark.parametrize("rows,chans", [(1, 8), (2, 64), (5, 128), (1, 136), (3, 400)])
def test_host_path_channel_slices(cell, K, bf16, rows, chans, cuda_device):
    # slices of rows x channels (strided 2-D copies, the weights and h0 cut
    # to the slice): the same bits as the device path on the whole batch
    B, T, D = 5, 300, 136
    px, w = _inputs(cell, B, T, D, seed=cell * 10 + rows + chans, bf16=bf16)
    S = binding.pararnn_state_width(cell)
    h0 = torch.randn((B, S, D), device=DEV, generator=torch.Generator(device=DEV).manual_seed(chans))
    ref = binding.newton_forward(cell, px.to(DEV), w, h0, K=K).cpu()
    H = binding.newton_forward_host(cell, px.pin_memory(), w, h0, K=K, rows_per_slice=rows, channels_per_slice=chans)
    assert torch.equal(H, ref)


# ---- forward + adjoint on host buffers (pararnn_newton_step_host) ----------

@pytest.mark.parametrize("cell,K,bf16", [(binding.LINEAR, 1, False), (binding.DIAG_GRU, 3, False),
                                         (binding.DIAG_GRU, 2, True), (binding.DIAG_LSTM, 3, False),
                                         (binding.DIAG_LSTM, 0, True)])
@pytest.mark.parametrize("chans", [0, 8, 64, 136, 48])
def test_step_host_matches_device_path(cell, K, bf16, chans, cuda_device):
    # H, dL/dpx and dL/da of the sliced pipeline are the device path's bits
    B, T, D = 3, 300, 136
    px, w = _inputs(cell, B, T, D, seed=cell * 7 + chans, bf16=bf16)
    S = binding.pararnn_state_width(cell)
    gen = torch.Generator().manual_seed(100 + chans)
    g = torch.randn((B, T, S, D), generator=gen)
    h0 = torch.randn((B, S, D), generator=gen).to(DEV)
    pxd = px.to(DEV)
    Hd = binding.newton_forward(cell, pxd, w, h0, K=K)
    dpxd, dad, _ = binding.newton_backward(cell, pxd, Hd, g.to(DEV), w, h0)
    H, dpx, da = binding.newton_step_host(cell, px.pin_memory(), g.pin_memory(), w, h0, K=K, channels_per_slice=chans)
    torch.cuda.synchronize()
    assert torch.equal(H, Hd.cpu())
    assert torch.equal(dpx, dpxd.cpu())
    if cell == binding.LINEAR:
        assert da is None
    else:
        assert torch.equal(da.cpu(), dad.cpu())


def test_step_host_pageable_memory_without_h0_or_weights(cuda_device):
    B, T, D = 2, 500, 64
    px, _ = _inputs(binding.DIAG_GRU, B, T, D, seed=11)
    g = torch.randn((B, T, 1, D), generator=torch.Generator().manual_seed(12))
    Hd = binding.newton_forward(binding.DIAG_GRU, px.to(DEV), None, None, K=2)
    dpxd, dad, _ = binding.newton_backward(binding.DIAG_GRU, px.to(DEV), Hd, g.to(DEV), None, None)
    H, dpx, da = binding.newton_step_host(binding.DIAG_GRU, px, g, None, None, K=2, channels_per_slice=16)
    assert torch.equal(H, Hd.cpu()) and torch.equal(dpx, dpxd.cpu()) and torch.equal(da.cpu(), dad.cpu())


def test_step_host_reports_nonfinite_and_bad_arguments(cuda_device):
    B, T, D = 2, 100, 64
    px, w = _inputs(binding.DIAG_GRU, B, T, D, seed=13)
    g = torch.randn((B, T, 1, D))
    g[1, 40, 0, 50] = float("inf")  # in the last of four slices
    with pytest.raises(binding.PararnnError) as e:
        binding.newton_step_host(binding.DIAG_GRU, px.pin_memory(), g.pin_memory(), w, None, K=2,
                                 channels_per_slice=16)
    assert e.value.status == binding.ENONFINITE
    g[1, 40, 0, 50] = 0.0
    n = binding.pararnn_newton_step_host_workspace_bytes(binding.DIAG_GRU, B, T, D, 2, binding.F32, 16)
    ws = torch.empty(n, dtype=torch.uint8, device=DEV)
    H, dpx = torch.empty((B, T, 1, D)), torch.empty((B, T, 3, D))
    da = torch.empty((3, D), device=DEV)
    f = binding.pararnn_newton_step_host
    assert f(binding.DIAG_GRU, B, T, D, binding.F32, px, w, None, 2, g, H, dpx, da, ws, n - 256, 16, None) == binding.EINVAL
    assert f(binding.DIAG_GRU, B, T, D, binding.F32, px, w, None, 2, g, H, dpx, da, ws, n, 12, None) == binding.EINVAL
    # the weights and dL/da live on the device
    assert f(binding.DIAG_GRU, B, T, D, binding.F32, px, w.cpu(), None, 2, g, H, dpx, da, ws, n, 16,
             None) == binding.EINVAL
    assert f(binding.DIAG_GRU, B, T, D, binding.F32, px, w, None, 2, g, H, dpx, da.cpu(), ws, n, 16,
             None) == binding.EINVAL
    assert f(binding.DIAG_GRU, B, T, D, binding.F32, px, w, None, 2, None, H, dpx, da, ws, n, 16,
             None) == binding.EINVAL
    assert f(binding.DIAG_GRU, B, T, D, binding.F32, px, w, None, 2, g, H, dpx, da, ws, n, 16, None) == binding.OK
    assert binding.pararnn_status_sync(ws, None) == binding.OK
