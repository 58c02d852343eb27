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
