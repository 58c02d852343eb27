"""GPU parity of the head-wise GRU forward (block-diagonal recurrent weights)
against the fp64 oracle, through the C ABI.

Tolerances as for the diagonal cells (gpu_util.rel_err): H <= 1e-4; the
residual history within 1e-4 of the largest residual; bf16 pre-activations
against the oracle on the same bf16 values <= 1e-4.  Cases cover every
supported head width (16, 32, 64; 64 runs the chunk products on tcgen05,
the narrower widths on mma.sync), one and several heads, a single step,
sequences that end inside a chunk or one step into a new one, an initial
state, K = 1..3 and K = T.
"""
import numpy as np
import pytest
import torch

import oracle
import slow_inputs
from gpu_util import rel_err, to_np
from nonlinear_rnn_iteration_b200 import binding, workloads

pytestmark = pytest.mark.gpu
TOL_H = 1e-4
DEV = "cuda:0"


def _case(B, T, D, nh, seed, h0=False):
    x = workloads.head_host_inputs(B, T, D, nh, seed)
    hz = (0.5 * np.random.default_rng(seed + 1).standard_normal((B, D))).astype(np.float32) if h0 else None
    t = lambda a: None if a is None else torch.from_numpy(np.ascontiguousarray(a)).to(DEV)
    return x["px"], x["U"], hz, t(x["px"]), t(x["U"]), t(hz)


CASES = [  # (B, T, D, n_heads, K)
    (2, 100, 64, 1, 3),
    (1, 77, 96, 3, 2),
    (2, 40, 48, 3, 1),
    (1, 130, 128, 2, 3),
    (2, 64, 256, 4, 2),
    # head width 64 (the tcgen05 products): one step, a last chunk of one
    # step, two whole chunks of 128 steps, three chunks (the first chunk's
    # product then carries into the last)
    (1, 1, 64, 1, 1),
    (3, 129, 64, 1, 2),
    (1, 256, 128, 2, 2),
    (1, 300, 64, 1, 3),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "B%dT%dD%dh%dK%d" % c)
@pytest.mark.parametrize("h0", [False, True])
def test_head_forward_small(case, h0, cuda_device):
    B, T, D, nh, K = case
    px, U, hz, pxt, Ut, h0t = _case(B, T, D, nh, seed=D + T, h0=h0)
    resid = torch.zeros(K + 1, device=DEV)
    H = binding.head_gru_forward(pxt, Ut, h0t, K=K, resid_hist=resid)
    ref, rref = oracle.head_gru_newton(px, U, hz, K=K)
    assert rel_err(to_np(H), ref) <= TOL_H
    r = resid.cpu().numpy().astype(np.float64)
    assert np.all(np.abs(r - rref) <= 1e-4 * max(1.0, rref.max()) + 1e-6 * np.abs(rref))


# Slow memory (slow_inputs.py): p_z shifted down by 5 keeps the update gate
# almost closed, so the product of a chunk's 128 Jacobians keeps a norm of
# about 0.4 and a wrong chunk product would show.  Every head width,
# several chunks.
SLOW_CASES = [  # (B, T, D, n_heads, K)
    (1, 300, 64, 1, 3),
    (2, 260, 128, 2, 2),
    (1, 300, 32, 1, 3),
    (1, 280, 48, 3, 2),
]


def _slow_case(B, T, D, nh, seed, h0=False):
    px, U = slow_inputs.head_host(B, T, D, nh, seed)
    hz = (0.5 * np.random.default_rng(seed + 1).standard_normal((B, D))).astype(np.float32) if h0 else None
    t = lambda a: None if a is None else torch.from_numpy(np.ascontiguousarray(a)).to(DEV)
    return px, U, hz, t(px), t(U), t(hz)


@pytest.mark.parametrize("case", SLOW_CASES, ids=lambda c: "B%dT%dD%dh%dK%d" % c)
def test_head_forward_slow_memory(case, cuda_device):
    B, T, D, nh, K = case
    px, U, hz, pxt, Ut, h0t = _slow_case(B, T, D, nh, seed=D + T + 1, h0=True)
    H = binding.head_gru_forward(pxt, Ut, h0t, K=K)
    ref, _ = oracle.head_gru_newton(px, U, hz, K=K)
    assert rel_err(to_np(H), ref) <= TOL_H


def test_head_forward_bf16(cuda_device):
    B, T, D, nh, K = 2, 90, 128, 2, 3
    px, U, _, _, Ut, _ = _case(B, T, D, nh, seed=7)
    pxb = workloads.round_bf16(px)
    H = binding.head_gru_forward(torch.from_numpy(px).to(DEV).to(torch.bfloat16), Ut, None, K=K)
    ref, _ = oracle.head_gru_newton(pxb, U, None, K=K)
    assert rel_err(to_np(H), ref) <= TOL_H


def test_head_k_equal_t_is_the_unroll(cuda_device):
    B, T, D, nh = 1, 10, 64, 2
    px, U, hz, pxt, Ut, h0t = _case(B, T, D, nh, seed=9, h0=True)
    H = binding.head_gru_forward(pxt, Ut, h0t, K=T)
    assert rel_err(to_np(H), oracle.head_gru_unroll(px, U, hz)) <= 5e-5


def test_head_deterministic(cuda_device):
    B, T, D, nh = 2, 200, 128, 2
    _, _, _, pxt, Ut, _ = _case(B, T, D, nh, seed=11)
    a = binding.head_gru_forward(pxt, Ut, None, K=3)
    b = binding.head_gru_forward(pxt, Ut, None, K=3)
    assert torch.equal(a, b)


def test_head_full_size_sampled(cuda_device):
    w = workloads.HEAD_WORKLOADS["headgru_8x4096x512_h8_k3"]
    x = workloads.head_device_inputs(w, DEV)
    resid = torch.zeros(w.K + 1, device=DEV)
    H = binding.head_gru_forward(x["px"], x["U"], None, K=w.K, resid_hist=resid)
    U = x["U"].cpu().numpy()
    rng = np.random.default_rng(5)
    for b, h in [(int(rng.integers(w.B)), int(rng.integers(w.n_heads))) for _ in range(3)]:
        sl = slice(h * w.d, (h + 1) * w.d)
        px = x["px"][b:b + 1, :, :, sl].cpu().numpy()
        ref, _ = oracle.head_gru_newton(px, U[:, h:h + 1], None, K=w.K)
        assert rel_err(to_np(H[b:b + 1, :, sl]), ref) <= TOL_H, (b, h)
    r = resid.cpu().numpy()
    assert np.isfinite(r).all() and r[-1] < 1e-2 * r[0]


def test_head_rejects_bad_arguments(cuda_device):
    px = torch.zeros((1, 4, 3, 16), device=DEV)
    U = torch.zeros((3, 2, 8, 8), device=DEV)
    H = torch.zeros((1, 4, 16), device=DEV)
    ws = torch.zeros(1 << 20, dtype=torch.uint8, device=DEV)
    # head width 8 is not supported; D not a multiple of n_heads; K out of range
    assert binding.pararnn_head_gru_workspace_bytes(1, 4, 16, 2, 1) == 0
    assert binding.pararnn_head_gru_workspace_bytes(1, 4, 50, 3, 1) == 0
    assert binding.pararnn_head_gru_workspace_bytes(1, 4, 64, 1, 0) == 0
    assert binding.pararnn_head_gru_forward(1, 4, 16, 2, binding.F32, px, U, None, 1, H, ws, ws.numel(), None,
                                            None) == binding.EINVAL
    # a workspace that is too small
    n = binding.pararnn_head_gru_workspace_bytes(1, 4, 64, 1, 2)
    px = torch.zeros((1, 4, 3, 64), device=DEV)
    U = torch.zeros((3, 1, 64, 64), device=DEV)
    H = torch.zeros((1, 4, 64), device=DEV)
    assert binding.pararnn_head_gru_forward(1, 4, 64, 1, binding.F32, px, U, None, 2, H, ws, n - 1, None,
                                            None) == binding.EINVAL
    # host memory
    assert binding.pararnn_head_gru_forward(1, 4, 64, 1, binding.F32, px.cpu().data_ptr(), U, None, 2, H, ws,
                                            ws.numel(), None, None) == binding.EINVAL


def test_head_empty_and_nonfinite(cuda_device):
    px = torch.zeros((0, 5, 3, 64), device=DEV)
    U = torch.zeros((3, 1, 64, 64), device=DEV)
    assert binding.head_gru_forward(px, U, None, K=2).shape == (0, 5, 64)
    px = torch.randn((1, 40, 3, 64), device=DEV)
    px[0, 17, 2, 5] = float("nan")
    with pytest.raises(binding.PararnnError) as e:
        binding.head_gru_forward(px, U, None, K=2)
    assert e.value.status == binding.ENONFINITE


# ---- the adjoint ---------------------------------------------------------
TOL_G = 1e-3

BWD_CASES = [  # (B, T, D, n_heads, K)
    (2, 100, 64, 1, 3),
    (1, 150, 96, 3, 2),
    (2, 40, 64, 2, 1),
    (1, 200, 128, 2, 3),
    (1, 1, 64, 1, 1),
    (3, 129, 64, 1, 2),
    (1, 300, 64, 1, 3),
]


@pytest.mark.parametrize("case", BWD_CASES, ids=lambda c: "B%dT%dD%dh%dK%d" % c)
@pytest.mark.parametrize("h0", [False, True])
def test_head_backward_small(case, h0, cuda_device):
    B, T, D, nh, K = case
    px, U, hz, pxt, Ut, h0t = _case(B, T, D, nh, seed=3 * D + T, h0=h0)
    g = np.random.default_rng(T + D).standard_normal((B, T, D)).astype(np.float32)
    H = binding.head_gru_forward(pxt, Ut, h0t, K=K)
    dpx, dU, dh0 = binding.head_gru_backward(pxt, Ut, H, torch.from_numpy(g).to(DEV), h0=h0t, want_dh0=True)
    r_dpx, r_dU, r_dh0 = oracle.head_gru_adjoint(px, U, to_np(H), g, hz)
    assert rel_err(to_np(dpx), r_dpx) <= TOL_G
    assert rel_err(to_np(dU), r_dU) <= TOL_G
    assert rel_err(to_np(dh0), r_dh0) <= TOL_G


@pytest.mark.parametrize("case", SLOW_CASES, ids=lambda c: "B%dT%dD%dh%dK%d" % c)
def test_head_backward_slow_memory(case, cuda_device):
    B, T, D, nh, K = case
    px, U, hz, pxt, Ut, h0t = _slow_case(B, T, D, nh, seed=3 * D + T + 1, h0=True)
    g = np.random.default_rng(T + D + 1).standard_normal((B, T, D)).astype(np.float32)
    H = binding.head_gru_forward(pxt, Ut, h0t, K=K)
    dpx, dU, dh0 = binding.head_gru_backward(pxt, Ut, H, torch.from_numpy(g).to(DEV), h0=h0t, want_dh0=True)
    r_dpx, r_dU, r_dh0 = oracle.head_gru_adjoint(px, U, to_np(H), g, hz)
    assert rel_err(to_np(dpx), r_dpx) <= TOL_G
    assert rel_err(to_np(dU), r_dU) <= TOL_G
    assert rel_err(to_np(dh0), r_dh0) <= TOL_G


@pytest.mark.parametrize("D,nh", [(128, 2), (64, 2)], ids=["d64", "d32"])
def test_head_backward_bf16(D, nh, cuda_device):
    # bf16 pre-activations (widened on load) against the oracle on the same
    # bf16 values, slow memory, three chunks
    B, T, K = 2, 300, 3
    px, U = slow_inputs.head_host(B, T, D, nh, seed=D + 5)
    pxb = workloads.round_bf16(px)
    pxt = torch.from_numpy(px).to(DEV).to(torch.bfloat16)
    Ut = torch.from_numpy(U).to(DEV)
    g = np.random.default_rng(D + 6).standard_normal((B, T, D)).astype(np.float32)
    H = binding.head_gru_forward(pxt, Ut, None, K=K)
    ref, _ = oracle.head_gru_newton(pxb, U, None, K=K)
    assert rel_err(to_np(H), ref) <= TOL_H
    dpx, dU, _ = binding.head_gru_backward(pxt, Ut, H, torch.from_numpy(g).to(DEV))
    r_dpx, r_dU, _ = oracle.head_gru_adjoint(pxb, U, to_np(H), g, None)
    assert rel_err(to_np(dpx), r_dpx) <= TOL_G
    assert rel_err(to_np(dU), r_dU) <= TOL_G


def test_head_backward_deterministic_and_optional_outputs(cuda_device):
    B, T, D, nh = 2, 300, 128, 2
    _, _, _, pxt, Ut, _ = _case(B, T, D, nh, seed=21)
    H = binding.head_gru_forward(pxt, Ut, None, K=3)
    g = torch.randn((B, T, D), device=DEV)
    a = binding.head_gru_backward(pxt, Ut, H, g, want_dh0=True)
    b = binding.head_gru_backward(pxt, Ut, H, g, want_dh0=True)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1]) and torch.equal(a[2], b[2])
    c = binding.head_gru_backward(pxt, Ut, H, g, want_dU=False)
    assert c[1] is None and c[2] is None and torch.equal(c[0], a[0])


def test_head_backward_full_size_sampled(cuda_device):
    w = workloads.HEAD_WORKLOADS["headgru_8x4096x512_h8_k3"]
    x = workloads.head_device_inputs(w, DEV)
    H = binding.head_gru_forward(x["px"], x["U"], None, K=w.K)
    g = torch.randn((w.B, w.T, w.D), device=DEV, generator=torch.Generator(device=DEV).manual_seed(77))
    dpx, dU, _ = binding.head_gru_backward(x["px"], x["U"], H, g)
    # dL/dpx per sampled (b, head) sequence; dL/dU of one head summed over all b
    U = x["U"].cpu().numpy()
    h = 5
    sl = slice(h * w.d, (h + 1) * w.d)
    dU_ref = np.zeros((3, 1, w.d, w.d))
    for b in range(w.B):
        px = x["px"][b:b + 1, :, :, sl].cpu().numpy()
        r_dpx, r_dU, _ = oracle.head_gru_adjoint(px, U[:, h:h + 1], to_np(H[b:b + 1, :, sl]),
                                                 to_np(g[b:b + 1, :, sl]))
        dU_ref += r_dU
        if b in (0, 5):
            assert rel_err(to_np(dpx[b:b + 1, :, :, sl]), r_dpx) <= TOL_G, b
    assert rel_err(to_np(dU[:, h:h + 1]), dU_ref) <= TOL_G


# ---- the sequential unroll on the GPU (pararnn_head_gru_unroll) -------------

@pytest.mark.parametrize("case", [(2, 100, 64, 1), (1, 77, 96, 3), (2, 40, 48, 3), (1, 130, 128, 2),
                                  (3, 33, 256, 4), (1, 1, 64, 1)], ids=lambda c: "B%dT%dD%dh%d" % c)
@pytest.mark.parametrize("h0", [False, True])
def test_head_unroll_matches_oracle(case, h0, cuda_device):
    B, T, D, nh = case
    px, U, hz, pxt, Ut, hzt = _case(B, T, D, nh, seed=T + D, h0=h0)
    H = binding.head_gru_unroll(pxt, Ut, hzt)
    ref = oracle.head_gru_unroll(px, U, hz)
    assert rel_err(to_np(H), ref) <= TOL_H


def test_head_unroll_bf16_slow_memory_and_newton(cuda_device):
    # bf16 pre-activations against the oracle on the same values
    x = workloads.head_host_inputs(2, 300, 128, 2, 31)
    pxb = torch.from_numpy(x["px"]).to(DEV).to(torch.bfloat16)
    H = binding.head_gru_unroll(pxb, torch.from_numpy(x["U"]).to(DEV))
    ref = oracle.head_gru_unroll(pxb.float().cpu().numpy(), x["U"], None)
    assert rel_err(to_np(H), ref) <= TOL_H
    # slow memory, several chunks of pre-activations
    px, U = slow_inputs.head_host(1, 400, 128, 2, 32)
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(DEV)
    H = binding.head_gru_unroll(t(px), t(U))
    assert rel_err(to_np(H), oracle.head_gru_unroll(px, U, None)) <= TOL_H
    # the Newton forward at K = T reaches the same sequence
    px, U, hz, pxt, Ut, hzt = _case(1, 20, 64, 1, seed=33, h0=True)
    Hn = binding.head_gru_forward(pxt, Ut, hzt, K=20)
    Hu = binding.head_gru_unroll(pxt, Ut, hzt)
    assert rel_err(to_np(Hn), to_np(Hu)) <= TOL_H


def test_head_unroll_rejects_bad_arguments(cuda_device):
    px = torch.zeros((1, 8, 3, 64), device=DEV)
    U = torch.zeros((3, 1, 64, 64), device=DEV)
    H = torch.empty((1, 8, 64), device=DEV)
    ws = torch.empty(256, dtype=torch.uint8, device=DEV)
    s = torch.cuda.current_stream()
    assert binding.pararnn_head_gru_unroll(1, 8, 64, 3, binding.F32, px, U, None, H, ws, 256, s) == binding.EINVAL
    assert binding.pararnn_head_gru_unroll(1, 8, 64, 8, binding.F32, px, U, None, H, ws, 256, s) == binding.EINVAL
    assert binding.pararnn_head_gru_unroll(1, 8, 64, 1, binding.F32, px, U, None, H, ws, 16, s) == binding.EINVAL
    assert binding.pararnn_head_gru_unroll(1, 8, 64, 1, binding.F32, px.cpu(), U, None, H, ws, 256, s) == binding.EINVAL
    bad = torch.full((1, 8, 3, 64), float("nan"), device=DEV)
    assert binding.pararnn_head_gru_unroll(1, 8, 64, 1, binding.F32, bad, U, None, H, ws, 256, s) == binding.OK
    assert binding.pararnn_status_sync(ws, s) == binding.ENONFINITE
