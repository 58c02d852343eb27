"""The C-ABI library on the CPU: it loads, it exports every symbol that
include/pararnn_b200.h declares, and its pure host functions and argument
checks behave as documented.  No kernel is launched here."""
import ctypes
import os
import re
import subprocess

import pytest

from nonlinear_rnn_iteration_b200 import binding, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "pararnn_b200.h")


def declared_symbols():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(pararnn_[a-z_0-9]+)\s*\(", text)))


def test_header_declares_the_boundary():
    syms = declared_symbols()
    for name in ("pararnn_newton_forward", "pararnn_newton_backward", "pararnn_workspace_bytes",
                 "pararnn_status_sync", "pararnn_status_string"):
        assert name in syms


def test_library_exports_every_declared_symbol():
    so = build.build()
    out = subprocess.run(["nm", "-D", "--defined-only", so], capture_output=True, text=True, check=True).stdout
    exported = set(re.findall(r"\bT\s+(pararnn_\w+)", out))
    missing = [s for s in declared_symbols() if s not in exported]
    assert not missing, "declared but not exported: %s" % missing
    lib = ctypes.CDLL(so)
    for s in declared_symbols():
        assert getattr(lib, s) is not None


def test_binding_covers_every_declared_symbol():
    assert sorted(binding.SIGNATURES) == declared_symbols()
    for s in declared_symbols():
        assert callable(getattr(binding, s))


def test_library_links_no_shared_cudart():
    out = subprocess.run(["ldd", build.build()], capture_output=True, text=True).stdout
    assert "libcudart" not in out  # runtime linked statically: loads on a machine without the toolkit


def test_cell_tables_and_status_strings():
    assert [binding.pararnn_num_gates(c) for c in (0, 1, 2)] == [2, 3, 4]
    assert [binding.pararnn_state_width(c) for c in (0, 1, 2)] == [1, 1, 2]
    assert binding.pararnn_num_gates(7) == -1
    for code, name in binding.STATUS.items():
        assert binding.pararnn_status_string(code) == name
    assert binding.pararnn_status_string(99) == "PARARNN_UNKNOWN"


def test_workspace_bytes():
    f = binding.pararnn_workspace_bytes
    assert f(9, 1, 1, 1, 1) == 0
    assert f(1, -1, 1, 1, 1) == 0
    assert f(1, 0, 0, 0, 1) >= 256
    small = f(1, 1, 1024, 64, 3)
    assert small > 256
    assert f(1, 2, 1024, 64, 3) > small  # grows with the problem
    assert f(1, 1, 1024, 64, 4) > small  # one carry set per Newton iteration
    assert f(0, 1, 1024, 64, 3) == f(0, 1, 1024, 64, 1)  # the linear cell does one scan for any K
    # one buffer serves forward and backward
    assert f(2, 4, 32768, 1024, 4) >= f(2, 4, 32768, 1024, 1)


@pytest.mark.parametrize("case", ["cell", "dtype", "K0", "K65", "ws_null", "ws_small", "ws_misaligned", "neg"])
def test_forward_rejects_bad_arguments(case):
    fake = 1 << 40  # never dereferenced: the checks fail first
    args = dict(cell=1, B=1, T=8, D=8, px_dtype=0, preacts=fake, diag_w=None, h0=None, K=2, H_out=fake,
                workspace=fake, ws_bytes=1 << 30, resid_hist=None, stream=None)
    if case == "cell":
        args["cell"] = 5
    elif case == "dtype":
        args["px_dtype"] = 3
    elif case == "K0":
        args["K"] = 0
    elif case == "K65":
        args["K"] = 65
    elif case == "ws_null":
        args["workspace"] = None
    elif case == "ws_small":
        args["ws_bytes"] = 16
    elif case == "ws_misaligned":
        args["workspace"] = fake + 4
    elif case == "neg":
        args["T"] = -3
    st = binding.pararnn_newton_forward(**args)
    assert st == binding.EINVAL
    assert binding.pararnn_last_error() != ""


def test_backward_rejects_bad_arguments():
    fake = 1 << 40
    st = binding.pararnn_newton_backward(1, 1, 8, 8, 0, fake, None, None, None, fake, fake, None, None, fake,
                                         1 << 30, None)
    assert st == binding.EINVAL  # H is NULL
    st = binding.pararnn_newton_backward(1, 1, 8, 8, 0, fake, None, None, fake, fake, fake, None, None, fake, 8,
                                         None)
    assert st == binding.EINVAL  # workspace too small


def test_probe_rejects_bad_arguments():
    assert binding.pararnn_probe_wait_timeout(None, 1024, 1000, None) == binding.EINVAL
    assert binding.pararnn_probe_wait_timeout(1 << 40, 16, 1000, None) == binding.EINVAL
    assert binding.pararnn_probe_wait_timeout(1 << 40, 1024, 0, None) == binding.EINVAL


def test_head_gru_workspace_bytes():
    f, fb = binding.pararnn_head_gru_workspace_bytes, binding.pararnn_head_gru_backward_workspace_bytes
    # invalid: head width 8, D not a multiple of n_heads, K outside 1..64
    assert f(1, 16, 64, 8, 2) == 0
    assert f(1, 16, 100, 3, 2) == 0
    assert f(1, 16, 128, 2, 0) == 0 and f(1, 16, 128, 2, 65) == 0
    assert fb(1, 16, 64, 8) == 0 and fb(1, 16, 100, 3) == 0
    B, T, D, nh = 2, 300, 128, 2
    n = B * T * D * 4
    one, two = f(B, T, D, nh, 1), f(B, T, D, nh, 2)
    # six float row factors per element; K >= 2 adds the second iterate buffer
    assert one >= 6 * n and two - one >= n
    assert f(B, T, D, nh, 3) == two
    assert f(B, 2 * T, D, nh, 2) > two
    # lambda * gamma and five float row factors per element, plus the products
    assert fb(B, T, D, nh) >= 6 * n
    assert f(0, T, D, nh, 2) >= 256 and fb(0, T, D, nh) >= 256


def test_head_gru_rejects_bad_arguments():
    fake = 1 << 40  # never dereferenced: the checks fail first
    ws = binding.pararnn_head_gru_workspace_bytes(1, 8, 64, 1, 2)
    fwd = binding.pararnn_head_gru_forward
    assert fwd(1, 8, 64, 1, binding.F32, fake, fake, None, 0, fake, fake, ws, None, None) == binding.EINVAL  # K
    assert fwd(1, 8, 48, 2, binding.F32, fake, fake, None, 2, fake, fake, ws, None, None) == binding.EINVAL  # d = 24
    assert fwd(1, 8, 64, 1, 7, fake, fake, None, 2, fake, fake, ws, None, None) == binding.EINVAL  # dtype
    assert fwd(1, 8, 64, 1, binding.F32, fake, fake, None, 2, fake, None, ws, None, None) == binding.EINVAL
    assert fwd(1, 8, 64, 1, binding.F32, fake, fake, None, 2, fake, fake, ws - 1, None, None) == binding.EINVAL
    assert binding.pararnn_last_error() != ""
    wsb = binding.pararnn_head_gru_backward_workspace_bytes(1, 8, 64, 1)
    bwd = binding.pararnn_head_gru_backward
    assert bwd(1, 8, 64, 1, binding.F32, fake, fake, None, fake, fake, fake, None, None, fake, wsb - 1,
               None) == binding.EINVAL
    assert bwd(1, 8, 60, 1, binding.F32, fake, fake, None, fake, fake, fake, None, None, fake, 1 << 30,
               None) == binding.EINVAL  # d = 60


def test_host_path_workspace_bytes():
    f = binding.pararnn_newton_forward_host_workspace_bytes
    gru = 1
    assert f(gru, 8, 1024, 256, 3, 7, 1) == 0  # dtype
    assert f(gru, 8, 1024, 256, 3, binding.F32, 0) == 0  # rows per slice
    assert f(9, 8, 1024, 256, 3, binding.F32, 1) == 0  # cell
    one, two = f(gru, 8, 1024, 256, 3, binding.F32, 1), f(gru, 8, 1024, 256, 3, binding.F32, 2)
    # three device slots, each holding one slice's pre-activations, H and solver workspace
    row_px, row_h = 1024 * 3 * 256 * 4, 1024 * 256 * 4
    assert one >= 3 * (row_px + row_h) and two - one >= 3 * (row_px + row_h)
    assert f(gru, 8, 1024, 256, 3, binding.BF16, 1) < one  # bf16 slices are smaller
    # channel slices: a multiple of 8 of a D that is a multiple of 8; 0 or
    # >= D means whole rows
    assert f(gru, 8, 1024, 256, 3, binding.F32, 1, 12) == 0
    assert f(gru, 8, 1024, 100, 3, binding.F32, 1, 8) == 0
    assert f(gru, 8, 1024, 256, 3, binding.F32, 1, -8) == 0
    assert f(gru, 8, 1024, 256, 3, binding.F32, 1, 256) == one == f(gru, 8, 1024, 256, 3, binding.F32, 1, 512)
    assert 0 < f(gru, 8, 1024, 256, 3, binding.F32, 1, 64) < one
    # a slice never exceeds the batch
    assert f(gru, 2, 1024, 256, 3, binding.F32, 5) == f(gru, 2, 1024, 256, 3, binding.F32, 2)


def test_step_host_workspace_bytes():
    f = binding.pararnn_newton_step_host_workspace_bytes
    gru = 1
    assert f(gru, 2, 1024, 256, 3, 7, 0) == 0  # dtype
    assert f(9, 2, 1024, 256, 3, binding.F32, 0) == 0  # cell
    assert f(gru, 2, 1024, 256, 3, binding.F32, 12) == 0  # not a multiple of 8
    assert f(gru, 2, 1024, 100, 3, binding.F32, 8) == 0  # D not a multiple of 8
    assert f(gru, 2, 1024, 256, 3, binding.F32, -8) == 0
    whole = f(gru, 2, 1024, 256, 3, binding.F32, 0)
    assert whole == f(gru, 2, 1024, 256, 3, binding.F32, 256) == f(gru, 2, 1024, 256, 3, binding.F32, 1000)
    # three slots of pre-activations, dL/dH, H, dL/dpx (float32) and a solver workspace
    n = 2 * 1024 * 256
    assert whole >= 3 * n * (3 * 4 + 4 + 4 + 3 * 4) + 3 * binding.pararnn_workspace_bytes(gru, 2, 1024, 256, 3)
    assert 0 < f(gru, 2, 1024, 256, 3, binding.F32, 64) < whole
    assert f(gru, 2, 1024, 256, 3, binding.BF16, 64) < f(gru, 2, 1024, 256, 3, binding.F32, 64)


def test_debug_hooks_reject_long_limits():
    # pure host function: it only records the limits for later calls on this thread
    assert binding.pararnn_debug_hooks(20_000_000_000, 0) == binding.EINVAL
    assert "10 s" in binding.pararnn_last_error()
    assert binding.pararnn_debug_hooks(20_000_000, 1) == binding.OK
    assert binding.pararnn_debug_hooks(0, 0) == binding.OK


def test_kstar_table_lookup():
    # K = 0 selects K*(cell, T): the linear cell needs its one scan; a length
    # between grid points takes the next grid point's entry, past the grid the
    # last entry
    assert binding.pararnn_kstar(binding.LINEAR, 1000) == 1
    assert binding.pararnn_kstar(7, 1000) == -1
    assert binding.pararnn_kstar(binding.DIAG_GRU, -1) == -1
    for cell in (binding.DIAG_GRU, binding.DIAG_LSTM):
        ks = [binding.pararnn_kstar(cell, T) for T in (1, 16, 17, 64, 1000, 1024, 4096, 131072, 262144, 10 ** 7)]
        assert all(1 <= k <= 8 for k in ks)
        assert ks == sorted(ks)  # an envelope: never fewer iterations for a longer sequence
        assert binding.pararnn_kstar(cell, 17) == binding.pararnn_kstar(cell, 64)
        assert binding.pararnn_kstar(cell, 10 ** 7) == binding.pararnn_kstar(cell, 262144)
    # the workspace for K = 0 is the one for K = K*
    for cell in (binding.DIAG_GRU, binding.DIAG_LSTM):
        assert binding.pararnn_workspace_bytes(cell, 2, 5000, 64, 0) == binding.pararnn_workspace_bytes(
            cell, 2, 5000, 64, binding.pararnn_kstar(cell, 5000))


def test_picard_iters_outside_range_is_rejected():
    # checked before any pointer: nothing is launched
    for p in (-1, 5):
        st = binding.pararnn_newton_forward_picard(binding.DIAG_GRU, 1, 10, 8, binding.F32, None, None, None, p, 2,
                                                   None, None, 0, None, None)
        assert st == binding.EINVAL
        assert "picard_iters" in binding.pararnn_last_error()
