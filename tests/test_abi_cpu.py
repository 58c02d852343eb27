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
