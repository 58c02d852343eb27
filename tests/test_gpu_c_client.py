"""The C ABI from a plain C program: tests/c_abi_client.c (cudaMalloc'd
buffers, no Python between it and the library) runs the forward and the
adjoint through libpararnn_b200, and its outputs must match the fp64 oracle.
The compile step runs on any machine; the run needs the GPU."""
import os
import subprocess

import numpy as np
import pytest

import oracle
from gpu_util import rel_err
from nonlinear_rnn_iteration_b200 import build as lib_build

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CUDA = os.environ.get("CUDA_HOME", "/usr/local/cuda")
TOL_H, TOL_G = 1e-4, 1e-3


def _compile(tmp_path):
    so = lib_build.build()
    exe = str(tmp_path / "c_abi_client")
    cmd = ["gcc", "-O2", "-std=c99", "-I", os.path.join(ROOT, "include"), "-I", os.path.join(CUDA, "include"),
           os.path.join(HERE, "c_abi_client.c"), "-o", exe, so, "-L", os.path.join(CUDA, "lib64"), "-lcudart",
           "-Wl,-rpath," + os.path.dirname(so) + ":" + os.path.join(CUDA, "lib64")]
    subprocess.check_call(cmd)
    return exe


def test_c_client_compiles_and_links(tmp_path):
    # no GPU needed: the header and the library's exported symbols are enough
    exe = _compile(tmp_path)
    assert os.path.exists(exe)


@pytest.mark.gpu
@pytest.mark.parametrize("cell,B,T,D,K", [(oracle.DIAG_GRU, 2, 700, 100, 3), (oracle.DIAG_LSTM, 1, 450, 40, 4),
                                          (oracle.LINEAR, 2, 300, 64, 1)])
def test_c_client_matches_oracle(tmp_path, cell, B, T, D, K, cuda_device):
    exe = _compile(tmp_path)
    rng = np.random.default_rng(cell * 31 + T)
    G, S = oracle.NUM_GATES[cell], oracle.STATE_WIDTH[cell]
    px = rng.standard_normal((B, T, G, D)).astype(np.float32)
    if cell == oracle.LINEAR:
        px[:, :, 0, :] = 1.0 / (1.0 + np.exp(-px[:, :, 0, :]))
    w = rng.uniform(-0.5, 0.5, (G, D)).astype(np.float32)
    g = rng.standard_normal((B, T, S, D)).astype(np.float32)
    for name, a in (("px", px), ("w", w), ("g", g)):
        a.tofile(str(tmp_path / ("%s.f32" % name)))
    subprocess.run([exe, str(tmp_path), str(cell), str(B), str(T), str(D), str(K)], check=True,
                   capture_output=True, text=True)
    H = np.fromfile(str(tmp_path / "H.f32"), dtype=np.float32).reshape(B, T, S, D)
    dpx = np.fromfile(str(tmp_path / "dpx.f32"), dtype=np.float32).reshape(B, T, G, D)
    da = np.fromfile(str(tmp_path / "da.f32"), dtype=np.float32).reshape(G, D)
    wo = None if cell == oracle.LINEAR else w
    Ho, _ = oracle.newton(cell, px, wo, None, K=K)
    dpxo, dao, _ = oracle.adjoint(cell, px, wo, None, H.astype(np.float64), g)
    assert rel_err(H, Ho) <= TOL_H
    assert rel_err(dpx, dpxo) <= TOL_G
    if cell != oracle.LINEAR:
        assert rel_err(da, dao) <= TOL_G
