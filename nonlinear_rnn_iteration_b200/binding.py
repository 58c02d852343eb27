"""ctypes binding of libpararnn_b200 -- argument marshalling only.

The ``pararnn_*`` functions here have the names and argument order of the C
ABI in ``include/pararnn_b200.h``; pointer arguments accept a torch tensor
(its ``data_ptr()``), an int address, or None (NULL).  ``stream`` accepts a
``torch.cuda.Stream``, an int handle or None (the legacy default stream).

Above them, :func:`newton_forward` and :func:`newton_backward` allocate the
outputs and the workspace with torch (device memory is torch's job here) and
raise :class:`PararnnError` on a non-OK status.  Every step of the
computation runs in the library's CUDA kernels; nothing here computes.  If
the library cannot be loaded, this module raises: there is no fallback.
"""
from __future__ import annotations

import ctypes
import os

from . import build as _build

LINEAR, DIAG_GRU, DIAG_LSTM = 0, 1, 2
F32, BF16 = 0, 1
CELLS = {"linear": LINEAR, "diag_gru": DIAG_GRU, "diag_lstm": DIAG_LSTM}
STATUS = {0: "PARARNN_OK", 1: "PARARNN_EINVAL", 2: "PARARNN_ENONFINITE", 3: "PARARNN_ETIMEOUT", 4: "PARARNN_ECUDA"}
OK, EINVAL, ENONFINITE, ETIMEOUT, ECUDA = 0, 1, 2, 3, 4

# every exported symbol of include/pararnn_b200.h, with its C signature
_P, _I64, _I, _SZ, _U64 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t, ctypes.c_uint64
SIGNATURES = {
    "pararnn_num_gates": (_I, [_I]),
    "pararnn_state_width": (_I, [_I]),
    "pararnn_workspace_bytes": (_SZ, [_I, _I64, _I64, _I64, _I]),
    "pararnn_kstar": (_I, [_I, _I64]),
    "pararnn_newton_forward": (_I, [_I, _I64, _I64, _I64, _I, _P, _P, _P, _I, _P, _P, _SZ, _P, _P]),
    "pararnn_newton_forward_picard": (_I, [_I, _I64, _I64, _I64, _I, _P, _P, _P, _I, _I, _P, _P, _SZ, _P, _P]),
    "pararnn_unroll": (_I, [_I, _I64, _I64, _I64, _I, _P, _P, _P, _P, _P, _SZ, _P]),
    "pararnn_newton_backward": (_I, [_I, _I64, _I64, _I64, _I, _P, _P, _P, _P, _P, _P, _P, _P, _P, _SZ, _P]),
    "pararnn_status_sync": (_I, [_P, _P]),
    "pararnn_status_string": (ctypes.c_char_p, [_I]),
    "pararnn_last_error": (ctypes.c_char_p, []),
    "pararnn_probe_wait_timeout": (_I, [_P, _SZ, _U64, _P]),
    "pararnn_debug_hooks": (_I, [_U64, _I]),
    "pararnn_newton_forward_noalloc": (_I, [_I, _I64, _I64, _I64, _I, _P, _P, _P, _I, _P, _P, _I, _P]),
    "pararnn_newton_forward_host_workspace_bytes": (_SZ, [_I, _I64, _I64, _I64, _I, _I, _I64, _I64]),
    "pararnn_newton_forward_host": (_I, [_I, _I64, _I64, _I64, _I, _P, _P, _P, _I, _P, _P, _SZ, _I64, _I64, _P]),
    "pararnn_newton_step_host_workspace_bytes": (_SZ, [_I, _I64, _I64, _I64, _I, _I, _I64]),
    "pararnn_newton_step_host": (_I, [_I, _I64, _I64, _I64, _I, _P, _P, _P, _I, _P, _P, _P, _P, _P, _SZ, _I64, _P]),
    "pararnn_head_gru_workspace_bytes": (_SZ, [_I64, _I64, _I64, _I, _I]),
    "pararnn_head_gru_forward": (_I, [_I64, _I64, _I64, _I, _I, _P, _P, _P, _I, _P, _P, _SZ, _P, _P]),
    "pararnn_head_gru_backward_workspace_bytes": (_SZ, [_I64, _I64, _I64, _I]),
    "pararnn_head_gru_backward": (_I, [_I64, _I64, _I64, _I, _I, _P, _P, _P, _P, _P, _P, _P, _P, _P, _SZ, _P]),
    "pararnn_head_gru_unroll": (_I, [_I64, _I64, _I64, _I, _I, _P, _P, _P, _P, _P, _SZ, _P]),
}

_lib = None


class PararnnError(RuntimeError):
    def __init__(self, status: int, where: str, detail: str = ""):
        self.status = status
        msg = "%s returned %s" % (where, STATUS.get(status, status))
        if detail:
            msg += ": " + detail
        super().__init__(msg)


def load(path: str | None = None):
    """Load (building first if missing or stale) the in-tree library."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    so = path or _build.build()
    if not os.path.exists(so):
        raise RuntimeError("libpararnn_b200.so not found at %s" % so)
    lib = ctypes.CDLL(so)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    if path is None:
        _lib = lib
    return lib


def _ptr(x):
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(s):
    if s is None:
        return None
    if isinstance(s, int):
        return s
    return s.cuda_stream


# ---- the C ABI, one to one -------------------------------------------------

def pararnn_num_gates(cell):
    return load().pararnn_num_gates(cell)


def pararnn_state_width(cell):
    return load().pararnn_state_width(cell)


def pararnn_workspace_bytes(cell, B, T, D, K):
    return load().pararnn_workspace_bytes(cell, B, T, D, K)


def pararnn_newton_forward(cell, B, T, D, px_dtype, preacts, diag_w, h0, K, H_out, workspace, ws_bytes,
                           resid_hist, stream):
    return load().pararnn_newton_forward(cell, B, T, D, px_dtype, _ptr(preacts), _ptr(diag_w), _ptr(h0), K,
                                         _ptr(H_out), _ptr(workspace), ws_bytes, _ptr(resid_hist), _stream(stream))


def pararnn_kstar(cell, T):
    return load().pararnn_kstar(cell, T)


def pararnn_newton_forward_picard(cell, B, T, D, px_dtype, preacts, diag_w, h0, picard_iters, K, H_out, workspace,
                                  ws_bytes, resid_hist, stream):
    return load().pararnn_newton_forward_picard(cell, B, T, D, px_dtype, _ptr(preacts), _ptr(diag_w), _ptr(h0),
                                                picard_iters, K, _ptr(H_out), _ptr(workspace), ws_bytes,
                                                _ptr(resid_hist), _stream(stream))


def pararnn_unroll(cell, B, T, D, px_dtype, preacts, diag_w, h0, H_out, workspace, ws_bytes, stream):
    return load().pararnn_unroll(cell, B, T, D, px_dtype, _ptr(preacts), _ptr(diag_w), _ptr(h0), _ptr(H_out),
                                 _ptr(workspace), ws_bytes, _stream(stream))


def pararnn_newton_backward(cell, B, T, D, px_dtype, preacts, diag_w, h0, H, dL_dH, dL_dpx, dL_da, dL_dh0,
                            workspace, ws_bytes, stream):
    return load().pararnn_newton_backward(cell, B, T, D, px_dtype, _ptr(preacts), _ptr(diag_w), _ptr(h0), _ptr(H),
                                          _ptr(dL_dH), _ptr(dL_dpx), _ptr(dL_da), _ptr(dL_dh0), _ptr(workspace),
                                          ws_bytes, _stream(stream))


def pararnn_status_sync(workspace, stream):
    return load().pararnn_status_sync(_ptr(workspace), _stream(stream))


def pararnn_status_string(status):
    return load().pararnn_status_string(status).decode()


def pararnn_last_error():
    return load().pararnn_last_error().decode()


def pararnn_probe_wait_timeout(workspace, ws_bytes, timeout_ns, stream):
    return load().pararnn_probe_wait_timeout(_ptr(workspace), ws_bytes, timeout_ns, _stream(stream))


def pararnn_debug_hooks(wait_limit_ns, stall_first_tile):
    return load().pararnn_debug_hooks(wait_limit_ns, int(stall_first_tile))


def pararnn_newton_forward_noalloc(cell, B, T, D, px_dtype, preacts, diag_w, h0, K, H_out, resid_hist, wait_status,
                                   stream):
    return load().pararnn_newton_forward_noalloc(cell, B, T, D, px_dtype, _ptr(preacts), _ptr(diag_w), _ptr(h0), K,
                                                 _ptr(H_out), _ptr(resid_hist), int(wait_status), _stream(stream))


def pararnn_newton_forward_host_workspace_bytes(cell, B, T, D, K, px_dtype, rows_per_slice, channels_per_slice=0):
    return load().pararnn_newton_forward_host_workspace_bytes(cell, B, T, D, K, px_dtype, rows_per_slice,
                                                              channels_per_slice)


def pararnn_newton_forward_host(cell, B, T, D, px_dtype, preacts_host, diag_w, h0, K, H_host, workspace, ws_bytes,
                                rows_per_slice, channels_per_slice, stream):
    return load().pararnn_newton_forward_host(cell, B, T, D, px_dtype, _ptr(preacts_host), _ptr(diag_w), _ptr(h0), K,
                                              _ptr(H_host), _ptr(workspace), ws_bytes, rows_per_slice,
                                              channels_per_slice, _stream(stream))


def pararnn_newton_step_host_workspace_bytes(cell, B, T, D, K, px_dtype, channels_per_slice=0):
    return load().pararnn_newton_step_host_workspace_bytes(cell, B, T, D, K, px_dtype, channels_per_slice)


def pararnn_newton_step_host(cell, B, T, D, px_dtype, preacts_host, diag_w, h0, K, dL_dH_host, H_host, dL_dpx_host,
                             dL_da, workspace, ws_bytes, channels_per_slice, stream):
    return load().pararnn_newton_step_host(cell, B, T, D, px_dtype, _ptr(preacts_host), _ptr(diag_w), _ptr(h0), K,
                                           _ptr(dL_dH_host), _ptr(H_host), _ptr(dL_dpx_host), _ptr(dL_da),
                                           _ptr(workspace), ws_bytes, channels_per_slice, _stream(stream))


def pararnn_head_gru_workspace_bytes(B, T, D, n_heads, K):
    return load().pararnn_head_gru_workspace_bytes(B, T, D, n_heads, K)


def pararnn_head_gru_forward(B, T, D, n_heads, px_dtype, preacts, U, h0, K, H_out, workspace, ws_bytes, resid_hist,
                             stream):
    return load().pararnn_head_gru_forward(B, T, D, n_heads, px_dtype, _ptr(preacts), _ptr(U), _ptr(h0), K,
                                           _ptr(H_out), _ptr(workspace), ws_bytes, _ptr(resid_hist),
                                           _stream(stream))


def pararnn_head_gru_backward_workspace_bytes(B, T, D, n_heads):
    return load().pararnn_head_gru_backward_workspace_bytes(B, T, D, n_heads)


def pararnn_head_gru_backward(B, T, D, n_heads, px_dtype, preacts, U, h0, H, dL_dH, dL_dpx, dL_dU, dL_dh0, workspace,
                              ws_bytes, stream):
    return load().pararnn_head_gru_backward(B, T, D, n_heads, px_dtype, _ptr(preacts), _ptr(U), _ptr(h0), _ptr(H),
                                            _ptr(dL_dH), _ptr(dL_dpx), _ptr(dL_dU), _ptr(dL_dh0), _ptr(workspace),
                                            ws_bytes, _stream(stream))


def pararnn_head_gru_unroll(B, T, D, n_heads, px_dtype, preacts, U, h0, H_out, workspace, ws_bytes, stream):
    return load().pararnn_head_gru_unroll(B, T, D, n_heads, px_dtype, _ptr(preacts), _ptr(U), _ptr(h0), _ptr(H_out),
                                          _ptr(workspace), ws_bytes, _stream(stream))


# ---- tensor-level helpers (allocation through torch, compute in the library) ----

def _check(status, where):
    if status != OK:
        raise PararnnError(status, where, pararnn_last_error())


def _dtype_code(t):
    import torch

    if t.dtype == torch.float32:
        return F32
    if t.dtype == torch.bfloat16:
        return BF16
    raise TypeError("pre-activations must be float32 or bfloat16, got %s" % t.dtype)


def _shape(cell, px):
    G = pararnn_num_gates(cell)
    if px.dim() != 4 or px.shape[2] != G:
        raise ValueError("preacts must be (B, T, %d, D), got %s" % (G, tuple(px.shape)))
    if not px.is_contiguous():
        raise ValueError("preacts must be contiguous")
    B, T, _, D = px.shape
    return B, T, D


def workspace_for(cell, B, T, D, K, device):
    """An uninitialised workspace: every call clears what it reads."""
    import torch

    n = pararnn_workspace_bytes(cell, B, T, D, K)
    return torch.empty(n, dtype=torch.uint8, device=device)


def newton_forward(cell, px, diag_w=None, h0=None, K=1, out=None, workspace=None, resid_hist=None, stream=None,
                   sync_status=True, picard_iters=0):
    """H = h^(K) of shape (B,T,S,D), float32, on px's device.  K=0 (or None)
    takes the measured K*(cell, T); picard_iters > 0 runs that many Picard
    sweeps before the Newton iterations."""
    import torch

    cell = CELLS.get(cell, cell)
    K = 0 if K is None else K
    B, T, D = _shape(cell, px)
    S = pararnn_state_width(cell)
    if out is None:
        out = torch.empty((B, T, S, D), dtype=torch.float32, device=px.device)
    if workspace is None:
        workspace = workspace_for(cell, B, T, D, K, px.device)
    st = stream if stream is not None else torch.cuda.current_stream(px.device)
    if picard_iters:
        _check(pararnn_newton_forward_picard(cell, B, T, D, _dtype_code(px), px, diag_w, h0, picard_iters, K, out,
                                             workspace, workspace.numel(), resid_hist, st),
               "pararnn_newton_forward_picard")
    else:
        _check(pararnn_newton_forward(cell, B, T, D, _dtype_code(px), px, diag_w, h0, K, out, workspace,
                                      workspace.numel(), resid_hist, st), "pararnn_newton_forward")
    if sync_status:
        _check(pararnn_status_sync(workspace, st), "pararnn_newton_forward (device status)")
    return out


def unroll(cell, px, diag_w=None, h0=None, out=None, workspace=None, stream=None, sync_status=True):
    """The sequential recurrence on the GPU: H (B,T,S,D) float32."""
    import torch

    cell = CELLS.get(cell, cell)
    B, T, D = _shape(cell, px)
    S = pararnn_state_width(cell)
    if out is None:
        out = torch.empty((B, T, S, D), dtype=torch.float32, device=px.device)
    if workspace is None:
        workspace = torch.empty(256, dtype=torch.uint8, device=px.device)
    st = stream if stream is not None else torch.cuda.current_stream(px.device)
    _check(pararnn_unroll(cell, B, T, D, _dtype_code(px), px, diag_w, h0, out, workspace, workspace.numel(), st),
           "pararnn_unroll")
    if sync_status:
        _check(pararnn_status_sync(workspace, st), "pararnn_unroll (device status)")
    return out


def newton_backward(cell, px, H, dL_dH, diag_w=None, h0=None, workspace=None, want_da=True, want_dh0=False,
                    stream=None, sync_status=True):
    """Returns (dL_dpx (B,T,G,D), dL_da (G,D) or None, dL_dh0 (B,S,D) or None), float32."""
    import torch

    cell = CELLS.get(cell, cell)
    B, T, D = _shape(cell, px)
    G, S = pararnn_num_gates(cell), pararnn_state_width(cell)
    dpx = torch.empty((B, T, G, D), dtype=torch.float32, device=px.device)
    da = torch.empty((G, D), dtype=torch.float32, device=px.device) if (want_da and cell != LINEAR) else None
    dh0 = torch.empty((B, S, D), dtype=torch.float32, device=px.device) if want_dh0 else None
    if workspace is None:
        workspace = workspace_for(cell, B, T, D, 1, px.device)
    st = stream if stream is not None else torch.cuda.current_stream(px.device)
    _check(pararnn_newton_backward(cell, B, T, D, _dtype_code(px), px, diag_w, h0, H, dL_dH, dpx, da, dh0,
                                   workspace, workspace.numel(), st), "pararnn_newton_backward")
    if sync_status:
        _check(pararnn_status_sync(workspace, st), "pararnn_newton_backward (device status)")
    return dpx, da, dh0


def head_gru_forward(px, U, h0=None, K=1, out=None, workspace=None, resid_hist=None, stream=None, sync_status=True):
    """Head-wise GRU: px (B,T,3,D), U (3, n_heads, d, d) -> H = h^(K) (B,T,D), float32."""
    import torch

    if px.dim() != 4 or px.shape[2] != 3 or not px.is_contiguous():
        raise ValueError("preacts must be contiguous (B, T, 3, D), got %s" % (tuple(px.shape),))
    if U.dim() != 4 or U.shape[0] != 3 or U.shape[2] != U.shape[3] or not U.is_contiguous():
        raise ValueError("U must be contiguous (3, n_heads, d, d), got %s" % (tuple(U.shape),))
    B, T, _, D = px.shape
    nh = U.shape[1]
    if out is None:
        out = torch.empty((B, T, D), dtype=torch.float32, device=px.device)
    if workspace is None:
        n = pararnn_head_gru_workspace_bytes(B, T, D, nh, K)
        if n == 0:
            raise PararnnError(EINVAL, "pararnn_head_gru_workspace_bytes", "invalid sizes")
        workspace = torch.empty(n, dtype=torch.uint8, device=px.device)
    st = stream if stream is not None else torch.cuda.current_stream(px.device)
    _check(pararnn_head_gru_forward(B, T, D, nh, _dtype_code(px), px, U, h0, K, out, workspace, workspace.numel(),
                                    resid_hist, st), "pararnn_head_gru_forward")
    if sync_status:
        _check(pararnn_status_sync(workspace, st), "pararnn_head_gru_forward (device status)")
    return out


def head_gru_backward(px, U, H, dL_dH, h0=None, want_dU=True, want_dh0=False, workspace=None, stream=None,
                      sync_status=True):
    """Head-wise GRU adjoint: returns (dL/dpx (B,T,3,D), dL/dU (3,n_heads,d,d) or None, dL/dh0 (B,D) or None)."""
    import torch

    B, T, _, D = px.shape
    nh = U.shape[1]
    dpx = torch.empty((B, T, 3, D), dtype=torch.float32, device=px.device)
    dU = torch.empty(tuple(U.shape), dtype=torch.float32, device=px.device) if want_dU else None
    dh0 = torch.empty((B, D), dtype=torch.float32, device=px.device) if want_dh0 else None
    if workspace is None:
        n = pararnn_head_gru_backward_workspace_bytes(B, T, D, nh)
        if n == 0:
            raise PararnnError(EINVAL, "pararnn_head_gru_backward_workspace_bytes", "invalid sizes")
        workspace = torch.empty(n, dtype=torch.uint8, device=px.device)
    st = stream if stream is not None else torch.cuda.current_stream(px.device)
    _check(pararnn_head_gru_backward(B, T, D, nh, _dtype_code(px), px, U, h0, H, dL_dH, dpx, dU, dh0, workspace,
                                     workspace.numel(), st), "pararnn_head_gru_backward")
    if sync_status:
        _check(pararnn_status_sync(workspace, st), "pararnn_head_gru_backward (device status)")
    return dpx, dU, dh0


def head_gru_unroll(px, U, h0=None, out=None, workspace=None, stream=None, sync_status=True):
    """Head-wise GRU, sequential unroll on the GPU: px (B,T,3,D), U (3,n_heads,d,d) -> H (B,T,D), float32."""
    import torch

    if px.dim() != 4 or px.shape[2] != 3 or not px.is_contiguous():
        raise ValueError("preacts must be contiguous (B, T, 3, D), got %s" % (tuple(px.shape),))
    B, T, _, D = px.shape
    nh = U.shape[1]
    if out is None:
        out = torch.empty((B, T, D), dtype=torch.float32, device=px.device)
    if workspace is None:
        workspace = torch.empty(256, dtype=torch.uint8, device=px.device)
    st = stream if stream is not None else torch.cuda.current_stream(px.device)
    _check(pararnn_head_gru_unroll(B, T, D, nh, _dtype_code(px), px, U, h0, out, workspace, workspace.numel(), st),
           "pararnn_head_gru_unroll")
    if sync_status:
        _check(pararnn_status_sync(workspace, st), "pararnn_head_gru_unroll (device status)")
    return out


def newton_forward_host(cell, px_host, diag_w=None, h0=None, K=1, out_host=None, rows_per_slice=1,
                        channels_per_slice=0, workspace=None, stream=None, sync_status=True):
    """The forward on host tensors (pinned for overlap): H (B,T,S,D) float32 on the host."""
    import torch

    cell = CELLS.get(cell, cell)
    B, T, D = _shape(cell, px_host)
    S = pararnn_state_width(cell)
    code = _dtype_code(px_host)
    if out_host is None:
        out_host = torch.empty((B, T, S, D), dtype=torch.float32, pin_memory=px_host.is_pinned())
    dev = diag_w.device if diag_w is not None else torch.device("cuda", torch.cuda.current_device())
    if workspace is None:
        n = pararnn_newton_forward_host_workspace_bytes(cell, B, T, D, K, code, rows_per_slice, channels_per_slice)
        if n == 0:
            raise PararnnError(EINVAL, "pararnn_newton_forward_host_workspace_bytes", "invalid arguments")
        workspace = torch.zeros(n, dtype=torch.uint8, device=dev)
    st = stream if stream is not None else torch.cuda.current_stream(dev)
    _check(pararnn_newton_forward_host(cell, B, T, D, code, px_host, diag_w, h0, K, out_host, workspace,
                                       workspace.numel(), rows_per_slice, channels_per_slice, st),
           "pararnn_newton_forward_host")
    if sync_status:
        _check(pararnn_status_sync(workspace, st), "pararnn_newton_forward_host (device status)")
    return out_host


def newton_step_host(cell, px_host, dL_dH_host, diag_w=None, h0=None, K=1, channels_per_slice=0, outs=None,
                     workspace=None, stream=None, sync_status=True):
    """Forward + adjoint on host tensors (pinned for overlap): returns
    (H, dL/dpx) on the host and dL/da (G, D) on the device (None for the
    linear cell)."""
    import torch

    cell = CELLS.get(cell, cell)
    B, T, D = _shape(cell, px_host)
    S, G = pararnn_state_width(cell), pararnn_num_gates(cell)
    code = _dtype_code(px_host)
    dev = diag_w.device if diag_w is not None else torch.device("cuda", torch.cuda.current_device())
    if outs is None:
        pin = px_host.is_pinned()
        outs = (torch.empty((B, T, S, D), dtype=torch.float32, pin_memory=pin),
                torch.empty((B, T, G, D), dtype=torch.float32, pin_memory=pin),
                None if cell == LINEAR else torch.empty((G, D), dtype=torch.float32, device=dev))
    H_host, dpx_host, da = outs
    if workspace is None:
        n = pararnn_newton_step_host_workspace_bytes(cell, B, T, D, K, code, channels_per_slice)
        if n == 0:
            raise PararnnError(EINVAL, "pararnn_newton_step_host_workspace_bytes", "invalid arguments")
        workspace = torch.empty(n, dtype=torch.uint8, device=dev)
    st = stream if stream is not None else torch.cuda.current_stream(dev)
    _check(pararnn_newton_step_host(cell, B, T, D, code, px_host, diag_w, h0, K, dL_dH_host, H_host, dpx_host, da,
                                    workspace, workspace.numel(), channels_per_slice, st),
           "pararnn_newton_step_host")
    if sync_status:
        _check(pararnn_status_sync(workspace, st), "pararnn_newton_step_host (device status)")
    return H_host, dpx_host, da
