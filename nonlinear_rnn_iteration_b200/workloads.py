"""Seeded synthetic workloads: shapes, Newton budgets and input distributions.

This module only draws random inputs.  It holds none of the method's
arithmetic, and it is the one piece shared by the CUDA path's callers and by
the oracle's callers, so that both read identical buffers.

Workloads (named by what they are and their sizes):

========================  ======  ====  =======  =====  ===  ===============
name                      cell    B     T        D      K    pre-activations
========================  ======  ====  =======  =====  ===  ===============
gru_1x1024x64_k3          GRU     1     1024     64     3    f32
linear_8x16384x1024       linear  8     16384    1024   1    f32
gru_8x4096x2048_k3        GRU     8     4096     2048   3    f32
gru_8x4096x2048_k3_bf16   GRU     8     4096     2048   3    bf16 (f32 state)
lstm_4x32768x1024_k4      LSTM    4     32768    1024   4    f32, + backward
gru_1x131072x4096_k2_bf16 GRU     1     131072   4096   2    bf16, + backward
========================  ======  ====  =======  =====  ===  ===============

Head-wise GRU (block-diagonal recurrent weights, ParaGRU(mix='head')):

===========================  ====  ====  ===  =======  ===  ===  ====
name                         B     T     D    n_heads  d    K    px
===========================  ====  ====  ===  =======  ===  ===  ====
headgru_8x4096x512_h8_k3     8     4096  512  8        64   3    f32
===========================  ====  ====  ===  =======  ===  ===  ====

with px ~ N(0,1), recurrent blocks U_g ~ U(-1, 1) / sqrt(d) entrywise (so
that U_g s stays O(1)), h0 = 0; draw order px, U; seed 5.

Distributions: GRU / LSTM pre-activations px ~ N(0,1), diagonal recurrent
weights a ~ U(-0.5, 0.5) per gate and channel, initial state h0 = 0.  Linear:
decay a_t = sigmoid(N(0,1)) in gate slot 0 and input b_t ~ N(0,1) in slot 1.
Upstream gradient dL/dH ~ N(0,1).  bf16 pre-activations are the f32 draws
rounded to nearest-even.  Draw order: px, a, dL/dH.  Seed = the workload's
index in the table above.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

CELL_IDS = {"linear": 0, "diag_gru": 1, "diag_lstm": 2}
NUM_GATES = {"linear": 2, "diag_gru": 3, "diag_lstm": 4}
STATE_WIDTH = {"linear": 1, "diag_gru": 1, "diag_lstm": 2}


@dataclass(frozen=True)
class Workload:
    name: str
    cell: str
    B: int
    T: int
    D: int
    K: int
    px_dtype: str  # "f32" or "bf16"
    seed: int
    backward: bool = False

    @property
    def G(self) -> int:
        return NUM_GATES[self.cell]

    @property
    def S(self) -> int:
        return STATE_WIDTH[self.cell]

    @property
    def cell_id(self) -> int:
        return CELL_IDS[self.cell]

    @property
    def elements(self) -> int:
        return self.B * self.T * self.D

    def with_shape(self, B=None, T=None, D=None, K=None, name=None):
        return Workload(name or self.name, self.cell, B or self.B, T or self.T, D or self.D,
                        K or self.K, self.px_dtype, self.seed, self.backward)


WORKLOADS = {
    w.name: w
    for w in [
        Workload("gru_1x1024x64_k3", "diag_gru", 1, 1024, 64, 3, "f32", 0),
        Workload("linear_8x16384x1024", "linear", 8, 16384, 1024, 1, "f32", 1),
        Workload("gru_8x4096x2048_k3", "diag_gru", 8, 4096, 2048, 3, "f32", 2),
        Workload("gru_8x4096x2048_k3_bf16", "diag_gru", 8, 4096, 2048, 3, "bf16", 2),
        Workload("lstm_4x32768x1024_k4", "diag_lstm", 4, 32768, 1024, 4, "f32", 3, backward=True),
        Workload("gru_1x131072x4096_k2_bf16", "diag_gru", 1, 131072, 4096, 2, "bf16", 4, backward=True),
    ]
}

HEADLINE = "gru_1x131072x4096_k2_bf16"


# --------------------------------------------------------------------------
# host (numpy) draws: used for sizes the oracle handles whole
# --------------------------------------------------------------------------

def host_inputs(w: Workload, seed: int | None = None, with_grad: bool = False) -> dict:
    """Draw a workload's inputs on the host (numpy PCG64).

    Returns float32 arrays: ``px`` (B,T,G,D), ``a`` (G,D) or None for the
    linear cell, ``h0`` None (zero initial state), and ``dLdH`` (B,T,S,D)
    when ``with_grad``.  For bf16 workloads ``px`` holds the f32 draws; the
    caller rounds them (see :func:`round_bf16`).
    """
    rng = np.random.Generator(np.random.PCG64(w.seed if seed is None else seed))
    shape = (w.B, w.T, w.G, w.D)
    if w.cell == "linear":
        px = np.empty(shape, dtype=np.float32)
        px[:, :, 0, :] = 1.0 / (1.0 + np.exp(-rng.standard_normal((w.B, w.T, w.D))))
        px[:, :, 1, :] = rng.standard_normal((w.B, w.T, w.D))
        a = None
    else:
        px = rng.standard_normal(shape, dtype=np.float32)
        a = rng.uniform(-0.5, 0.5, size=(w.G, w.D)).astype(np.float32)
    out = {"px": px, "a": a, "h0": None}
    if with_grad:
        out["dLdH"] = rng.standard_normal((w.B, w.T, w.S, w.D), dtype=np.float32)
    return out


def round_bf16(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16 (nearest-even), returned as float32."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    r = ((u + 0x7FFF + lsb) >> 16) << 16
    nan = np.isnan(x)
    out = r.astype(np.uint32).view(np.float32).copy()
    out[nan] = np.nan
    return out


# --------------------------------------------------------------------------
# device (torch) draws: used at full size, where a host draw would be slow
# --------------------------------------------------------------------------

def device_inputs(w: Workload, device, seed: int | None = None, with_grad: bool = False) -> dict:
    """Draw a workload's inputs directly in device memory (torch generator).

    Returns torch tensors: ``px32`` (B,T,G,D) float32 draws, ``px`` in the
    workload's dtype (bf16 rounding of ``px32`` or ``px32`` itself), ``a``
    (G,D) float32 or None, ``h0`` None, and ``dLdH`` when ``with_grad``.
    """
    import torch

    g = torch.Generator(device=device)
    g.manual_seed(w.seed if seed is None else seed)
    shape = (w.B, w.T, w.G, w.D)
    if w.cell == "linear":
        px32 = torch.empty(shape, dtype=torch.float32, device=device)
        px32[:, :, 0, :] = torch.sigmoid(torch.randn((w.B, w.T, w.D), generator=g, device=device))
        px32[:, :, 1, :] = torch.randn((w.B, w.T, w.D), generator=g, device=device)
        a = None
    else:
        px32 = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
        a = torch.rand((w.G, w.D), generator=g, device=device, dtype=torch.float32) - 0.5
    px = px32.to(torch.bfloat16) if w.px_dtype == "bf16" else px32
    out = {"px32": px32, "px": px, "a": a, "h0": None}
    if with_grad:
        out["dLdH"] = torch.randn((w.B, w.T, w.S, w.D), generator=g, device=device, dtype=torch.float32)
    return out


def sample_channels(w: Workload, n: int, seed: int = 12345):
    """A seeded sample of n distinct (b, d) channels, sorted."""
    rng = np.random.Generator(np.random.PCG64(seed))
    n = min(n, w.B * w.D)
    flat = np.sort(rng.choice(w.B * w.D, size=n, replace=False))
    return [(int(c // w.D), int(c % w.D)) for c in flat]


# --------------------------------------------------------------------------
# head-wise GRU (block-diagonal recurrent weights)
# --------------------------------------------------------------------------

@dataclass(frozen=True)
class HeadWorkload:
    name: str
    B: int
    T: int
    D: int
    n_heads: int
    K: int
    px_dtype: str
    seed: int

    @property
    def d(self) -> int:
        return self.D // self.n_heads

    @property
    def elements(self) -> int:
        return self.B * self.T * self.D


HEAD_WORKLOADS = {
    w.name: w
    for w in [
        HeadWorkload("headgru_8x4096x512_h8_k3", 8, 4096, 512, 8, 3, "f32", 5),
    ]
}


def head_host_inputs(B: int, T: int, D: int, n_heads: int, seed: int) -> dict:
    """px (B,T,3,D) ~ N(0,1) and U (3, n_heads, d, d) ~ U(-1,1)/sqrt(d), float32."""
    rng = np.random.Generator(np.random.PCG64(seed))
    d = D // n_heads
    px = rng.standard_normal((B, T, 3, D), dtype=np.float32)
    U = (rng.uniform(-1.0, 1.0, size=(3, n_heads, d, d)) / np.sqrt(d)).astype(np.float32)
    return {"px": px, "U": U, "h0": None}


def head_device_inputs(w: HeadWorkload, device, seed: int | None = None) -> dict:
    """The same distributions drawn in device memory (torch generator)."""
    import torch

    g = torch.Generator(device=device)
    g.manual_seed(w.seed if seed is None else seed)
    px32 = torch.randn((w.B, w.T, 3, w.D), generator=g, device=device, dtype=torch.float32)
    U = (torch.rand((3, w.n_heads, w.d, w.d), generator=g, device=device, dtype=torch.float32) * 2.0 - 1.0) / float(
        np.sqrt(w.d))
    px = px32.to(torch.bfloat16) if w.px_dtype == "bf16" else px32
    return {"px32": px32, "px": px, "U": U, "h0": None}
