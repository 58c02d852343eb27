"""Helpers for the GPU parity tests: the error metric and oracle runs on
channel samples.  Parity is always GPU (through the C ABI) vs the fp64 oracle
on the same seeded inputs."""
import numpy as np
import torch

import oracle


def rel_err(got, ref, floor_frac=1e-2):
    """max_i |g_i - o_i| / max(|o_i|, floor_frac * max|o|): a relative error
    whose floor keeps near-zero entries from dominating."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    if ref.size == 0:
        return 0.0
    if not np.all(np.isfinite(got)):
        return float("inf")
    scale = np.maximum(np.abs(ref), floor_frac * max(float(np.max(np.abs(ref))), 1e-30))
    return float(np.max(np.abs(got - ref) / scale))


def norm_err(got, ref):
    """max_i |g_i - o_i| / max_i |o_i|: the normwise relative error.  Used for
    bf16 pre-activations against the unrounded f32 draws, where rounding the
    inputs to 8 significant bits moves every output by an amount set by the
    input perturbation, not by the output's own size, so an element-wise
    relative error near zero crossings measures the rounding, not the solver
    (the fp64 oracle fed the same two inputs shows the same element-wise gap)."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    if ref.size == 0:
        return 0.0
    if not np.all(np.isfinite(got)):
        return float("inf")
    return float(np.max(np.abs(got - ref)) / max(float(np.max(np.abs(ref))), 1e-30))


def to_np(t):
    return None if t is None else t.detach().float().cpu().numpy().astype(np.float64)


def gather_channels(t, chans):
    """(B,T,X,D) tensor -> (T,X,n) numpy for the listed (b, d) channels."""
    bs = torch.tensor([b for b, _ in chans], device=t.device)
    ds = torch.tensor([d for _, d in chans], device=t.device)
    sub = t[bs, :, :, ds]  # (n, T, X)
    return to_np(sub).transpose(1, 2, 0)
