"""Benchmark: Newton-solve B*T*D elements per second on B200, through the C ABI.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl native|reference]
                    [--workload NAME] [--no-extra]

A step is one pass of the hot path over one batch of the workload: one
``pararnn_newton_forward`` call (all K Newton iterations; the linear workload
is one exact scan), plus ``pararnn_newton_backward`` for workloads that carry
a backward pass.  The default workload is the largest: the long-sequence
diagonal GRU (B=1, T=131072, D=4096, K=2, bf16 pre-activations with float32
state), forward and adjoint in every step.  Inputs are resident in HBM before timing and are larger
than L2, so no flush is needed between steps.  The device time of the K
timed steps is measured with CUDA events on the launching stream between a
barrier and a synchronize on both sides; with N > 1 processes (one per GPU,
launched by torchrun) each rank solves its own independent problem of the
full workload size (channels never interact), the time is the max over ranks,
and ``value`` counts the elements of all ranks (weak scaling).

``--impl reference`` times the fp64 CPU oracle -- the slow, obviously correct
program every GPU result is checked against -- on a bounded sample of the same
workload on this machine's host cores (rank 0 only).
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "Newton-solve B·T·D elements/sec at K iters; achieved HBM GB/s vs B200 peak"
UNIT = "elem/s"

# HBM bytes per (b,t,d) element for one call, two ways.
#
# Fused minimum (what these kernels move): every pre-activation read once,
# every output written once; the Newton iterate never leaves the chip between
# iterations.
#   linear f32 fwd: a, b read (8) + h written (4)                         = 12
#   GRU fwd: px read (3 x 4 f32 | 3 x 2 bf16) + h written (4)            = 16 | 10
#   LSTM fwd f32: px read (4 x 4) + (c, h) written (8)                    = 24
#   GRU bwd: px (3 x 4 | 3 x 2) + H (4) + dL/dH (4) read, dL/dpx (3 x 4) written
#                                                                        = 32 | 26
# Streaming design (one HBM pass per Newton iteration, the method's plain
# form): the first iteration reads px and writes the state, each later one
# reads px and the state and writes the state; the backward moves the same
# bytes in both designs.  This is the figure the HBM roofline fraction is
# taken on.
ALGO_BYTES = {
    ("linear", "f32", "fwd"): 12, ("diag_gru", "f32", "fwd"): 16, ("diag_gru", "bf16", "fwd"): 10,
    ("diag_lstm", "f32", "fwd"): 24, ("diag_lstm", "bf16", "fwd"): 16,
    ("linear", "f32", "bwd"): 24, ("diag_gru", "f32", "bwd"): 32, ("diag_gru", "bf16", "bwd"): 26,
    ("diag_lstm", "f32", "bwd"): 48, ("diag_lstm", "bf16", "bwd"): 40,
}
PX_BYTES = {"f32": 4, "bf16": 2}
# nominal B200 HBM3e bandwidth, reported beside the measured copy bandwidth
NOMINAL_HBM_GBS = 8000.0


def streaming_bytes_per_elem(w, direction):
    """Bytes per element of the streaming design (see above)."""
    if direction == "bwd" or w.cell == "linear":
        return ALGO_BYTES[(w.cell, w.px_dtype, direction)]
    px = w.G * PX_BYTES[w.px_dtype]
    state = 4 * w.S
    return (px + state) + (px + 2 * state) * (w.K - 1)
# channels per slice of the host-buffer pipeline in the e2e measurement:
# 8 x 1024 channels in slices of 256 make 32 slices, whose shorter fill and
# drain beat whole rows (8 slices)
E2E_CHANNELS = 256
# channels per slice of the forward + adjoint host-buffer pipeline: each
# slice holds all B rows.  Measured on the long-sequence GRU (1 x 131072 x
# 4096): 128 channels 285 ms, 256: 224, 512: 199, 1024: 186, 2048: 214, one
# slice 254 ms.  Narrow slices of a long sequence leave few channel groups,
# each with a long chain of tiles, and the solver becomes the bottleneck;
# wide ones lengthen the pipeline's fill and drain.
E2E_STEP_CHANNELS = 1024

KERNEL_SOURCES = ["newton_fwd.cuh", "adjoint_bwd.cuh", "lookback.cuh", "cells.cuh", "common.cuh", "tma.cuh", "pararnn_abi.cu"]


# --------------------------------------------------------------------------
# distributed plumbing (host only; testable with gloo on CPU)
# --------------------------------------------------------------------------

def dist_env():
    return int(os.environ.get("RANK", "0")), int(os.environ.get("LOCAL_RANK", "0")), int(os.environ.get("WORLD_SIZE", "1"))


def dist_init(backend, world):
    import torch.distributed as dist

    if world > 1 and not dist.is_initialized():
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))
    return dist if world > 1 else None


def barrier(dist, device=None):
    if dist is not None:
        if device is not None and dist.get_backend() == "nccl":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


def reduce_max(dist, value, device):
    """Max of a float over ranks (the timing rule: the slowest rank counts)."""
    if dist is None:
        return value
    import torch

    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def rank_seed(base_seed, rank):
    """Each rank draws an independent problem of the full workload size."""
    return base_seed + 1000 * rank


def aggregate_throughput(elements_per_rank, world, steps, max_ms):
    """Whole-job units/s: every rank's elements over the slowest rank's time."""
    return elements_per_rank * world * steps / (max_ms / 1e3)


# --------------------------------------------------------------------------
# measurement helpers
# --------------------------------------------------------------------------

def kernel_source_hash():
    h = hashlib.sha256()
    for name in KERNEL_SOURCES:
        with open(os.path.join(ROOT, "nonlinear_rnn_iteration_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p.get("bf16_tflops", 1590.0)),
                "source": "of measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "source": "of fallback"}


# TF32 / BF16 dense tensor throughput, nominal (1.1 / 2.25 PFLOP/s on B200):
# the head-wise products run in TF32, so their peak is the measured bf16
# figure scaled by this ratio
TF32_PER_BF16 = 1.1 / 2.25


def time_head(w, device, steps, warmup):
    """Device times of one head-wise GRU forward call and one adjoint call at
    its output (CUDA events on the launching stream); returns
    (forward ms, backward ms, status name)."""
    import torch

    from nonlinear_rnn_iteration_b200 import binding, workloads

    x = workloads.head_device_inputs(w, device)
    H = torch.empty((w.B, w.T, w.D), device=device)
    n = binding.pararnn_head_gru_workspace_bytes(w.B, w.T, w.D, w.n_heads, w.K)
    ws = torch.empty(n, dtype=torch.uint8, device=device)
    nb = binding.pararnn_head_gru_backward_workspace_bytes(w.B, w.T, w.D, w.n_heads)
    wsb = torch.empty(nb, dtype=torch.uint8, device=device)
    g = torch.randn((w.B, w.T, w.D), device=device, generator=torch.Generator(device=device).manual_seed(w.seed + 100))
    stream = torch.cuda.current_stream(device)

    def fwd():
        binding.head_gru_forward(x["px"], x["U"], None, K=w.K, out=H, workspace=ws, stream=stream,
                                 sync_status=False)

    def bwd():
        binding.head_gru_backward(x["px"], x["U"], H, g, workspace=wsb, stream=stream, sync_status=False)

    Hu = torch.empty_like(H)
    wsu = torch.empty(256, dtype=torch.uint8, device=device)

    def unroll():
        binding.head_gru_unroll(x["px"], x["U"], None, out=Hu, workspace=wsu, stream=stream, sync_status=False)

    times = []
    for f in (fwd, bwd, unroll):
        for _ in range(warmup):
            f()
        torch.cuda.synchronize(device)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(steps):
            f()
        e1.record(stream)
        torch.cuda.synchronize(device)
        times.append(e0.elapsed_time(e1) / steps)
    st = binding.pararnn_status_sync(ws, stream)
    if st == binding.OK:
        st = binding.pararnn_status_sync(wsb, stream)
    if st == binding.OK:
        st = binding.pararnn_status_sync(wsu, stream)
    del x, H, Hu, ws, wsb, wsu, g
    torch.cuda.empty_cache()
    return times[0], times[1], binding.STATUS.get(st, st), times[2]


def head_line(w, ms, bwd_ms, status, unroll_ms=None):
    """A head-wise forward's line: time, elements/s, and the FLOP rate of its
    Jacobian products -- 2 d^3 useful FLOP per step and (batch row, head),
    issued as three TF32 products -- against the TF32 tensor peak; beside it
    the sequential unroll on the GPU (pararnn_head_gru_unroll) of the same
    problem."""
    peaks = measured_peaks()
    useful = 2.0 * w.d ** 3 * w.B * w.T * w.n_heads * w.K
    tf32_peak = peaks["bf16_tflops"] * TF32_PER_BF16
    extra = {}
    if unroll_ms is not None:
        extra = {"unroll_ms": round(unroll_ms, 4), "unroll_elem_per_s": w.elements / (unroll_ms / 1e3)}
    return {"ms_per_step": round(ms, 4), "elem_per_s": w.elements / (ms / 1e3), "K": w.K,
            "n_heads": w.n_heads, "d": w.d, "status": status, "bwd_ms": round(bwd_ms, 4),
            "bwd_elem_per_s": w.elements / (bwd_ms / 1e3), **extra,
            "roofline": {"bound": "tensor", "kernel": "head_chunk_tc_kernel (Jacobian products, tcgen05 TF32)",
                         "achieved_useful": round(useful / (ms / 1e3) / 1e12, 2),
                         "achieved_issued": round(3 * useful / (ms / 1e3) / 1e12, 2),
                         "peak": round(tf32_peak, 1), "peak_source": peaks["source"] + " (bf16 x TF32 ratio)",
                         "unit": "TFLOP/s", "frac_issued": round(3 * useful / (ms / 1e3) / 1e12 / tf32_peak, 4)}}


def head_workloads(device):
    """Device-time lines for the head-wise GRU workloads."""
    from nonlinear_rnn_iteration_b200 import workloads

    out = {}
    for name, w in workloads.HEAD_WORKLOADS.items():
        ms, bms, status, ums = time_head(w, device, steps=5, warmup=3)
        out[name] = head_line(w, ms, bms, status, ums)
    return out


def recorded_traffic(kernel, w):
    """DRAM bytes per launch of `kernel` on workload `w` from the committed
    ncu records (profiles/traffic.json), if they were taken on the current
    kernel sources; else None.  A record taken on a shorter sequence of the
    same workload (every tile moves the same bytes) is scaled to the full
    launch by the ratio of elements."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        rec = json.load(f)
    for key, e in rec.items():
        if key != "%s/%s" % (kernel, w.name) and not key.startswith("%s/%s@" % (kernel, w.name)):
            continue
        if e.get("kernel_source_hash") != kernel_source_hash():
            continue
        n = e.get("elements", w.elements)
        return {"dram_bytes_per_launch": int(round(e["dram_bytes_per_launch"] * w.elements / n)),
                "captured_on": key, "scaled_by": round(w.elements / n, 3)}
    return None


def kernel_roofline(w, direction, ms, peaks):
    """The HBM roofline record of one kernel launch on workload `w`."""
    kernel = "newton_fwd_kernel" if direction == "fwd" else "adjoint_bwd_kernel"
    sb = streaming_bytes_per_elem(w, direction) * w.elements
    fb = ALGO_BYTES[(w.cell, w.px_dtype, direction)] * w.elements
    achieved = sb / (ms / 1e3) / 1e9
    tr = recorded_traffic(kernel, w)
    return {"bound": "hbm", "kernel": kernel, "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"],
            "peak_source": peaks["source"], "unit": "GB/s", "frac": round(achieved / peaks["hbm_gbs"], 4),
            "frac_of_nominal_8tbs": round(achieved / NOMINAL_HBM_GBS, 4),
            "traffic": None if tr is None else tr["dram_bytes_per_launch"],
            "traffic_record": tr,
            "bytes_per_elem": sb // w.elements, "bytes_model": "streaming design (one HBM pass per iteration)",
            "fused_bytes_per_elem": fb // w.elements,
            "fused_achieved": round(fb / (ms / 1e3) / 1e9, 1),
            "algorithmic_bytes_per_launch": sb, "launch_ms": round(ms, 4)}


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled during the timed region."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(prefix="clocks_", suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), "--query-gpu=" + self.QUERY,
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.2)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        rows = []
        if self.path and os.path.exists(self.path):
            for line in open(self.path):
                f = [x.strip() for x in line.split(",")]
                if len(f) >= 9:
                    try:
                        rows.append((float(f[1]), float(f[2]), float(f[3]), f[4], f[5], f[6], f[7], f[8]))
                    except ValueError:
                        pass
            os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}
        loaded = [r for r in rows if r[2] > 200.0] or rows
        sm = sorted(r[0] for r in loaded)
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in loaded for i in range(4) if r[4 + i].lower() == "active"})
        return {"sm_mhz": sm[len(sm) // 2], "sm_max_mhz": max(r[1] for r in rows), "reasons": reasons,
                "samples": len(rows)}


# --------------------------------------------------------------------------
# the native arm
# --------------------------------------------------------------------------

class Problem:
    """One workload's device buffers and its C-ABI step."""

    def __init__(self, w, device, seed):
        import torch

        from nonlinear_rnn_iteration_b200 import binding, workloads

        self.w, self.dev, self.b = w, device, binding
        x = workloads.device_inputs(w, device, seed=seed, with_grad=w.backward)
        self.px, self.a = x["px"], x["a"]
        self.g = x.get("dLdH")
        del x
        self.H = torch.empty((w.B, w.T, w.S, w.D), dtype=torch.float32, device=device)
        self.ws = binding.workspace_for(w.cell_id, w.B, w.T, w.D, w.K, device)
        if w.backward:
            self.dpx = torch.empty((w.B, w.T, w.G, w.D), dtype=torch.float32, device=device)
            self.da = torch.empty((w.G, w.D), dtype=torch.float32, device=device)
        self.code = binding.BF16 if w.px_dtype == "bf16" else binding.F32
        self.stream = torch.cuda.current_stream(device)
        # the C entry points with their arguments resolved once (device
        # addresses and the stream handle), called as a C caller would call
        # them: the per-call cost is the library's, not Python's
        lib = binding.load()
        ptr = lambda t: None if t is None else t.data_ptr()
        self._fwd = lib.pararnn_newton_forward
        self._fwd_args = (w.cell_id, w.B, w.T, w.D, self.code, ptr(self.px), ptr(self.a), None, w.K, ptr(self.H),
                          ptr(self.ws), self.ws.numel(), None, self.stream.cuda_stream)
        if w.backward:
            self._bwd = lib.pararnn_newton_backward
            self._bwd_args = (w.cell_id, w.B, w.T, w.D, self.code, ptr(self.px), ptr(self.a), None, ptr(self.H),
                              ptr(self.g), ptr(self.dpx), ptr(self.da), None, ptr(self.ws), self.ws.numel(),
                              self.stream.cuda_stream)

    def forward(self, px=None, H=None):
        w = self.w
        if px is None and H is None:
            st = self._fwd(*self._fwd_args)
        else:
            st = self.b.pararnn_newton_forward(w.cell_id, w.B, w.T, w.D, self.code, self.px if px is None else px,
                                               self.a, None, w.K, self.H if H is None else H, self.ws,
                                               self.ws.numel(), None, self.stream)
        if st != 0:
            raise RuntimeError("forward: %s %s" % (self.b.STATUS[st], self.b.pararnn_last_error()))

    def backward(self):
        st = self._bwd(*self._bwd_args)
        if st != 0:
            raise RuntimeError("backward: %s %s" % (self.b.STATUS[st], self.b.pararnn_last_error()))

    def unroll(self):
        """The sequential recurrence on the GPU (pararnn_unroll) over the same
        inputs, for the Newton-vs-sequential comparison."""
        import torch

        w = self.w
        if not hasattr(self, "ws_unroll"):
            self.ws_unroll = torch.empty(256, dtype=torch.uint8, device=self.dev)
        st = self.b.pararnn_unroll(w.cell_id, w.B, w.T, w.D, self.code, self.px, self.a, None, self.H,
                                   self.ws_unroll, 256, self.stream)
        if st != 0:
            raise RuntimeError("unroll: %s %s" % (self.b.STATUS[st], self.b.pararnn_last_error()))

    def step(self):
        self.forward()
        if self.w.backward:
            self.backward()

    def launches_per_step(self):
        return 1 + (2 if self.w.backward else 0)

    def check_status(self):
        st = self.b.pararnn_status_sync(self.ws, self.stream)
        if st != 0:
            raise RuntimeError("device status %s" % self.b.STATUS[st])


def time_device(prob, steps, warmup, dist, device):
    """Returns (ms_per_step max over ranks, fwd_ms, bwd_ms) with CUDA events.

    The step time is the contract's: `steps` whole steps back to back between
    two events, bracketed by a barrier and a synchronize.  The per-kernel
    times come from separate passes of `steps` forward calls, then `steps`
    backward calls, back to back between two events each (no event between
    calls, so that on a small problem the host's enqueueing of the next call
    overlaps the device's work on the last)."""
    import torch

    for _ in range(warmup):
        prob.step()
    prob.check_status()
    barrier(dist, device)
    torch.cuda.synchronize(device)

    def timed(fn):
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record(prob.stream)
        for _ in range(steps):
            fn()
        t1.record(prob.stream)
        torch.cuda.synchronize(device)
        return t0.elapsed_time(t1)

    total = timed(prob.step)
    barrier(dist, device)
    prob.check_status()
    fwd = timed(prob.forward) / steps
    bwd = timed(prob.backward) / steps if prob.w.backward else 0.0
    torch.cuda.synchronize(device)
    prob.check_status()
    return reduce_max(dist, total, device) / steps, fwd, bwd


def time_graph(prob, steps=50, replays=4):
    """Device time per forward call with the calls replayed from a CUDA graph
    (captured once on a side stream): the kernel's own time without the
    per-launch overhead, for launch-bound (small) problems."""
    import torch

    side = torch.cuda.Stream(prob.dev)
    args = list(prob._fwd_args)
    args[-1] = side.cuda_stream
    side.wait_stream(prob.stream)
    with torch.cuda.stream(side):
        for _ in range(3):
            prob._fwd(*args)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=side):
        for _ in range(steps):
            prob._fwd(*args)
    # a graph replays on the current stream: replay and time on the side stream
    with torch.cuda.stream(side):
        g.replay()
        torch.cuda.synchronize()
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record(side)
        for _ in range(replays):
            g.replay()
        t1.record(side)
    torch.cuda.synchronize()
    del g
    prob.check_status()
    return t0.elapsed_time(t1) / (steps * replays)


def time_unroll(prob, steps=3):
    """Device time of the sequential recurrence on the GPU (CUDA events, calls
    back to back); the forward's H buffer is reused as its output."""
    import torch

    prob.unroll()
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(prob.stream)
    for _ in range(steps):
        prob.unroll()
    t1.record(prob.stream)
    torch.cuda.synchronize()
    st = prob.b.pararnn_status_sync(prob.ws_unroll, prob.stream)
    if st != 0:
        raise RuntimeError("unroll device status %s" % prob.b.STATUS[st])
    return t0.elapsed_time(t1) / steps


def time_e2e(prob, steps):
    """Same step through the public API with host buffers, all copies inside
    the timed region: the host-buffer entry points take pinned host inputs
    and write pinned host outputs, their copies overlapped with the solve --
    pararnn_newton_forward_host for a forward-only step,
    pararnn_newton_step_host (pre-activations and dL/dH in, H and dL/dpx out)
    for a step with the adjoint backward."""
    import torch

    from nonlinear_rnn_iteration_b200 import binding

    w = prob.w
    s = prob.stream
    px_host = torch.empty(prob.px.shape, dtype=prob.px.dtype, pin_memory=True)
    px_host.copy_(prob.px)
    H_host = torch.empty(prob.H.shape, dtype=torch.float32, pin_memory=True)
    code = binding.BF16 if prob.px.dtype == torch.bfloat16 else binding.F32
    if w.backward:
        g_host = torch.empty(prob.g.shape, dtype=torch.float32, pin_memory=True)
        g_host.copy_(prob.g)
        dpx_host = torch.empty(prob.dpx.shape, dtype=torch.float32, pin_memory=True)
        chans = E2E_STEP_CHANNELS if (w.D % 8 == 0 and w.D > E2E_STEP_CHANNELS) else 0
        n = binding.pararnn_newton_step_host_workspace_bytes(w.cell_id, w.B, w.T, w.D, w.K, code, chans)
        ws_host = torch.empty(n, dtype=torch.uint8, device=prob.px.device)
        da = prob.da

        def one():
            st = binding.pararnn_newton_step_host(w.cell_id, w.B, w.T, w.D, code, px_host, prob.a, None, w.K,
                                                  g_host, H_host, dpx_host, da, ws_host, n, chans, s)
            if st != binding.OK:
                raise RuntimeError("pararnn_newton_step_host: %s" % binding.pararnn_last_error())

        h2d = px_host.numel() * px_host.element_size() + g_host.numel() * 4
        d2h = H_host.numel() * 4 + dpx_host.numel() * 4
        path = "pararnn_newton_step_host, %s" % ("%d-channel slices" % chans if chans else "one slice")
    else:
        # slices of one batch row and E2E_CHANNELS channels
        chans = E2E_CHANNELS if (w.D % 8 == 0 and w.D > E2E_CHANNELS) else 0
        n = binding.pararnn_newton_forward_host_workspace_bytes(w.cell_id, w.B, w.T, w.D, w.K, code, 1, chans)
        ws_host = torch.empty(n, dtype=torch.uint8, device=prob.px.device)

        def one():
            st = binding.pararnn_newton_forward_host(w.cell_id, w.B, w.T, w.D, code, px_host, prob.a, None, w.K,
                                                     H_host, ws_host, n, 1, chans, s)
            if st != binding.OK:
                raise RuntimeError("pararnn_newton_forward_host: %s" % binding.pararnn_last_error())

        h2d = px_host.numel() * px_host.element_size()
        d2h = H_host.numel() * 4
        path = "pararnn_newton_forward_host, one-row %s" % ("x %d-channel slices" % chans if chans else "slices")
    one()
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(s)
    for _ in range(steps):
        one()
    t1.record(s)
    torch.cuda.synchronize()
    st = binding.pararnn_status_sync(ws_host, s)
    if st != binding.OK:
        raise RuntimeError("host-buffer step device status %s" % binding.STATUS[st])
    return t0.elapsed_time(t1) / steps, h2d, d2h, path


def cpu_baseline(w, device, seed, target_s=12.0, max_bytes=2.0e9):
    """The oracle as it stands -- Newton with sequential solves, plus the
    sequential adjoint for a workload with a backward -- on a bounded sample
    of the workload's channels (full length T each), on this host's cores and
    on one core."""
    import numpy as np
    import torch

    import oracle
    from nonlinear_rnn_iteration_b200 import workloads

    threads = os.cpu_count() or 1
    x = workloads.device_inputs(w, device, seed=seed, with_grad=w.backward)

    def sample(n):
        chans = workloads.sample_channels(w, n, seed=5)
        bi = torch.tensor([b for b, _ in chans], device=device)
        di = torch.tensor([d for _, d in chans], device=device)
        # (1, T, X, n) contiguous fp64, prepared outside the timed region
        prep = lambda t: np.ascontiguousarray(t[bi, :, :, di].float().cpu().numpy().transpose(1, 2, 0)[None],
                                              dtype=np.float64)
        a = None if x["a"] is None else np.ascontiguousarray(x["a"][:, di].cpu().numpy(), dtype=np.float64)
        return prep(x["px"]), a, (prep(x["dLdH"]) if w.backward else None)

    def run(inp, nthreads):
        px, a, g = inp
        t = time.perf_counter()
        if w.cell == "linear":
            H = oracle.unroll(w.cell_id, px, a, None, nthreads=nthreads)
        else:
            H, _ = oracle.newton(w.cell_id, px, a, None, K=w.K, nthreads=nthreads)
        if w.backward:
            oracle.adjoint(w.cell_id, px, a, None, H, g, nthreads=nthreads)
        return time.perf_counter() - t

    # bytes of fp64 host arrays per sampled channel (inputs, H, gradients)
    per_chan = 8 * w.T * (w.G + w.S + (w.S + w.G if w.backward else 0))
    n_cap = max(1, min(w.B * w.D, int(max_bytes // per_chan)))
    n = min(n_cap, max(threads, 8))
    dt = run(sample(n), threads)
    while dt < 1.0 and n < n_cap:
        n = min(n_cap, n * 4)
        dt = run(sample(n), threads)
    n_final = int(min(n_cap, max(n, n * target_s / max(dt, 1e-3))))
    if n_final > n:
        n = n_final
        dt = run(sample(n), threads)
    # one core, on a sample sized for a few seconds
    n1 = max(1, min(n, int(n * 3.0 / max(dt * threads, 1e-3))))
    dt1 = run(sample(n1), 1)
    del x
    kind = "sequential unroll" if w.cell == "linear" else "Newton K=%d with sequential solves" % w.K
    if w.backward:
        kind += " + sequential adjoint"
    return {"value": n * w.T / dt, "unit": UNIT, "cores": threads, "kind": "oracle",
            "sample": "%d of %d channels at full T=%d (%s, fp64), %.1f s" % (n, w.B * w.D, w.T, kind, dt),
            "value_1_core": n1 * w.T / dt1, "cores_1_core": 1,
            "sample_1_core": "%d channels at full T=%d, %.1f s" % (n1, w.T, dt1)}


def extra_workloads(names, device, seed_base):
    """Device-time lines for the other workloads (parity cases, not bench lines)."""
    import torch

    from nonlinear_rnn_iteration_b200 import workloads

    peaks = measured_peaks()
    out = {}
    for name in names:
        w = workloads.WORKLOADS[name]
        prob = Problem(w, device, seed_base + w.seed)
        ms, fwd, bwd = time_device(prob, steps=20, warmup=3, dist=None, device=device)
        in_bytes = prob.px.numel() * prob.px.element_size()
        rec = {"ms_per_step": round(ms, 4), "elem_per_s": w.elements / (ms / 1e3), "fwd_ms": round(fwd, 4),
               "fwd": kernel_roofline(w, "fwd", fwd, peaks),
               "l2": ("inputs larger than L2 (%.2f GB)" % (in_bytes / 1e9)) if in_bytes > 126e6 else
                     ("inputs L2-resident (%.2f MB): a latency measurement" % (in_bytes / 1e6))}
        if w.backward:
            rec.update(bwd_ms=round(bwd, 4), bwd=kernel_roofline(w, "bwd", bwd, peaks))
        ums = time_unroll(prob)
        rec.update(unroll_ms=round(ums, 4), newton_fwd_speedup_vs_gpu_unroll=round(ums / fwd, 2))
        if fwd < 0.1:
            # launch-bound: the forward's device time without launch overhead
            rec["fwd_ms_graph_replay"] = round(time_graph(prob), 4)
        out[name] = rec
        del prob
        torch.cuda.empty_cache()
    return out


def run_native(args):
    import torch

    from nonlinear_rnn_iteration_b200 import workloads

    rank, local, world = dist_env()
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    dist = dist_init("nccl", world)
    w = workloads.WORKLOADS[args.workload]
    if args.B or args.T or args.D:
        w = w.with_shape(B=args.B, T=args.T, D=args.D, name="%s@B%dT%dD%d" % (w.name, args.B or w.B, args.T or w.T,
                                                                           args.D or w.D))
    prob = Problem(w, device, rank_seed(w.seed, rank))
    with ClockSampler(local) as clk:
        ms, fwd_ms, bwd_ms = time_device(prob, args.steps, args.warmup, dist, device)
    clocks = clk.summary()
    value = aggregate_throughput(w.elements, world, 1, ms)
    peaks = measured_peaks()
    kernels = {"fwd": kernel_roofline(w, "fwd", fwd_ms, peaks)}
    if w.backward:
        kernels["bwd"] = kernel_roofline(w, "bwd", bwd_ms, peaks)
    # the dominant kernel: the one that takes longer per step
    dominant = "bwd" if (w.backward and bwd_ms > fwd_ms) else "fwd"
    roof = dict(kernels[dominant])
    roof["all_kernels"] = kernels
    if args.quick:
        e2e = None
    else:
        e2e_ms, h2d, d2h, e2e_path = time_e2e(prob, steps=3)
        e2e = {"value": w.elements / (e2e_ms / 1e3) * world, "unit": UNIT, "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "ms_per_step": round(e2e_ms, 3),
               "path": e2e_path, "host_memory": "pinned"}
    step = "forward (K=%d Newton iterations)" % w.K if w.cell != "linear" else "forward (one exact scan)"
    if w.backward:
        step += " + adjoint backward"
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32" if w.px_dtype == "f32" else "bf16 px / f32 state", "data": "synthetic",
        "config": {"workload": w.name, "cell": w.cell, "B": w.B, "T": w.T, "D": w.D, "K": w.K,
                   "px_dtype": w.px_dtype, "backward": w.backward, "step": step,
                   "fwd_ms": round(fwd_ms, 4), "bwd_ms": round(bwd_ms, 4) if w.backward else None,
                   "l2": "inputs larger than L2 (%.2f GB pre-activations per rank), no flush"
                         % (prob.px.numel() * prob.px.element_size() / 1e9),
                   "parallelism": "replicas%d" % world},
        "roofline": roof, "e2e": e2e, "gpu_launches": prob.launches_per_step() * args.steps, "clocks": clocks,
    }
    del prob
    torch.cuda.empty_cache()
    if rank == 0 and world == 1 and not args.quick:
        prob = Problem(w, device, rank_seed(w.seed, rank))
        ums = time_unroll(prob)
        line["config"]["sequential_unroll_on_gpu_ms"] = round(ums, 4)
        line["config"]["newton_fwd_speedup_vs_gpu_unroll"] = round(ums / fwd_ms, 2)
        del prob
        torch.cuda.empty_cache()
        line["cpu_baseline"] = cpu_baseline(w, device, rank_seed(w.seed, rank))
        if not args.no_extra:
            line["workloads"] = extra_workloads([n for n in workloads.WORKLOADS if n != w.name], device, 0)
            line["workloads"].update(head_workloads(device))
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.destroy_process_group()


def run_head(args):
    """--workload <head-wise>: time that forward alone and print its line
    (a profiling and inspection mode, not the bench contract's line)."""
    import torch

    from nonlinear_rnn_iteration_b200 import workloads

    w = workloads.HEAD_WORKLOADS[args.workload]
    if args.B or args.T:
        w = workloads.HeadWorkload("%s@B%dT%d" % (w.name, args.B or w.B, args.T or w.T), args.B or w.B,
                                   args.T or w.T, w.D, w.n_heads, w.K, w.px_dtype, w.seed)
    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    ms, bms, status, ums = time_head(w, device, args.steps, args.warmup)
    line = {"workload": w.name, "metric": METRIC, "unit": UNIT, "data": "synthetic",
            **head_line(w, ms, bms, status, ums)}
    print(json.dumps(line), flush=True)


def run_reference(args):
    """The oracle as the reference arm, rank 0 only, on the host cores."""
    rank, local, world = dist_env()
    if rank != 0:
        return
    import numpy as np

    import oracle
    from nonlinear_rnn_iteration_b200 import workloads

    w = workloads.WORKLOADS[args.workload]
    threads = os.cpu_count() or 1
    # a bounded sample per step: whole channels (full T), sized so that one step
    # takes a few seconds on this host
    n = max(threads, 8)
    per_step = []
    # fp64 host arrays per channel (inputs, H, gradients): the sample stays
    # within about 2 GB of host memory
    per_chan = 8 * w.T * (w.G + w.S + (w.S + w.G if w.backward else 0))
    n_cap = max(1, min(w.B * w.D, int(2.0e9 // per_chan)))
    n = min(n, n_cap)

    def prepare(xx):
        # fp64 contiguous inputs, converted outside the timed region
        return {k: (None if v is None else np.ascontiguousarray(v, dtype=np.float64)) for k, v in xx.items()}

    x = prepare(workloads.host_inputs(w.with_shape(B=1, D=n), seed=w.seed, with_grad=w.backward))

    def one():
        t = time.perf_counter()
        if w.cell == "linear":
            H = oracle.unroll(w.cell_id, x["px"], x["a"], None, nthreads=threads)
        else:
            H, _ = oracle.newton(w.cell_id, x["px"], x["a"], None, K=w.K, nthreads=threads)
        if w.backward:
            oracle.adjoint(w.cell_id, x["px"], x["a"], None, H, x["dLdH"], nthreads=threads)
        return time.perf_counter() - t

    probe = one()
    scale = max(1, int(2.0 / max(probe, 1e-3)))
    n = min(n_cap, n * scale)
    x = prepare(workloads.host_inputs(w.with_shape(B=1, D=n), seed=w.seed, with_grad=w.backward))
    for _ in range(args.warmup):
        one()
    for _ in range(args.steps):
        per_step.append(one())
    ms = 1e3 * sum(per_step) / len(per_step)
    value = n * w.T / (ms / 1e3)
    sample = "%d of %d channels at full T=%d per step (fp64 oracle: %s)" % (
        n, w.B * w.D, w.T, "Newton K=%d + adjoint" % w.K if w.backward else "Newton K=%d" % w.K)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms, 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "cell": w.cell, "B": w.B, "T": w.T, "D": w.D, "K": w.K,
                   "px_dtype": w.px_dtype, "parallelism": "host threads"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main(argv=None):
    from nonlinear_rnn_iteration_b200 import workloads

    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["native", "reference"], default="native")
    ap.add_argument("--workload", default=workloads.HEADLINE,
                    choices=sorted(workloads.WORKLOADS) + sorted(workloads.HEAD_WORKLOADS),
                    help="a head-wise workload is timed alone (profiling mode)")
    ap.add_argument("--no-extra", action="store_true", help="skip the other workloads' lines")
    ap.add_argument("--quick", action="store_true",
                    help="device timing only (no e2e, CPU baseline or other workloads): for profiling runs")
    ap.add_argument("--B", type=int, default=None, help="override the workload's batch (profiling cases)")
    ap.add_argument("--T", type=int, default=None, help="override the workload's length (profiling cases)")
    ap.add_argument("--D", type=int, default=None, help="override the workload's channels (profiling cases)")
    args = ap.parse_args(argv)
    args.warmup = max(3, args.warmup)
    args.steps = max(1, args.steps)
    if args.impl == "reference":
        run_reference(args)
    elif args.workload in workloads.HEAD_WORKLOADS:
        run_head(args)
    else:
        run_native(args)


if __name__ == "__main__":
    main()
