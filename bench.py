#!/usr/bin/env python
"""Benchmark of the WKV hot path on B200: prints one JSON line.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

A step is one pass of the whole operator over one batch of synthetic inputs
already resident in HBM.  The default workload is the long-context stream:
B=1, C=4096, T=1,048,576 bfloat16 tokens fed as 1024 chunks of 1024 tokens,
the state (num, den, max) carried in place from the empty state; one step is
the whole stream, 1024 wkv_forward calls replayed from one CUDA graph.  Other
workloads (layer_1b5, layer_14b, stream_1m_chunk: one chunk per step,
stream_1m_single: the whole stream in one call, decode: one wkv_step over 24
layers) are available with --workload.

Timing: W warm-up steps, then exactly K steps between a barrier +
synchronize on both sides, timed with CUDA events on the launching stream;
the inputs exceed the 126 MB L2 (the stream: 25.8 GB; the others rotate over
sets larger than twice L2), so no step finds its inputs in L2.  With N GPUs
(torchrun) every rank runs the same per-GPU workload on its own seeds
(independent sequences: no collective on the data path), the time is the max
over ranks and the value is the total.

`--impl reference` times the fp64 CPU oracle on the host cores on a bounded
lane sample per step (rank 0 only).
"""
import argparse
import math
import hashlib
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "WKV elements/s (B·T·C) and achieved HBM GB/s as % of B200 peak, 1 GPU"
METRIC_BWD = "WKV backward elements/s (B·T·C) and achieved HBM GB/s as % of B200 peak, 1 GPU"
METRIC_SHIFT = "token shift elements/s (B·T·C) and achieved HBM GB/s as % of B200 peak, 1 GPU"
METRIC_WKV5 = "matrix-state WKV elements/s (B·T·C) and achieved FP32 rate as % of B200 peak, 1 GPU"
# FP32 pipe of one B200: 148 SMs x 128 fused multiply-adds per clock at the
# 1965 MHz clocks.max.sm (the recipe's unit counts and clock)
FP32_PEAK_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12
SHIFT_MIXES = 3   # RWKV-4 time mixing: one mix each for K, V and R
UNIT = "elements/s"
SPEC_HBM_GBS = 8000.0
L2_BYTES = 126 * 1024 * 1024
PROFILE_TRAFFIC = os.path.join(ROOT, "profiles", "traffic.json")
CSRC = os.path.join(ROOT, "rwkv_wkv_recurrence_02_b200", "csrc")


# ---------------------------------------------------------------------------
# helpers that need no GPU (unit-tested on CPU)
# ---------------------------------------------------------------------------
# Sources that hold only the token shift kernel: no WKV kernel is built from
# them, so the WKV kernels' traffic records do not depend on them.
SHIFT_ONLY_SOURCES = ("wkv_shift.cuh",)


def kernel_source_hash(kernel: str = "") -> str:
    """Hash of the CUDA sources a recorded kernel is built from (a recorded
    DRAM traffic figure is only reported while it still describes the built
    kernel): every source for the token shift, every source but the
    token-shift-only ones for the WKV kernels."""
    h = hashlib.sha256()
    for name in sorted(os.listdir(CSRC)):
        if kernel != "token_shift" and name in SHIFT_ONLY_SOURCES:
            continue
        if name.endswith((".cu", ".cuh")):
            with open(os.path.join(CSRC, name), "rb") as f:
                h.update(name.encode())
                h.update(f.read())
    return h.hexdigest()[:16]


def algorithmic_bytes(wl, B, T, C, layers=0) -> int:
    """Bytes one call must move at minimum: every input element read once,
    every output written once, the state read and written once, w and u once."""
    eb = wl.elem_bytes
    if layers:  # decode step over `layers` layers
        n = layers * B * C
        io = n * eb * (3 if wl.gate else 2) + n * eb          # k, v, (r) in; y out
        return io + n * 12 * 2 + layers * C * 8               # state in + out; w, u
    n = B * T * C
    io = n * eb * (3 if wl.gate else 2) + n * eb
    state = B * C * 12 * (2 if wl.random_state or wl.chunk else 1)
    return io + state + C * 8


def algorithmic_bytes_backward(wl, B, T, C) -> int:
    """Bytes one backward call must move at minimum: k, v, dy (and r) read
    once, dk, dv (and dr) written once, the initial state and dL/d(a, b) of
    the returned state read, dL/d(initial state) written, w and u read, dw and
    du written."""
    eb = wl.elem_bytes
    n = B * T * C
    narr = 3 if wl.gate else 2
    io = n * eb * ((narr + 1) + narr)
    state = B * C * (12 * (1 if wl.random_state or wl.chunk else 0) + 8 + 12)
    return io + state + C * 16


def algorithmic_bytes_shift(wl, B, T, C, nmix=SHIFT_MIXES) -> int:
    """Bytes one token-shift call must move at minimum: x read once, nmix
    output rows written per input row, the carried previous token read and
    the next one written, mu read."""
    eb = wl.elem_bytes
    return B * T * C * eb * (1 + nmix) + 2 * B * C * eb + nmix * C * 4


def algorithmic_bytes_wkv5(wl, B, T, C, H, state=False) -> int:
    """Bytes one wkv5_forward call must move at minimum: r, k, v read and y
    written once, the decay rates (per channel, or per token and channel),
    u, and the (B, H, N, N) state written (and read when given)."""
    eb = wl.elem_bytes
    n = B * T * C
    N = C // H
    w = n * 4 if wl.per_token_decay else C * 4
    return n * eb * 4 + w + C * 4 + B * H * N * N * 4 * (2 if state else 1)


def flops_wkv5(B, T, C, H) -> int:
    """FP32 operations of the recurrence: per token, head and state entry a
    multiply-add for the output, a multiply-add and a multiply for the update
    (5 flops), N^2 entries per head: 5 N per element."""
    return B * T * C * 5 * (C // H)


def max_over_ranks(value: float, dist=None) -> float:
    """Largest value across ranks (the slowest rank's time)."""
    if dist is None or not dist.is_initialized() or dist.get_world_size() == 1:
        return value
    import torch
    backend = dist.get_backend()
    dev = torch.device("cuda", torch.cuda.current_device()) if backend == "nccl" else torch.device("cpu")
    t = torch.tensor([value], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def rank_seed(base: int, rank: int) -> int:
    """Per-rank seed: each rank processes its own independent sequences."""
    return base + 7919 * rank


def whole_job_rate(units_per_rank_step: int, world: int, steps: int, seconds: float) -> float:
    return units_per_rank_step * world * steps / seconds


def load_traffic(workload: str):
    """ncu DRAM bytes per launch recorded for this workload, if the kernel
    sources are unchanged since they were taken."""
    try:
        with open(PROFILE_TRAFFIC) as f:
            rec = json.load(f).get(workload)
    except (OSError, ValueError):
        return None
    if not rec or rec.get("source_hash") != kernel_source_hash(rec.get("kernel", "")):
        return None
    return rec.get("traffic_bytes_per_launch")


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except (OSError, ValueError, KeyError):
        return 6650.0, "fallback"


# ---------------------------------------------------------------------------
# clocks during the timed region (NVML reads only; nothing is changed)
# ---------------------------------------------------------------------------
class ClockSampler:
    REASONS = {
        "sw_power_cap": 0x4, "hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20,
        "hw_thermal_slowdown": 0x40, "hw_power_brake_slowdown": 0x80,
    }

    def __init__(self, device_index: int, period_s: float = 0.02):
        self.samples = []
        self.period = period_s
        self.stop_evt = threading.Event()
        self.ok = False
        self.max_mhz = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.ok = False
        self.thread = threading.Thread(target=self._run, daemon=True)

    def _one(self):
        try:
            mhz = self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM)
            reasons = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
            util = self.nv.nvmlDeviceGetUtilizationRates(self.h).gpu
            self.samples.append((time.time(), mhz, reasons, util))
        except Exception:
            pass

    def _run(self):
        while not self.stop_evt.is_set():
            self._one()
            time.sleep(self.period)

    def sample_now(self):
        """One extra sample now (the timed region's edges, so that a short
        region still has samples inside it)."""
        if self.ok:
            self._one()

    def start(self):
        if self.ok:
            self.thread.start()
        return self

    def stop(self):
        self.stop_evt.set()
        if self.ok:
            self.thread.join(timeout=2)

    def summary(self, t0: float, t1: float):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvml unavailable"]}
        inside = [s for s in sorted(self.samples) if t0 - 1e-3 <= s[0] <= t1 + 1e-3]
        src = inside if inside else [s for s in self.samples if s[0] >= t0 - 1.0]
        if not src:
            src = self.samples[-3:]
        mhz = [s[1] for s in src]
        reasons = sorted({name for s in src for name, bit in self.REASONS.items() if s[2] & bit})
        return {"sm_mhz": statistics.median(mhz) if mhz else None, "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(src), "in_window": bool(inside)}


# ---------------------------------------------------------------------------
# workloads on the GPU
# ---------------------------------------------------------------------------
class ForwardCase:
    """Two resident input sets of one wkv_forward workload (rotated per step)."""

    def __init__(self, wl, device, seed_base, T=None):
        import torch
        from rwkv_wkv_recurrence_02_b200 import inputs as I
        self.wl = wl
        T = (wl.chunk or wl.T) if T is None else T
        self.B, self.T, self.C = wl.B, T, wl.C
        self.sets = []
        nsets = 2
        one = algorithmic_bytes(wl, self.B, self.T, self.C)
        while nsets * one < 2 * L2_BYTES:
            nsets += 1
        for i in range(nsets):
            d = I.make_forward_inputs(wl, T=T, device=device, seed_offset=seed_base + i)
            if wl.chunk and d["state"] is None:
                d["state"] = I.fresh_state(self.B, self.C, device=device)
            self.sets.append(d)
        self.y = [torch.empty((self.B, T, self.C), dtype=wl.torch_dtype, device=device) for _ in range(nsets)]
        self.s_out = [torch.empty((3, self.B, self.C), dtype=torch.float32, device=device) for _ in range(nsets)]
        self.elements = self.B * self.T * self.C
        self.bytes = algorithmic_bytes(wl, self.B, self.T, self.C)
        self.launches_per_step = 1
        self.roofline_per_step = False
        self.period = nsets

    def step(self, i, wkv, ws):
        d = self.sets[i % len(self.sets)]
        if self.wl.chunk:   # streaming: the state is carried in place
            wkv.wkv_forward(d["w"], d["u"], d["k"], d["v"], d["r"], d["state"], y=self.y[i % len(self.y)],
                            state_out=d["state"], workspace=ws)
        else:
            wkv.wkv_forward(d["w"], d["u"], d["k"], d["v"], d["r"], d["state"], y=self.y[i % len(self.y)],
                            state_out=self.s_out[i % len(self.s_out)], workspace=ws)


class StreamCase:
    """The streaming workload as its definition reads: one step feeds the whole
    stream (T = 1,048,576 tokens) through wkv_forward as T / chunk carried
    chunks, the state in place and reset to the empty state at the start of
    the step.  k, v and y of the whole stream are resident (25.8 GB for the
    1M-token stream), so every chunk reads fresh inputs from HBM.
    inputs_ready passes WKV_FLAG_INPUTS_READY: the chunks' inputs are written
    before the step and never by the chain itself.  chain passes the chunk
    chain flags instead (WKV_FLAG_CHAIN_BEGIN on the first call of the step,
    WKV_FLAG_CHAIN_NEXT on the others, which imply WKV_FLAG_INPUTS_READY):
    each call takes the state the previous one publishes in the workspace."""

    def __init__(self, wl, device, seed_base, inputs_ready=True, chain=True):
        import dataclasses
        import torch
        from rwkv_wkv_recurrence_02_b200 import inputs as I
        self.wl = wl
        self.B, self.T, self.C, self.chunk = wl.B, wl.T, wl.C, wl.chunk
        self.n = wl.T // wl.chunk
        wr = dataclasses.replace(wl, seed=wl.seed + seed_base)
        self.w, self.u = I.make_params(wr, device=device)
        dt = wl.torch_dtype
        self.k = torch.empty((self.B, self.T, self.C), dtype=dt, device=device)
        self.v = torch.empty_like(self.k)
        for i in range(self.n):
            kc, vc, _ = I.make_chunk(wr, i, device=device)
            self.k[:, i * self.chunk:(i + 1) * self.chunk] = kc
            self.v[:, i * self.chunk:(i + 1) * self.chunk] = vc
        self.y = torch.empty_like(self.k)
        self.fresh = I.fresh_state(self.B, self.C, device=device)
        self.state = self.fresh.clone()
        self.ready = inputs_ready
        self.chain = chain and inputs_ready
        self.elements = self.B * self.T * self.C
        self.bytes = algorithmic_bytes(wl, self.B, self.chunk, self.C)      # per launch (one chunk)
        self.launches_per_step = self.n
        self.roofline_per_step = False
        self.period = 1

    def chunk_slice(self, i):
        return slice(i * self.chunk, (i + 1) * self.chunk)

    def step(self, i, wkv, ws):
        self.state.copy_(self.fresh)
        for j in range(self.n):
            sl = self.chunk_slice(j)
            wkv.wkv_forward(self.w, self.u, self.k[:, sl], self.v[:, sl], None, self.state, y=self.y[:, sl],
                            state_out=self.state, workspace=ws, inputs_ready=self.ready,
                            chain=("begin" if j == 0 else "next") if self.chain else None)


class DecodeCase:
    """Decode: one wkv_step over all layers per step, inputs from the ring; or,
    per_layer, one wkv_step per layer (L = 1 each)."""

    def __init__(self, wl, device, seed_base, per_layer=False):
        import torch
        from rwkv_wkv_recurrence_02_b200 import inputs as I
        self.wl, self.I = wl, I
        self.w, self.u = I.make_params(wl, layers=wl.layers, device=device, seed=wl.seed + seed_base)
        self.k, self.v, self.r = I.make_decode_ring(wl, device=device)
        self.state = I.fresh_state(wl.B, wl.C, layers=wl.layers, device=device)
        self.y = torch.empty((wl.layers, wl.B, wl.C), dtype=wl.torch_dtype, device=device)
        self.elements = wl.layers * wl.B * wl.C
        self.bytes = algorithmic_bytes(wl, wl.B, 1, wl.C, layers=wl.layers)
        self.per_layer = per_layer
        self.launches_per_step = wl.layers if per_layer else 1
        self.roofline_per_step = per_layer
        # steps whose inputs coincide: the ring start advances by `layers` mod `ring`
        self.period = wl.ring // math.gcd(wl.layers, wl.ring)

    def step(self, i, wkv, ws):
        a = self.I.decode_ring_start(self.wl, i)
        L = self.wl.layers
        if not self.per_layer:
            wkv.wkv_step(self.w, self.u, self.k[a:a + L], self.v[a:a + L], self.state,
                         None if self.r is None else self.r[a:a + L], y=self.y)
            return
        for l in range(L):
            sl = slice(l, l + 1)
            wkv.wkv_step(self.w[sl], self.u[sl], self.k[a + l:a + l + 1], self.v[a + l:a + l + 1], self.state[sl],
                         None if self.r is None else self.r[a + l:a + l + 1], y=self.y[sl])


class BackwardCase:
    """Backward: one wkv_backward call per step on the workload's shape, inputs
    (forward inputs, dy, dL/d(returned state)) rotating over sets larger than
    L2, outputs preallocated."""

    def __init__(self, wl, device, seed_base):
        import torch
        from rwkv_wkv_recurrence_02_b200 import inputs as I
        self.wl = wl
        T = wl.chunk or wl.T
        self.B, self.T, self.C = wl.B, T, wl.C
        one = algorithmic_bytes_backward(wl, self.B, self.T, self.C)
        nsets = 2
        while nsets * one < 2 * L2_BYTES:
            nsets += 1
        self.sets = []
        for i in range(nsets):
            d = I.make_forward_inputs(wl, T=T, device=device, seed_offset=seed_base + i)
            g = torch.Generator(device="cpu").manual_seed(9000 + seed_base + i)
            d["dy"] = torch.randn(self.B, T, self.C, generator=g).to(wl.torch_dtype).to(device)
            d["ds"] = torch.randn(3, self.B, self.C, generator=g).to(device)
            self.sets.append(d)
        mk = lambda: torch.empty((self.B, T, self.C), dtype=wl.torch_dtype, device=device)
        self.out = [dict(dk=mk(), dv=mk(), dr=mk() if wl.gate else None,
                         dw=torch.empty(self.C, device=device), du=torch.empty(self.C, device=device),
                         dstate_in=torch.empty((3, self.B, self.C), device=device)) for _ in range(2)]
        self.elements = self.B * T * self.C
        self.bytes = algorithmic_bytes_backward(wl, self.B, T, self.C)
        self.launches_per_step = 3   # checkpoint sweep, reverse walk, dw/du reduction
        self.roofline_per_step = True
        self.period = len(self.sets) * 2 // math.gcd(len(self.sets), 2)

    def step(self, i, wkv, ws):
        d = self.sets[i % len(self.sets)]
        wkv.wkv_backward(d["w"], d["u"], d["k"], d["v"], d["r"], d["state"], dy=d["dy"], dstate_out=d["ds"],
                         workspace=ws, **self.out[i % 2])


class Wkv5Case:
    """wkv5_forward on a matrix-state workload: inputs rotating over sets
    larger than twice L2, outputs preallocated, a fresh state per call."""

    def __init__(self, wl, device, seed_base):
        import torch
        from rwkv_wkv_recurrence_02_b200 import inputs as I
        self.wl = wl
        self.B, self.T, self.C, self.H = wl.B, wl.T, wl.C, wl.H
        one = algorithmic_bytes_wkv5(wl, self.B, self.T, self.C, self.H)
        nsets = 2
        while nsets * one < 2 * L2_BYTES:
            nsets += 1
        self.sets = [I.make_matrix_inputs(wl, device=device, seed_offset=seed_base + i) for i in range(nsets)]
        N = self.C // self.H
        self.y = [torch.empty((self.B, self.T, self.C), dtype=wl.torch_dtype, device=device) for _ in range(2)]
        self.s_out = [torch.empty((self.B, self.H, N, N), device=device) for _ in range(2)]
        self.elements = self.B * self.T * self.C
        self.bytes = one
        self.flops = flops_wkv5(self.B, self.T, self.C, self.H)
        self.launches_per_step = 1
        self.roofline_per_step = False
        self.period = nsets * 2 // math.gcd(nsets, 2)

    def step(self, i, wkv, ws):
        d = self.sets[i % len(self.sets)]
        wkv.wkv5_forward(d["w"], d["u"], d["r"], d["k"], d["v"], self.H, None, y=self.y[i % 2],
                         state_out=self.s_out[i % 2])


class TokenShiftCase:
    """Token shift on a workload's shape (decode: one token of one layer):
    x of the workload's dtype, SHIFT_MIXES mixes, the previous token carried;
    inputs rotate over sets larger than L2, outputs preallocated."""

    def __init__(self, wl, device, seed_base):
        import torch
        self.wl = wl
        T = 1 if wl.layers else (wl.chunk or wl.T)
        self.B, self.T, self.C = wl.B, T, wl.C
        one = algorithmic_bytes_shift(wl, self.B, T, self.C)
        nsets = 2
        while nsets * one < 2 * L2_BYTES:
            nsets += 1
        self.sets = []
        for i in range(nsets):
            g = torch.Generator(device="cpu").manual_seed(7000 + seed_base + i)
            self.sets.append({"x": torch.randn(self.B, T, self.C, generator=g).to(wl.torch_dtype).to(device),
                              "mu": torch.rand(SHIFT_MIXES, self.C, generator=g).to(device),
                              "xp": torch.randn(self.B, self.C, generator=g).to(wl.torch_dtype).to(device)})
        self.out = [torch.empty((SHIFT_MIXES, self.B, T, self.C), dtype=wl.torch_dtype, device=device)
                    for _ in range(2)]
        self.last = [torch.empty((self.B, self.C), dtype=wl.torch_dtype, device=device) for _ in range(2)]
        self.elements = self.B * T * self.C
        self.bytes = one
        self.launches_per_step = 1
        self.roofline_per_step = False
        self.period = nsets * 2 // math.gcd(nsets, 2)

    def step(self, i, wkv, ws):
        d = self.sets[i % len(self.sets)]
        wkv.wkv_token_shift(d["x"], d["mu"], d["xp"], out=self.out[i % 2], x_last=self.last[i % 2])


WORKLOAD_NAMES = ["stream_1m", "stream_1m_chunk", "stream_1m_single", "layer_1b5", "layer_14b", "decode", "tiny",
                  "v5_layer", "v6_layer"]


def workload(name):
    """A workload by name.  `stream_1m` is the whole stream as 1024 carried
    chunks per step; `stream_1m_chunk` one of those chunks per step;
    `stream_1m_single` the whole 1M-token sequence in one call."""
    import dataclasses
    from rwkv_wkv_recurrence_02_b200 import inputs as I
    if name == "stream_1m_single":
        return dataclasses.replace(I.WORKLOADS["stream_1m"], name=name, chunk=0)
    if name == "stream_1m_chunk":
        return dataclasses.replace(I.WORKLOADS["stream_1m"], name=name)
    if name in I.MATRIX_WORKLOADS:
        return I.MATRIX_WORKLOADS[name]
    return I.WORKLOADS[name]


def whole_stream(name) -> bool:
    return name == "stream_1m"


def make_case(name, device, seed_base, op="forward", per_layer=False, inputs_ready=True, chain=True):
    wl = workload(name)
    if op == "wkv5" or hasattr(wl, "H"):
        if not hasattr(wl, "H"):
            raise SystemExit("--op wkv5 takes the matrix-state workloads (v5_layer, v6_layer)")
        return Wkv5Case(wl, device, seed_base)
    if op == "token_shift":
        return TokenShiftCase(wl, device, seed_base)
    if op == "backward":
        if wl.layers:
            raise SystemExit("--op backward takes the forward workloads (the decode step has no reverse mode)")
        return BackwardCase(wl, device, seed_base)
    if wl.layers:
        return DecodeCase(wl, device, seed_base, per_layer)
    if whole_stream(name):
        return StreamCase(wl, device, seed_base, inputs_ready, chain)
    return ForwardCase(wl, device, seed_base)


def e2e_measure_wkv5(case, wkv, steps, warmup, stream):
    """wkv5_forward through the public API with host buffers: r, k, v, w, u
    in from pinned host memory, y and the state out."""
    import torch
    d = case.sets[0]
    names = ("w", "u", "r", "k", "v")
    host = {n: d[n].to("cpu").pin_memory() for n in names}
    dev = {n: torch.empty_like(x, device=d["k"].device) for n, x in host.items()}
    y_h = torch.empty(case.y[0].shape, dtype=case.y[0].dtype).pin_memory()
    s_h = torch.empty(case.s_out[0].shape).pin_memory()
    h2d = sum(x.numel() * x.element_size() for x in host.values())
    d2h = y_h.numel() * y_h.element_size() + s_h.numel() * 4

    def one():
        for n, x in host.items():
            dev[n].copy_(x, non_blocking=True)
        wkv.wkv5_forward(dev["w"], dev["u"], dev["r"], dev["k"], dev["v"], case.H, None, y=case.y[0],
                         state_out=case.s_out[0])
        y_h.copy_(case.y[0], non_blocking=True)
        s_h.copy_(case.s_out[0], non_blocking=True)

    for _ in range(warmup):
        one()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        one()
    e1.record(stream)
    torch.cuda.synchronize()
    return {"seconds": e0.elapsed_time(e1) / 1e3, "steps": steps, "h2d": h2d, "d2h": d2h,
            "path": "pinned host -> wkv5_forward (C ABI) -> pinned host"}


def cpu_baseline_wkv5(name: str, budget_s: float, max_reps: int = 1000):
    """The oracle's matrix-state WKV on this host's cores over a sample of
    (sequence, head) pairs of the workload, repeated for about `budget_s`."""
    import oracle
    from rwkv_wkv_recurrence_02_b200 import inputs as I
    wl = workload(name)
    heads = max(1, oracle.max_threads())
    N = wl.C // wl.H
    d = I.make_matrix_inputs(wl, B=1, C=heads * N, H=heads)
    f = lambda x: x.float().numpy()
    run = lambda: oracle.wkv5_forward(f(d["w"]), f(d["u"]), f(d["k"]), f(d["v"]), f(d["r"]), heads)
    t0 = time.perf_counter()
    reps = 0
    while True:
        run()
        reps += 1
        if time.perf_counter() - t0 >= budget_s or reps >= max_reps:
            break
    sec = time.perf_counter() - t0
    return {"value": wl.T * heads * N * reps / sec, "unit": UNIT, "cores": oracle.max_threads(), "kind": "oracle",
            "sample": f"{heads} heads of one sequence (T={wl.T}, N={N}), repeated {reps}x over {sec:.1f} s"}


def e2e_measure(case, wkv, ws, steps, warmup, stream):
    """Same metric through the public API with host buffers: each step copies
    its inputs from pinned host memory and reads the result back."""
    import torch
    if isinstance(case, Wkv5Case):
        return e2e_measure_wkv5(case, wkv, steps, warmup, stream)
    if isinstance(case, BackwardCase):
        return e2e_measure_backward(case, wkv, ws, steps, warmup, stream)
    if isinstance(case, DecodeCase):
        return e2e_measure_decode(case, wkv, steps, warmup, stream)
    if isinstance(case, TokenShiftCase):
        return e2e_measure_shift(case, wkv, steps, warmup, stream)
    if isinstance(case, StreamCase):
        return e2e_measure_stream(case, wkv, ws, steps, warmup, stream)
    d = case.sets[0]
    host = {k: (None if v is None else v.to("cpu").pin_memory()) for k, v in d.items()}
    y_host = torch.empty(case.y[0].shape, dtype=case.y[0].dtype).pin_memory()
    s_host = torch.empty((3, case.B, case.C), dtype=torch.float32).pin_memory()
    dev = {k: (None if v is None else torch.empty_like(v, device=d["k"].device)) for k, v in host.items()}
    h2d = sum(v.numel() * v.element_size() for v in host.values() if v is not None)
    d2h = y_host.numel() * y_host.element_size() + s_host.numel() * 4

    def one():
        for k, v in host.items():
            if v is not None:
                dev[k].copy_(v, non_blocking=True)
        y, s = wkv.wkv_forward(dev["w"], dev["u"], dev["k"], dev["v"], dev["r"], dev["state"], y=case.y[0],
                               state_out=case.s_out[0], workspace=ws)
        y_host.copy_(y, non_blocking=True)
        s_host.copy_(s, non_blocking=True)

    for _ in range(warmup):
        one()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        one()
    e1.record(stream)
    torch.cuda.synchronize()
    sec = e0.elapsed_time(e1) / 1e3
    return {"seconds": sec, "steps": steps, "h2d": h2d, "d2h": d2h}


def e2e_measure_stream(case, wkv, ws, steps, warmup, stream, ring=8):
    """The whole stream through the public API from pinned host memory: every
    chunk's k, v are copied in on one stream, the chunk's wkv_forward runs on
    the compute stream, and its y is copied back on a third, with two device
    buffers per array so that chunk i+1's upload and chunk i-1's download
    overlap chunk i's kernel.  The host side cycles over `ring` pinned chunks
    (the bytes per step are those of the whole stream)."""
    import torch
    ch, n = case.chunk, case.n
    host_k = [case.k[:, case.chunk_slice(j)].to("cpu").pin_memory() for j in range(ring)]
    host_v = [case.v[:, case.chunk_slice(j)].to("cpu").pin_memory() for j in range(ring)]
    host_y = [torch.empty_like(host_k[0]).pin_memory() for _ in range(ring)]
    s_host = torch.empty((3, case.B, case.C), dtype=torch.float32).pin_memory()
    dk = [torch.empty_like(host_k[0], device=case.k.device) for _ in range(2)]
    dv = [torch.empty_like(dk[0]) for _ in range(2)]
    dy = [torch.empty_like(dk[0]) for _ in range(2)]
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_comp = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]
    h2d = n * 2 * host_k[0].numel() * host_k[0].element_size()
    d2h = n * host_y[0].numel() * host_y[0].element_size() + s_host.numel() * 4

    def one():
        case.state.copy_(case.fresh)
        s_in.wait_stream(stream)
        for j in range(n):
            b = j & 1
            with torch.cuda.stream(s_in):
                if j >= 2:
                    s_in.wait_event(ev_comp[b])          # the kernel that read buffer b is done
                dk[b].copy_(host_k[j % ring], non_blocking=True)
                dv[b].copy_(host_v[j % ring], non_blocking=True)
                ev_in[b].record(s_in)
            stream.wait_event(ev_in[b])
            if j >= 2:
                stream.wait_event(ev_out[b])             # y buffer b has been read back
            wkv.wkv_forward(case.w, case.u, dk[b], dv[b], None, case.state, y=dy[b], state_out=case.state,
                            workspace=ws, stream=stream)
            ev_comp[b].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_comp[b])
                host_y[j % ring].copy_(dy[b], non_blocking=True)
                ev_out[b].record(s_out)
        s_host.copy_(case.state, non_blocking=True)
        stream.wait_stream(s_out)

    for _ in range(warmup):
        one()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        one()
    e1.record(stream)
    torch.cuda.synchronize()
    return {"seconds": e0.elapsed_time(e1) / 1e3, "steps": steps, "h2d": h2d, "d2h": d2h,
            "path": (f"pinned host (ring of {ring} chunks) -> {n} x wkv_forward (C ABI), uploads, kernels and "
                     "downloads on three streams with double-buffered chunks -> pinned host")}


def e2e_measure_decode(case, wkv, steps, warmup, stream):
    """Decode through the public API with host buffers: each step copies the
    token's k, v (and r) for every layer from pinned host memory, runs the
    step in the bench's form, and reads y of every layer back."""
    import torch
    L = case.wl.layers
    a = case.I.decode_ring_start(case.wl, 0)
    host = [None if t is None else t[a:a + L].to("cpu").pin_memory() for t in (case.k, case.v, case.r)]
    dev = [None if t is None else torch.empty_like(t, device=case.k.device) for t in host]
    y_host = torch.empty(case.y.shape, dtype=case.y.dtype).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in host if t is not None)
    d2h = y_host.numel() * y_host.element_size()

    def one():
        for dv, hv in zip(dev, host):
            if hv is not None:
                dv.copy_(hv, non_blocking=True)
        k, v, r = dev
        if case.per_layer:
            for l in range(L):
                sl = slice(l, l + 1)
                wkv.wkv_step(case.w[sl], case.u[sl], k[sl], v[sl], case.state[sl],
                             None if r is None else r[sl], y=case.y[sl])
        else:
            wkv.wkv_step(case.w, case.u, k, v, case.state, r, y=case.y)
        y_host.copy_(case.y, non_blocking=True)

    for _ in range(warmup):
        one()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        one()
    e1.record(stream)
    torch.cuda.synchronize()
    return {"seconds": e0.elapsed_time(e1) / 1e3, "steps": steps, "h2d": h2d, "d2h": d2h,
            "path": "pinned host -> wkv_step (C ABI) -> pinned host"}


def e2e_measure_shift(case, wkv, steps, warmup, stream):
    """Token shift through the public API with host buffers: x and the
    previous token in from pinned host memory, every mix and x_last out."""
    import torch
    d = case.sets[0]
    host = {n: d[n].to("cpu").pin_memory() for n in ("x", "mu", "xp")}
    dev = {n: torch.empty_like(v, device=d["x"].device) for n, v in host.items()}
    out_h = torch.empty(case.out[0].shape, dtype=case.out[0].dtype).pin_memory()
    last_h = torch.empty(case.last[0].shape, dtype=case.last[0].dtype).pin_memory()
    h2d = sum(v.numel() * v.element_size() for v in host.values())
    d2h = out_h.numel() * out_h.element_size() + last_h.numel() * last_h.element_size()

    def one():
        for n, v in host.items():
            dev[n].copy_(v, non_blocking=True)
        wkv.wkv_token_shift(dev["x"], dev["mu"], dev["xp"], out=case.out[0], x_last=case.last[0])
        out_h.copy_(case.out[0], non_blocking=True)
        last_h.copy_(case.last[0], non_blocking=True)

    for _ in range(warmup):
        one()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        one()
    e1.record(stream)
    torch.cuda.synchronize()
    return {"seconds": e0.elapsed_time(e1) / 1e3, "steps": steps, "h2d": h2d, "d2h": d2h,
            "path": "pinned host -> wkv_token_shift (C ABI) -> pinned host"}


def cpu_baseline_shift(name: str, budget_s: float, max_reps: int = 1000):
    """The oracle's token shift as it stands, on this host, over a channel
    sample of one call repeated for about `budget_s`."""
    import numpy as np
    import oracle
    wl = workload(name)
    T = 1 if wl.layers else (wl.chunk or wl.T)
    B, C = wl.B, wl.C
    csub = max(1, min(C, int(2e7 // (B * T))))
    g = np.random.default_rng(3)
    x = g.standard_normal((B, T, csub)).astype(np.float32)
    mu = g.uniform(0, 1, (SHIFT_MIXES, csub)).astype(np.float32)
    xp = g.standard_normal((B, csub)).astype(np.float32)
    t0 = time.perf_counter()
    reps = 0
    while True:
        oracle.token_shift(x, mu, xp)
        reps += 1
        if time.perf_counter() - t0 >= budget_s or reps >= max_reps:
            break
    sec = time.perf_counter() - t0
    sample = f"B={B}, T={T}, C={csub} of {C}, {SHIFT_MIXES} mixes"
    return {"value": B * T * csub * reps / sec, "unit": UNIT, "cores": 1, "kind": "oracle",
            "sample": f"{sample}, repeated {reps}x over {sec:.1f} s"}


def e2e_measure_backward(case, wkv, ws, steps, warmup, stream):
    """The backward through the public API with host buffers: every step copies
    k, v, r, dy, the state and dL/d(returned state) from pinned host memory and
    reads every gradient back."""
    import torch
    d = case.sets[0]
    names = ("w", "u", "k", "v", "r", "state", "dy", "ds")
    host = {n: (None if d[n] is None else d[n].to("cpu").pin_memory()) for n in names}
    dev = {n: (None if v is None else torch.empty_like(v, device=d["k"].device)) for n, v in host.items()}
    outs = case.out[0]
    back = {n: (None if v is None else torch.empty(v.shape, dtype=v.dtype).pin_memory()) for n, v in outs.items()}
    h2d = sum(v.numel() * v.element_size() for v in host.values() if v is not None)
    d2h = sum(v.numel() * v.element_size() for v in back.values() if v is not None)

    def one():
        for n, v in host.items():
            if v is not None:
                dev[n].copy_(v, non_blocking=True)
        wkv.wkv_backward(dev["w"], dev["u"], dev["k"], dev["v"], dev["r"], dev["state"], dy=dev["dy"],
                         dstate_out=dev["ds"], workspace=ws, **outs)
        for n, v in back.items():
            if v is not None:
                v.copy_(outs[n], non_blocking=True)

    for _ in range(warmup):
        one()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        one()
    e1.record(stream)
    torch.cuda.synchronize()
    return {"seconds": e0.elapsed_time(e1) / 1e3, "steps": steps, "h2d": h2d, "d2h": d2h,
            "path": "pinned host -> wkv_backward (C ABI) -> pinned host"}


def cpu_baseline_backward(name: str, budget_s: float, max_reps: int = 1000):
    """The oracle's reverse mode as it stands, on this host's cores, over a
    lane sample of the workload repeated for about `budget_s`."""
    import oracle
    from rwkv_wkv_recurrence_02_b200 import inputs as I
    import numpy as np
    wl = workload(name)
    T, B, C = wl.chunk or wl.T, wl.B, wl.C
    cap = max(1, int(1e7 // T))
    csub = C if B * C <= cap else max(1, cap // B)
    d = I.make_forward_inputs(wl, T=T, C=csub)
    f = lambda x: None if x is None else x.float().numpy()
    st = None if d["state"] is None else d["state"].double().numpy()
    g = np.random.default_rng(0)
    dy = g.normal(0, 1, (B, T, csub))
    ds = g.normal(0, 1, (3, B, csub))
    run = lambda: oracle.wkv_backward(f(d["w"]), f(d["u"]), f(d["k"]), f(d["v"]), f(d["r"]), st, dy, ds)
    t0 = time.perf_counter()
    reps = 0
    while True:
        run()
        reps += 1
        if time.perf_counter() - t0 >= budget_s or reps >= max_reps:
            break
    sec = time.perf_counter() - t0
    sample = f"lane sample B={B}, T={T}, C={csub} of {C}" if csub < C else f"full step B={B}, T={T}, C={C}"
    return {"value": B * T * csub * reps / sec, "unit": UNIT, "cores": oracle.max_threads(), "kind": "oracle",
            "sample": f"{sample}, repeated {reps}x over {sec:.1f} s"}


def cpu_baseline_sample(name: str, budget_s: float, max_reps: int = 1000):
    """Time the oracle as it stands on this host's cores: whole steps of the
    workload (or a lane sample of one) repeated for about `budget_s`."""
    import numpy as np
    import oracle
    from rwkv_wkv_recurrence_02_b200 import inputs as I
    wl = workload(name)
    if wl.layers:
        B, C = wl.B, wl.C
        w, u = I.make_params(wl, layers=wl.layers)
        k, v, r = I.make_decode_ring(wl)
        L = wl.layers
        st = np.zeros((L, 3, B, C))
        st[:, 2] = -1e38
        f = lambda x: x.float().numpy()
        args = (f(w), f(u), f(k[:L]), f(v[:L]), st, f(r[:L]))
        run = lambda: oracle.wkv_step(args[0], args[1], args[2], args[3], args[4], args[5])
        elems, sample = L * B * C, f"one decode step of all {L} layers (B={B}, C={C})"
    else:
        T = wl.T if whole_stream(name) else (wl.chunk or wl.T)
        B, C = wl.B, wl.C
        # lanes so that one repetition takes a bounded time
        lanes_total = B * C
        cap = max(1, int(2e7 // T))
        csub = C if lanes_total <= cap else max(1, cap // B)
        d = I.make_forward_inputs(wl, T=T, C=csub)
        f = lambda x: None if x is None else x.float().numpy()
        st = None if d["state"] is None else d["state"].double().numpy()
        run = lambda: oracle.wkv_forward(f(d["w"]), f(d["u"]), f(d["k"]), f(d["v"]), f(d["r"]), st)
        elems = B * T * csub
        sample = (f"full step B={B}, T={T}, C={C}" if csub == C else
                  f"lane sample B={B}, T={T}, C={csub} of {C}")
        if whole_stream(name):
            sample += " (the whole stream in one oracle call, which equals the carried chunks exactly)"
    t0 = time.perf_counter()
    reps = 0
    while True:
        run()
        reps += 1
        if time.perf_counter() - t0 >= budget_s or reps >= max_reps:
            break
    sec = time.perf_counter() - t0
    return {"value": elems * reps / sec, "unit": UNIT, "cores": oracle.max_threads(), "kind": "oracle",
            "sample": f"{sample}, repeated {reps}x over {sec:.1f} s"}


# ---------------------------------------------------------------------------
# arms
# ---------------------------------------------------------------------------
def config_of(case, workload, world):
    wl = case.wl
    cfg = {"workload": workload, "B": wl.B, "T": (getattr(wl, "chunk", 0) or wl.T), "C": wl.C,
           "io_dtype": wl.dtype, "gate": getattr(wl, "gate", False),
           "parallelism": f"dp{world}" if world > 1 else "single",
           "l2": "inputs rotate over sets totalling >2x the 126 MB L2"}
    if getattr(wl, "layers", 0):
        cfg.update({"layers": wl.layers, "T": 1, "steps_per_sequence": wl.steps})
    if whole_stream(workload):
        cfg.update({"T": wl.T, "chunk": wl.chunk,
                    "stream": (f"the whole stream per step: {wl.T // wl.chunk} wkv_forward calls of {wl.chunk} "
                               "tokens, state carried in place from the empty state"),
                    "inputs_ready": bool(getattr(case, "ready", False)),
                    "chain": bool(getattr(case, "chain", False)),
                    "l2": "inputs of the whole stream resident (25.8 GB), far above the 126 MB L2"})
    elif getattr(wl, "chunk", 0):
        cfg["stream"] = f"one chunk of {wl.chunk} tokens per step, state carried in place"
    return cfg


def shift_config(case):
    """Config keys of the token shift: its mixes, and for the decode workload
    that one step is one layer's token."""
    cfg = {"nmix": SHIFT_MIXES, "x_prev": "carried"}
    if case.wl.layers:
        cfg.update({"T": 1, "layers": 1, "decode": "one layer's token per step"})
    return cfg


def run_ours(args):
    import torch
    import torch.distributed as dist
    import rwkv_wkv_recurrence_02_b200 as wkv

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=device)
    wkv.lib()
    case = make_case(args.workload, device, rank_seed(0, rank), args.op, args.decode_per_layer,
                     not args.no_inputs_ready, not args.no_chain)
    ws = wkv.Workspace(device)
    stream = torch.cuda.current_stream()
    for i in range(args.warmup):
        case.step(i, wkv, ws)
    torch.cuda.synchronize()
    graphs = None
    if args.graph or (isinstance(case, StreamCase) and not args.no_graph):
        # one CUDA graph per distinct step (inputs rotate with period case.period)
        graphs = []
        for p in range(case.period):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                case.step(args.warmup + p, wkv, ws)
            graphs.append(g)
        for p in range(case.period):
            graphs[p].replay()
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clocks = ClockSampler(local).start()
    time.sleep(0.05)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clocks.sample_now()
    t0 = time.time()
    e0.record(stream)
    # an NVTX range around the timed launches, so a profiler's launch list can
    # be restricted to them (ncu --nvtx --nvtx-include bench_timed/)
    torch.cuda.nvtx.range_push("bench_timed")
    for i in range(args.steps):
        if graphs is not None:
            graphs[i % len(graphs)].replay()
        else:
            case.step(args.warmup + i, wkv, ws)
    torch.cuda.nvtx.range_pop()
    e1.record(stream)
    clocks.sample_now()
    torch.cuda.synchronize()
    t1 = time.time()
    if world > 1:
        dist.barrier()
    clocks.stop()
    sec = max_over_ranks(e0.elapsed_time(e1) / 1e3, dist if world > 1 else None)
    if ws.buf is not None and ws.status() != 0:
        raise SystemExit("the GPU reported a cross-block wait timeout during the benchmark")
    value = whole_job_rate(case.elements, world, args.steps, sec)
    # the roofline of a multi-kernel step (the backward) is taken over the whole
    # step: its algorithmic bytes over the step's time, a lower bound on the
    # dominant kernel's fraction
    per_launch = sec / args.steps / (1 if case.roofline_per_step else case.launches_per_step)
    peak, peak_kind = load_peaks()
    achieved = case.bytes / per_launch / 1e9
    out = {
        "metric": {"backward": METRIC_BWD, "token_shift": METRIC_SHIFT}.get(args.op, METRIC), "value": value,
        "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": sec / args.steps * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "io_dtype": case.wl.dtype,
        "data": "synthetic (seeded; distributions of the workload definition)",
        "config": dict(config_of(case, args.workload, world), **({"op": args.op} if args.op != "forward" else {}),
                       **(shift_config(case) if args.op == "token_shift" else {}),
                       **({"graph": (f"{len(graphs)} captured step(s) of {case.launches_per_step} launches "
                                     "replayed")} if graphs is not None else {}),
                       **({"decode_form": "one wkv_step per layer (L = 1)"} if args.decode_per_layer else {})),
        "hbm_gbs": achieved, "hbm_pct_of_spec_8tbs": 100.0 * achieved / SPEC_HBM_GBS,
        "hbm_pct_of_measured": 100.0 * achieved / peak,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "scope": ("whole step: checkpoint sweep + reverse walk + dw/du reduction"
                               if isinstance(case, BackwardCase) else
                               "whole step: one launch per layer" if case.roofline_per_step else "the step's one kernel"),
                     "frac": achieved / peak, "peak_kind": peak_kind,
                     "algorithmic_bytes_per_launch": case.bytes,
                     "traffic": load_traffic(args.workload + ("" if args.op == "forward" else "_" + args.op))},
        "gpu_launches": args.steps * case.launches_per_step,
        "clocks": clocks.summary(t0, t1),
    }
    if isinstance(case, Wkv5Case):
        # the recurrence on the CUDA cores is bound by FP32 arithmetic: its
        # roofline is the FP32 pipe; the tensor-core blocks move that work onto
        # the tensor cores, and their bound is the memory traffic
        tflops = case.flops / per_launch / 1e12
        tc_kernel = (os.environ.get("WKV5_KERNEL") != "recurrent" and case.wl.dtype == "bf16"
                     and case.C // case.H == 64)
        out["metric"] = METRIC_WKV5
        out["config"].update({"H": case.H, "head_size": case.C // case.H, "decay": (
            "per token and channel (v6)" if case.wl.per_token_decay else "per channel (v5)"), "gate": False,
            "kernel": ("recurrence on the CUDA cores (WKV5_KERNEL=recurrent)"
                       if os.environ.get("WKV5_KERNEL") == "recurrent" or case.wl.dtype != "bf16" or case.C // case.H != 64
                       else "blocks of 64 tokens on the tensor cores (tcgen05, tf32)")})
        if tc_kernel:
            out["roofline"] = {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                               "frac": achieved / peak, "peak_kind": peak_kind,
                               "algorithmic_bytes_per_launch": case.bytes, "scope": "the step's one kernel",
                               "recurrence_tflops": tflops, "recurrence_flops_per_launch": case.flops,
                               "traffic": load_traffic(args.workload + "_wkv5")}
        else:
            out["roofline"] = {"bound": "alu", "achieved": tflops, "peak": FP32_PEAK_TFLOPS, "unit": "TFLOP/s",
                               "frac": tflops / FP32_PEAK_TFLOPS,
                               "peak_kind": "derived: 148 SMs x 128 FP32 FMA/clock x 2 x 1965 MHz",
                               "flops_per_launch": case.flops, "algorithmic_bytes_per_launch": case.bytes,
                               "hbm_frac_of_measured": achieved / peak, "scope": "the step's one kernel",
                               "traffic": load_traffic(args.workload + "_wkv5")}
    if not args.no_e2e:
        e2e_steps = min(args.steps, 2 if isinstance(case, StreamCase) else args.e2e_steps)
        e = e2e_measure(case, wkv, ws, e2e_steps, 1 if isinstance(case, StreamCase) else 2, stream)
        if e is not None:
            out["e2e"] = {"value": whole_job_rate(case.elements, world, e["steps"],
                                                  max_over_ranks(e["seconds"], dist if world > 1 else None)),
                          "unit": UNIT, "h2d_bytes_per_step": e["h2d"], "d2h_bytes_per_step": e["d2h"],
                          "steps": e["steps"], "path": e.get("path", "pinned host -> wkv_forward (C ABI) -> pinned host")}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = {"backward": cpu_baseline_backward, "token_shift": cpu_baseline_shift,
                               "wkv5": cpu_baseline_wkv5}.get(
            "wkv5" if isinstance(case, Wkv5Case) else args.op, cpu_baseline_sample)(args.workload, args.cpu_seconds)
    if rank == 0:
        print(json.dumps(out), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def run_reference(args):
    """The oracle on the host cores, as it stands, on a bounded lane sample
    per step, so that the whole run stays within a few minutes."""
    import numpy as np
    import oracle
    from rwkv_wkv_recurrence_02_b200 import inputs as I
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    wl = workload(args.workload)
    budget = args.ref_budget_s
    f = lambda x: None if x is None else x.float().numpy()
    if args.op == "token_shift":
        return run_reference_shift(args, wl)
    if wl.layers:
        raise SystemExit("--impl reference times the forward workloads")
    T, B, C = (wl.T if whole_stream(args.workload) else (wl.chunk or wl.T)), wl.B, wl.C
    backward = args.op == "backward"

    def call(d, n):
        st = None if d["state"] is None else d["state"].double().numpy()
        a = (f(d["w"]), f(d["u"]), f(d["k"]), f(d["v"]), f(d["r"]), st)
        if not backward:
            return lambda: oracle.wkv_forward(*a)
        g = np.random.default_rng(1)
        dy, ds = g.normal(0, 1, (1, T, n)), g.normal(0, 1, (3, 1, n))
        return lambda: oracle.wkv_backward(*a, dy, ds)

    # calibrate: seconds per lane (all T tokens) with all cores busy
    ncal = min(C, 256 if T <= 65536 else 16)
    cal = I.make_forward_inputs(wl, B=1, T=T, C=ncal)
    run = call(cal, ncal)
    t0 = time.perf_counter()
    run()
    per_lane = (time.perf_counter() - t0) / ncal
    lanes = int(max(1, min(B * C, budget / max(1, args.steps + args.warmup) / per_lane)))
    csub = max(1, min(C, lanes))
    d = I.make_forward_inputs(wl, B=1, T=T, C=csub)
    run = call(d, csub)
    for _ in range(args.warmup):
        run()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        run()
    sec = time.perf_counter() - t0
    elems = T * csub
    value = elems * args.steps / sec
    sample = f"lane sample B=1, T={T}, C={csub} of the workload's B={B}, C={C} per step"
    if whole_stream(args.workload):
        sample += " (the whole stream in one oracle call, which equals the carried chunks exactly)"
    out = {
        "metric": METRIC_BWD if backward else METRIC, "value": value, "unit": UNIT, "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": sec / args.steps * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
        "config": {"workload": args.workload, "B": B, "T": T, "C": C, "io_dtype": wl.dtype, "gate": wl.gate},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": oracle.max_threads(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(out), flush=True)


def run_reference_shift(args, wl):
    """The oracle's token shift on a channel sample of the workload's call,
    sized so that every step takes a bounded share of the budget."""
    import numpy as np
    import oracle
    T = 1 if wl.layers else (wl.chunk or wl.T)
    B, C = wl.B, wl.C
    g = np.random.default_rng(3)
    per_step = args.ref_budget_s / max(1, args.steps + args.warmup)
    cal = 64
    xc = g.standard_normal((B, T, cal)).astype(np.float32)
    muc = g.uniform(0, 1, (SHIFT_MIXES, cal)).astype(np.float32)
    t0 = time.perf_counter()
    oracle.token_shift(xc, muc, None)
    per_chan = (time.perf_counter() - t0) / cal
    csub = int(max(1, min(C, per_step / max(per_chan, 1e-12))))
    x = g.standard_normal((B, T, csub)).astype(np.float32)
    mu = g.uniform(0, 1, (SHIFT_MIXES, csub)).astype(np.float32)
    xp = g.standard_normal((B, csub)).astype(np.float32)
    for _ in range(args.warmup):
        oracle.token_shift(x, mu, xp)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle.token_shift(x, mu, xp)
    sec = time.perf_counter() - t0
    value = B * T * csub * args.steps / sec
    sample = f"channel sample B={B}, T={T}, C={csub} of {C}, {SHIFT_MIXES} mixes per step"
    out = {
        "metric": METRIC_SHIFT, "value": value, "unit": UNIT, "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": sec / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
        "config": {"workload": args.workload, "B": B, "T": T, "C": C, "io_dtype": wl.dtype, "op": "token_shift",
                   "nmix": SHIFT_MIXES},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": 1, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(out), flush=True)


# the workload each operation is measured on unless --workload names another
DEFAULT_WORKLOAD = {"forward": "stream_1m", "backward": "layer_1b5", "token_shift": "layer_14b", "wkv5": "v5_layer"}


def parse_args(argv=None):
    p = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=None,
                   help="timed steps (default: 20 for the whole stream, 3000 for the other workloads)")
    p.add_argument("--warmup", type=int, default=None, help="warm-up steps (default: 5 / 20)")
    p.add_argument("--workload", default=None, choices=WORKLOAD_NAMES,
                   help="default per --op: " + ", ".join(f"{k}: {v}" for k, v in DEFAULT_WORKLOAD.items()))
    p.add_argument("--no-graph", action="store_true",
                   help="the whole stream: launch the chunk calls instead of replaying a CUDA graph")
    p.add_argument("--no-chain", action="store_true",
                   help="the whole stream: plain calls (state read after the previous kernel ends) instead of a "
                        "chunk chain")
    p.add_argument("--no-inputs-ready", action="store_true",
                   help="the whole stream: do not pass WKV_FLAG_INPUTS_READY")
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--graph", action="store_true",
                   help="replay each step from a captured CUDA graph instead of launching it")
    p.add_argument("--decode-per-layer", action="store_true",
                   help="decode: one wkv_step per layer (L = 1) instead of one call over all layers")
    p.add_argument("--op", default="forward", choices=["forward", "backward", "token_shift", "wkv5"],
                   help="forward (the headline), the reverse mode, or the token shift on the workload's shape")
    p.add_argument("--e2e-steps", type=int, default=20)
    p.add_argument("--cpu-seconds", type=float, default=10.0)
    p.add_argument("--ref-budget-s", type=float, default=90.0)
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-cpu-baseline", action="store_true")
    a = p.parse_args(argv)
    if a.workload is None:
        a.workload = DEFAULT_WORKLOAD[a.op]
    if a.op in ("backward", "token_shift") and whole_stream(a.workload):
        p.error(f"--op {a.op} takes a single-call workload, not the whole stream {a.workload}")
    if a.steps is None:
        a.steps = 20 if whole_stream(a.workload) and a.op == "forward" else 3000
    if a.warmup is None:
        a.warmup = 5 if whole_stream(a.workload) and a.op == "forward" else 20
    if a.warmup < 3:
        p.error("--warmup must be >= 3")
    return a


def main(argv=None):
    args = parse_args(argv)
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
