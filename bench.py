#!/usr/bin/env python
"""Benchmark of the WKV hot path on B200: prints one JSON line.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

A step is one pass of the whole operator over one batch of synthetic inputs
already resident in HBM.  The default workload is the RWKV-4 1.5B-shaped layer
(B=8, T=1024, C=2048, float32 k/v/r/y, sigmoid gate, random initial state):
one wkv_forward call per step.  Other workloads (layer_14b, stream_1m: one
1024-token chunk with the state carried, decode: one wkv_step over 24 layers)
are available with --workload.

Timing: W warm-up steps, then exactly K steps between a barrier +
synchronize on both sides, timed with CUDA events on the launching stream;
the inputs rotate over two sets whose size exceeds the 126 MB L2, so no step
finds its inputs in L2.  With N GPUs (torchrun) every rank runs the same
per-GPU workload on its own seeds (independent sequences: no collective on the
data path), the time is the max over ranks and the value is the total.

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

    def _run(self):
        while not self.stop_evt.is_set():
            try:
                mhz = self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM)
                reasons = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                util = self.nv.nvmlDeviceGetUtilizationRates(self.h).gpu
                self.samples.append((time.time(), mhz, reasons, util))
            except Exception:
                pass
            time.sleep(self.period)

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
        inside = [s for s in self.samples if t0 <= s[0] <= t1]
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


def workload(name):
    """A workload by name.  `stream_1m_single` is the streaming workload's
    whole 1M-token sequence in one call instead of 1024-token chunks."""
    import dataclasses
    from rwkv_wkv_recurrence_02_b200 import inputs as I
    if name == "stream_1m_single":
        return dataclasses.replace(I.WORKLOADS["stream_1m"], name=name, chunk=0)
    return I.WORKLOADS[name]


def make_case(name, device, seed_base, op="forward", per_layer=False):
    from rwkv_wkv_recurrence_02_b200 import inputs as I
    wl = workload(name)
    if op == "token_shift":
        return TokenShiftCase(wl, device, seed_base)
    if op == "backward":
        if wl.layers:
            raise SystemExit("--op backward takes the forward workloads (the decode step has no reverse mode)")
        return BackwardCase(wl, device, seed_base)
    if wl.layers:
        return DecodeCase(wl, device, seed_base, per_layer)
    return ForwardCase(wl, device, seed_base)


def e2e_measure(case, wkv, ws, steps, warmup, stream):
    """Same metric through the public API with host buffers: each step copies
    its inputs from pinned host memory and reads the result back."""
    import torch
    if isinstance(case, BackwardCase):
        return e2e_measure_backward(case, wkv, ws, steps, warmup, stream)
    if isinstance(case, DecodeCase):
        return e2e_measure_decode(case, wkv, steps, warmup, stream)
    if isinstance(case, TokenShiftCase):
        return e2e_measure_shift(case, wkv, steps, warmup, stream)
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
        T = wl.chunk or wl.T
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
    cfg = {"workload": workload, "B": wl.B, "T": (wl.chunk or wl.T), "C": wl.C, "io_dtype": wl.dtype,
           "gate": wl.gate, "parallelism": f"dp{world}" if world > 1 else "single",
           "l2": "inputs rotate over sets totalling >2x the 126 MB L2"}
    if wl.layers:
        cfg.update({"layers": wl.layers, "T": 1, "steps_per_sequence": wl.steps})
    if wl.chunk:
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
    case = make_case(args.workload, device, rank_seed(0, rank), args.op, args.decode_per_layer)
    ws = wkv.Workspace(device)
    stream = torch.cuda.current_stream()
    for i in range(args.warmup):
        case.step(i, wkv, ws)
    torch.cuda.synchronize()
    graphs = None
    if args.graph:
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
    t0 = time.time()
    e0.record(stream)
    for i in range(args.steps):
        if graphs is not None:
            graphs[i % len(graphs)].replay()
        else:
            case.step(args.warmup + i, wkv, ws)
    e1.record(stream)
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
                       **({"graph": f"{len(graphs)} captured steps replayed"} if graphs is not None else {}),
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
    if not args.no_e2e:
        e = e2e_measure(case, wkv, ws, min(args.steps, args.e2e_steps), 2, stream)
        if e is not None:
            out["e2e"] = {"value": whole_job_rate(case.elements, world, e["steps"],
                                                  max_over_ranks(e["seconds"], dist if world > 1 else None)),
                          "unit": UNIT, "h2d_bytes_per_step": e["h2d"], "d2h_bytes_per_step": e["d2h"],
                          "steps": e["steps"], "path": e.get("path", "pinned host -> wkv_forward (C ABI) -> pinned host")}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = {"backward": cpu_baseline_backward, "token_shift": cpu_baseline_shift}.get(
            args.op, cpu_baseline_sample)(args.workload, args.cpu_seconds)
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
    T, B, C = (wl.chunk or wl.T), wl.B, wl.C
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
    cal = I.make_forward_inputs(wl, B=1, T=T, C=min(C, 256))
    run = call(cal, min(C, 256))
    t0 = time.perf_counter()
    run()
    per_lane = (time.perf_counter() - t0) / min(C, 256)
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


def parse_args(argv=None):
    p = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=3000)
    p.add_argument("--warmup", type=int, default=20)
    p.add_argument("--workload", default="layer_1b5",
                   choices=["tiny", "layer_1b5", "layer_14b", "stream_1m", "stream_1m_single", "decode"])
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--graph", action="store_true",
                   help="replay each step from a captured CUDA graph instead of launching it")
    p.add_argument("--decode-per-layer", action="store_true",
                   help="decode: one wkv_step per layer (L = 1) instead of one call over all layers")
    p.add_argument("--op", default="forward", choices=["forward", "backward", "token_shift"],
                   help="forward (the headline), the reverse mode, or the token shift on the workload's shape")
    p.add_argument("--e2e-steps", type=int, default=20)
    p.add_argument("--cpu-seconds", type=float, default=10.0)
    p.add_argument("--ref-budget-s", type=float, default=90.0)
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-cpu-baseline", action="store_true")
    a = p.parse_args(argv)
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
