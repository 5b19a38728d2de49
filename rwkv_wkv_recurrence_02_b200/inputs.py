"""Seeded synthetic inputs for the WKV workloads.

This module only draws random numbers; it holds none of the WKV arithmetic.
Both the CUDA path's tests/benchmark and the CPU oracle are fed from it.

Workloads (sizes and distributions of the five synthetic cases this library is
measured on; N(m, s) means mean m and standard deviation s):

  tiny        B=1, T=64, C=32, fp32.  decay~U(-3,1), u~N(0,1), k,v~N(0,1),
              fresh state, no gate.
  layer_1b5   RWKV-4 1.5B-shaped layer: B=8, T=1024, C=2048, fp32.
              decay~U(-3,1), u~N(0,0.5), k,v,r~N(0,1), gate, random state with
              p~U(-5,5), b~U(0.5,1.5), a=b*N(0,1).
  layer_14b   RWKV-4 14B-shaped layer: B=4, T=8192, C=5120, bf16 k/v/r.
              decay~U(-4,2), u~N(0,1), k~N(0,2), v,r~N(0,1), gate, fresh state.
  stream_1m   B=1, C=4096, T=1,048,576 fed as 1024 chunks of 1024, bf16,
              no gate, fresh state.  decay~U(-3,1), u~N(0,1), v~N(0,1),
              k~N(0,1) with each element independently replaced, with
              probability 1e-3, by +50 or -50 (equal odds).
  decode      batched T=1 steps: L=24 layers, B=256, C=4096, bf16 k/v/r, fp32
              state, 1000 steps, gate.  decay~U(-3,1), u~N(0,1), k~N(0,3),
              v,r~N(0,1), fresh state.  Step s of layer l reads input set
              (s*24 + l) mod 64 of a ring of 64 sets.

w = exp(decay) is the parameterisation of the decay (w > 0); it is formed
here once, in float32, because the library takes w itself.

Matrix-state workloads (multi-head WKV, v5 / v6), from the training
configuration on the pages (n_embd 2048, head size 64, context 4096):

  v5_layer    B=8, T=4096, C=2048 in H=32 heads of 64, bf16 r/k/v, fp32 state,
              decay rate w = exp(d) per channel with d ~ U(-4, 0.5),
              u ~ N(0, 1), r, k, v ~ N(0, 1), fresh (zero) state.
  v6_layer    the same with a decay rate per token and channel,
              w = exp(d), d ~ U(-4, 0.5) drawn per element (float32).
"""
from dataclasses import dataclass
from typing import Optional

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    T: int
    C: int
    dtype: str            # "f32" or "bf16": dtype of k, v, r, y
    gate: bool
    decay_lo: float
    decay_hi: float
    u_std: float
    k_std: float
    random_state: bool
    outlier_prob: float = 0.0
    outlier_mag: float = 0.0
    chunk: int = 0        # >0: the sequence is fed as chunks of this length
    layers: int = 0       # >0: decode workload (wkv_step over this many layers)
    steps: int = 0        # decode steps
    ring: int = 0         # decode input-set ring size
    seed: int = 0

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    @property
    def elem_bytes(self) -> int:
        return 4 if self.dtype == "f32" else 2


WORKLOADS = {
    "tiny": Workload("tiny", 1, 64, 32, "f32", False, -3.0, 1.0, 1.0, 1.0, False, seed=1000),
    "layer_1b5": Workload("layer_1b5", 8, 1024, 2048, "f32", True, -3.0, 1.0, 0.5, 1.0, True, seed=1001),
    "layer_14b": Workload("layer_14b", 4, 8192, 5120, "bf16", True, -4.0, 2.0, 1.0, 2.0, False, seed=1002),
    "stream_1m": Workload("stream_1m", 1, 1 << 20, 4096, "bf16", False, -3.0, 1.0, 1.0, 1.0, False,
                          outlier_prob=1e-3, outlier_mag=50.0, chunk=1024, seed=1003),
    "decode": Workload("decode", 256, 1, 4096, "bf16", True, -3.0, 1.0, 1.0, 3.0, False,
                       layers=24, steps=1000, ring=64, seed=1004),
}


def _gen(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def make_params(wl: Workload, C: Optional[int] = None, layers: int = 0, device="cpu", seed=None):
    """Per-channel (w, u) as float32: (C,), or (layers, C) when layers > 0."""
    C = wl.C if C is None else C
    g = _gen(device, wl.seed if seed is None else seed)
    shape = (layers, C) if layers > 0 else (C,)
    decay = torch.empty(shape, dtype=torch.float32, device=device).uniform_(wl.decay_lo, wl.decay_hi, generator=g)
    w = torch.exp(decay)
    u = torch.randn(shape, dtype=torch.float32, device=device, generator=g) * wl.u_std
    return w.contiguous(), u.contiguous()


def make_sequence(wl: Workload, B: int, T: int, C: int, device="cpu", seed: int = 0, gate=None):
    """k, v, r of shape (B, T, C) in the workload's dtype (r is None without a gate).
    Values are drawn in float32 and rounded to bf16 (nearest-even) where needed."""
    gate = wl.gate if gate is None else gate
    g = _gen(device, seed)
    k = torch.randn((B, T, C), dtype=torch.float32, device=device, generator=g) * wl.k_std
    if wl.outlier_prob > 0.0:
        hit = torch.rand((B, T, C), device=device, generator=g) < wl.outlier_prob
        sign = torch.where(torch.rand((B, T, C), device=device, generator=g) < 0.5, -1.0, 1.0)
        k = torch.where(hit, sign * wl.outlier_mag, k)
    v = torch.randn((B, T, C), dtype=torch.float32, device=device, generator=g)
    r = torch.randn((B, T, C), dtype=torch.float32, device=device, generator=g) if gate else None
    dt = wl.torch_dtype
    return k.to(dt).contiguous(), v.to(dt).contiguous(), (None if r is None else r.to(dt).contiguous())


def make_state(wl: Workload, B: int, C: int, device="cpu", seed: int = 0):
    """Initial (3, B, C) float32 state {a, b, p}, or None for a fresh state."""
    if not wl.random_state:
        return None
    g = _gen(device, seed)
    p = torch.empty((B, C), dtype=torch.float32, device=device).uniform_(-5.0, 5.0, generator=g)
    b = torch.empty((B, C), dtype=torch.float32, device=device).uniform_(0.5, 1.5, generator=g)
    a = b * torch.randn((B, C), dtype=torch.float32, device=device, generator=g)
    return torch.stack([a, b, p]).contiguous()


def make_forward_inputs(name_or_wl, B=None, T=None, C=None, device="cpu", seed_offset: int = 0):
    """All inputs of one wkv_forward call of a workload (optionally resized)."""
    wl = WORKLOADS[name_or_wl] if isinstance(name_or_wl, str) else name_or_wl
    B = wl.B if B is None else B
    T = (wl.chunk or wl.T) if T is None else T
    C = wl.C if C is None else C
    w, u = make_params(wl, C=C, device=device)
    base = wl.seed * 1000 + seed_offset * 7
    k, v, r = make_sequence(wl, B, T, C, device=device, seed=base + 1)
    s0 = make_state(wl, B, C, device=device, seed=base + 2)
    return dict(w=w, u=u, k=k, v=v, r=r, state=s0)


def make_chunk(wl: Workload, index: int, B=None, C=None, device="cpu"):
    """k, v, r of chunk `index` of a chunked (streaming) workload."""
    B = wl.B if B is None else B
    C = wl.C if C is None else C
    return make_sequence(wl, B, wl.chunk, C, device=device, seed=wl.seed * 1000003 + index)


def make_decode_ring(wl: Workload, B=None, C=None, device="cpu"):
    """k, v, r of the decode ring: shape (ring + layers - 1, B, C).  Rows
    0..ring-1 are the ring's input sets (one (B, C) set per layer-step); the
    last layers-1 rows repeat the first ones, so the sets of step s,
    (s*layers + l) mod ring for l = 0..layers-1, are the contiguous slice
    starting at row (s*layers) mod ring."""
    B = wl.B if B is None else B
    C = wl.C if C is None else C
    g = _gen(device, wl.seed * 1000003)
    k = torch.randn((wl.ring, B, C), dtype=torch.float32, device=device, generator=g) * wl.k_std
    v = torch.randn((wl.ring, B, C), dtype=torch.float32, device=device, generator=g)
    r = torch.randn((wl.ring, B, C), dtype=torch.float32, device=device, generator=g) if wl.gate else None
    dt = wl.torch_dtype
    k, v, r = k.to(dt), v.to(dt), (None if r is None else r.to(dt))
    ext = lambda x: None if x is None else torch.cat([x, x[: wl.layers - 1]]).contiguous()
    return ext(k), ext(v), ext(r)


def decode_ring_start(wl: Workload, step: int) -> int:
    """First ring row of decode step `step` (see make_decode_ring)."""
    return (step * wl.layers) % wl.ring


def fresh_state(B: int, C: int, layers: int = 0, device="cpu"):
    """The empty state (0, 0, -1e38): (3, B, C), or (layers, 3, B, C)."""
    shape = (layers, 3, B, C) if layers > 0 else (3, B, C)
    s = torch.zeros(shape, dtype=torch.float32, device=device)
    s[..., 2, :, :] = -1e38
    return s


@dataclass(frozen=True)
class MatrixWorkload:
    name: str
    B: int
    T: int
    C: int
    H: int
    dtype: str            # "f32" or "bf16": dtype of r, k, v, y
    per_token_decay: bool
    decay_lo: float = -4.0
    decay_hi: float = 0.5
    seed: int = 0

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    @property
    def elem_bytes(self) -> int:
        return 4 if self.dtype == "f32" else 2


MATRIX_WORKLOADS = {
    "v5_layer": MatrixWorkload("v5_layer", 8, 4096, 2048, 32, "bf16", False, seed=1005),
    "v6_layer": MatrixWorkload("v6_layer", 8, 4096, 2048, 32, "bf16", True, seed=1006),
}


def make_matrix_inputs(wl, B=None, T=None, C=None, H=None, device="cpu", seed_offset: int = 0, state=False):
    """r, k, v (B, T, C) in the workload's dtype, w (C,) or (B, T, C) and u
    (C,) float32, and the state (B, H, N, N) float32 (None unless `state`)."""
    B = wl.B if B is None else B
    T = wl.T if T is None else T
    C = wl.C if C is None else C
    H = wl.H if H is None else H
    g = _gen(device, wl.seed * 1000 + seed_offset * 7 + 3)
    wshape = (B, T, C) if wl.per_token_decay else (C,)
    d = torch.empty(wshape, dtype=torch.float32, device=device).uniform_(wl.decay_lo, wl.decay_hi, generator=g)
    w = torch.exp(d)
    u = torch.randn((C,), dtype=torch.float32, device=device, generator=g)
    r, k, v = (torch.randn((B, T, C), dtype=torch.float32, device=device, generator=g).to(wl.torch_dtype)
               for _ in range(3))
    s0 = torch.randn((B, H, C // H, C // H), dtype=torch.float32, device=device, generator=g) if state else None
    return dict(w=w.contiguous(), u=u, r=r.contiguous(), k=k.contiguous(), v=v.contiguous(), state=s0)
