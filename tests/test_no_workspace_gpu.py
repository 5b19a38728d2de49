"""wkv_forward without a caller workspace, on every kind of shape.

The operator's plain call form has no workspace argument; a NULL (or too
small) workspace must therefore be accepted for every shape and give the
oracle's results.  Calls go through the C ABI with raw pointers.  The shapes
reach each scratch-free schedule: the cluster kernel (17..1024 tokens), the
lane-resident kernel over whole lane blocks (more lane blocks than the GPU
holds at once, and a single long sequence), and the per-lane recurrence for
layouts the TMA kernels cannot take.
"""
import numpy as np
import pytest
import torch

import rwkv_wkv_recurrence_02_b200 as wkv
from rwkv_wkv_recurrence_02_b200 import inputs as I
from tests.parity import (TOL, argmax_index, gpu_argmax_index, oracle_forward, output_error, sample_channels,
                          state_error, to_np32, to_np64)

pytestmark = pytest.mark.gpu

DEV = "cuda"
WKV_ERR_WORKSPACE = -8


def abi_forward(d, y, s_out, ws=None, ws_bytes=0):
    """wkv_forward through the C ABI; returns the status."""
    B, T, C = d["k"].shape
    code = 0 if d["k"].dtype == torch.float32 else 1
    p = lambda t: None if t is None else t.data_ptr()
    rc = wkv.lib().wkv_forward(B, T, C, code, p(d["w"]), p(d["u"]), p(d["k"]), p(d["v"]), p(d["r"]),
                               p(d["state"]), p(y), p(s_out), ws, ws_bytes,
                               torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    return rc


def gen_case(B, T, C, dtype, gate, state, seed):
    wl = I.Workload("nows", B, T, C, "f32" if dtype == torch.float32 else "bf16", gate, -3.0, 1.0, 1.0, 1.0,
                    state, seed=seed)
    d = I.make_forward_inputs(wl, device="cpu")
    return {k: (None if v is None else v.to(DEV)) for k, v in d.items()}


def check(d, y, s, idx=None):
    if idx is not None:
        f = lambda x: None if x is None else x[..., idx].contiguous()
        ref = oracle_forward(d["w"][idx], d["u"][idx], f(d["k"]), f(d["v"]), f(d["r"]), f(d["state"]))
        y, s = y[..., idx.to(DEV)], s[..., idx.to(DEV)]
    else:
        ref = oracle_forward(d["w"], d["u"], d["k"], d["v"], d["r"], d["state"])
    y_ref, s_ref, scale = ref
    tol = TOL[d["k"].dtype]
    assert output_error(y, y_ref, scale) <= tol
    assert max(state_error(s, s_ref)) <= tol
    return s_ref


SHAPES = [
    # B, T, C, dtype, gate, state: which schedule a NULL workspace reaches
    (5, 200, 3840, torch.float32, True, True),     # lane-resident, more lane blocks than slots: whole blocks
    (7, 1300, 2724, torch.bfloat16, True, True),   # same, ragged channel block and last chunk
    (1, 5000, 256, torch.float32, False, True),    # few lane blocks, T > 1024: lane-resident over whole blocks
    (2, 2000, 4096, torch.bfloat16, True, False),
    (3, 3000, 130, torch.float32, True, True),     # C not a multiple of 4: per-lane recurrence
    (2, 2000, 7, torch.bfloat16, False, True),     # odd C
    (2, 700, 96, torch.float32, True, True),       # cluster kernel
]


@pytest.mark.parametrize("B,T,C,dtype,gate,state", SHAPES)
def test_null_workspace_every_schedule(B, T, C, dtype, gate, state):
    d = gen_case(B, T, C, dtype, gate, state, seed=B * 31 + T + C)
    assert wkv.lib().wkv_forward_workspace_bytes(B, T, C, 0 if dtype == torch.float32 else 1) > 0
    y = torch.full_like(d["k"], float("nan"))
    s = torch.full((3, B, C), float("nan"), device=DEV)
    assert abi_forward(d, y, s) == 0
    check(d, y, s)


def test_too_small_workspace_is_not_touched():
    """A workspace smaller than required is ignored (the call runs without
    one); its contents stay as they were."""
    B, T, C = 5, 200, 3840
    d = gen_case(B, T, C, torch.float32, True, True, seed=3)
    need = wkv.lib().wkv_forward_workspace_bytes(B, T, C, 0)
    buf = torch.full((need // 4 + 64,), 424242.0, device=DEV)
    base = (buf.data_ptr() + 255) & ~255
    y = torch.empty_like(d["k"])
    s = torch.empty((3, B, C), device=DEV)
    assert abi_forward(d, y, s, ws=base, ws_bytes=need - 256) == 0
    assert torch.all(buf == 424242.0)
    check(d, y, s)


def test_layer_14b_full_without_workspace():
    """The 14B-shaped layer (4 x 8192 x 5120, bf16, gated) with a NULL
    workspace, at full size; the oracle on sampled lanes, and the argmax
    index of the final running max."""
    d = I.make_forward_inputs("layer_14b", device=DEV)
    B, T, C = d["k"].shape
    y = torch.empty_like(d["k"])
    s = torch.empty((3, B, C), device=DEV)
    assert abi_forward(d, y, s) == 0
    idx = sample_channels(C, n=48)
    check(d, y, s, idx)
    j_ref, gap, cand = argmax_index(to_np32(d["k"][..., idx.to(DEV)]), to_np32(d["w"][idx.to(DEV)]), T)
    j_gpu = gpu_argmax_index(to_np64(s[2][..., idx.to(DEV)]), cand, 0)
    clear = gap > 1e-2
    assert np.array_equal(j_gpu[clear], j_ref[clear])
    # and the same as the call with a workspace, everywhere
    y2, s2 = wkv.wkv_forward(d["w"], d["u"], d["k"], d["v"], d["r"], None)
    torch.cuda.synchronize()
    assert (y.float() - y2.float()).abs().max().item() <= 2e-2


def test_long_stream_without_workspace():
    """One sequence of 65,536 tokens of the streaming workload's kind (4096
    channels, bf16, +-50 outliers) with a NULL workspace: a call the
    workspace schedules would split across many CTAs."""
    wl = I.WORKLOADS["stream_1m"]
    T, C = 65536, wl.C
    w, u = I.make_params(wl, device=DEV)
    k, v, _ = I.make_sequence(wl, 1, T, C, device=DEV, seed=77)
    d = dict(w=w, u=u, k=k, v=v, r=None, state=None)
    y = torch.empty_like(k)
    s = torch.empty((3, 1, C), device=DEV)
    assert abi_forward(d, y, s) == 0
    idx = sample_channels(C, n=16)
    check(d, y, s, idx)
