"""wkv5_forward (multi-head matrix-state WKV, v5 and v6) against the fp64
oracle, element by element, through the C ABI.

Error metric: |y_gpu - y_oracle| / s with s the oracle's magnitude scale of
the output (the same sum over the absolute value of every term), so the
error is measured against the size of what is summed even where y cancels
to near zero.  Tolerances: 2e-5 for float32 inputs and outputs, 1e-2 for
bfloat16 (its output rounding alone is up to 2^-9 of |y|).  The state is
compared against the largest |S| of its head."""
import numpy as np
import pytest
import torch

import oracle
import rwkv_wkv_recurrence_02_b200 as wkv
from rwkv_wkv_recurrence_02_b200 import inputs as I

pytestmark = pytest.mark.gpu

DEV = "cuda"
TOL = {torch.float32: 2e-5, torch.bfloat16: 1e-2}
STATE_TOL = 2e-5


def case(B, T, C, H, dtype, v6, state, seed):
    wl = I.MatrixWorkload("t", B, T, C, H, "f32" if dtype == torch.float32 else "bf16", v6, seed=seed)
    d = I.make_matrix_inputs(wl, state=state)
    return {k: (None if x is None else x.to(DEV)) for k, x in d.items()}


def np32(t):
    return None if t is None else t.detach().float().cpu().numpy()


def ref(d, H):
    s0 = None if d["state"] is None else d["state"].double().cpu().numpy()
    return oracle.wkv5_forward(np32(d["w"]), np32(d["u"]), np32(d["k"]), np32(d["v"]), np32(d["r"]), H, s0,
                               want_scale=True)


def check(d, H, y, s, tol):
    y_ref, s_ref, scale = ref(d, H)
    yg = y.double().cpu().numpy()
    assert np.all(np.isfinite(yg))
    err = float(np.max(np.abs(yg - y_ref) / np.maximum(scale, 1e-30))) if yg.size else 0.0
    assert err <= tol, err
    if s is not None:
        sg = s.double().cpu().numpy()
        hs = np.maximum(np.abs(s_ref).max(axis=(2, 3), keepdims=True), 1e-30)
        serr = float(np.max(np.abs(sg - s_ref) / hs))
        assert serr <= STATE_TOL, serr
    return err


SHAPES = [
    # B, T, C, H, dtype, v6, state
    (1, 1, 64, 1, torch.float32, False, False),
    (1, 2, 64, 1, torch.float32, True, True),
    (2, 33, 128, 2, torch.float32, False, True),     # one block and a ragged one
    (2, 33, 128, 4, torch.float32, True, False),     # head size 32
    (3, 100, 256, 4, torch.bfloat16, False, True),
    (2, 257, 192, 6, torch.bfloat16, True, True),    # head size 32, several blocks
    (1, 500, 128, 2, torch.float32, True, True),
]


@pytest.mark.parametrize("B,T,C,H,dtype,v6,state", SHAPES)
def test_wkv5_shapes(B, T, C, H, dtype, v6, state):
    d = case(B, T, C, H, dtype, v6, state, seed=B * 7 + T + C + H)
    y, s = wkv.wkv5_forward(d["w"], d["u"], d["r"], d["k"], d["v"], H, d["state"])
    torch.cuda.synchronize()
    check(d, H, y, s, TOL[dtype])


@pytest.mark.parametrize("v6", [False, True])
def test_wkv5_chain_in_place_equals_one_pass(v6):
    B, T, C, H = 2, 300, 128, 2
    d = case(B, T, C, H, torch.float32, v6, True, seed=41)
    y_full, s_full = wkv.wkv5_forward(d["w"], d["u"], d["r"], d["k"], d["v"], H, d["state"])
    st = d["state"].clone()
    ys = []
    for a, b in [(0, 1), (1, 40), (40, 40), (40, 300)]:
        sl = lambda x: x[:, a:b].contiguous()
        w = sl(d["w"]) if v6 else d["w"]
        y, _ = wkv.wkv5_forward(w, d["u"], sl(d["r"]), sl(d["k"]), sl(d["v"]), H, st, state_out=st)
        ys.append(y)
    torch.cuda.synchronize()
    # identical arithmetic in the same order: bit-equal to one call
    assert torch.equal(torch.cat(ys, dim=1), y_full)
    assert torch.equal(st, s_full)
    check(d, H, y_full, s_full, TOL[torch.float32])


def test_wkv5_guard_bands_untouched():
    B, T, C, H, pad = 2, 70, 128, 2, 4096
    d = case(B, T, C, H, torch.bfloat16, True, True, seed=43)
    n, ns = B * T * C, B * H * 64 * 64
    ybuf = torch.full((n + 2 * pad,), 12345.0, dtype=torch.bfloat16, device=DEV)
    sbuf = torch.full((ns + 2 * pad,), 777.0, device=DEV)
    y = ybuf[pad:pad + n].view(B, T, C)
    s = sbuf[pad:pad + ns].view(B, H, 64, 64)
    wkv.wkv5_forward(d["w"], d["u"], d["r"], d["k"], d["v"], H, d["state"], y=y, state_out=s)
    torch.cuda.synchronize()
    assert torch.all(ybuf[:pad] == 12345.0) and torch.all(ybuf[pad + n:] == 12345.0)
    assert torch.all(sbuf[:pad] == 777.0) and torch.all(sbuf[pad + ns:] == 777.0)
    check(d, H, y, s, TOL[torch.bfloat16])


def test_wkv5_empty_sequence_passes_the_state():
    d = case(2, 4, 128, 2, torch.float32, False, True, seed=47)
    s = torch.empty_like(d["state"])
    y = torch.empty((2, 0, 128), device=DEV)
    z = torch.empty((2, 0, 128), device=DEV)
    rc = wkv.lib().wkv5_forward(2, 0, 128, 2, 0, d["w"].data_ptr(), 0, d["u"].data_ptr(), z.data_ptr(),
                                z.data_ptr(), z.data_ptr(), d["state"].data_ptr(), y.data_ptr(), s.data_ptr(), None)
    torch.cuda.synchronize()
    assert rc == 0 and torch.equal(s, d["state"])


@pytest.mark.parametrize("name", ["v5_layer", "v6_layer"])
def test_wkv5_workloads_full_size(name):
    """The pages' layer shape (8 x 4096 x 2048, 32 heads of 64, bf16) at full
    size; the oracle on sampled (sequence, head) pairs (heads are
    independent, so a sampled head is checked exactly)."""
    wl = I.MATRIX_WORKLOADS[name]
    d = I.make_matrix_inputs(wl, device=DEV)
    y, s = wkv.wkv5_forward(d["w"], d["u"], d["r"], d["k"], d["v"], wl.H)
    torch.cuda.synchronize()
    N = wl.C // wl.H
    for b, h in [(0, 0), (3, 17), (7, 31)]:
        cs = slice(h * N, (h + 1) * N)
        sub = {k: x[b:b + 1, :, cs].contiguous() for k, x in d.items() if k in ("r", "k", "v")}
        sub["w"] = d["w"][b:b + 1, :, cs].contiguous() if wl.per_token_decay else d["w"][cs].contiguous()
        sub["u"] = d["u"][cs].contiguous()
        sub["state"] = None
        check(sub, 1, y[b:b + 1, :, cs], s[b:b + 1, h:h + 1], TOL[torch.bfloat16])
