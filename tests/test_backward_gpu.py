"""CUDA reverse mode (wkv_backward through the C ABI) against the fp64 oracle's
reverse mode, on identical seeded inputs.

Errors are measured per lane: the largest |gpu - oracle| over a lane's tokens
divided by the largest |oracle| of that lane, so a small gradient next to a
large one in the same lane is measured at the lane's scale.  dw, du and the
state's gradient are measured per channel (per lane for the state): each
against its own |oracle|, floored at FLOOR times the largest |oracle| of the
array (or of dv, where the array's sums cancel to zero), so a channel whose
gradient is small is still checked at its own scale down to that floor.
"""
import numpy as np
import pytest
import torch

import oracle
import rwkv_wkv_recurrence_02_b200 as wkv
from rwkv_wkv_recurrence_02_b200 import inputs as I
from tests.parity import to_np32, to_np64

pytestmark = pytest.mark.gpu

DEV = "cuda"
# Tolerances from the largest errors the kernels reach on the cases below,
# with a margin of about 3x: float32 1.35e-4 (dw of one channel against its
# own value; dk 7.2e-5 against its lane), bfloat16 3.9e-3 (dk, dv, dr: the
# bf16 rounding of the outputs, 2^-8 relative).
TOL = {torch.float32: 4e-4, torch.bfloat16: 1e-2}
FLOOR = 1e-3


def gen(B, T, C, dtype, gate, state, with_ds, seed):
    wl = I.Workload("bwd", B, T, C, "f32" if dtype == torch.float32 else "bf16", gate, -3.0, 1.0, 1.0, 1.0, state,
                    seed=seed + 101)
    d = {k: (None if v is None else v.to(DEV)) for k, v in I.make_forward_inputs(wl, device="cpu").items()}
    g = torch.Generator(device="cpu").manual_seed(seed + 7)
    d["dy"] = torch.randn(B, T, C, generator=g).to(dtype).to(DEV)
    d["ds"] = torch.randn(3, B, C, generator=g).to(DEV) if with_ds else None
    return d


def run(d, **kw):
    out = wkv.wkv_backward(d["w"], d["u"], d["k"], d["v"], d["r"], d["state"], dy=d["dy"], dstate_out=d["ds"], **kw)
    torch.cuda.synchronize()
    return out


def reference(d):
    return oracle.wkv_backward(to_np32(d["w"]), to_np32(d["u"]), to_np32(d["k"]), to_np32(d["v"]),
                               None if d["r"] is None else to_np32(d["r"]),
                               None if d["state"] is None else to_np64(d["state"]),
                               to_np64(d["dy"]), None if d["ds"] is None else to_np64(d["ds"]))


def lane_error(got, ref):
    got = to_np64(got)
    scale = np.abs(ref).max(axis=1, keepdims=True)
    scale = np.where(scale > 0, scale, 1.0)
    return float((np.abs(got - ref) / scale).max()) if got.size else 0.0


def check(d, out, tol=None):
    tol = TOL[d["k"].dtype] if tol is None else tol
    dk, dv, dr, dw, du, dsi = out
    rk, rv, rr, rw, ru, rs = reference(d)
    errs = {"dk": lane_error(dk, rk), "dv": lane_error(dv, rv)}
    if rr is not None:
        errs["dr"] = lane_error(dr, rr)
    # sums over many tokens can cancel to ~0 (T = 1 from the empty state:
    # du = 0 exactly): the floor then comes from the call's dv scale
    g_scale = max(np.abs(rv).max(), 1e-30)

    def per_element(got, ref):
        ref = np.asarray(ref)
        floor = FLOOR * max(np.abs(ref).max(), g_scale if np.abs(ref).max() == 0 else 0.0, 1e-30)
        return float((np.abs(to_np64(got) - ref) / np.maximum(np.abs(ref), floor)).max())

    errs["dw"] = per_element(dw, rw)
    errs["du"] = per_element(du, ru)
    if dsi is not None and d["state"] is not None:
        for i, name in enumerate(("ds_a", "ds_b", "ds_p")):
            errs[name] = per_element(dsi[i], rs[i])
    bad = {k: v for k, v in errs.items() if not v <= tol}
    assert not bad, (bad, errs)
    return errs


SHAPES = [
    # B, T, C, dtype, gate, state, dstate_out
    (1, 1, 4, torch.float32, False, False, False),
    (2, 17, 64, torch.float32, True, True, True),
    (1, 64, 64, torch.bfloat16, False, False, True),
    (2, 65, 128, torch.float32, True, False, False),
    (3, 200, 72, torch.bfloat16, True, True, True),     # ragged channel block
    (2, 1000, 128, torch.float32, False, True, True),
    (1, 4099, 64, torch.bfloat16, True, True, False),   # ragged last chunk, long
    (4, 333, 256, torch.float32, True, True, True),
    (300, 40, 64, torch.bfloat16, True, False, True),   # more lane blocks than CTA slots
    # more lane blocks than CTA slots with several chunks each: CTAs take
    # equal shares of the chunk order and hand one reverse state to the
    # CTA before them
    (5, 200, 3840, torch.float32, True, True, True),
    (7, 130, 2728, torch.bfloat16, True, True, True),   # ragged channel block and last chunk
]


@pytest.mark.parametrize("B,T,C,dtype,gate,state,with_ds", SHAPES)
def test_backward_shapes(B, T, C, dtype, gate, state, with_ds):
    d = gen(B, T, C, dtype, gate, state, with_ds, seed=B * 31 + T + C)
    check(d, run(d))


def test_backward_extreme_keys():
    """Keys of +-60 on alternate tokens: every weight and reverse weight spans
    the whole fp32 exponent range the max form has to keep apart."""
    d = gen(2, 300, 64, torch.float32, True, True, True, seed=3)
    t = torch.arange(300, device=DEV)[None, :, None]
    d["k"] = torch.where(t % 2 == 0, 60.0, -60.0).expand(2, 300, 64).contiguous()
    check(d, run(d))


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_backward_mixed_paths(dtype):
    """Sparse +-50 outliers among N(0, 1) keys: within one launch some
    segments take the fixed-scale fast path and others the exact one, and
    reverse states cross between them."""
    B, T, C = 3, 700, 128
    d = gen(B, T, C, dtype, True, True, True, seed=21)
    g = torch.Generator(device="cpu").manual_seed(4)
    k = torch.randn(B, T, C, generator=g)
    hit = torch.rand(B, T, C, generator=g) < 0.01
    k = torch.where(hit, torch.where(torch.rand(B, T, C, generator=g) < 0.5, -50.0, 50.0), k)
    d["k"] = k.to(dtype).to(DEV).contiguous()
    check(d, run(d))


def test_backward_chunked_equals_one_pass():
    """dstate_in of the later chunk, fed as dstate_out of the earlier one,
    reproduces one backward pass; dw and du add up."""
    B, T, C, T1 = 2, 300, 128, 130
    d = gen(B, T, C, torch.float32, True, True, True, seed=5)
    full = run(d)
    y, s_mid = wkv.wkv_forward(d["w"], d["u"], d["k"][:, :T1].contiguous(), d["v"][:, :T1].contiguous(),
                               d["r"][:, :T1].contiguous(), d["state"])
    sl = lambda x, a, b: x[:, a:b].contiguous()
    late = wkv.wkv_backward(d["w"], d["u"], sl(d["k"], T1, T), sl(d["v"], T1, T), sl(d["r"], T1, T), s_mid,
                            dy=sl(d["dy"], T1, T), dstate_out=d["ds"])
    early = wkv.wkv_backward(d["w"], d["u"], sl(d["k"], 0, T1), sl(d["v"], 0, T1), sl(d["r"], 0, T1),
                             d["state"], dy=sl(d["dy"], 0, T1), dstate_out=late[5].clone())
    torch.cuda.synchronize()
    for i in range(3):
        joined = torch.cat([early[i], late[i]], dim=1)
        assert lane_error(joined, to_np64(full[i])) <= 1e-3
    for i in (3, 4):
        ref = to_np64(full[i])
        assert np.abs(to_np64(early[i] + late[i]) - ref).max() <= 1e-3 * np.abs(ref).max()
    ref = to_np64(full[5])
    assert np.abs(to_np64(early[5]) - ref).max() <= 1e-3 * np.abs(ref).max()


def test_backward_guard_bands():
    """Every gradient lands exactly in its buffer."""
    B, T, C, pad = 2, 150, 72, 4096
    d = gen(B, T, C, torch.bfloat16, True, True, True, seed=9)
    n = B * T * C
    bufs = {name: torch.full((n + 2 * pad,), 321.0, dtype=torch.bfloat16, device=DEV) for name in ("dk", "dv", "dr")}
    views = {name: b[pad:pad + n].view(B, T, C) for name, b in bufs.items()}
    wbuf = torch.full((2 * C + 2 * pad,), 55.0, device=DEV)
    sbuf = torch.full((3 * B * C + 2 * pad,), 77.0, device=DEV)
    out = run(d, dk=views["dk"], dv=views["dv"], dr=views["dr"], dw=wbuf[pad:pad + C], du=wbuf[pad + C:pad + 2 * C],
              dstate_in=sbuf[pad:pad + 3 * B * C].view(3, B, C))
    for b in bufs.values():
        assert torch.all(b[:pad] == 321.0) and torch.all(b[pad + n:] == 321.0)
    assert torch.all(wbuf[:pad] == 55.0) and torch.all(wbuf[pad + 2 * C:] == 55.0)
    assert torch.all(sbuf[:pad] == 77.0) and torch.all(sbuf[pad + 3 * B * C:] == 77.0)
    check(d, out)


def test_backward_empty_sequence():
    """T == 0: dw = du = 0 and the state's gradient passes through."""
    B, C = 2, 64
    d = gen(B, 1, C, torch.float32, False, True, True, seed=11)
    k0 = torch.empty((B, 0, C), device=DEV)
    dk, dv, dr, dw, du, dsi = wkv.wkv_backward(d["w"], d["u"], k0, k0.clone(), None, d["state"], dy=k0.clone(),
                                               dstate_out=d["ds"])
    torch.cuda.synchronize()
    assert torch.all(dw == 0) and torch.all(du == 0)
    assert torch.equal(dsi[:2], d["ds"][:2])
    s = d["state"]
    assert torch.allclose(dsi[2], s[0] * d["ds"][0] + s[1] * d["ds"][1], rtol=1e-6, atol=1e-6)


def test_backward_layer_1b5_sampled():
    """The 1.5B-shaped layer (8 x 1024 x 2048, fp32, gated, random state) at full
    size, checked on sampled channels (lanes are independent; dw and du of a
    channel depend only on its own lanes)."""
    d = I.make_forward_inputs("layer_1b5", device=DEV)
    B, T, C = d["k"].shape
    g = torch.Generator(device="cpu").manual_seed(17)
    d["dy"] = torch.randn(B, T, C, generator=g).to(DEV)
    d["ds"] = torch.randn(3, B, C, generator=g).to(DEV)
    out = run(d)
    idx = torch.tensor(sorted(np.random.default_rng(3).choice(C, 48, replace=False)), device=DEV)
    sub = {k: (None if v is None else (v[..., idx].contiguous() if v.dim() > 1 else v[idx].contiguous()))
           for k, v in d.items()}
    outs = [None if o is None else (o[..., idx].contiguous() if o.dim() > 1 else o[idx].contiguous()) for o in out]
    check(sub, outs)
