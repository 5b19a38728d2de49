"""Token shift (wkv_token_shift) against the oracle, element by element, on
seeded inputs: both access widths (16-byte vectors, and single elements for
rows or pointers that do not allow them), ragged token tails of the 8-token
units, several mixes, a carried or fresh previous token, in-place x_last,
chaining, T = 0, untouched guard bands, and the full-size parallel and decode
shapes on sampled channels.

Error metric: |gpu - oracle| over |mu x_t| + |(1 - mu) x_{t-1}|, the scale of
the convex mix (a float32 evaluation rounds three times at that scale; a
bfloat16 output once more, by at most 2^-9 of it).  x_last is a copy and must
be bit-exact."""
import numpy as np
import pytest
import torch

import oracle
import rwkv_wkv_recurrence_02_b200 as wkv

pytestmark = pytest.mark.gpu
DEV = "cuda"
TOL = {torch.float32: 1e-6, torch.bfloat16: 4e-3}


def gen(B, T, C, nmix, dtype, prev, seed):
    g = torch.Generator(device="cpu").manual_seed(seed)
    x = torch.randn(B, T, C, generator=g).to(dtype)
    mu = torch.rand(nmix, C, generator=g)
    xp = torch.randn(B, C, generator=g).to(dtype) if prev else None
    return x, mu, xp


def oracle_ref(x, mu, xp):
    f = lambda t: None if t is None else t.float().cpu().numpy()
    out, last = oracle.token_shift(f(x), f(mu), f(xp))
    xf = x.double().cpu().numpy()
    pf = np.zeros((x.shape[0], x.shape[2])) if xp is None else xp.double().cpu().numpy()
    prev = np.concatenate([pf[:, None, :], xf[:, :-1, :]], axis=1)
    m = mu.double().cpu().numpy()[:, None, None, :]
    scale = np.abs(m * xf[None]) + np.abs((1.0 - m) * prev[None]) + 1e-30
    return out, last, scale


def check(x, mu, xp, out, last):
    ref, ref_last, scale = oracle_ref(x, mu, xp)
    err = float(np.max(np.abs(out.double().cpu().numpy() - ref) / scale)) if ref.size else 0.0
    assert err <= TOL[x.dtype], f"error {err:.3e}"
    if last is not None:
        assert torch.equal(last.cpu(), torch.from_numpy(ref_last).to(x.dtype))


SHAPES = [
    # B, T, C, nmix, dtype, carried previous token
    (1, 1, 1, 1, torch.float32, False),
    (2, 17, 64, 3, torch.float32, True),      # vector path, ragged 8-token unit
    (3, 5, 130, 3, torch.float32, True),      # C not a multiple of 4: element-wise
    (2, 33, 72, 3, torch.bfloat16, True),     # vector path
    (1, 9, 7, 2, torch.bfloat16, False),      # element-wise
    (4, 1, 4096, 3, torch.bfloat16, True),    # decode: one token
    (2, 16, 96, 8, torch.bfloat16, True),     # eight mixes, whole units
    (3, 1000, 2048, 1, torch.float32, True),
]


@pytest.mark.parametrize("B,T,C,nmix,dtype,prev", SHAPES)
def test_token_shift_shapes(B, T, C, nmix, dtype, prev):
    x, mu, xp = gen(B, T, C, nmix, dtype, prev, seed=B * 100 + T + C)
    out, last = wkv.wkv_token_shift(x.to(DEV), mu.to(DEV), None if xp is None else xp.to(DEV))
    torch.cuda.synchronize()
    check(x, mu, xp, out, last)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_token_shift_in_place_chaining_equals_one_call(dtype):
    """x_last == x_prev (in place); four chunks reproduce one call bit for bit."""
    x, mu, xp = gen(2, 4 * 37, 256, 3, dtype, True, seed=77)
    x, mu, xp = x.to(DEV), mu.to(DEV), xp.to(DEV)
    whole, last = wkv.wkv_token_shift(x, mu, xp)
    carry = xp.clone()
    parts = []
    for i in range(4):
        o, _ = wkv.wkv_token_shift(x[:, i * 37:(i + 1) * 37].contiguous(), mu, carry, x_last=carry)
        parts.append(o)
    torch.cuda.synchronize()
    assert torch.equal(torch.cat(parts, dim=2), whole)
    assert torch.equal(carry, last)
    check(x, mu, xp, whole, last)


def test_token_shift_empty_sequence_passes_the_state():
    xp = torch.randn(3, 64, device=DEV)
    x = torch.empty(3, 0, 64, device=DEV)
    mu = torch.rand(2, 64, device=DEV)
    out, last = wkv.wkv_token_shift(x, mu, xp)
    _, zeros = wkv.wkv_token_shift(x, mu, None)
    torch.cuda.synchronize()
    assert out.shape == (2, 3, 0, 64)
    assert torch.equal(last, xp) and torch.equal(zeros, torch.zeros_like(xp))


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_token_shift_guard_bands_untouched(dtype):
    B, T, C, nmix = 2, 19, 72, 3
    x, mu, xp = gen(B, T, C, nmix, dtype, True, seed=5)
    n, pad = nmix * B * T * C, 1024
    buf = torch.full((n + 2 * pad,), 7.0, dtype=dtype, device=DEV)
    lbuf = torch.full((B * C + 2 * pad,), 7.0, dtype=dtype, device=DEV)
    out = buf[pad:pad + n].view(nmix, B, T, C)
    last = lbuf[pad:pad + B * C].view(B, C)
    wkv.wkv_token_shift(x.to(DEV), mu.to(DEV), xp.to(DEV), out=out, x_last=last)
    torch.cuda.synchronize()
    check(x, mu, xp, out, last)
    for b in (buf, lbuf):
        assert torch.all(b[:pad] == 7.0) and torch.all(b[-pad:] == 7.0)


@pytest.mark.parametrize("B,T,C", [(4, 8192, 5120), (256, 1, 4096)])
def test_token_shift_full_size_sampled(B, T, C):
    """The parallel-mode layer shape and the decode shape, bfloat16, three
    mixes; channels are independent, so sampled channels are checked exactly."""
    x, mu, xp = gen(B, T, C, 3, torch.bfloat16, True, seed=B + T)
    out, last = wkv.wkv_token_shift(x.to(DEV), mu.to(DEV), xp.to(DEV))
    torch.cuda.synchronize()
    idx = torch.arange(3, C, 61)
    check(x[..., idx].contiguous(), mu[:, idx].contiguous(), xp[:, idx].contiguous(), out[..., idx.to(DEV)],
          last[:, idx.to(DEV)])
