"""Seeded random shapes through every forward kernel and the reverse mode,
against the oracle: sizes, dtypes, gates, states and alignments drawn at
random.  Odd channel counts take the register-load kernels, multiples of 4
the TMA ones; few lane blocks take the part kernel, many the lane-resident
one."""
import numpy as np
import pytest
import torch

import rwkv_wkv_recurrence_02_b200 as wkv
from tests.test_backward_gpu import check as check_backward
from tests.test_backward_gpu import gen as gen_backward
from tests.test_parity_gpu import check_forward, gen_case

pytestmark = pytest.mark.gpu


def draws(n, seed):
    g = np.random.default_rng(seed)
    for _ in range(n):
        B = int(g.integers(1, 6))
        T = int(g.choice([int(g.integers(1, 20)), int(g.integers(20, 400)), int(g.integers(400, 1500))]))
        C = int(g.choice([int(g.integers(1, 200)), 4 * int(g.integers(1, 100))]))
        dtype = torch.float32 if g.random() < 0.5 else torch.bfloat16
        yield B, T, C, dtype, bool(g.random() < 0.5), bool(g.random() < 0.5), int(g.integers(0, 1 << 30))


@pytest.mark.parametrize("B,T,C,dtype,gate,state,seed", list(draws(24, 2026)))
def test_random_forward(B, T, C, dtype, gate, state, seed):
    d = gen_case(B, T, C, dtype, gate, state, seed=seed % 100000)
    y, s = wkv.wkv_forward(d["w"], d["u"], d["k"], d["v"], d["r"], d["state"])
    torch.cuda.synchronize()
    check_forward(d, y, s)


def backward_draws(n, seed):
    for B, T, C, dtype, gate, state, s in draws(n, seed):
        # the reverse mode takes the TMA tiles only: rows of a multiple of 16 bytes
        step = 4 if dtype == torch.float32 else 8
        C = step * max(1, C // step)
        yield B, T, C, dtype, gate, state, bool(s % 2), s


@pytest.mark.parametrize("B,T,C,dtype,gate,state,with_ds,seed", list(backward_draws(12, 7)))
def test_random_backward(B, T, C, dtype, gate, state, with_ds, seed):
    d = gen_backward(B, T, C, dtype, gate, state, with_ds, seed=seed % 100000)
    out = wkv.wkv_backward(d["w"], d["u"], d["k"], d["v"], d["r"], d["state"], dy=d["dy"], dstate_out=d["ds"])
    torch.cuda.synchronize()
    check_backward(d, out)
