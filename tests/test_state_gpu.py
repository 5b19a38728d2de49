"""wkv_state and wkv_state_combine against the oracle, and the T-sharded
forward's three steps emulated on one GPU.

wkv_state is the state a chunk leaves behind (no outputs); from the empty
state it is the chunk's summary.  wkv_state_combine folds summaries of
consecutive chunks onto a state.  A sequence split into chunks, each chunk's
entering state folded from the summaries of the chunks before it, and every
chunk run from there, must reproduce one pass over the whole sequence: that
is the T-sharded forward with its ranks played one after another on one
device (no cross-rank waits)."""
import numpy as np
import pytest
import torch

import oracle
import rwkv_wkv_recurrence_02_b200 as wkv
from rwkv_wkv_recurrence_02_b200 import inputs as I
from tests.parity import TOL, oracle_forward, output_error, sample_channels, state_error, to_np32, to_np64

pytestmark = pytest.mark.gpu

DEV = "cuda"


def gen(B, T, C, dtype, gate, state, seed, outliers=0.0):
    wl = I.Workload("st", B, T, C, "f32" if dtype == torch.float32 else "bf16", gate, -3.0, 1.0, 1.0, 1.0,
                    state, outlier_prob=outliers, outlier_mag=50.0, seed=seed)
    d = I.make_forward_inputs(wl, device="cpu")
    return {k: (None if v is None else v.to(DEV)) for k, v in d.items()}


@pytest.mark.parametrize("B,T,C,dtype,state,ws", [
    (2, 1, 64, torch.float32, True, True),
    (3, 16, 130, torch.bfloat16, True, True),     # sequential kernel
    (1, 700, 256, torch.float32, False, False),   # cluster kernel, no workspace
    (2, 3000, 512, torch.bfloat16, True, True),   # part kernel (look-back)
    (2, 3000, 512, torch.bfloat16, True, False),  # lane-resident over whole lane blocks
    (40, 500, 512, torch.float32, True, True),    # lane-resident
    (2, 999, 70, torch.float32, True, True),      # register-load look-back kernel
])
def test_state_matches_oracle(B, T, C, dtype, state, ws):
    d = gen(B, T, C, dtype, True, state, seed=B + T + C)
    s = wkv.wkv_state(d["w"], d["k"], d["v"], d["state"], use_workspace=ws)
    torch.cuda.synchronize()
    _, s_ref, _ = oracle_forward(d["w"], d["u"], d["k"], d["v"], None, d["state"])
    assert max(state_error(s, s_ref)) <= TOL[dtype]
    # in place, and the same state as the forward's
    st = d["state"].clone() if state else I.fresh_state(B, C, device=DEV)
    wkv.wkv_state(d["w"], d["k"], d["v"], st, state_out=st, use_workspace=ws)
    _, s_fwd = wkv.wkv_forward(d["w"], d["u"], d["k"], d["v"], d["r"], d["state"], use_workspace=ws)
    torch.cuda.synchronize()
    assert max(state_error(st, s_ref)) <= TOL[dtype]
    assert max(state_error(s_fwd, to_np64(st))) <= TOL[dtype]


def test_state_combine_matches_oracle():
    B, C, n = 3, 96, 5
    g = np.random.default_rng(3)
    w = torch.from_numpy(np.exp(g.uniform(-3, 1, C)).astype(np.float32))
    lens = [0, 1, 17, 300, 64]
    seg = np.zeros((n, 3, B, C), np.float32)
    seg[:, 0] = g.normal(0, 1, (n, B, C))
    seg[:, 1] = g.uniform(0.5, 2.0, (n, B, C))
    seg[:, 2] = g.uniform(-40, 40, (n, B, C))
    seg[0, 0], seg[0, 1], seg[0, 2] = 0.0, 0.0, -1e38      # an empty chunk's summary
    s0 = np.stack([g.normal(0, 1, (B, C)), g.uniform(0.5, 1.5, (B, C)), g.uniform(-5, 5, (B, C))]).astype(np.float32)
    out = wkv.wkv_state_combine(w.to(DEV), lens, torch.from_numpy(seg).to(DEV), torch.from_numpy(s0).to(DEV))
    torch.cuda.synchronize()
    ref = s0.astype(np.float64).copy()
    for j in range(n):
        for b in range(B):
            for c in range(C):
                p, a, bb = oracle.combine(float(w[c]), (ref[2, b, c], ref[0, b, c], ref[1, b, c]),
                                          (float(seg[j, 2, b, c]), float(seg[j, 0, b, c]), float(seg[j, 1, b, c])),
                                          lens[j])
                ref[0, b, c], ref[1, b, c], ref[2, b, c] = a, bb, p
    assert max(state_error(out, ref)) <= 2e-6
    # n = 0 passes the state through; the empty state from NULL
    same = wkv.wkv_state_combine(w.to(DEV), [], torch.from_numpy(seg).to(DEV), torch.from_numpy(s0).to(DEV))
    fresh = wkv.wkv_state_combine(w.to(DEV), [3], torch.from_numpy(seg[:1]).to(DEV))
    torch.cuda.synchronize()
    assert torch.equal(same.cpu(), torch.from_numpy(s0))
    assert torch.all(fresh[0] == 0) and torch.all(fresh[1] == 0) and torch.all(fresh[2] == -1e38)


@pytest.mark.parametrize("cuts,dtype,gate,ws", [
    ([0, 3000, 5000, 5001, 9000], torch.bfloat16, False, True),
    ([0, 100, 100, 1024, 2048], torch.float32, True, False),
    ([0, 20000, 40000, 65536], torch.bfloat16, False, True),
])
def test_tsharded_steps_on_one_gpu(cuts, dtype, gate, ws):
    """The T-sharded forward's steps for len(cuts)-1 ranks, played one after
    another: summaries (wkv_state), folds (wkv_state_combine), forwards from
    the folded states.  Equals one pass over the sequence."""
    T, C = cuts[-1], 512
    d = gen(1, T, C, dtype, gate, True, seed=len(cuts), outliers=1e-3)
    ops = __import__("rwkv_wkv_recurrence_02_b200.tshard", fromlist=["CudaOps"]).CudaOps(use_workspace=ws)
    chunk = lambda x, i: None if x is None else x[:, cuts[i]:cuts[i + 1]].contiguous()
    n = len(cuts) - 1
    summaries = torch.stack([ops.state(d["w"], chunk(d["k"], i), chunk(d["v"], i)) for i in range(n)])
    lens = [cuts[i + 1] - cuts[i] for i in range(n)]
    ys, states = [], []
    for i in range(n):
        entering = ops.combine(d["w"], lens[:i], summaries[:i].contiguous(), d["state"]) if i else d["state"]
        y, s = ops.forward(d["w"], d["u"], chunk(d["k"], i), chunk(d["v"], i), chunk(d["r"], i), entering, None)
        ys.append(y)
        states.append(s)
    torch.cuda.synchronize()
    y = torch.cat(ys, dim=1)
    idx = sample_channels(C, n=24)
    f = lambda x: None if x is None else x[..., idx.to(DEV)].contiguous()
    y_ref, s_ref, scale = oracle_forward(d["w"][idx.to(DEV)], d["u"][idx.to(DEV)], f(d["k"]), f(d["v"]), f(d["r"]),
                                         f(d["state"]))
    assert output_error(f(y), y_ref, scale) <= TOL[dtype]
    assert max(state_error(f(states[-1]), s_ref)) <= TOL[dtype]
