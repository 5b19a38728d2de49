"""The T-sharded forward's exchange, with ranks on CPU (gloo).

One sequence is cut into consecutive chunks, one per rank; every rank runs
forward_tsharded on its chunk.  The per-rank arithmetic (chunk summary, fold
of summaries, forward from a state) is the fp64 oracle's here, injected
through ``ops``, so what is checked is the exchange itself: that every rank
gathers the lengths and summaries in rank order, folds exactly the chunks
before its own with their own lengths, and starts its chunk from the result.
The concatenated outputs and the last rank's state must equal one oracle
pass over the whole sequence.  (The CUDA steps are checked against the
oracle on the GPU by tests/test_state_gpu.py.)
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle


class OracleOps:
    """The three per-rank steps in fp64 by the oracle."""

    def state(self, w, k, v):
        C = k.shape[2]
        _, st = oracle.wkv_forward(w.numpy(), np.zeros(C, np.float32), k.numpy(), v.numpy())
        return torch.from_numpy(st)

    def combine(self, w, lens, states, state_in):
        _, B, C = states.shape[1:]
        s = oracle.fresh_state(B, C) if state_in is None else state_in.numpy().astype(np.float64)
        s = s.copy()
        for j, n in enumerate(lens):
            x = states[j].numpy()
            for b in range(B):
                for c in range(C):
                    p, a, bb = oracle.combine(float(w[c]), (s[2, b, c], s[0, b, c], s[1, b, c]),
                                              (x[2, b, c], x[0, b, c], x[1, b, c]), n)
                    s[0, b, c], s[1, b, c], s[2, b, c] = a, bb, p
        return torch.from_numpy(s)

    def forward(self, w, u, k, v, r, state_in, y):
        yy, st = oracle.wkv_forward(w.numpy(), u.numpy(), k.numpy(), v.numpy(),
                                    None if r is None else r.numpy(),
                                    None if state_in is None else state_in.numpy())
        return torch.from_numpy(yy), torch.from_numpy(st)


def make_sequence(B, T, C, gate, seed):
    g = np.random.default_rng(seed)
    w = np.exp(g.uniform(-3, 1, C)).astype(np.float32)
    u = g.normal(0, 1, C).astype(np.float32)
    k = g.normal(0, 1, (B, T, C)).astype(np.float32)
    k[g.random((B, T, C)) < 0.01] = 50.0
    v = g.normal(0, 1, (B, T, C)).astype(np.float32)
    r = g.normal(0, 1, (B, T, C)).astype(np.float32) if gate else None
    p = g.uniform(-5, 5, (B, C))
    b = g.uniform(0.5, 1.5, (B, C))
    s0 = np.stack([b * g.normal(0, 1, (B, C)), b, p])
    return w, u, k, v, r, s0


def _worker(rank, world, port, cuts, gate, seed, out_q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from rwkv_wkv_recurrence_02_b200.tshard import forward_tsharded
        B, T, C = 2, cuts[-1], 5
        w, u, k, v, r, s0 = make_sequence(B, T, C, gate, seed)
        a, b = cuts[rank], cuts[rank + 1]
        t = lambda x: None if x is None else torch.from_numpy(np.ascontiguousarray(x[:, a:b]))
        y, s = forward_tsharded(torch.from_numpy(w), torch.from_numpy(u), t(k), t(v), t(r), torch.from_numpy(s0),
                                ops=OracleOps())
        out_q.put((rank, y.numpy(), s.numpy()))
    finally:
        dist.destroy_process_group()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("cuts,gate", [([0, 70, 160], True), ([0, 50, 50, 137], False), ([0, 1, 2, 90, 91], True)])
def test_tsharded_equals_one_pass(cuts, gate):
    world = len(cuts) - 1
    seed = sum(cuts)
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, cuts, gate, seed, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = dict()
    for _ in range(world):
        rank, y, s = q.get(timeout=240)
        got[rank] = (y, s)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    B, T, C = 2, cuts[-1], 5
    w, u, k, v, r, s0 = make_sequence(B, T, C, gate, seed)
    y_ref, s_ref = oracle.wkv_forward(w, u, k, v, r, s0)
    y = np.concatenate([got[i][0] for i in range(world)], axis=1)
    assert y.shape == y_ref.shape
    np.testing.assert_allclose(y, y_ref, rtol=1e-9, atol=1e-12)
    # every rank's state is the state after its own last token
    for i in range(world):
        _, s_i = oracle.wkv_forward(w, u, k[:, :cuts[i + 1]], v[:, :cuts[i + 1]],
                                    None if r is None else r[:, :cuts[i + 1]], s0)
        np.testing.assert_allclose(oracle.represented(got[i][1])[0], oracle.represented(s_i)[0], rtol=1e-9,
                                   atol=1e-9)
        np.testing.assert_allclose(oracle.represented(got[i][1])[2], oracle.represented(s_i)[2], rtol=1e-9,
                                   atol=1e-9)
    np.testing.assert_allclose(got[world - 1][1][2], s_ref[2], rtol=1e-12, atol=1e-9)


def test_a_misordered_fold_is_caught():
    """The check above would see a fold in the wrong order: chunks folded
    last-to-first give a different entering state."""
    B, T, C = 1, 120, 3
    w, u, k, v, r, s0 = make_sequence(B, T, C, False, 5)
    ops = OracleOps()
    cut = [0, 40, 80, 120]
    summ = [ops.state(torch.from_numpy(w), torch.from_numpy(np.ascontiguousarray(k[:, a:b])),
                      torch.from_numpy(np.ascontiguousarray(v[:, a:b]))) for a, b in zip(cut[:-1], cut[1:])]
    good = ops.combine(torch.from_numpy(w), [40, 40], torch.stack(summ[:2]), torch.from_numpy(s0)).numpy()
    bad = ops.combine(torch.from_numpy(w), [40, 40], torch.stack(summ[:2][::-1]), torch.from_numpy(s0)).numpy()
    _, ref = oracle.wkv_forward(w, u, k[:, :80], v[:, :80], None, s0)
    assert np.allclose(oracle.represented(good)[2], oracle.represented(ref)[2], rtol=1e-9)
    assert not np.allclose(oracle.represented(bad)[2], oracle.represented(ref)[2], rtol=1e-6)
