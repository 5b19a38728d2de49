"""Chunk chains (WKV_FLAG_CHAIN_BEGIN / WKV_FLAG_CHAIN_NEXT): each call of a
chain takes its entering state from the word the previous call publishes in
the workspace, instead of waiting for the previous kernel to end.  The
results must be those of the plain chunk calls: the oracle over the whole
sequence, in eager launches and in a replayed CUDA graph; a broken chain (a
foreign state, another call on the workspace) must fall back to reading
state_in; and a word that never comes must time out with NaN and
WKV_ERR_TIMEOUT instead of hanging."""
import os
import subprocess
import sys

import pytest
import torch

import rwkv_wkv_recurrence_02_b200 as wkv
from tests.test_parity_gpu import check_forward, gen_case

pytestmark = pytest.mark.gpu

DEV = "cuda"
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def chunked(d, n, T):
    """d's k, v, r cut into n contiguous chunks of T tokens (the last may be
    shorter), and one output buffer per chunk."""
    Ttot = d["k"].shape[1]
    sls = [slice(i * T, min((i + 1) * T, Ttot)) for i in range(n)]
    pick = (lambda x, sl: None if x is None else x[:, sl].contiguous())
    return [(pick(d["k"], sl), pick(d["v"], sl), pick(d["r"], sl), torch.empty_like(d["k"][:, sl])) for sl in sls]


def run_chain(d, n, T, ws, parts=None, state=None, first="begin"):
    """n chunk calls of T tokens over d's sequence, the state carried in
    place; returns the outputs joined along T and the state."""
    if state is None:
        state = d["state"].clone()
    parts = chunked(d, n, T) if parts is None else parts
    for i, (k, v, r, y) in enumerate(parts):
        wkv.wkv_forward(d["w"], d["u"], k, v, r, state, y=y, state_out=state, workspace=ws,
                        chain=first if i == 0 else "next")
    return torch.cat([p[3] for p in parts], dim=1), state


CHAINS = [
    # n, T, B, C, dtype, gate: the last chunk of the ragged cases is shorter
    (12, 1024, 1, 512, torch.bfloat16, False),
    (6, 1000, 2, 200, torch.float32, True),
    (5, 2048, 1, 4096, torch.bfloat16, False),
    (7, 300, 3, 72, torch.bfloat16, True),
]


@pytest.mark.parametrize("n,T,B,C,dtype,gate", CHAINS)
def test_chain_equals_oracle(n, T, B, C, dtype, gate):
    total = n * T - (T // 3 if T % 2 == 0 else 0)
    d = gen_case(B, total, C, dtype, gate, True, seed=n * 31 + C)
    d["k"][:, ::997] = 50.0    # outliers: the exact path inside a chain
    ws = wkv.Workspace()
    y, s = run_chain(d, n, T, ws)
    torch.cuda.synchronize()
    assert ws.status() == 0
    check_forward(d, y, s)


def test_chain_matches_plain_calls():
    """The chained calls run the same kernel as plain calls with
    WKV_FLAG_INPUTS_READY; only the hand-off differs (the published word
    carries the base-2 exponent the plain path converts to and from natural
    units), so outputs agree to rounding."""
    n, T, C = 8, 1024, 4096
    d = gen_case(1, n * T, C, torch.bfloat16, False, True, seed=3)
    ws = wkv.Workspace()
    y_c, s_c = run_chain(d, n, T, ws)
    s_p = d["state"].clone()
    y_p = torch.empty_like(d["k"])
    for i in range(n):
        sl = slice(i * T, (i + 1) * T)
        wkv.wkv_forward(d["w"], d["u"], d["k"][:, sl], d["v"][:, sl], None, s_p, y=y_p[:, sl], state_out=s_p,
                        workspace=ws, inputs_ready=True)
    torch.cuda.synchronize()
    diff = (y_c.float() - y_p.float()).abs()
    assert diff.max().item() <= 1e-2 * max(1.0, y_p.float().abs().max().item())
    torch.testing.assert_close(s_c, s_p, rtol=1e-4, atol=1e-6)


def test_chain_in_cuda_graph_replays():
    """A captured chain (its first call clears the words by a memset node)
    replays to the eager chain's results, every replay from the reset state."""
    n, T, C = 16, 1024, 2048
    d = gen_case(1, n * T, C, torch.bfloat16, False, True, seed=11)
    ws = wkv.Workspace()
    y_e, s_e = run_chain(d, n, T, ws)
    torch.cuda.synchronize()
    fresh = d["state"].clone()
    state = fresh.clone()
    parts = chunked(d, n, T)
    run_chain(d, n, T, ws, parts=parts, state=state)   # warm the launch configuration outside the capture
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            state.copy_(fresh)
            run_chain(d, n, T, ws, parts=parts, state=state)
    torch.cuda.current_stream().wait_stream(s)
    for _ in range(3):
        for p in parts:
            p[3].zero_()
        state.fill_(float("nan"))
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(torch.cat([p[3] for p in parts], dim=1), y_e)
        assert torch.equal(state, s_e)
    assert ws.status() == 0
    del g


def test_broken_chains_fall_back_to_state_in():
    """A 'next' call whose state_in is not the previous state_out, and one
    after another call on the same workspace, read state_in: still exact."""
    n, T, C = 6, 1024, 512
    d = gen_case(1, n * T, C, torch.bfloat16, True, True, seed=21)
    ws = wkv.Workspace()
    state = d["state"].clone()
    y = torch.empty_like(d["k"])

    def call(i, chain, st_in, st_out):
        sl = slice(i * T, (i + 1) * T)
        wkv.wkv_forward(d["w"], d["u"], d["k"][:, sl], d["v"][:, sl], d["r"][:, sl], st_in, y=y[:, sl],
                        state_out=st_out, workspace=ws, chain=chain)

    call(0, "begin", state, state)
    call(1, "next", state, state)
    moved = state.clone()                     # a foreign buffer holding the same state
    call(2, "next", moved, moved)             # no matching predecessor: reads state_in
    call(3, "next", moved, moved)
    other = gen_case(1, 300, 64, torch.float32, False, True, seed=2)
    wkv.wkv_forward(other["w"], other["u"], other["k"], other["v"], None, other["state"], workspace=ws)
    call(4, "next", moved, moved)             # the workspace served another call in between
    call(5, "next", moved, moved)
    torch.cuda.synchronize()
    assert ws.status() == 0
    check_forward(d, y, moved)


def test_two_chains_interleaved_on_one_stream():
    """Two chains with their own workspaces and states, their calls
    alternating on one stream."""
    n, T, C = 5, 1024, 256
    a = gen_case(1, n * T, C, torch.bfloat16, False, True, seed=41)
    b = gen_case(2, n * T, C, torch.float32, True, False, seed=42)
    wa, wb = wkv.Workspace(), wkv.Workspace()
    sa = a["state"].clone()
    sb = torch.empty((3, 2, C), device=DEV)
    pa, pb = chunked(a, n, T), chunked(b, n, T)
    for i in range(n):
        ch = "begin" if i == 0 else "next"
        k, v, _, y = pa[i]
        wkv.wkv_forward(a["w"], a["u"], k, v, None, sa, y=y, state_out=sa, workspace=wa, chain=ch)
        k, v, r, y = pb[i]
        wkv.wkv_forward(b["w"], b["u"], k, v, r, None if i == 0 else sb, y=y, state_out=sb, workspace=wb, chain=ch)
    torch.cuda.synchronize()
    check_forward(a, torch.cat([p[3] for p in pa], dim=1), sa)
    check_forward(b, torch.cat([p[3] for p in pb], dim=1), sb)


def test_flag_validation():
    d = gen_case(1, 64, 64, torch.float32, False, False, seed=1)
    with pytest.raises(ValueError):
        wkv.wkv_forward(d["w"], d["u"], d["k"], d["v"], chain="middle")
    L = wkv.lib()
    st = L.wkv_forward_ex(1, 64, 64, 0, d["w"].data_ptr(), d["u"].data_ptr(), d["k"].data_ptr(), d["v"].data_ptr(),
                          None, None, torch.empty_like(d["k"]).data_ptr(), None, None, 0,
                          wkv.WKV_FLAG_CHAIN_BEGIN | wkv.WKV_FLAG_CHAIN_NEXT, None)
    assert wkv.STATUS[st] == "WKV_ERR_SHAPE"


MISSING_WORD = r"""
import sys, torch
sys.path.insert(0, %r)
import rwkv_wkv_recurrence_02_b200 as wkv
from rwkv_wkv_recurrence_02_b200 import inputs as I
T, C = 1024, 512
wl = I.Workload("t", 1, 2 * T, C, "bf16", False, -3.0, 1.0, 1.0, 1.0, True, seed=5)
d = I.make_forward_inputs(wl, device="cuda")
ws = wkv.Workspace()
state = d["state"].clone()
y = torch.empty_like(d["k"])
wkv.wkv_forward(d["w"], d["u"], d["k"][:, :T], d["v"][:, :T], None, state, y=y[:, :T], state_out=state,
                workspace=ws, chain="begin")
torch.cuda.synchronize()
# wipe the published words behind the library's back: the next call's word never comes
base = ws._aligned_ptr() - ws.buf.data_ptr()
ws.buf[base + 256: base + 256 + 16 * C].zero_()
wkv.wkv_forward(d["w"], d["u"], d["k"][:, T:], d["v"][:, T:], None, state, y=y[:, T:], state_out=state,
                workspace=ws, chain="next")
torch.cuda.synchronize()
print("STATUS", ws.status(), "NAN", bool(torch.isnan(y[:, T:].float()).all().item()),
      "STATE_NAN", bool(torch.isnan(state[:2]).all().item()))
ws.reset()
print("AFTER_RESET", ws.status())
"""


def test_missing_word_times_out():
    """The wait for the previous call's word is bounded (the limit forced to
    1 ms here): the call records WKV_ERR_TIMEOUT and writes NaN outputs and
    a NaN state (its a and b; the exponent of a NaN state is not defined).  Runs in a child process so the limit does not leak."""
    env = dict(os.environ, WKV_WAIT_LIMIT_NS="1000000")
    r = subprocess.run([sys.executable, "-c", MISSING_WORD % ROOT], env=env, capture_output=True, text=True,
                       timeout=300)
    assert r.returncode == 0, r.stderr
    out = dict(zip(r.stdout.split()[::2], r.stdout.split()[1::2]))
    assert out["STATUS"] == "-7"           # WKV_ERR_TIMEOUT
    assert out["NAN"] == "True" and out["STATE_NAN"] == "True"
    assert out["AFTER_RESET"] == "0"


# Calls longer than one stream launch (8 parts) with few lane blocks and a
# workspace: ungated bfloat16 calls with at least 48 lane blocks run as a
# chain of 4-part launches (forced with WKV_FORWARD_KERNEL=stream for the
# others in test_forced_kernels_gpu.py).
LONG = [
    # B, T, C, dtype, gate, state
    (1, 5000, 4096, torch.bfloat16, False, True),     # 5 launches, the last one ragged
    (1, 2049, 4096, torch.bfloat16, False, False),    # one token past a single launch
    (2, 3000, 2048, torch.bfloat16, False, True),
    (1, 9000, 3100, torch.bfloat16, False, True),     # ragged channel block (49 lane blocks)
]


@pytest.mark.parametrize("B,T,C,dtype,gate,state", LONG)
def test_long_call_equals_oracle(B, T, C, dtype, gate, state):
    d = gen_case(B, T, C, dtype, gate, state, seed=T + C)
    d["k"][:, ::991] = 50.0
    ws = wkv.Workspace()
    y, s = wkv.wkv_forward(d["w"], d["u"], d["k"], d["v"], d["r"], d["state"], workspace=ws)
    torch.cuda.synchronize()
    assert ws.status() == 0
    check_forward(d, y, s)
    # the state alone (no outputs) takes the same launches
    s2 = wkv.wkv_state(d["w"], d["k"], d["v"], d["state"], workspace=ws)
    torch.cuda.synchronize()
    torch.testing.assert_close(s2, s, rtol=1e-5, atol=1e-6)


def test_long_calls_in_a_chain():
    """A chain whose calls are themselves several launches long: positions
    continue across the calls."""
    T1, T2, T3, C = 5000, 3001, 4096, 4096
    d = gen_case(1, T1 + T2 + T3, C, torch.bfloat16, False, True, seed=77)
    ws = wkv.Workspace()
    state = d["state"].clone()
    ys = []
    for i, (a, b) in enumerate(((0, T1), (T1, T1 + T2), (T1 + T2, T1 + T2 + T3))):
        k, v = d["k"][:, a:b].contiguous(), d["v"][:, a:b].contiguous()
        y, _ = wkv.wkv_forward(d["w"], d["u"], k, v, None, state, state_out=state, workspace=ws,
                               chain="begin" if i == 0 else "next")
        ys.append(y)
    torch.cuda.synchronize()
    assert ws.status() == 0
    check_forward(d, torch.cat(ys, dim=1), state)
