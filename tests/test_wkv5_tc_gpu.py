"""The tensor-core form of wkv5_forward (bf16, heads of 64: blocks of tokens
as five 64 x 64 products per block, the default for those shapes) against
the fp64 oracle, with the
tolerances of tests/test_wkv5_gpu.py: 1e-2 of the output's magnitude scale
for the bf16 outputs, 2e-5 of the head's largest |S| for the state.

Decays large enough that a 64-token block would leave the range of its
factors make the kernel cut windows into blocks of 16, 4 or 1 token; those
cases are pinned here too, as are windows of one sequence that alternate
between the two (per-token decays staged in the state's tile, or read from
global memory), ragged windows, the carried state and the
fallback to the recurrent kernel for outputs it cannot store 16 bytes at a
time, and the full layer workloads.  The cases run in a child process, and
the same cases with WKV5_KERNEL=recurrent keep the CUDA-core recurrence
covered on these shapes."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r"""
import sys, torch
sys.path.insert(0, @ROOT@)
import rwkv_wkv_recurrence_02_b200 as wkv
from rwkv_wkv_recurrence_02_b200 import inputs as I
from tests.test_wkv5_gpu import TOL, case, check
BF = torch.bfloat16
DEV = "cuda"
res = []

def run(d, H, **kw):
    y, s = wkv.wkv5_forward(d["w"], d["u"], d["r"], d["k"], d["v"], H, d["state"], **kw)
    torch.cuda.synchronize()
    return y, s

# shapes: one token, one window, ragged windows, carried states, 64 windows
for (B, T, C, H, v6, st) in [(1, 1, 64, 1, False, False), (1, 1, 64, 1, True, True), (1, 64, 64, 1, True, True),
                            (2, 63, 128, 2, False, True),
                            (3, 200, 256, 4, True, True), (2, 1000, 512, 8, False, False),
                            (1, 4096, 128, 2, True, True)]:
    d = case(B, T, C, H, BF, v6, st, seed=B * 5 + T + C)
    y, s = run(d, H)
    res.append(("shape", check(d, H, y, s, TOL[BF])))

# decays large enough for blocks of 16, 4 and 1 token
for wmax, v6 in [(5.0, False), (20.0, False), (200.0, False), (12.0, True), (300.0, True)]:
    B, T, C, H = 2, 300, 128, 2
    d = case(B, T, C, H, BF, v6, True, seed=int(wmax) + v6)
    g = torch.Generator(device="cpu").manual_seed(int(wmax * 10))
    if v6:
        spikes = torch.rand(d["w"].shape, generator=g) < 0.05
        big = torch.rand(d["w"].shape, generator=g) * wmax
        d["w"] = torch.where(spikes.to(DEV), big.to(DEV), d["w"]).contiguous()
    else:
        sel = torch.rand(C, generator=g) < 0.25
        d["w"] = torch.where(sel.to(DEV), torch.full_like(d["w"], wmax), d["w"]).contiguous()
    y, s = run(d, H)
    res.append(("decay", check(d, H, y, s, TOL[BF])))

# per-token decays large in some windows only: a sequence's windows alternate between blocks of 64 tokens (the
# decays staged in the state's tile, the quarter sums) and shorter blocks (the decays read from global memory),
# while the other sequence keeps 64-token blocks throughout; the last window is ragged
B, T, C, H = 2, 5 * 64 + 17, 128, 2
d = case(B, T, C, H, BF, True, True, seed=71)
w = d["w"].clone()
w[1, 64:128] = 40.0          # sequence 1, window 1: blocks of one token
w[1, 192:256, :64] = 3.0     # window 3, head 0: blocks of 16
w[1, 320:, 64:] = 2.5        # the ragged last window, head 1
d["w"] = w.contiguous()
y, s = run(d, H)
res.append(("mixed", check(d, H, y, s, TOL[BF])))

# calls of 1, 63, 64, 65 and 307 tokens chained in place, and one call
B, T, C, H = 2, 500, 128, 2
d = case(B, T, C, H, BF, True, True, seed=61)
st = d["state"].clone()
ys = []
for a, b in [(0, 1), (1, 64), (64, 128), (128, 193), (193, 500)]:
    sl = lambda x: x[:, a:b].contiguous()
    y, _ = wkv.wkv5_forward(sl(d["w"]), d["u"], sl(d["r"]), sl(d["k"]), sl(d["v"]), H, st, state_out=st)
    ys.append(y)
torch.cuda.synchronize()
res.append(("chain", check(d, H, torch.cat(ys, dim=1), st, TOL[BF])))

# outputs only 2-byte aligned: the recurrent kernel takes them
B, T, C, H = 1, 100, 128, 2
d = case(B, T, C, H, BF, False, True, seed=67)
ybuf = torch.empty(B * T * C + 1, dtype=BF, device=DEV)
y = ybuf[1:].view(B, T, C)
s = torch.empty_like(d["state"])
run(d, H, y=y, state_out=s)
res.append(("unaligned", check(d, H, y, s, TOL[BF])))

# the full layer workloads on sampled (sequence, head) pairs
for name in ("v5_layer", "v6_layer"):
    wl = I.MATRIX_WORKLOADS[name]
    d = I.make_matrix_inputs(wl, device=DEV)
    y, s = wkv.wkv5_forward(d["w"], d["u"], d["r"], d["k"], d["v"], wl.H)
    torch.cuda.synchronize()
    N = wl.C // wl.H
    for b, h in [(0, 0), (3, 17), (5, 4), (7, 31)]:
        cs = slice(h * N, (h + 1) * N)
        sub = {k: x[b:b + 1, :, cs].contiguous() for k, x in d.items() if k in ("r", "k", "v")}
        sub["w"] = d["w"][b:b + 1, :, cs].contiguous() if wl.per_token_decay else d["w"][cs].contiguous()
        sub["u"] = d["u"][cs].contiguous()
        sub["state"] = None
        res.append((name, check(sub, 1, y[b:b + 1, :, cs], s[b:b + 1, h:h + 1], TOL[BF])))
for name, err in res:
    print("OK", name, err)
"""


@pytest.mark.parametrize("kernel", ["tensor cores", "recurrent"])
def test_matrix_state_kernels_match_the_oracle(kernel):
    env = dict(os.environ)
    env.pop("WKV5_KERNEL", None)
    if kernel == "recurrent":
        env["WKV5_KERNEL"] = "recurrent"
    r = subprocess.run([sys.executable, "-c", CHILD.replace("@ROOT@", repr(ROOT))], env=env, capture_output=True,
                       text=True, timeout=900, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-3000:]
    assert r.stdout.count("OK ") == 7 + 5 + 1 + 1 + 1 + 8, r.stdout
