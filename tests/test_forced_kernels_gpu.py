"""Each forward kernel outside the shapes that select it: a child process
forces one kernel (environment knob read once per process), runs a list of
shapes through wkv_forward and saves the results; this process compares them
with the oracle on the same seeded inputs.

- part: short sequences of few lane blocks, which take the cluster kernel
  when the call brings no workspace (at most 64 tokens need none);
- cluster: few lane blocks (where the stream kernel runs) and many (more
  clusters than fit the GPU at once), which with a workspace take the
  lane-resident kernel;
- stream: many lane blocks, which take the lane-resident kernel; and calls
  longer than one launch that are gated, float32 or have few lane blocks,
  which take the part kernel (forced, they run as a chain of launches).
"""
import os
import subprocess
import sys

import pytest
import torch

from tests.test_parity_gpu import check_forward, gen_case

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r"""
import sys, torch
sys.path.insert(0, %r)
import rwkv_wkv_recurrence_02_b200 as wkv
from tests.test_parity_gpu import gen_case
cases, out = %r, %r
res = []
for (B, T, C, dt, gate, state, seed) in cases:
    d = gen_case(B, T, C, getattr(torch, dt), gate, state, seed=seed)
    y, s = wkv.wkv_forward(d["w"], d["u"], d["k"], d["v"], d["r"], d["state"])
    torch.cuda.synchronize()
    res.append((y.cpu(), s.cpu()))
torch.save(res, out)
"""

FORCED = {
    "part": [
        # B, T, C, dtype, gate, state
        (1, 17, 64, "float32", True, True),
        (1, 64, 64, "bfloat16", False, True),
        (1, 65, 128, "float32", True, False),
        (1, 129, 128, "float32", True, False),
        (2, 1000, 72, "bfloat16", True, True),
        (3, 777, 1000, "bfloat16", False, True),
    ],
    "cluster": [
        (1, 100, 64, "float32", True, True),         # few lane blocks (where the stream kernel runs by default)
        (2, 1000, 72, "bfloat16", True, True),
        (1, 1024, 4096, "bfloat16", False, True),
        (40, 130, 256, "bfloat16", True, False),     # 160 lane blocks
        (160, 64, 64, "float32", False, True),
        (300, 40, 64, "bfloat16", True, True),
        (5, 1000, 3840, "float32", True, True),      # 300 clusters of 8 CTAs
        (7, 130, 2728, "bfloat16", True, True),      # ragged channel block
    ],
    "stream": [
        (40, 130, 256, "bfloat16", True, False),     # 160 lane blocks: more clusters than fit at once
        (300, 40, 64, "bfloat16", True, True),
        (5, 1000, 3840, "float32", True, True),      # 300 clusters of 8 CTAs
        (7, 130, 2728, "bfloat16", True, True),      # ragged channel block
        (3, 2048, 4096, "bfloat16", False, True),    # 8 parts of 256 tokens, 192 lane blocks
        (2, 3000, 128, "float32", True, True),       # a chain of six 512-token launches
        (1, 5000, 256, "bfloat16", True, False),     # five 1024-token launches, the last ragged
        (3, 2500, 72, "bfloat16", False, True),      # ragged channel block
    ],
}


@pytest.mark.parametrize("kernel", sorted(FORCED))
def test_forced_kernel_matches_oracle(kernel, tmp_path):
    cases = [c + (c[0] * 19 + c[1] + c[2],) for c in FORCED[kernel]]
    out = str(tmp_path / "res.pt")
    env = dict(os.environ, WKV_FORWARD_KERNEL=kernel)
    r = subprocess.run([sys.executable, "-c", CHILD % (ROOT, cases, out)], env=env, capture_output=True, text=True,
                       timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    res = torch.load(out)
    for (B, T, C, dt, gate, state, seed), (y, s) in zip(cases, res):
        d = gen_case(B, T, C, getattr(torch, dt), gate, state, seed=seed, device="cpu")
        check_forward(d, y, s)
