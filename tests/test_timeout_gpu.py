"""A cross-block wait that runs out is reported, not hung: with the wait limit
forced to 1 ns (environment knob read once per process) the look-back waits of
a 300-chunk launch expire before their predecessors publish.  The kernel must
record WKV_ERR_TIMEOUT in the workspace and write NaN for the affected
outputs, and the workspace must work again after a reset.  Runs in a child
process so the knob does not leak into other tests."""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r"""
import sys, torch
sys.path.insert(0, %r)
import rwkv_wkv_recurrence_02_b200 as wkv
from rwkv_wkv_recurrence_02_b200 import inputs as I
wl = I.Workload("t", 1, 64 * 300, 64, "f32", False, -3.0, 1.0, 1.0, 1.0, False, seed=5)
d = I.make_forward_inputs(wl, device="cuda")
ws = wkv.Workspace()
y, s = wkv.wkv_forward(d["w"], d["u"], d["k"], d["v"], workspace=ws)
st = ws.status()
print("STATUS", st, "NAN", bool(torch.isnan(y).any().item()))
ws.reset()
print("AFTER_RESET", ws.status())
"""


@pytest.mark.gpu
def test_expired_wait_is_reported():
    env = dict(os.environ, WKV_WAIT_LIMIT_NS="1", WKV_FORWARD_KERNEL="chunk")
    r = subprocess.run([sys.executable, "-c", CHILD % ROOT], env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    out = dict(zip(r.stdout.split()[::2], r.stdout.split()[1::2]))
    assert out["STATUS"] == "-7"           # WKV_ERR_TIMEOUT
    assert out["NAN"] == "True"            # affected outputs are NaN, not stale values
    assert out["AFTER_RESET"] == "0"
