"""A cross-block wait that runs out is reported, not hung: with the wait limit
forced to 1 ns (environment knob read once per process), the look-back waits
of the kernels whose CTAs wait on one another expire before their
predecessors publish.  The kernel must record WKV_ERR_TIMEOUT in the workspace and write
NaN for the affected outputs, and the workspace must work again after a
reset.  Waits for a CTA's own TMA copies keep their fixed limit, so no copy is
left in flight.  Each case runs in a child process so the knob does not leak
into other tests."""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

FORWARD = r"""
import sys, torch
sys.path.insert(0, %r)
import rwkv_wkv_recurrence_02_b200 as wkv
from rwkv_wkv_recurrence_02_b200 import inputs as I
B, T, C = %d, %d, %d
wl = I.Workload("t", B, T, C, "f32", False, -3.0, 1.0, 1.0, 1.0, False, seed=5)
d = I.make_forward_inputs(wl, device="cuda")
ws = wkv.Workspace()
y, s = wkv.wkv_forward(d["w"], d["u"], d["k"], d["v"], workspace=ws)
st = ws.status()
print("STATUS", st, "NAN", bool(torch.isnan(y).any().item()))
ws.reset()
print("AFTER_RESET", ws.status())
"""

# The two look-back kernels: parts and chunks of one lane block run in
# different CTAs at the same time, so a part waits for the ones before it.
# The lane-resident forward and the reverse walk hand one state between
# neighbouring CTAs, but a CTA publishes its word from its first work item and
# reads its neighbour's only in its last, so that word is there by then and a
# 1 ns limit cannot expire it; its wait is the same bounded loop.
CASES = [
    # name, script, forced kernel, (B, T, C)
    ("register-load look-back", FORWARD, "chunk", (1, 64 * 300, 64)),
    ("part kernel look-back", FORWARD, "part", (1, 64 * 300, 64)),
]


@pytest.mark.gpu
@pytest.mark.parametrize("name,script,kernel,shape", CASES, ids=[c[0] for c in CASES])
def test_expired_wait_is_reported(name, script, kernel, shape):
    env = dict(os.environ, WKV_WAIT_LIMIT_NS="1")
    if kernel is not None:
        env["WKV_FORWARD_KERNEL"] = kernel
    r = subprocess.run([sys.executable, "-c", script % ((ROOT,) + shape)], env=env, capture_output=True, text=True,
                       timeout=300)
    assert r.returncode == 0, r.stderr
    out = dict(zip(r.stdout.split()[::2], r.stdout.split()[1::2]))
    assert out["STATUS"] == "-7"           # WKV_ERR_TIMEOUT
    assert out["NAN"] == "True"            # affected outputs are NaN, not stale values
    assert out["AFTER_RESET"] == "0"


NOALLOC = r"""
import sys, torch
sys.path.insert(0, %r)
import rwkv_wkv_recurrence_02_b200 as wkv
from rwkv_wkv_recurrence_02_b200 import inputs as I
B, T, C = %d, %d, %d
wl = I.Workload("t", B, T, C, "f32", False, -3.0, 1.0, 1.0, 1.0, False, seed=5)
d = I.make_forward_inputs(wl, device="cuda")
print("BEFORE", wkv.wkv_forward_noalloc_status())
y = torch.empty_like(d["k"])
wkv.wkv_forward_noalloc(d["w"], d["u"], d["k"], d["v"], y=y)
print("STATUS", wkv.wkv_forward_noalloc_status(), "NAN", bool(torch.isnan(y).any().item()))
"""


@pytest.mark.gpu
def test_noalloc_expired_wait_is_reported():
    """The allocation-free entry point keeps its error word in the built-in
    array; wkv_forward_noalloc_status reads it.  C = 130 (not a multiple of
    4) takes the register-load look-back kernel, whose chunks wait on one
    another."""
    env = dict(os.environ, WKV_WAIT_LIMIT_NS="1")
    env.pop("WKV_FORWARD_KERNEL", None)
    r = subprocess.run([sys.executable, "-c", NOALLOC % (ROOT, 1, 64 * 300, 130)], env=env, capture_output=True,
                       text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    out = dict(zip(r.stdout.split()[::2], r.stdout.split()[1::2]))
    assert out["BEFORE"] == "0"            # nothing has used the array yet
    assert out["STATUS"] == "-7"           # WKV_ERR_TIMEOUT
    assert out["NAN"] == "True"
