"""wkv_forward_noalloc: the entry point for callers that cannot allocate
device memory (plug-ins whose host owns every allocation, runtimes that hand
out only pre-registered buffers).  Its cross-block scratch is a fixed array
inside the library, so it must give the same results as wkv_forward with a
caller workspace, call after call, and refuse problems larger than that
array.  Calls whose sequences fit one cluster of parts use no scratch at
all.  This file is collected last on purpose."""
import ctypes

import pytest
import torch

import rwkv_wkv_recurrence_02_b200 as wkv
from rwkv_wkv_recurrence_02_b200 import inputs as I
from tests.parity import TOL, oracle_forward, output_error, state_error, to_np64

WKV_ERR_SCRATCH = -9
SCRATCH_MAX = 32 << 20


def case(B, T, C, dtype, seed):
    wl = I.Workload("noalloc", B, T, C, "f32" if dtype == torch.float32 else "bf16", True, -3.0, 1.0, 1.0, 1.0,
                    True, seed=seed)
    d = I.make_forward_inputs(wl, device="cpu")
    return {k: (None if x is None else x.to("cuda")) for k, x in d.items()}


@pytest.mark.gpu
@pytest.mark.parametrize("B,T,C,dtype", [(3, 700, 130, torch.float32), (2, 1100, 96, torch.bfloat16),
                                         (1, 333, 7, torch.float32)])
def test_noalloc_matches_workspace_entry_point(B, T, C, dtype):
    d = case(B, T, C, dtype, seed=B + T + C)
    need = wkv.lib().wkv_forward_noalloc_scratch_bytes(B, T, C, 0 if dtype == torch.float32 else 1)
    assert 0 < need <= SCRATCH_MAX          # the call really uses the built-in scratch
    y_ref, s_ref = wkv.wkv_forward(d["w"], d["u"], d["k"], d["v"], d["r"], d["state"])
    scale = oracle_forward(d["w"], d["u"], d["k"], d["v"], d["r"], d["state"])[2]
    for _ in range(2):                      # two calls in a row share the array
        y = torch.full_like(y_ref, float("nan"))
        s = torch.full_like(s_ref, float("nan"))
        wkv.wkv_forward_noalloc(d["w"], d["u"], d["k"], d["v"], d["r"], d["state"], y=y, state_out=s)
        torch.cuda.synchronize()
        assert output_error(y, to_np64(y_ref), scale) <= TOL[dtype]
        assert max(state_error(s, to_np64(s_ref))) <= TOL[dtype]


@pytest.mark.gpu
def test_noalloc_cluster_calls_share_nothing():
    """Calls that fit the cluster kernel use no scratch: two of them running
    at the same time on unordered streams, each far beyond the built-in
    array's size limit, both give the oracle's results."""
    B, T, C = 17, 1024, 4096
    assert wkv.lib().wkv_forward_noalloc_scratch_bytes(B, T, C, 1) > SCRATCH_MAX
    cases = [case(B, T, C, torch.bfloat16, seed=s) for s in (11, 12)]
    outs = [(torch.empty_like(d["k"]), torch.empty((3, B, C), device="cuda")) for d in cases]
    torch.cuda.synchronize()
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    for d, (y, s), st in zip(cases, outs, streams):
        with torch.cuda.stream(st):
            wkv.wkv_forward_noalloc(d["w"], d["u"], d["k"], d["v"], d["r"], d["state"], y=y, state_out=s)
    torch.cuda.synchronize()
    idx = torch.arange(0, C, 97)
    for d, (y, s) in zip(cases, outs):
        y_ref, s_ref, scale = oracle_forward(d["w"][idx], d["u"][idx], d["k"][..., idx], d["v"][..., idx],
                                             d["r"][..., idx], d["state"][..., idx])
        assert output_error(y[..., idx.cuda()], y_ref, scale) <= TOL[torch.bfloat16]
        assert max(state_error(s[..., idx.cuda()], s_ref)) <= TOL[torch.bfloat16]


@pytest.mark.gpu
def test_noalloc_rejects_problems_beyond_its_scratch():
    B, T, C = 64, 65536, 4096
    assert wkv.lib().wkv_forward_noalloc_scratch_bytes(B, T, C, 1) > SCRATCH_MAX
    base = 1 << 44   # never dereferenced: the size check comes first (arrays 1 TiB apart)
    rc = wkv.lib().wkv_forward_noalloc(B, T, C, 1, base, base + 65536, base + (1 << 40), base + (2 << 40), None,
                                       None, base + (3 << 40), None, None)
    assert rc == WKV_ERR_SCRATCH
