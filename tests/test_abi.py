"""The C ABI on the host: the library loads without a GPU, exports every
function include/wkv.h declares, and rejects bad arguments before launching
anything (these calls return before any CUDA runtime call)."""
import ctypes
import os
import re

import pytest

import rwkv_wkv_recurrence_02_b200 as wkv

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "wkv.h")

OK, NULLPTR, SHAPE, DTYPE, ALIGN, ALIAS, CUDA, TIMEOUT, WORKSPACE = 0, -1, -2, -3, -4, -5, -6, -7, -8
F32, BF16 = 0, 1
# fake, well-aligned device addresses: every call below must fail validation
# (or be a no-op) before it could dereference them
BASE = 1 << 40


def _gpu_present():
    try:
        import torch
        return torch.cuda.is_available()
    except Exception:
        return True


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[a-z_0-9]+\s*\**\s*(wkv[0-9]*_[a-z_0-9]+)\s*\(", text, flags=re.M)))


@pytest.fixture(scope="module")
def L():
    return wkv.lib()


def test_header_declares_the_binding_exports():
    assert declared_functions() == sorted(wkv.EXPORTS)


def test_library_exports_every_declared_symbol(L):
    for name in declared_functions():
        assert hasattr(L, name), name
    # and through dlsym of the raw handle, not just the ctypes cache
    raw = ctypes.CDLL(wkv.LIB_PATH)
    for name in declared_functions():
        assert ctypes.cast(getattr(raw, name), ctypes.c_void_p).value


def test_abi_version_and_strerror(L):
    assert L.wkv_abi_version() == 1
    msgs = {L.wkv_strerror(s).decode() for s in (OK, NULLPTR, SHAPE, DTYPE, ALIGN, ALIAS, CUDA, TIMEOUT, WORKSPACE)}
    assert len(msgs) == 9
    assert L.wkv_strerror(12345).decode() == "unknown wkv status"


def fwd(L, B=2, T=100, C=64, dt=F32, w=BASE, u=BASE + 4096, k=BASE + (1 << 30), v=BASE + (2 << 30),
        r=None, s_in=None, y=BASE + (3 << 30), s_out=None, ws=None, ws_bytes=0):
    return L.wkv_forward(B, T, C, dt, w, u, k, v, r, s_in, y, s_out, ws, ws_bytes, None)


def test_forward_rejects_bad_dtype_and_shapes(L):
    assert fwd(L, dt=7) == DTYPE
    assert fwd(L, B=-1) == SHAPE
    assert fwd(L, T=-5) == SHAPE
    assert fwd(L, B=1 << 21, T=1 << 21, C=1 << 21) == SHAPE


def test_forward_ex_flag_validation(L):
    def ex(flags, **kw):
        return L.wkv_forward_ex(2, 100, 64, F32, BASE, BASE + 4096, BASE + (1 << 30), BASE + (2 << 30), None, None,
                                BASE + (3 << 30), None, None, 0, flags, None)
    assert ex(8) == SHAPE                          # an unknown bit
    assert ex(wkv.WKV_FLAG_CHAIN_BEGIN | wkv.WKV_FLAG_CHAIN_NEXT) == SHAPE
    assert ex(0x80000000) == SHAPE
    # a valid flag reaches the argument checks (a null k is reported, nothing launches)
    for f in (wkv.WKV_FLAG_INPUTS_READY, wkv.WKV_FLAG_CHAIN_BEGIN, wkv.WKV_FLAG_CHAIN_NEXT):
        assert L.wkv_forward_ex(2, 100, 64, F32, BASE, BASE + 4096, None, BASE + (2 << 30), None, None,
                                BASE + (3 << 30), None, None, 0, f, None) == NULLPTR


def test_forward_empty_is_a_noop(L):
    assert fwd(L, B=0) == OK
    assert fwd(L, C=0) == OK
    assert fwd(L, T=0) == OK            # no state_out: nothing to write
    s = BASE + (5 << 30)
    assert fwd(L, T=0, s_in=s, s_out=s) == OK   # in place: nothing to copy


def test_forward_null_pointers(L):
    assert fwd(L, w=None) == NULLPTR
    assert fwd(L, k=None) == NULLPTR
    assert fwd(L, y=None) == NULLPTR


def test_forward_alignment(L):
    assert fwd(L, k=BASE + (1 << 30) + 2) == ALIGN
    assert fwd(L, dt=BF16, k=BASE + (1 << 30) + 1) == ALIGN
    assert fwd(L, s_out=BASE + (6 << 30) + 1) == ALIGN
    ws = BASE + (7 << 30)
    n = L.wkv_forward_workspace_bytes(2, 100, 64, F32)
    assert fwd(L, ws=ws + 16, ws_bytes=n) == ALIGN


def test_forward_aliasing(L):
    k = BASE + (1 << 30)
    assert fwd(L, y=k) == ALIAS
    assert fwd(L, y=k + 64) == ALIAS                    # partial overlap
    s = BASE + (5 << 30)
    assert fwd(L, s_in=s, s_out=s + 8) == ALIAS         # partial state overlap
    assert fwd(L, s_out=k) == ALIAS
    assert fwd(L, s_out=BASE + (3 << 30)) == ALIAS      # state_out inside y


@pytest.mark.skipif(_gpu_present(), reason="launches on fake addresses; only where no GPU can run them")
@pytest.mark.parametrize("B,T,C,dt", [(2, 100, 64, F32), (4, 8192, 5120, BF16), (1, 65536, 4096, BF16),
                                      (1, 1 << 20, 4096, BF16), (3, 5000, 130, F32), (2, 2000, 7, BF16),
                                      (64, 4096, 4096, F32)])
def test_forward_runs_without_a_workspace(L, B, T, C, dt):
    """No shape needs a caller workspace: with none (or too small a one) the
    call passes every host check and goes on to a launch.  Without a GPU the
    launch itself fails (WKV_ERR_CUDA); WKV_ERR_WORKSPACE never comes."""
    assert L.wkv_forward_workspace_bytes(B, T, C, dt) > 0
    ext = dict(k=BASE + (1 << 36), v=BASE + (2 << 36), y=BASE + (3 << 36))
    assert fwd(L, B=B, T=T, C=C, dt=dt, ws=None, ws_bytes=0, **ext) not in (WORKSPACE, NULLPTR, ALIGN, ALIAS, SHAPE)
    n = L.wkv_forward_workspace_bytes(B, T, C, dt)
    assert fwd(L, B=B, T=T, C=C, dt=dt, ws=BASE + (7 << 36), ws_bytes=n - 1, **ext) not in (WORKSPACE, ALIGN)


def test_workspace_size_rules(L):
    # short sequences take the sequential kernel and need no workspace
    assert L.wkv_forward_workspace_bytes(4, 16, 128, F32) == 0
    assert L.wkv_forward_workspace_bytes(4, 32, 128, F32) == 0     # a single chunk
    assert L.wkv_forward_workspace_bytes(-1, 64, 128, F32) == 0
    small = L.wkv_forward_workspace_bytes(8, 1024, 2048, F32)
    big = L.wkv_forward_workspace_bytes(8, 4096, 2048, F32)
    assert 0 < small < big
    # two 16-byte words per lane per 32-token chunk: about one byte per element
    assert small < 2 * 8 * 1024 * 2048


def test_workspace_init_and_status_validation(L):
    assert L.wkv_workspace_init(None, 0, None) == OK
    assert L.wkv_workspace_init(None, 100, None) == NULLPTR
    assert L.wkv_workspace_init(BASE + 8, 100, None) == ALIGN
    assert L.wkv_workspace_status(None, None) == NULLPTR
    assert L.wkv_workspace_status(BASE + 8, None) == ALIGN


def step(L, Lr=2, B=3, C=64, dt=BF16, w=BASE, u=BASE + 4096, k=BASE + (1 << 30), v=BASE + (2 << 30), r=None,
         state=BASE + (4 << 30), y=BASE + (3 << 30)):
    return L.wkv_step(Lr, B, C, dt, w, u, k, v, r, state, y, None)


def test_step_validation(L):
    assert step(L, dt=3) == DTYPE
    assert step(L, Lr=-1) == SHAPE
    assert step(L, Lr=0) == OK
    assert step(L, state=None) == NULLPTR
    assert step(L, y=None) == NULLPTR
    assert step(L, state=BASE + (4 << 30) + 2) == ALIGN
    assert step(L, y=BASE + (4 << 30)) == ALIAS      # y inside the state
    assert step(L, state=BASE + (1 << 30)) == ALIAS  # state over k


def test_python_front_end_refuses_cpu_tensors():
    import torch
    k = torch.zeros(1, 4, 8)
    with pytest.raises(ValueError):
        wkv.wkv_forward(torch.ones(8), torch.zeros(8), k, k)
    with pytest.raises(ValueError):
        wkv.wkv_step(torch.ones(1, 8), torch.zeros(1, 8), k, k, torch.zeros(1, 3, 4, 8))


def bwd(L, B=2, T=100, C=64, dt=F32, w=BASE, u=BASE + 4096, k=BASE + (1 << 30), v=BASE + (2 << 30), r=None,
        s_in=None, dy=BASE + (8 << 30), ds_out=None, dk=BASE + (9 << 30), dv=BASE + (10 << 30), dr=None,
        dw=BASE + 8192, du=BASE + 12288, ds_in=None, ws=BASE + (7 << 30), ws_bytes=None):
    if ws_bytes is None:
        ws_bytes = L.wkv_backward_workspace_bytes(B, T, C, dt)
    return L.wkv_backward(B, T, C, dt, w, u, k, v, r, s_in, dy, ds_out, dk, dv, dr, dw, du, ds_in, ws, ws_bytes,
                          None)


def test_backward_workspace_size(L):
    assert L.wkv_backward_workspace_bytes(-1, 64, 128, F32) == 0
    assert L.wkv_backward_workspace_bytes(2, 64, 128, 9) == 0
    assert L.wkv_backward_workspace_bytes(2, 0, 128, F32) == 0
    small = L.wkv_backward_workspace_bytes(8, 1024, 2048, F32)
    big = L.wkv_backward_workspace_bytes(8, 4096, 2048, F32)
    # one 12-byte checkpoint per lane per 64 tokens, plus fixed parts
    assert 0 < small < big < 2 * 8 * 4096 * 2048


def test_backward_validation(L):
    assert bwd(L, dt=5) == DTYPE
    assert bwd(L, T=-1) == SHAPE
    assert bwd(L, C=0) == OK
    assert bwd(L, dw=None) == NULLPTR
    assert bwd(L, dy=None) == NULLPTR
    assert bwd(L, dk=None) == NULLPTR
    assert bwd(L, r=BASE + (11 << 30)) == NULLPTR                 # a gate needs dr
    assert bwd(L, dr=BASE + (11 << 30)) == NULLPTR                # and dr needs a gate
    assert bwd(L, dk=BASE + (9 << 30) + 4) == ALIGN               # 16-byte aligned arrays
    assert bwd(L, C=66) == ALIGN                                  # C a multiple of 4
    assert bwd(L, dk=BASE + (1 << 30)) == ALIAS                   # dk over k
    assert bwd(L, dv=BASE + (9 << 30) + 1024) == ALIAS            # dv inside dk
    assert bwd(L, du=BASE + 8192 + 16) == ALIAS                   # du inside dw
    assert bwd(L, ds_in=BASE + (8 << 30), s_in=BASE + (12 << 30)) == ALIAS   # dstate_in over dy
    assert bwd(L, ws=None) == WORKSPACE
    assert bwd(L, ws_bytes=L.wkv_backward_workspace_bytes(2, 100, 64, F32) - 1) == WORKSPACE
    assert bwd(L, ws=BASE + (7 << 30) + 16) == ALIGN


def test_token_shift_validation(L):
    ts = L.wkv_token_shift
    x, mu, xp, out, xl = BASE, BASE + (1 << 36), BASE + (2 << 36), BASE + (3 << 36), BASE + (4 << 36)
    assert ts(2, 8, 64, 7, 3, x, mu, xp, out, xl, None) == DTYPE
    assert ts(-1, 8, 64, F32, 3, x, mu, xp, out, xl, None) == SHAPE
    assert ts(2, 8, 64, F32, 0, x, mu, xp, out, xl, None) == SHAPE          # nmix 1..8
    assert ts(2, 8, 64, F32, 9, x, mu, xp, out, xl, None) == SHAPE
    assert ts(1 << 30, 1 << 30, 8, F32, 1, x, mu, xp, out, xl, None) == SHAPE
    assert ts(0, 8, 64, F32, 3, None, None, None, None, None, None) == OK    # nothing to do
    assert ts(2, 8, 64, F32, 3, None, mu, xp, out, xl, None) == NULLPTR
    assert ts(2, 8, 64, F32, 3, x, None, xp, out, xl, None) == NULLPTR
    assert ts(2, 8, 64, F32, 3, x, mu, xp, None, xl, None) == NULLPTR
    assert ts(2, 8, 64, F32, 3, x + 2, mu, xp, out, xl, None) == ALIGN
    assert ts(2, 8, 64, BF16, 3, x, mu + 2, xp, out, xl, None) == ALIGN
    assert ts(2, 8, 64, BF16, 3, x, mu, xp + 1, out, xl, None) == ALIGN
    assert ts(2, 8, 64, F32, 3, x, mu, xp, x + 64, xl, None) == ALIAS           # out over x
    assert ts(2, 8, 64, F32, 3, x, mu, xp, out, out + 4096, None) == ALIAS      # x_last inside out
    assert ts(2, 8, 64, F32, 3, x, mu, xp, out, x, None) == ALIAS               # x_last over x
    assert ts(2, 8, 64, F32, 3, x, mu, xp, out, xp + 4, None) == ALIAS          # x_last partly over x_prev
    assert ts(2, 8, 64, F32, 3, x, mu, xp, xp, xl, None) == ALIAS               # out over x_prev


def test_token_shift_front_end_refuses_bad_arguments():
    import torch
    x = torch.zeros(2, 4, 8)
    with pytest.raises(ValueError):
        wkv.wkv_token_shift(x, torch.rand(3, 8))                       # CPU tensors
    with pytest.raises(ValueError):
        wkv.wkv_token_shift(torch.zeros(4, 8), torch.rand(3, 8))       # x not (B, T, C)
    with pytest.raises(ValueError):
        wkv.wkv_token_shift(x, torch.rand(8))                          # mu not (nmix, C)


def test_state_validation(L):
    st = BASE + (5 << 30)
    call = lambda B=2, T=100, C=64, dt=F32, w=BASE, k=BASE + (1 << 30), v=BASE + (2 << 30), s_in=None, s_out=st: \
        L.wkv_state(B, T, C, dt, w, k, v, s_in, s_out, None, 0, None)
    assert call(dt=5) == DTYPE
    assert call(B=-1) == SHAPE
    assert call(B=0) == OK and call(C=0) == OK
    assert call(s_out=None) == NULLPTR
    assert call(k=None) == NULLPTR and call(w=None) == NULLPTR
    assert call(k=BASE + (1 << 30) + 2) == ALIGN
    assert call(s_out=BASE + (1 << 30)) == ALIAS                  # state_out inside k
    assert call(s_in=st + 4, s_out=st) == ALIAS                   # partial state overlap


def test_state_combine_validation(L):
    import ctypes as ct
    lens = (ct.c_int64 * 3)(5, 0, 7)
    neg = (ct.c_int64 * 1)(-1)
    st, seg = BASE + (5 << 30), BASE + (6 << 30)
    call = lambda B=2, C=64, n=3, w=BASE, ln=lens, sg=seg, s_in=None, s_out=st: \
        L.wkv_state_combine(B, C, n, w, ln, sg, s_in, s_out, None)
    assert call(n=-1) == SHAPE and call(n=65) == SHAPE
    assert call(n=1, ln=neg) == SHAPE
    assert call(B=0) == OK
    assert call(s_out=None) == NULLPTR
    assert call(ln=None) == NULLPTR and call(sg=None) == NULLPTR and call(w=None) == NULLPTR
    assert call(s_out=st + 2) == ALIGN
    assert call(s_out=seg + 64) == ALIAS                          # state_out inside the summaries


def test_wkv5_validation(L):
    y, st = BASE + (3 << 30), BASE + (5 << 30)
    call = lambda B=2, T=10, C=128, H=2, dt=BF16, w=BASE, pt=0, u=BASE + 4096, r=BASE + (4 << 30), \
        k=BASE + (1 << 30), v=BASE + (2 << 30), s_in=None, yy=y, s_out=st: \
        L.wkv5_forward(B, T, C, H, dt, w, pt, u, r, k, v, s_in, yy, s_out, None)
    assert call(dt=3) == DTYPE
    assert call(H=0) == SHAPE and call(H=3) == SHAPE              # C not a multiple of H
    assert call(C=96, H=2) == SHAPE                               # head size 48
    assert call(B=0) == OK
    assert call(r=None) == NULLPTR and call(w=None) == NULLPTR
    assert call(k=BASE + (1 << 30) + 1) == ALIGN
    assert call(yy=BASE + (1 << 30)) == ALIAS                     # y is k
    assert call(s_out=BASE + (2 << 30) + 64) == ALIAS             # state_out inside v
    assert call(pt=1, w=y - 64) == ALIAS                          # per-token w (B, T, C) runs into y
