"""bench.py's host-side logic: byte accounting, rank helpers and the
max-over-ranks reduction (two gloo ranks on CPU)."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

import bench
from rwkv_wkv_recurrence_02_b200 import inputs as I

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_algorithmic_bytes_layer_1b5():
    wl = I.WORKLOADS["layer_1b5"]
    n = 8 * 1024 * 2048
    # k, v, r read + y written (4 B each), state in and out, w and u
    assert bench.algorithmic_bytes(wl, 8, 1024, 2048) == n * 16 + 8 * 2048 * 24 + 2048 * 8


def test_algorithmic_bytes_bf16_and_decode():
    wl = I.WORKLOADS["layer_14b"]
    n = 4 * 8192 * 5120
    assert bench.algorithmic_bytes(wl, 4, 8192, 5120) == n * 8 + 4 * 5120 * 12 + 5120 * 8
    st = I.WORKLOADS["stream_1m"]
    assert bench.algorithmic_bytes(st, 1, 1024, 4096) == 1024 * 4096 * 6 + 4096 * 24 + 4096 * 8
    dec = I.WORKLOADS["decode"]
    lanes = 24 * 256 * 4096
    assert bench.algorithmic_bytes(dec, 256, 1, 4096, layers=24) == lanes * 8 + lanes * 24 + 24 * 4096 * 8


def test_algorithmic_bytes_backward():
    wl = I.WORKLOADS["layer_1b5"]
    n = 8 * 1024 * 2048
    # k, v, dy, r read + dk, dv, dr written (4 B each); state read, dL/d(a, b)
    # of the returned state read, dL/d(state) written; w, u read, dw, du written
    assert bench.algorithmic_bytes_backward(wl, 8, 1024, 2048) == n * 28 + 8 * 2048 * (12 + 8 + 12) + 2048 * 16
    st = I.WORKLOADS["layer_14b"]       # bf16, gated, no initial state
    assert bench.algorithmic_bytes_backward(st, 4, 8192, 5120) == 4 * 8192 * 5120 * 14 + 4 * 5120 * 20 + 5120 * 16


def test_single_call_stream_workload():
    wl = bench.workload("stream_1m_single")
    base = I.WORKLOADS["stream_1m"]
    assert wl.chunk == 0 and wl.T == base.T == 1 << 20
    assert (wl.B, wl.C, wl.dtype, wl.gate, wl.seed) == (base.B, base.C, base.dtype, base.gate, base.seed)
    assert bench.algorithmic_bytes(wl, 1, wl.T, wl.C) == wl.T * 4096 * 6 + 4096 * 12 + 4096 * 8
    assert bench.parse_args(["--workload", "stream_1m_single", "--op", "backward"]).op == "backward"


def test_rates_and_seeds():
    assert bench.whole_job_rate(100, 4, 10, 2.0) == 2000.0
    assert len({bench.rank_seed(0, r) for r in range(8)}) == 8


def test_traffic_record_invalidated_by_source_change(tmp_path, monkeypatch):
    p = tmp_path / "traffic.json"
    p.write_text(json.dumps({"layer_1b5": {"traffic_bytes_per_launch": 123, "source_hash": "stale"}}))
    monkeypatch.setattr(bench, "PROFILE_TRAFFIC", str(p))
    assert bench.load_traffic("layer_1b5") is None
    p.write_text(json.dumps({"layer_1b5": {"traffic_bytes_per_launch": 123,
                                           "source_hash": bench.kernel_source_hash()}}))
    assert bench.load_traffic("layer_1b5") == 123


def test_traffic_hash_scopes(tmp_path, monkeypatch):
    """A WKV kernel's record does not depend on the token-shift-only sources;
    the token shift's record depends on every source."""
    csrc = tmp_path / "csrc"
    csrc.mkdir()
    (csrc / "wkv_api.cu").write_text("api")
    (csrc / "wkv_lane.cuh").write_text("lane")
    (csrc / "wkv_shift.cuh").write_text("shift v1")
    monkeypatch.setattr(bench, "CSRC", str(csrc))
    wkv1, ts1 = bench.kernel_source_hash("lane_forward"), bench.kernel_source_hash("token_shift")
    (csrc / "wkv_shift.cuh").write_text("shift v2")
    assert bench.kernel_source_hash("lane_forward") == wkv1
    assert bench.kernel_source_hash("token_shift") != ts1
    (csrc / "wkv_lane.cuh").write_text("lane v2")
    assert bench.kernel_source_hash("lane_forward") != wkv1


def _rank_main(rank, world, port, q):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    t = bench.max_over_ranks(1.0 + rank * 0.5, dist)
    q.put((rank, t))
    dist.barrier()
    dist.destroy_process_group()


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def test_max_over_ranks_gloo_world_2():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=5) for _ in range(2))
    assert got == [(0, 1.5), (1, 1.5)]


def test_reference_arm_nonzero_rank_exits_quietly():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "3",
                        "--warmup", "3"], env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0 and r.stdout.strip() == ""


def test_reference_arm_prints_one_line():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "3",
                        "--warmup", "3", "--ref-budget-s", "3"], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    out = json.loads(lines[0])
    assert out["impl"] == "reference" and out["unit"] == "elements/s" and out["value"] > 0
    assert out["cpu_baseline"]["kind"] == "oracle" and out["e2e"]["h2d_bytes_per_step"] == 0
    assert out["config"]["workload"] == "stream_1m" and out["config"]["T"] == 1 << 20


def test_decode_forms_and_graph_period():
    """The per-layer decode form issues one L = 1 call per layer on the same rows
    as the one-call form, and steps one graph period apart read the same rows."""
    import dataclasses
    wl = dataclasses.replace(I.WORKLOADS["decode"], B=2, C=8)

    class Rec:
        def __init__(self):
            self.calls = []

        def wkv_step(self, w, u, k, v, state, r, y):
            self.calls.append((w.shape[0], k.data_ptr(), state.data_ptr(), y.data_ptr()))

    one = bench.DecodeCase(wl, "cpu", 0)
    per = bench.DecodeCase(wl, "cpu", 0, per_layer=True)
    assert one.launches_per_step == 1 and per.launches_per_step == wl.layers
    assert one.period == per.period == 8
    for i in range(3 * one.period):
        assert I.decode_ring_start(wl, i) == I.decode_ring_start(wl, i + one.period)
        a, b = Rec(), Rec()
        one.step(i, a, None)
        per.step(i, b, None)
        assert len(a.calls) == 1 and a.calls[0][0] == wl.layers
        assert len(b.calls) == wl.layers and all(c[0] == 1 for c in b.calls)
        row = one.k[0].numel() * one.k.element_size()
        assert a.calls[0][1] - one.k.data_ptr() == b.calls[0][1] - per.k.data_ptr()
        assert [c[1] - per.k.data_ptr() for c in b.calls] == [(I.decode_ring_start(wl, i) + l) * row
                                                              for l in range(wl.layers)]


def test_decode_e2e_bytes():
    """The decode end-to-end leg copies k, v, r of every layer in and y out."""
    import dataclasses
    import torch
    wl = dataclasses.replace(I.WORKLOADS["decode"], B=2, C=8)
    case = bench.DecodeCase(wl, "cpu", 0, per_layer=True)
    calls = []

    class Rec:
        def wkv_step(self, w, u, k, v, state, r, y):
            calls.append(k.shape[0])

    class Ev:
        def __init__(self, **kw):
            pass

        def record(self, stream):
            pass

        def elapsed_time(self, other):
            return 1.0

    orig_pin, orig_ev, orig_sync = torch.Tensor.pin_memory, torch.cuda.Event, torch.cuda.synchronize
    torch.Tensor.pin_memory, torch.cuda.Event, torch.cuda.synchronize = (lambda t: t), Ev, (lambda: None)
    try:
        e = bench.e2e_measure(case, Rec(), None, 3, 1, None)
    finally:
        torch.Tensor.pin_memory, torch.cuda.Event, torch.cuda.synchronize = orig_pin, orig_ev, orig_sync
    el = torch.tensor([], dtype=wl.torch_dtype).element_size()
    assert e["h2d"] == 3 * wl.layers * wl.B * wl.C * el
    assert e["d2h"] == wl.layers * wl.B * wl.C * el
    assert calls == [1] * (wl.layers * 4) and "wkv_step" in e["path"]


def test_token_shift_bytes_and_reference_arm(capsys):
    """Token-shift byte accounting, and its reference arm (the oracle on a
    channel sample) prints one line with the op's metric."""
    wl = I.WORKLOADS["layer_14b"]
    n = 4 * 8192 * 5120
    assert bench.algorithmic_bytes_shift(wl, 4, 8192, 5120) == n * 2 * 4 + 2 * 4 * 5120 * 2 + 3 * 5120 * 4
    bench.main(["--impl", "reference", "--op", "token_shift", "--workload", "decode", "--steps", "3",
                "--warmup", "3", "--ref-budget-s", "2"])
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["metric"] == bench.METRIC_SHIFT and line["value"] > 0
    assert line["config"]["T"] == 1 and line["config"]["op"] == "token_shift"


def test_token_shift_cpu_baseline_is_bounded():
    r = bench.cpu_baseline_shift("layer_1b5", 0.5)
    assert r["value"] > 0 and r["kind"] == "oracle" and "mixes" in r["sample"]


def test_defaults_follow_the_workload():
    a = bench.parse_args([])
    assert a.workload == "stream_1m" and a.steps == 20 and a.warmup == 5
    b = bench.parse_args(["--workload", "layer_1b5"])
    assert b.steps == 3000 and b.warmup == 20
    c = bench.parse_args(["--gpus", "1", "--steps", "20", "--warmup", "5"])
    assert (c.steps, c.warmup, c.workload) == (20, 5, "stream_1m")
    # the other operations default to their own single-call workloads
    assert bench.parse_args(["--op", "backward"]).workload == "layer_1b5"
    assert bench.parse_args(["--op", "token_shift"]).workload == "layer_14b"
    assert bench.parse_args(["--op", "wkv5"]).workload == "v5_layer"
    with pytest.raises(SystemExit):
        bench.parse_args(["--op", "backward", "--workload", "stream_1m"])


def test_whole_stream_bytes_and_names():
    wl = bench.workload("stream_1m")
    assert bench.whole_stream("stream_1m") and not bench.whole_stream("stream_1m_chunk")
    assert wl.T == 1 << 20 and wl.chunk == 1024 and wl.T // wl.chunk == 1024
    assert bench.workload("stream_1m_chunk").chunk == 1024
    # per launch (one chunk): k, v read, y written (2 B each), state in and out, w and u
    assert bench.algorithmic_bytes(wl, 1, wl.chunk, wl.C) == 1024 * 4096 * 6 + 4096 * 24 + 4096 * 8
