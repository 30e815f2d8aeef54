"""bench.py's multi-rank logic on CPU: two gloo ranks, max-over-ranks timing,
weak-scaling aggregate, and the reference arm running on rank 0 only."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import datetime

    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import bench
    m = bench.dist_max(10.0 + 5.0 * rank, dist, "cpu")          # rank 1 is the slower one
    v = bench.weak_scaling_value(2e9, 4, world, m)
    dist.barrier()
    dist.destroy_process_group()
    q.put((rank, m, v))


def test_two_gloo_ranks_max_time_and_weak_scaling_value():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    for rank, m, v in res:
        assert m == 15.0                                        # the max over ranks on every rank
        assert v == pytest.approx(2e9 * 4 * 2 / 0.015 / 1e9)    # all ranks' bytes / the slowest rank's time


def test_reference_arm_runs_on_rank_zero_only():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload", "tiny_f32",
                        "--steps", "1", "--warmup", "0"], env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0 and r.stdout.strip() == ""
    env = dict(os.environ, RANK="0", WORLD_SIZE="2", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload", "tiny_f32",
                        "--steps", "1", "--warmup", "0"], env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["e2e"]["h2d_bytes_per_step"] == 0


def test_traffic_summary_is_used_only_while_its_sources_are_unchanged(tmp_path):
    sys.path.insert(0, ROOT)
    import bench
    srcs = "sparse_top_kv_std_b200/csrc/attn_tc.cu sparse_top_kv_std_b200/csrc/tc100.cuh"
    sha = bench.sources_sha256(srcs.split())
    p = tmp_path / "t.txt"
    body = ("# header\nkernel: dense_verify_attn\nworkload: video_140k\nsources: %s\nsources_sha256: %s\n"
            "dram_bytes_per_launch: 8.3e9\ncommand: x: y\n")
    p.write_text(body % (srcs, sha))
    assert bench.load_traffic("dense_verify_attn", "video_140k", str(p)) == 8.3e9
    assert bench.load_traffic("dense_verify_attn", "layer_16k", str(p)) is None
    p.write_text(body % (srcs, "0" * 64))
    assert bench.load_traffic("dense_verify_attn", "video_140k", str(p)) is None
    assert bench.load_traffic("dense_verify_attn", "video_140k", str(tmp_path / "missing.txt")) is None


def test_clock_summary_keeps_samples_of_the_timed_region():
    sys.path.insert(0, ROOT)
    import datetime

    import bench

    def row(t, mhz, reason="Not Active", power="600.0"):
        ts = datetime.datetime.fromtimestamp(t).strftime("%Y/%m/%d %H:%M:%S.%f")[:-3]
        return [ts, "0", str(mhz), "1965", power, "0x0", "Not Active", "Not Active", "Not Active", reason]

    t = 1_800_000_000.0
    rows = [row(t, 1000), row(t + 1.0, 1600, "Active"), row(t + 1.1, 1700), row(t + 2.0, 900)]
    s = bench.ClockSampler.summarise(rows, window=(t + 0.95, t + 1.15))
    assert s["samples"] == 2 and s["window"] == "timed region"
    assert s["sm_mhz"] == 1650 and s["reasons"] == ["sw_power_cap"] and s["sm_max_mhz"] == 1965
    # a region shorter than the sampling interval: the two nearest samples, marked
    s = bench.ClockSampler.summarise(rows, window=(t + 1.5, t + 1.52))
    assert s["samples"] == 2 and s["window"] == "nearest to the timed region"
    assert bench.ClockSampler.summarise([], window=(t, t + 1)) is None


def test_draft_launch_modes_issue_per_layer_slices(monkeypatch):
    """The per-layer draft launches get L = 1 dims and the layer's slices of every operand, the
    CUDA-graph mode captures exactly those launches, and a failure becomes an "error" entry
    instead of an exception (CUDA events, graphs and the library replaced by fakes)."""
    import types

    import torch
    sys.path.insert(0, ROOT)
    import bench

    class Ev:
        def __init__(self, **kw):
            self.t = 0.0

        def record(self, stream=None):
            pass

        def elapsed_time(self, other):
            return 2.0

    class Graph:
        def __init__(self):
            self.calls = None

        def replay(self):
            calls.extend(self.calls)

    class Capture:
        def __init__(self, g, capture_error_mode=None):
            self.g = g

        def __enter__(self):
            self.n0 = len(calls)

        def __exit__(self, *exc):
            self.g.calls = calls[self.n0:]
            del calls[self.n0:]

    monkeypatch.setattr(torch.cuda, "Event", Ev)
    monkeypatch.setattr(torch.cuda, "synchronize", lambda: None)
    monkeypatch.setattr(torch.cuda, "CUDAGraph", Graph)
    monkeypatch.setattr(torch.cuda, "graph", Capture)
    calls = []
    L, Bn, Hq, Hkv, d, K, T = 3, 1, 4, 2, 8, 5, 2
    fake = types.SimpleNamespace(
        dims=lambda *a: ("dims",) + a,
        std_get_device_error=lambda clear=True: 0,
        STD_ATTN_EARLY_KV=1,
        std_sparse_decode_attn_append=lambda dims, q, k, v, ln, off, kn, vn, o, sp, ws: calls.append(
            (dims, q, k, v, ln, off, kn, vn, o, None)),
        std_sparse_decode_attn_append_ex=lambda dims, q, k, v, ln, off, kn, vn, o, sp, fl, ws: calls.append(
            (dims, q, k, v, ln, off, kn, vn, o, fl)))
    wl = types.SimpleNamespace(L=L, B=Bn, Hq=Hq, Hkv=Hkv, d=d, K=K, T=T, cap_full=20, cap_sparse=12)
    sess = types.SimpleNamespace(dims="batched-dims", k_sparse=torch.zeros(L, Bn, Hkv, 12, d),
                                 v_sparse=torch.ones(L, Bn, Hkv, 12, d), len_sparse=torch.zeros(Bn, dtype=torch.int32))
    q, kn, vn = torch.randn(L, Bn, Hq, 1, d), torch.randn(L, Bn, Hkv, 1, d), torch.randn(L, Bn, Hkv, 1, d)
    o = torch.zeros(L, Bn, Hq, 1, d)
    res = bench.draft_launch_modes(fake, sess, wl, 1, q, kn, vn, o, None, None, reps=2)
    assert "error" not in res, res
    assert sess.len_sparse.tolist() == [K + T]
    # batched: 1 + 2 calls; per-layer eager: (1 + 2) x L; each of the two graphs: capture L, then
    # 1 + 2 replays of L (the second graph's launches fetch K/V early)
    assert len(calls) == 3 + 3 * L + 3 * L + 3 * L
    assert res["launches_per_step"] == {"batched": 1, "per_layer": L}
    assert res["batched_us"] == res["per_layer_eager_us"] == res["per_layer_graph_us"] == 1e3
    assert res["per_layer_graph_early_kv_us"] == 1e3
    assert [c[9] for c in calls[3:3 + 6 * L]] == [0] * (6 * L)
    assert [c[9] for c in calls[3 + 6 * L:]] == [1] * (3 * L)
    first = calls[0]
    assert first[0] == "batched-dims" and first[1] is q and first[5] == 1
    for l, c in enumerate(calls[3:3 + L]):
        assert c[0][:3] == ("dims", 1, Bn)                  # one layer per launch
        for got, full in zip((c[1], c[2], c[3], c[6], c[7], c[8]), (q, sess.k_sparse, sess.v_sparse, kn, vn, o)):
            assert got.data_ptr() == full[l].data_ptr() and got.shape == full.shape[1:]
    replayed = calls[3 + 3 * L:3 + 6 * L]
    assert [c[1].data_ptr() for c in replayed] == [q[l].data_ptr() for l in range(L)] * 3
    # a failing library call is reported, not raised
    fake.std_sparse_decode_attn_append = lambda *a: (_ for _ in ()).throw(RuntimeError("boom"))
    assert bench.draft_launch_modes(fake, sess, wl, 1, q, kn, vn, o, None, None)["error"] == "RuntimeError: boom"


def test_selection_figures_at_the_long_video_sizes():
    """2 passes x 2 x (7 x 256) x 143,360 x 128 flops x 112 heads = 14.73 TFLOP and 2 x 1,792 x
    143,360 x 112 exponentials per selection; rates and fractions against the given peaks."""
    sys.path.insert(0, ROOT)
    import bench
    import synth
    wl = synth.workload("video_140k")
    assert bench.select_flops(wl) == 2 * 2 * 1792 * 143360 * 128 * 112
    assert bench.select_exps(wl) == 2 * 1792 * 143360 * 112
    f = bench.select_figures(wl, 18.0, {"bf16_tflops": 1647.5, "bf16_tflops_sustained": 1399.2}, "measured")
    assert abs(f["mma_TFLOPs"] - 14.7307e12 / 0.018 / 1e12) < 0.5
    assert abs(f["one_pass_TFLOPs"] - 0.5 * f["mma_TFLOPs"]) < 1e-9
    assert abs(f["frac_of_burst_bf16"] - f["mma_TFLOPs"] / 1647.5) < 1e-12
    assert abs(f["frac_of_sustained_bf16"] - f["mma_TFLOPs"] / 1399.2) < 1e-12
    assert abs(f["exp2_G_per_s"] - 2 * 1792 * 143360 * 112 / 0.018 / 1e9) < 1e-6


def test_attention_byte_model_at_the_long_video_sizes():
    """K/V bytes the draft and verify calls read: 2 (K, V) x 128 x 2 B x 28 layers x 4 KV heads
    = 57,344 B per position.  Round 0's verify reads nvis + T + gamma + 1 = 143,625 positions
    (8.236 GB); draft step j reads K + T + j + 1; accepted tokens advance both caches."""
    sys.path.insert(0, ROOT)
    import bench
    import synth
    wl = synth.workload("video_140k")
    row = 57344
    d, v, per = bench.attention_bytes(wl, 1, [[9]])
    assert v == per[0] == 143625 * row == 8_236_032_000
    assert d == sum(4096 + 256 + j + 1 for j in range(8)) * row
    d2, v2, per2 = bench.attention_bytes(wl, 3, [[1], [9], [4]])
    assert per2 == [143625 * row, (143625 + 1) * row, (143625 + 10) * row]
    assert v2 == sum(per2)
    assert d2 == sum((4352 + c + j + 1) * row for c in (0, 1, 10) for j in range(8))
