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
