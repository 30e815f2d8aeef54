#!/usr/bin/env python
"""Benchmark of the Sparse-to-Dense (StD) decoding hot path on B200.

One step = one whole StD decode of a synthetic long-video prompt: the prefill
top-K selection (selection scores, top-K, gather) followed by R draft+verify
rounds (gamma sparse draft attentions, one dense verify attention over the
full cache, acceptance, commit).  All inputs are resident in HBM before the
timed region; the full KV cache (8.2 GB at the default workload) is larger
than L2, so no flush is needed between steps.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload video_140k]
    python bench.py --impl reference ...   # the fp64 CPU oracle on a bounded sample

Multi-GPU (torchrun, one rank per GPU): every rank decodes its own prompt
(independent sequences, no data-path collective), "scaling": "weak"; time is
the max over ranks.  Rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "decode-attn HBM GB/s (sparse draft, dense verify) vs 8 TB/s; µs per draft+verify round"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["std", "reference"], default="std")
    ap.add_argument("--workload", default="video_140k")
    ap.add_argument("--rounds", type=int, default=None, help="draft+verify rounds per step (default: workload's)")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--e2e-steps", type=int, default=4)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-draft-modes", action="store_true",
                    help="skip the draft launch-mode figures (batched / per layer / per-layer CUDA graph)")
    ap.add_argument("--threads", type=int, default=0, help="host threads for input generation")
    ap.add_argument("--eager", action="store_true",
                    help="issue every step's launches from the host instead of replaying a CUDA graph of one step")
    return ap.parse_args(argv)


def dist_env():
    return (int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)),
            int(os.environ.get("LOCAL_RANK", 0)))


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in FALLBACK_PEAKS if k in d}, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ----------------------------------------------------------------------------- byte / flop model

def attention_bytes(wl, rounds, accepted):
    """Algorithmic K/V bytes of the draft and verify attention over `rounds` rounds.

    accepted[r][b] = n + 1 of round r.  A step reads, per (layer, KV head), every
    K and V row each attention call attends to: the verify of round r reads
    len_full_r + gamma + 1 rows, draft step j reads len_sparse_r + j + 1 rows.
    Returns (draft_bytes, verify_bytes, per-round verify bytes list).
    """
    row = 2 * wl.d * wl.elem_bytes * wl.L * wl.Hkv          # K + V of one position, all layers/heads
    lf = [n + wl.T for n in wl.nvis]
    ls = [wl.K + wl.T] * wl.B
    draft = verify = 0
    per_round_verify = []
    for r in range(rounds):
        v = sum(lf[b] + wl.gamma + 1 for b in range(wl.B)) * row
        verify += v
        per_round_verify.append(v)
        for j in range(wl.gamma):
            draft += sum(ls[b] + j + 1 for b in range(wl.B)) * row
        for b in range(wl.B):
            lf[b] += int(accepted[r][b])
            ls[b] += int(accepted[r][b])
    return draft, verify, per_round_verify


def dist_max(x, pg, device):
    """Max of a per-rank float over all ranks (pg: torch.distributed or None)."""
    import torch
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    if pg is not None:
        pg.all_reduce(t, op=pg.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_value(bytes_per_step, steps, world, elapsed_ms):
    """Whole-job GB/s: every rank processed `steps` steps of `bytes_per_step` in `elapsed_ms`
    (the max over ranks)."""
    return bytes_per_step * steps * world / (elapsed_ms / 1e3) / 1e9


def select_flops(wl):
    """Executed MMA flops of the selection (2 passes over the M x Nv logits)."""
    M = wl.G * wl.T
    return 2 * sum(2 * M * n * wl.d for n in wl.nvis) * wl.L * wl.Hkv


def select_exps(wl):
    """Exponentials of the selection: one per logit in each of the 2 passes."""
    return 2 * sum(wl.G * wl.T * n for n in wl.nvis) * wl.L * wl.Hkv


def select_figures(wl, ms, peaks, peak_src):
    """Rates of one selection call (scores, top-K, gather) that took `ms`: executed MMA flops
    (both passes) against the bf16 GEMM peaks, the one-pass algorithmic rate, exponentials/s."""
    s = ms / 1e3
    mma = select_flops(wl) / s / 1e12
    out = {"ms_per_launch": ms, "mma_TFLOPs": mma, "one_pass_TFLOPs": 0.5 * mma,
           "exp2_G_per_s": select_exps(wl) / s / 1e9}
    for key, name in (("bf16_tflops", "burst"), ("bf16_tflops_sustained", "sustained")):
        if key in peaks:
            out[f"frac_of_{name}_bf16"] = mma / peaks[key]
    out["peak_source"] = f"{peak_src} cuBLAS bf16 GEMM"
    return out


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi samples every 50 ms, started before the warm-up so that the tool is up by
    the time the timed region starts; stop(window) keeps the samples whose timestamps fall
    inside the timed region (host wall-clock seconds), or the two nearest ones, marked, if the
    region was shorter than the sampling interval."""
    FIELDS = ["timestamp", "index", "clocks.sm", "clocks.max.sm", "power.draw", "clocks_event_reasons.active",
              "clocks_event_reasons.hw_slowdown", "clocks_event_reasons.hw_thermal_slowdown",
              "clocks_event_reasons.sw_thermal_slowdown", "clocks_event_reasons.sw_power_cap"]

    def __init__(self, gpu_id, interval_ms=50):
        self.gpu_id = gpu_id
        self.interval_ms = interval_ms
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.f = open(self.path, "w")
            cmd = ["nvidia-smi", "--query-gpu=" + ",".join(self.FIELDS), "--format=csv,noheader,nounits",
                   "-lms", str(self.interval_ms)]
            if self.gpu_id is not None:
                cmd += ["-i", str(self.gpu_id)]
            self.proc = subprocess.Popen(cmd, stdout=self.f, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    @staticmethod
    def _when(ts):
        try:
            return datetime.datetime.strptime(ts.strip(), "%Y/%m/%d %H:%M:%S.%f").timestamp()
        except ValueError:
            return None

    def stop(self, window=None):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.f.close()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) == len(self.FIELDS):
                    rows.append(parts)
        os.unlink(self.path)
        return self.summarise(rows, window)

    @classmethod
    def summarise(cls, rows, window=None):
        """Clock summary of nvidia-smi rows (FIELDS order); window = (t0, t1) host seconds."""
        kept, where = rows, "all"
        if window is not None:
            timed = [(cls._when(r[0]), r) for r in rows]
            timed = [(t, r) for t, r in timed if t is not None]
            kept = [r for t, r in timed if window[0] <= t <= window[1]]
            where = "timed region"
            if not kept and timed:
                mid = 0.5 * (window[0] + window[1])
                kept = [r for _, r in sorted(timed, key=lambda tr: abs(tr[0] - mid))[:2]]
                where = "nearest to the timed region"
        if not kept:
            return None

        def num(x):
            try:
                return float(x)
            except ValueError:
                return None
        sm = [num(r[2]) for r in kept if num(r[2]) is not None]
        pw = [num(r[4]) for r in kept if num(r[4]) is not None]
        reasons = set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in kept:
            for n, v in zip(names, r[6:10]):
                if v.lower() == "active":
                    reasons.add(n)
        load = [x for x, p in zip(sm, pw) if pw and p >= 0.5 * max(pw)] or sm
        return {"sm_mhz": statistics.median(load) if load else None,
                "sm_max_mhz": num(kept[0][3]), "power_w_max": max(pw) if pw else None,
                "samples": len(kept), "window": where, "reasons": sorted(reasons)}


# ----------------------------------------------------------------------------- oracle (CPU) sample

def oracle_sample(wl, seed, rounds_sample, heads=((0, 0, 0),)):
    """Time the fp64 oracle on a bounded sample: for each listed (layer, batch, KV head)
    slice, its prefill selection and `rounds_sample` draft+verify rounds.
    Returns (select seconds per head, round seconds per head and round)."""
    import numpy as np

    import oracle
    import synth
    f = lambda a: synth.storage_to_f64(synth.storage(a, wl.dtype), wl.dtype)  # noqa: E731
    t_sel = t_round = 0.0
    for (l, b, h) in heads:
        nv = wl.nvis[b]
        k, v = synth.kv_head(wl, seed, l, b, h)
        cap_f = nv + wl.T + rounds_sample * (wl.gamma + 1)
        cap_s = wl.K + wl.T + rounds_sample * (wl.gamma + 1)
        kf = np.zeros((1, 1, 1, cap_f, wl.d))
        vf = np.zeros_like(kf)
        kf[0, 0, 0, :nv + wl.T] = f(k)
        vf[0, 0, 0, :nv + wl.T] = f(v)
        qt = f(synth.q_text_head(wl, seed, l, b, h))[None, None]
        t0 = time.perf_counter()
        _, _, ksp, vsp, lsp = oracle.select_topk(qt, kf, vf, np.array([nv]), wl.T, wl.K, cap_s)
        t_sel += time.perf_counter() - t0
        qd, qv = synth.decode_queries(wl, seed, l, b, h)
        kd, vd, kv, vv = synth.decode_kv(wl, seed, l, b, h)
        dense, draft = synth.tokens(wl, seed, b)
        st = {"k_full": kf, "v_full": vf, "k_sp": ksp, "v_sp": vsp,
              "len_full": np.array([nv + wl.T]), "len_sp": lsp.astype(np.int64)}
        t0 = time.perf_counter()
        for r in range(rounds_sample):
            oracle.decode_round(st, f(qd[r])[:, None, None, :, None, :], f(kd[r])[:, None, None, None, None, :],
                                f(vd[r])[:, None, None, None, None, :], f(qv[r])[None, None],
                                f(kv[r])[None, None, None], f(vv[r])[None, None, None],
                                draft[r][None], dense[r][None])
        t_round += time.perf_counter() - t0
    n = len(heads)
    return t_sel / n, t_round / (n * rounds_sample)


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return os.cpu_count() or 1


def cpu_estimate(wl, seed, rounds, step_attn_bytes, rounds_sample, heads):
    """Oracle GB/s on the sample, scaled to a whole step (all heads, all rounds)."""
    t_sel, t_round = oracle_sample(wl, seed, rounds_sample, heads)
    probs = wl.L * wl.B * wl.Hkv
    est = probs * (t_sel + rounds * t_round)
    return step_attn_bytes / est / 1e9, t_sel, t_round, est


# ----------------------------------------------------------------------------- reference arm

def run_reference(args, rank, world):
    if rank != 0:
        return 0
    import numpy as np

    import oracle
    import synth
    wl = synth.workload(args.workload)
    R = args.rounds or wl.rounds
    if R > wl.rounds:
        wl = wl.replace(rounds=R)
    # acceptance counts of the byte model: the oracle's greedy prefix rule on the token streams
    streams = [synth.tokens(wl, args.seed, b) for b in range(wl.B)]
    acc = [oracle.accept_prefix(np.array([s[1][r] for s in streams]), np.array([s[0][r] for s in streams]))[0]
           for r in range(R)]
    draft_b, verify_b, _ = attention_bytes(wl, R, acc)
    step_bytes = draft_b + verify_b
    heads = [(l, b, h) for l in range(wl.L) for b in range(wl.B) for h in range(wl.Hkv)]
    vals = []
    times = []
    for i in range(args.warmup + args.steps):
        lbh = heads[i % len(heads)]
        t0 = time.perf_counter()
        v, t_sel, t_round, est = cpu_estimate(wl, args.seed, R, step_bytes, 1, [lbh])
        dt = time.perf_counter() - t0
        if i >= args.warmup:
            vals.append(v)
            times.append(dt)
    value = statistics.median(vals)
    cores = blas_threads()
    sample = (f"each step: the fp64 oracle on one (layer, KV head) slice of {wl.name} -- its prefill "
              f"selection and 1 draft+verify round -- scaled to all {wl.L * wl.B * wl.Hkv} slices and {R} rounds")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * statistics.median(times),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": workload_config(wl, R),
            "cpu_baseline": {"value": value, "unit": "GB/s", "cores": cores, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def draft_launch_modes(B, sess, wl, dt, q, k_new, v_new, o, ws, stream, reps=20):
    """One sparse draft step (the step's row appended in the same launch) issued three ways,
    each repeated `reps` times after one untimed pass and timed with CUDA events on `stream`:
    one layer-batched launch (what a decode round issues), one launch per layer issued from
    the host, and those per-layer launches captured once in a CUDA graph and replayed.
    Runs outside the timed region on a sparse cache of K + T rows (the length right after the
    prefill selection); the repeated appends write the same row each time.  Returns
    microseconds per draft step for each mode, or {"error": ...} if a mode could not run."""
    import torch
    try:
        d1 = B.dims(1, wl.B, wl.Hq, wl.Hkv, wl.d, dt, wl.cap_full, wl.cap_sparse)
        sess.len_sparse.fill_(wl.K + wl.T)

        def batched():
            B.std_sparse_decode_attn_append(sess.dims, q, sess.k_sparse, sess.v_sparse, sess.len_sparse, 1,
                                            k_new, v_new, o, 0, ws)

        def per_layer(flags=0):
            for l in range(wl.L):
                B.std_sparse_decode_attn_append_ex(d1, q[l], sess.k_sparse[l], sess.v_sparse[l], sess.len_sparse, 1,
                                                   k_new[l], v_new[l], o[l], 0, flags, ws)

        def timed(fn):
            fn()
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for _ in range(reps):
                fn()
            e1.record(stream)
            torch.cuda.synchronize()
            return 1e3 * e0.elapsed_time(e1) / reps

        res = {"batched_us": timed(batched), "per_layer_eager_us": timed(per_layer)}
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, capture_error_mode="thread_local"):
            per_layer()
        res["per_layer_graph_us"] = timed(g.replay)
        del g
        # the same graph with each layer's K/V tiles fetched while the previous layer finishes
        # (its predecessor writes only another layer's rows; q is still read after the wait)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, capture_error_mode="thread_local"):
            per_layer(B.STD_ATTN_EARLY_KV)
        res["per_layer_graph_early_kv_us"] = timed(g.replay)
        del g
        res["launches_per_step"] = {"batched": 1, "per_layer": wl.L}
        res["reps"] = reps
        flags = B.std_get_device_error(clear=True)
        if flags:
            res["device_error_flags"] = flags
        return res
    except Exception as ex:  # an extra figure: never lose the bench line to it
        return {"error": f"{type(ex).__name__}: {ex}"}


def workload_config(wl, R):
    return {"workload": wl.name, "L": wl.L, "B": wl.B, "Hq": wl.Hq, "Hkv": wl.Hkv, "d": wl.d,
            "nvis": list(wl.nvis) if wl.B > 1 else wl.nvis[0], "T": wl.T, "K": wl.K, "gamma": wl.gamma,
            "rounds_per_step": R, "p_match": wl.p_match, "storage": wl.dtype,
            "step": f"prefill top-K selection + {R} draft/verify rounds (one StD decode)",
            "l2": ("inputs larger than L2 (no flush)" if not needs_l2_flush(wl)
                   else "L2 flushed before every timed step (256 MB written outside the step's events)")}


# The KV cache must exceed the 126 MB L2 by a margin for back-to-back steps to start cold;
# smaller workloads get the L2 overwritten between timed steps instead.
L2_BYTES = 126e6


def needs_l2_flush(wl):
    return kv_bytes(wl) < 2 * L2_BYTES


def kv_bytes(wl):
    return 2 * wl.L * wl.B * wl.Hkv * wl.cap_full * wl.d * wl.elem_bytes


# ----------------------------------------------------------------------------- GPU arm

def run_std(args, rank, world, local_rank):
    import numpy as np
    import torch

    import synth
    from sparse_top_kv_std_b200 import binding as B
    from sparse_top_kv_std_b200.session import DecodeSession

    if not torch.cuda.is_available():
        raise RuntimeError("bench.py needs a CUDA GPU")
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    pg = None
    if world > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=dev)
        pg = dist
    B.lib()

    wl = synth.workload(args.workload)
    R = args.rounds or wl.rounds
    if R > wl.rounds:
        wl = wl.replace(rounds=R)
    seed = args.seed + rank
    dt = B.STD_F32 if wl.dtype == "f32" else B.STD_BF16
    sess = DecodeSession(wl.L, wl.B, wl.Hq, wl.Hkv, wl.d, dt, wl.cap_full, wl.cap_sparse, wl.T, wl.K, wl.gamma,
                         wl.nvis_max, device=dev)
    stream = torch.cuda.current_stream(dev)

    # ---- inputs: generated on the host (pinned), copied once to HBM
    host_t = torch.int16 if dt == B.STD_BF16 else torch.float32
    np_t = np.uint16 if dt == B.STD_BF16 else np.float32
    pin_k = torch.zeros(tuple(sess.k_full.shape), dtype=host_t, pin_memory=True)
    pin_v = torch.zeros(tuple(sess.v_full.shape), dtype=host_t, pin_memory=True)
    nk, nvw = pin_k.numpy().view(np_t), pin_v.numpy().view(np_t)

    def sink(l, b, h, ks, vs):
        nk[l, b, h, :ks.shape[0]] = ks
        nvw[l, b, h, :vs.shape[0]] = vs

    t_gen = time.perf_counter()
    threads = args.threads or min(16, os.cpu_count() or 8)
    x = synth.host_inputs(wl, seed=seed, threads=threads, kv_sink=sink)
    t_gen = time.perf_counter() - t_gen
    names = ["q_text", "q_draft", "k_draft", "v_draft", "q_verify", "k_verify", "v_verify"]
    pin = {}
    for n in names:
        a = np.ascontiguousarray(x[n])
        t = torch.from_numpy(a.view(np.int16) if a.dtype == np.uint16 else a)
        pin[n] = t.pin_memory()
    pin["draft_tokens"] = torch.from_numpy(x["draft_tokens"]).pin_memory()
    pin["dense_tokens"] = torch.from_numpy(x["dense_tokens"]).pin_memory()
    sd = torch.bfloat16 if dt == B.STD_BF16 else torch.float32

    def to_dev(t):
        d = torch.empty(t.shape, dtype=t.dtype, device=dev)
        return d

    dv = {n: to_dev(pin[n]) for n in pin}

    def h2d_inputs():
        sess.k_full.view(host_t).copy_(pin_k, non_blocking=True)
        sess.v_full.view(host_t).copy_(pin_v, non_blocking=True)
        for n in pin:
            dv[n].copy_(pin[n], non_blocking=True)

    h2d_inputs()
    torch.cuda.synchronize()

    def view(n, r=None):
        t = dv[n] if r is None else dv[n][r]
        return t.view(sd) if t.dtype == torch.int16 else t

    EARLY_CHAIN = B.STD_ATTN_EARLY_KV | B.STD_ATTN_EARLY_Q
    len0 = torch.tensor([n + wl.T for n in wl.nvis], dtype=torch.int32, device=dev)
    nvis_dev = torch.tensor(list(wl.nvis), dtype=torch.int32, device=dev)
    sess.nvis.copy_(nvis_dev)
    outs = [sess.round_outputs() for _ in range(R)]
    # draft CTAs: step 0 of a round, and the early-started steps after it
    sp_d = ({"step_0": B.std_attn_splits(sess.dims, 1, wl.cap_sparse, 0),
             "steps_1_on": B.std_attn_splits_ex(sess.dims, 1, wl.cap_sparse, 0,
                                                B.STD_ATTN_EARLY_KV | B.STD_ATTN_EARLY_Q)}
            if wl.gamma > 0 else 1)
    sp_v = B.std_attn_splits(sess.dims, wl.gamma + 1, wl.cap_full, 0)
    ws = sess.ws_round
    q_text = view("q_text")

    class BufSet:
        """One decode's device state: a session (caches, lengths, workspaces), the round
        inputs on the device and the round outputs."""

        def __init__(self, s, d, o):
            self.sess, self.dv, self.outs, self.ws = s, d, o, s.ws_round

        def view(self, n, r=None):
            t = self.dv[n] if r is None else self.dv[n][r]
            return t.view(sd) if t.dtype == torch.int16 else t

    bs0 = BufSet(sess, dv, outs)

    def step(ev=None, draft_ev=False):
        """One StD decode: reset lengths, select, R rounds.  ev: dict of event lists to record
        (selection and verify only, unless draft_ev: events between kernels cost overlap)."""
        sess.len_full.copy_(len0, non_blocking=True)
        if ev is not None:
            ev["sel0"].record()
        sess.select(q_text, keep_scores=False)
        if ev is not None:
            ev["sel1"].record()
        rounds(ev, draft_ev)

    def rounds(ev=None, draft_ev=False, bs=None):
        bs = bs or bs0
        sess, outs, ws, view, dv = bs.sess, bs.outs, bs.ws, bs.view, bs.dv
        for r in range(R):
            o = outs[r]
            if ev is not None and not draft_ev:
                ev["dc0"][r].record()
            for j in range(wl.gamma):  # draft step j: append its input's row, attend (one launch)
                if draft_ev:
                    ev["d0"][r * wl.gamma + j].record()
                # steps after the first follow the previous step, which writes no length, no q and
                # only the sparse row before this step's: they may start reading early (not after
                # an event, which ends the overlap anyway)
                flags = EARLY_CHAIN if j > 0 and not draft_ev else 0
                B.std_sparse_decode_attn_append_ex(sess.dims, view("q_draft", r)[j], sess.k_sparse, sess.v_sparse,
                                                   sess.len_sparse, j + 1, view("k_draft", r)[j],
                                                   view("v_draft", r)[j], o["o_draft"][j], 0, flags, ws)
                if draft_ev:
                    ev["d1"][r * wl.gamma + j].record()
            if ev is not None and not draft_ev:
                ev["dc1"][r].record()
            B.std_kv_append(sess.dims, sess.k_full, sess.v_full, wl.cap_full, sess.len_full, 0,
                            view("k_verify", r), view("v_verify", r), wl.gamma + 1)
            if ev is not None:
                ev["v0"][r].record()
            B.std_dense_verify_attn(sess.dims, view("q_verify", r), wl.gamma, sess.k_full, sess.v_full,
                                    sess.len_full, o["o_verify"], 0, ws)
            if ev is not None:
                ev["v1"][r].record()
            B.std_accept_prefix(wl.B, wl.gamma, dv["draft_tokens"][r], dv["dense_tokens"][r], o["n_plus_1"],
                                o["accepted"])
            B.std_kv_commit(sess.dims, sess.k_full, sess.v_full, sess.k_sparse, sess.v_sparse, sess.len_full,
                            sess.len_sparse, o["n_plus_1"], wl.gamma + 1)
        if ev is not None:
            ev["end"].record()

    def new_events(external=False):
        # external: recorded as event nodes when captured in a CUDA graph, so that every replay
        # records them and their times can be read afterwards
        E = lambda: torch.cuda.Event(enable_timing=True, external=external)  # noqa: E731
        return {"sel0": E(), "sel1": E(), "end": E(), "d0": [E() for _ in range(R * wl.gamma)],
                "d1": [E() for _ in range(R * wl.gamma)], "v0": [E() for _ in range(R)],
                "v1": [E() for _ in range(R)], "dc0": [E() for _ in range(R)], "dc1": [E() for _ in range(R)]}

    # ---- warm-up (also yields the acceptance counts of the byte model); the clock sampler
    # starts here so that nvidia-smi is sampling by the time the timed region begins
    clk = ClockSampler(gpu_uuid(dev))
    clk.start()
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    flags = B.std_get_device_error(clear=True)
    if flags:
        raise RuntimeError(f"device error flags {flags:#x} after warm-up")
    accepted = [o["n_plus_1"].cpu().tolist() for o in outs]
    draft_b, verify_b, verify_round_b = attention_bytes(wl, R, accepted)
    step_attn = draft_b + verify_b

    # ---- one step captured in a CUDA graph (as a serving loop runs its decode steps): the
    # timed steps replay it, so the launches of a step are not issued one by one from Python.
    # The library counts its launches while the graph is captured: that count per step is
    # what every replay launches.
    graph, graph_error, gev = None, None, None
    if not args.eager:
        try:
            gev = new_events(external=True)
            graph = torch.cuda.CUDAGraph()
            n0 = B.std_launch_count()
            with torch.cuda.graph(graph, capture_error_mode="thread_local"):
                step(gev)
            per_step_launches = B.std_launch_count() - n0
            graph.replay()  # one untimed replay
            torch.cuda.synchronize()
            flags = B.std_get_device_error(clear=True)
            if flags:
                raise RuntimeError(f"device error flags {flags:#x} in the graph replay")
        except Exception as ex:  # the eager loop below still measures the step
            graph, graph_error = None, f"{type(ex).__name__}: {ex}"
            torch.cuda.synchronize()

    # ---- timed region
    evs = [gev] if graph is not None else [new_events() for _ in range(args.steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    # small workloads: overwrite L2 before every step, outside that step's own events
    flush = torch.empty(int(2 * L2_BYTES), dtype=torch.uint8, device=dev) if needs_l2_flush(wl) else None
    step_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(args.steps)] if flush is not None else None
    if pg:
        pg.barrier()
    torch.cuda.synchronize()
    w0 = time.time()
    launches0 = B.std_launch_count()  # the library's own count of the kernels it launches
    t0.record(stream)
    for i in range(args.steps):
        if flush is not None:
            flush.zero_()
            step_ev[i][0].record(stream)
        if graph is not None:
            graph.replay()  # the per-kernel events inside it keep the last replay's times
        else:
            step(evs[i])
        if flush is not None:
            step_ev[i][1].record(stream)
    t1.record(stream)
    torch.cuda.synchronize()
    w1 = time.time()
    launches = per_step_launches * args.steps if graph is not None else B.std_launch_count() - launches0
    clocks = clk.stop(window=(w0, w1))
    if pg:
        pg.barrier()
    elapsed_ms = t0.elapsed_time(t1) if flush is None else sum(a.elapsed_time(b) for a, b in step_ev)
    flags = B.std_get_device_error(clear=True)
    if flags:
        raise RuntimeError(f"device error flags {flags:#x} in the timed region")

    sel_ms = [e["sel0"].elapsed_time(e["sel1"]) for e in evs]
    v_ms = [e["v0"][r].elapsed_time(e["v1"][r]) for e in evs for r in range(R)]
    rounds_ms = [e["sel1"].elapsed_time(e["end"]) for e in evs]
    # the gamma draft launches of each round as one chain (events around the chain only, so the
    # launches inside it overlap as they do untimed)
    dchain_ms = [e["dc0"][r].elapsed_time(e["dc1"][r]) for e in evs for r in range(R)] if wl.gamma > 0 else [0.0]
    # per-launch draft timing from one instrumented step outside the timed region
    dev_ev = new_events()
    step(dev_ev, draft_ev=True)
    torch.cuda.synchronize()
    d_ms = [dev_ev["d0"][k].elapsed_time(dev_ev["d1"][k]) for k in range(R * wl.gamma)]
    elapsed_ms = dist_max(elapsed_ms, pg, dev)

    # ---- e2e through the public API with host buffers (H2D of inputs, D2H of the accepted tokens)
    e2e = None
    if not args.no_e2e and args.e2e_steps > 0:
        acc_host = torch.zeros((R, wl.B, wl.gamma + 1), dtype=torch.int32, pin_memory=True)
        acc_dev = torch.zeros((R, wl.B, wl.gamma + 1), dtype=torch.int32, device=dev)

        copy_stream = torch.cuda.Stream(device=dev)
        d1 = B.dims(1, wl.B, wl.Hq, wl.Hkv, wl.d, dt, wl.cap_full, wl.cap_sparse)
        # two buffer sets, taken in turn: the next prompt's cache uploads while this one decodes
        sets = [bs0]
        if args.e2e_steps >= 2:
            s2 = DecodeSession(wl.L, wl.B, wl.Hq, wl.Hkv, wl.d, dt, wl.cap_full, wl.cap_sparse, wl.T, wl.K,
                               wl.gamma, wl.nvis_max, device=dev)
            s2.nvis.copy_(nvis_dev)
            sets.append(BufSet(s2, {n: to_dev(pin[n]) for n in pin}, [s2.round_outputs() for _ in range(R)]))
        layer_ev = [[torch.cuda.Event() for _ in range(wl.L)] for _ in sets]
        rest_ev = [torch.cuda.Event() for _ in sets]
        done_ev = [torch.cuda.Event() for _ in sets]

        def e2e_step(k):
            # the prompt cache and the text queries arrive layer by layer on a copy stream, and
            # each layer's selection starts as soon as its rows have landed; the rounds need
            # every layer, so they wait for the whole copy
            bs = sets[k]
            s = bs.sess
            copy_stream.wait_event(done_ev[k])  # the step before on this set is done with it
            with torch.cuda.stream(copy_stream):
                kf_h, vf_h = s.k_full.view(host_t), s.v_full.view(host_t)
                for l in range(wl.L):
                    kf_h[l].copy_(pin_k[l], non_blocking=True)
                    vf_h[l].copy_(pin_v[l], non_blocking=True)
                    bs.dv["q_text"][l].copy_(pin["q_text"][l], non_blocking=True)
                    layer_ev[k][l].record(copy_stream)
                for n in pin:
                    if n != "q_text":
                        bs.dv[n].copy_(pin[n], non_blocking=True)
                rest_ev[k].record(copy_stream)
            s.len_full.copy_(len0, non_blocking=True)
            qt = bs.view("q_text")
            for l in range(wl.L):
                stream.wait_event(layer_ev[k][l])
                B.std_select_topk(d1, qt[l], wl.T, s.k_full[l], s.v_full[l], s.nvis, wl.nvis_max, wl.K, s.idx[l],
                                  s.k_sparse[l], s.v_sparse[l], s.len_sparse, None, s.ws_select)
            stream.wait_event(rest_ev[k])
            rounds(bs=bs)
            for r in range(R):
                acc_dev[r].copy_(bs.outs[r]["accepted"], non_blocking=True)
            acc_host.copy_(acc_dev, non_blocking=True)
            done_ev[k].record(stream)

        for k in range(len(sets)):
            e2e_step(k)
        torch.cuda.synchronize()
        a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        if pg:
            pg.barrier()
        torch.cuda.synchronize()
        a0.record(stream)
        for i in range(args.e2e_steps):
            e2e_step(i % len(sets))
        a1.record(stream)
        torch.cuda.synchronize()
        e_ms = dist_max(a0.elapsed_time(a1), pg, dev)
        # the same prompt in either buffer set: the accepted tokens read back must equal the
        # timed region's
        if not torch.equal(acc_host, torch.stack([o["accepted"] for o in outs]).cpu()):
            raise RuntimeError("end-to-end steps accepted other tokens than the timed steps")
        h2d = pin_k.numel() * pin_k.element_size() * 2 + sum(t.numel() * t.element_size() for t in pin.values())
        d2h = acc_host.numel() * 4
        e2e = {"value": weak_scaling_value(step_attn, args.e2e_steps, world, e_ms), "unit": "GB/s",
               "ms_per_step": e_ms / args.e2e_steps, "steps": args.e2e_steps,
               "pipeline": "two buffer sets taken in turn: each prompt's cache is copied layer by layer on a "
                           "second stream while the previous prompt decodes, and each layer is selected as it "
                           "lands",
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h)}

    if rank != 0:
        if pg:
            pg.destroy_process_group()
        return 0

    draft_modes = None
    if not args.no_draft_modes and wl.gamma > 0:
        draft_modes = draft_launch_modes(B, sess, wl, dt, view("q_draft", 0)[0], view("k_draft", 0)[0],
                                         view("v_draft", 0)[0], outs[0]["o_draft"][0], ws, stream)

    peaks, peak_src = load_peaks()
    value = weak_scaling_value(step_attn, args.steps, world, elapsed_ms)
    v_avg_ms = statistics.mean(v_ms)
    v_bytes_avg = verify_b / R
    achieved = v_bytes_avg / (v_avg_ms / 1e3) / 1e9
    d_avg_ms = statistics.mean(dchain_ms) / max(1, wl.gamma)   # per launch, inside the timed region
    d_iso_ms = statistics.mean(d_ms)                            # per launch, each between events
    d_bytes_avg = draft_b / max(1, R * wl.gamma)
    sel_avg = statistics.mean(sel_ms)
    traffic = load_traffic("dense_verify_attn", wl.name)
    line = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": elapsed_ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16" if dt == B.STD_BF16 else "f32",
        "data": "synthetic", "config": workload_config(wl, R),
        "us_per_round": 1e3 * statistics.mean(rounds_ms) / R,
        # the same draft + verify bytes over the rounds' own time (the step without its selection)
        "rounds_GBps": step_attn / (statistics.mean(rounds_ms) / 1e3) / 1e9,
        "select_ms": sel_avg,
        "kernels": {
            "dense_verify_attn": {"ms_per_launch": v_avg_ms, "bytes_per_launch": v_bytes_avg,
                                  "GBps": achieved, "frac_of_8TBps": achieved / 8000.0, "ctas": sp_v},
            "sparse_decode_attn": {"timing": "the round's draft chain (gamma launches) between CUDA events in "
                                             "the timed region, divided by gamma",
                                   "us_per_launch": 1e3 * d_avg_ms, "bytes_per_launch": d_bytes_avg,
                                   "GBps": d_bytes_avg / (d_avg_ms / 1e3) / 1e9,
                                   "frac_of_8TBps": d_bytes_avg / (d_avg_ms / 1e3) / 8e12, "ctas": sp_d,
                                   "us_per_launch_isolated": 1e3 * d_iso_ms,
                                   "isolated_timing": "each launch between CUDA events, one step outside the "
                                                      "timed region, no early start",
                                   "launch_modes": draft_modes},
            "select_topk": select_figures(wl, sel_avg, peaks, peak_src),
        },
        "roofline": {"kernel": "dense_verify_attn (verify attention + split merge)", "bound": "hbm",
                     "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": achieved / peaks["hbm_gbs"], "traffic": traffic,
                     "peak_source": f"{peak_src} HBM copy bandwidth"},
        "gpu_launches": launches,
        "launch": ("one CUDA graph per step (captured once, replayed each step; the library's launch count is "
                   "taken while capturing)" if graph is not None else "eager (host-issued launches)"
                   + (f"; graph capture failed: {graph_error}" if graph_error else "")),
        "clocks": clocks,
        "e2e": e2e,
        "input_gen_s": t_gen,
    }
    if world == 1 and not args.no_cpu_baseline:
        v, t_sel, t_round, est = cpu_estimate(wl, seed, R, step_attn, 2, [(0, 0, 0)])
        line["cpu_baseline"] = {
            "value": v, "unit": "GB/s", "cores": blas_threads(), "kind": "oracle",
            "sample": (f"fp64 oracle on one (layer, KV head) slice of {wl.name}: its prefill selection "
                       f"({t_sel:.1f} s) and 2 draft+verify rounds ({2 * t_round:.1f} s), scaled to all "
                       f"{wl.L * wl.B * wl.Hkv} slices and {R} rounds (est. {est:.0f} s per step)")}
    print(json.dumps(line), flush=True)
    if pg:
        pg.destroy_process_group()
    return 0


def gpu_uuid(dev):
    try:
        import torch
        u = str(torch.cuda.get_device_properties(dev).uuid)
        return u if u.startswith("GPU-") else "GPU-" + u
    except Exception:
        return None


TRAFFIC_FILE = os.path.join(ROOT, "profiles", "dram_traffic_dense_verify_attn_video_140k.txt")


def sources_sha256(paths):
    """sha256 over the concatenated bytes of the given repo-relative files."""
    h = hashlib.sha256()
    for rel in paths:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def load_traffic(kernel, workload, path=TRAFFIC_FILE):
    """DRAM bytes per launch from a committed ncu summary ("key: value" lines), or None when the
    summary is missing, is for another kernel or workload, or its kernel sources changed since."""
    if not os.path.exists(path):
        return None
    kv = {}
    with open(path) as f:
        for line in f:
            if ":" in line and not line.startswith((" ", "#")):
                k, v = line.split(":", 1)
                kv[k.strip()] = v.strip()
    if kv.get("kernel") != kernel or kv.get("workload") != workload:
        return None
    srcs = kv.get("sources", "").split()
    if not srcs or not all(os.path.exists(os.path.join(ROOT, r)) for r in srcs):
        return None
    if sources_sha256(srcs) != kv.get("sources_sha256"):
        return None
    return float(kv["dram_bytes_per_launch"])


def main(argv=None):
    args = parse_args(argv)
    rank, world, local_rank = dist_env()
    if args.impl == "reference":
        return run_reference(args, rank, world)
    return run_std(args, rank, world, local_rank)


if __name__ == "__main__":
    sys.exit(main())
