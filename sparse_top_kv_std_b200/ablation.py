"""Gamma / K ablation of Sparse-to-Dense decoding on the batch-8 ragged sweep.

    python -m sparse_top_kv_std_b200.ablation [--rounds 32] [--reps 3] [--json out.json]

The gist.science summary ("Experimentelle Ergebnisse", item "Hyperparameter")
reports that a longer draft raises the speed-up up to about gamma = 9 and lowers
it beyond.  This sweep asks the same question of the decode attention on one
GPU: for K in {512, 1024, 4096}, gamma in {2, 4, 6, 8, 10} and draft/dense match
probability p in {0.6, 0.9} it measures, through the library,

  * us per round: gamma x (append + sparse draft attention), append + dense
    verify attention, acceptance, commit, for a batch of 8 sequences with visual
    lengths uniform in [16k, 64k] (one attention layer, 28 query / 4 KV heads,
    d = 128, bf16);
  * tokens per round: the mean of n + 1 over the sequences and rounds (the
    acceptance streams draw i.i.d. matches with probability p);
  * us per token, and the speed-up over plain dense decoding (append + one-row
    dense attention per token, the same batch and lengths);

next to the attention-I/O model: with i.i.d. matches E[n + 1] =
sum_{i <= gamma} p^i, and a round reads gamma x K' sparse rows plus
N_ctx + gamma + 1 full rows against N_ctx per dense token, so the I/O speed-up
is N_ctx E / (gamma K' + N_ctx + gamma + 1) (summed over the batch).

The prompt cache of the first sweep point serves every point (its values do not
change the timings); queries, new rows and token streams are drawn per point.
Everything runs on the CUDA library; nothing here computes a step of the method.
"""
from __future__ import annotations

import argparse
import json
import statistics
import sys

import numpy as np
import torch

import synth
from sparse_top_kv_std_b200 import binding as B
from sparse_top_kv_std_b200.session import DecodeSession

KS = (512, 1024, 4096)
GAMMAS = (2, 4, 6, 8, 10)
PS = (0.6, 0.9)


def _dev(x):
    x = np.ascontiguousarray(x)
    if x.dtype == np.uint16:
        return torch.from_numpy(x.view(np.int16)).cuda().view(torch.bfloat16)
    return torch.from_numpy(x).cuda()


def io_model(nvis, T, K, gamma, p):
    """Attention-I/O speed-up of one round over dense decoding, i.i.d. matches."""
    e = sum(p ** i for i in range(gamma + 1))
    n_ctx = np.asarray(nvis, np.float64) + T
    k_sp = K + T
    return float((n_ctx * e).sum() / (gamma * k_sp + n_ctx + gamma + 1).sum()), e


def dense_us_per_token(master_k, master_v, wl, steps, reps):
    """Plain greedy decoding's attention: append one row, attend over the whole cache."""
    cap = master_k.shape[3]
    d = B.dims(1, wl.B, wl.Hq, wl.Hkv, wl.d, B.STD_BF16, cap, cap)
    g = torch.Generator(device="cuda").manual_seed(7)
    q = torch.randn((1, wl.B, wl.Hq, 1, wl.d), generator=g, device="cuda").to(torch.bfloat16)
    kn = torch.randn((1, wl.B, wl.Hkv, 1, wl.d), generator=g, device="cuda").to(torch.bfloat16)
    o = torch.empty((1, wl.B, wl.Hq, 1, wl.d), device="cuda")
    ws = torch.empty(max(16, B.std_attn_workspace_size(d, 1, cap, 0)), dtype=torch.uint8, device="cuda")
    base = torch.tensor([n + wl.T for n in wl.nvis], dtype=torch.int32, device="cuda")
    times = []
    for rep in range(reps + 1):
        ln = base.clone()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        e0.record()
        for _ in range(steps):
            B.std_kv_append(d, master_k, master_v, cap, ln, 0, kn, kn, 1)
            B.std_dense_verify_attn(d, q, 0, master_k, master_v, ln, o, 0, ws)
            ln += 1
        e1.record()
        torch.cuda.synchronize()
        if rep > 0:  # the first repetition warms up
            times.append(e0.elapsed_time(e1) * 1e3 / steps)
    return statistics.median(times)


def run_point(master_k, master_v, K, gamma, p, rounds, reps, seed=0):
    wl = synth.ragged_workload(K, gamma, p, seed=seed, rounds=rounds)
    x = synth.host_inputs(wl, seed=seed, heads=[], kv_sink=lambda *a: None)
    s = DecodeSession(wl.L, wl.B, wl.Hq, wl.Hkv, wl.d, B.STD_BF16, wl.cap_full, wl.cap_sparse, wl.T, K, gamma,
                      wl.nvis_max)
    n = master_k.shape[3]
    s.k_full[..., :n, :].copy_(master_k)
    s.v_full[..., :n, :].copy_(master_v)
    q_text = _dev(x["q_text"])
    ios = []
    for r in range(rounds):
        io = {k: _dev(x[k][r]) for k in ("q_draft", "k_draft", "v_draft", "q_verify", "k_verify", "v_verify")}
        io["draft_tokens"] = torch.from_numpy(x["draft_tokens"][r]).cuda()
        io["dense_tokens"] = torch.from_numpy(x["dense_tokens"][r]).cuda()
        io.update(s.round_outputs())
        ios.append(io)
    times, toks = [], []
    for rep in range(reps + 1):
        s.start(x["nvis"])
        s.select(q_text, keep_scores=False)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        e0.record()
        for io in ios:
            s.round(io)
        e1.record()
        torch.cuda.synchronize()
        if rep > 0:
            times.append(e0.elapsed_time(e1) * 1e3 / rounds)
            toks.append(float(np.mean([io["n_plus_1"].float().mean().item() for io in ios])))
    flags = B.std_get_device_error()
    if flags:
        raise RuntimeError(f"device error flags {flags:#x}")
    return wl, statistics.median(times), statistics.mean(toks)


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--rounds", type=int, default=32)
    ap.add_argument("--reps", type=int, default=3)
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--json", default=None)
    args = ap.parse_args(argv)
    if not torch.cuda.is_available():
        print("needs a CUDA device", file=sys.stderr)
        return 2
    B.lib()
    wl0 = synth.ragged_workload(KS[0], GAMMAS[0], PS[0], seed=args.seed, rounds=args.rounds)
    n = max(wl0.nvis) + wl0.T
    master_k = torch.zeros((1, wl0.B, wl0.Hkv, n + args.rounds + 1, wl0.d), dtype=torch.bfloat16, device="cuda")
    master_v = torch.zeros_like(master_k)

    def sink(l, b, h, ks, vs):
        master_k[l, b, h, :ks.shape[0]].copy_(_dev(ks))
        master_v[l, b, h, :vs.shape[0]].copy_(_dev(vs))
    synth.host_inputs(wl0, seed=args.seed, kv_sink=sink)
    dense_us = dense_us_per_token(master_k, master_v, wl0, args.rounds, args.reps)
    mk, mv = master_k[..., :n, :].contiguous(), master_v[..., :n, :].contiguous()
    rows = []
    for K in KS:
        for p in PS:
            for gamma in GAMMAS:
                wl, us_round, tok = run_point(mk, mv, K, gamma, p, args.rounds, args.reps, args.seed)
                model, e = io_model(wl.nvis, wl.T, K, gamma, p)
                rows.append({"K": K, "p": p, "gamma": gamma, "us_per_round": us_round, "tokens_per_round": tok,
                             "us_per_token": us_round / tok, "speedup": dense_us / (us_round / tok),
                             "io_model_speedup": model, "io_model_tokens_per_round": e})
    best = {}
    for r in rows:
        key = (r["K"], r["p"])
        if key not in best or r["speedup"] > best[key]["speedup"]:
            best[key] = r
    print(f"dense decoding: {dense_us:.1f} us per token (batch 8, visual lengths {list(wl0.nvis)} + "
          f"{wl0.T} text)")
    print("| K | p | gamma | us/round | tokens/round (i.i.d. model) | us/token | speed-up measured | "
          "speed-up I/O model |")
    print("|---|---|---|---|---|---|---|---|")
    for r in rows:
        mark = " **best**" if best[(r["K"], r["p"])] is r else ""
        print(f"| {r['K']} | {r['p']} | {r['gamma']} | {r['us_per_round']:.1f} | {r['tokens_per_round']:.2f} "
              f"({r['io_model_tokens_per_round']:.2f}) | {r['us_per_token']:.1f} | {r['speedup']:.2f}x{mark} | "
              f"{r['io_model_speedup']:.2f}x |")
    if args.json:
        with open(args.json, "w") as f:
            json.dump({"dense_us_per_token": dense_us, "nvis": list(wl0.nvis), "T": wl0.T, "rows": rows}, f, indent=1)
    return 0


if __name__ == "__main__":
    sys.exit(main())
