"""The prefill selection over a cache split by position (sparse_top_kv_std_b200.seqshard),
on CPU: which visual keys each rank holds and where they start, and three gloo ranks that
each score only their own keys and exchange the row statistics and the top-K candidates
with the module's all-gather.  The per-rank steps are the fp64 oracle's (test side), so
this checks the host bookkeeping -- the ranks' visual ranges and offsets, the rank-major
gathered layouts -- against the selection over the whole cache."""
import os
import socket
import sys

import numpy as np
import torch.multiprocessing as mp

from sparse_top_kv_std_b200 import seqshard

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_visual_part_and_offset_cover_every_visual_key_once():
    for prompt, cap, world, n_prefix, nvis in ((1000, 1100, 3, 40, (900, 700)), (4200, 4400, 4, 0, (4000, 3100)),
                                               (700, 760, 2, 100, (550,))):
        shards = seqshard.partition(prompt, cap, world)
        for b, nv in enumerate(nvis):
            seen = []
            for sh in shards:
                p_loc, counts = seqshard.visual_part(sh, n_prefix, nvis)
                off = seqshard.visual_offset(sh, n_prefix)
                for n in range(off, off + counts[b]):
                    assert sh.pos0 + p_loc + (n - off) == n_prefix + n     # the key's global position
                seen += list(range(off, off + counts[b]))
            assert seen == list(range(nv))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _inputs(seed=31):
    rng = np.random.default_rng(seed)
    L, B, Hq, Hkv, d, T, K, P = 2, 2, 4, 2, 16, 5, 24, 30
    nvis = np.array([520, 410])
    cap = P + int(nvis.max()) + T + 10
    k = rng.standard_normal((L, B, Hkv, cap, d)) * 1.5
    v = rng.standard_normal((L, B, Hkv, cap, d))
    q = rng.standard_normal((L, B, Hq, T, d)) * 1.5
    return q, k, v, nvis, T, K, P, cap


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import datetime

    import torch
    import torch.distributed as dist

    import oracle
    from sparse_top_kv_std_b200 import seqshard as ss
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    q, k, v, nvis, T, K, P, cap = _inputs()
    L, B, Hq = q.shape[:3]
    Hkv = k.shape[2]
    G = Hq // Hkv
    shards = ss.partition(P + int(nvis.max()) + T, cap, world)
    mine = shards[rank]
    k_loc = k[:, :, :, mine.pos0:mine.end].copy()           # this rank holds only its rows
    p_loc, counts = ss.visual_part(mine, P, nvis)
    # pass 1 on this rank's visual keys; exchange; merge
    m = np.zeros((L, B, Hkv, G * T))
    l = np.zeros_like(m)
    for li in range(L):
        for b in range(B):
            for h in range(Hkv):
                m[li, b, h], l[li, b, h] = oracle.selection_rowstats(
                    q[li, b, h * G:(h + 1) * G], k_loc[li, b, h, p_loc:p_loc + counts[b]])
    m_all = ss.all_gather_rank_major(torch.from_numpy(m)).numpy()
    l_all = ss.all_gather_rank_major(torch.from_numpy(l)).numpy()
    mg, lg = oracle.merge_rowstats(m_all, l_all)
    # pass 2 against the merged statistics; this rank's candidates; exchange; merge
    ci = np.zeros((L, B, Hkv, K), np.int32)
    cs = np.zeros((L, B, Hkv, K))
    for li in range(L):
        for b in range(B):
            for h in range(Hkv):
                sc = oracle.selection_scores_given_rowstats(q[li, b, h * G:(h + 1) * G],
                                                            k_loc[li, b, h, p_loc:p_loc + counts[b]],
                                                            mg[li, b, h], lg[li, b, h])
                ci[li, b, h], cs[li, b, h] = oracle.topk_candidates(sc, K)
    ci_all = ss.all_gather_rank_major(torch.from_numpy(ci)).numpy()
    cs_all = ss.all_gather_rank_major(torch.from_numpy(cs)).numpy()
    offs = [ss.visual_offset(sh, P) for sh in shards]
    idx = np.zeros((L, B, Hkv, K), np.int32)
    for li in range(L):
        for b in range(B):
            for h in range(Hkv):
                idx[li, b, h] = oracle.merge_candidates(
                    [(offs[r], ci_all[r, li, b, h], cs_all[r, li, b, h]) for r in range(world)], K)
    dist.barrier()
    dist.destroy_process_group()
    out.put((rank, idx))


def test_three_ranks_select_what_the_whole_cache_selects():
    world = 3
    port = _free_port()
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    got = dict(out.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    sys.path.insert(0, ROOT)
    import oracle
    q, k, v, nvis, T, K, P, cap = _inputs()
    idx, *_ = oracle.select_topk(q, k, v, nvis, T, K, K + T + P, n_prefix=P)
    for r in range(world):
        np.testing.assert_array_equal(got[r], idx)
