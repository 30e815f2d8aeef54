"""The cache split by position over ranks (sparse_top_kv_std_b200.seqshard), on CPU:
the partition, position ownership, and two gloo ranks that each attend only their own
shard and exchange partials with the module's all-gather.  The per-rank partials and
the merge are the fp64 oracle's (test side), so this checks the host bookkeeping --
which rows each rank holds, the shard's first position, the rank-major gathered
layout -- against dense verify attention over the whole cache."""
import os
import socket
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

from sparse_top_kv_std_b200 import seqshard

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_partition_covers_the_cache_and_puts_the_tail_on_the_last_rank():
    for prompt, cap, world in ((143616, 143904, 8), (1000, 1100, 3), (100, 120, 4), (0, 10, 2), (5000, 5000, 1)):
        sh = seqshard.partition(prompt, cap, world)
        assert [s.rank for s in sh] == list(range(world))
        assert sh[0].pos0 == 0 and sh[-1].end == cap
        for a, b in zip(sh[:-1], sh[1:]):
            assert a.end == b.pos0 and a.pos0 % seqshard.ALIGN == 0
        assert sh[-1].pos0 <= prompt                      # appended rows land on the last rank
        sizes = [s.rows for s in sh[:-1]]
        if world > 1 and prompt >= world * seqshard.ALIGN:
            assert max(sizes) - min(sizes) <= seqshard.ALIGN
    sh = seqshard.partition(1000, 1100, 3)
    for pos in (0, 127, sh[1].pos0, sh[1].pos0 - 1, 1099):
        r, loc = seqshard.owner(sh, pos)
        assert sh[r].pos0 + loc == pos and 0 <= loc < sh[r].rows
    with pytest.raises(IndexError):
        seqshard.owner(sh, 1100)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _inputs(seed=21):
    rng = np.random.default_rng(seed)
    L, B, Hq, Hkv, d, gamma = 2, 2, 4, 2, 16, 3
    n_ctx = np.array([700, 455])
    cap = 720
    k = rng.standard_normal((L, B, Hkv, cap, d)) * 1.5
    v = rng.standard_normal((L, B, Hkv, cap, d))
    q = rng.standard_normal((L, B, Hq, gamma + 1, d)) * 1.5
    return q, k, v, n_ctx, cap


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import datetime

    import torch
    import torch.distributed as dist

    import oracle
    from sparse_top_kv_std_b200 import seqshard as ss
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    q, k, v, n_ctx, cap = _inputs()
    shards = ss.partition(int(n_ctx.max()), cap, world)
    mine = shards[rank]
    k_loc = k[:, :, :, mine.pos0:mine.end].copy()        # this rank holds only its rows
    v_loc = v[:, :, :, mine.pos0:mine.end].copy()
    o, m, l = oracle.attn_range_partial(q, k_loc, v_loc, n_ctx + 1, mine.pos0, 0, mine.rows)
    ml = np.stack([m, l], axis=-1)
    o_all, ml_all = ss.all_gather_partials(torch.from_numpy(o), torch.from_numpy(ml))
    merged = oracle.merge_partials(o_all.numpy(), ml_all[..., 0].numpy(), ml_all[..., 1].numpy())
    dist.barrier()
    dist.destroy_process_group()
    out.put((rank, mine.pos0, mine.rows, merged))


@pytest.mark.parametrize("world", [2, 3])
def test_gloo_ranks_attend_their_shards_and_merge_to_dense_verify(world):
    import oracle
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted((out.get(timeout=180) for _ in range(world)), key=lambda t: t[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    q, k, v, n_ctx, cap = _inputs()
    want = oracle.dense_verify_attn(q, k, v, n_ctx)
    assert sum(r[2] for r in res) == cap
    for rank, pos0, rows, merged in res:
        np.testing.assert_allclose(merged, want, atol=1e-12, rtol=0)
