"""A KV cache split by sequence position over several GPUs (one process per GPU).

The summary keeps every KV cache in one GPU's HBM ("Bedeutung"); at 140k visual
tokens per prompt one GPU's memory bounds the context.  Splitting the cache by
position needs one exchange per attention call: every rank attends its own rows
(``std_dense_verify_attn_partial`` / ``std_sparse_decode_attn_partial``), the
per-row partials (o, m, l) -- a few KB -- are all-gathered, and
``std_merge_partials`` combines them.  This module holds the host side of that:
which rows each rank keeps, where a global position lives, and the all-gather
into the [world][rows][...] layout the merge reads.  The prefill selection over
such a cache (``sharded_select``) needs two exchanges: the text rows' softmax
statistics (m, l) after the first score pass, and each rank's top-K candidates
after the second; the selected rows are then copied by the rank that holds them
and summed into every rank's sparse cache.  torch is used for the collectives
and for buffers only; every step of the attention and the selection runs in the
library's kernels.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import List, Tuple

# shard boundaries fall on multiples of the attention kernel's 128-key tile
ALIGN = 128


@dataclass(frozen=True)
class Shard:
    """Rows [pos0, pos0 + rows) of every sequence's cache live on `rank`."""

    rank: int
    pos0: int
    rows: int

    @property
    def end(self) -> int:
        return self.pos0 + self.rows


def partition(prompt_len: int, cap: int, world: int, align: int = ALIGN) -> List[Shard]:
    """Contiguous shards of a cache with capacity `cap` positions.

    The prompt's `prompt_len` positions are spread evenly over the ranks (shard
    starts rounded to `align`); the last rank also holds every position after the
    prompt, so the rows a decode appends (verify inputs, accepted tokens) always
    land on it and only it.  Returns one Shard per rank, in rank order, covering
    [0, cap) without overlap.
    """
    if world < 1:
        raise ValueError("world must be >= 1")
    if not 0 <= prompt_len <= cap:
        raise ValueError("need 0 <= prompt_len <= cap")
    starts = [0]
    for r in range(1, world):
        s = (prompt_len * r // world) // align * align
        starts.append(max(s, starts[-1]))
    ends = starts[1:] + [cap]
    return [Shard(r, s, e - s) for r, (s, e) in enumerate(zip(starts, ends))]


def owner(shards: List[Shard], pos: int) -> Tuple[int, int]:
    """(rank, local row) of global position `pos`."""
    for sh in shards:
        if sh.pos0 <= pos < sh.end:
            return sh.rank, pos - sh.pos0
    raise IndexError(f"position {pos} outside the cache")


def visual_part(shard: Shard, n_prefix: int, nvis) -> Tuple[int, List[int]]:
    """This shard's share of every sequence's visual block, for a cache [n_prefix rows |
    nvis[b] visual rows | text rows]: (the shard-local row of its first visual key, the
    number of visual keys of each sequence it holds).  Visual key n of sequence b sits at
    global position n_prefix + n."""
    lo = max(shard.pos0, n_prefix)
    return lo - shard.pos0, [max(0, min(shard.end, n_prefix + int(nv)) - lo) for nv in nvis]


def visual_offset(shard: Shard, n_prefix: int) -> int:
    """Global visual index of the shard's first visual key (the same for every sequence)."""
    return max(shard.pos0, n_prefix) - n_prefix


def all_gather_rank_major(x, group=None):
    """All-gather this rank's tensor into [world][*x.shape], rank-major."""
    import torch
    import torch.distributed as dist
    world = dist.get_world_size(group)
    x = x.contiguous()
    flat = torch.empty((world * x.shape[0],) + tuple(x.shape[1:]), dtype=x.dtype, device=x.device)
    dist.all_gather_into_tensor(flat, x, group=group)
    return flat.view((world,) + tuple(x.shape))


def all_gather_partials(o_part, ml_part, group=None):
    """All-gather this rank's partials into ([world][*o_part.shape], [world][*ml_part.shape])
    tensors, rank-major: the layout std_merge_partials reads as [n_parts][rows][...]."""
    # the concatenated form (every backend takes it), viewed rank-major afterwards
    return all_gather_rank_major(o_part, group), all_gather_rank_major(ml_part, group)


def sharded_verify(dims_local, shard: Shard, q, gamma, k_local, v_local, len_full, o, ws=None, group=None,
                   splits=0, stream=None):
    """Dense verify attention over a cache split by position: this rank's partial over its
    shard (buffers k_local / v_local [L][B][Hkv][shard rows][d], dims_local.cap_full = shard
    rows, len_full the global committed lengths), the all-gather, and the merge into o
    [L][B][Hq][gamma + 1][d].  Every rank ends with the full output."""
    import torch

    from . import binding as B
    rows = o.numel() // o.shape[-1]
    o_part = torch.empty_like(o)
    ml_part = torch.empty(o.shape[:-1] + (2,), dtype=torch.float32, device=o.device)
    B.std_dense_verify_attn_partial(dims_local, q, gamma, k_local, v_local, len_full, shard.pos0, 0, shard.rows,
                                    o_part, ml_part, splits, ws, stream)
    o_all, ml_all = all_gather_partials(o_part, ml_part, group)
    B.std_merge_partials(rows, o.shape[-1], o_all.shape[0], o_all, ml_all, o, stream)
    return o


def sharded_select(dims_local, shards: List[Shard], rank: int, q_text, T: int, k_local, v_local, nvis, nvis_dev,
                   n_prefix: int, K: int, idx_out, k_sparse, v_sparse, len_sparse, group=None, stream=None):
    """Prefill selection over a cache split by position: this rank holds global positions
    [shards[rank].pos0, shards[rank].end) of every (layer, sequence, KV head) in k_local /
    v_local (dims_local.cap_full = that buffer's capacity), q_text is every rank's copy of
    the text queries, nvis the host list and nvis_dev the device copy of the visual counts.
    Every rank ends with idx_out [L][B][Hkv][K] (global visual indices, ascending) and the
    whole sparse cache [n_prefix | K selected | T text rows] in k_sparse / v_sparse, as
    std_select_topk_ex (flags 0) gives on the unsplit cache.  Every shard must hold at
    least K visual keys of every sequence."""
    import torch
    import torch.distributed as dist

    from . import binding as B
    shard = shards[rank]
    world = len(shards)
    p_loc, counts = visual_part(shard, n_prefix, nvis)
    if min(counts) < K:
        raise ValueError(f"rank {rank} holds {min(counts)} visual keys of some sequence, fewer than K = {K}")
    dev = k_local.device
    L, Bn, Hq, Hkv = dims_local.L, dims_local.B, dims_local.Hq, dims_local.Hkv
    probs, rows = L * Bn * Hkv, (Hq // Hkv) * T
    nv_loc = torch.tensor(counts, dtype=torch.int32, device=dev)
    nv_max = max(counts)
    # pass 1 on this rank's keys, the exchange of (m, l), their merge
    m = torch.empty((probs, rows), dtype=torch.float32, device=dev)
    l = torch.empty_like(m)
    B.std_select_rowstats(dims_local, q_text, T, k_local, nv_loc, nv_max, p_loc, m, l, stream)
    m_all, l_all = all_gather_rank_major(m, group), all_gather_rank_major(l, group)
    B.std_merge_rowstats(probs * rows, world, m_all, l_all, m, l, stream)
    # pass 2 against the merged statistics, this rank's candidates, their exchange and merge
    cand_idx = torch.empty((probs, K), dtype=torch.int32, device=dev)
    cand_score = torch.empty((probs, K), dtype=torch.float32, device=dev)
    ws = torch.empty(B.std_select_candidates_workspace_size(dims_local, nv_max), dtype=torch.uint8, device=dev)
    B.std_select_candidates(dims_local, q_text, T, k_local, nv_loc, nv_max, p_loc, m, l, K, cand_idx, cand_score,
                            None, ws, stream)
    ci_all, cs_all = all_gather_rank_major(cand_idx, group), all_gather_rank_major(cand_score, group)
    offsets = torch.tensor([[visual_offset(sh, n_prefix)] * Bn for sh in shards], dtype=torch.int32, device=dev)
    ws2 = torch.empty(B.std_merge_candidates_workspace_size(dims_local, world, K), dtype=torch.uint8, device=dev)
    B.std_merge_candidates(dims_local, world, K, ci_all, cs_all, offsets, idx_out, ws2, stream)
    # the selected rows this rank holds, zeros for the others, summed over the ranks
    k_sparse.zero_()
    v_sparse.zero_()
    B.std_gather_sparse_part(dims_local, k_local, v_local, nvis_dev, idx_out, K, T, n_prefix, shard.pos0, shard.rows,
                             k_sparse, v_sparse, len_sparse, stream)
    dist.all_reduce(k_sparse, group=group)
    dist.all_reduce(v_sparse, group=group)
    return idx_out
