"""A KV cache split by sequence position over several GPUs (one process per GPU).

The summary keeps every KV cache in one GPU's HBM ("Bedeutung"); at 140k visual
tokens per prompt one GPU's memory bounds the context.  Splitting the cache by
position needs one exchange per attention call: every rank attends its own rows
(``std_dense_verify_attn_partial`` / ``std_sparse_decode_attn_partial``), the
per-row partials (o, m, l) -- a few KB -- are all-gathered, and
``std_merge_partials`` combines them.  This module holds the host side of that:
which rows each rank keeps, where a global position lives, and the all-gather
into the [world][rows][...] layout the merge reads.  torch is used for the
collective and for buffers only; every step of the attention runs in the
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


def all_gather_partials(o_part, ml_part, group=None):
    """All-gather this rank's partials into ([world][*o_part.shape], [world][*ml_part.shape])
    tensors, rank-major: the layout std_merge_partials reads as [n_parts][rows][...]."""
    import torch
    import torch.distributed as dist
    world = dist.get_world_size(group)
    out = []
    for x in (o_part.contiguous(), ml_part.contiguous()):
        # the concatenated form (every backend takes it), viewed rank-major afterwards
        flat = torch.empty((world * x.shape[0],) + tuple(x.shape[1:]), dtype=x.dtype, device=x.device)
        dist.all_gather_into_tensor(flat, x, group=group)
        out.append(flat.view((world,) + tuple(x.shape)))
    return out[0], out[1]


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
