"""Test helpers: move generator arrays to the GPU and compare with the oracle."""
from __future__ import annotations

import numpy as np
import torch

import synth
from sparse_top_kv_std_b200 import binding as B


def dtype_code(wl) -> int:
    return B.STD_F32 if wl.dtype == "f32" else B.STD_BF16


def to_dev(x: np.ndarray) -> torch.Tensor:
    """Host array -> CUDA tensor with the same bits (uint16 bf16 bits -> torch.bfloat16)."""
    x = np.ascontiguousarray(x)
    if x.dtype == np.uint16:
        return torch.from_numpy(x.view(np.int16)).cuda().view(torch.bfloat16)
    return torch.from_numpy(x).cuda()


def to_host_bits(t: torch.Tensor) -> np.ndarray:
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).cpu().numpy().view(np.uint16)
    return t.cpu().numpy()


def f64(x: np.ndarray, wl) -> np.ndarray:
    return synth.storage_to_f64(x, wl.dtype)


def attn_tol(wl) -> float:
    """Max-abs tolerance on attention outputs: 1e-5 for fp32 operands, 2e-2 for bf16."""
    return 1e-5 if wl.dtype == "f32" else 2e-2


def score_rtol(wl) -> float:
    """Relative tolerance on selection scores (see the design notes for the derivation)."""
    return 1e-4 if wl.dtype == "f32" else 2e-3


def assert_topk_boundary(gpu_idx, orc_idx, orc_scores, K, rtol):
    """GPU and oracle index sets may differ only between entries whose oracle scores
    are within rtol of the K-th largest score (near-ties at the cut)."""
    g = np.asarray(gpu_idx)
    o = np.asarray(orc_idx)
    assert len(g) == K and np.all(np.diff(g) > 0), "indices must be unique and ascending"
    only_g = np.setdiff1d(g, o)
    only_o = np.setdiff1d(o, g)
    assert len(only_g) == len(only_o)
    if len(only_g):
        kth = np.sort(orc_scores)[::-1][K - 1]
        for i in np.concatenate([only_g, only_o]):
            assert abs(orc_scores[i] - kth) <= rtol * kth, (i, orc_scores[i], kth)
    return len(only_g)


def session_for(wl, K=None, gamma=None, splits_draft=0, splits_verify=0):
    from sparse_top_kv_std_b200.session import DecodeSession
    return DecodeSession(wl.L, wl.B, wl.Hq, wl.Hkv, wl.d, dtype_code(wl), wl.cap_full, wl.cap_sparse,
                         wl.T, wl.K if K is None else K, wl.gamma if gamma is None else gamma,
                         wl.nvis_max, splits_draft, splits_verify)


# ----------------------------------------------------------------------------- canaries

GUARD_BYTES = 256
_GUARD_BYTE = 0xA5


class Canaries:
    """Device buffers with GUARD_BYTES of a fixed byte pattern before and after each one:
    a kernel that writes past either end of an output or workspace changes the pattern,
    which check() reports (a cheap stand-in for a memory checker)."""

    def __init__(self):
        self._bufs = []

    def tensor(self, shape, dtype, fill=None):
        import math
        n = math.prod(shape) * torch.empty((), dtype=dtype).element_size()
        raw = torch.full((GUARD_BYTES * 2 + n,), _GUARD_BYTE, dtype=torch.uint8, device="cuda")
        inner = raw[GUARD_BYTES:GUARD_BYTES + n].view(dtype).view(shape)
        if fill is not None:
            inner.fill_(fill)
        self._bufs.append((raw, n))
        return inner

    def like(self, t, fill=None):
        c = self.tensor(tuple(t.shape), t.dtype)
        c.copy_(t)
        if fill is not None:
            c.fill_(fill)
        return c

    def check(self):
        torch.cuda.synchronize()
        for i, (raw, n) in enumerate(self._bufs):
            head = raw[:GUARD_BYTES]
            tail = raw[GUARD_BYTES + n:]
            assert bool((head == _GUARD_BYTE).all()), f"buffer {i}: bytes before it were overwritten"
            assert bool((tail == _GUARD_BYTE).all()), f"buffer {i}: bytes after it were overwritten"
