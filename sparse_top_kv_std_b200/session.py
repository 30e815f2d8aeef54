"""Device-resident state of one Sparse-to-Dense decode, driven through the C ABI.

``DecodeSession`` owns the full and the sparse KV caches, the device lengths,
the selection outputs and the workspaces (allocated once with torch, which is
used here only for device memory and streams), and exposes the method's steps
as calls into ``libstd_b200.so``:

    s = DecodeSession(L=28, B=1, Hq=28, Hkv=4, d=128, dtype=STD_BF16, ...)
    s.k_full[...] = prompt keys; s.v_full[...] = prompt values
    s.start(nvis)            # committed context = nvis + T
    s.select(q_text)         # prefill top-K selection + gather  (std_select_topk_ex)
    s.round(io)              # gamma drafts + verify + accept + commit  (std_decode_round)
"""
from __future__ import annotations

from typing import Dict, Optional

import torch

from . import binding as B_


def storage_dtype(dtype: int) -> torch.dtype:
    return torch.bfloat16 if dtype == B_.STD_BF16 else torch.float32


class DecodeSession:
    def __init__(self, L: int, B: int, Hq: int, Hkv: int, d: int, dtype: int, cap_full: int,
                 cap_sparse: int, T: int, K: int, gamma: int, nvis_max: int,
                 splits_draft: int = 0, splits_verify: int = 0, device="cuda"):
        self.L, self.B, self.Hq, self.Hkv, self.d, self.dtype = L, B, Hq, Hkv, d, dtype
        self.T, self.K, self.gamma, self.nvis_max = T, K, gamma, nvis_max
        self.cap_full, self.cap_sparse = cap_full, cap_sparse
        self.splits_draft, self.splits_verify = splits_draft, splits_verify
        self.dims = B_.dims(L, B, Hq, Hkv, d, dtype, cap_full, cap_sparse)
        dev = torch.device(device)
        st = storage_dtype(dtype)
        self.k_full = torch.zeros((L, B, Hkv, cap_full, d), dtype=st, device=dev)
        self.v_full = torch.zeros_like(self.k_full)
        self.k_sparse = torch.zeros((L, B, Hkv, cap_sparse, d), dtype=st, device=dev)
        self.v_sparse = torch.zeros_like(self.k_sparse)
        self.len_full = torch.zeros(B, dtype=torch.int32, device=dev)
        self.len_sparse = torch.zeros(B, dtype=torch.int32, device=dev)
        self.nvis = torch.zeros(B, dtype=torch.int32, device=dev)
        self.idx = torch.zeros((L, B, Hkv, K), dtype=torch.int32, device=dev)
        self.scores = torch.zeros((L, B, Hkv, nvis_max), dtype=torch.float32, device=dev)
        self.ws_select = torch.empty(max(16, B_.std_select_workspace_size(self.dims, T, nvis_max)),
                                     dtype=torch.uint8, device=dev)
        self.ws_round = torch.empty(max(16, B_.std_round_workspace_size(self.dims, gamma, splits_draft,
                                                                        splits_verify)),
                                    dtype=torch.uint8, device=dev)

    # -- prompt
    def start(self, nvis, stream=None) -> None:
        """Set the visual lengths (device copy) and the committed context nvis + T."""
        nv = torch.as_tensor(nvis, dtype=torch.int32).to(self.nvis.device, non_blocking=True)
        self.nvis.copy_(nv, non_blocking=True)
        self.len_full.copy_(self.nvis + self.T, non_blocking=True)

    def select(self, q_text: torch.Tensor, stream=None, keep_scores: bool = True, flags: int = 0,
               n_prefix: int = 0) -> None:
        """Prefill selection; flags = binding.STD_SELECT_CAUSAL_TEXT for the causal full-row score,
        n_prefix = prompt rows (a system prompt) before the visual block of the full cache."""
        B_.std_select_topk_ex(self.dims, q_text, self.T, self.k_full, self.v_full, self.nvis, self.nvis_max,
                              self.K, n_prefix, flags, self.idx, self.k_sparse, self.v_sparse, self.len_sparse,
                              self.scores if keep_scores else None, self.ws_select, stream)

    # -- decoding
    def round(self, io: Dict[str, torch.Tensor], stream=None) -> None:
        cache = {"k_full": self.k_full, "v_full": self.v_full, "k_sparse": self.k_sparse,
                 "v_sparse": self.v_sparse, "len_full": self.len_full, "len_sparse": self.len_sparse}
        B_.std_decode_round(self.dims, self.gamma, cache, io, self.splits_draft, self.splits_verify,
                            self.ws_round, stream)

    def round_outputs(self, device=None) -> Dict[str, torch.Tensor]:
        """Output buffers of one round: o_draft, o_verify, n_plus_1, accepted."""
        dev = device or self.k_full.device
        L, B, Hq, d, g = self.L, self.B, self.Hq, self.d, self.gamma
        return {"o_draft": torch.zeros((g, L, B, Hq, 1, d), dtype=torch.float32, device=dev),
                "o_verify": torch.zeros((L, B, Hq, g + 1, d), dtype=torch.float32, device=dev),
                "n_plus_1": torch.zeros(B, dtype=torch.int32, device=dev),
                "accepted": torch.zeros((B, g + 1), dtype=torch.int32, device=dev)}

    def device_error(self, clear: bool = True, stream=None) -> int:
        return B_.std_get_device_error(clear, stream)
