"""Verify attention through the entry point that allocates nothing.

Some callers cannot give the library device memory while they decode -- an
engine that owns every allocation, or a service that forbids cudaMalloc after
start-up because it can stall the device -- so std_dense_verify_attn_noalloc
keeps its split-K partials in a scratch array built into the library.  These
tests call it through the C ABI and compare it with std_dense_verify_attn
(which takes a caller workspace) on two calls in a row.  The file is named so
that pytest collects it last; it builds all of its own inputs, so it also
passes when run alone in a fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

import synth
from sparse_top_kv_std_b200 import binding as B
from tests import harness as H

pytestmark = pytest.mark.gpu


def _case(seed):
    wl = synth.Workload("noalloc", 110, "bf16", 2, 2, 28, 4, 128, (3000, 1777), 64, 256, 8, 0.01, 0.8, 2)
    x = synth.host_inputs(wl, seed=seed)
    kf = x["k_full"].copy()
    vf = x["v_full"].copy()
    for b in range(wl.B):
        p = wl.nvis[b] + wl.T
        kf[:, b, :, p:p + wl.gamma + 1] = x["k_verify"][0][:, b]
        vf[:, b, :, p:p + wl.gamma + 1] = x["v_verify"][0][:, b]
    ctx = torch.tensor([n + wl.T for n in wl.nvis], dtype=torch.int32, device="cuda")
    return wl, H.to_dev(x["q_verify"][0]), H.to_dev(kf), H.to_dev(vf), ctx


@pytest.mark.parametrize("splits", [3, 0])
def test_noalloc_verify_matches_workspace_verify_twice(splits):
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    for call, seed in enumerate((11, 12)):            # two calls in a row, different inputs
        wl, q, kf, vf, ctx = _case(seed)
        d = B.dims(wl.L, wl.B, wl.Hq, wl.Hkv, wl.d, B.STD_BF16, wl.cap_full, wl.cap_sparse)
        shape = (wl.L, wl.B, wl.Hq, wl.gamma + 1, wl.d)
        ws = torch.empty(max(16, B.std_attn_workspace_size(d, wl.gamma + 1, wl.cap_full, splits)),
                         dtype=torch.uint8, device="cuda")
        assert ws.numel() <= B.STD_NOALLOC_SCRATCH_BYTES
        o_ws = torch.full(shape, float("nan"), device="cuda")
        o_na = torch.full(shape, float("nan"), device="cuda")
        B.std_dense_verify_attn(d, q, wl.gamma, kf, vf, ctx, o_ws, splits, ws)
        B.std_dense_verify_attn_noalloc(d, q, wl.gamma, kf, vf, ctx, o_na, splits)
        torch.cuda.synchronize()
        assert B.std_get_device_error() == 0
        assert torch.isfinite(o_na).all(), f"call {call}"
        err = (o_na - o_ws).abs().max().item()
        assert err <= H.attn_tol(wl), (call, err)


def test_noalloc_rejects_more_scratch_than_built_in():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    # 28 layers x 4 KV heads, 63 rows padded to 64, 64 splits: 112*64*64*130*4 B > 16 MiB
    d = B.dims(28, 1, 28, 4, 128, B.STD_BF16, 200000, 5000)
    fake = 1 << 40                                     # never dereferenced: the size check fails first
    rc = B.lib().std_dense_verify_attn_noalloc(ctypes.byref(d), fake, 8, fake, fake, fake, fake, 64, None)
    assert rc == B.STD_ERR_WORKSPACE
    assert "scratch" in B.std_last_error()
