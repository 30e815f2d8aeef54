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
    """A call whose partials would not fit the built-in array is refused before launch.
    Every buffer is a real device allocation of the size the dims declare, with valid
    lengths, so the call would be in bounds even if the size check ever let it through."""
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    L, Bn, Hq, Hkv, dh, gamma, cap, splits = 1, 1, 28, 4, 128, 8, 4096, 256
    d = B.dims(L, Bn, Hq, Hkv, dh, B.STD_BF16, cap, 1024)
    # the tensor-core plan: (probs + splits * probs) partial slots of 63 rows x (128 + 2)
    # floats, plus one 8-byte merge counter per problem = 1028 * 63 * 130 * 4 + 4 * 8 bytes
    need = B.std_attn_workspace_size(d, gamma + 1, cap, splits)
    assert need == (4 + splits * 4) * 63 * 130 * 4 + 4 * 8
    assert need > B.STD_NOALLOC_SCRATCH_BYTES
    q = torch.zeros((L, Bn, Hq, gamma + 1, dh), dtype=torch.bfloat16, device="cuda")
    kf = torch.zeros((L, Bn, Hkv, cap, dh), dtype=torch.bfloat16, device="cuda")
    vf = torch.zeros_like(kf)
    ctx = torch.tensor([1000], dtype=torch.int32, device="cuda")
    o = torch.full((L, Bn, Hq, gamma + 1, dh), 7.0, device="cuda")
    n0 = B.std_launch_count()
    rc = B.lib().std_dense_verify_attn_noalloc(ctypes.byref(d), q.data_ptr(), gamma, kf.data_ptr(), vf.data_ptr(),
                                               ctx.data_ptr(), o.data_ptr(), splits, None)
    torch.cuda.synchronize()
    assert rc == B.STD_ERR_WORKSPACE
    assert "scratch" in B.std_last_error()
    assert B.std_launch_count() == n0                  # nothing was launched
    assert bool((o == 7.0).all())
