"""Every output and workspace of the library's calls inside canary guard regions
(harness.Canaries: fixed bytes before and after each buffer), checked after the calls,
with the results against the fp64 oracle on small cases of each path: selection (tensor
core, ragged rows), verify (M = 64 and M = 128 layouts, fp32 split-K), the draft with its
row appended in the same launch (SPLIT layout), a whole round, key-range partials and
their merge.  The same module runs against the debug build (libstd_b200_debug.so, every
index and cache row bounds-checked on the device) from test_gpu_debug_build.py; there any
failed device check shows as STD_DEVERR_DEBUG in the error word, which every case reads."""
import os

import numpy as np
import pytest
import torch

import oracle
import synth
from sparse_top_kv_std_b200 import binding as B
from tests import harness as H

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    B.lib()
    B.std_get_device_error(clear=True)


def _wl(name, dtype="bf16", L=2, Bsz=2, Hq=28, Hkv=4, d=128, nvis=(1100, 300), T=37, K=100, gamma=6, wl_id=130):
    return synth.Workload(name, wl_id, dtype, L, Bsz, Hq, Hkv, d, tuple(nvis), T, K, gamma, 0.02, 0.7, 2)


def test_the_library_loaded_is_the_one_asked_for():
    want = "libstd_b200_debug.so" if os.environ.get("STD_B200_DEBUG") == "1" else "libstd_b200.so"
    assert os.path.basename(B.LIB_PATH) == want
    with open("/proc/self/maps") as f:
        assert want in f.read()


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_select_inside_canaries(dtype):
    wl = _wl("c_sel", dtype=dtype, d=128 if dtype == "bf16" else 64, wl_id=131)
    x = synth.host_inputs(wl, seed=1)
    cv = H.Canaries()
    st = torch.bfloat16 if dtype == "bf16" else torch.float32
    d = B.dims(wl.L, wl.B, wl.Hq, wl.Hkv, wl.d, H.dtype_code(wl), wl.cap_full, wl.cap_sparse)
    kf, vf = cv.like(H.to_dev(x["k_full"])), cv.like(H.to_dev(x["v_full"]))
    q = cv.like(H.to_dev(x["q_text"]))
    nvis = cv.like(torch.tensor(wl.nvis, dtype=torch.int32, device="cuda"))
    idx = cv.tensor((wl.L, wl.B, wl.Hkv, wl.K), torch.int32, fill=-1)
    ksp = cv.tensor((wl.L, wl.B, wl.Hkv, wl.cap_sparse, wl.d), st, fill=0)
    vsp = cv.tensor((wl.L, wl.B, wl.Hkv, wl.cap_sparse, wl.d), st, fill=0)
    lsp = cv.tensor((wl.B,), torch.int32, fill=0)
    sc = cv.tensor((wl.L, wl.B, wl.Hkv, wl.nvis_max), torch.float32, fill=0)
    ws = cv.tensor((B.std_select_workspace_size(d, wl.T, wl.nvis_max),), torch.uint8)
    B.std_select_topk(d, q, wl.T, kf, vf, nvis, wl.nvis_max, wl.K, idx, ksp, vsp, lsp, sc, ws)
    cv.check()
    assert B.std_get_device_error() == 0
    idx_o, sc_o, _, _, _ = oracle.select_topk(H.f64(x["q_text"], wl), H.f64(x["k_full"], wl),
                                              H.f64(x["v_full"], wl), x["nvis"], wl.T, wl.K, wl.cap_sparse)
    ig, sg = idx.cpu().numpy(), sc.cpu().numpy()
    for l in range(wl.L):
        for b in range(wl.B):
            for h in range(wl.Hkv):
                nv = wl.nvis[b]
                H.assert_topk_boundary(ig[l, b, h], idx_o[l, b, h], sc_o[l, b, h, :nv], wl.K, H.score_rtol(wl))
    assert lsp.cpu().tolist() == [wl.K + wl.T] * wl.B


@pytest.mark.parametrize("dtype,gamma", [("bf16", 6), ("bf16", 10), ("f32", 3)])
def test_verify_inside_canaries(dtype, gamma):
    # fp32: the tiny workload's head geometry (4 query heads on 2 KV heads, d = 64), for which
    # the method states its 1e-5 bound
    wl = (_wl("c_ver", gamma=gamma, wl_id=132) if dtype == "bf16" else
          _wl("c_ver32", dtype="f32", Hq=4, Hkv=2, d=64, gamma=gamma, wl_id=132))
    x = synth.host_inputs(wl, seed=2)
    kf, vf = x["k_full"].copy(), x["v_full"].copy()
    for b in range(wl.B):
        p = wl.nvis[b] + wl.T
        kf[:, b, :, p:p + gamma + 1] = x["k_verify"][0][:, b]
        vf[:, b, :, p:p + gamma + 1] = x["v_verify"][0][:, b]
    n_ctx = np.array(wl.nvis) + wl.T
    cv = H.Canaries()
    d = B.dims(wl.L, wl.B, wl.Hq, wl.Hkv, wl.d, H.dtype_code(wl), wl.cap_full, wl.cap_sparse)
    for splits in (0, 3):
        ws = cv.tensor((max(16, B.std_attn_workspace_size(d, gamma + 1, wl.cap_full, splits)),), torch.uint8)
        o = cv.tensor((wl.L, wl.B, wl.Hq, gamma + 1, wl.d), torch.float32, fill=float("nan"))
        B.std_dense_verify_attn(d, cv.like(H.to_dev(x["q_verify"][0])), gamma, cv.like(H.to_dev(kf)),
                                cv.like(H.to_dev(vf)), cv.like(torch.from_numpy(n_ctx.astype(np.int32)).cuda()), o,
                                splits, ws)
        cv.check()
        assert B.std_get_device_error() == 0
        want = oracle.dense_verify_attn(H.f64(x["q_verify"][0], wl), H.f64(kf, wl), H.f64(vf, wl), n_ctx)
        assert np.abs(o.cpu().numpy() - want).max() <= H.attn_tol(wl)


def test_draft_append_and_round_inside_canaries():
    wl = _wl("c_round", wl_id=133)
    x = synth.host_inputs(wl, seed=3)
    cv = H.Canaries()
    d = B.dims(wl.L, wl.B, wl.Hq, wl.Hkv, wl.d, B.STD_BF16, wl.cap_full, wl.cap_sparse)
    kf, vf = cv.like(H.to_dev(x["k_full"])), cv.like(H.to_dev(x["v_full"]))
    nvis = cv.like(torch.tensor(wl.nvis, dtype=torch.int32, device="cuda"))
    idx = cv.tensor((wl.L, wl.B, wl.Hkv, wl.K), torch.int32, fill=-1)
    ksp = cv.tensor((wl.L, wl.B, wl.Hkv, wl.cap_sparse, wl.d), torch.bfloat16, fill=0)
    vsp = cv.tensor((wl.L, wl.B, wl.Hkv, wl.cap_sparse, wl.d), torch.bfloat16, fill=0)
    lsp = cv.tensor((wl.B,), torch.int32, fill=0)
    lfull = cv.like(torch.tensor([n + wl.T for n in wl.nvis], dtype=torch.int32, device="cuda"))
    ws_sel = cv.tensor((B.std_select_workspace_size(d, wl.T, wl.nvis_max),), torch.uint8)
    B.std_select_topk(d, cv.like(H.to_dev(x["q_text"])), wl.T, kf, vf, nvis, wl.nvis_max, wl.K, idx, ksp, vsp, lsp,
                      None, ws_sel)
    ws = cv.tensor((B.std_round_workspace_size(d, wl.gamma, 0, 0),), torch.uint8)
    kf64, vf64 = H.f64(x["k_full"], wl), H.f64(x["v_full"], wl)
    torch.cuda.synchronize()
    ksp64, vsp64, lsp_o = oracle.gather_sparse(kf64, vf64, x["nvis"], idx.cpu().numpy(), wl.T, wl.cap_sparse)
    state = {"k_full": kf64, "v_full": vf64, "k_sp": ksp64, "v_sp": vsp64,
             "len_full": np.array(wl.nvis) + wl.T, "len_sp": lsp_o.astype(np.int64)}
    for r in range(wl.rounds):
        io = {k: cv.like(H.to_dev(x[k][r])) for k in ("q_draft", "k_draft", "v_draft", "q_verify", "k_verify",
                                                      "v_verify")}
        io["draft_tokens"] = cv.like(torch.from_numpy(x["draft_tokens"][r]).cuda())
        io["dense_tokens"] = cv.like(torch.from_numpy(x["dense_tokens"][r]).cuda())
        io["o_draft"] = cv.tensor((wl.gamma, wl.L, wl.B, wl.Hq, 1, wl.d), torch.float32, fill=float("nan"))
        io["o_verify"] = cv.tensor((wl.L, wl.B, wl.Hq, wl.gamma + 1, wl.d), torch.float32, fill=float("nan"))
        io["n_plus_1"] = cv.tensor((wl.B,), torch.int32, fill=0)
        io["accepted"] = cv.tensor((wl.B, wl.gamma + 1), torch.int32, fill=0)
        cache = {"k_full": kf, "v_full": vf, "k_sparse": ksp, "v_sparse": vsp, "len_full": lfull, "len_sparse": lsp}
        B.std_decode_round(d, wl.gamma, cache, io, 0, 0, ws)
        cv.check()
        assert B.std_get_device_error() == 0
        want = oracle.decode_round(state, *(H.f64(x[k][r], wl) for k in ("q_draft", "k_draft", "v_draft",
                                                                          "q_verify", "k_verify", "v_verify")),
                                   x["draft_tokens"][r], x["dense_tokens"][r])
        np.testing.assert_array_equal(io["n_plus_1"].cpu().numpy(), want["n_plus_1"])
        assert np.abs(io["o_draft"].cpu().numpy() - want["o_draft"]).max() <= 2e-2
        assert np.abs(io["o_verify"].cpu().numpy() - want["o_verify"]).max() <= 2e-2
    np.testing.assert_array_equal(lsp.cpu().numpy(), state["len_sp"])


def test_partials_and_merge_inside_canaries():
    wl = _wl("c_part", wl_id=134)
    x = synth.host_inputs(wl, seed=4)
    g = wl.gamma
    kf, vf = x["k_full"].copy(), x["v_full"].copy()
    for b in range(wl.B):
        p = wl.nvis[b] + wl.T
        kf[:, b, :, p:p + g + 1] = x["k_verify"][0][:, b]
        vf[:, b, :, p:p + g + 1] = x["v_verify"][0][:, b]
    n_ctx = np.array(wl.nvis) + wl.T
    cv = H.Canaries()
    d = B.dims(wl.L, wl.B, wl.Hq, wl.Hkv, wl.d, B.STD_BF16, wl.cap_full, wl.cap_sparse)
    q, kd, vd = cv.like(H.to_dev(x["q_verify"][0])), cv.like(H.to_dev(kf)), cv.like(H.to_dev(vf))
    ctx = cv.like(torch.from_numpy(n_ctx.astype(np.int32)).cuda())
    shape = (wl.L, wl.B, wl.Hq, g + 1, wl.d)
    cuts = (0, 500, 1100, wl.cap_full)
    o_all = cv.tensor((3,) + shape, torch.float32, fill=float("nan"))
    ml_all = cv.tensor((3,) + shape[:-1] + (2,), torch.float32, fill=float("nan"))
    ws = cv.tensor((B.std_attn_workspace_size(d, g + 1, wl.cap_full, 0),), torch.uint8)
    for i, (r0, r1) in enumerate(zip(cuts[:-1], cuts[1:])):
        B.std_dense_verify_attn_partial(d, q, g, kd, vd, ctx, 0, r0, r1, o_all[i], ml_all[i], 0, ws)
    out = cv.tensor(shape, torch.float32, fill=float("nan"))
    B.std_merge_partials(out.numel() // wl.d, wl.d, 3, o_all, ml_all, out)
    cv.check()
    assert B.std_get_device_error() == 0
    want = oracle.dense_verify_attn(H.f64(x["q_verify"][0], wl), H.f64(kf, wl), H.f64(vf, wl), n_ctx)
    assert np.abs(out.cpu().numpy() - want).max() <= 2e-2
