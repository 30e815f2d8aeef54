"""Prefill selection over a cache split by position, on one GPU: the parts' buffers are
slices of the whole cache, and the two exchanges (row statistics, candidates) are done by
stacking the parts' outputs -- what the all-gathers deliver rank-major.  Checked against
the oracle's selection over the whole cache (indices up to near-ties at the K-th score),
against the library's own single-buffer selection, and the parts' summed sparse caches
against the single-buffer gather at the same indices (bit-exact)."""
import numpy as np
import pytest
import torch

import oracle
import synth
from sparse_top_kv_std_b200 import binding as B
from sparse_top_kv_std_b200 import seqshard
from tests import harness as H

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    B.lib()
    B.std_get_device_error(clear=True)
    yield
    torch.cuda.synchronize()


def _wl(name, dtype="bf16", L=2, Bsz=2, Hq=28, Hkv=4, d=128, nvis=(1500, 1100), T=40, K=64, wl_id=120):
    return synth.Workload(name, wl_id, dtype, L, Bsz, Hq, Hkv, d, tuple(nvis), T, K, 4, 0.02, 0.8, 2)


CASES = {
    "bf16_ragged_3parts": (_wl("bf16_ragged_3parts"), 3, 0),
    "bf16_prefix_2parts": (_wl("bf16_prefix_2parts", L=1, Bsz=1, nvis=(2000,), K=128, wl_id=121), 2, 20),
    "bf16_d64_4parts": (_wl("bf16_d64_4parts", L=1, Bsz=2, Hq=8, Hkv=2, d=64, nvis=(1800, 1700), T=17, K=50,
                            wl_id=122), 4, 7),
    "f32_2parts": (_wl("f32_2parts", dtype="f32", L=1, Bsz=1, Hq=4, Hkv=2, d=32, nvis=(900,), T=9, K=40,
                       wl_id=123), 2, 0),
    "bf16_16k_4parts": (_wl("bf16_16k_4parts", L=1, Bsz=1, nvis=(16384,), T=128, K=1024, wl_id=124), 4, 0),
}


def _run_split(wl, x, world, P):
    """Steps 1-4 of the split selection over `world` parts of the cache; returns (idx, the
    parts' summed sparse K and V, the merged row statistics, the parts' candidates)."""
    dev = torch.device("cuda")
    kf, vf = x["k_full"], x["v_full"]
    cap_full = kf.shape[3]
    prompt = P + int(max(wl.nvis)) + wl.T
    shards = seqshard.partition(prompt, cap_full, world)
    nvis = [int(n) for n in wl.nvis]
    G, T, K = wl.Hq // wl.Hkv, wl.T, wl.K
    probs, rows = wl.L * wl.B * wl.Hkv, G * T
    cap_sp = P + K + T
    q = H.to_dev(x["q_text"])
    parts = []
    for sh in shards:
        kl = H.to_dev(np.ascontiguousarray(kf[:, :, :, sh.pos0:sh.end]))
        vl = H.to_dev(np.ascontiguousarray(vf[:, :, :, sh.pos0:sh.end]))
        dl = B.dims(wl.L, wl.B, wl.Hq, wl.Hkv, wl.d, H.dtype_code(wl), sh.rows, cap_sp)
        p_loc, counts = seqshard.visual_part(sh, P, nvis)
        assert min(counts) >= K
        parts.append((sh, kl, vl, dl, p_loc, counts))
    ms, ls = [], []
    for sh, kl, vl, dl, p_loc, counts in parts:
        m = torch.empty((probs, rows), dtype=torch.float32, device=dev)
        l = torch.empty_like(m)
        B.std_select_rowstats(dl, q, T, kl, torch.tensor(counts, dtype=torch.int32, device=dev), max(counts), p_loc,
                              m, l)
        ms.append(m)
        ls.append(l)
    m_all, l_all = torch.stack(ms), torch.stack(ls)
    mg = torch.empty((probs, rows), dtype=torch.float32, device=dev)
    lg = torch.empty_like(mg)
    B.std_merge_rowstats(probs * rows, world, m_all, l_all, mg, lg)
    cis, css = [], []
    for sh, kl, vl, dl, p_loc, counts in parts:
        ci = torch.empty((probs, K), dtype=torch.int32, device=dev)
        cs = torch.empty((probs, K), dtype=torch.float32, device=dev)
        ws = torch.empty(B.std_select_candidates_workspace_size(dl, max(counts)), dtype=torch.uint8, device=dev)
        B.std_select_candidates(dl, q, T, kl, torch.tensor(counts, dtype=torch.int32, device=dev), max(counts), p_loc,
                                mg, lg, K, ci, cs, None, ws)
        cis.append(ci)
        css.append(cs)
    offs = torch.tensor([[seqshard.visual_offset(sh, P)] * wl.B for sh in shards], dtype=torch.int32, device=dev)
    idx = torch.empty((probs, K), dtype=torch.int32, device=dev)
    d0 = parts[0][3]
    ws2 = torch.empty(B.std_merge_candidates_workspace_size(d0, world, K), dtype=torch.uint8, device=dev)
    B.std_merge_candidates(d0, world, K, torch.stack(cis), torch.stack(css), offs, idx, ws2)
    nvis_dev = torch.tensor(nvis, dtype=torch.int32, device=dev)
    elem = torch.bfloat16 if wl.dtype == "bf16" else torch.float32
    ksum = torch.zeros((wl.L, wl.B, wl.Hkv, cap_sp, wl.d), dtype=torch.float32, device=dev)
    vsum = torch.zeros_like(ksum)
    lsp = torch.empty(wl.B, dtype=torch.int32, device=dev)
    for sh, kl, vl, dl, p_loc, counts in parts:
        ksp = torch.full((wl.L, wl.B, wl.Hkv, cap_sp, wl.d), float("nan"), dtype=elem, device=dev)
        vsp = torch.full_like(ksp, float("nan"))
        B.std_gather_sparse_part(dl, kl, vl, nvis_dev, idx, K, T, P, sh.pos0, sh.rows, ksp, vsp, lsp)
        ksum += ksp.float()      # every row comes from exactly one part, zeros elsewhere
        vsum += vsp.float()
    torch.cuda.synchronize()
    assert B.std_get_device_error() == 0
    assert lsp.cpu().tolist() == [P + K + T] * wl.B
    return idx, ksum.to(elem), vsum.to(elem), (mg, lg), (torch.stack(cis), torch.stack(css))


@pytest.mark.parametrize("name", sorted(CASES))
def test_split_selection_matches_the_whole_cache(name):
    wl, world, P = CASES[name]
    x = synth.host_inputs(wl, seed=3)
    if P:
        rng = np.random.default_rng(29)
        for key in ("k_full", "v_full"):
            pre = rng.standard_normal(x[key].shape[:3] + (P, wl.d)).astype(np.float32)
            x[key] = np.concatenate([synth.storage(pre, wl.dtype), x[key]], axis=3)
    idx, ksp, vsp, (mg, lg), (ci, cs) = _run_split(wl, x, world, P)
    K, T = wl.K, wl.T
    idx_o, sc_o, *_ = oracle.select_topk(H.f64(x["q_text"], wl), H.f64(x["k_full"], wl), H.f64(x["v_full"], wl),
                                         x["nvis"], T, K, P + K + T, n_prefix=P)
    rtol = H.score_rtol(wl)
    idx_g = idx.view(wl.L, wl.B, wl.Hkv, K).cpu().numpy()
    # merged row statistics against the oracle's over all visual keys (exp2 domain)
    G = wl.Hq // wl.Hkv
    mg_h = mg.view(wl.L, wl.B, wl.Hkv, G * T).cpu().numpy().astype(np.float64)
    lg_h = lg.view(wl.L, wl.B, wl.Hkv, G * T).cpu().numpy().astype(np.float64)
    qf, kf = H.f64(x["q_text"], wl), H.f64(x["k_full"], wl)
    for l in range(wl.L):
        for b in range(wl.B):
            nv = wl.nvis[b]
            for h in range(wl.Hkv):
                m0, l0 = oracle.selection_rowstats(qf[l, b, h * G:(h + 1) * G], kf[l, b, h, P:P + nv])
                np.testing.assert_allclose(mg_h[l, b, h], m0 * np.log2(np.e), rtol=rtol, atol=rtol * 10)
                np.testing.assert_allclose(lg_h[l, b, h], l0, rtol=rtol)
                H.assert_topk_boundary(idx_g[l, b, h], idx_o[l, b, h], sc_o[l, b, h, :nv], K, rtol)
    # the parts' summed sparse caches equal the single-buffer gather at the same indices
    dev = torch.device("cuda")
    cap_sp = P + K + T
    d1 = B.dims(wl.L, wl.B, wl.Hq, wl.Hkv, wl.d, H.dtype_code(wl), x["k_full"].shape[3], cap_sp)
    elem = torch.bfloat16 if wl.dtype == "bf16" else torch.float32
    k1 = torch.empty((wl.L, wl.B, wl.Hkv, cap_sp, wl.d), dtype=elem, device=dev)
    v1 = torch.empty_like(k1)
    lsp = torch.empty(wl.B, dtype=torch.int32, device=dev)
    B.std_gather_sparse(d1, H.to_dev(x["k_full"]), H.to_dev(x["v_full"]),
                        torch.tensor([int(n) for n in wl.nvis], dtype=torch.int32, device=dev), idx, K, T, k1, v1,
                        lsp, n_prefix=P)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(H.to_host_bits(ksp), H.to_host_bits(k1))
    np.testing.assert_array_equal(H.to_host_bits(vsp), H.to_host_bits(v1))


def test_split_selection_agrees_with_the_single_buffer_call():
    """Same indices as std_select_topk_ex on the whole cache except near-ties."""
    wl, world, P = CASES["bf16_ragged_3parts"]
    x = synth.host_inputs(wl, seed=4)
    idx, *_ = _run_split(wl, x, world, P)
    from sparse_top_kv_std_b200.session import DecodeSession
    s = DecodeSession(wl.L, wl.B, wl.Hq, wl.Hkv, wl.d, H.dtype_code(wl), x["k_full"].shape[3], wl.K + wl.T, wl.T,
                      wl.K, wl.gamma, wl.nvis_max)
    s.k_full.copy_(H.to_dev(x["k_full"]))
    s.v_full.copy_(H.to_dev(x["v_full"]))
    s.start(x["nvis"])
    s.select(H.to_dev(x["q_text"]))
    torch.cuda.synchronize()
    sc = s.scores.cpu().numpy().astype(np.float64)
    one = s.idx.cpu().numpy()
    split = idx.view(one.shape).cpu().numpy()
    for l in range(wl.L):
        for b in range(wl.B):
            for h in range(wl.Hkv):
                H.assert_topk_boundary(split[l, b, h], one[l, b, h], sc[l, b, h, :wl.nvis[b]], wl.K, 2e-5)


def test_a_part_with_fewer_than_K_keys_is_flagged():
    """K above a part's visual count: the device error word says so; nothing faults."""
    wl, world, P = CASES["bf16_prefix_2parts"]
    dev = torch.device("cuda")
    x = synth.host_inputs(wl, seed=6)
    G, T = wl.Hq // wl.Hkv, wl.T
    probs, rows = wl.L * wl.B * wl.Hkv, G * T
    d = B.dims(wl.L, wl.B, wl.Hq, wl.Hkv, wl.d, H.dtype_code(wl), x["k_full"].shape[3], wl.K + T)
    q, kf = H.to_dev(x["q_text"]), H.to_dev(x["k_full"])
    nv = torch.tensor([100], dtype=torch.int32, device=dev)
    m = torch.empty((probs, rows), dtype=torch.float32, device=dev)
    l = torch.empty_like(m)
    B.std_select_rowstats(d, q, T, kf, nv, 100, 0, m, l)
    ci = torch.empty((probs, wl.K), dtype=torch.int32, device=dev)
    cs = torch.empty((probs, wl.K), dtype=torch.float32, device=dev)
    ws = torch.empty(B.std_select_candidates_workspace_size(d, 100), dtype=torch.uint8, device=dev)
    B.std_select_candidates(d, q, T, kf, nv, 100, 0, m, l, 100, ci, cs, None, ws)   # K = 100 keys: fine
    torch.cuda.synchronize()
    assert B.std_get_device_error() == 0
    nv.fill_(90)                                                                      # now fewer than K
    B.std_select_candidates(d, q, T, kf, nv, 100, 0, m, l, 100, ci, cs, None, ws)
    torch.cuda.synchronize()
    assert B.std_get_device_error(clear=True) & B.STD_DEVERR_K_RANGE
