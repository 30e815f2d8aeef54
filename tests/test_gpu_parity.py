"""CUDA path vs the fp64 oracle, element by element, through the C ABI.

Tolerances (fixed by the method's targets): attention max-abs 1e-5 for fp32
operands and 2e-2 for bf16 operands with fp32 accumulation; top-K indices on
identical fp32 scores and acceptance results bit-exact; cache copies
byte-exact.  Selection scores use the relative tolerance in harness.score_rtol.
"""
import math

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
    yield
    torch.cuda.synchronize()


def small_wl(name, dtype="bf16", L=1, Bsz=1, Hq=28, Hkv=4, d=128, nvis=(1000,), T=40, K=128,
             gamma=4, rounds=3, p=0.7, wl_id=90):
    return synth.Workload(name, wl_id, dtype, L, Bsz, Hq, Hkv, d, tuple(nvis), T, K, gamma, 0.02, p, rounds)


SELECT_CASES = {
    "tiny_f32": synth.workload("tiny_f32"),
    "layer_16k": synth.workload("layer_16k"),
    "ragged_bf16": small_wl("ragged_bf16", L=2, Bsz=3, nvis=(777, 1500, 64), T=33, K=64, wl_id=91),
    "d64_bf16_G1": small_wl("d64_bf16_G1", Hq=4, Hkv=4, d=64, nvis=(300,), T=7, K=300, wl_id=92),
    "f32_G4_K1": small_wl("f32_G4_K1", dtype="f32", Hq=8, Hkv=2, d=32, nvis=(513,), T=5, K=1, wl_id=93),
    # more than 2048 text rows per KV head: the mma.sync fallback of the score passes
    "rows2100_fallback": small_wl("rows2100_fallback", nvis=(700,), T=300, K=64, wl_id=102),
    # ragged rows: G*T = 7*37 = 259 (two 128-row blocks, two 256-row chunks), ragged keys
    "tc_ragged_rows": small_wl("tc_ragged_rows", L=2, Bsz=2, nvis=(1025, 300), T=37, K=100, wl_id=103),
}


# ----------------------------------------------------------------------------- selection

@pytest.mark.parametrize("name", sorted(SELECT_CASES))
def test_select_topk_matches_oracle(name):
    wl = SELECT_CASES[name]
    _check_select(wl, synth.host_inputs(wl, seed=0))


def test_select_row_max_jumps_and_ramps():
    """A per-key logit bias shared by every text row: all queries get +8 on component 0
    and visual key n gets component 0 = t_n, which adds 8 t_n / sqrt(d) (about t_n in the
    exp2 domain) to every row's logit of key n.  t jumps 0 -> 80, ramps 80 -> 110, drops
    to 20, jumps to 118, so each row's running maximum rises within a tile by more than
    the online-softmax rescale thresholds (2^8 and 2^64), while the softmax inside each
    group of keys stays smooth (scores are not saturated)."""
    wl = small_wl("max_jumps", nvis=(1500,), T=40, K=16, wl_id=104)
    x = synth.host_inputs(wl, seed=0)
    nv = wl.nvis[0]
    t = np.zeros(nv)
    t[300:600] = 80.0
    t[600:900] = 80.0 + 0.1 * np.arange(300)
    t[900:1100] = 20.0
    t[1100:] = 118.0
    q = H.f64(x["q_text"], wl)
    q[..., 0] += 8.0
    k = H.f64(x["k_full"], wl)
    k[:, :, :, :nv, 0] = t
    x["q_text"] = synth.storage(q.astype(np.float32), wl.dtype)
    x["k_full"] = synth.storage(k.astype(np.float32), wl.dtype)
    _check_select(wl, x)


CAUSAL_CASES = ["tiny_f32", "ragged_bf16", "d64_bf16_G1", "f32_G4_K1", "rows2100_fallback", "tc_ragged_rows"]


@pytest.mark.parametrize("name", CAUSAL_CASES)
def test_select_causal_text_matches_oracle(name):
    """The causal full-row score (text keys 0..t join row (g, t)'s softmax) on the
    tensor-core, bf16 fallback and fp32 paths."""
    wl = SELECT_CASES[name]
    _check_select(wl, synth.host_inputs(wl, seed=3), flags=B.STD_SELECT_CAUSAL_TEXT)


PREFIX_CASES = [("ragged_bf16", 0), ("ragged_bf16", 1), ("tiny_f32", 0), ("tiny_f32", 1),
                ("rows2100_fallback", 0), ("tc_ragged_rows", 1)]


@pytest.mark.parametrize("name,causal", PREFIX_CASES)
def test_select_with_prompt_prefix(name, causal):
    """A system prompt of 13 rows before the video in the full cache: scores, indices and the
    sparse layout [prefix | selected visual | text], on the tensor-core, bf16 and fp32 paths,
    with both readings of the score."""
    wl = SELECT_CASES[name]
    x = synth.host_inputs(wl, seed=5)
    P = 13
    rng = np.random.default_rng(17)
    for key in ("k_full", "v_full"):
        pre = rng.standard_normal(x[key].shape[:3] + (P, wl.d)).astype(np.float32)
        x[key] = np.concatenate([synth.storage(pre, wl.dtype), x[key]], axis=3)
    _check_select(wl, x, flags=B.STD_SELECT_CAUSAL_TEXT if causal else 0, n_prefix=P)


def _check_select(wl, x, flags=0, n_prefix=0):
    """Selection through the library against the oracle; x["k_full"] / x["v_full"] hold
    [n_prefix rows | visual | text] per (layer, sequence, KV head)."""
    from sparse_top_kv_std_b200.session import DecodeSession
    P = n_prefix
    cap_full, cap_sparse = x["k_full"].shape[3], wl.cap_sparse + P
    s = DecodeSession(wl.L, wl.B, wl.Hq, wl.Hkv, wl.d, H.dtype_code(wl), cap_full, cap_sparse, wl.T, wl.K,
                      wl.gamma, wl.nvis_max)
    s.k_full.copy_(H.to_dev(x["k_full"]))
    s.v_full.copy_(H.to_dev(x["v_full"]))
    s.start(x["nvis"])
    q_text = H.to_dev(x["q_text"])
    s.select(q_text, flags=flags, n_prefix=P)
    torch.cuda.synchronize()
    assert B.std_get_device_error() == 0

    idx_o, sc_o, ksp_o, vsp_o, lsp_o = oracle.select_topk(
        H.f64(x["q_text"], wl), H.f64(x["k_full"], wl), H.f64(x["v_full"], wl), x["nvis"], wl.T, wl.K,
        cap_sparse, causal_text=bool(flags), n_prefix=P)
    sc_g = s.scores.cpu().numpy().astype(np.float64)
    idx_g = s.idx.cpu().numpy()
    rtol = H.score_rtol(wl)
    kf, vf = x["k_full"], x["v_full"]
    ksp_g = H.to_host_bits(s.k_sparse)
    vsp_g = H.to_host_bits(s.v_sparse)
    K, T = wl.K, wl.T
    assert s.len_sparse.cpu().tolist() == [P + K + T] * wl.B
    for l in range(wl.L):
        for b in range(wl.B):
            nv = wl.nvis[b]
            for h in range(wl.Hkv):
                o_s, g_s = sc_o[l, b, h, :nv], sc_g[l, b, h, :nv]
                np.testing.assert_allclose(g_s, o_s, rtol=rtol, atol=rtol * 1e-3 * o_s.max())
                H.assert_topk_boundary(idx_g[l, b, h], idx_o[l, b, h], o_s, K, rtol)
                # gather: byte-exact prefix rows, rows at the GPU's own indices, then the text rows
                ix = idx_g[l, b, h]
                for got, full in ((ksp_g, kf), (vsp_g, vf)):
                    np.testing.assert_array_equal(got[l, b, h, :P], full[l, b, h, :P])
                    np.testing.assert_array_equal(got[l, b, h, P:P + K], full[l, b, h, P + ix])
                    np.testing.assert_array_equal(got[l, b, h, P + K:P + K + T], full[l, b, h, P + nv:P + nv + T])
                # top-K step bit-exact on the GPU's own fp32 scores
                want = oracle.topk_indices(s.scores[l, b, h, :nv].cpu().numpy(), K)
                np.testing.assert_array_equal(ix, want)


TOPK_CASES = [(1, 1, 1), (3, 100, 1), (3, 100, 100), (2, 1000, 37), (5, 4097, 1024), (1, 143360, 4096),
              (4, 16384, 1024), (2, 33, 32)]


@pytest.mark.parametrize("rows,n,K", TOPK_CASES)
@pytest.mark.parametrize("kind", ["normal", "ties", "signed_zero"])
def test_topk_from_scores_bitexact(rows, n, K, kind):
    rng = np.random.default_rng(rows * 7 + n + K)
    if kind == "normal":
        sc = rng.standard_normal((rows, n)).astype(np.float32)
    elif kind == "ties":
        sc = (rng.integers(0, 5, size=(rows, n)) / 4).astype(np.float32)
    else:
        sc = rng.choice(np.array([0.0, -0.0, 1.0, -1.0, 2.5], np.float32), size=(rows, n))
    dev = torch.from_numpy(sc).cuda()
    out = torch.full((rows, K), -7, dtype=torch.int32, device="cuda")
    B.std_topk_from_scores(dev, rows, n, K, out)
    got = out.cpu().numpy()
    for r in range(rows):
        want = oracle.topk_indices(sc[r].astype(np.float64) + 0.0, K)   # +0.0 folds -0.0 into +0.0
        np.testing.assert_array_equal(got[r], want)


# ----------------------------------------------------------------------------- attention

ATTN_CASES = {
    "tiny_f32": synth.workload("tiny_f32"),
    "layer_16k": synth.workload("layer_16k"),
    "ragged_g10": small_wl("ragged_g10", L=2, Bsz=3, nvis=(911, 64, 2500), T=17, K=60, gamma=10, wl_id=94),
    "d64_G2_g0": small_wl("d64_G2_g0", Hq=4, Hkv=2, d=64, nvis=(190,), T=3, K=50, gamma=0, wl_id=95),
    "G16_g7": small_wl("G16_g7", Hq=32, Hkv=2, nvis=(700,), T=9, K=64, gamma=7, wl_id=96),
    "f32_d128_g6": small_wl("f32_d128_g6", dtype="f32", Hq=6, Hkv=3, d=128, nvis=(300,), T=11, K=40,
                            gamma=6, wl_id=97),
    # query rows per problem at the edges of the M = 64 layout: 8 * 8 = 64 (d = 64), 13 * 5 = 65
    "rows64_d64": small_wl("rows64_d64", Hq=16, Hkv=2, d=64, nvis=(1300,), T=5, K=200, gamma=7, wl_id=105),
    "rows65": small_wl("rows65", Hq=13, Hkv=1, nvis=(800,), T=6, K=100, gamma=4, wl_id=106),
}


def _verify_inputs(wl, x):
    """Full cache with the verify rows of round 0 appended at n_ctx = nvis + T."""
    kf = x["k_full"].copy()
    vf = x["v_full"].copy()
    for b in range(wl.B):
        p = wl.nvis[b] + wl.T
        kf[:, b, :, p:p + wl.gamma + 1] = x["k_verify"][0][:, b]
        vf[:, b, :, p:p + wl.gamma + 1] = x["v_verify"][0][:, b]
    return kf, vf


@pytest.mark.parametrize("name", sorted(ATTN_CASES))
@pytest.mark.parametrize("splits", [1, 3, 0])
def test_dense_verify_matches_oracle(name, splits):
    wl = ATTN_CASES[name]
    x = synth.host_inputs(wl, seed=1)
    kf, vf = _verify_inputs(wl, x)
    n_ctx = np.array(wl.nvis) + wl.T
    d = B.dims(wl.L, wl.B, wl.Hq, wl.Hkv, wl.d, H.dtype_code(wl), wl.cap_full, wl.cap_sparse)
    ws_bytes = B.std_attn_workspace_size(d, wl.gamma + 1, wl.cap_full, splits)
    ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device="cuda")
    o = torch.full((wl.L, wl.B, wl.Hq, wl.gamma + 1, wl.d), float("nan"), device="cuda")
    B.std_dense_verify_attn(d, H.to_dev(x["q_verify"][0]), wl.gamma, H.to_dev(kf), H.to_dev(vf),
                            torch.from_numpy(n_ctx.astype(np.int32)).cuda(), o, splits, ws)
    torch.cuda.synchronize()
    assert B.std_get_device_error() == 0
    want = oracle.dense_verify_attn(H.f64(x["q_verify"][0], wl), H.f64(kf, wl), H.f64(vf, wl), n_ctx)
    err = np.abs(o.cpu().numpy() - want).max()
    assert err <= H.attn_tol(wl), err


@pytest.mark.parametrize("name", sorted(ATTN_CASES))
@pytest.mark.parametrize("splits", [1, 5, 0])
def test_sparse_decode_matches_oracle(name, splits):
    wl = ATTN_CASES[name]
    x = synth.host_inputs(wl, seed=2)
    # a sparse cache of K + T committed rows plus `extra` appended draft rows
    rng = np.random.default_rng(5)
    st = np.float32 if wl.dtype == "f32" else np.uint16
    ksp = np.zeros((wl.L, wl.B, wl.Hkv, wl.cap_sparse, wl.d), st)
    vsp = np.zeros_like(ksp)
    base = wl.K + wl.T
    for b in range(wl.B):
        take = np.sort(rng.choice(wl.nvis[b], size=wl.K, replace=False))
        nv = wl.nvis[b]
        rows = np.concatenate([take, np.arange(nv, nv + wl.T)])
        ksp[:, b, :, :base] = x["k_full"][:, b][:, :, rows]
        vsp[:, b, :, :base] = x["v_full"][:, b][:, :, rows]
    extra = 3
    ksp[:, :, :, base:base + extra] = x["k_full"][:, :, :, 1:1 + extra]
    vsp[:, :, :, base:base + extra] = x["v_full"][:, :, :, 1:1 + extra]
    lens = np.full(wl.B, base, np.int32)
    d = B.dims(wl.L, wl.B, wl.Hq, wl.Hkv, wl.d, H.dtype_code(wl), wl.cap_full, wl.cap_sparse)
    ws_bytes = B.std_attn_workspace_size(d, 1, wl.cap_sparse, splits)
    ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device="cuda")
    q = x["q_draft"][0, 0] if wl.gamma > 0 else x["q_verify"][0][:, :, :, :1]
    q = np.ascontiguousarray(q)
    o = torch.full((wl.L, wl.B, wl.Hq, 1, wl.d), float("nan"), device="cuda")
    B.std_sparse_decode_attn(d, H.to_dev(q), H.to_dev(ksp), H.to_dev(vsp), torch.from_numpy(lens).cuda(), extra,
                             o, splits, ws)
    torch.cuda.synchronize()
    assert B.std_get_device_error() == 0
    want = oracle.sparse_decode_attn(H.f64(q, wl), H.f64(ksp, wl), H.f64(vsp, wl), lens + extra)
    err = np.abs(o.cpu().numpy() - want).max()
    assert err <= H.attn_tol(wl), err


def test_full_k_sparse_equals_dense_on_gpu():
    """K = Nv: the sparse cache is the prompt in order, so the draft equals a gamma=0 verify."""
    wl = small_wl("fullk", Hq=8, Hkv=2, nvis=(400,), T=16, K=400, gamma=0, wl_id=98)
    x = synth.host_inputs(wl, seed=3)
    s = H.session_for(wl)
    s.k_full.copy_(H.to_dev(x["k_full"]))
    s.v_full.copy_(H.to_dev(x["v_full"]))
    s.start(x["nvis"])
    s.select(H.to_dev(x["q_text"]))
    q = H.to_dev(np.ascontiguousarray(x["q_verify"][0][:, :, :, :1]))
    o_sp = torch.zeros((1, 1, 8, 1, 128), device="cuda")
    o_dn = torch.zeros_like(o_sp)
    ws = torch.empty(1 << 20, dtype=torch.uint8, device="cuda")
    B.std_sparse_decode_attn(s.dims, q, s.k_sparse, s.v_sparse, s.len_sparse, 0, o_sp, 1, ws)
    ctx = torch.tensor([400 + 16 - 1], dtype=torch.int32, device="cuda")
    B.std_dense_verify_attn(s.dims, q, 0, s.k_full, s.v_full, ctx, o_dn, 1, ws)
    torch.cuda.synchronize()
    assert s.idx.cpu().numpy()[0, 0, 0].tolist() == list(range(400))
    assert torch.equal(o_sp, o_dn)


# ----------------------------------------------------------------------------- acceptance

@pytest.mark.parametrize("gamma", [0, 1, 4, 8, 10, 31])
@pytest.mark.parametrize("p", [0.5, 0.95])
def test_accept_bitexact(gamma, p):
    rng = np.random.default_rng(gamma * 100 + int(p * 10))
    Bn = 67
    dense = rng.integers(0, 32000, size=(Bn, gamma + 1)).astype(np.int32)
    match = rng.random((Bn, gamma)) < p
    draft = np.where(match, dense[:, :gamma], (dense[:, :gamma] + 1) % 32000).astype(np.int32)
    n1 = torch.zeros(Bn, dtype=torch.int32, device="cuda")
    acc = torch.zeros((Bn, gamma + 1), dtype=torch.int32, device="cuda")
    dr = torch.from_numpy(draft).cuda() if gamma else torch.zeros(1, dtype=torch.int32, device="cuda")
    B.std_accept_prefix(Bn, gamma, dr, torch.from_numpy(dense).cuda(), n1, acc)
    w_n1, w_acc = oracle.accept_prefix(draft.reshape(Bn, gamma), dense)
    np.testing.assert_array_equal(n1.cpu().numpy(), w_n1)
    np.testing.assert_array_equal(acc.cpu().numpy(), w_acc)


# ----------------------------------------------------------------------------- bookkeeping

def test_append_and_commit_byte_exact():
    wl = small_wl("bk", L=2, Bsz=3, Hq=8, Hkv=2, nvis=(50, 60, 70), T=5, K=20, gamma=3, wl_id=99)
    rng = np.random.default_rng(11)
    kf = rng.integers(0, 65535, size=(2, 3, 2, wl.cap_full, 128)).astype(np.uint16)
    vf = rng.integers(0, 65535, size=kf.shape).astype(np.uint16)
    ks = rng.integers(0, 65535, size=(2, 3, 2, wl.cap_sparse, 128)).astype(np.uint16)
    vs = rng.integers(0, 65535, size=ks.shape).astype(np.uint16)
    lf = np.array([55, 65, 75], np.int32)
    ls = np.array([25, 26, 27], np.int32)
    newk = rng.integers(0, 65535, size=(2, 3, 2, 4, 128)).astype(np.uint16)
    newv = rng.integers(0, 65535, size=newk.shape).astype(np.uint16)
    n1 = np.array([1, 4, 2], np.int32)
    d = B.dims(2, 3, 8, 2, 128, B.STD_BF16, wl.cap_full, wl.cap_sparse)
    t = {k: H.to_dev(v) for k, v in dict(kf=kf, vf=vf, ks=ks, vs=vs, nk=newk, nv=newv).items()}
    tlf, tls, tn1 = (torch.from_numpy(a).cuda() for a in (lf, ls, n1))
    B.std_kv_append(d, t["kf"], t["vf"], wl.cap_full, tlf, 0, t["nk"], t["nv"], 4)
    B.std_kv_append(d, t["ks"], t["vs"], wl.cap_sparse, tls, 2, t["nk"][:, :, :, :1].contiguous(),
                    t["nv"][:, :, :, :1].contiguous(), 1)
    B.std_kv_commit(d, t["kf"], t["vf"], t["ks"], t["vs"], tlf, tls, tn1, 4)
    torch.cuda.synchronize()
    assert B.std_get_device_error() == 0
    # oracle on the same bits, as exact integers in float64
    o = {k: v.astype(np.float64) for k, v in dict(kf=kf, vf=vf, ks=ks, vs=vs).items()}
    olf, ols = lf.copy(), ls.copy()
    oracle.kv_append(o["kf"], olf, 0, newk.astype(np.float64))
    oracle.kv_append(o["vf"], olf, 0, newv.astype(np.float64))
    oracle.kv_append(o["ks"], ols, 2, newk[:, :, :, :1].astype(np.float64))
    oracle.kv_append(o["vs"], ols, 2, newv[:, :, :, :1].astype(np.float64))
    oracle.kv_commit(o["kf"], o["vf"], o["ks"], o["vs"], olf, ols, n1)
    for k in ("kf", "vf", "ks", "vs"):
        np.testing.assert_array_equal(H.to_host_bits(t[k]).astype(np.float64), o[k])
    np.testing.assert_array_equal(tlf.cpu().numpy(), olf)
    np.testing.assert_array_equal(tls.cpu().numpy(), ols)


def test_device_error_flags_capacity_and_k_range():
    wl = small_wl("err", Hq=4, Hkv=2, d=64, nvis=(100, 30), Bsz=2, T=4, K=40, gamma=2, wl_id=100)
    d = B.dims(1, 2, 4, 2, 64, B.STD_BF16, wl.cap_full, wl.cap_sparse)
    kc = torch.zeros((1, 2, 2, wl.cap_full, 64), dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    nk = torch.ones((1, 2, 2, 2, 64), dtype=torch.bfloat16, device="cuda")
    lens = torch.tensor([wl.cap_full - 1, 0], dtype=torch.int32, device="cuda")
    B.std_get_device_error(clear=True)
    B.std_kv_append(d, kc, vc, wl.cap_full, lens, 0, nk, nk, 2)
    flags = B.std_get_device_error(clear=True)
    assert flags & B.STD_DEVERR_CAPACITY
    assert float(kc[0, 0].abs().sum()) == 0.0          # the overflowing sequence wrote nothing
    assert float(kc[0, 1, :, :2].float().sum()) == 2 * 2 * 64
    # K = 40 > nvis[1] = 30: that sequence is flagged, the other is still selected
    x = synth.host_inputs(wl, seed=0)
    s = H.session_for(wl)
    s.k_full.copy_(H.to_dev(x["k_full"]))
    s.v_full.copy_(H.to_dev(x["v_full"]))
    s.start(x["nvis"])
    s.select(H.to_dev(x["q_text"]))
    flags = B.std_get_device_error(clear=True)
    assert flags & B.STD_DEVERR_K_RANGE
    idx_o = oracle.select_topk(H.f64(x["q_text"][:, :1], wl), H.f64(x["k_full"][:, :1], wl),
                               H.f64(x["v_full"][:, :1], wl), x["nvis"][:1], wl.T, wl.K, wl.cap_sparse)[0]
    np.testing.assert_array_equal(s.idx[:, :1].cpu().numpy(), idx_o)


# ----------------------------------------------------------------------------- whole rounds

ROUND_CASES = {
    "tiny_f32": (synth.workload("tiny_f32"), 4),
    "layer_16k": (synth.workload("layer_16k"), 3),
    "ragged_b3": (small_wl("ragged_b3", L=2, Bsz=3, Hq=14, Hkv=2, nvis=(900, 333, 1200), T=20, K=96,
                           gamma=5, rounds=4, p=0.6, wl_id=101), 4),
}


@pytest.mark.parametrize("name", sorted(ROUND_CASES))
def test_decode_rounds_match_oracle(name):
    wl, R = ROUND_CASES[name]
    x = synth.host_inputs(wl, seed=4)
    s = H.session_for(wl)
    s.k_full.copy_(H.to_dev(x["k_full"]))
    s.v_full.copy_(H.to_dev(x["v_full"]))
    s.start(x["nvis"])
    s.select(H.to_dev(x["q_text"]))
    kf64, vf64 = H.f64(x["k_full"], wl), H.f64(x["v_full"], wl)
    idx_o, sc_o, _, _, _ = oracle.select_topk(H.f64(x["q_text"], wl), kf64, vf64, x["nvis"], wl.T, wl.K,
                                              wl.cap_sparse)
    # the GPU's index sets may differ from the oracle's only at near-ties of the cut; once that
    # is checked, the oracle's sparse cache is gathered from the GPU's own indices so every
    # head's draft attention is compared
    idx_g = s.idx.cpu().numpy()
    for l in range(wl.L):
        for b in range(wl.B):
            for h in range(wl.Hkv):
                nv = wl.nvis[b]
                H.assert_topk_boundary(idx_g[l, b, h], idx_o[l, b, h], sc_o[l, b, h, :nv], wl.K, H.score_rtol(wl))
    ksp, vsp, lsp = oracle.gather_sparse(kf64, vf64, x["nvis"], idx_g, wl.T, wl.cap_sparse)
    state = {"k_full": kf64, "v_full": vf64, "k_sp": ksp, "v_sp": vsp,
             "len_full": np.array(wl.nvis) + wl.T, "len_sp": lsp.astype(np.int64)}
    tol = H.attn_tol(wl)
    for r in range(R):
        io = {k: H.to_dev(x[k][r]) for k in ("q_draft", "k_draft", "v_draft", "q_verify", "k_verify",
                                             "v_verify")}
        io["draft_tokens"] = torch.from_numpy(x["draft_tokens"][r]).cuda()
        io["dense_tokens"] = torch.from_numpy(x["dense_tokens"][r]).cuda()
        io.update(s.round_outputs())
        s.round(io)
        want = oracle.decode_round(state, *(H.f64(x[k][r], wl) for k in ("q_draft", "k_draft", "v_draft",
                                                                          "q_verify", "k_verify", "v_verify")),
                                   x["draft_tokens"][r], x["dense_tokens"][r])
        torch.cuda.synchronize()
        assert B.std_get_device_error() == 0
        np.testing.assert_array_equal(io["n_plus_1"].cpu().numpy(), want["n_plus_1"])
        np.testing.assert_array_equal(io["accepted"].cpu().numpy(), want["accepted"])
        assert np.abs(io["o_draft"].cpu().numpy() - want["o_draft"]).max(initial=0.0) <= tol
        assert np.abs(io["o_verify"].cpu().numpy() - want["o_verify"]).max() <= tol
        np.testing.assert_array_equal(s.len_full.cpu().numpy(), state["len_full"])
        np.testing.assert_array_equal(s.len_sparse.cpu().numpy(), state["len_sp"])
    # caches after all rounds: byte-exact
    np.testing.assert_array_equal(H.f64(H.to_host_bits(s.k_sparse), wl), state["k_sp"])
    np.testing.assert_array_equal(H.f64(H.to_host_bits(s.v_sparse), wl), state["v_sp"])
    np.testing.assert_array_equal(H.f64(H.to_host_bits(s.v_full), wl), state["v_full"])


# ----------------------------------------------------------------------------- FMA-pipe exponential

def test_exp2_polynomial_error_bound():
    """The polynomial 2^x used beside the special-function unit: relative error
    against float64 exp2 within 4e-6 on x in [-125, 0] (a degree-4 fit whose
    exact-arithmetic error is 2.6e-6; the selection scores it feeds are compared
    at a relative 2e-3), and the SFU's own ex2.approx within 4e-7."""
    x = np.concatenate([-np.linspace(0.0, 125.0, 1 << 20), -np.random.default_rng(0).random(1 << 16) * 30,
                        np.array([0.0, -0.5, -1e-8, -0.49999997, -124.99])]).astype(np.float32)
    xd = torch.from_numpy(x).cuda()
    yf = torch.empty_like(xd)
    ys = torch.empty_like(xd)
    B.std_probe_exp2(xd, yf, ys)
    torch.cuda.synchronize()
    ref = np.exp2(x.astype(np.float64))
    rel_f = np.abs(yf.cpu().numpy() - ref) / ref
    rel_s = np.abs(ys.cpu().numpy() - ref) / ref
    assert rel_f.max() < 4e-6, rel_f.max()
    assert rel_f.mean() < 2e-6
    assert rel_s.max() < 4e-7     # the SFU reference the polynomial stands beside


# ----------------------------------------------------------------------------- streaming baseline

@pytest.mark.parametrize("name,n_sink,P", [("ragged_bf16", 4, 0), ("tiny_f32", 0, 0), ("d64_bf16_G1", 300, 0),
                                            ("ragged_bf16", 4, 9)])
def test_streaming_indices_and_gather(name, n_sink, P):
    wl = SELECT_CASES[name]
    x = synth.host_inputs(wl, seed=4)
    if P:  # a prompt prefix before the visual block
        for key in ("k_full", "v_full"):
            pre = np.random.default_rng(3).standard_normal(x[key].shape[:3] + (P, wl.d)).astype(np.float32)
            x[key] = np.concatenate([synth.storage(pre, wl.dtype), x[key]], axis=3)
    cap_sparse = wl.cap_sparse + P
    d = B.dims(wl.L, wl.B, wl.Hq, wl.Hkv, wl.d, H.dtype_code(wl), x["k_full"].shape[3], cap_sparse)
    nvis = torch.tensor(wl.nvis, dtype=torch.int32, device="cuda")
    idx = torch.full((wl.L, wl.B, wl.Hkv, wl.K), -1, dtype=torch.int32, device="cuda")
    st = torch.float32 if wl.dtype == "f32" else torch.int16
    ksp = torch.zeros((wl.L, wl.B, wl.Hkv, cap_sparse, wl.d), dtype=st, device="cuda")
    vsp = torch.zeros_like(ksp)
    lsp = torch.zeros(wl.B, dtype=torch.int32, device="cuda")
    B.std_streaming_indices(d, nvis, wl.K, n_sink, idx)
    B.std_gather_sparse(d, H.to_dev(x["k_full"]), H.to_dev(x["v_full"]), nvis, idx, wl.K, wl.T, ksp, vsp, lsp,
                        n_prefix=P)
    torch.cuda.synchronize()
    assert B.std_get_device_error() == 0
    idx_h = idx.cpu().numpy()
    for b in range(wl.B):
        want = oracle.streaming_indices(wl.nvis[b], wl.K, n_sink)
        for l in range(wl.L):
            for h in range(wl.Hkv):
                np.testing.assert_array_equal(idx_h[l, b, h], want)
    kw, vw, lw = oracle.gather_sparse(x["k_full"], x["v_full"], np.array(wl.nvis), idx_h, wl.T, cap_sparse, P)
    n = P + wl.K + wl.T
    got_k = ksp.cpu().numpy().view(x["k_full"].dtype)[..., :n, :]
    got_v = vsp.cpu().numpy().view(x["v_full"].dtype)[..., :n, :]
    np.testing.assert_array_equal(got_k, kw[..., :n, :].astype(x["k_full"].dtype))
    np.testing.assert_array_equal(got_v, vw[..., :n, :].astype(x["v_full"].dtype))
    assert lsp.cpu().tolist() == lw.tolist()


def test_streaming_window_larger_than_the_sequence_is_flagged():
    wl = SELECT_CASES["ragged_bf16"]  # nvis (777, 1500, 64)
    d = B.dims(wl.L, wl.B, wl.Hq, wl.Hkv, wl.d, H.dtype_code(wl), wl.cap_full, wl.cap_sparse)
    nvis = torch.tensor(wl.nvis, dtype=torch.int32, device="cuda")
    idx = torch.full((wl.L, wl.B, wl.Hkv, 65), -7, dtype=torch.int32, device="cuda")
    B.std_streaming_indices(d, nvis, 65, 4, idx)
    torch.cuda.synchronize()
    assert B.std_get_device_error() == B.STD_DEVERR_K_RANGE
    h = idx.cpu().numpy()
    assert (h[:, 2] == -7).all()                              # the 64-token sequence was skipped
    assert h[0, 0, 0].tolist() == list(range(4)) + list(range(777 - 61, 777))


def test_topk_keeps_more_attention_mass_than_the_streaming_window():
    """Selection quality on the generator's long-video layer: the share of each draft
    query's dense softmax mass (over the prompt) that falls on the sparse cache's rows.
    The method's top-K (chosen from the text queries) keeps more of it than the sink +
    recent window of the same size.  The mass is computed in torch from the library's
    own index sets (test-side arithmetic only)."""
    wl = synth.workload("layer_16k")
    x = synth.host_inputs(wl, seed=0)
    s = H.session_for(wl)
    s.k_full.copy_(H.to_dev(x["k_full"]))
    s.v_full.copy_(H.to_dev(x["v_full"]))
    s.start(x["nvis"])
    s.select(H.to_dev(x["q_text"]))
    idx_top = s.idx.clone()
    idx_str = torch.empty_like(s.idx)
    B.std_streaming_indices(s.dims, s.nvis, wl.K, 4, idx_str)
    torch.cuda.synchronize()
    assert B.std_get_device_error() == 0
    nv, G, N = wl.nvis[0], wl.G, wl.nvis[0] + wl.T
    keys = s.k_full[:, 0, :, :N].float()                                   # [L, Hkv, N, d]
    q = H.to_dev(np.ascontiguousarray(x["q_draft"][0, 0])).float()[:, 0, :, 0]   # [L, Hq, d]
    q = q.reshape(wl.L, wl.Hkv, G, wl.d)
    p = torch.softmax(torch.einsum("lhgd,lhnd->lhgn", q, keys) / math.sqrt(wl.d), dim=-1)
    text = p[..., nv:].sum(-1)

    def kept(idx):
        ix = idx[:, 0].long()[:, :, None, :].expand(-1, -1, G, -1)             # [L, Hkv, G, K]
        return float((torch.gather(p, 3, ix).sum(-1) + text).mean())
    m_top, m_str = kept(idx_top), kept(idx_str)
    print(f"\nmean dense attention mass kept by K = {wl.K} of {nv} visual rows + {wl.T} text rows: "
          f"top-K {m_top:.3f}, sink + window {m_str:.3f}")
    assert m_top > 1.5 * m_str, (m_top, m_str)


# ----------------------------------------------------------------------------- append + attention

@pytest.mark.parametrize("name", ["layer_16k", "ragged_g10", "d64_G2_g0", "rows64_d64", "f32_d128_g6"])
def test_append_then_attend_in_one_launch(name):
    """std_*_attn_append equal std_kv_append followed by the attention call: the caches
    byte for byte and the outputs exactly (the same kernel reads the same rows)."""
    wl = ATTN_CASES[name]
    x = synth.host_inputs(wl, seed=6)
    d = B.dims(wl.L, wl.B, wl.Hq, wl.Hkv, wl.d, H.dtype_code(wl), wl.cap_full, wl.cap_full)
    n_ctx = torch.tensor(np.array(wl.nvis) + wl.T, dtype=torch.int32, device="cuda")
    g = wl.gamma
    ws = torch.empty(max(16, B.std_attn_workspace_size(d, g + 1, wl.cap_full, 0)), dtype=torch.uint8, device="cuda")
    kv_new = H.to_dev(x["k_verify"][0]), H.to_dev(x["v_verify"][0])
    q_ver = H.to_dev(x["q_verify"][0])
    outs = []
    for fused in (False, True):
        kf, vf = H.to_dev(x["k_full"]), H.to_dev(x["v_full"])
        o_v = torch.full((wl.L, wl.B, wl.Hq, g + 1, wl.d), float("nan"), device="cuda")
        o_d = torch.full((wl.L, wl.B, wl.Hq, 1, wl.d), float("nan"), device="cuda")
        k1, v1 = kv_new[0][:, :, :, :1].contiguous(), kv_new[1][:, :, :, :1].contiguous()
        q1 = q_ver[:, :, :, :1].contiguous()
        if fused:
            B.std_dense_verify_attn_append(d, q_ver, g, kf, vf, n_ctx, kv_new[0], kv_new[1], o_v, 0, ws)
            # a draft-style step on the cache just extended: one more row at n_ctx + g + 1
            B.std_sparse_decode_attn_append(d, q1, kf, vf, n_ctx, g + 2, k1, v1, o_d, 0, ws)
        else:
            B.std_kv_append(d, kf, vf, wl.cap_full, n_ctx, 0, kv_new[0], kv_new[1], g + 1)
            B.std_dense_verify_attn(d, q_ver, g, kf, vf, n_ctx, o_v, 0, ws)
            B.std_kv_append(d, kf, vf, wl.cap_full, n_ctx, g + 1, k1, v1, 1)
            B.std_sparse_decode_attn(d, q1, kf, vf, n_ctx, g + 2, o_d, 0, ws)
        torch.cuda.synchronize()
        assert B.std_get_device_error() == 0
        outs.append((H.to_host_bits(kf), H.to_host_bits(vf), o_v.cpu().numpy(), o_d.cpu().numpy()))
    for a, b in zip(outs[0], outs[1]):
        np.testing.assert_array_equal(a, b)
    # and against the oracle for the verify rows
    want = oracle.dense_verify_attn(H.f64(x["q_verify"][0], wl), H.f64(outs[1][0], wl), H.f64(outs[1][1], wl),
                                    np.array(wl.nvis) + wl.T)
    assert np.abs(outs[1][2] - want).max() <= H.attn_tol(wl)


def test_launch_count_matches_the_calls():
    """std_launch_count counts the library's kernel launches: 4 for a tensor-core selection
    (two score passes, top-K, gather), gamma + 5 for a round (gamma fused draft attentions,
    append + verify, acceptance, two commit kernels)."""
    wl = synth.workload("layer_16k").replace(rounds=1)
    x = synth.host_inputs(wl, seed=0)
    s = H.session_for(wl)
    s.k_full.copy_(H.to_dev(x["k_full"]))
    s.v_full.copy_(H.to_dev(x["v_full"]))
    s.start(x["nvis"])
    torch.cuda.synchronize()
    n0 = B.std_launch_count()
    s.select(H.to_dev(x["q_text"]))
    n1 = B.std_launch_count()
    io = {k: H.to_dev(x[k][0]) for k in ("q_draft", "k_draft", "v_draft", "q_verify", "k_verify", "v_verify")}
    io["draft_tokens"] = torch.from_numpy(x["draft_tokens"][0]).cuda()
    io["dense_tokens"] = torch.from_numpy(x["dense_tokens"][0]).cuda()
    io.update(s.round_outputs())
    s.round(io)
    n2 = B.std_launch_count()
    torch.cuda.synchronize()
    assert B.std_get_device_error() == 0
    assert (n1 - n0, n2 - n1) == (4, wl.gamma + 5)



@pytest.mark.parametrize("early", [False, True])
@pytest.mark.parametrize("splits", [1, 2, 7, 16, 40, 0])
def test_sparse_decode_ragged_lengths_problem_aligned_parts(splits, early):
    """The keys-on-lanes draft kernel over sequences of different lengths -- one shorter
    than a 128-key tile, one with fewer tiles than a 7- or 40-part split, one over nine
    tiles -- with the step's row appended in the same launch: explicit splits (equal parts
    of every problem; 2 to 16 of them merge inside a thread-block cluster, 16 being the
    largest, non-portable size), the automatic plan, and the early start behind another
    attention call on the same stream and workspace.  Against the oracle's sparse draft attention
    over rows j < len[b] + 1 after the append [S-M2, S-M3]; the appended rows bit-exact."""
    L, Bn, Hq, Hkv, d, cap = 2, 3, 28, 4, 128, 1200
    lens = np.array([90, 300, 1100], np.int32)
    rng = np.random.default_rng(11)

    def draw(shape, scale=1.0):
        return synth.storage(rng.standard_normal(shape).astype(np.float32) * scale, "bf16")

    k, v = draw((L, Bn, Hkv, cap, d), 0.5), draw((L, Bn, Hkv, cap, d))
    q = draw((L, Bn, Hq, 1, d))
    kn, vn = draw((L, Bn, Hkv, 1, d), 0.5), draw((L, Bn, Hkv, 1, d))
    dims = B.dims(L, Bn, Hq, Hkv, d, B.STD_BF16, cap, cap)
    ws = torch.empty(max(B.std_attn_workspace_size(dims, 1, cap, splits), 16), dtype=torch.uint8, device="cuda")
    kd, vd, qd = H.to_dev(k), H.to_dev(v), H.to_dev(q)
    lens_d = torch.from_numpy(lens).cuda()
    o = torch.full((L, Bn, Hq, 1, d), float("nan"), device="cuda")
    flags = 0
    if early:
        # the predecessor writes only its own output and the workspace: the rows below the
        # appended one, the lengths and q may be read before it finishes
        o0 = torch.empty_like(o)
        B.std_sparse_decode_attn(dims, qd, kd, vd, lens_d, 0, o0, splits, ws)
        flags = B.STD_ATTN_EARLY_KV | B.STD_ATTN_EARLY_Q
    B.std_sparse_decode_attn_append_ex(dims, qd, kd, vd, lens_d, 1, H.to_dev(kn), H.to_dev(vn), o, splits, flags, ws)
    torch.cuda.synchronize()
    assert B.std_get_device_error() == 0
    k_ref, v_ref = k.copy(), v.copy()
    for b in range(Bn):
        k_ref[:, b, :, lens[b]] = kn[:, b, :, 0]
        v_ref[:, b, :, lens[b]] = vn[:, b, :, 0]
    assert np.array_equal(H.to_host_bits(kd), k_ref) and np.array_equal(H.to_host_bits(vd), v_ref)
    wl = type("W", (), {"dtype": "bf16"})()
    want = oracle.sparse_decode_attn(H.f64(q, wl), H.f64(k_ref, wl), H.f64(v_ref, wl), lens + 1)
    err = np.abs(o.cpu().numpy() - want).max()
    assert err <= H.attn_tol(wl), err
    if early:
        want0 = oracle.sparse_decode_attn(H.f64(q, wl), H.f64(k, wl), H.f64(v, wl), lens)
        assert np.abs(o0.cpu().numpy() - want0).max() <= H.attn_tol(wl)


def test_automatic_draft_grids():
    """The planner's automatic grid for the draft kernel on this device: a single layer's
    draft (4 problems of up to 4640 keys) is cut into equal parts of at least three tiles
    at cap, at most 16 and at most half as many CTAs as SMs; the 28-layer draft takes one
    CTA per SM, or one CTA per problem when it starts early; an early plan never needs
    more workspace than the plain one."""
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    cap = 4640
    d1 = B.dims(1, 1, 28, 4, 128, B.STD_BF16, 200000, cap)
    parts = max(1, min((cap + 127) // 128 // 3, 16, sms // (2 * 4)))
    assert B.std_attn_splits(d1, 1, cap, 0) == 4 * parts
    d28 = B.dims(28, 1, 28, 4, 128, B.STD_BF16, 200000, cap)
    assert B.std_attn_splits(d28, 1, cap, 0) == sms
    early = B.STD_ATTN_EARLY_KV | B.STD_ATTN_EARLY_Q
    if 112 <= sms <= 224:
        assert B.std_attn_splits_ex(d28, 1, cap, 0, early) == 112
    # explicit splits are parts of every problem, with or without the flags
    assert B.std_attn_splits_ex(d1, 1, cap, 7, early) == 28
    # the early plan's grid (one CTA per problem) is that of splits = 1
    assert B.std_attn_workspace_size(d28, 1, cap, 0) >= B.std_attn_workspace_size(d28, 1, cap, 1)
