"""Decode attention over key ranges (std_dense_verify_attn_partial,
std_sparse_decode_attn_partial) and their merge (std_merge_partials) through the C ABI,
against the fp64 oracle: the cache split into 1-4 row ranges -- and into shard buffers
that start at a later position -- then merged, equals the full attention.  Per range the
determined quantities of a partial, o / l and m + ln l, are compared with the oracle's."""
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


def _wl(name, L=2, Bsz=2, Hq=28, Hkv=4, d=128, nvis=(1500, 700), T=40, K=128, gamma=6, wl_id=120):
    return synth.Workload(name, wl_id, "bf16", L, Bsz, Hq, Hkv, d, tuple(nvis), T, K, gamma, 0.02, 0.7, 1)


CASES = {
    "G7_g6": _wl("G7_g6"),                                           # 49 rows, M = 64 layout
    "G7_g10": _wl("G7_g10", gamma=10, wl_id=121),                    # 77 rows, M = 128 layout
    "G2_d64": _wl("G2_d64", Hq=4, Hkv=2, d=64, nvis=(900, 2100, 33), Bsz=3, wl_id=122),  # 14 rows: SPLIT layout
}


def _verify_inputs(wl, x):
    kf = x["k_full"].copy()
    vf = x["v_full"].copy()
    for b in range(wl.B):
        p = wl.nvis[b] + wl.T
        kf[:, b, :, p:p + wl.gamma + 1] = x["k_verify"][0][:, b]
        vf[:, b, :, p:p + wl.gamma + 1] = x["v_verify"][0][:, b]
    return kf, vf


def _run_verify_partial(wl, d, q, kf, vf, ctx, pos0, r0, r1, splits=0):
    shape = (wl.L, wl.B, wl.Hq, wl.gamma + 1, wl.d)
    o = torch.full(shape, float("nan"), device="cuda")
    ml = torch.full(shape[:-1] + (2,), float("nan"), device="cuda")
    ws = torch.empty(max(16, B.std_attn_workspace_size(d, wl.gamma + 1, d.cap_full, splits)), dtype=torch.uint8,
                     device="cuda")
    B.std_dense_verify_attn_partial(d, q, wl.gamma, kf, vf, ctx, pos0, r0, r1, o, ml, splits, ws)
    return o, ml


def _check_partial(o, ml, want):
    """o / l and m + ln l against the oracle's partial (rows without keys: o = 0, m = -inf, l = 0)."""
    wo, wm, wl_ = want
    o, ml = o.cpu().numpy().astype(np.float64), ml.cpu().numpy().astype(np.float64)
    m, l = ml[..., 0], ml[..., 1]
    empty = wl_ == 0
    assert (np.isneginf(m[empty])).all() and (l[empty] == 0).all() and (o[empty] == 0).all()
    live = ~empty
    assert (l[live] > 0).all()
    np.testing.assert_allclose(o[live] / l[live][..., None], wo[live] / wl_[live][..., None], atol=2e-2, rtol=0)
    np.testing.assert_allclose(m[live] + np.log(l[live]), wm[live] + np.log(wl_[live]), atol=2e-3, rtol=0)


@pytest.mark.parametrize("name", sorted(CASES))
# (0, 1543, None): the second range starts inside sequence 0's verify rows (positions 1540..1546),
# so its first query rows attend no key there while the later ones do
@pytest.mark.parametrize("cuts", [(0, None), (0, 640, None), (0, 128, 1000, 1600, None), (0, 0, 300, None),
                                  (0, 1543, None)])
def test_verify_ranges_merge_to_full_verify(name, cuts):
    wl = CASES[name]
    x = synth.host_inputs(wl, seed=7)
    kf, vf = _verify_inputs(wl, x)
    cap = wl.cap_full
    cuts = tuple(cap if c is None else min(c, cap) for c in cuts)
    n_ctx = np.array(wl.nvis) + wl.T
    d = B.dims(wl.L, wl.B, wl.Hq, wl.Hkv, wl.d, B.STD_BF16, cap, wl.cap_sparse)
    q, kd, vd = H.to_dev(x["q_verify"][0]), H.to_dev(kf), H.to_dev(vf)
    ctx = torch.from_numpy(n_ctx.astype(np.int32)).cuda()
    q64, k64, v64 = H.f64(x["q_verify"][0], wl), H.f64(kf, wl), H.f64(vf, wl)
    parts = []
    for r0, r1 in zip(cuts[:-1], cuts[1:]):
        o, ml = _run_verify_partial(wl, d, q, kd, vd, ctx, 0, r0, r1)
        torch.cuda.synchronize()
        assert B.std_get_device_error() == 0
        _check_partial(o, ml, oracle.attn_range_partial(q64, k64, v64, n_ctx + 1, 0, r0, r1))
        parts.append((o, ml))
    o_all = torch.stack([p[0] for p in parts]).contiguous()
    ml_all = torch.stack([p[1] for p in parts]).contiguous()
    out = torch.full_like(parts[0][0], float("nan"))
    rows = out.numel() // wl.d
    B.std_merge_partials(rows, wl.d, len(parts), o_all, ml_all, out)
    torch.cuda.synchronize()
    want = oracle.dense_verify_attn(q64, k64, v64, n_ctx)
    assert np.abs(out.cpu().numpy() - want).max() <= 2e-2


def test_verify_shard_buffers_starting_at_later_positions():
    """Each 'rank' holds only its rows in a buffer of its own (row r = position pos0 + r), as
    when the cache is split over GPUs; the last shard holds the verify rows."""
    wl = CASES["G7_g6"]
    x = synth.host_inputs(wl, seed=8)
    kf, vf = _verify_inputs(wl, x)
    cap = wl.cap_full
    n_ctx = np.array(wl.nvis) + wl.T
    ctx = torch.from_numpy(n_ctx.astype(np.int32)).cuda()
    q = H.to_dev(x["q_verify"][0])
    parts = []
    for pos0, pos1 in ((0, 512), (512, 1280), (1280, cap)):
        rows = pos1 - pos0
        d = B.dims(wl.L, wl.B, wl.Hq, wl.Hkv, wl.d, B.STD_BF16, rows, wl.cap_sparse)
        ks = H.to_dev(np.ascontiguousarray(kf[:, :, :, pos0:pos1]))
        vs = H.to_dev(np.ascontiguousarray(vf[:, :, :, pos0:pos1]))
        parts.append(_run_verify_partial(wl, d, q, ks, vs, ctx, pos0, 0, rows))
    torch.cuda.synchronize()
    assert B.std_get_device_error() == 0
    out = torch.empty_like(parts[0][0])
    B.std_merge_partials(out.numel() // wl.d, wl.d, 3, torch.stack([p[0] for p in parts]).contiguous(),
                         torch.stack([p[1] for p in parts]).contiguous(), out)
    torch.cuda.synchronize()
    want = oracle.dense_verify_attn(H.f64(x["q_verify"][0], wl), H.f64(kf, wl), H.f64(vf, wl), n_ctx)
    assert np.abs(out.cpu().numpy() - want).max() <= 2e-2


@pytest.mark.parametrize("splits", [0, 1, 3])
def test_draft_ranges_merge_to_full_draft(splits):
    wl = CASES["G7_g6"]
    x = synth.host_inputs(wl, seed=9)
    rng = np.random.default_rng(4)
    cap = wl.cap_sparse
    ksp = np.zeros((wl.L, wl.B, wl.Hkv, cap, wl.d), np.uint16)
    vsp = np.zeros_like(ksp)
    base = wl.K + wl.T
    for b in range(wl.B):
        rows = np.concatenate([np.sort(rng.choice(wl.nvis[b], wl.K, replace=False)),
                               np.arange(wl.nvis[b], wl.nvis[b] + wl.T)])
        ksp[:, b, :, :base] = x["k_full"][:, b][:, :, rows]
        vsp[:, b, :, :base] = x["v_full"][:, b][:, :, rows]
    lens = np.full(wl.B, base - 3, np.int32)
    off = 3                                              # attends rows < len + 3 = base
    d = B.dims(wl.L, wl.B, wl.Hq, wl.Hkv, wl.d, B.STD_BF16, wl.cap_full, cap)
    q = np.ascontiguousarray(x["q_draft"][0, 0])
    qd, kd, vd = H.to_dev(q), H.to_dev(ksp), H.to_dev(vsp)
    ln = torch.from_numpy(lens).cuda()
    ws = torch.empty(max(16, B.std_attn_workspace_size(d, 1, cap, splits)), dtype=torch.uint8, device="cuda")
    parts = []
    for r0, r1 in ((0, 100), (100, 101), (101, cap)):
        o = torch.full((wl.L, wl.B, wl.Hq, 1, wl.d), float("nan"), device="cuda")
        ml = torch.full((wl.L, wl.B, wl.Hq, 1, 2), float("nan"), device="cuda")
        B.std_sparse_decode_attn_partial(d, qd, kd, vd, ln, off, 0, r0, r1, o, ml, splits, ws)
        torch.cuda.synchronize()
        assert B.std_get_device_error() == 0
        _check_partial(o, ml, oracle.attn_range_partial(H.f64(q, wl), H.f64(ksp, wl), H.f64(vsp, wl), lens + off,
                                                        0, r0, r1))
        parts.append((o, ml))
    out = torch.empty_like(parts[0][0])
    B.std_merge_partials(out.numel() // wl.d, wl.d, 3, torch.stack([p[0] for p in parts]).contiguous(),
                         torch.stack([p[1] for p in parts]).contiguous(), out)
    torch.cuda.synchronize()
    want = oracle.sparse_decode_attn(H.f64(q, wl), H.f64(ksp, wl), H.f64(vsp, wl), lens + off)
    assert np.abs(out.cpu().numpy() - want).max() <= 2e-2


def test_long_video_verify_split_over_four_ranges():
    """143,616 + 9 rows per head, 28 layers (the long-video verify) split into 4 ranges as 4
    GPUs would hold them; merged output against the oracle on sampled heads."""
    wl = synth.workload("video_140k").replace(rounds=1)
    s = H.session_for(wl)

    def sink(l, b, h, ks, vs):
        s.k_full[l, b, h, :ks.shape[0]].copy_(H.to_dev(ks))
        s.v_full[l, b, h, :vs.shape[0]].copy_(H.to_dev(vs))

    x = synth.host_inputs(wl, seed=0, kv_sink=sink)
    n_ctx = wl.nvis[0] + wl.T
    ctx = torch.tensor([n_ctx], dtype=torch.int32, device="cuda")
    B.std_kv_append(s.dims, s.k_full, s.v_full, wl.cap_full, ctx, 0, H.to_dev(x["k_verify"][0]),
                    H.to_dev(x["v_verify"][0]), wl.gamma + 1)
    q = H.to_dev(x["q_verify"][0])
    shape = (wl.L, 1, wl.Hq, wl.gamma + 1, wl.d)
    cuts = (0, 35840, 71680, 107520, wl.cap_full)
    o_all = torch.empty((4,) + shape, device="cuda")
    ml_all = torch.empty((4,) + shape[:-1] + (2,), device="cuda")
    for i, (r0, r1) in enumerate(zip(cuts[:-1], cuts[1:])):
        B.std_dense_verify_attn_partial(s.dims, q, wl.gamma, s.k_full, s.v_full, ctx, 0, r0, r1, o_all[i], ml_all[i],
                                        0, s.ws_round)
    out = torch.empty(shape, device="cuda")
    B.std_merge_partials(out.numel() // wl.d, wl.d, 4, o_all, ml_all, out)
    o_full = torch.empty(shape, device="cuda")
    B.std_dense_verify_attn(s.dims, q, wl.gamma, s.k_full, s.v_full, ctx, o_full, 0, s.ws_round)
    torch.cuda.synchronize()
    assert B.std_get_device_error() == 0
    assert (out - o_full).abs().max().item() <= 1e-2       # two GPU paths, same bf16 products
    f = lambda a: synth.storage_to_f64(synth.storage(a, wl.dtype), wl.dtype)  # noqa: E731
    qv = H.f64(x["q_verify"][0], wl)
    for (l, h) in ((0, 0), (17, 3)):
        k, v = synth.kv_head(wl, 0, l, 0, h)
        kk = np.concatenate([f(k), H.f64(x["k_verify"][0][l, 0, h], wl)])
        vv = np.concatenate([f(v), H.f64(x["v_verify"][0][l, 0, h], wl)])
        want = oracle.dense_verify_attn(qv[l:l + 1, :, h * wl.G:(h + 1) * wl.G], kk[None, None, None],
                                        vv[None, None, None], np.array([n_ctx]))
        got = out[l, 0, h * wl.G:(h + 1) * wl.G].cpu().numpy()
        assert np.abs(got - want[0, 0]).max() <= 2e-2, (l, h)


def test_partial_rejections():
    wl = CASES["G7_g6"]
    d = B.dims(wl.L, wl.B, wl.Hq, wl.Hkv, wl.d, B.STD_BF16, wl.cap_full, wl.cap_sparse)
    t = torch.zeros(16, device="cuda")
    with pytest.raises(B.StdError) as e:
        B.std_dense_verify_attn_partial(d, t, wl.gamma, t, t, t, 0, 10, 5, t, t)
    assert e.value.code == B.STD_ERR_INVALID_ARG
    with pytest.raises(B.StdError) as e:
        B.std_dense_verify_attn_partial(d, t, wl.gamma, t, t, t, 0, 0, wl.cap_full + 1, t, t)
    assert e.value.code == B.STD_ERR_INVALID_ARG
    f = B.dims(1, 1, 4, 2, 64, B.STD_F32, 100, 100)
    with pytest.raises(B.StdError) as e:
        B.std_dense_verify_attn_partial(f, t, 1, t, t, t, 0, 0, 50, t, t, 0, torch.zeros(1 << 16, device="cuda"))
    assert e.value.code == B.STD_ERR_UNSUPPORTED
