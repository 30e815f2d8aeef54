"""Parity at the workloads' full sizes, in the launch configuration bench.py times
(DecodeSession, automatic splits), on outputs the oracle can compute head by head.

* long video (28 layers, 143,360 visual + 256 text tokens, K = 4096, gamma = 8):
  selection scores / indices / gather and two draft+verify rounds on sampled
  (layer, KV head) slices; acceptance and lengths in full.
* 28-layer stack with 32,768 visual tokens: all 32 rounds, sampled slices.
* batch-8 ragged sweep: three points with everything checked on every head, and
  every (K, gamma) pair of the sweep at p = 0.9 with two rounds, draft and verify
  checked on one KV head of each sequence and selection on two heads.
"""
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


def _load_session(wl, seed):
    """Session with the full prompt cache generated head by head straight into HBM."""
    s = H.session_for(wl)

    def sink(l, b, h, ks, vs):
        n = ks.shape[0]
        s.k_full[l, b, h, :n].copy_(H.to_dev(ks))
        s.v_full[l, b, h, :n].copy_(H.to_dev(vs))

    x = synth.host_inputs(wl, seed=seed, kv_sink=sink)
    s.start(x["nvis"])
    return s, x


def _head_state(wl, seed, l, b, h):
    """fp64 oracle inputs of one (layer, batch, KV head) slice, shaped [1][1][1]..."""
    f = lambda a: synth.storage_to_f64(synth.storage(a, wl.dtype), wl.dtype)  # noqa: E731
    nv = wl.nvis[b]
    k, v = synth.kv_head(wl, seed, l, b, h)
    kf = np.zeros((1, 1, 1, wl.cap_full, wl.d))
    vf = np.zeros_like(kf)
    kf[0, 0, 0, :nv + wl.T] = f(k)
    vf[0, 0, 0, :nv + wl.T] = f(v)
    qt = f(synth.q_text_head(wl, seed, l, b, h))[None, None]
    return kf, vf, qt, f


def _run_rounds_and_check(wl, seed, R, heads, select_heads=None):
    """R rounds through the library; acceptance and lengths checked for every sequence,
    draft and verify outputs on `heads`, selection scores and index sets on `select_heads`
    (default: all of `heads`)."""
    s, x = _load_session(wl, seed)
    s.select(H.to_dev(x["q_text"]))
    idx_g = s.idx.cpu().numpy()
    sc_g = s.scores.cpu().numpy()
    outs = []
    for r in range(R):
        io = {k: H.to_dev(x[k][r]) for k in ("q_draft", "k_draft", "v_draft", "q_verify", "k_verify", "v_verify")}
        io["draft_tokens"] = torch.from_numpy(x["draft_tokens"][r]).cuda()
        io["dense_tokens"] = torch.from_numpy(x["dense_tokens"][r]).cuda()
        io.update(s.round_outputs())
        s.round(io)
        outs.append({k: io[k].cpu().numpy() for k in ("o_draft", "o_verify", "n_plus_1", "accepted")})
    torch.cuda.synchronize()
    assert B.std_get_device_error() == 0
    # acceptance and lengths for every sequence
    lf = np.array(wl.nvis) + wl.T
    ls = np.full(wl.B, wl.K + wl.T)
    for r in range(R):
        n1, acc = oracle.accept_prefix(x["draft_tokens"][r], x["dense_tokens"][r])
        np.testing.assert_array_equal(outs[r]["n_plus_1"], n1)
        np.testing.assert_array_equal(outs[r]["accepted"], acc)
        lf += n1
        ls += n1
    np.testing.assert_array_equal(s.len_full.cpu().numpy(), lf)
    np.testing.assert_array_equal(s.len_sparse.cpu().numpy(), ls)

    tol = H.attn_tol(wl)
    rtol = H.score_rtol(wl)
    G = wl.G
    for (l, b, h) in heads:
        kf, vf, qt, f = _head_state(wl, seed, l, b, h)
        nv = wl.nvis[b]
        if select_heads is None or (l, b, h) in select_heads:
            idx_o, sc_o, _, _, _ = oracle.select_topk(qt, kf, vf, np.array([nv]), wl.T, wl.K, wl.cap_sparse)
            np.testing.assert_allclose(sc_g[l, b, h, :nv], sc_o[0, 0, 0, :nv], rtol=rtol,
                                       atol=rtol * 1e-3 * sc_o[0, 0, 0, :nv].max())
            H.assert_topk_boundary(idx_g[l, b, h], idx_o[0, 0, 0], sc_o[0, 0, 0, :nv], wl.K, rtol)
        # the boundary check vouches for the GPU's index set; the oracle's sparse cache is
        # gathered from it, so the draft is compared on every sampled head
        ksp, vsp, lsp = oracle.gather_sparse(kf, vf, np.array([nv]), idx_g[l, b, h][None, None, None], wl.T,
                                             wl.cap_sparse)
        qd, qv = synth.decode_queries(wl, seed, l, b, h)
        kd, vd, kvv, vvv = synth.decode_kv(wl, seed, l, b, h)
        st = {"k_full": kf, "v_full": vf, "k_sp": ksp, "v_sp": vsp,
              "len_full": np.array([nv + wl.T]), "len_sp": lsp.astype(np.int64)}
        dense, draft = synth.tokens(wl, seed, b)
        for r in range(R):
            want = oracle.decode_round(st, f(qd[r])[:, None, None, :, None, :], f(kd[r])[:, None, None, None, None, :],
                                       f(vd[r])[:, None, None, None, None, :], f(qv[r])[None, None],
                                       f(kvv[r])[None, None, None], f(vvv[r])[None, None, None],
                                       draft[r][None], dense[r][None])
            got_v = outs[r]["o_verify"][l, b, h * G:(h + 1) * G]
            assert np.abs(got_v - want["o_verify"][0, 0]).max() <= tol, (l, b, h, r)
            got_d = outs[r]["o_draft"][:, l, b, h * G:(h + 1) * G]
            assert np.abs(got_d - want["o_draft"][:, 0, 0]).max(initial=0.0) <= tol, (l, b, h, r)
    return s


def test_long_video_full_size_sampled_heads():
    wl = synth.workload("video_140k").replace(rounds=2)
    _run_rounds_and_check(wl, 0, 2, heads=[(0, 0, 0), (13, 0, 2), (27, 0, 3)])


def test_stack28_32k_all_32_rounds_sampled_heads():
    wl = synth.workload("stack28_32k")
    _run_rounds_and_check(wl, 0, 32, heads=[(0, 0, 1), (27, 0, 0)])


@pytest.mark.parametrize("K,gamma,p", [(1024, 10, 0.6), (4096, 2, 0.9), (512, 6, 0.6)])
def test_ragged_batch8_sweep_points(K, gamma, p):
    wl = synth.ragged_workload(K, gamma, p, rounds=3)
    heads = [(0, b, h) for b in range(wl.B) for h in range(wl.Hkv)]
    _run_rounds_and_check(wl, 0, 3, heads=heads)


@pytest.mark.parametrize("gamma", [2, 4, 6, 8, 10])
@pytest.mark.parametrize("K", [512, 1024, 4096])
def test_ragged_batch8_every_K_gamma_pair(K, gamma):
    """Every (K, gamma) point of the batch-8 ragged sweep at p = 0.9: both MMA layouts
    (G * (gamma + 1) = 77 rows at gamma = 10 takes M = 128, the rest M = 64), every
    ragged length, commits of up to gamma + 1 rows."""
    wl = synth.ragged_workload(K, gamma, 0.9, rounds=2)
    heads = [(0, b, b % wl.Hkv) for b in range(wl.B)]
    longest = int(np.argmax(wl.nvis))
    shortest = int(np.argmin(wl.nvis))
    _run_rounds_and_check(wl, 0, 2, heads=heads,
                          select_heads={(0, longest, longest % wl.Hkv), (0, shortest, shortest % wl.Hkv)})
