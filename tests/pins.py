"""Checks that pin the fp64 oracle to facts outside itself.

Each ``check_*`` takes the oracle module (or a stand-in with the same
functions) and raises AssertionError on a mismatch, so the same checks can be
run against deliberately broken copies of the oracle to show that they catch
plausible mistakes (dropped scale, wrong GQA grouping, off-by-one mask,
wrong tie rule, non-prefix acceptance, wrong commit window).

Sources of truth used here, none of them the oracle's own formulas:
  * hand-derived closed forms stored under tests/golden/ (logits ln 1, ln 2, ...
    make the softmax weights small integers over their sum);
  * brute-force enumeration on tiny inputs;
  * library routines: heapq.nlargest, torch's scaled_dot_product_attention in
    float64, the logistic function written via tanh;
  * mathematical invariants (a mean of distributions sums to 1, uniform
    attention when all logits are equal).
"""
from __future__ import annotations

import heapq
import itertools
import json
import math
import os

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def load_golden(name: str) -> dict:
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


# ----------------------------------------------------------------------------- attention

def check_golden_attention(orc) -> None:
    g = load_golden("attention_3key.json")
    o = orc.attend(np.array(g["q"]), np.array(g["k"]), np.array(g["v"]))
    np.testing.assert_allclose(o, g["expected"], atol=g["atol"], rtol=0)


def check_golden_verify(orc) -> None:
    g = load_golden("verify_causal_2row.json")
    k = np.array(g["k"])[None, None, None]          # [L=1][B=1][Hkv=1][n][d]
    v = np.array(g["v"])[None, None, None]
    q = np.array(g["q"])[None, None, None]          # [1][1][Hq=1][2][d]
    o = orc.dense_verify_attn(q, k, v, np.array([g["n_ctx"]]))
    np.testing.assert_allclose(o[0, 0, 0], g["expected"], atol=g["atol"], rtol=0)


def check_attention_vs_sdpa(orc, seed: int = 3) -> None:
    """Decode and verify attention against torch SDPA (float64) with an explicit mask."""
    import torch
    rng = np.random.default_rng(seed)
    L, B, Hq, Hkv, d, gamma = 2, 2, 6, 2, 16, 3
    G = Hq // Hkv
    n_ctx = np.array([11, 5])
    cap = 20
    k = rng.standard_normal((L, B, Hkv, cap, d)) * 2
    v = rng.standard_normal((L, B, Hkv, cap, d))
    q = rng.standard_normal((L, B, Hq, gamma + 1, d)) * 2
    o = orc.dense_verify_attn(q, k, v, n_ctx)
    o_sp = orc.sparse_decode_attn(q[:, :, :, :1], k, v, n_ctx + 1)
    for l in range(L):
        for b in range(B):
            n = int(n_ctx[b]) + gamma + 1
            kk = torch.from_numpy(np.repeat(k[l, b, :, :n], G, axis=0))    # [Hq][n][d]
            vv = torch.from_numpy(np.repeat(v[l, b, :, :n], G, axis=0))
            qq = torch.from_numpy(q[l, b])                                  # [Hq][rows][d]
            i = torch.arange(gamma + 1)[:, None]
            j = torch.arange(n)[None, :]
            mask = j < (int(n_ctx[b]) + i + 1)
            ref = torch.nn.functional.scaled_dot_product_attention(qq, kk, vv, attn_mask=mask)
            np.testing.assert_allclose(o[l, b], ref.numpy(), atol=1e-12, rtol=1e-12)
            np.testing.assert_allclose(o_sp[l, b], ref.numpy()[:, :1], atol=1e-12, rtol=1e-12)


def check_attention_closed_forms(orc, seed: int = 4) -> None:
    rng = np.random.default_rng(seed)
    d = 8
    q = rng.standard_normal(d)
    # one key: the output is that value row
    v1 = rng.standard_normal((1, d))
    np.testing.assert_allclose(orc.attend(q, rng.standard_normal((1, d)), v1), v1[0], atol=1e-14)
    # identical keys: uniform weights, the mean of the values
    kk = np.repeat(rng.standard_normal((1, d)), 5, axis=0)
    vv = rng.standard_normal((5, d))
    np.testing.assert_allclose(orc.attend(q, kk, vv), vv.mean(axis=0), atol=1e-14)
    # two keys: logistic weighting sigma(x) = (1 + tanh(x/2)) / 2 of the logit gap
    k2 = rng.standard_normal((2, d))
    v2 = rng.standard_normal((2, d))
    x = (q @ k2[0] - q @ k2[1]) / math.sqrt(d)
    w = 0.5 * (1.0 + math.tanh(0.5 * x))
    np.testing.assert_allclose(orc.attend(q, k2, v2), w * v2[0] + (1 - w) * v2[1], atol=1e-14)


# ----------------------------------------------------------------------------- selection

def check_golden_selection(orc) -> None:
    g = load_golden("selection_gqa.json")
    q_text = np.array(g["q_text"])[None, None]                     # [1][1][Hq][T][d]
    kv = np.array(g["k_vis"])
    Hkv, nv, d = 2, kv.shape[0], kv.shape[1]
    T = q_text.shape[3]
    k_full = np.zeros((1, 1, Hkv, nv + T, d))
    k_full[0, 0, :, :nv] = kv
    v_full = np.zeros_like(k_full)
    for K, key in ((1, "expected_top1"), (2, "expected_top2")):
        idx, scores, _, _, _ = orc.select_topk(q_text, k_full, v_full, np.array([nv]), T, K, nv + T)
        np.testing.assert_allclose(scores[0, 0], g["expected_scores"], atol=g["atol"], rtol=0)
        assert idx[0, 0].tolist() == g[key], (idx[0, 0].tolist(), g[key])


def check_golden_selection_causal(orc) -> None:
    """Hand-derived causal full-row and visual-only scores, with and without a prompt prefix
    (exact rationals; derivation in the fixture)."""
    g = load_golden("selection_causal.json")
    q = np.array(g["q_text"])[None, None]                          # [1][1][1][T][d]
    rows, pre = np.array(g["k_rows"]), np.array(g["k_prefix"])
    nv, T, P = g["nvis"], q.shape[3], pre.shape[0]
    cases = ((rows, 0, True, "expected_causal"), (rows, 0, False, "expected_visual_only"),
             (np.concatenate([pre, rows]), P, True, "expected_causal_prefix"),
             (np.concatenate([pre, rows]), P, False, "expected_visual_only"))
    for kr, n_prefix, causal, key in cases:
        kf = kr[None, None, None]
        vf = kf + 1.0
        idx, sc, ksp, vsp, lsp = orc.select_topk(q, kf, vf, np.array([nv]), T, 1, n_prefix + 1 + T,
                                                 causal_text=causal, n_prefix=n_prefix)
        np.testing.assert_allclose(sc[0, 0, 0], g[key], atol=g["atol"], rtol=0)
        assert idx[0, 0, 0].tolist() == g["expected_top1"]
        # sparse cache: [prefix rows | the selected visual row | text rows]
        want = np.concatenate([kr[:n_prefix], kr[n_prefix:n_prefix + 1], kr[n_prefix + nv:n_prefix + nv + T]])
        np.testing.assert_array_equal(ksp[0, 0, 0], want)
        np.testing.assert_array_equal(vsp[0, 0, 0], want + 1.0)
        assert lsp.tolist() == [n_prefix + 1 + T]
    # the score functions themselves, on the same rows
    qg, kv, kt = q[0, 0], rows[:nv], rows[nv:nv + T]
    np.testing.assert_allclose(orc.selection_scores_causal(qg, kv, kt), g["expected_causal"], atol=g["atol"], rtol=0)
    np.testing.assert_allclose(orc.selection_scores_causal(qg, kv, kt, pre), g["expected_causal_prefix"],
                               atol=g["atol"], rtol=0)
    np.testing.assert_allclose(orc.selection_scores(qg, kv), g["expected_visual_only"], atol=g["atol"], rtol=0)


def check_selection_invariants(orc, seed: int = 5) -> None:
    rng = np.random.default_rng(seed)
    G, T, d, nv = 3, 7, 16, 50
    q = rng.standard_normal((G, T, d)) * 3
    k = rng.standard_normal((nv, d))
    s = orc.selection_scores(q, k)
    assert s.shape == (nv,)
    assert abs(s.sum() - 1.0) < 1e-12                       # a mean of distributions
    assert (s > 0).all()
    np.testing.assert_allclose(orc.selection_scores(np.zeros_like(q), k), np.full(nv, 1 / nv),
                               atol=1e-15)                   # zero queries: uniform
    np.testing.assert_allclose(orc.selection_scores(q, np.repeat(k[:1], nv, axis=0)),
                               np.full(nv, 1 / nv), atol=1e-15)  # identical keys: uniform
    # a key that dominates every row's softmax collects almost all mass
    k2 = k.copy()
    k2[17] = 40.0 * q.reshape(-1, d).mean(axis=0) / np.linalg.norm(q.reshape(-1, d).mean(axis=0))
    s2 = orc.selection_scores(q, k2)
    assert int(np.argmax(s2)) == 17



def check_selection_causal(orc, seed: int = 11) -> None:
    """The causal full-row reading of the selection score, against (1) the prompt's full
    causal attention matrix for the text rows, masked and normalised by torch in float64;
    (2) a closed form; (3) invariants."""
    import torch
    rng = np.random.default_rng(seed)
    G, T, d, nv = 3, 6, 8, 11
    q = rng.standard_normal((G, T, d)) * 2
    kv = rng.standard_normal((nv, d))
    kt = rng.standard_normal((T, d))
    s = orc.selection_scores_causal(q, kv, kt)
    # (1) logits of every text query against [visual keys, text keys], mask text key j > t
    keys = torch.from_numpy(np.concatenate([kv, kt]))
    qt = torch.from_numpy(q.reshape(G * T, d))
    logits = (qt @ keys.T) / math.sqrt(d)
    t_of_row = torch.arange(G * T) % T
    mask = torch.arange(nv + T)[None, :] >= (nv + t_of_row[:, None] + 1)
    p = torch.softmax(logits.masked_fill(mask, float("-inf")), dim=-1)
    np.testing.assert_allclose(s, p[:, :nv].mean(dim=0).numpy(), rtol=1e-12, atol=1e-15)
    # (2) one visual key, one text key, d = 1: score = logistic((b - c) a), written via tanh
    a, b, c = 0.7, 1.9, -0.4
    s1 = orc.selection_scores_causal(np.array([[[a]]]), np.array([[b]]), np.array([[c]]))
    assert abs(s1[0] - 0.5 * (1 + math.tanh(0.5 * (b - c) * a))) < 1e-15
    # (3) text keys can only take mass away; with text logits far below, the visual-only score
    sv = orc.selection_scores(q, kv)
    assert (s <= sv + 1e-15).all() and s.sum() < 1.0
    q2 = q.copy()
    q2[..., 0] = 5.0
    kt2 = kt.copy()
    kt2[:, 0] = -1000.0
    np.testing.assert_allclose(orc.selection_scores_causal(q2, kv, kt2), orc.selection_scores(q2, kv),
                               rtol=0, atol=1e-12)
    # (4) a prompt prefix (system prompt) before the video: its keys are visible to every row
    P = 4
    kp = rng.standard_normal((P, d))
    sp = orc.selection_scores_causal(q, kv, kt, kp)
    keys = torch.from_numpy(np.concatenate([kp, kv, kt]))
    logits = (qt @ keys.T) / math.sqrt(d)
    mask = torch.arange(P + nv + T)[None, :] >= (P + nv + t_of_row[:, None] + 1)
    p = torch.softmax(logits.masked_fill(mask, float("-inf")), dim=-1)
    np.testing.assert_allclose(sp, p[:, P:P + nv].mean(dim=0).numpy(), rtol=1e-12, atol=1e-15)
    assert (sp <= s + 1e-15).all()


def check_selection_prefix(orc, seed: int = 13) -> None:
    """A prompt prefix before the visual block: the visual-only scores and indices are those
    of the same prompt without it (softmax over the visual keys, which did not change), and
    the sparse cache is [prefix rows | selected visual rows | text rows]."""
    rng = np.random.default_rng(seed)
    L, B, Hq, Hkv, d, T, K, P = 1, 2, 4, 2, 8, 3, 4, 5
    nvis = np.array([11, 7])
    cap = P + 11 + T
    q = rng.standard_normal((L, B, Hq, T, d)) * 2
    kf = rng.standard_normal((L, B, Hkv, cap, d))
    vf = rng.standard_normal((L, B, Hkv, cap, d))
    idx_p, sc_p, ksp, vsp, lsp = orc.select_topk(q, kf, vf, nvis, T, K, P + K + T, n_prefix=P)
    idx_0, sc_0, k0, _, _ = orc.select_topk(q, kf[:, :, :, P:], vf[:, :, :, P:], nvis, T, K, K + T)
    np.testing.assert_array_equal(idx_p, idx_0)
    np.testing.assert_allclose(sc_p, sc_0, rtol=0, atol=0)
    assert lsp.tolist() == [P + K + T] * B
    for b in range(B):
        nv = nvis[b]
        np.testing.assert_array_equal(ksp[0, b, 1, :P], kf[0, b, 1, :P])
        np.testing.assert_array_equal(ksp[0, b, 1, P:P + K], kf[0, b, 1, P + idx_p[0, b, 1]])
        np.testing.assert_array_equal(vsp[0, b, 0, P + K:P + K + T], vf[0, b, 0, P + nv:P + nv + T])
        np.testing.assert_array_equal(ksp[0, b, 1, P:P + K + T], k0[0, b, 1, :K + T])



def check_streaming_and_gather(orc, seed: int = 12) -> None:
    """Streaming index sets written out by hand; gather_sparse on the top-K indices equals
    select_topk's own sparse cache, and on a hand-made index set copies the named rows."""
    assert orc.streaming_indices(10, 4, 1).tolist() == [0, 7, 8, 9]
    assert orc.streaming_indices(10, 4, 0).tolist() == [6, 7, 8, 9]
    assert orc.streaming_indices(10, 4, 4).tolist() == [0, 1, 2, 3]
    assert orc.streaming_indices(5, 5, 2).tolist() == [0, 1, 2, 3, 4]
    rng = np.random.default_rng(seed)
    L, B, Hq, Hkv, d, T, K = 2, 2, 4, 2, 8, 3, 5
    nvis = np.array([12, 9])
    cap = 12 + T
    q = rng.standard_normal((L, B, Hq, T, d))
    kf = rng.standard_normal((L, B, Hkv, cap, d))
    vf = rng.standard_normal((L, B, Hkv, cap, d))
    idx, _, ksp, vsp, lsp = orc.select_topk(q, kf, vf, nvis, T, K, K + T + 2)
    k2, v2, l2 = orc.gather_sparse(kf, vf, nvis, idx, T, K + T + 2)
    np.testing.assert_array_equal(k2, ksp)
    np.testing.assert_array_equal(v2, vsp)
    np.testing.assert_array_equal(l2, lsp)
    mine = np.zeros((L, B, Hkv, 2), np.int32)
    mine[..., 0], mine[..., 1] = 3, 0
    k3, v3, _ = orc.gather_sparse(kf, vf, nvis, mine, T, 2 + T)
    np.testing.assert_array_equal(k3[1, 1, 0, 0], kf[1, 1, 0, 3])
    np.testing.assert_array_equal(v3[0, 1, 1, 1], vf[0, 1, 1, 0])
    np.testing.assert_array_equal(k3[0, 1, 1, 2:2 + T], kf[0, 1, 1, 9:9 + T])
    # with a 2-row prompt prefix before the video: [prefix | named visual rows | text]
    P = 2
    kp = rng.standard_normal((L, B, Hkv, P + cap, d))
    vp = rng.standard_normal((L, B, Hkv, P + cap, d))
    k4, v4, l4 = orc.gather_sparse(kp, vp, nvis, mine, T, P + 2 + T, P)
    assert l4.tolist() == [P + 2 + T] * B
    np.testing.assert_array_equal(k4[1, 0, 1, :P], kp[1, 0, 1, :P])
    np.testing.assert_array_equal(k4[1, 0, 1, P], kp[1, 0, 1, P + 3])
    np.testing.assert_array_equal(v4[0, 1, 0, P + 1], vp[0, 1, 0, P + 0])
    np.testing.assert_array_equal(v4[0, 1, 0, P + 2:P + 2 + T], vp[0, 1, 0, P + 9:P + 9 + T])
    np.testing.assert_array_equal(k4[1, 0, 0, P + 2:P + 2 + T], kp[1, 0, 0, P + 12:P + 12 + T])


def _brute_topk(s, K):
    """The unique K-subset whose members all beat all non-members under (score desc, pos asc)."""
    n = len(s)
    found = []
    for sub in itertools.combinations(range(n), K):
        ins = set(sub)
        if all((s[a] > s[b]) or (s[a] == s[b] and a < b) for a in ins for b in range(n) if b not in ins):
            found.append(list(sub))
    assert len(found) == 1
    return found[0]


def check_topk_bruteforce(orc, seed: int = 6) -> None:
    rng = np.random.default_rng(seed)
    for trial in range(40):
        n = int(rng.integers(1, 8))
        s = rng.integers(0, 4, size=n).astype(np.float64) / 4   # many ties
        for K in range(n + 1):
            got = orc.topk_indices(s, K).tolist()
            assert got == _brute_topk(s, K), (s, K, got)
            want = sorted(heapq.nlargest(K, range(n), key=lambda i: (s[i], -i)))
            assert got == want


def check_topk_special(orc, seed: int = 7) -> None:
    rng = np.random.default_rng(seed)
    s = rng.random(300)
    s[[10, 200]] = 2.0                                        # tie at the maximum
    assert orc.topk_indices(s, 1).tolist() == [int(np.argmax(s))] == [10]
    assert orc.topk_indices(s, 300).tolist() == list(range(300))
    assert orc.topk_indices(s, 0).tolist() == []


def check_full_k_sparse_equals_dense(orc, seed: int = 8) -> None:
    """K = Nv keeps every visual row in order, so sparse attention equals dense attention."""
    rng = np.random.default_rng(seed)
    L, B, Hq, Hkv, d, nv, T = 1, 1, 4, 2, 8, 30, 5
    cap = nv + T + 4
    k = np.zeros((L, B, Hkv, cap, d))
    v = np.zeros((L, B, Hkv, cap, d))
    k[..., :nv + T, :] = rng.standard_normal((L, B, Hkv, nv + T, d))
    v[..., :nv + T, :] = rng.standard_normal((L, B, Hkv, nv + T, d))
    qt = rng.standard_normal((L, B, Hq, T, d))
    idx, _, ksp, vsp, lsp = orc.select_topk(qt, k, v, np.array([nv]), T, nv, cap)
    assert idx[0, 0, 0].tolist() == list(range(nv))
    np.testing.assert_array_equal(ksp[..., :nv + T, :], k[..., :nv + T, :])
    q = rng.standard_normal((L, B, Hq, 1, d))
    a = orc.sparse_decode_attn(q, ksp, vsp, lsp)
    bb = orc.dense_verify_attn(q, k, v, np.array([nv + T - 1]))
    np.testing.assert_allclose(a, bb, atol=1e-14)


# ----------------------------------------------------------------------------- acceptance

def check_golden_accept(orc) -> None:
    g = load_golden("accept_cases.json")
    for c in g["cases"]:
        gm = len(c["draft"])
        n1, acc = orc.accept_prefix(np.array(c["draft"], dtype=np.int64).reshape(1, gm),
                                    np.array(c["dense"]).reshape(1, gm + 1))
        assert int(n1[0]) == c["n_plus_1"], c
        assert acc[0].tolist() == c["accepted"], c


def check_accept_bruteforce(orc) -> None:
    """Every match pattern for gamma <= 10: n + 1 = (index of the lowest 0 bit) + 1."""
    for gamma in range(0, 11):
        pats = np.arange(2 ** gamma)
        dense = np.tile(np.arange(100, 100 + gamma + 1), (len(pats), 1))
        bits = (pats[:, None] >> np.arange(gamma)[None, :]) & 1
        draft = np.where(bits == 1, dense[:, :gamma], dense[:, :gamma] + 7)
        n1, acc = orc.accept_prefix(draft, dense)
        for p in range(len(pats)):
            expect = (~int(p) & (int(p) + 1)).bit_length()
            assert int(n1[p]) == expect, (gamma, p)
            assert 1 <= expect <= gamma + 1
            assert acc[p, :expect].tolist() == dense[p, :expect].tolist()
            assert (acc[p, expect:] == -1).all()


# ----------------------------------------------------------------------------- round bookkeeping

def check_commit(orc, seed: int = 9) -> None:
    rng = np.random.default_rng(seed)
    L, B, Hkv, d = 2, 3, 2, 4
    kf = rng.standard_normal((L, B, Hkv, 20, d))
    vf = rng.standard_normal((L, B, Hkv, 20, d))
    ks = np.zeros((L, B, Hkv, 12, d))
    vs = np.zeros((L, B, Hkv, 12, d))
    lf = np.array([10, 4, 7])
    ls = np.array([3, 2, 5])
    n1 = np.array([1, 4, 2])
    orc.kv_commit(kf, vf, ks, vs, lf, ls, n1)
    assert lf.tolist() == [11, 8, 9] and ls.tolist() == [4, 6, 7]
    for b, (a, s, n) in enumerate(((10, 3, 1), (4, 2, 4), (7, 5, 2))):
        np.testing.assert_array_equal(ks[:, b, :, s:s + n], kf[:, b, :, a:a + n])
        np.testing.assert_array_equal(vs[:, b, :, s:s + n], vf[:, b, :, a:a + n])
        assert (ks[:, b, :, s + n:] == 0).all()


def check_round_lossless_extremes(orc, seed: int = 10) -> None:
    """All drafts right: gamma + 1 tokens per round; all wrong: only the bonus token."""
    rng = np.random.default_rng(seed)
    L, B, Hq, Hkv, d, gamma = 1, 2, 2, 1, 4, 3
    for agree in (True, False):
        st = {"k_full": np.zeros((L, B, Hkv, 40, d)), "v_full": np.zeros((L, B, Hkv, 40, d)),
              "k_sp": np.zeros((L, B, Hkv, 30, d)), "v_sp": np.zeros((L, B, Hkv, 30, d)),
              "len_full": np.array([6, 9]), "len_sp": np.array([3, 4])}
        st["k_full"][..., :9, :] = rng.standard_normal((L, B, Hkv, 9, d))
        dense = rng.integers(0, 50, size=(B, gamma + 1))
        draft = dense[:, :gamma] if agree else dense[:, :gamma] + 1
        kvv = rng.standard_normal((L, B, Hkv, gamma + 1, d))
        out = orc.decode_round(st, rng.standard_normal((gamma, L, B, Hq, 1, d)),
                               rng.standard_normal((gamma, L, B, Hkv, 1, d)),
                               rng.standard_normal((gamma, L, B, Hkv, 1, d)),
                               rng.standard_normal((L, B, Hq, gamma + 1, d)), kvv, kvv.copy(),
                               draft, dense)
        n = gamma + 1 if agree else 1
        assert out["n_plus_1"].tolist() == [n, n]
        assert out["accepted"][:, :n].tolist() == dense[:, :n].tolist()
        assert st["len_full"].tolist() == [6 + n, 9 + n] and st["len_sp"].tolist() == [3 + n, 4 + n]
        np.testing.assert_array_equal(st["k_sp"][:, 0, :, 3:3 + n], kvv[:, 0, :, :n])
        np.testing.assert_array_equal(st["k_full"][:, 1, :, 9:9 + gamma + 1], kvv[:, 1])


def check_golden_draft_round(orc) -> None:
    """A whole 2-draft round with hand-derived rational outputs: each draft step's row lands
    at len_sparse + j and the step attends over len_sparse + j + 1 rows; the verify, the
    acceptance and the commit (which overwrites the draft rows) follow (derivation in the
    fixture)."""
    g = load_golden("draft_round_2step.json")
    d = 4
    st = {"k_sp": np.zeros((1, 1, 1, g["cap_sparse"], d)), "v_sp": np.zeros((1, 1, 1, g["cap_sparse"], d)),
          "k_full": np.zeros((1, 1, 1, g["cap_full"], d)), "v_full": np.zeros((1, 1, 1, g["cap_full"], d)),
          "len_sp": np.array([g["len_sparse"]]), "len_full": np.array([g["len_full"]])}
    st["k_sp"][0, 0, 0, :g["len_sparse"]] = g["k_sparse_rows"]
    st["v_sp"][0, 0, 0, :g["len_sparse"]] = g["v_sparse_rows"]
    st["k_full"][0, 0, 0, :g["len_full"]] = g["k_full_rows"]
    st["v_full"][0, 0, 0, :g["len_full"]] = g["v_full_rows"]
    gamma = len(g["draft_tokens"])
    per_step = lambda a: np.array(a).reshape(gamma, 1, 1, 1, 1, d)  # noqa: E731  [gamma][L][B][H][1][d]
    out = orc.decode_round(st, per_step(g["q_draft"]), per_step(g["k_draft"]), per_step(g["v_draft"]),
                           np.array(g["q_verify"])[None, None, None], np.array(g["k_verify"])[None, None, None],
                           np.array(g["v_verify"])[None, None, None], np.array([g["draft_tokens"]]),
                           np.array([g["dense_tokens"]]))
    np.testing.assert_allclose(out["o_draft"][:, 0, 0, 0, 0], g["expected_o_draft"], atol=g["atol"], rtol=0)
    np.testing.assert_allclose(out["o_verify"][0, 0, 0], g["expected_o_verify"], atol=g["atol"], rtol=0)
    assert out["n_plus_1"].tolist() == [g["expected_n_plus_1"]]
    assert out["accepted"][0].tolist() == g["expected_accepted"]
    assert st["len_full"].tolist() == [g["expected_len_full"]]
    assert st["len_sp"].tolist() == [g["expected_len_sparse"]]
    n = g["expected_len_sparse"]
    np.testing.assert_allclose(st["k_sp"][0, 0, 0, :n], g["expected_k_sparse_after"], atol=g["atol"], rtol=0)
    np.testing.assert_array_equal(st["v_sp"][0, 0, 0, :n], g["expected_v_sparse_after"])


def check_append_offsets(orc, seed: int = 14) -> None:
    """kv_append writes row r of sequence b at length[b] + offset + r and nothing else."""
    rng = np.random.default_rng(seed)
    L, B, H, cap, d = 2, 3, 2, 12, 3
    cache = np.zeros((L, B, H, cap, d))
    length = np.array([0, 4, 7])
    rows = rng.standard_normal((L, B, H, 2, d))
    orc.kv_append(cache, length, 3, rows)
    for b, start in enumerate((3, 7, 10)):
        np.testing.assert_array_equal(cache[:, b, :, start:start + 2], rows[:, b])
        untouched = np.delete(cache[:, b], [start, start + 1], axis=2)
        assert (untouched == 0).all()


# ----------------------------------------------------------------------------- attention over key ranges

def check_golden_partials(orc) -> None:
    """Hand-derived partials of three key ranges (one empty) and their merge (fixture)."""
    g = load_golden("attention_partials_3key.json")
    q, k, v = np.array(g["q"]), np.array(g["k"]), np.array(g["v"])
    parts = [orc.attend_partial(q, k[a:b], v[a:b]) for a, b in g["ranges"]]
    for (o, m, l), eo, em, el in zip(parts, g["expected_o"], g["expected_m"], g["expected_l"]):
        np.testing.assert_allclose(o, eo, atol=g["atol"], rtol=0)
        assert (m == -math.inf) if em == "-inf" else abs(m - em) <= g["atol"], (m, em)
        assert abs(l - el) <= g["atol"], (l, el)
    merged = orc.merge_partials(np.array([p[0] for p in parts]), np.array([p[1] for p in parts]),
                                np.array([p[2] for p in parts]))
    np.testing.assert_allclose(merged, g["expected_merged"], atol=g["atol"], rtol=0)


def check_range_partials_vs_torch(orc, seed: int = 15) -> None:
    """attn_range_partial against torch (float64): m is the max of the masked logits, l is
    exp(logsumexp - m), o / l is SDPA over the range with the causal limit; and merging the
    partials of any split of the rows into ranges gives dense verify attention."""
    import torch
    rng = np.random.default_rng(seed)
    L, B, Hq, Hkv, d, rows = 2, 2, 4, 2, 8, 3
    G = Hq // Hkv
    n_ctx = np.array([13, 6])
    cap = 20
    k = rng.standard_normal((L, B, Hkv, cap, d)) * 2
    v = rng.standard_normal((L, B, Hkv, cap, d))
    q = rng.standard_normal((L, B, Hq, rows, d)) * 2
    limit = n_ctx + 1
    for (r0, r1) in ((0, 20), (4, 11), (7, 7), (9, 16)):
        o, m, l = orc.attn_range_partial(q, k, v, limit, 0, r0, r1)
        for li in range(L):
            for b in range(B):
                for hq in range(Hq):
                    kk = torch.from_numpy(k[li, b, hq // G])
                    logits = torch.from_numpy(q[li, b, hq]) @ kk.T / math.sqrt(d)       # [rows][cap]
                    j = torch.arange(cap)[None, :]
                    i = torch.arange(rows)[:, None]
                    ok = (j >= r0) & (j < r1) & (j < int(limit[b]) + i)
                    for r in range(rows):
                        if not bool(ok[r].any()):
                            assert m[li, b, hq, r] == -math.inf and l[li, b, hq, r] == 0
                            assert not o[li, b, hq, r].any()
                            continue
                        lg = logits[r][ok[r]]
                        mm = float(lg.max())
                        assert abs(m[li, b, hq, r] - mm) < 1e-12
                        assert abs(l[li, b, hq, r] - math.exp(float(torch.logsumexp(lg, 0)) - mm)) < 1e-12
                        ref = torch.nn.functional.scaled_dot_product_attention(
                            torch.from_numpy(q[li, b, hq, r])[None], kk, torch.from_numpy(v[li, b, hq // G]),
                            attn_mask=ok[r][None])
                        np.testing.assert_allclose(o[li, b, hq, r] / l[li, b, hq, r], ref[0].numpy(), atol=1e-12)
    dense = orc.dense_verify_attn(q, k, v, n_ctx)
    for cuts in ((0, 20), (0, 5, 20), (0, 3, 8, 14, 20), (0, 0, 19, 20)):
        parts = [orc.attn_range_partial(q, k, v, limit, 0, a, b) for a, b in zip(cuts[:-1], cuts[1:])]
        merged = orc.merge_partials(*(np.array([p[t] for p in parts]) for t in range(3)))
        np.testing.assert_allclose(merged, dense, atol=1e-12, rtol=0)
    # a shard that stores positions [pos0, pos0 + n): the same partials as rows [pos0, pos0 + n)
    o1, m1, l1 = orc.attn_range_partial(q, k[:, :, :, 5:], v[:, :, :, 5:], limit, 5, 0, 10)
    o2, m2, l2 = orc.attn_range_partial(q, k, v, limit, 0, 5, 15)
    np.testing.assert_allclose(o1, o2, atol=1e-14)
    np.testing.assert_array_equal(m1, m2)
    np.testing.assert_allclose(l1, l2, atol=1e-14)


# ----------------------------------------------------------------------------- selection over parts

def check_split_selection(orc, seed: int = 16) -> None:
    """The selection over a cache split by position: each part's (m, l) against torch
    (max, exp(logsumexp - max)); the parts' merged (m, l), the parts' scores against them
    and the top-K of the parts' candidates against the whole-cache selection; the
    candidates' tie rule on a hand-made case."""
    import torch
    rng = np.random.default_rng(seed)
    G, T, d, nv = 3, 4, 8, 90
    q = rng.standard_normal((G, T, d)) * 1.5
    k = rng.standard_normal((nv, d)) * 1.5
    k[17] += 3 * q[0, 0]                              # a salient key
    whole = orc.selection_scores(q, k)
    for cuts in ((0, 90), (0, 1, 90), (0, 30, 31, 64, 90), (0, 45, 89, 90), (0, 20, 55, 90), (0, 12, 90)):
        ranges = list(zip(cuts[:-1], cuts[1:]))
        stats = [orc.selection_rowstats(q, k[a:b]) for a, b in ranges]
        for (a, b), (m, l) in zip(ranges, stats):
            x = torch.from_numpy(q.reshape(-1, d)) @ torch.from_numpy(k[a:b]).T / math.sqrt(d)
            mx = x.max(dim=1).values
            np.testing.assert_allclose(m, mx.numpy(), atol=1e-12, rtol=0)
            np.testing.assert_allclose(l, torch.exp(torch.logsumexp(x, 1) - mx).numpy(), rtol=1e-12)
        m, l = orc.merge_rowstats([s[0] for s in stats], [s[1] for s in stats])
        m0, l0 = orc.selection_rowstats(q, k)
        np.testing.assert_allclose(m, m0, atol=1e-12, rtol=0)
        np.testing.assert_allclose(l, l0, rtol=1e-12)
        part_scores = [orc.selection_scores_given_rowstats(q, k[a:b], m, l) for a, b in ranges]
        np.testing.assert_allclose(np.concatenate(part_scores), whole, rtol=1e-11)
        smallest = min(b - a for a, b in ranges)   # every part holds at least K keys
        for K in sorted({1, min(5, smallest), smallest}):
            parts = []
            for (a, b), sc in zip(ranges, part_scores):
                idx, val = orc.topk_candidates(sc, K)
                np.testing.assert_array_equal(idx, orc.topk_indices(sc, K))
                np.testing.assert_array_equal(val, sc[idx])
                parts.append((a, idx, val))
            np.testing.assert_array_equal(orc.merge_candidates(parts, K), orc.topk_indices(whole, K))
    # ties across parts go to the lower global index
    parts = [(0, np.array([1, 2]), np.array([0.5, 0.3])), (10, np.array([0, 4]), np.array([0.5, 0.5]))]
    np.testing.assert_array_equal(orc.merge_candidates(parts, 2), [1, 10])
    np.testing.assert_array_equal(orc.merge_candidates(parts, 3), [1, 10, 14])


ALL_CHECKS = [
    check_golden_attention, check_golden_verify, check_golden_draft_round, check_append_offsets,
    check_attention_vs_sdpa,
    check_attention_closed_forms, check_golden_selection, check_golden_selection_causal,
    check_selection_invariants, check_selection_causal,
    check_selection_prefix, check_streaming_and_gather,
    check_topk_bruteforce, check_topk_special, check_full_k_sparse_equals_dense,
    check_golden_accept, check_accept_bruteforce, check_commit, check_round_lossless_extremes,
    check_golden_partials, check_range_partials_vs_torch, check_split_selection,
]
