"""The pins catch plausible mistakes: each test breaks one step of a copy of the
oracle (on the CPU) and expects at least one pin to fail."""
import math
import types

import numpy as np
import pytest

import oracle
from oracle import std_oracle as so
from tests import pins


def _mutant(**overrides):
    ns = types.SimpleNamespace(**{k: getattr(so, k) for k in dir(so) if not k.startswith("__")})
    for k, v in overrides.items():
        setattr(ns, k, v)
    return ns


def _attend_scale_1_over_d(q, k, v):
    w = so.softmax((np.asarray(k, np.float64) @ q) / q.shape[-1])
    return w @ v


def _scores_sum_not_mean(q_text, k_vis):
    return so.selection_scores(q_text, k_vis) * (q_text.shape[0] * q_text.shape[1])


def _select_interleaved_groups(q_text, k_full, v_full, nvis, T, K, cap_sparse, causal_text=False, n_prefix=0):
    L, B, Hq = q_text.shape[:3]
    Hkv = k_full.shape[2]
    res = so.select_topk(q_text, k_full, v_full, nvis, T, K, cap_sparse, causal_text, n_prefix)
    idx, scores = res[0].copy(), res[1].copy()
    for h in range(Hkv):
        q = q_text[0, 0, h::Hkv]                               # hq % Hkv grouping
        s = so.selection_scores(q, k_full[0, 0, h, n_prefix:n_prefix + int(nvis[0])])
        scores[0, 0, h, :len(s)] = s
        idx[0, 0, h] = so.topk_indices(s, K)
    return (idx, scores) + tuple(res[2:])



def _causal_text_off_by_one(q_text, k_vis, k_text):
    # row t sees text keys 0..t-1 only (row 0 sees none)
    q = np.asarray(q_text, np.float64)
    G, T, d = q.shape
    total = np.zeros(k_vis.shape[0])
    for g in range(G):
        for t in range(T):
            keys = np.concatenate([k_vis, k_text[:t]], axis=0)
            total += oracle.softmax(keys @ q[g, t] / math.sqrt(d))[:k_vis.shape[0]]
    return total / (G * T)


def _topk_ties_high(scores, K):
    s = np.asarray(scores)
    order = np.lexsort((-np.arange(len(s)), -s))
    return np.sort(order[:K]).astype(np.int32)


def _verify_off_by_one(q, k_full, v_full, n_ctx):
    return so.dense_verify_attn(q, k_full, v_full, np.asarray(n_ctx) - 1)


def _accept_count_all(draft, dense):
    B, gamma = draft.shape
    n1 = np.zeros(B, np.int32)
    acc = np.full((B, gamma + 1), -1, np.int32)
    for b in range(B):
        n = int((draft[b] == dense[b, :gamma]).sum())
        n1[b] = n + 1
        acc[b, :n + 1] = dense[b, :n + 1]
    return n1, acc


def _accept_bonus_from_draft(draft, dense):
    n1, acc = so.accept_prefix(draft, dense)
    for b in range(draft.shape[0]):
        n = int(n1[b]) - 1
        if n < draft.shape[1]:
            acc[b, n] = draft[b, n]
    return n1, acc


def _commit_shifted(k_full, v_full, k_sp, v_sp, len_full, len_sp, n_plus_1):
    for b in range(k_full.shape[1]):
        a, s, n = int(len_full[b]) + 1, int(len_sp[b]), int(n_plus_1[b])
        k_sp[:, b, :, s:s + n] = k_full[:, b, :, a:a + n]
        v_sp[:, b, :, s:s + n] = v_full[:, b, :, a:a + n]
        len_full[b] += n
        len_sp[b] += n


MUTANTS = {
    "attention scale 1/d": _mutant(attend=_attend_scale_1_over_d),
    "selection sum not mean": _mutant(selection_scores=_scores_sum_not_mean),
    "causal text mask off by one": _mutant(selection_scores_causal=_causal_text_off_by_one),
    "causal variant ignores text keys": _mutant(selection_scores_causal=lambda q, kv, kt: oracle.selection_scores(q, kv)),
    "GQA grouping hq % Hkv": _mutant(select_topk=_select_interleaved_groups),
    "top-K ties to higher position": _mutant(topk_indices=_topk_ties_high),
    "verify mask off by one": _mutant(dense_verify_attn=_verify_off_by_one),
    "accept counts all matches": _mutant(accept_prefix=_accept_count_all),
    "bonus token from the draft": _mutant(accept_prefix=_accept_bonus_from_draft),
    "commit window shifted": _mutant(kv_commit=_commit_shifted),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(name):
    orc = MUTANTS[name]
    failed = []
    for check in pins.ALL_CHECKS:
        try:
            check(orc)
        except AssertionError:
            failed.append(check.__name__)
    assert failed, f"no pin caught the mutant: {name}"


def test_unmutated_copy_passes():
    orc = _mutant()
    for check in pins.ALL_CHECKS:
        check(orc)
