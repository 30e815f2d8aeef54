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


def _streaming_window_early(nv, K, n_sink):
    # the recent window ends one position before the last visual row
    return np.concatenate([np.arange(n_sink), np.arange(nv - (K - n_sink) - 1, nv - 1)]).astype(np.int32)


def _gather_prefix_after_selected(k_full, v_full, nvis, idx, T, cap_sparse, n_prefix=0):
    k_sp, v_sp, lsp = so.gather_sparse(k_full, v_full, nvis, idx, T, cap_sparse, n_prefix)
    K, P = idx.shape[3], n_prefix
    for t in (k_sp, v_sp):
        t[..., :P + K, :] = np.concatenate([t[..., P:P + K, :], t[..., :P, :]], axis=-2)
    return k_sp, v_sp, lsp


def _gather_text_at_nvis_max(k_full, v_full, nvis, idx, T, cap_sparse, n_prefix=0):
    nmax = np.full_like(np.asarray(nvis), int(np.max(nvis)))
    k_sp, v_sp, _ = so.gather_sparse(k_full, v_full, nmax, idx, T, cap_sparse, n_prefix)
    return k_sp, v_sp, np.full(idx.shape[1], n_prefix + idx.shape[3] + T, np.int32)


def _select_prefix_in_softmax(q_text, k_full, v_full, nvis, T, K, cap_sparse, causal_text=False, n_prefix=0):
    # the default score's softmax also covers the prompt prefix keys
    res = so.select_topk(q_text, k_full, v_full, nvis, T, K, cap_sparse, causal_text, n_prefix)
    if n_prefix == 0 or causal_text:
        return res
    L, B, Hq = q_text.shape[:3]
    Hkv = k_full.shape[2]
    G = Hq // Hkv
    idx, scores = res[0].copy(), res[1].copy()
    for l in range(L):
        for b in range(B):
            nv = int(nvis[b])
            for h in range(Hkv):
                s = so.selection_scores(q_text[l, b, h * G:(h + 1) * G], k_full[l, b, h, :n_prefix + nv])[n_prefix:]
                scores[l, b, h, :nv] = s
                idx[l, b, h] = so.topk_indices(s, K)
    k_sp, v_sp, lsp = so.gather_sparse(k_full, v_full, nvis, idx, T, cap_sparse, n_prefix)
    return idx, scores, k_sp, v_sp, lsp


def _sparse_attn_one_row_short(q, k_sp, v_sp, length):
    return so.sparse_decode_attn(q, k_sp, v_sp, np.asarray(length) - 1)


def _verify_sees_next_row(q, k_full, v_full, n_ctx):
    return so.dense_verify_attn(q, k_full, v_full, np.asarray(n_ctx) + 1)


def _round_with_draft(append_offset, attended):
    """decode_round with the draft leg changed: step j appends at len_sp + append_offset(j)
    and attends over len_sp + attended(j) rows; verify, accept and commit unchanged."""
    def decode_round(state, q_draft, k_draft, v_draft, q_verify, k_verify, v_verify, draft_tokens, dense_tokens):
        o_draft = []
        for j in range(q_draft.shape[0]):
            so.kv_append(state["k_sp"], state["len_sp"], append_offset(j), k_draft[j])
            so.kv_append(state["v_sp"], state["len_sp"], append_offset(j), v_draft[j])
            o_draft.append(so.sparse_decode_attn(q_draft[j], state["k_sp"], state["v_sp"],
                                                 state["len_sp"] + attended(j)))
        so.kv_append(state["k_full"], state["len_full"], 0, k_verify)
        so.kv_append(state["v_full"], state["len_full"], 0, v_verify)
        o_verify = so.dense_verify_attn(q_verify, state["k_full"], state["v_full"], state["len_full"])
        n_plus_1, acc = so.accept_prefix(draft_tokens, dense_tokens)
        so.kv_commit(state["k_full"], state["v_full"], state["k_sp"], state["v_sp"], state["len_full"],
                     state["len_sp"], n_plus_1)
        return {"o_draft": np.stack(o_draft), "o_verify": o_verify, "n_plus_1": n_plus_1, "accepted": acc}
    return decode_round


def _append_offset_ignored(cache, length, offset, rows):
    so.kv_append(cache, length, 0, rows)


def _merge_without_rescale(o, m, l):
    o, l = np.asarray(o, np.float64), np.asarray(l, np.float64)
    L = l.sum(axis=0)
    return np.where(L[..., None] > 0, o.sum(axis=0) / np.where(L > 0, L, 1.0)[..., None], 0.0)


def _partial_normalised(q, k, v):
    o, m, l = so.attend_partial(q, k, v)
    return (o / l if l > 0 else o), m, l


def _range_end_inclusive(q, k, v, limit, pos0, row_begin, row_end):
    return so.attn_range_partial(q, k, v, limit, pos0, row_begin, row_end + 1)


def _range_ignores_pos0(q, k, v, limit, pos0, row_begin, row_end):
    return so.attn_range_partial(q, k, v, limit, 0, row_begin, row_end)


def _merge_rowstats_no_rescale(ms, ls):
    return np.max(ms, axis=0), np.sum(ls, axis=0)


def _part_scores_own_stats(q_text, k_vis, m, l):
    return so.selection_scores(q_text, k_vis)


def _merge_candidates_ties_high(parts, K):
    gidx = np.concatenate([np.asarray(i, np.int64) + off for off, i, _ in parts])
    sc = np.concatenate([np.asarray(v, np.float64) for _, _, v in parts])
    order = np.lexsort((-gidx, -sc))
    return np.sort(gidx[order[:K]]).astype(np.int32)


def _merge_candidates_local_idx(parts, K):
    return so.merge_candidates([(0, i, v) for _, i, v in parts], K)


MUTANTS = {
    "merge without the exp(m_k - M) rescale": _mutant(merge_partials=_merge_without_rescale),
    "partial returns the normalised output": _mutant(attend_partial=_partial_normalised),
    "key range end inclusive": _mutant(attn_range_partial=_range_end_inclusive),
    "key range ignores the shard's first position": _mutant(attn_range_partial=_range_ignores_pos0),
    "draft appends at offset 0 every step": _mutant(decode_round=_round_with_draft(lambda j: 0, lambda j: j + 1)),
    "draft step attends len_sp + j rows": _mutant(decode_round=_round_with_draft(lambda j: j, lambda j: j)),
    "draft step attends one row past its own": _mutant(decode_round=_round_with_draft(lambda j: j, lambda j: j + 2)),
    "append ignores the offset": _mutant(kv_append=_append_offset_ignored),
    "streaming window ends one row early": _mutant(streaming_indices=_streaming_window_early),
    "gather puts the prefix after the selected rows": _mutant(gather_sparse=_gather_prefix_after_selected),
    "gather reads text rows at the longest visual length": _mutant(gather_sparse=_gather_text_at_nvis_max),
    "default score's softmax covers the prefix keys": _mutant(select_topk=_select_prefix_in_softmax),
    "sparse attention one row short": _mutant(sparse_decode_attn=_sparse_attn_one_row_short),
    "verify row sees the next row": _mutant(dense_verify_attn=_verify_sees_next_row),
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
    "row statistics merged without the exp(m_i - m) rescale": _mutant(merge_rowstats=_merge_rowstats_no_rescale),
    "part scores use the part's own row statistics": _mutant(selection_scores_given_rowstats=_part_scores_own_stats),
    "candidate merge ties to the higher index": _mutant(merge_candidates=_merge_candidates_ties_high),
    "candidate merge ignores the part offsets": _mutant(merge_candidates=_merge_candidates_local_idx),
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
