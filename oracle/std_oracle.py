"""fp64 CPU oracle of the Sparse-to-Dense (StD) decoding hot path.

TEST INFRASTRUCTURE.  Only the test-suite, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
module.  It shares no code with the CUDA library and the library never calls
it.

Every function is the plain definition of one step, in float64, written from
the method as the pages state it:

  [P-M2] Sparse-to-Dense summary (gist.science, de/fr/ar), "Methodik" item 2:
         the sparse model M_s attends only to the top-K KV entries chosen by
         text-to-visual attention weight; the dense model M uses the full KV
         cache with standard attention.  Same weights in both modes.
  [P-M3] same page, "Methodik" item 3 (decoding procedure): M_s drafts gamma
         tokens autoregressively; M verifies all of them in parallel in one
         pass over the full cache; the longest prefix matching M's predictions
         (n tokens) is kept plus one bonus token; the accepted tokens are
         appended to the context.
  [P-M4] same page, "Methodik" item 4 (KV-cache selection): top-K visual KV
         chosen once at prefill from the attention scores from text tokens to
         visual tokens, averaged; the choice differs per layer and head.
  [P-A]  Sparse-to-Dense abstract (khansong-paper-with-me.hf.space): sparse
         top-K attention module + dense full-attention module, lossless.

Readings of points the pages leave open (each also listed in the design notes):
  * softmax of the selection score runs over the visual keys only;
  * one index set per (layer, KV head), averaging over the G query heads of
    the group (query head hq uses KV head hq // G);
  * the logit scale is 1/sqrt(d); the score is the mean (not the sum);
  * ties in top-K go to the lower position; indices are returned ascending;
  * the sparse cache is [K selected visual rows | T text rows | generated rows];
  * verify row i (0..gamma) sees the committed context plus new rows <= i;
  * the bonus token is the dense prediction at the first mismatch;
  * accepted rows are copied from the full cache into the sparse tail.

Array conventions match the library: caches [L][B][Hkv][cap][d], queries
[L][B][Hq][rows][d], outputs [L][B][Hq][rows][d].
"""
from __future__ import annotations

import math
from typing import Tuple

import numpy as np

# query rows per matmul while forming the selection score; only bounds memory,
# the score is still the plain mean of the per-row softmax distributions.
_ROW_CHUNK = 64


def softmax(x: np.ndarray) -> np.ndarray:
    """Softmax along the last axis, max-subtracted, fp64."""
    x = np.asarray(x, dtype=np.float64)
    m = x.max(axis=-1, keepdims=True)
    e = np.exp(x - m)
    return e / e.sum(axis=-1, keepdims=True)


# --------------------------------------------------------------------------- selection [P-M4]

def selection_scores(q_text: np.ndarray, k_vis: np.ndarray) -> np.ndarray:
    """Mean text-to-visual attention of one (layer, KV head).

    q_text: [G, T, d] text queries of the G query heads sharing the KV head.
    k_vis:  [Nv, d] visual keys.
    Returns score[n] = mean over (g, t) of softmax_n(q[g, t] . k_n / sqrt(d)), fp64.
    """
    q = np.asarray(q_text, np.float64).reshape(-1, q_text.shape[-1])
    k = np.asarray(k_vis, np.float64)
    scale = 1.0 / math.sqrt(q.shape[-1])
    total = np.zeros(k.shape[0], np.float64)
    for r0 in range(0, q.shape[0], _ROW_CHUNK):
        p = softmax(scale * (q[r0:r0 + _ROW_CHUNK] @ k.T))
        total += p.sum(axis=0)
    return total / q.shape[0]


def selection_scores_causal(q_text: np.ndarray, k_vis: np.ndarray, k_text: np.ndarray,
                            k_prefix: np.ndarray = None) -> np.ndarray:
    """The causal full-row reading of the selection score [P-M4] (the pages do not say
    which keys the text queries' softmax runs over; this variant lets each text query see
    what it sees in the prompt's causal attention: every visual key and the text keys up to
    its own position).

    q_text: [G, T, d]; k_vis: [Nv, d]; k_text: [T, d], the text keys of the prompt;
    k_prefix: [P, d], keys of a prompt prefix before the video (a system prompt), or None.
    Row (g, t) takes the softmax over [k_prefix; k_vis; k_text[0..t]] of q[g, t] . k / sqrt(d);
    score[n] = mean over (g, t) of that row's probability at visual key n, fp64.
    The scores sum to 1 minus the mean probability mass the rows put on other keys.
    """
    q = np.asarray(q_text, np.float64)
    kv = np.asarray(k_vis, np.float64)
    kt = np.asarray(k_text, np.float64)
    kp = np.zeros((0, kv.shape[1])) if k_prefix is None else np.asarray(k_prefix, np.float64)
    G, T, d = q.shape
    P, nv = kp.shape[0], kv.shape[0]
    scale = 1.0 / math.sqrt(d)
    total = np.zeros(nv, np.float64)
    for g in range(G):
        for t in range(T):
            keys = np.concatenate([kp, kv, kt[:t + 1]], axis=0)
            total += softmax(scale * (keys @ q[g, t]))[P:P + nv]
    return total / (G * T)


def topk_indices(scores: np.ndarray, K: int) -> np.ndarray:
    """The K highest scores' positions, ties to the lower position, ascending. int32."""
    s = np.asarray(scores)
    n = s.shape[0]
    if not 0 <= K <= n:
        raise ValueError("K out of range")
    order = np.lexsort((np.arange(n), -s))   # primary: score descending; then position ascending
    return np.sort(order[:K]).astype(np.int32)


def select_topk(q_text: np.ndarray, k_full: np.ndarray, v_full: np.ndarray, nvis: np.ndarray,
                T: int, K: int, cap_sparse: int, causal_text: bool = False, n_prefix: int = 0):
    """Prefill selection for every (layer, batch, KV head) [P-M4], [P-M2].

    causal_text: score with selection_scores_causal (text keys join each row's softmax)
    instead of selection_scores (visual keys only).
    n_prefix: rows of a prompt prefix (a system prompt) before the visual block; the
    cache is then [prefix | visual | text], the indices stay positions within the visual
    block, and the sparse cache is [prefix | K selected visual | text] (length
    n_prefix + K + T).  With causal_text the prefix keys join every text row's softmax.

    q_text [L][B][Hq][T][d]; k_full, v_full [L][B][Hkv][cap_full][d] (visual rows
    [0, nvis_b), text rows [nvis_b, nvis_b + T)).  Returns
      idx      [L][B][Hkv][K] int32, ascending visual positions;
      scores   [L][B][Hkv][max nvis] fp64 (0 beyond nvis_b);
      k_sparse, v_sparse [L][B][Hkv][cap_sparse][d]: rows [0, K) the selected
               visual rows in ascending position, rows [K, K + T) the text rows;
      len_sparse [B] int32 = K + T.
    """
    L, B, Hq = q_text.shape[:3]
    Hkv, d = k_full.shape[2], k_full.shape[4]
    G = Hq // Hkv
    nmax = int(np.max(nvis))
    idx = np.zeros((L, B, Hkv, K), np.int32)
    scores = np.zeros((L, B, Hkv, nmax), np.float64)
    k_sp = np.zeros((L, B, Hkv, cap_sparse, d), np.float64)
    v_sp = np.zeros((L, B, Hkv, cap_sparse, d), np.float64)
    for l in range(L):
        for b in range(B):
            nv = int(nvis[b])
            for h in range(Hkv):
                qh = q_text[l, b, h * G:(h + 1) * G]
                P = n_prefix
                kvis = k_full[l, b, h, P:P + nv]
                if causal_text:
                    s = selection_scores_causal(qh, kvis, k_full[l, b, h, P + nv:P + nv + T], k_full[l, b, h, :P])
                else:
                    s = selection_scores(qh, kvis)
                scores[l, b, h, :nv] = s
                idx[l, b, h] = topk_indices(s, K)
    k_sp, v_sp, lsp = gather_sparse(k_full, v_full, nvis, idx, T, cap_sparse, n_prefix)
    return idx, scores, k_sp, v_sp, lsp


# --------------------------------------------------------------------------- selection over parts [P-M4]
#
# The selection score of [P-M4] for a cache split by position into parts (one per GPU).
# Each text row's softmax over all visual keys is exp(x_n - m) / l with m the row's
# maximum and l its sum of exp(x_n - m); a part can form its rows' (m, l) over its own
# keys, the parts' pairs give the whole row's, and each part then scores its own keys
# with the whole row's (m, l).  The global top-K keys are each among their own part's
# top-K, so the top-K of the parts' candidates is the selection.

def selection_rowstats(q_text: np.ndarray, k_vis: np.ndarray) -> Tuple[np.ndarray, np.ndarray]:
    """Per text row of one (layer, KV head) over the given visual keys: m[r] = max_n
    x_rn and l[r] = sum_n exp(x_rn - m[r]), x = q . k / sqrt(d).  q_text [G, T, d],
    k_vis [n, d]; returns (m, l), each [G * T], fp64."""
    q = np.asarray(q_text, np.float64).reshape(-1, q_text.shape[-1])
    x = (q @ np.asarray(k_vis, np.float64).T) / math.sqrt(q.shape[-1])
    m = x.max(axis=1)
    return m, np.exp(x - m[:, None]).sum(axis=1)


def merge_rowstats(ms, ls) -> Tuple[np.ndarray, np.ndarray]:
    """(m, l) over the union of the parts' keys from each part's (m_i, l_i): m = max_i m_i,
    l = sum_i l_i exp(m_i - m)."""
    ms = np.asarray(ms, np.float64)
    ls = np.asarray(ls, np.float64)
    m = ms.max(axis=0)
    return m, (ls * np.exp(ms - m)).sum(axis=0)


def selection_scores_given_rowstats(q_text: np.ndarray, k_vis: np.ndarray, m: np.ndarray,
                                    l: np.ndarray) -> np.ndarray:
    """The selection score of the given keys when (m, l) are the whole rows' statistics:
    score[n] = mean over rows r of exp(x_rn - m[r]) / l[r].  With (m, l) over exactly these
    keys this is selection_scores."""
    q = np.asarray(q_text, np.float64).reshape(-1, q_text.shape[-1])
    x = (q @ np.asarray(k_vis, np.float64).T) / math.sqrt(q.shape[-1])
    return (np.exp(x - m[:, None]) / l[:, None]).mean(axis=0)


def topk_candidates(scores: np.ndarray, K: int) -> Tuple[np.ndarray, np.ndarray]:
    """A part's candidates: its K highest scores' positions (ties to the lower position,
    ascending) and those scores."""
    idx = topk_indices(scores, K)
    return idx, np.asarray(scores)[idx]


def merge_candidates(parts, K: int) -> np.ndarray:
    """The top-K of the parts' candidates.  parts: (offset, idx, score) per part, offset the
    global index of the part's first key; returns the K highest candidates' global indices,
    ties to the lower global index, ascending.  int32."""
    gidx = np.concatenate([np.asarray(i, np.int64) + off for off, i, _ in parts])
    sc = np.concatenate([np.asarray(v, np.float64) for _, _, v in parts])
    order = np.lexsort((gidx, -sc))   # primary: score descending; then global index ascending
    return np.sort(gidx[order[:K]]).astype(np.int32)


# --------------------------------------------------------------------------- streaming draft baseline

def streaming_indices(nv: int, K: int, n_sink: int) -> np.ndarray:
    """Index set of the "Streaming" draft baseline (gist.science summary, "Experimentelle
    Ergebnisse", item "Vergleich": a baseline that drafts with streaming attention; no
    detail printed).  Read as attention sinks plus a recent window: the first n_sink
    visual positions and the last K - n_sink, ascending.  int32."""
    if not (0 <= n_sink <= K <= nv):
        raise ValueError("need 0 <= n_sink <= K <= nv")
    return np.concatenate([np.arange(n_sink), np.arange(nv - (K - n_sink), nv)]).astype(np.int32)


def gather_sparse(k_full: np.ndarray, v_full: np.ndarray, nvis: np.ndarray, idx: np.ndarray, T: int,
                  cap_sparse: int, n_prefix: int = 0):
    """Sparse cache from given indices [P-M2].  The full cache holds [P prefix rows |
    nvis_b visual rows | T text rows] with P = n_prefix; the sparse cache gets the P
    prefix rows, then the visual rows P + idx[l, b, h, j] in the given order, then the
    text rows.  Returns (k_sparse, v_sparse [L][B][Hkv][cap_sparse][d],
    len_sparse [B] = P + K + T)."""
    L, B, Hkv, K = idx.shape
    d = k_full.shape[4]
    P = n_prefix
    k_sp = np.zeros((L, B, Hkv, cap_sparse, d), np.float64)
    v_sp = np.zeros((L, B, Hkv, cap_sparse, d), np.float64)
    for l in range(L):
        for b in range(B):
            nv = int(nvis[b])
            for h in range(Hkv):
                for dst, src in ((k_sp, k_full), (v_sp, v_full)):
                    dst[l, b, h, :P] = src[l, b, h, :P]
                    dst[l, b, h, P:P + K] = src[l, b, h, P + idx[l, b, h]]
                    dst[l, b, h, P + K:P + K + T] = src[l, b, h, P + nv:P + nv + T]
    return k_sp, v_sp, np.full(B, P + K + T, np.int32)


# --------------------------------------------------------------------------- attention [P-M2]

def attend(q: np.ndarray, k: np.ndarray, v: np.ndarray) -> np.ndarray:
    """softmax(k . q / sqrt(d)) @ v for one query q [d] over rows k, v [n, d]."""
    q = np.asarray(q, np.float64)
    w = softmax((np.asarray(k, np.float64) @ q) / math.sqrt(q.shape[-1]))
    return w @ np.asarray(v, np.float64)


def sparse_decode_attn(q: np.ndarray, k_sp: np.ndarray, v_sp: np.ndarray,
                       length: np.ndarray) -> np.ndarray:
    """Sparse draft attention [P-M2]: each query row attends to sparse rows j < length[b].

    q [L][B][Hq][rows][d] (rows = 1 in decoding); caches [L][B][Hkv][cap][d].
    """
    L, B, Hq, rows, d = q.shape
    G = Hq // k_sp.shape[2]
    o = np.zeros(q.shape, np.float64)
    for l in range(L):
        for b in range(B):
            n = int(length[b])
            for hq in range(Hq):
                h = hq // G
                for r in range(rows):
                    o[l, b, hq, r] = attend(q[l, b, hq, r], k_sp[l, b, h, :n], v_sp[l, b, h, :n])
    return o


def dense_verify_attn(q: np.ndarray, k_full: np.ndarray, v_full: np.ndarray,
                      n_ctx: np.ndarray) -> np.ndarray:
    """Dense verify attention [P-M3]: row i of gamma + 1 attends full rows j < n_ctx[b] + i + 1.

    q [L][B][Hq][gamma + 1][d]; n_ctx = committed context length before the
    gamma + 1 new rows, which sit at [n_ctx, n_ctx + gamma + 1) in the cache.
    """
    L, B, Hq, rows, d = q.shape
    G = Hq // k_full.shape[2]
    o = np.zeros(q.shape, np.float64)
    for l in range(L):
        for b in range(B):
            for hq in range(Hq):
                h = hq // G
                for i in range(rows):
                    n = int(n_ctx[b]) + i + 1
                    o[l, b, hq, i] = attend(q[l, b, hq, i], k_full[l, b, h, :n], v_full[l, b, h, :n])
    return o


# --------------------------------------------------------------------------- attention over key ranges

def attend_partial(q: np.ndarray, k: np.ndarray, v: np.ndarray):
    """Attention of one query q [d] restricted to the rows k, v [n, d], left unnormalised
    so that ranges of one key sequence can be combined later (the cache split by position
    over several devices; the pages keep the whole cache on one GPU, "Bedeutung", so this
    is the plain decomposition of the softmax, not a step the pages describe).

    With logits s_j = q . k_j / sqrt(d): m = max_j s_j, l = sum_j exp(s_j - m),
    o = sum_j exp(s_j - m) v_j.  An empty range gives (o = 0, m = -inf, l = 0).
    Returns (o [d], m, l), fp64; attend(q, k, v) = o / l.
    """
    q = np.asarray(q, np.float64)
    if k.shape[0] == 0:
        return np.zeros(q.shape[-1]), -math.inf, 0.0
    s = (np.asarray(k, np.float64) @ q) / math.sqrt(q.shape[-1])
    m = float(s.max())
    e = np.exp(s - m)
    return e @ np.asarray(v, np.float64), m, float(e.sum())


def merge_partials(o: np.ndarray, m: np.ndarray, l: np.ndarray) -> np.ndarray:
    """Combine partials (o_k, m_k, l_k), k over the first axis, of disjoint key ranges:
    M = max_k m_k, weights w_k = exp(m_k - M), result sum_k w_k o_k / sum_k w_k l_k
    (0 where no range holds a key).  o [n_parts][..., d], m and l [n_parts][...]."""
    o = np.asarray(o, np.float64)
    m = np.asarray(m, np.float64)
    l = np.asarray(l, np.float64)
    M = m.max(axis=0)
    ref = np.where(np.isfinite(M), M, 0.0)
    w = np.exp(m - ref)                                    # exp(-inf) = 0 for empty ranges
    L = (w * l).sum(axis=0)
    O = (w[..., None] * o).sum(axis=0)
    out = np.zeros(O.shape)
    nz = L > 0
    out[nz] = O[nz] / L[nz][..., None]
    return out


def attn_range_partial(q: np.ndarray, k: np.ndarray, v: np.ndarray, limit: np.ndarray, pos0: int,
                       row_begin: int, row_end: int):
    """Partials of decode attention over one range of cache rows [P-M2], [P-M3].

    q [L][B][Hq][rows][d]; k, v [L][B][Hkv][cap][d] whose row r holds sequence position
    pos0 + r; limit [B]: query row i of sequence b attends positions j < limit[b] + i
    (limit = n_ctx + 1 for the dense verify, the sparse length for the draft).  Row i
    attends cache rows r in [row_begin, row_end) with pos0 + r < limit[b] + i.
    Returns (o [L][B][Hq][rows][d], m [L][B][Hq][rows], l [L][B][Hq][rows]) as attend_partial.
    """
    L, B, Hq, rows, d = q.shape
    G = Hq // k.shape[2]
    o = np.zeros(q.shape, np.float64)
    m = np.full(q.shape[:4], -math.inf)
    l = np.zeros(q.shape[:4])
    for li in range(L):
        for b in range(B):
            for hq in range(Hq):
                h = hq // G
                for i in range(rows):
                    hi = min(row_end, int(limit[b]) + i - pos0)
                    lo = row_begin
                    kk = k[li, b, h, lo:max(lo, hi)]
                    vv = v[li, b, h, lo:max(lo, hi)]
                    o[li, b, hq, i], m[li, b, hq, i], l[li, b, hq, i] = attend_partial(q[li, b, hq, i], kk, vv)
    return o, m, l


# --------------------------------------------------------------------------- acceptance [P-M3]

def accept_prefix(draft: np.ndarray, dense: np.ndarray) -> Tuple[np.ndarray, np.ndarray]:
    """Greedy acceptance: n = leading positions where draft == dense; keep n + 1 tokens.

    draft [B][gamma], dense [B][gamma + 1] (dense prediction after each input).
    Returns n_plus_1 [B] int32 and accepted [B][gamma + 1] int32 = dense[b][0..n],
    -1 after that.
    """
    draft = np.asarray(draft)
    dense = np.asarray(dense)
    B, gamma = draft.shape
    n_plus_1 = np.zeros(B, np.int32)
    acc = np.full((B, gamma + 1), -1, np.int32)
    for b in range(B):
        n = 0
        while n < gamma and draft[b, n] == dense[b, n]:
            n += 1
        n_plus_1[b] = n + 1
        acc[b, :n + 1] = dense[b, :n + 1]
    return n_plus_1, acc


# --------------------------------------------------------------------------- cache bookkeeping [P-M3]

def kv_append(cache: np.ndarray, length: np.ndarray, offset: int, rows: np.ndarray) -> None:
    """Write rows [L][B][Hkv][n][d] at positions length[b] + offset + r (in place)."""
    n = rows.shape[3]
    for b in range(cache.shape[1]):
        p = int(length[b]) + offset
        cache[:, b, :, p:p + n] = rows[:, b]


def kv_commit(k_full, v_full, k_sp, v_sp, len_full, len_sp, n_plus_1) -> None:
    """Append the accepted inputs to the context (in place).

    The n + 1 verified rows at full positions [len_full, len_full + n + 1) are
    copied to sparse positions [len_sp, len_sp + n + 1); both lengths grow by n + 1.
    """
    for b in range(k_full.shape[1]):
        a, s, n = int(len_full[b]), int(len_sp[b]), int(n_plus_1[b])
        k_sp[:, b, :, s:s + n] = k_full[:, b, :, a:a + n]
        v_sp[:, b, :, s:s + n] = v_full[:, b, :, a:a + n]
        len_full[b] += n
        len_sp[b] += n


def decode_round(state: dict, q_draft, k_draft, v_draft, q_verify, k_verify, v_verify,
                 draft_tokens, dense_tokens) -> dict:
    """One draft + verify round [P-M3], updating `state` in place.

    state: k_full, v_full, k_sp, v_sp (fp64 caches), len_full, len_sp ([B] int).
    q_draft [gamma][L][B][Hq][1][d], k_draft/v_draft [gamma][L][B][Hkv][1][d],
    q_verify [L][B][Hq][gamma+1][d], k_verify/v_verify [L][B][Hkv][gamma+1][d],
    draft_tokens [B][gamma], dense_tokens [B][gamma+1].
    Draft step j appends its input row to the sparse cache and attends over the
    committed sparse rows plus the j + 1 new ones; verify appends gamma + 1 rows
    to the full cache and attends causally; then accept and commit.
    """
    gamma = q_draft.shape[0]
    o_draft = []
    for j in range(gamma):
        kv_append(state["k_sp"], state["len_sp"], j, k_draft[j])
        kv_append(state["v_sp"], state["len_sp"], j, v_draft[j])
        o_draft.append(sparse_decode_attn(q_draft[j], state["k_sp"], state["v_sp"],
                                          state["len_sp"] + j + 1))
    kv_append(state["k_full"], state["len_full"], 0, k_verify)
    kv_append(state["v_full"], state["len_full"], 0, v_verify)
    o_verify = dense_verify_attn(q_verify, state["k_full"], state["v_full"], state["len_full"])
    n_plus_1, acc = accept_prefix(draft_tokens, dense_tokens)
    kv_commit(state["k_full"], state["v_full"], state["k_sp"], state["v_sp"],
              state["len_full"], state["len_sp"], n_plus_1)
    o_draft = np.stack(o_draft) if o_draft else np.zeros((0,) + q_draft.shape[1:])
    return {"o_draft": o_draft, "o_verify": o_verify, "n_plus_1": n_plus_1, "accepted": acc}
