"""A tiny random-weight attention-only language model for the losslessness test.

Sparse-to-Dense claims that its output is identical to the dense model's greedy
output (gist.science summary, "Methodik" item 3 and "Hauptbeiträge"; "lossless"
in the abstract): the sparse mode only proposes tokens, and every kept token is
the dense model's own prediction.  This module runs the whole loop on a toy
model, so that the claim is checked with real draft tokens (the sparse model's
own argmax) instead of synthetic token streams:

* ``ToyLM``: token and position embeddings, L layers of grouped-query attention
  with residual connections, an LM head; random weights.  Q/K/V are rounded to
  bf16 (the storage type of the library's caches) before attention.
* ``prefill``: the causal prompt pass in plain torch fp32 (test infrastructure,
  not a library step) -> full K/V cache, text queries, first token.
* ``std_decode``: Sparse-to-Dense decoding through the C ABI -- selection, per
  layer sparse draft attention, one batched dense verify, acceptance, commit.
* ``dense_decode_gpu``: plain greedy decoding with the library's dense
  attention, one query per step.
* ``dense_decode_f64``: the same greedy decoding in numpy float64, on the
  oracle's attention.

The projections and the LM head are torch matmuls: the language-model layers
around attention are not part of the library.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np
import torch

import oracle
import synth


@dataclass(frozen=True)
class ToyConfig:
    vocab: int = 256
    dm: int = 256
    L: int = 2
    Hq: int = 4
    Hkv: int = 2
    d: int = 64
    nvis: int = 2048
    T: int = 32
    q_scale: float = 2.0      # scale of Wq, Wk: how peaked attention is
    vis_scale: float = 0.5    # scale of the visual embeddings
    pos_scale: float = 0.5    # scale of the position embeddings
    logit_scale: float = 4.0
    max_pos: int = 4096


class ToyLM:
    """Random weights (float64 masters; fp32 copies on the GPU), fixed by `seed`."""

    def __init__(self, cfg: ToyConfig, seed: int = 0):
        c = self.cfg = cfg
        g = torch.Generator().manual_seed(seed)
        r = lambda *s: torch.randn(*s, generator=g, dtype=torch.float64)  # noqa: E731
        self.G = c.Hq // c.Hkv
        self.E = r(c.vocab, c.dm)
        self.Wq = r(c.L, c.dm, c.Hq * c.d) / math.sqrt(c.dm) * c.q_scale
        self.Wk = r(c.L, c.dm, c.Hkv * c.d) / math.sqrt(c.dm) * c.q_scale
        self.Wv = r(c.L, c.dm, c.Hkv * c.d) / math.sqrt(c.dm)
        self.Wo = r(c.L, c.Hq * c.d, c.dm) / math.sqrt(c.Hq * c.d)
        self.Wlm = r(c.dm, c.vocab) / math.sqrt(c.dm) * c.logit_scale
        self.P = r(c.max_pos, c.dm) * c.pos_scale
        # the prompt: visual embeddings and text tokens
        self.vis = r(c.nvis, c.dm) * c.vis_scale
        self.text = torch.randint(0, c.vocab, (c.T,), generator=g)
        self._dev = None

    def dev(self):
        if self._dev is None:
            names = ("E", "Wq", "Wk", "Wv", "Wo", "Wlm", "P", "vis")
            self._dev = {n: getattr(self, n).float().cuda() for n in names}
            self._dev["text"] = self.text.cuda()
        return self._dev

    def qkv(self, l, x):
        """x [n, dm] fp32 -> q [Hq, n, d], k, v [Hkv, n, d] as contiguous bf16."""
        c, W = self.cfg, self.dev()
        n = x.shape[0]
        q = (x @ W["Wq"][l]).view(n, c.Hq, c.d).transpose(0, 1)
        k = (x @ W["Wk"][l]).view(n, c.Hkv, c.d).transpose(0, 1)
        v = (x @ W["Wv"][l]).view(n, c.Hkv, c.d).transpose(0, 1)
        bf = lambda t: t.to(torch.bfloat16).contiguous()  # noqa: E731
        return bf(q), bf(k), bf(v)

    def embed(self, tokens, pos0):
        W = self.dev()
        t = torch.as_tensor(tokens, device="cuda").reshape(-1)
        return W["E"][t] + W["P"][pos0:pos0 + t.numel()]


# ----------------------------------------------------------------------------- GPU paths

def prefill(m: ToyLM, cap_full: int):
    """Causal prompt pass (torch fp32).

    Returns (k_full, v_full [L][1][Hkv][cap_full][d] bf16, q_text [L][1][Hq][T][d] bf16,
    first generated token).
    """
    c, W = m.cfg, m.dev()
    N = c.nvis + c.T
    x = torch.cat([W["vis"], W["E"][W["text"]]], 0) + W["P"][:N]
    k_full = torch.zeros((c.L, 1, c.Hkv, cap_full, c.d), dtype=torch.bfloat16, device="cuda")
    v_full = torch.zeros_like(k_full)
    q_text = torch.zeros((c.L, 1, c.Hq, c.T, c.d), dtype=torch.bfloat16, device="cuda")
    mask = torch.ones(N, N, dtype=torch.bool, device="cuda").tril()
    for l in range(c.L):
        q, k, v = m.qkv(l, x)
        k_full[l, 0, :, :N] = k
        v_full[l, 0, :, :N] = v
        q_text[l, 0] = q[:, c.nvis:]
        kk = k.float().repeat_interleave(m.G, 0)
        vv = v.float().repeat_interleave(m.G, 0)
        s = (q.float() @ kk.transpose(1, 2)) / math.sqrt(c.d)
        o = torch.softmax(s.masked_fill(~mask, float("-inf")), -1) @ vv      # [Hq, N, d]
        x = x + o.transpose(0, 1).reshape(N, -1) @ W["Wo"][l]
    first = int(torch.argmax(x[-1] @ W["Wlm"]))
    return k_full, v_full, q_text, first


def _attn_layer(B, m, l, x, q_rows, k_cache, v_cache, length, offset, attn):
    """Append layer l's K/V rows of `x` to the cache at length + offset, attend with
    `attn(dims, q, k_layer, v_layer, o)`; returns x + the attention block's output."""
    c, W = m.cfg, m.dev()
    q, k, v = m.qkv(l, x)
    cap = k_cache.shape[3]
    kl, vl = k_cache[l:l + 1], v_cache[l:l + 1]
    d1 = B.dims(1, 1, c.Hq, c.Hkv, c.d, B.STD_BF16, cap, cap)
    B.std_kv_append(d1, kl, vl, cap, length, offset, k[None, None].contiguous(), v[None, None].contiguous(),
                    q_rows)
    o = torch.empty((1, 1, c.Hq, q_rows, c.d), device="cuda")
    attn(d1, q[None, None].contiguous(), kl, vl, o)
    return x + o[0, 0].transpose(0, 1).reshape(q_rows, -1) @ W["Wo"][l]


def dense_decode_gpu(m: ToyLM, k_full, v_full, first: int, n_tokens: int):
    """Greedy decoding, one token per step, dense attention through the library."""
    from sparse_top_kv_std_b200 import binding as B
    c, W = m.cfg, m.dev()
    k_full, v_full = k_full.clone(), v_full.clone()
    cap = k_full.shape[3]
    d1 = B.dims(1, 1, c.Hq, c.Hkv, c.d, B.STD_BF16, cap, cap)
    ws = torch.empty(max(16, B.std_attn_workspace_size(d1, 1, cap, 0)), dtype=torch.uint8, device="cuda")
    ln = torch.tensor([c.nvis + c.T], dtype=torch.int32, device="cuda")
    n_ctx = c.nvis + c.T
    out, tok = [first], first
    while len(out) < n_tokens:
        x = m.embed([tok], n_ctx)
        for l in range(c.L):
            x = _attn_layer(B, m, l, x, 1, k_full, v_full, ln, 0,
                            lambda d, q, kl, vl, o: B.std_dense_verify_attn(d, q, 0, kl, vl, ln, o, 0, ws))
        ln += 1
        n_ctx += 1
        tok = int(torch.argmax(x[0] @ W["Wlm"]))
        out.append(tok)
    assert B.std_get_device_error() == 0
    return out


def std_decode(m: ToyLM, k_full, v_full, q_text, first: int, K: int, gamma: int, n_tokens: int,
               select: str = "topk", n_sink: int = 4):
    """Sparse-to-Dense decoding through the library.  Returns (tokens, n + 1 of every round).

    select: "topk" -- the method's selection (std_select_topk); "stream" -- the streaming
    draft baseline (n_sink attention sinks + the most recent visual positions, through
    std_streaming_indices and std_gather_sparse)."""
    from sparse_top_kv_std_b200 import binding as B
    c, W = m.cfg, m.dev()
    k_full, v_full = k_full.clone(), v_full.clone()
    cap_full = k_full.shape[3]
    cap_sp = K + c.T + n_tokens + gamma + 1
    dims = B.dims(c.L, 1, c.Hq, c.Hkv, c.d, B.STD_BF16, cap_full, cap_sp)
    k_sp = torch.zeros((c.L, 1, c.Hkv, cap_sp, c.d), dtype=torch.bfloat16, device="cuda")
    v_sp = torch.zeros_like(k_sp)
    len_full = torch.tensor([c.nvis + c.T], dtype=torch.int32, device="cuda")
    len_sp = torch.zeros(1, dtype=torch.int32, device="cuda")
    nvis = torch.tensor([c.nvis], dtype=torch.int32, device="cuda")
    idx = torch.zeros((c.L, 1, c.Hkv, K), dtype=torch.int32, device="cuda")
    if select == "topk":
        ws_sel = torch.empty(B.std_select_workspace_size(dims, c.T, c.nvis), dtype=torch.uint8, device="cuda")
        B.std_select_topk(dims, q_text, c.T, k_full, v_full, nvis, c.nvis, K, idx, k_sp, v_sp, len_sp, None, ws_sel)
    else:
        B.std_streaming_indices(dims, nvis, K, n_sink, idx)
        B.std_gather_sparse(dims, k_full, v_full, nvis, idx, K, c.T, k_sp, v_sp, len_sp)
    d1 = B.dims(1, 1, c.Hq, c.Hkv, c.d, B.STD_BF16, cap_full, cap_sp)
    ws = torch.empty(max(16, B.std_round_workspace_size(d1, gamma)), dtype=torch.uint8, device="cuda")
    n1 = torch.zeros(1, dtype=torch.int32, device="cuda")
    acc = torch.zeros((1, gamma + 1), dtype=torch.int32, device="cuda")
    n_ctx = c.nvis + c.T                      # committed context length, on the host too
    out, counts, bonus = [first], [], first
    while len(out) < n_tokens:
        # gamma draft steps of the sparse model, each on its own previous argmax
        drafts, tok = [], bonus
        for j in range(gamma):
            x = m.embed([tok], n_ctx + j)
            for l in range(c.L):
                x = _attn_layer(B, m, l, x, 1, k_sp, v_sp, len_sp, j,
                                lambda d, q, kl, vl, o, j=j: B.std_sparse_decode_attn(d, q, kl, vl, len_sp, j + 1,
                                                                                      o, 0, ws))
            tok = int(torch.argmax(x[0] @ W["Wlm"]))
            drafts.append(tok)
        # one dense pass over the inputs [bonus, d_0 .. d_{gamma-1}]
        x = m.embed([bonus] + drafts, n_ctx)
        for l in range(c.L):
            x = _attn_layer(B, m, l, x, gamma + 1, k_full, v_full, len_full, 0,
                            lambda d, q, kl, vl, o: B.std_dense_verify_attn(d, q, gamma, kl, vl, len_full, o, 0,
                                                                            ws))
        dense = torch.argmax(x @ W["Wlm"], -1).to(torch.int32).reshape(1, gamma + 1).contiguous()
        draft_t = torch.tensor(drafts, dtype=torch.int32, device="cuda").reshape(1, gamma)
        B.std_accept_prefix(1, gamma, draft_t, dense, n1, acc)
        B.std_kv_commit(dims, k_full, v_full, k_sp, v_sp, len_full, len_sp, n1, gamma + 1)
        n = int(n1.item())
        out.extend(acc[0, :n].tolist())
        counts.append(n)
        n_ctx += n
        bonus = out[-1]
    assert B.std_get_device_error() == 0
    return out[:n_tokens], counts


# ----------------------------------------------------------------------------- fp64 oracle path

def dense_decode_f64(m: ToyLM, n_tokens: int):
    """Greedy decoding of the same model in numpy float64, Q/K/V rounded to bf16 as in the
    library's caches.  Returns (tokens, top-1 minus top-2 logit gap of every step)."""
    c = m.cfg
    bf = lambda a: synth.bf16_bits_to_f64(synth.storage(a.astype(np.float32), "bf16"))  # noqa: E731
    E, Wq, Wk, Wv, Wo, Wlm, P = (getattr(m, n).numpy() for n in ("E", "Wq", "Wk", "Wv", "Wo", "Wlm", "P"))
    N = c.nvis + c.T
    x = np.concatenate([m.vis.numpy(), E[m.text.numpy()]], 0) + P[:N]
    causal = np.tril(np.ones((N, N), bool))
    ks, vs = [], []
    for l in range(c.L):
        q = bf(x @ Wq[l]).reshape(N, c.Hq, c.d)
        k = bf(x @ Wk[l]).reshape(N, c.Hkv, c.d)
        v = bf(x @ Wv[l]).reshape(N, c.Hkv, c.d)
        ks.append(k)
        vs.append(v)
        o = np.zeros((N, c.Hq, c.d))
        for hq in range(c.Hq):
            h = hq // m.G
            s = np.where(causal, (q[:, hq] @ k[:, h].T) / math.sqrt(c.d), -np.inf)
            o[:, hq] = oracle.softmax(s) @ v[:, h]
        x = x + o.reshape(N, -1) @ Wo[l]

    def pick(logits):
        top2 = np.sort(logits)[-2:]
        return int(np.argmax(logits)), float(top2[1] - top2[0])

    tok, gap = pick(x[-1] @ Wlm)
    out, gaps, pos = [tok], [gap], N
    while len(out) < n_tokens:
        h_ = E[tok][None] + P[pos]
        for l in range(c.L):
            q = bf(h_ @ Wq[l]).reshape(c.Hq, c.d)
            ks[l] = np.concatenate([ks[l], bf(h_ @ Wk[l]).reshape(1, c.Hkv, c.d)], 0)
            vs[l] = np.concatenate([vs[l], bf(h_ @ Wv[l]).reshape(1, c.Hkv, c.d)], 0)
            o = np.stack([oracle.attend(q[hq], ks[l][:, hq // m.G], vs[l][:, hq // m.G]) for hq in range(c.Hq)])
            h_ = h_ + o.reshape(1, -1) @ Wo[l]
        tok, gap = pick(h_[0] @ Wlm)
        out.append(tok)
        gaps.append(gap)
        pos += 1
    return out, gaps


def causal_recompute_f64(m: ToyLM, tokens):
    """Argmax after every position of prompt + tokens[:-1], recomputed from scratch with
    full causal attention (no cache) in float64: the greedy stream a correct incremental
    decoder must reproduce.  Returns the predictions for positions N-1 .. N-2+len(tokens)."""
    c = m.cfg
    bf = lambda a: synth.bf16_bits_to_f64(synth.storage(a.astype(np.float32), "bf16"))  # noqa: E731
    E, Wq, Wk, Wv, Wo, Wlm, P = (getattr(m, n).numpy() for n in ("E", "Wq", "Wk", "Wv", "Wo", "Wlm", "P"))
    N0 = c.nvis + c.T
    ids = np.asarray(tokens[:-1], dtype=np.int64)
    x = np.concatenate([m.vis.numpy(), E[m.text.numpy()], E[ids]], 0)
    N = x.shape[0]
    x = x + P[:N]
    for l in range(c.L):
        q = bf(x @ Wq[l]).reshape(N, c.Hq, c.d)
        k = bf(x @ Wk[l]).reshape(N, c.Hkv, c.d)
        v = bf(x @ Wv[l]).reshape(N, c.Hkv, c.d)
        o = np.zeros((N, c.Hq, c.d))
        for hq in range(c.Hq):
            h = hq // m.G
            for i in range(N):
                o[i, hq] = oracle.attend(q[i, hq], k[:i + 1, h], v[:i + 1, h])
        x = x + o.reshape(N, -1) @ Wo[l]
    return [int(t) for t in np.argmax(x[N0 - 1:] @ Wlm, axis=-1)]
