"""Seeded synthetic workloads for Sparse-to-Dense decoding.

The pages describe Video-LLM decoding over >140k visual tokens (gist.science
"Sparse-to-Dense", Problemstellung / problem statement) with a top-K selection
of visual KV (Methodik §4) and a draft/verify loop (Methodik §3).  Their
evaluation data (MLVU, VideoMME, 7B checkpoints) is not available, so these
tensors stand in for it with the same shapes and a planted structure:

* Q, K, V ~ N(0, 1) in fp32, rounded once to the storage type (bf16 by
  round-to-nearest-even on the bit pattern) so both consumers read the same
  bits.
* Per (layer, batch, KV head) a random unit direction u; a fraction of the
  visual positions (never position 0) are "salient": key += 4u.  Position 0 is
  a sink: its key is scaled by 6.  Text and decode queries of every query head
  of the group get += 4u.
* V and the decode-time K/V rows carry no planted structure.
* Token streams: dense token t ~ U[0, 32000); the draft equals t with
  probability p, else (t + 1 + U[0, 31999)) mod 32000, which never equals t.

Every tensor comes from its own PCG64 stream keyed by
SeedSequence([seed, workload id, tensor id, gamma, layer, batch, head]) so a
single (layer, batch, head) slice can be regenerated without the rest.

Nothing here computes any part of the method (no attention, no softmax, no
selection, no acceptance).
"""
from __future__ import annotations

import dataclasses
from concurrent.futures import ThreadPoolExecutor
from typing import Callable, Dict, Optional, Sequence, Tuple

import numpy as np

VOCAB = 32000
PLANT = 4.0
SINK_SCALE = 6.0

# tensor ids of the seed tree
_T_PLANT, _T_SALIENT, _T_K, _T_V, _T_QTEXT, _T_QDEC, _T_KVDEC, _T_TOK, _T_NVIS = range(9)


@dataclasses.dataclass(frozen=True)
class Workload:
    """Shapes and generator knobs of one synthetic workload."""

    name: str
    wl_id: int
    dtype: str            # "f32" or "bf16": storage type of Q, K, V
    L: int                # layers
    B: int                # batch
    Hq: int               # query heads
    Hkv: int              # KV heads
    d: int                # head dim
    nvis: Tuple[int, ...]  # visual tokens per sequence
    T: int                # text tokens
    K: int                # kept visual KV per (layer, KV head)
    gamma: int            # draft length
    salient_frac: float
    p_match: float
    rounds: int           # draft+verify rounds of one decode

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    @property
    def nvis_max(self) -> int:
        return max(self.nvis)

    @property
    def cap_full(self) -> int:
        return _round_up(self.nvis_max + self.T + self.rounds * (self.gamma + 1), 16)

    @property
    def cap_sparse(self) -> int:
        return _round_up(self.K + self.T + self.rounds * (self.gamma + 1), 16)

    @property
    def elem_bytes(self) -> int:
        return 4 if self.dtype == "f32" else 2

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


def _round_up(x: int, m: int) -> int:
    return (x + m - 1) // m * m


def _rng(seed: int, wl: Workload, tid: int, *coords: int) -> np.random.Generator:
    key = [int(seed), int(wl.wl_id), int(tid), int(wl.gamma), int(round(wl.p_match * 1000))]
    key += [int(c) for c in coords]
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence(key)))


def ragged_lengths(seed: int, B: int, lo: int = 16384, hi: int = 65536) -> Tuple[int, ...]:
    """Visual lengths of the ragged batch: uniform integers in [lo, hi]."""
    g = np.random.Generator(np.random.PCG64(np.random.SeedSequence([int(seed), 5, _T_NVIS])))
    return tuple(int(x) for x in g.integers(lo, hi + 1, size=B))


def ragged_workload(K: int, gamma: int, p: float, seed: int = 0, rounds: int = 32) -> Workload:
    """One point of the batch-8 ragged sweep (28 q-heads / 4 KV heads / d=128, bf16)."""
    return Workload(name=f"ragged_b8_K{K}_g{gamma}_p{int(p * 100)}", wl_id=5, dtype="bf16",
                    L=1, B=8, Hq=28, Hkv=4, d=128, nvis=ragged_lengths(seed, 8), T=128,
                    K=K, gamma=gamma, salient_frac=0.01, p_match=p, rounds=rounds)


WORKLOADS: Dict[str, Workload] = {
    # 1 layer, 4 q-heads over 2 KV heads, d=64, fp32, 2048 visual + 64 text, K=256, gamma=4
    "tiny_f32": Workload("tiny_f32", 1, "f32", 1, 1, 4, 2, 64, (2048,), 64, 256, 4, 0.02, 0.8, 4),
    # one Qwen2-VL-7B-shaped attention layer, bf16, 16384 visual + 128 text, K=1024, gamma=4
    "layer_16k": Workload("layer_16k", 2, "bf16", 1, 1, 28, 4, 128, (16384,), 128, 1024, 4,
                          0.01, 0.8, 32),
    # 28-layer attention-only stack, 32768 visual + 256 text, K=2048, gamma=6, 32 rounds, p=0.75
    "stack28_32k": Workload("stack28_32k", 3, "bf16", 28, 1, 28, 4, 128, (32768,), 256, 2048, 6,
                            0.01, 0.75, 32),
    # long video: 28 layers, 143360 visual + 256 text (~8.2 GB of KV), K=4096, gamma=8
    "video_140k": Workload("video_140k", 4, "bf16", 28, 1, 28, 4, 128, (143360,), 256, 4096, 8,
                           0.005, 0.8, 32),
}


def workload(name: str) -> Workload:
    if name in WORKLOADS:
        return WORKLOADS[name]
    if name.startswith("ragged_b8"):
        # ragged_b8_K<k>_g<gamma>_p<pct>
        parts = dict((p[0], p[1:]) for p in name.split("_")[2:])
        return ragged_workload(int(parts["K"]), int(parts["g"]), int(parts["p"]) / 100.0)
    raise KeyError(name)


# --------------------------------------------------------------------------- storage

def storage(x: np.ndarray, dtype: str) -> np.ndarray:
    """fp32 values -> storage bits: float32 for "f32", uint16 bf16 (RNE) for "bf16"."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    if dtype == "f32":
        return x
    u = x.view(np.uint32)
    r = (u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def storage_to_f64(x: np.ndarray, dtype: str) -> np.ndarray:
    if dtype == "f32":
        return np.asarray(x, dtype=np.float32).astype(np.float64)
    return bf16_bits_to_f64(np.asarray(x, dtype=np.uint16))


# --------------------------------------------------------------------------- per-head draws

def planted(wl: Workload, seed: int, l: int, b: int, h: int) -> Tuple[np.ndarray, np.ndarray]:
    """(u, salient positions) of one (layer, batch, KV head)."""
    g = _rng(seed, wl, _T_PLANT, l, b, h)
    u = g.standard_normal(wl.d)
    u = (u / np.linalg.norm(u)).astype(np.float32)
    nv = wl.nvis[b]
    n_sal = int(round(wl.salient_frac * nv))
    gs = _rng(seed, wl, _T_SALIENT, l, b, h)
    sal = np.sort(gs.choice(np.arange(1, nv), size=min(n_sal, nv - 1), replace=False))
    return u, sal.astype(np.int64)


def kv_head(wl: Workload, seed: int, l: int, b: int, h: int) -> Tuple[np.ndarray, np.ndarray]:
    """Prompt K and V rows of one (layer, batch, KV head): [nvis_b + T, d] fp32 each.

    Rows [0, nvis_b) are visual, rows [nvis_b, nvis_b + T) are the text tokens.
    """
    n = wl.nvis[b] + wl.T
    u, sal = planted(wl, seed, l, b, h)
    k = _rng(seed, wl, _T_K, l, b, h).standard_normal((n, wl.d), dtype=np.float32)
    k[sal] += np.float32(PLANT) * u
    k[0] *= np.float32(SINK_SCALE)
    v = _rng(seed, wl, _T_V, l, b, h).standard_normal((n, wl.d), dtype=np.float32)
    return k, v


def q_text_head(wl: Workload, seed: int, l: int, b: int, h: int) -> np.ndarray:
    """Text-token queries of the G query heads of KV head h: [G, T, d] fp32."""
    u, _ = planted(wl, seed, l, b, h)
    q = _rng(seed, wl, _T_QTEXT, l, b, h).standard_normal((wl.G, wl.T, wl.d), dtype=np.float32)
    return q + np.float32(PLANT) * u


def decode_queries(wl: Workload, seed: int, l: int, b: int, h: int):
    """Decode queries of the G query heads of KV head h for every round.

    Returns (q_draft [R, gamma, G, d], q_verify [R, G, gamma + 1, d]) fp32.
    """
    u, _ = planted(wl, seed, l, b, h)
    g = _rng(seed, wl, _T_QDEC, l, b, h)
    R, gm, G, d = wl.rounds, wl.gamma, wl.G, wl.d
    qd = g.standard_normal((R, gm, G, d), dtype=np.float32) + np.float32(PLANT) * u
    qv = g.standard_normal((R, G, gm + 1, d), dtype=np.float32) + np.float32(PLANT) * u
    return qd, qv


def decode_kv(wl: Workload, seed: int, l: int, b: int, h: int):
    """K/V rows appended during decoding, for every round.

    Returns (k_draft [R, gamma, d], v_draft, k_verify [R, gamma + 1, d], v_verify) fp32:
    draft step j appends one row to the sparse cache, verify appends gamma + 1 rows
    to the full cache.
    """
    g = _rng(seed, wl, _T_KVDEC, l, b, h)
    R, gm, d = wl.rounds, wl.gamma, wl.d
    kd = g.standard_normal((R, gm, d), dtype=np.float32)
    vd = g.standard_normal((R, gm, d), dtype=np.float32)
    kv = g.standard_normal((R, gm + 1, d), dtype=np.float32)
    vv = g.standard_normal((R, gm + 1, d), dtype=np.float32)
    return kd, vd, kv, vv


def tokens(wl: Workload, seed: int, b: int) -> Tuple[np.ndarray, np.ndarray]:
    """(dense [R, gamma + 1], draft [R, gamma]) int32 token streams of sequence b."""
    g = _rng(seed, wl, _T_TOK, b)
    R, gm = wl.rounds, wl.gamma
    dense = g.integers(0, VOCAB, size=(R, gm + 1))
    match = g.random((R, gm)) < wl.p_match
    other = (dense[:, :gm] + 1 + g.integers(0, VOCAB - 1, size=(R, gm))) % VOCAB
    draft = np.where(match, dense[:, :gm], other)
    return dense.astype(np.int32), draft.astype(np.int32)


# --------------------------------------------------------------------------- assembly

KVSink = Callable[[int, int, int, np.ndarray, np.ndarray], None]


def host_inputs(wl: Workload, seed: int = 0, threads: int = 8,
                kv_sink: Optional[KVSink] = None,
                heads: Optional[Sequence[Tuple[int, int, int]]] = None) -> Dict[str, np.ndarray]:
    """All inputs of one decode in the library's layouts, as storage-typed host arrays.

    Layouts (d innermost):
      k_full, v_full    [L][B][Hkv][cap_full][d]   rows < nvis_b + T filled, rest 0
      q_text            [L][B][Hq][T][d]
      q_draft           [R][gamma][L][B][Hq][1][d]
      q_verify          [R][L][B][Hq][gamma + 1][d]
      k_draft, v_draft  [R][gamma][L][B][Hkv][1][d]
      k_verify, v_verify[R][L][B][Hkv][gamma + 1][d]
      dense_tokens      [R][B][gamma + 1] int32,  draft_tokens [R][B][gamma] int32
      nvis              [B] int32
    If kv_sink is given, the prompt K/V of each head is handed to it as storage
    arrays instead of being assembled into k_full / v_full (which are then absent).
    heads restricts the prompt K/V draws to the listed (l, b, h).
    """
    L, B, Hq, Hkv, d, G = wl.L, wl.B, wl.Hq, wl.Hkv, wl.d, wl.G
    R, gm, T = wl.rounds, wl.gamma, wl.T
    st = np.float32 if wl.dtype == "f32" else np.uint16
    out: Dict[str, np.ndarray] = {}
    if kv_sink is None:
        out["k_full"] = np.zeros((L, B, Hkv, wl.cap_full, d), st)
        out["v_full"] = np.zeros((L, B, Hkv, wl.cap_full, d), st)
    out["q_text"] = np.zeros((L, B, Hq, T, d), st)
    out["q_draft"] = np.zeros((R, gm, L, B, Hq, 1, d), st)
    out["q_verify"] = np.zeros((R, L, B, Hq, gm + 1, d), st)
    out["k_draft"] = np.zeros((R, gm, L, B, Hkv, 1, d), st)
    out["v_draft"] = np.zeros((R, gm, L, B, Hkv, 1, d), st)
    out["k_verify"] = np.zeros((R, L, B, Hkv, gm + 1, d), st)
    out["v_verify"] = np.zeros((R, L, B, Hkv, gm + 1, d), st)

    all_heads = [(l, b, h) for l in range(L) for b in range(B) for h in range(Hkv)]
    kv_heads = set(all_heads if heads is None else heads)

    def one(lbh):
        l, b, h = lbh
        if lbh in kv_heads:
            k, v = kv_head(wl, seed, l, b, h)
            ks, vs = storage(k, wl.dtype), storage(v, wl.dtype)
            if kv_sink is None:
                n = ks.shape[0]
                out["k_full"][l, b, h, :n] = ks
                out["v_full"][l, b, h, :n] = vs
            else:
                kv_sink(l, b, h, ks, vs)
        out["q_text"][l, b, h * G:(h + 1) * G] = storage(q_text_head(wl, seed, l, b, h), wl.dtype)
        qd, qv = decode_queries(wl, seed, l, b, h)
        out["q_draft"][:, :, l, b, h * G:(h + 1) * G, 0] = storage(qd, wl.dtype)
        out["q_verify"][:, l, b, h * G:(h + 1) * G] = storage(qv, wl.dtype)
        kd, vd, kv, vv = decode_kv(wl, seed, l, b, h)
        out["k_draft"][:, :, l, b, h, 0] = storage(kd, wl.dtype)
        out["v_draft"][:, :, l, b, h, 0] = storage(vd, wl.dtype)
        out["k_verify"][:, l, b, h] = storage(kv, wl.dtype)
        out["v_verify"][:, l, b, h] = storage(vv, wl.dtype)

    if threads > 1 and len(all_heads) > 1:
        with ThreadPoolExecutor(threads) as ex:
            list(ex.map(one, all_heads))
    else:
        for x in all_heads:
            one(x)

    dense = np.zeros((R, B, gm + 1), np.int32)
    draft = np.zeros((R, B, gm), np.int32)
    for b in range(B):
        dn, dr = tokens(wl, seed, b)
        dense[:, b] = dn
        draft[:, b] = dr
    out["dense_tokens"] = dense
    out["draft_tokens"] = draft
    out["nvis"] = np.asarray(wl.nvis, np.int32)
    return out
