"""Pins of the toy language model's fp64 greedy decoder, which the losslessness
test uses as the expected token stream.

The incremental decoder (KV cache, one query per step) must give the same
tokens as recomputing every position from scratch with plain causal attention
-- an independent route through the model, so a wrong cache position, a missing
residual or a mis-grouped head shows up here.
"""
import numpy as np

from tests.toy_lm import ToyConfig, ToyLM, causal_recompute_f64, dense_decode_f64

SMALL = ToyConfig(nvis=192, T=16, max_pos=512)


def test_incremental_greedy_equals_causal_recompute():
    for seed in (0, 1):
        m = ToyLM(SMALL, seed)
        toks, gaps = dense_decode_f64(m, 24)
        assert causal_recompute_f64(m, toks) == toks


def test_greedy_gaps_are_top1_minus_top2():
    m = ToyLM(SMALL, 3)
    toks, gaps = dense_decode_f64(m, 8)
    assert len(toks) == len(gaps) == 8
    assert all(g >= 0 for g in gaps)


def test_toy_weights_fixed_by_seed():
    a, b, c = ToyLM(SMALL, 5), ToyLM(SMALL, 5), ToyLM(SMALL, 6)
    assert np.array_equal(a.Wq.numpy(), b.Wq.numpy()) and np.array_equal(a.text.numpy(), b.text.numpy())
    assert not np.array_equal(a.Wq.numpy(), c.Wq.numpy())
