"""The seeded generator: determinism, storage rounding, planted structure, token streams."""
import numpy as np
import torch

import synth
from synth import generator as gen


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(10000).astype(np.float32) * 7,
                        np.array([0.0, -0.0, 1.0, 1.00390625, 1.01171875, 3.4e38, -1e-40],
                                 np.float32)])
    bits = gen.storage(x, "bf16")
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(bits, ref)
    back = gen.bf16_bits_to_f64(bits)
    np.testing.assert_array_equal(back, torch.from_numpy(x).to(torch.bfloat16).double().numpy())


def test_deterministic_and_head_independent():
    wl = synth.workload("tiny_f32")
    a = synth.host_inputs(wl, seed=0, threads=1)
    b = synth.host_inputs(wl, seed=0, threads=4)
    for k in a:
        np.testing.assert_array_equal(a[k], b[k])
    c = synth.host_inputs(wl, seed=1, threads=1)
    assert not np.array_equal(a["k_full"], c["k_full"])
    k, v = synth.kv_head(wl, 0, 0, 0, 1)
    np.testing.assert_array_equal(a["k_full"][0, 0, 1, :k.shape[0]], k)


def test_planted_structure():
    wl = synth.workload("tiny_f32")
    u, sal = synth.planted(wl, 0, 0, 0, 0)
    assert abs(np.linalg.norm(u) - 1) < 1e-6
    assert len(sal) == round(0.02 * 2048) and 0 not in sal and len(set(sal.tolist())) == len(sal)
    k, _ = synth.kv_head(wl, 0, 0, 0, 0)
    proj = k[:2048] @ u
    others = np.setdiff1d(np.arange(1, 2048), sal)
    assert proj[sal].mean() > 3.0 and abs(proj[others].mean()) < 0.3
    assert np.linalg.norm(k[0]) > 4 * np.median(np.linalg.norm(k[1:2048], axis=1))
    q = synth.q_text_head(wl, 0, 0, 0, 0)
    assert (q @ u).mean() > 3.0


def test_token_streams():
    wl = synth.workload("layer_16k")
    dense, draft = synth.tokens(wl, 0, 0)
    assert dense.shape == (wl.rounds, wl.gamma + 1) and draft.shape == (wl.rounds, wl.gamma)
    assert dense.min() >= 0 and dense.max() < 32000 and draft.min() >= 0 and draft.max() < 32000
    big = wl.replace(rounds=4000)
    dn, dr = synth.tokens(big, 0, 0)
    rate = (dn[:, :-1] == dr).mean()
    assert abs(rate - 0.8) < 0.02


def test_workload_shapes():
    wl = synth.workload("video_140k")
    assert (wl.L, wl.Hq, wl.Hkv, wl.d, wl.nvis, wl.T, wl.K, wl.gamma) == \
        (28, 28, 4, 128, (143360,), 256, 4096, 8)
    assert wl.cap_full >= 143360 + 256 + wl.rounds * 9
    r = synth.workload("ragged_b8_K1024_g6_p60")
    assert r.B == 8 and r.K == 1024 and r.gamma == 6 and abs(r.p_match - 0.6) < 1e-12
    assert all(16384 <= n <= 65536 for n in r.nvis) and len(set(r.nvis)) > 1
