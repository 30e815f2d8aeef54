"""Losslessness of Sparse-to-Dense decoding on a toy language model.

The method's claim (gist.science summary, "Methodik" item 3 and
"Hauptbeiträge"; "lossless" in the abstract): whatever the sparse draft model
proposes, the kept tokens are exactly the dense model's greedy tokens.  Here the
whole loop runs through the library -- prefill selection, gamma sparse draft
steps that feed on their own argmax, one dense verify pass, acceptance, commit
-- and its stream must equal plain greedy decoding, both with the library's
dense attention and with the fp64 oracle.  The seeds are ones whose fp64
greedy stream keeps a top-1 / top-2 logit gap of at least 0.03, far above the
fp32 and bf16 rounding of the GPU path, so the streams must agree exactly.
"""
import pytest
import torch

from tests.toy_lm import ToyConfig, ToyLM, dense_decode_f64, dense_decode_gpu, prefill, std_decode

pytestmark = pytest.mark.gpu

N_TOKENS = 64
CFG = ToyConfig()
CAP_FULL = CFG.nvis + CFG.T + N_TOKENS + 32 + 1


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    torch.backends.cuda.matmul.allow_tf32 = False


_cache = {}


def _model(seed):
    if seed not in _cache:
        m = ToyLM(CFG, seed)
        want, gaps = dense_decode_f64(m, N_TOKENS)
        assert min(gaps) > 0.03, "seed without a clear greedy stream"
        kf, vf, qt, first = prefill(m, CAP_FULL)
        _cache[seed] = (m, want, kf, vf, qt, first)
    return _cache[seed]


def _first_diff(a, b):
    return next((i for i, (x, y) in enumerate(zip(a, b)) if x != y), None)


@pytest.mark.parametrize("seed", [1, 2, 6])
def test_dense_gpu_greedy_matches_fp64(seed):
    m, want, kf, vf, qt, first = _model(seed)
    got = dense_decode_gpu(m, kf, vf, first, N_TOKENS)
    assert got == want, _first_diff(got, want)


@pytest.mark.parametrize("seed,K,gamma", [(1, 512, 6), (2, 512, 6), (6, 256, 8), (1, 64, 4), (2, 2048, 8),
                                          (6, 512, 1), (1, 512, 0), (2, 512, 31)])
def test_std_stream_equals_dense_greedy(seed, K, gamma):
    m, want, kf, vf, qt, first = _model(seed)
    got, counts = std_decode(m, kf, vf, qt, first, K, gamma, N_TOKENS)
    assert got == want, (_first_diff(got, want), counts)
    assert all(1 <= n <= gamma + 1 for n in counts)
    if gamma >= 4 and K < CFG.nvis:
        # both outcomes of the acceptance step happened: a rejected first draft and a multi-token accept
        assert min(counts) == 1 and max(counts) > 2, counts


def test_full_selection_drafts_are_accepted():
    """K = nvis: the sparse cache holds every visual row in order, so the draft model is
    the dense model and (nearly) every draft is accepted."""
    m, want, kf, vf, qt, first = _model(2)
    got, counts = std_decode(m, kf, vf, qt, first, CFG.nvis, 8, N_TOKENS)
    assert got == want
    full = sum(n == 9 for n in counts[:-1])
    assert full >= 0.8 * (len(counts) - 1), counts


def test_streaming_baseline_is_lossless_and_compared_with_topk():
    """The streaming draft baseline (sinks + recent window, same kernels) is lossless too:
    any index set only changes how many drafts are accepted.  Prints the mean tokens per
    round of both index sets at equal K."""
    rows = []
    for seed, K, gamma in [(1, 512, 6), (2, 512, 6), (6, 256, 8), (1, 128, 6)]:
        m, want, kf, vf, qt, first = _model(seed)
        got_t, cnt_t = std_decode(m, kf, vf, qt, first, K, gamma, N_TOKENS)
        got_s, cnt_s = std_decode(m, kf, vf, qt, first, K, gamma, N_TOKENS, select="stream")
        assert got_t == want, _first_diff(got_t, want)
        assert got_s == want, _first_diff(got_s, want)
        rows.append((seed, K, gamma, sum(cnt_t) / len(cnt_t), sum(cnt_s) / len(cnt_s)))
    print("\nseed  K  gamma  tokens/round top-K  tokens/round streaming")
    for r in rows:
        print("%4d %4d %5d %12.2f %18.2f" % r)
