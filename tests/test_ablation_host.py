"""Host-side arithmetic of the gamma / K ablation (no GPU): the attention-I/O model."""
import math

from sparse_top_kv_std_b200.ablation import io_model


def test_io_model_closed_forms():
    # p = 0: one token per round; the round reads gamma sparse caches plus the full cache
    s, e = io_model([1000], 24, 100, 3, 0.0)
    assert e == 1.0 and math.isclose(s, 1024 / (3 * 124 + 1024 + 4))
    # p = 1: every draft matches, gamma + 1 tokens per round
    s, e = io_model([1000, 3000], 24, 100, 4, 1.0)
    assert e == 5.0 and math.isclose(s, (1024 + 3024) * 5 / (2 * 4 * 124 + 1024 + 3024 + 2 * 5))
    # geometric sum for 0 < p < 1
    _, e = io_model([10], 2, 1, 3, 0.5)
    assert math.isclose(e, 1 + 0.5 + 0.25 + 0.125)
