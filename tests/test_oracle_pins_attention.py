"""Pins of the oracle's attention: closed forms a softmax must satisfy."""
import numpy as np

from golden_io import round_to_bf16_bits


def test_attention_single_key_returns_its_value(orc):
    rng = np.random.default_rng(0)
    q = round_to_bf16_bits(rng.standard_normal((5, 2, 16)))
    k = round_to_bf16_bits(rng.standard_normal((1, 2, 16)))
    v = round_to_bf16_bits(rng.standard_normal((1, 2, 16)))
    out = orc.attention(q, k, v, 5, 1, 2, 16, 0.25)
    vf = (v.astype(np.uint32) << 16).view(np.float32).reshape(1, 2, 16)
    np.testing.assert_allclose(out, np.broadcast_to(vf, (5, 2, 16)), rtol=0, atol=0)


def test_attention_equal_scores_average_the_values(orc):
    rng = np.random.default_rng(1)
    q = np.zeros((3, 1, 16), np.uint16)  # zero queries: every score 0, uniform weights
    k = round_to_bf16_bits(rng.standard_normal((7, 1, 16)))
    v = round_to_bf16_bits(rng.standard_normal((7, 1, 16)))
    out = orc.attention(q, k, v, 3, 7, 1, 16, 1.0)
    vf = (v.astype(np.uint32) << 16).view(np.float32).reshape(7, 1, 16).astype(np.float64)
    np.testing.assert_allclose(out, np.broadcast_to(vf.mean(axis=0), (3, 1, 16)), rtol=1e-12)


def test_attention_large_score_gap_selects_one_key(orc):
    k = np.zeros((4, 1, 16), np.float64)
    k[2, 0, 0] = 64.0
    q = np.zeros((1, 1, 16))
    q[0, 0, 0] = 64.0  # score 4096 for key 2, 0 for the others
    v = np.arange(4 * 16, dtype=np.float64).reshape(4, 1, 16)
    out = orc.attention(round_to_bf16_bits(q), round_to_bf16_bits(k), round_to_bf16_bits(v), 1, 4, 1, 16, 1.0)
    np.testing.assert_allclose(out[0, 0], v[2, 0], rtol=0, atol=1e-12)
