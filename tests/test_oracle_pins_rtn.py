"""Pins of the oracle's RTN integer codecs (the study's RTN_INT4 / RTN_INT2 / K2_V4):
a hand-worked example, the study's own compression figure, brute force and invariants."""
import numpy as np
import pytest
import torch

from golden_io import floats_to_bf16_bits, read_sections, round_to_bf16_bits


def _hex16(tokens):
    return np.array([int(t, 16) for t in tokens], dtype=np.uint16)


def _hex8(tokens):
    return np.array([int(t, 16) for t in tokens], dtype=np.uint8)


def _f64(bits):
    return torch.from_numpy(bits.astype(np.int16)).view(torch.bfloat16).double().numpy()


def _codes(packed, bits):
    per = 8 // bits
    v = np.stack([(packed >> (bits * k)) & ((1 << bits) - 1) for k in range(per)], 1).reshape(-1).astype(np.int64)
    return np.where(v >= (1 << (bits - 1)), v - (1 << bits), v)


@pytest.mark.parametrize("bits", [4, 2])
def test_rtn_worked_example(orc, bits):
    g = read_sections("rtn_worked_example.txt")
    x = floats_to_bf16_bits(g[f"int{bits}.input"])
    p, s = orc.rtn_quantize(x, 16, bits)
    np.testing.assert_array_equal(s, _hex16(g[f"int{bits}.scales"]))
    np.testing.assert_array_equal(p, _hex8(g[f"int{bits}.packed"]))
    y = orc.rtn_dequantize(p, s, 16, bits)
    np.testing.assert_array_equal(_f64(y), _f64(floats_to_bf16_bits(g[f"int{bits}.dequant"])))


@pytest.mark.parametrize("bits,ratio", [(2, 5.33), (4, 3.20)])
def test_rtn_compression_matches_the_study(orc, bits, ratio):
    """The study reports 5.33x for RTN INT2 (Table 4): 16 bf16 bits over bits + 16/16
    scale bits per value. That fixes a 16-bit scale per 16 values."""
    x = round_to_bf16_bits(np.random.default_rng(0).standard_normal(16 * 1000))
    p, s = orc.rtn_quantize(x, 128, bits)
    stored = p.nbytes + s.nbytes
    assert round(x.nbytes / stored, 2) == ratio


@pytest.mark.parametrize("bits", [4, 2])
def test_rtn_levels_are_nearest_to_x_over_s(orc, bits):
    """Brute force: every level is the nearest integer in [-qmax, qmax] to x / S (fp64),
    ties to the even integer, for 2000 random blocks."""
    qmax = (1 << (bits - 1)) - 1
    rng = np.random.default_rng(bits)
    for trial in range(2000):
        v = rng.standard_t(3, 16) * 2.0 ** int(rng.integers(-10, 10))
        x = round_to_bf16_bits(v)
        p, s = orc.rtn_quantize(x, 16, bits)
        S = float(_f64(s.astype(np.uint16))[0])
        q = _codes(p, bits)
        t = _f64(x) / S
        cand = np.arange(-qmax, qmax + 1)
        for i in range(16):
            d = np.abs(cand - t[i])
            best = cand[d == d.min()]
            if best.size > 1:
                best = best[best % 2 == 0]
            assert q[i] == best[0], (trial, i, t[i], q[i])


@pytest.mark.parametrize("bits", [4, 2])
def test_rtn_integer_blocks_round_trip_exactly(orc, bits):
    qmax = (1 << (bits - 1)) - 1
    rng = np.random.default_rng(5)
    for j in (-20, 0, 9):
        q = rng.integers(-qmax, qmax + 1, 16 * 40)
        q[::16] = qmax  # every block's amax is qmax * 2^j, so S = 2^j exactly
        x = floats_to_bf16_bits(q * 2.0 ** j)
        p, s = orc.rtn_quantize(x, 16, bits)
        np.testing.assert_array_equal(_codes(p, bits), q)
        np.testing.assert_array_equal(orc.rtn_dequantize(p, s, 16, bits), x)


@pytest.mark.parametrize("bits", [4, 2])
def test_rtn_sign_symmetry_and_zero_block(orc, bits):
    x = round_to_bf16_bits(np.random.default_rng(1).standard_normal(16 * 64))
    x[:16] = 0
    p, s = orc.rtn_quantize(x, 128, bits)
    pn, sn = orc.rtn_quantize(x ^ np.uint16(0x8000), 128, bits)
    np.testing.assert_array_equal(s, sn)
    np.testing.assert_array_equal(_codes(pn, bits), -_codes(p, bits))
    assert s[0] == 0 and not p[:16 * bits // 8].any()


@pytest.mark.parametrize("bits,bound", [(4, 2.5e-2), (2, 0.45)])
def test_rtn_relative_mse(orc, bits, bound):
    from nvfp4_kv_cache_kvq_b200 import inputs

    x = inputs.bits(inputs.single_k())
    p, s = orc.rtn_quantize(x, 128, bits)
    y = _f64(orc.rtn_dequantize(p, s, 128, bits))
    xf = _f64(x)
    rel = np.sum((y - xf) ** 2) / np.sum(xf ** 2)
    assert rel <= bound, rel


# ---------------------------------------------------------------- exact restatement

def _round_half_even(t):
    from fractions import Fraction

    n = t.numerator // t.denominator
    rem = t - n
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and n % 2 == 1):
        n += 1
    return n


@pytest.mark.parametrize("bits", [4, 2])
def test_rtn_equals_exact_restatement(orc, bits):
    """The RTN codec restated with exact rationals, each IEEE step rounded once (the
    reading of the study's appendix Table 3 that the oracle lists): S = bf16(fp32(amax_b /
    qmax)), q = round-half-even(fp32(x / S)) clamped to [-qmax, qmax] (0 when S = 0),
    y = bf16(fp32(q * S)). Blocks from bf16 subnormals to 2^100, bit for bit."""
    import exact_fp32 as ex

    qmax = (1 << (bits - 1)) - 1
    rng = np.random.default_rng(40 + bits)
    for trial in range(300):
        v = rng.standard_t(3, 16) * 2.0 ** int(rng.integers(-136, 100))
        if trial % 7 == 0:
            v[rng.integers(0, 16)] = 0.0
        x = round_to_bf16_bits(v)
        p, s = orc.rtn_quantize(x, 16, bits)
        y = orc.rtn_dequantize(p, s, 16, bits)
        xs = [ex.bf16_value(int(b)) for b in x]
        amax_b = max(abs(t) for t in xs)
        S = ex.rn_bf16(ex.rn32(amax_b / qmax))
        assert ex.bf16_value(int(s[0])) == S, (trial, float(S))
        q = [0 if S == 0 else max(-qmax, min(qmax, _round_half_even(ex.rn32(t / S)))) for t in xs]
        assert _codes(p, bits).tolist() == q, trial
        want = [ex.rn_bf16(ex.rn32(qi * S)) for qi in q]
        assert [abs(ex.bf16_value(int(b))) for b in y] == [abs(w) for w in want], trial
        assert all(ex.bf16_value(int(b)) == w for b, w in zip(y, want) if w != 0), trial
