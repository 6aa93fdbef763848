"""Pins of the oracle's mse rule where the order of the squared-error sum decides.

The oracle evaluates each candidate's error as stated in its header: residuals as one
fused multiply-add, squares fused-multiply-added into an even-position and an
odd-position sum, then one addition. These tests hold that evaluation to things outside
the oracle:

* hand-worked near-tie blocks (tests/golden/mse_near_ties.txt), whose candidate errors
  are equal in exact arithmetic, worked on paper in both the oracle's order and the
  multiply / subtract / pairwise-tree order; the two orders choose differently, so the
  blocks tell the orders apart;
* an exact-rational restatement of the whole block quantizer (tests/exact_fp32.py:
  Fractions, each IEEE operation rounded once by a rounding function written from the
  IEEE definition), compared bit for bit with the oracle's codes, scale codes and both
  candidate errors on random, heavy-tailed, grid-valued and near-tie blocks under many
  global scales.
"""
from fractions import Fraction

import numpy as np
import pytest

import exact_fp32 as ex
from golden_io import floats_to_bf16_bits, hex_bytes, read_sections, round_to_bf16_bits


def _golden():
    g = read_sections("mse_near_ties.txt")
    x = floats_to_bf16_bits(g["input"]).reshape(-1, 16)
    return g, x


def _packed(codes):
    return [codes[2 * j] | (codes[2 * j + 1] << 4) for j in range(8)]


def test_near_tie_blocks_oracle_follows_its_order(orc):
    g, x = _golden()
    packed, scales, amax = orc.quantize(x.reshape(-1), 16, "mse")
    assert amax == float(g["amax"][0])
    np.testing.assert_array_equal(scales, hex_bytes(g["fma_even_odd.scales"]))
    np.testing.assert_array_equal(packed, hex_bytes(g["fma_even_odd.packed"]))
    errs = np.array([float(t) for t in g["fma_even_odd.errors"]]).reshape(-1, 2)
    for row, (e6_want, e4_want) in zip(x, errs):
        _, _, e6, e4 = orc.quantize_block_detail(row, amax, "mse")
        assert (e6, e4) == (e6_want, e4_want)


@pytest.mark.parametrize("order", ["fma_even_odd", "mul_sub_pairwise"])
def test_near_tie_blocks_exact_restatement(order):
    """The exact restatement reproduces the paper derivation of both orders."""
    g, x = _golden()
    amax_t = Fraction(g["amax"][0])
    want_scales = hex_bytes(g[f"{order}.scales"])
    want_packed = hex_bytes(g[f"{order}.packed"]).reshape(-1, 8)
    errs = [Fraction(t) for t in g[f"{order}.errors"]]
    for i, row in enumerate(x):
        c, codes, e6, e4 = ex.mse_block([int(b) for b in row], amax_t, order)
        assert c == want_scales[i]
        assert _packed(codes) == want_packed[i].tolist()
        assert (e6, e4) == (errs[2 * i], errs[2 * i + 1])


def test_near_tie_blocks_separate_the_orders():
    g, _ = _golden()
    a, b = hex_bytes(g["fma_even_odd.scales"]), hex_bytes(g["mul_sub_pairwise.scales"])
    assert (a[1:] != b[1:]).all()
    # one block goes each way: the oracle's order keeps R = 4 in row 1 and R = 6 in row 2
    assert a[1] == 0x3C and a[2] == 0x38


def _bf16_f64(bits):
    import torch

    return torch.from_numpy(bits.astype(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()


def _random_blocks(rng, n):
    """(block bits, global amax) pairs of several kinds; the amax is an fp32 value."""
    tau = 2.0 ** -12
    out = []
    for k in range(n):
        kind = k % 5
        if kind == 0:
            v = rng.standard_normal(16)
        elif kind == 1:
            v = rng.standard_t(3, 16)
        elif kind == 2:
            v = rng.choice([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0], 16) * rng.choice([-1, 1], 16)
        elif kind == 3:  # near ties: grid midpoints and neighbours over tiny residuals
            v = rng.choice([0.0, 0.0, tau, tau / 2, 2 * tau], 16)
            v[0] = 6.0
            for p in rng.choice(np.arange(1, 16), 3, replace=False):
                v[p] = rng.choice([4.0, 2.5, 0.75, 5.0, 3.5, 1.25, 2.0, 1.0, 0.5])
        else:  # a wide dynamic range inside one block
            v = rng.standard_normal(16) * 2.0 ** rng.integers(-30, 10, 16)
        x = round_to_bf16_bits(v * 2.0 ** int(rng.integers(-20, 20)))
        amax_b = float(np.abs(_bf16_f64(x)).max())
        if amax_b == 0.0:
            continue
        if kind == 3 and k % 2:
            amax_t = amax_b * 448.0  # gs = amax_b / 6: every product val * S is exact
        else:
            # up to 1e3: normal e4m3 scales; 1e5 and 3e6: subnormal e4m3 scales and scales
            # that round to zero (448 * amax_b / amax_t below 2^-6 and 2^-10)
            amax_t = amax_b * float(rng.choice([1.0, 1.0, 2.5, 37.0, 1e3, 1e5, 3e6]))
        out.append((x, float(np.float32(amax_t))))
    return out


def test_oracle_equals_exact_restatement_bit_for_bit(orc):
    rng = np.random.default_rng(2026)
    blocks = _random_blocks(rng, 600)
    assert len(blocks) > 500
    chose4 = 0
    subnormal_scales = 0
    for x, amax_f in blocks:
        amax_t = Fraction(amax_f)
        bits = [int(b) for b in x]
        c, codes, e6, e4 = ex.mse_block(bits, amax_t, "fma_even_odd")
        oc, opk, oe6, oe4 = orc.quantize_block_detail(x, amax_f, "mse")
        assert oc == c and opk.tolist() == _packed(codes)
        assert Fraction(oe6) == e6 and Fraction(oe4) == e4
        chose4 += e4 < e6
        subnormal_scales += 0 < (c & 0x7F) < 8  # e4m3 exponent field 0: a subnormal scale
        for R, rule in ((6, "static_6"), (4, "static_4")):
            sc, _, scodes = ex.candidate(bits, amax_t, R)
            occ, opk2, _, _ = orc.quantize_block_detail(x, amax_f, rule)
            assert occ == sc and opk2.tolist() == _packed(scodes)
    assert 0 < chose4 < len(blocks)
    assert subnormal_scales > 10
