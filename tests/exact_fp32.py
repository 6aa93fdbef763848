"""Exact-rational restatement of the NVFP4 block quantizer, for pinning the oracle.

Every quantity is a ``fractions.Fraction``; every IEEE binary32 operation of the
specification is "compute the exact real result, then round it once to binary32" with
``rn32``, written here from the IEEE 754 definition of round-to-nearest-even (including
subnormals). Nothing here calls the C oracle, numpy's float32 or the CUDA library, so a
slip in the oracle's use of ``fmaf``, its summation order, or its encodes shows up as a
disagreement.

The specification restated (the pages' formulas, with the readings the oracle lists):
  * global scale gs = RN(amax_t / 2688)   ("How NVFP4 Quantization Works in LongLive 2.0
    for Transformer Inference", "Stage 3", step 3: amax / (e2m1_max * e4m3_max))
  * candidate R: r = RN(RN(amax_b / R) / gs); c = e4m3 nearest-even, saturating at 448
    ("Understanding the NVFP4 Format": block scales in FP8 e4m3)
  * S = RN(e4m3(c) * gs); inv = RN(1 / S), or 0 when that is infinite
  * codes: e2m1 nearest-even of RN(x * inv), saturating at 6, sign kept
    ("Stage 1", step 3)
  * mse ("How to Use KV Cache Quantization with LongLive's LongLiveQuantizationConfig",
    "Configuration Parameters Reference": the rule that minimises the squared error),
    with two orders of evaluating that error:
      ``fma_even_odd``  d_i = RN(x_i - val_i * S)   (one rounding: a fused multiply-add)
                        s_even = RN(s_even + d_i^2) for even i, s_odd likewise for odd
                        i, both in index order (one rounding each: fused multiply-adds);
                        err = RN(s_even + s_odd)
      ``mul_sub_pairwise``  p_i = RN(val_i * S); d_i = RN(x_i - p_i); q_i = RN(d_i^2);
                        err = pairwise tree ((q0 + q1) + (q2 + q3)) + ..., each sum
                        rounded
    R = 4 is kept only when its error is strictly smaller than R = 6's.
"""
from __future__ import annotations

from fractions import Fraction

E2M1_GRID = [Fraction(0), Fraction(1, 2), Fraction(1), Fraction(3, 2), Fraction(2), Fraction(3), Fraction(4),
             Fraction(6)]
E4M3_MAX = Fraction(448)


def _floor_log2(a: Fraction) -> int:
    """floor(log2(a)) for a > 0."""
    e = a.numerator.bit_length() - a.denominator.bit_length()
    if Fraction(2) ** e > a:
        e -= 1
    elif Fraction(2) ** (e + 1) <= a:
        e += 1
    return e


def rn32(q: Fraction) -> Fraction:
    """Round an exact real to the nearest binary32 value, ties to even mantissa. Finite
    results only (the quantities here never overflow)."""
    if q == 0:
        return Fraction(0)
    neg = q < 0
    a = -q if neg else q
    e = max(_floor_log2(a), -126)  # below 2^-126 the spacing stays 2^-149 (subnormals)
    quantum = Fraction(2) ** (e - 23)
    m = a / quantum
    n = m.numerator // m.denominator
    rem = m - n
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and n % 2 == 1):
        n += 1
    r = n * quantum
    assert r < Fraction(2) ** 128, "binary32 overflow"
    return -r if neg else r


def rn_bf16(q: Fraction) -> Fraction:
    """Round an exact real to the nearest bf16 value (8 significant bits), ties to even
    mantissa, subnormals included. Finite results only."""
    if q == 0:
        return Fraction(0)
    a = abs(q)
    e = max(_floor_log2(a), -126)
    quantum = Fraction(2) ** (e - 7)
    m = a / quantum
    n = m.numerator // m.denominator
    rem = m - n
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and n % 2 == 1):
        n += 1
    r = n * quantum
    return -r if q < 0 else r


def bf16_value(bits: int) -> Fraction:
    """Exact value of a bf16 bit pattern (finite)."""
    sign = -1 if bits & 0x8000 else 1
    e = (bits >> 7) & 0xFF
    m = bits & 0x7F
    assert e != 0xFF, "finite inputs only"
    if e == 0:
        return sign * Fraction(m, 128) * Fraction(2) ** -126
    return sign * (1 + Fraction(m, 128)) * Fraction(2) ** (e - 127)


def e4m3_value(code: int) -> Fraction:
    f = code & 0x7F
    e, m = f >> 3, f & 7
    if e == 0:
        return Fraction(m, 8) * Fraction(2) ** -6
    return (1 + Fraction(m, 8)) * Fraction(2) ** (e - 7)


E4M3_VALUES = [e4m3_value(c) for c in range(127)]  # codes 0..126, increasing


def e4m3_encode(r: Fraction) -> int:
    """Nearest e4m3 code to r >= 0, ties to the even code, saturating at 448 (code 126)."""
    if r >= E4M3_MAX:
        return 126
    best = 0
    for c in range(127):
        d, db = abs(r - E4M3_VALUES[c]), abs(r - E4M3_VALUES[best])
        if d < db or (d == db and c % 2 == 0):
            best = c
    return best


def e2m1_encode(v: Fraction, negative: bool) -> int:
    """Nearest e2m1 magnitude to |v|, ties to the even code, saturating at 6; bit 3 is
    the sign of v (kept when the magnitude rounds to zero)."""
    a = abs(v)
    best = 7
    if a <= 6:
        for f in range(8):
            d, db = abs(a - E2M1_GRID[f]), abs(a - E2M1_GRID[best])
            if d < db or (d == db and f % 2 == 0):
                best = f
    return (8 if negative else 0) | best


def e2m1_value(code: int) -> Fraction:
    mag = E2M1_GRID[code & 7]
    return -mag if code & 8 else mag


def candidate(x_bits: list[int], amax_t: Fraction, R: int):
    """Scale code, decoded scale and the 16 codes of one block under denominator R."""
    x = [bf16_value(b) for b in x_bits]
    amax_b = max(abs(v) for v in x)
    gs = rn32(amax_t / 2688)
    c = 0 if gs == 0 else e4m3_encode(rn32(rn32(amax_b / R) / gs))
    S = rn32(e4m3_value(c) * gs)
    inv = Fraction(0) if S == 0 or abs(1 / S) >= Fraction(2) ** 128 else rn32(1 / S)
    codes = [e2m1_encode(rn32(v * inv), bool(b & 0x8000)) for v, b in zip(x, x_bits)]
    return c, S, codes


def sq_error(x_bits: list[int], S: Fraction, codes: list[int], order: str) -> Fraction:
    x = [bf16_value(b) for b in x_bits]
    val = [e2m1_value(q) for q in codes]
    if order == "fma_even_odd":
        s = [Fraction(0), Fraction(0)]
        for i in range(16):
            d = rn32(x[i] - val[i] * S)
            s[i & 1] = rn32(s[i & 1] + d * d)
        return rn32(s[0] + s[1])
    if order == "mul_sub_pairwise":
        q = []
        for i in range(16):
            d = rn32(x[i] - rn32(val[i] * S))
            q.append(rn32(d * d))
        while len(q) > 1:
            q = [rn32(q[2 * j] + q[2 * j + 1]) for j in range(len(q) // 2)]
        return q[0]
    raise ValueError(order)


def mse_block(x_bits: list[int], amax_t: Fraction, order: str = "fma_even_odd"):
    """(chosen scale code, codes, err6, err4) of one block under rule mse."""
    c6, S6, q6 = candidate(x_bits, amax_t, 6)
    c4, S4, q4 = candidate(x_bits, amax_t, 4)
    e6, e4 = sq_error(x_bits, S6, q6, order), sq_error(x_bits, S4, q4, order)
    return (c4, q4, e6, e4) if e4 < e6 else (c6, q6, e6, e4)
