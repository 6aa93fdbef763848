"""Error bound of the fused attention's FMA-pipe exp2 (Cody and Waite range reduction plus
a cubic for 2^f on [-1/2, 1/2]): the kernel's own constants, read from its source,
evaluated with the kernel's fp32 operation sequence (each fused multiply-add rounded once)
against 2^x in fp64. The kernel relies on a relative error below 1.5e-4, far under the
2^-9 of P's bf16 rounding."""
import os
import re

import numpy as np

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "nvfp4_kv_cache_kvq_b200", "csrc",
                   "kvq_attention.cu")


def _constants():
    src = open(SRC).read()
    body = src[src.index("uint64_t exp2_poly(uint64_t x2)"):]
    body = body[:body.index("\n}\n")]
    # the polynomial coefficients, highest degree first, as they appear in Horner order
    coef = [float(c) for c in re.findall(r"f32x2_pack\((0\.\d+)f, \1f\)", body)]
    assert len(coef) == 4, coef
    assert "-125.0f" in body and "12582912.0f" in body
    return coef


def _f32(x):
    return np.asarray(x, dtype=np.float64).astype(np.float32)


def _fma(a, b, c):
    # fp32 fused multiply-add: the exact a*b + c (exact in fp64 for fp32 inputs of these
    # magnitudes) rounded once to fp32
    return _f32(a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64))


def _exp2_poly(x):
    c3, c2, c1, c0 = [np.float32(c) for c in _constants()]
    x = np.maximum(_f32(x), np.float32(-125.0))
    one = np.float32(1.0)
    magic = np.float32(12582912.0)
    t = _fma(x, one, magic)
    n = _fma(t, one, -magic)
    f = _fma(n, np.float32(-1.0), x)
    p = _fma(np.full_like(f, c3), f, np.full_like(f, c2))
    p = _fma(p, f, np.full_like(f, c1))
    p = _fma(p, f, np.full_like(f, c0))
    bits = p.view(np.uint32) + (t.view(np.uint32) << np.uint32(23))
    return bits.astype(np.uint32).view(np.float32)


def test_exp2_poly_relative_error_bound():
    rng = np.random.default_rng(0)
    x = np.concatenate([np.linspace(-125.0, 8.0, 400001), rng.uniform(-125.0, 8.0, 200000),
                        np.arange(-125, 9, dtype=np.float64) + 0.5, np.arange(-125, 9, dtype=np.float64)])
    x = _f32(x)
    got = _exp2_poly(x).astype(np.float64)
    want = np.exp2(x.astype(np.float64))
    rel = np.abs(got / want - 1.0)
    assert rel.max() < 1.5e-4, rel.max()


def test_exp2_poly_clamps_below():
    # far below the row maximum the result is the clamp 2^-125 (normal), never garbage
    got = _exp2_poly(np.array([-200.0, -1e6, -np.inf], dtype=np.float32))
    assert np.all(np.isfinite(got)) and np.all(got > 0) and np.all(got <= 2.0 ** -124.9)
