"""The fused attention's division-free global scale: gs = RN(amax / 2688) by Markstein's
correction step (P. Markstein, "Computation of elementary functions on the IBM RISC
System/6000 processor", IBM J. Res. Dev. 34(1), 1990) with y = RN(1/2688):
q = RN(amax y), r = fma(-q, 2688, amax), gs = fma(r, y, q). The kernel takes this path
only when every chunk amax of a CTA's keys is in [kMarkMinAmax, FLT_MAX]; this test reads
the kernel's constants from its source and checks, with C's correctly rounded fmaf, that
the step equals the IEEE quotient there (every fp32 value in the binades next to the
threshold, and a seeded sample of the whole range) and that it does not just below (where
the quotient is subnormal, the kernel divides)."""
import ctypes
import os
import random
import re
import subprocess
import tempfile

import pytest

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "nvfp4_kv_cache_kvq_b200", "csrc",
                   "kvq_attention.cu")

C_SRC = r"""
#include <math.h>
#include <stdint.h>
#include <string.h>
static float f(uint32_t u) { float x; memcpy(&x, &u, 4); return x; }
static uint32_t u(float x) { uint32_t v; memcpy(&v, &x, 4); return v; }
static int same(float a, float y, float den) {
    const float q = a * y;
    const float r = fmaf(-q, den, a);
    const float m = fmaf(r, y, q);
    return u(m) == u(a / den);
}
/* mismatches over the fp32 bit patterns [lo, hi) */
uint64_t mismatches(uint32_t lo, uint32_t hi, float y, float den) {
    uint64_t bad = 0;
    for (uint32_t k = lo; k < hi; ++k)
        bad += !same(f(k), y, den);
    return bad;
}
/* mismatches over n given bit patterns */
uint64_t mismatches_at(const uint32_t* ks, uint64_t n, float y, float den) {
    uint64_t bad = 0;
    for (uint64_t i = 0; i < n; ++i)
        bad += !same(f(ks[i]), y, den);
    return bad;
}
"""


def _hexfloat(src: str, name: str) -> float:
    m = re.search(name + r"\s*=\s*(0x[0-9a-fA-F.]+p[-+]?\d+)f", src)
    assert m, name
    return float.fromhex(m.group(1))


@pytest.fixture(scope="module")
def lib():
    with tempfile.TemporaryDirectory() as d:
        c = os.path.join(d, "gs.c")
        so = os.path.join(d, "gs.so")
        with open(c, "w") as fh:
            fh.write(C_SRC)
        # no -ffast-math, no contraction: a * y and a / den round once each, fmaf is fused
        subprocess.run(["gcc", "-O2", "-ffp-contract=off", "-fPIC", "-shared", "-o", so, c, "-lm"], check=True)
        h = ctypes.CDLL(so)
        h.mismatches.restype = ctypes.c_uint64
        h.mismatches.argtypes = [ctypes.c_uint32, ctypes.c_uint32, ctypes.c_float, ctypes.c_float]
        h.mismatches_at.restype = ctypes.c_uint64
        h.mismatches_at.argtypes = [ctypes.POINTER(ctypes.c_uint32), ctypes.c_uint64, ctypes.c_float, ctypes.c_float]
        yield h


def _bits(x: float) -> int:
    return ctypes.c_uint32.from_buffer(ctypes.c_float(x)).value


def test_constants_and_threshold(lib):
    src = open(SRC).read()
    y = _hexfloat(src, "kInvDen")
    lo = _hexfloat(src, "kMarkMinAmax")
    assert ctypes.c_float(y).value == y  # an fp32 value
    # y is RN(1/2688): within half an ulp of the reciprocal
    ulp = 2.0 ** (-12 - 23)
    assert abs(y - 1.0 / 2688.0) <= ulp / 2
    assert "2688.0f" in src
    # every fp32 amax in the 5 binades from the threshold up, through the whole range where
    # the quotient amax / 2688 is subnormal (amax below about 2^-114.6) and into normal
    # quotients: the IEEE quotient
    assert lib.mismatches(_bits(lo), _bits(lo * 32.0), y, 2688.0) == 0
    # just below it the step is not exact (the quotient is subnormal): the kernel divides
    assert lib.mismatches(_bits(lo / 4.0), _bits(lo), y, 2688.0) > 0


def test_sample_of_the_whole_range(lib):
    src = open(SRC).read()
    y = _hexfloat(src, "kInvDen")
    lo = _bits(_hexfloat(src, "kMarkMinAmax"))
    hi = 0x7F800000  # +inf: the range ends at FLT_MAX
    rng = random.Random(2688)
    ks = [rng.randrange(lo, hi) for _ in range(1 << 20)]
    # the largest finite values, and powers of two across the range
    ks += list(range(hi - 4096, hi)) + [e << 23 for e in range((lo >> 23) + 1, 255)]
    arr = (ctypes.c_uint32 * len(ks))(*ks)
    assert lib.mismatches_at(arr, len(ks), y, 2688.0) == 0
