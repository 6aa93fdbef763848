"""Pins of the oracle's RECENT cache policy (RTN_INT4 RECENT2 of the Self-Forcing study,
appendix Table 3) against its definition written out directly: after appending blocks
x_0 .. x_{n-1}, the cache reads back RTN(x_b) round-tripped for b < n - R and x_b
itself for the R newest blocks."""
import numpy as np
import pytest

from nvfp4_kv_cache_kvq_b200 import inputs
from nvfp4_kv_cache_kvq_b200.inputs import bits

D = 128


def _blocks(n, rows, seed):
    return [bits(inputs.student_t((rows, D), 4, seed + b)) for b in range(n)]


@pytest.mark.parametrize("R,bits_,n", [(2, 4, 7), (1, 4, 3), (3, 2, 5), (2, 4, 1), (2, 4, 2)])
def test_recent_cache_matches_definition(orc, R, bits_, n):
    rows = 24
    xs = _blocks(n, rows, 40)
    c = orc.RecentCache(rows, D, bits_, R)
    for b, x in enumerate(xs):
        c.append(x)
        m = b + 1
        want = [orc.rtn_dequantize(*orc.rtn_quantize(xs[i], D, bits_), D, bits_) for i in range(max(0, m - R))]
        want += [xs[i] for i in range(max(0, m - R), m)]
        np.testing.assert_array_equal(c.read(), np.concatenate(want))


def test_recent_tail_is_exact_and_prefix_is_lossy(orc):
    rows = 32
    xs = _blocks(4, rows, 90)
    c = orc.RecentCache(rows, D, 4, 2)
    for x in xs:
        c.append(x)
    y = c.read().reshape(4, -1)
    # the two newest blocks are the inputs bit for bit; the quantized ones are not
    np.testing.assert_array_equal(y[2], xs[2])
    np.testing.assert_array_equal(y[3], xs[3])
    assert not np.array_equal(y[0], xs[0]) and not np.array_equal(y[1], xs[1])
