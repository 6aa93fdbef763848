"""Whole tensors through the oracle against the exact-rational restatement
(tests/exact_fp32.py): the tensor amax, every block's scale code and packed codes under the
three rules, and the dequantized bf16 values, y = bf16(fp32(e2m1(q) * S)) with
S = fp32(e4m3(c) * gs) ("How NVFP4 Quantization Works in LongLive 2.0 for Transformer
Inference", "Stage 3" steps 2-3; the even element in the low nibble)."""
from fractions import Fraction

import numpy as np
import pytest

import exact_fp32 as ex
from golden_io import round_to_bf16_bits


def _tensor(rng, blocks):
    v = rng.standard_t(4, 16 * blocks) * np.repeat(2.0 ** rng.integers(-12, 4, blocks), 16)
    v[rng.integers(0, v.size, 5)] = 0.0
    v[rng.integers(0, v.size, 3)] *= -0.0
    return round_to_bf16_bits(v * 2.0 ** int(rng.integers(-30, 30)))


@pytest.mark.parametrize("rule", ["static_6", "static_4", "mse"])
def test_whole_tensor_equals_exact_restatement(orc, rule):
    rng = np.random.default_rng({"static_6": 1, "static_4": 2, "mse": 3}[rule])
    for _ in range(6):
        blocks = int(rng.integers(1, 40))
        x = _tensor(rng, blocks)
        packed, scales, amax = orc.quantize(x, 16, rule)
        y = orc.dequantize(packed, scales, amax, 16)
        xs = [ex.bf16_value(int(b)) for b in x]
        amax_t = max(abs(t) for t in xs)
        assert Fraction(amax) == amax_t
        gs = ex.rn32(amax_t / 2688)
        for k in range(blocks):
            xb = [int(b) for b in x[16 * k:16 * k + 16]]
            if rule == "mse":
                c, codes, _, _ = ex.mse_block(xb, amax_t)
            else:
                c, _, codes = ex.candidate(xb, amax_t, 6 if rule == "static_6" else 4)
            assert scales[k] == c, (rule, k)
            want_packed = [codes[2 * j] | (codes[2 * j + 1] << 4) for j in range(8)]
            assert packed[8 * k:8 * k + 8].tolist() == want_packed, (rule, k)
            S = ex.rn32(ex.e4m3_value(c) * gs)
            for i in range(16):
                want = ex.rn_bf16(ex.rn32(ex.e2m1_value(codes[i]) * S))
                got = int(y[16 * k + i])
                assert ex.bf16_value(got) == want, (rule, k, i)
                if want == 0:  # the sign of zero is the code's sign
                    assert (got >> 15) == (codes[i] >> 3), (rule, k, i)
