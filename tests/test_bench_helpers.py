"""The bench line's reported quantities, on the CPU: the relative MSE summed in passes of
any size equals the sum taken at once (numpy, fp64), and the footprint of the NVFP4 form
is 4.5 bits per element plus one amax per tensor (the ratio 16 / 4.5 for large tensors)."""
import os
import sys

import numpy as np
import torch

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import bench  # noqa: E402


def _pair(n, seed):
    g = torch.Generator().manual_seed(seed)
    x = (torch.randn(n, generator=g) * 3).to(torch.bfloat16)
    y = (x.float() + torch.randn(n, generator=g) * 0.05).to(torch.bfloat16)
    return x, y


def test_rel_mse_in_passes_equals_one_sum():
    xs, ys = zip(*(_pair(n, s) for s, n in enumerate((1, 7, 1000, 4099))))
    xf = np.concatenate([x.float().numpy().astype(np.float64) for x in xs])
    yf = np.concatenate([y.float().numpy().astype(np.float64) for y in ys])
    want = ((yf - xf) ** 2).sum() / (xf ** 2).sum()
    for step in (1, 3, 7, 64, 1 << 26):
        got = bench.rel_mse(list(xs), list(ys), step=step)
        assert abs(got - want) <= 1e-12 * want


def test_rel_mse_of_zero_tensors_is_zero():
    z = torch.zeros(10, dtype=torch.bfloat16)
    assert bench.rel_mse([z], [z]) == 0.0


def test_footprint_of_the_nvfp4_form():
    elems = 60 * 93600 * 12 * 128
    f = bench.footprint(elems // 2, elems // 16, 60 * 60 * 4, elems, 575078400)
    assert f["quantized_bytes"] == elems // 2 + elems // 16 + 14400
    assert f["bf16_bytes"] == 2 * elems
    assert f["ratio"] == 2 * elems / (elems // 2 + elems // 16 + 14400)
    assert abs(f["ratio"] - 16 / 4.5) < 2e-5  # the amax words are 14.4 KB of 4.85 GB
    assert f["transient_bf16_bytes"] == 575078400
    assert bench.footprint(0, 0, 0, 0)["ratio"] is None
