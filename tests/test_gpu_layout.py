"""The blocked scale layout kernels against the oracle, on the scales of a real
quantization and on odd shapes."""
import numpy as np
import pytest
import torch

import nvfp4_kv_cache_kvq_b200 as kvq
from gpu_helpers import assert_same
from nvfp4_kv_cache_kvq_b200 import inputs
from nvfp4_kv_cache_kvq_b200.inputs import bits

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("rows,cols", [(1, 1), (5, 8), (128, 4), (130, 8), (300, 9), (4680 * 24, 8)])
def test_blocked_round_trip(orc, rows, cols):
    rng = np.random.default_rng(rows + cols)
    m = rng.integers(0, 256, rows * cols, dtype=np.uint8)
    d = torch.from_numpy(m).cuda()
    b = kvq.kvq_scales_to_blocked(d, rows, cols)
    back = kvq.kvq_scales_from_blocked(b, rows, cols)
    torch.cuda.synchronize()
    assert b.numel() == kvq.kvq_blocked_scale_bytes(rows, cols)
    assert_same(b.cpu().numpy(), orc.scales_to_blocked(m, rows, cols), "blocked")
    assert_same(back.cpu().numpy(), m, "from_blocked")


@pytest.mark.parametrize("cols", [4, 8])
def test_blocked_byte_path_for_unaligned_scales(orc, cols):
    """A plain buffer that is not 4-byte aligned takes the byte-by-byte path, in both
    directions, with the same results."""
    rows = 300
    rng = np.random.default_rng(cols)
    m = rng.integers(0, 256, rows * cols, dtype=np.uint8)
    buf = torch.zeros(rows * cols + 1, dtype=torch.uint8, device="cuda")
    d = buf[1:]
    d.copy_(torch.from_numpy(m))
    assert d.data_ptr() % 4 != 0
    b = kvq.kvq_scales_to_blocked(d, rows, cols)
    out = torch.zeros(rows * cols + 1, dtype=torch.uint8, device="cuda")
    back = kvq.kvq_scales_from_blocked(b, rows, cols, scales=out[1:])
    torch.cuda.synchronize()
    assert_same(b.cpu().numpy(), orc.scales_to_blocked(m, rows, cols), "blocked")
    assert_same(back.cpu().numpy(), m, "from_blocked")
    assert int(out[0].item()) == 0


def test_blocked_buffer_alignment_is_checked():
    m = torch.zeros(128 * 8, dtype=torch.uint8, device="cuda")
    buf = torch.zeros(kvq.kvq_blocked_scale_bytes(128, 8) + 16, dtype=torch.uint8, device="cuda")
    with pytest.raises(kvq.KvqError):
        kvq.kvq_scales_to_blocked(m, 128, 8, blocked=buf[4:4 + kvq.kvq_blocked_scale_bytes(128, 8)])
    with pytest.raises(kvq.KvqError):
        kvq.kvq_scales_from_blocked(buf[4:4 + kvq.kvq_blocked_scale_bytes(128, 8)], 128, 8)


def test_blocked_scales_of_a_quantized_layer(orc):
    x = inputs.layer_kv(0, heads=3, tokens=777, device="cuda")
    _, scales, _ = kvq.kvq_quantize(x, 128, "mse")
    rows, cols = x.numel() // 128, 8
    b = kvq.kvq_scales_to_blocked(scales, rows, cols)
    torch.cuda.synchronize()
    _, want_scales, _ = orc.quantize(bits(x), 128, "mse")
    assert_same(b.cpu().numpy(), orc.scales_to_blocked(want_scales, rows, cols), "blocked")
