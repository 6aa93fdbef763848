"""Shared helpers of the GPU parity tests: run the CUDA path through the C ABI binding,
run the oracle on the same bytes, compare bit for bit."""
import numpy as np
import torch

import nvfp4_kv_cache_kvq_b200 as kvq
from nvfp4_kv_cache_kvq_b200.inputs import bits


def gpu_round_trip(x: torch.Tensor, rule, head_dim: int):
    packed, scales, amax = kvq.kvq_quantize(x, head_dim, rule)
    y = kvq.kvq_dequantize(packed, scales, amax, head_dim)
    torch.cuda.synchronize()
    return packed.cpu().numpy(), scales.cpu().numpy(), float(amax.cpu()[0]), bits(y)


def assert_same(got: np.ndarray, want: np.ndarray, what: str):
    got = np.asarray(got).reshape(-1)
    want = np.asarray(want).reshape(-1)
    assert got.shape == want.shape, (what, got.shape, want.shape)
    bad = np.nonzero(got != want)[0]
    if bad.size:
        i = bad[:8]
        raise AssertionError(f"{what}: {bad.size} of {got.size} differ; first at {i.tolist()}: "
                             f"got {got[i].tolist()} want {want[i].tolist()}")


def check_full(orc, x: torch.Tensor, rule, head_dim: int):
    """Whole-tensor bit-exact parity of quantize and dequantize."""
    p, s, a, y = gpu_round_trip(x, rule, head_dim)
    xb = bits(x)
    pe, se, ae = orc.quantize(xb, head_dim, rule)
    assert a == ae, (a, ae)
    assert_same(s, se, f"scales[{rule}]")
    assert_same(p, pe, f"packed[{rule}]")
    assert_same(y, orc.dequantize(pe, se, ae, head_dim), f"dequant[{rule}]")
    return p, s, a, y


def check_sampled(orc, x: torch.Tensor, packed: torch.Tensor, scales: torch.Tensor, amax: float,
                  y: torch.Tensor, rule, n_samples: int = 4096, seed: int = 0):
    """Parity at any size: the kernel's amax against torch's max |x| (an exact library
    reduction), then n_samples random blocks quantized and dequantized one by one by the
    oracle under torch's amax. Nothing the CUDA path produced is fed to the oracle."""
    xf = x.reshape(-1)
    ref_amax = float(xf.abs().max().float())
    assert amax == ref_amax, ("amax", amax, ref_amax)
    amax = ref_amax
    nb = xf.numel() // 16
    g = torch.Generator().manual_seed(seed)
    idx = torch.randint(0, nb, (min(n_samples, nb),), generator=g)
    idx = torch.cat([idx, torch.tensor([0, nb - 1])])
    idx_d = idx.to(x.device)
    xb = bits(xf.view(-1, 16)[idx_d])
    pe, se, _ = orc.quantize(xb, 16, rule, amax_in=amax)
    assert_same(scales.reshape(-1)[idx_d].cpu().numpy(), se, "sampled scales")
    assert_same(packed.reshape(-1, 8)[idx_d].cpu().numpy(), pe, "sampled packed")
    if y is not None:
        assert_same(bits(y.reshape(-1, 16)[idx_d]), orc.dequantize(pe, se, amax, 16), "sampled dequant")
