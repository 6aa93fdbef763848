"""The one-launch amax + quantize path (fused_quantize_kernel, taken by batches of two or
more tensors) against the oracle, around every switch of its launch plan, and its bounded
wait made to give up on purpose.

Amax and quantize tiles of 896 blocks (7 quantize warps x 2 units x 2 blocks): ragged
last tiles, one and several tiles, two and three tensors, jobs within one wave of CTAs
and jobs over several waves (the amax warps then run ahead of the quantize warps, up to
a tensor and one and a half grids), the largest tensors the launch takes (64 MiB of bf16
each) and the next size, which takes the separate amax pass, as does a single tensor; two
blocks per thread and one (packed / scales alignment)."""
import numpy as np
import pytest
import torch

import nvfp4_kv_cache_kvq_b200 as kvq
from gpu_helpers import assert_same, check_sampled
from nvfp4_kv_cache_kvq_b200.inputs import bits

pytestmark = pytest.mark.gpu


def _x(rows, seed, device="cuda"):
    g = torch.Generator(device="cpu").manual_seed(seed)
    x = torch.randn(rows, 128, generator=g) * torch.exp(torch.randn(rows, 1, generator=g))
    return x.to(torch.bfloat16).to(device)


def _check_batch(orc, xs, rule, offset_bytes=0):
    """kvq_quantize_batch (amax computed) on xs, every output compared with the oracle.
    offset_bytes shifts packed and scales off their 16- and 2-byte alignment."""
    n = xs[0].numel()
    pk = [torch.empty(n // 2 + 16, dtype=torch.uint8, device="cuda")[offset_bytes:offset_bytes + n // 2]
          for _ in xs]
    sc = [torch.empty(n // 16 + 16, dtype=torch.uint8, device="cuda")[offset_bytes:offset_bytes + n // 16]
          for _ in xs]
    p, s, a = kvq.kvq_quantize_batch(xs, 128, rule, packed=pk, scales=sc)
    torch.cuda.synchronize()
    kvq.kvq_device_status()
    for x, pi, si, ai in zip(xs, p, s, a):
        pe, se, ae = orc.quantize(bits(x), 128, rule)
        assert float(ai.cpu()[0]) == ae
        assert_same(si.cpu().numpy(), se, f"scales[{rule}]")
        assert_same(pi.cpu().numpy(), pe, f"packed[{rule}]")


@pytest.mark.parametrize("blocks", [8, 888, 896, 904, 65536 + 8])
@pytest.mark.parametrize("n_tensors", [2, 3])
def test_plan_switch_tile_size(orc, blocks, n_tensors):
    rows = -(-blocks // 8)
    xs = [_x(rows, 100 * n_tensors + i) for i in range(n_tensors)]
    _check_batch(orc, xs, "mse")


@pytest.mark.parametrize("rule", ["static_6", "static_4", "mse"])
def test_two_tensors_and_unaligned_codes(orc, rule):
    xs = [_x(9001, 5), _x(9001, 6)]
    _check_batch(orc, xs, rule)
    _check_batch(orc, xs, rule, offset_bytes=8)  # packed not 16-byte aligned: one block per thread


def test_several_waves(orc):
    """Three tensors of 2^20 blocks (3072 tiles, several waves of CTAs): whole-tensor parity
    on the first, sampled on the others."""
    xs = [_x(131072, 7 + i) for i in range(3)]
    p, s, a = kvq.kvq_quantize_batch(xs, 128, "mse")
    torch.cuda.synchronize()
    kvq.kvq_device_status()
    pe, se, ae = orc.quantize(bits(xs[0]), 128, "mse")
    assert float(a[0].cpu()[0]) == ae
    assert_same(s[0].cpu().numpy(), se, "scales")
    assert_same(p[0].cpu().numpy(), pe, "packed")
    for i in (1, 2):
        check_sampled(orc, xs[i], p[i], s[i], float(a[i].cpu()[0]), None, "mse", seed=i)


def test_largest_one_launch_tensors_and_the_two_pass_above(orc):
    """2^21 blocks (64 MiB of bf16) is the largest tensor of the one-launch path; one row
    more takes the separate amax pass. A single tensor always does."""
    assert kvq.kvq_quantize_launches(1, 1024 * 128) == 3
    assert kvq.kvq_quantize_launches(65, 1024 * 128) == 2 + 3  # a group of 64, then one
    for rows in (262_144, 262_145):
        assert kvq.kvq_quantize_launches(2, rows * 128) == (2 if rows == 262_144 else 3)
        xs = [_x(rows, 9), _x(rows, 10)]
        p, s, a = kvq.kvq_quantize_batch(xs, 128, "mse")
        torch.cuda.synchronize()
        kvq.kvq_device_status()
        for i in range(2):
            check_sampled(orc, xs[i], p[i], s[i], float(a[i].cpu()[0]), None, "mse", seed=i)
        del xs, p, s, a


def test_bounded_wait_gives_up_and_the_next_call_is_correct(orc):
    """With the test hook, every quantize tile waits for one amax tile more than exist;
    the wait gives up after 2 ms: nothing is written, the amax is NaN, and
    kvq_device_status reports the timeout. Then the same calls without the hook are
    exact, on the same stream, in the same process."""
    xs = [_x(4096, 12), _x(4096, 13)]
    n = xs[0].numel()
    packed = [torch.full((n // 2,), 0xA5, dtype=torch.uint8, device="cuda") for _ in xs]
    scales = [torch.full((n // 16,), 0x5A, dtype=torch.uint8, device="cuda") for _ in xs]
    amax = [torch.zeros(1, dtype=torch.float32, device="cuda") for _ in xs]
    kvq.kvq_device_status()  # clear
    try:
        kvq.testing_set_fused_wait(1, 2_000_000)
        kvq.kvq_quantize_batch(xs, 128, "mse", amax_out=amax, packed=packed, scales=scales)
        torch.cuda.synchronize()
    finally:
        kvq.testing_set_fused_wait(0, 0)
    with pytest.raises(kvq.KvqError) as e:
        kvq.kvq_device_status()
    assert e.value.status == 6
    kvq.kvq_device_status()  # cleared by the call above
    for i in range(2):
        assert torch.isnan(amax[i]).all()
        assert bool((packed[i] == 0xA5).all()) and bool((scales[i] == 0x5A).all())
    # an append under the hook times out the same way
    caches = kvq.allocate_caches(1, 1, 4096, 128, 4096, "cuda")
    try:
        kvq.testing_set_fused_wait(1, 2_000_000)
        kvq.kvq_append_batch(caches, [0, 0], xs, "mse")
        torch.cuda.synchronize()
    finally:
        kvq.testing_set_fused_wait(0, 0)
    with pytest.raises(kvq.KvqError):
        kvq.kvq_device_status()
    # normal operation resumes
    kvq.kvq_quantize_batch(xs, 128, "mse", amax_out=amax, packed=packed, scales=scales)
    kvq.kvq_append_batch(caches, [0, 0], xs, "mse")
    torch.cuda.synchronize()
    kvq.kvq_device_status()
    for i in range(2):
        pe, se, ae = orc.quantize(bits(xs[i]), 128, "mse")
        assert float(amax[i].cpu()[0]) == ae and float(caches[i].amax.cpu()[0]) == ae
        assert_same(packed[i].cpu().numpy(), pe, "packed")
        assert_same(scales[i].cpu().numpy(), se, "scales")
        assert_same(caches[i].packed.cpu().numpy(), pe, "cache packed")
        assert np.array_equal(caches[i].scales.cpu().numpy(), se)
