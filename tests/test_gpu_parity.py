"""Bit-exact parity of the CUDA path (through the C ABI) against the CPU oracle:
packed codes, e4m3 scales, amax and dequantized bf16, on the five workloads' inputs and
on the edge cases. Floating point decides integers here (codes, scales), so the bar is
bit equality everywhere, including the sign of zero."""
import os

import numpy as np
import pytest
import torch

import nvfp4_kv_cache_kvq_b200 as kvq
from golden_io import floats_to_bf16_bits, hex_bytes, read_sections
from gpu_helpers import assert_same, check_full, check_sampled, gpu_round_trip
from nvfp4_kv_cache_kvq_b200 import inputs
from nvfp4_kv_cache_kvq_b200.inputs import bits

pytestmark = pytest.mark.gpu
RULES = ("static_6", "static_4", "mse")


def _bf16(bits_np: np.ndarray, device="cuda") -> torch.Tensor:
    return torch.from_numpy(bits_np.astype(np.uint16).view(np.int16).copy()).view(torch.bfloat16).to(device)


def test_library_loaded_in_tree():
    kvq.load()
    maps = open("/proc/self/maps").read()
    assert kvq.library_path() in maps
    assert os.path.dirname(os.path.dirname(kvq.library_path())) == os.path.dirname(kvq.__file__)


@pytest.mark.parametrize("rule", RULES)
def test_worked_example_on_gpu(rule):
    g = read_sections("worked_example.txt")
    x = _bf16(floats_to_bf16_bits(g["input"]))
    p, s, a, y = gpu_round_trip(x, rule, 16)
    assert a == float(g["amax"][0])
    assert_same(s, hex_bytes(g[f"{rule}.scales"]), "scales")
    assert_same(p, hex_bytes(g[f"{rule}.packed"]), "packed")
    assert_same(y, floats_to_bf16_bits(g[f"{rule}.dequant"]), "dequant")


def test_mse_near_tie_blocks_on_gpu(orc):
    """The hand-worked near-tie blocks, whose choice depends on the order of the error
    sum: as given, then tiled over many CTAs, through quantize and through append."""
    g = read_sections("mse_near_ties.txt")
    x = floats_to_bf16_bits(g["input"])
    p, s, a, y = gpu_round_trip(_bf16(x), "mse", 16)
    assert a == float(g["amax"][0])
    assert_same(s, hex_bytes(g["fma_even_odd.scales"]), "scales")
    assert_same(p, hex_bytes(g["fma_even_odd.packed"]), "packed")
    big = np.tile(x, 4096)  # 1536 rows of 128
    check_full(orc, _bf16(big), "mse", 128)
    rows = big.size // 128
    cache = kvq.allocate_caches(1, 1, rows, 128, rows, "cuda")[0]
    kvq.kvq_append(cache, 0, _bf16(big).view(rows, 128), "mse")
    torch.cuda.synchronize()
    pe, se, ae = orc.quantize(big, 128, "mse")
    assert float(cache.amax.cpu()[0]) == ae
    assert_same(cache.scales.cpu().numpy(), se, "append scales")
    assert_same(cache.packed.cpu().numpy(), pe, "append packed")


@pytest.mark.parametrize("rule", RULES)
def test_single_k(orc, rule):
    """[4096, 128] N(0,1), seed 0."""
    check_full(orc, inputs.single_k("cuda"), rule, 128)


@pytest.mark.parametrize("rule", RULES)
def test_layer_kv(orc, rule):
    """One layer's K and V, [1, 24, 4680, 128], Student-t(3) with outlier channels."""
    for kv in (0, 1):
        check_full(orc, inputs.layer_kv(kv, device="cuda"), rule, 128)


@pytest.mark.parametrize("rule", RULES)
def test_layer_kv_batched_as_the_benchmark_runs_it(orc, rule):
    """The layer workload in the benchmark's launch configuration: K and V in one
    kvq_quantize_batch (the amax and the codes in one launch) and one kvq_dequantize_batch,
    whole tensors against the oracle."""
    xs = [inputs.layer_kv(kv, device="cuda") for kv in (0, 1)]
    assert kvq.kvq_quantize_launches(2, xs[0].numel()) == 2
    p, s, a = kvq.kvq_quantize_batch(xs, 128, rule)
    ys = kvq.kvq_dequantize_batch(p, s, a, 128)
    torch.cuda.synchronize()
    kvq.kvq_device_status()
    for i, x in enumerate(xs):
        pe, se, ae = orc.quantize(bits(x), 128, rule)
        assert float(a[i][0]) == ae
        assert_same(s[i].cpu().numpy(), se, f"scales t{i}")
        assert_same(p[i].cpu().numpy(), pe, f"packed t{i}")
        assert_same(bits(ys[i]), orc.dequantize(pe, se, ae, 128), f"dequant t{i}")


def _all_bf16(lo: float, hi: float) -> np.ndarray:
    """Every finite bf16 bit pattern with lo <= value <= hi (both signs if lo < 0)."""
    u = np.arange(0, 1 << 16, dtype=np.uint32).astype(np.uint16)
    f = torch.from_numpy(u.view(np.int16)).view(torch.bfloat16).float().numpy()
    keep = np.isfinite(f) & (f >= lo) & (f <= hi)
    return u[keep]


@pytest.mark.parametrize("rule", ["static_6", "static_4"])
def test_e2m1_rounding_of_every_bf16(orc, rule):
    """Blocks of 15 swept values + one 6: with gs = 1 (a 2688 elsewhere) static_6 gives
    S = 1 (codes are e2m1(x) straight from the hardware cvt, every tie included) and
    static_4 gives S = 1.5 (codes of the fp32 products x * (1/1.5))."""
    vals = _all_bf16(-6.0, 6.0)
    pad = (-vals.size) % 15
    vals = np.concatenate([vals, np.zeros(pad, np.uint16)]).reshape(-1, 15)
    six = floats_to_bf16_bits([6.0])[0]
    blocks = np.concatenate([np.full((vals.shape[0], 1), six, np.uint16), vals], 1)
    head = np.concatenate([floats_to_bf16_bits([2688.0]), np.zeros(15, np.uint16)])[None]
    x = np.concatenate([head, blocks]).reshape(-1)
    check_full(orc, _bf16(x), rule, 16)


@pytest.mark.parametrize("rule", RULES)
def test_e4m3_scale_rounding_of_every_bf16_amax(orc, rule):
    """One block per positive bf16 amax in [2^-16, 2688] with gs = 1: covers every e4m3
    scale rounding, subnormal scales, ties and saturation."""
    amaxes = _all_bf16(2.0 ** -16, 2688.0)
    blocks = np.zeros((amaxes.size, 16), np.uint16)
    blocks[:, 0] = amaxes
    blocks[:, 1] = amaxes ^ 0x8000
    blocks[:, 2] = amaxes - 1
    blocks[:, 3:] = (amaxes[:, None] >> 1) & 0x7FFF
    head = np.concatenate([floats_to_bf16_bits([2688.0]), np.zeros(15, np.uint16)])[None]
    x = np.concatenate([head, blocks]).reshape(-1)
    check_full(orc, _bf16(x), rule, 16)


def _ulp_step(v, d):
    """v moved by d fp32 ulps."""
    v = np.float32(v)
    for _ in range(abs(d)):
        v = np.nextafter(v, np.float32(np.inf) if d > 0 else np.float32(0))
    return float(v)


@pytest.mark.parametrize("rule", ["static_6", "static_4", "mse"])
def test_scale_quotients_at_e4m3_midpoints(orc, rule):
    """The scale code is e4m3((amax_b / R) / gs): pick amax_in (hence gs) so that the
    quotient lands on, or a few ulps around, e4m3 rounding midpoints. The code then
    hinges on the correctly rounded quotient, which the kernel computes without a
    division (a corrected reciprocal product); the oracle divides."""
    R = 4.0 if rule == "static_4" else 6.0
    mags = np.array([orc.e4m3_decode(c) for c in range(127)])
    mids = (mags[:-1] + mags[1:]) / 2
    rng = np.random.default_rng(21)
    a_vals = np.float32([1.0, 0.75, 3.0, 0.5625, 11.0, 1.9375])
    n_checked = 0
    for k in range(0, 126, 3):
        a = float(a_vals[k % a_vals.size])
        s32 = np.float32(a) / np.float32(R) if R == 6.0 else np.float32(a) * np.float32(0.25)
        target = np.float32(float(s32) / mids[k] * 2688.0)
        for d in (-2, -1, 0, 1, 2):
            amax_in = _ulp_step(target, d)
            blk = np.concatenate([[a], rng.uniform(-a, a, 15)])
            x = torch.from_numpy(np.concatenate([blk, rng.standard_normal(16 * 7) * a / 3])).to(torch.bfloat16)
            p, sc, _ = kvq.kvq_quantize(x.cuda(), 16, rule, amax_in=torch.tensor([amax_in], device="cuda"))
            torch.cuda.synchronize()
            pe, se, _ = orc.quantize(bits(x), 16, rule, amax_in=amax_in)
            assert_same(sc.cpu().numpy(), se, f"scales at midpoint {k} d={d}")
            assert_same(p.cpu().numpy(), pe, f"packed at midpoint {k} d={d}")
            n_checked += 1
    assert n_checked == 42 * 5


def test_empty_tensor():
    x = torch.empty(0, dtype=torch.bfloat16, device="cuda")
    amax = torch.full((1,), 5.0, device="cuda")
    p, s, a = kvq.kvq_quantize(x, 128, "mse", amax_out=amax)
    y = kvq.kvq_dequantize(p, s, a, 128)
    torch.cuda.synchronize()
    assert p.numel() == 0 and s.numel() == 0 and y.numel() == 0 and float(amax[0]) == 0.0


@pytest.mark.parametrize("rule", RULES)
def test_zero_tensor_with_signed_zeros(orc, rule):
    x = np.zeros(128 * 5, np.uint16)
    x[1::3] = 0x8000
    p, s, a, y = check_full(orc, _bf16(x), rule, 128)
    assert a == 0.0 and not s.any()
    assert_same(y, x, "signed zeros round trip")


@pytest.mark.parametrize("head_dim,rows", [(16, 1), (16, 7), (48, 5), (144, 3), (256, 9), (128, 4097)])
@pytest.mark.parametrize("rule", RULES)
def test_ragged_shapes(orc, head_dim, rows, rule):
    """Odd block counts (the pair kernel's tail) and row lengths that are not powers of 2."""
    x = inputs.normal((rows, head_dim), seed=head_dim * 1000 + rows, device="cuda")
    check_full(orc, x, rule, head_dim)


@pytest.mark.parametrize("rule", RULES)
def test_unaligned_packed_takes_single_block_path(orc, rule):
    """packed only 8-byte aligned, scales odd: the one-block-per-thread kernel."""
    x = inputs.normal((33, 128), seed=5, device="cuda")
    n = x.numel()
    pbuf = torch.zeros(n // 2 + 8, dtype=torch.uint8, device="cuda")
    sbuf = torch.zeros(n // 16 + 1, dtype=torch.uint8, device="cuda")
    packed, scales = pbuf[8:], sbuf[1:]
    _, _, amax = kvq.kvq_quantize(x, 128, rule, packed=packed, scales=scales)
    y = kvq.kvq_dequantize(packed, scales, amax, 128)
    torch.cuda.synchronize()
    pe, se, ae = orc.quantize(bits(x), 128, rule)
    assert_same(packed.cpu().numpy(), pe, "packed")
    assert_same(scales.cpu().numpy(), se, "scales")
    assert_same(bits(y), orc.dequantize(pe, se, ae, 128), "dequant")


def test_extreme_magnitudes(orc):
    rng = np.random.default_rng(1)
    for scale in (1e-38, 1e-40, 2.0 ** -130, 1e30, 5.0e37):
        v = rng.standard_normal(128 * 8) * scale
        x = torch.from_numpy(v).to(torch.bfloat16).cuda()
        for rule in RULES:
            check_full(orc, x, rule, 128)


@pytest.mark.parametrize("rule", RULES)
def test_single_outlier(orc, rule):
    x = inputs.normal((64, 128), seed=3)
    x[17, 5] = -4096.0
    check_full(orc, x.cuda(), rule, 128)


@pytest.mark.parametrize("rule", RULES)
def test_amax_in(orc, rule):
    x = inputs.normal((257, 128), seed=8, device="cuda")
    true_amax = float(x.abs().max().float())
    for given in (true_amax, true_amax / 8, true_amax * 3, 0.0):
        amax_in = torch.tensor([given], dtype=torch.float32, device="cuda")
        amax_out = torch.full((1,), -1.0, device="cuda")
        p, s, _ = kvq.kvq_quantize(x, 128, rule, amax_in=amax_in, amax_out=amax_out)
        y = kvq.kvq_dequantize(p, s, amax_in, 128)
        torch.cuda.synchronize()
        assert float(amax_out[0]) == given
        pe, se, _ = orc.quantize(bits(x), 128, rule, amax_in=given)
        assert_same(s.cpu().numpy(), se, f"scales amax_in={given}")
        assert_same(p.cpu().numpy(), pe, f"packed amax_in={given}")
        assert_same(bits(y), orc.dequantize(pe, se, given, 128), f"dequant amax_in={given}")


def test_stream_ordering_on_side_stream(orc):
    x = inputs.normal((512, 128), seed=9, device="cuda")
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        p, sc, a = kvq.kvq_quantize(x, 128, "mse")
        y = kvq.kvq_dequantize(p, sc, a, 128)
    s.synchronize()
    pe, se, ae = orc.quantize(bits(x), 128, "mse")
    assert_same(bits(y), orc.dequantize(pe, se, ae, 128), "dequant on side stream")


# ---------------------------------------------------------------- cache (append / read)

def _rollout(orc, layers, heads, tokens, steps, capacity_frames, rule, check_every=1):
    """Append `steps` chunks to 2*layers caches through kvq_append_batch, reading the
    whole prefix back after each step through kvq_dequantize_cache_batch, against the
    oracle's caches."""
    D = 128
    caches = kvq.allocate_caches(layers, heads, capacity_frames * tokens, D, tokens)
    rpc = tokens * heads
    ocs = [orc.Cache(capacity_frames * rpc, rpc, D) for _ in caches]
    for step in range(steps):
        xs = [inputs.rollout_chunk(step, t, heads=heads, tokens=tokens, device="cuda") for t in range(len(caches))]
        kvq.kvq_append_batch(caches, [step * rpc] * len(caches), xs, rule)
        for oc, xt in zip(ocs, xs):
            assert oc.append(step * rpc, bits(xt), rule) == 0
        if step % check_every == 0 or step == steps - 1:
            ys = kvq.kvq_dequantize_cache_batch(caches, 0, (step + 1) * rpc)
            torch.cuda.synchronize()
            for i, (c, oc, yt) in enumerate(zip(caches, ocs, ys)):
                n = (step + 1) * rpc * D
                assert_same(c.packed[:n // 2].cpu().numpy(), oc.packed[:n // 2], f"packed t{i} s{step}")
                assert_same(c.scales[:n // 16].cpu().numpy(), oc.scales[:n // 16], f"scales t{i} s{step}")
                assert_same(c.amax[:step + 1].cpu().numpy(), oc.amax[:step + 1], f"amax t{i} s{step}")
                assert_same(bits(yt), oc.dequantize(0, (step + 1) * rpc), f"dequant t{i} s{step}")
    return caches, ocs


@pytest.mark.parametrize("rule", RULES)
def test_rollout_small(orc, rule):
    _rollout(orc, layers=3, heads=2, tokens=40, steps=5, capacity_frames=6, rule=rule)


def test_rollout_odd_geometry(orc):
    """tokens*heads*8 blocks per chunk is odd, so chunks and pairs are misaligned."""
    _rollout(orc, layers=2, heads=3, tokens=13, steps=4, capacity_frames=5, rule="mse")


def test_cache_ranges_and_partial_chunk(orc):
    D, heads, tokens = 128, 3, 21
    rpc = heads * tokens
    c = kvq.KVCache(5 * rpc, rpc, D)
    oc = orc.Cache(5 * rpc, rpc, D)
    for step, n_rows in enumerate([rpc, rpc, rpc - 5, rpc]):  # a short append leaves a gap
        x = inputs.normal((n_rows, D), seed=100 + step, device="cuda")
        kvq.kvq_append(c, step * rpc, x, "mse")
        assert oc.append(step * rpc, bits(x), "mse") == 0
    torch.cuda.synchronize()
    for r0, r1 in [(0, 4 * rpc), (1, 2), (rpc - 1, rpc + 1), (rpc // 2 + 1, 3 * rpc + 7), (3 * rpc, 3 * rpc)]:
        y = kvq.kvq_dequantize_cache(c, r0, r1)
        torch.cuda.synchronize()
        assert_same(bits(y), oc.dequantize(r0, r1), f"range [{r0}, {r1})")


def test_cache_capacity_error_leaves_cache_untouched():
    c = kvq.KVCache(32, 16, 128)
    x = inputs.normal((16, 128), seed=1, device="cuda")
    with pytest.raises(kvq.KvqError) as e:
        kvq.kvq_append(c, 32, x)
    assert e.value.status == 4
    torch.cuda.synchronize()
    assert not c.packed.any() and not c.scales.any()


# ---------------------------------------------------------------- batched and fused entry points

@pytest.mark.parametrize("rule", RULES)
def test_quantize_batch_matches_oracle_per_tensor(orc, rule):
    """K and V (and a third tensor) in one set of launches, each with its own amax."""
    xs = [inputs.layer_kv(kv, heads=3, tokens=331, device="cuda") for kv in (0, 1)]
    xs.append(inputs.normal(tuple(xs[0].shape), seed=77, device="cuda") * 1e-3)
    p, s, a = kvq.kvq_quantize_batch(xs, 128, rule)
    ys = kvq.kvq_dequantize_batch(p, s, a, 128)
    torch.cuda.synchronize()
    for i, x in enumerate(xs):
        pe, se, ae = orc.quantize(bits(x), 128, rule)
        assert float(a[i][0]) == ae
        assert_same(s[i].cpu().numpy(), se, f"scales t{i}")
        assert_same(p[i].cpu().numpy(), pe, f"packed t{i}")
        assert_same(bits(ys[i]), orc.dequantize(pe, se, ae, 128), f"dequant t{i}")


def test_batches_above_the_launch_limit_are_split(orc):
    n = kvq.MAX_BATCH + 7
    xs = [inputs.normal((3, 128), seed=500 + i, device="cuda") * (i + 1) for i in range(n)]
    p, s, a = kvq.kvq_quantize_batch(xs, 128, "mse")
    ys = kvq.kvq_dequantize_batch(p, s, a, 128)
    torch.cuda.synchronize()
    for i in (0, kvq.MAX_BATCH - 1, kvq.MAX_BATCH, n - 1):
        pe, se, ae = orc.quantize(bits(xs[i]), 128, "mse")
        assert float(a[i][0]) == ae
        assert_same(p[i].cpu().numpy(), pe, f"packed t{i}")
        assert_same(bits(ys[i]), orc.dequantize(pe, se, ae, 128), f"dequant t{i}")


@pytest.mark.parametrize("codes", [True, False])
@pytest.mark.parametrize("rule", RULES)
def test_fused_round_trip_equals_quantize_then_dequantize(orc, rule, codes):
    cases = [inputs.single_k("cuda"), inputs.normal((7, 48), seed=3, device="cuda"),
             inputs.layer_kv(1, heads=2, tokens=257, device="cuda")]
    for x in cases:
        D = x.shape[-1]
        y, p, s, a = kvq.kvq_quantize_dequantize(x, D, rule, codes=codes)
        torch.cuda.synchronize()
        pe, se, ae = orc.quantize(bits(x), D, rule)
        assert float(a[0]) == ae
        assert_same(bits(y), orc.dequantize(pe, se, ae, D), f"round trip {tuple(x.shape)}")
        if codes:
            assert_same(p.cpu().numpy(), pe, "packed")
            assert_same(s.cpu().numpy(), se, "scales")
        else:
            assert p is None and s is None


def test_fused_round_trip_with_amax_in(orc):
    x = inputs.normal((129, 128), seed=12, device="cuda")
    for given in (float(x.abs().max().float()) / 4, 0.0):
        amax_in = torch.tensor([given], device="cuda")
        y, _, _, _ = kvq.kvq_quantize_dequantize(x, 128, "mse", amax_in=amax_in, codes=False)
        torch.cuda.synchronize()
        pe, se, _ = orc.quantize(bits(x), 128, "mse", amax_in=given)
        assert_same(bits(y), orc.dequantize(pe, se, given, 128), f"round trip amax_in={given}")
