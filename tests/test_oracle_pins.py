"""Pins of the CPU oracle to facts fixed outside the oracle itself.

Each test ties one part of the oracle to something it cannot echo: a value worked by
hand from the pages' formulas (tests/golden/), an independent library conversion
(ml_dtypes, torch), a closed form of the format, an invariant, or brute force on tiny
inputs. A plausible slip in the oracle (a swapped nibble, a wrong bias, a wrong tie, an
inverted mse comparison, a dropped global scale) fails at least one of them.
"""
import math

import ml_dtypes
import numpy as np
import pytest
import torch

from golden_io import floats_to_bf16_bits, hex_bytes, read_sections, round_to_bf16_bits

E2M1_GRID = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def _bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    return torch.from_numpy(bits.astype(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()


def _f32(x) -> float:
    return float(np.float32(x))


# ---------------------------------------------------------------- hand-worked example

@pytest.mark.parametrize("rule", ["static_6", "static_4", "mse"])
def test_worked_example(orc, rule):
    g = read_sections("worked_example.txt")
    x = floats_to_bf16_bits(g["input"])
    packed, scales, amax = orc.quantize(x, 16, rule)
    assert amax == float(g["amax"][0])
    np.testing.assert_array_equal(scales, hex_bytes(g[f"{rule}.scales"]))
    np.testing.assert_array_equal(packed, hex_bytes(g[f"{rule}.packed"]))
    y = orc.dequantize(packed, scales, amax, 16)
    np.testing.assert_array_equal(y, floats_to_bf16_bits(g[f"{rule}.dequant"]))


def test_worked_example_mse_errors(orc):
    """Block 1 of the worked example: err6 = 2.878906 + 2^-26, err4 = 1.316406 + 2^-26."""
    g = read_sections("worked_example.txt")
    x = floats_to_bf16_bits(g["input"])[16:32]
    _, _, e6, e4 = orc.quantize_block_detail(x, 2688.0, "mse")
    assert e6 == _f32(2.87890625 + 2.0 ** -26)
    assert e4 == _f32(1.31640625 + 2.0 ** -26)


def test_zero_tensor_keeps_signed_zeros(orc):
    x = floats_to_bf16_bits(["0", "-0"] * 8)
    for rule in ("static_6", "static_4", "mse"):
        packed, scales, amax = orc.quantize(x, 16, rule)
        assert amax == 0.0
        assert scales.tolist() == [0]
        assert packed.tolist() == [0x80] * 8
        np.testing.assert_array_equal(orc.dequantize(packed, scales, amax, 16), x)


# ---------------------------------------------------------------- e2m1

def _minifloat(e_bits, m_bits, bias, field):
    """Generic minifloat magnitude from its bit fields (the textbook definition)."""
    e = field >> m_bits
    m = field & ((1 << m_bits) - 1)
    if e == 0:
        return math.ldexp(m / (1 << m_bits), 1 - bias)
    return math.ldexp(1.0 + m / (1 << m_bits), e - bias)


def test_e2m1_grid_from_bit_fields(orc):
    # 1 sign, 2 exponent, 1 mantissa bit, bias 1; the largest value is 6 (scale = amax / 6.0)
    grid = [_minifloat(2, 1, 1, f) for f in range(8)]
    assert grid == E2M1_GRID
    for nib in range(16):
        want = -grid[nib & 7] if nib & 8 else grid[nib & 7]
        got = orc.e2m1_decode(nib)
        assert got == want and math.copysign(1, got) == math.copysign(1, want)


def test_e2m1_all_256_bytes_decode_to_grid(orc):
    lib = np.arange(16, dtype=np.uint8).view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    allowed = set(E2M1_GRID) | {-v for v in E2M1_GRID}
    for byte in range(256):
        lo, hi = orc.e2m1_decode(byte & 15), orc.e2m1_decode(byte >> 4)
        assert lo in allowed and hi in allowed
        assert lo == lib[byte & 15] and hi == lib[byte >> 4]


def test_e2m1_encode_matches_ml_dtypes_sweep(orc):
    # every multiple of 2^-12 in [-8, 8], plus the exact midpoints and their fp32 neighbours
    v = np.arange(-8 * 4096, 8 * 4096 + 1, dtype=np.float64) / 4096.0
    mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0])
    near = np.concatenate([mids, np.nextafter(mids.astype(np.float32), 0), np.nextafter(mids.astype(np.float32), 10)])
    v = np.concatenate([v, near, -near, [7.0, 100.0, 1e30, -1e30, 1e-40, -1e-40, 0.0, -0.0]]).astype(np.float32)
    want = v.astype(ml_dtypes.float4_e2m1fn).view(np.uint8) & 15
    got = np.array([orc.e2m1_encode(float(t)) for t in v], dtype=np.uint8)
    bad = np.nonzero(got != want)[0]
    assert bad.size == 0, [(float(v[i]), int(got[i]), int(want[i])) for i in bad[:10]]


def test_e2m1_thresholds_and_ties(orc):
    # round to nearest, ties to the even code: 0.25->0, 0.75->1, 1.25->1, 1.75->2, 2.5->2, 3.5->4, 5->4
    cases = {0.25: 0, 0.75: 2, 1.25: 2, 1.75: 4, 2.5: 4, 3.5: 6, 5.0: 6, 6.0: 7, 6.5: 7,
             0.2500001: 1, 0.7499999: 1, 5.0000005: 7, 4.9999995: 6}
    for v, code in cases.items():
        assert orc.e2m1_encode(v) == code, v
        assert orc.e2m1_encode(-v) == code | 8, -v
    assert orc.e2m1_encode(-0.1) == 8  # negative values that round to zero keep the sign
    assert orc.e2m1_encode(float("inf")) == 7
    for f in range(8):
        assert orc.e2m1_encode(E2M1_GRID[f]) == f  # idempotent on the grid


# ---------------------------------------------------------------- e4m3

def test_e4m3_decode_matches_libraries(orc):
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], dtype=np.uint8)
    ml = codes.view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    th = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    for c, a, b in zip(codes, ml, th):
        got = orc.e4m3_decode(int(c))
        assert got == a == b
        assert got == (-1 if c & 0x80 else 1) * _minifloat(4, 3, 7, int(c) & 0x7F)
    assert math.isnan(orc.e4m3_decode(0x7F)) and math.isnan(orc.e4m3_decode(0xFF))
    assert orc.e4m3_decode(0x7E) == 448.0 and orc.e4m3_decode(0x01) == 2.0 ** -9


def test_e4m3_decode_encode_identity(orc):
    for c in range(127):
        assert orc.e4m3_encode(orc.e4m3_decode(c)) == c


def test_e4m3_encode_matches_libraries(orc):
    rng = np.random.default_rng(7)
    # log-uniform positives over the whole e4m3 range, plus every midpoint and its neighbours
    v = np.exp2(rng.uniform(-14, math.log2(463.9), 60000)).astype(np.float32)
    mags = np.array([orc.e4m3_decode(c) for c in range(127)])
    mids = ((mags[:-1] + mags[1:]) / 2).astype(np.float32)
    v = np.concatenate([v, mids, np.nextafter(mids, 0), np.nextafter(mids, 1000), mags.astype(np.float32),
                        np.float32([0.0, 2.0 ** -10, 2.0 ** -11, 1e-30, 463.99997])])
    want_ml = v.astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
    want_th = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(want_ml, want_th)
    got = np.array([orc.e4m3_encode(float(t)) for t in v], dtype=np.uint8)
    bad = np.nonzero(got != want_ml)[0]
    assert bad.size == 0, [(float(v[i]), int(got[i]), int(want_ml[i])) for i in bad[:10]]


def test_e4m3_saturates(orc):
    # the libraries return NaN above 464; the method's scale conversion saturates at 448
    for r in (448.0, 460.0, 464.0, 479.0, 480.0, 1e6, float("inf")):
        assert orc.e4m3_encode(r) == 0x7E
    assert orc.e4m3_encode(2.0 ** -10) == 0x00  # tie between 0 and the smallest subnormal -> even (0)
    assert orc.e4m3_encode(float(np.nextafter(np.float32(2.0 ** -10), 1))) == 0x01


# ---------------------------------------------------------------- bf16 rounding

def test_bf16_rne_matches_torch(orc):
    rng = np.random.default_rng(3)
    u = rng.integers(0, 2 ** 32, 50000, dtype=np.uint64).astype(np.uint32)
    u = u[((u >> 23) & 0xFF) != 0xFF]  # finite only
    ties = (rng.integers(0, 2 ** 16, 2000, dtype=np.uint32) << 16) | 0x8000
    ties = ties[((ties >> 23) & 0xFF) < 0xFE]
    u = np.concatenate([u, ties, ties + 1, ties - 1])
    f = u.view(np.float32)
    want = torch.from_numpy(f.copy()).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = np.array([orc.bf16_rne(float(t)) for t in f], dtype=np.uint16)
    np.testing.assert_array_equal(got, want)


# ---------------------------------------------------------------- quantizer properties

def _grid_block_tensor(rng, nblocks, k_t=0):
    """Tensor whose amax is 6*2^k_t, every block's values on the e2m1 grid times 2^j_b."""
    vals = []
    for b in range(nblocks):
        j = k_t if b == 0 else k_t - int(rng.integers(0, 9))
        blk = rng.choice(E2M1_GRID, 16) * rng.choice([-1.0, 1.0], 16)
        blk[int(rng.integers(0, 16))] = 6.0 * (1 if rng.random() < 0.5 else -1)
        vals.append(blk * 2.0 ** j)
    return np.concatenate(vals)


def test_grid_blocks_round_trip_exactly(orc):
    rng = np.random.default_rng(11)
    for k_t in (0, 5, -7):
        vals = _grid_block_tensor(rng, 32, k_t)
        x = floats_to_bf16_bits(vals)
        packed, scales, amax = orc.quantize(x, 128, "static_6")
        assert amax == 6.0 * 2.0 ** k_t
        y = orc.dequantize(packed, scales, amax, 128)
        np.testing.assert_array_equal(y, x)


def test_amax_element_maps_to_6_or_4(orc):
    rng = np.random.default_rng(5)
    x = round_to_bf16_bits(rng.standard_normal(128 * 64))
    xf = _bf16_bits_to_f64(x)
    for rule, R in (("static_6", 6), ("static_4", 4)):
        packed, scales, amax = orc.quantize(x, 128, rule)
        gs = np.float32(amax) / np.float32(2688)
        nib = np.stack([packed & 15, packed >> 4], 1).reshape(-1)
        checked = 0
        for b in range(xf.size // 16):
            blk = xf[16 * b:16 * b + 16]
            amax_b = np.abs(blk).max()
            r = amax_b / R / float(gs)
            if not (2.0 ** -6 <= r <= 448):
                continue
            i = int(np.argmax(np.abs(blk)))
            code = int(nib[16 * b + i])
            assert abs(orc.e2m1_decode(code)) == R and (code >> 3) == (blk[i] < 0), (rule, b)
            checked += 1
        assert checked > (0.95 if R == 6 else 0.5) * (xf.size // 16)


def test_single_outlier_block(orc):
    vals = np.full(128, 2.0 ** -7)
    vals[37] = -500.0
    x = floats_to_bf16_bits(vals)
    packed, scales, amax = orc.quantize(x, 128, "static_6")
    assert amax == 500.0
    assert scales[2] == 0x7E  # the outlier's block: (500/6) / (500/2688) = 448
    nib = np.stack([packed & 15, packed >> 4], 1).reshape(-1)
    assert nib[37] == 0xF
    # small blocks: r = (2^-7/6)/(500/2688) ~ 0.007 -> e4m3 subnormal scale 4*2^-9
    assert all(scales[b] != 0x7E for b in (0, 1, 3, 4, 5, 6, 7))
    y = _bf16_bits_to_f64(orc.dequantize(packed, scales, amax, 128))
    assert y[37] == -500.0


def test_static4_saturated_block(orc):
    # block amax == tensor amax: r4 = 672 saturates at 448, S = amax/6, the amax maps to 6
    vals = np.linspace(-1, 1, 32)
    vals[3] = 3.0
    x = round_to_bf16_bits(vals)
    packed, scales, _ = orc.quantize(x, 16, "static_4")
    assert scales[0] == 0x7E
    assert (packed[1] >> 4) == 7


def test_negative_values_rounding_to_zero_keep_sign(orc):
    vals = np.zeros(16)
    vals[0] = 6.0
    vals[1] = -0.1
    vals[2] = 0.1
    x = round_to_bf16_bits(vals)
    packed, _, _ = orc.quantize(x, 16, "static_6")
    assert packed[0] == (7 | (8 << 4)) and (packed[1] & 15) == 0


def test_zero_block_inside_nonzero_tensor(orc):
    vals = np.concatenate([np.zeros(16), np.arange(16) - 7.5])
    x = floats_to_bf16_bits(vals)
    packed, scales, _ = orc.quantize(x, 16, "mse")
    assert scales[0] == 0 and packed[:8].tolist() == [0] * 8


def test_sign_symmetry(orc):
    rng = np.random.default_rng(2)
    x = round_to_bf16_bits(rng.standard_normal(2048))
    xn = x ^ np.uint16(0x8000)
    for rule in ("static_6", "static_4", "mse"):
        p, s, a = orc.quantize(x, 128, rule)
        pn, sn, an = orc.quantize(xn, 128, rule)
        assert a == an
        np.testing.assert_array_equal(s, sn)
        np.testing.assert_array_equal(pn, p ^ np.uint8(0x88))


def test_power_of_two_equivariance(orc):
    rng = np.random.default_rng(4)
    x = round_to_bf16_bits(rng.standard_normal(4096))
    xf = _bf16_bits_to_f64(x)
    for rule in ("static_6", "static_4", "mse"):
        p, s, a = orc.quantize(x, 128, rule)
        y = _bf16_bits_to_f64(orc.dequantize(p, s, a, 128))
        for k in (-20, 3, 17):
            xk = floats_to_bf16_bits(xf * 2.0 ** k)
            pk, sk, ak = orc.quantize(xk, 128, rule)
            assert ak == a * 2.0 ** k
            np.testing.assert_array_equal(pk, p)
            np.testing.assert_array_equal(sk, s)
            np.testing.assert_array_equal(_bf16_bits_to_f64(orc.dequantize(pk, sk, ak, 128)), y * 2.0 ** k)


def test_block_permutation_equivariance(orc):
    rng = np.random.default_rng(6)
    x = round_to_bf16_bits(rng.standard_normal(16 * 64))
    perm = rng.permutation(64)
    xp = x.reshape(64, 16)[perm].reshape(-1)
    p, s, _ = orc.quantize(x, 16, "mse")
    pp, sp, _ = orc.quantize(xp, 16, "mse")
    np.testing.assert_array_equal(sp, s[perm])
    np.testing.assert_array_equal(pp.reshape(64, 8), p.reshape(64, 8)[perm])


def test_mse_brute_force_tiny_blocks(orc):
    """mse must keep the candidate with the lower squared error (computed here in fp64
    from the two static rules' own outputs); near-ties are left to the fp32 rule."""
    rng = np.random.default_rng(9)
    picked4 = 0
    for trial in range(3000):
        scale = 2.0 ** int(rng.integers(-8, 8))
        kind = trial % 3
        if kind == 0:
            v = rng.standard_normal(16)
        elif kind == 1:
            v = rng.standard_t(3, 16)
        else:
            v = rng.choice(E2M1_GRID, 16) * rng.uniform(0.5, 1.5) * rng.choice([-1, 1], 16)
        x = round_to_bf16_bits(v * scale)
        xf = _bf16_bits_to_f64(x)
        amax_t = float(np.abs(xf).max()) * float(rng.choice([1.0, 1.0, 3.0, 40.0]))
        amax_t = float(np.float32(amax_t))
        gs = float(np.float32(np.float32(amax_t) / np.float32(2688)))
        errs = {}
        outs = {}
        for rule in ("static_6", "static_4"):
            c, pk, _, _ = orc.quantize_block_detail(x, amax_t, rule)
            nib = np.stack([pk & 15, pk >> 4], 1).reshape(-1)
            vals = np.array([orc.e2m1_decode(int(q)) for q in nib])
            S = orc.e4m3_decode(c) * gs
            errs[rule] = float(np.sum((xf - vals * S) ** 2))
            outs[rule] = (c, pk)
        c, pk, e6, e4 = orc.quantize_block_detail(x, amax_t, "mse")
        tol = 1e-5 * max(errs["static_6"], errs["static_4"], 1e-300)
        if abs(errs["static_4"] - errs["static_6"]) <= tol:
            want = "static_4" if e4 < e6 else "static_6"
        else:
            want = "static_4" if errs["static_4"] < errs["static_6"] else "static_6"
        assert c == outs[want][0] and np.array_equal(pk, outs[want][1]), trial
        picked4 += want == "static_4"
    assert 0 < picked4 < 3000


def test_codes_are_nearest_grid_points(orc):
    """For a fixed decoded scale, each code is the grid point nearest to x / S (fp64
    brute force over all 16 codes), except within 1e-6 of a midpoint."""
    rng = np.random.default_rng(10)
    for trial in range(400):
        x = round_to_bf16_bits(rng.standard_normal(16) * 3)
        xf = _bf16_bits_to_f64(x)
        amax_t = float(np.float32(np.abs(xf).max() * 2))
        gs = float(np.float32(np.float32(amax_t) / np.float32(2688)))
        for rule in ("static_6", "static_4"):
            c, pk, _, _ = orc.quantize_block_detail(x, amax_t, rule)
            S = orc.e4m3_decode(c) * gs
            nib = np.stack([pk & 15, pk >> 4], 1).reshape(-1)
            allv = np.array([orc.e2m1_decode(q) for q in range(16)])
            for i in range(16):
                t = xf[i] / S
                d = np.abs(allv - t)
                order = np.sort(np.unique(d))
                if order.size > 1 and order[1] - order[0] < 1e-6:
                    continue
                assert abs(orc.e2m1_decode(int(nib[i])) - t) == order[0]


def test_relative_mse_bound_on_normal(orc):
    """Reconstruction error on N(0, 1): relative MSE <= 2e-2 for every rule."""
    from nvfp4_kv_cache_kvq_b200 import inputs

    x = inputs.bits(inputs.single_k())
    xf = _bf16_bits_to_f64(x)
    rel = {}
    for rule in ("static_6", "static_4", "mse"):
        p, s, a = orc.quantize(x, 128, rule)
        y = _bf16_bits_to_f64(orc.dequantize(p, s, a, 128))
        rel[rule] = float(np.sum((y - xf) ** 2) / np.sum(xf ** 2))
        assert rel[rule] <= 2e-2, rel
    assert rel["mse"] <= min(rel["static_6"], rel["static_4"]) * 1.02


def test_thread_count_does_not_change_results(orc):
    from nvfp4_kv_cache_kvq_b200 import inputs

    x = inputs.bits(inputs.layer_kv(0, heads=2, tokens=333))
    ref = orc.quantize(x, 128, "mse", threads=1)
    for t in (2, 7):
        got = orc.quantize(x, 128, "mse", threads=t)
        np.testing.assert_array_equal(got[0], ref[0])
        np.testing.assert_array_equal(got[1], ref[1])
        assert got[2] == ref[2]


def test_amax_in_overrides(orc):
    rng = np.random.default_rng(12)
    x = round_to_bf16_bits(rng.standard_normal(256))
    p, s, a = orc.quantize(x, 128, "static_6")
    p2, s2, a2 = orc.quantize(x, 128, "static_6", amax_in=a)
    assert a2 == a and np.array_equal(p, p2) and np.array_equal(s, s2)
    p3, s3, a3 = orc.quantize(x, 128, "static_6", amax_in=4 * a)
    assert a3 == 4 * a and not np.array_equal(s, s3)


# ---------------------------------------------------------------- cache

def test_append_equals_per_chunk_quantize(orc):
    from nvfp4_kv_cache_kvq_b200 import inputs

    heads, tok, D = 3, 40, 128
    rows_per_chunk = heads * tok
    cache = orc.Cache(capacity_rows=rows_per_chunk * 4, rows_per_chunk=rows_per_chunk, head_dim=D)
    chunks = [inputs.bits(inputs.rollout_chunk(s, 0, heads=heads, tokens=tok)) for s in range(3)]
    for s, xb in enumerate(chunks):
        assert cache.append(s * rows_per_chunk, xb, "mse") == 0
    for s, xb in enumerate(chunks):
        p, sc, a = orc.quantize(xb, D, "mse")
        e0 = s * rows_per_chunk * D
        np.testing.assert_array_equal(cache.packed[e0 // 2:e0 // 2 + p.size], p)
        np.testing.assert_array_equal(cache.scales[e0 // 16:e0 // 16 + sc.size], sc)
        assert cache.amax[s] == a
    y = cache.dequantize(0, 3 * rows_per_chunk)
    want = np.concatenate([orc.dequantize(*orc.quantize(xb, D, "mse")[:2], orc.quantize(xb, D, "mse")[2], D)
                           for xb in chunks])
    np.testing.assert_array_equal(y, want)
    # a range that starts and ends inside chunks
    r0, r1 = rows_per_chunk // 2 + 1, 2 * rows_per_chunk + 7
    np.testing.assert_array_equal(cache.dequantize(r0, r1), want[r0 * D:r1 * D])


def test_append_rejects_bad_offsets(orc):
    cache = orc.Cache(capacity_rows=64, rows_per_chunk=16, head_dim=128)
    x = np.zeros(16 * 128, np.uint16)
    assert cache.append(8, x, "static_6") == 1  # not chunk aligned
    assert cache.append(64, x, "static_6") == 4  # past capacity
    assert cache.append(0, np.zeros(17 * 128, np.uint16), "static_6") == 1  # larger than a chunk


def test_cache_bytes_closed_form(orc):
    # 30 layers x {K, V}, 12 heads, 93600 tokens, D 128, chunks of 1560 tokens
    p, s, a = orc.cache_bytes(30, 12, 93600, 128, 1560)
    elems = 60 * 93600 * 12 * 128
    assert p == elems // 2 and s == elems // 16 and a == 60 * 60 * 4
    bf16 = elems * 2
    assert abs(bf16 / (p + s + a) - 16 / 4.5) < 1e-3  # 4.5 bits per element
