"""Bit-exact parity of the RTN INT4 / INT2 kernels (through the C ABI) against the CPU
oracle: codes, bf16 scales and dequantized bf16."""
import numpy as np
import pytest
import torch

import nvfp4_kv_cache_kvq_b200 as kvq
from golden_io import floats_to_bf16_bits, read_sections
from gpu_helpers import assert_same
from nvfp4_kv_cache_kvq_b200 import inputs
from nvfp4_kv_cache_kvq_b200.inputs import bits

pytestmark = pytest.mark.gpu


def _bf16(b):
    return torch.from_numpy(b.astype(np.uint16).view(np.int16).copy()).view(torch.bfloat16).cuda()


def check(orc, x, nbits, head_dim):
    p, s = kvq.kvq_rtn_quantize(x, nbits, head_dim)
    y = kvq.kvq_rtn_dequantize(p, s, nbits, head_dim)
    torch.cuda.synchronize()
    pe, se = orc.rtn_quantize(bits(x), head_dim, nbits)
    assert_same(bits(s), se, f"rtn{nbits} scales")
    assert_same(p.cpu().numpy(), pe, f"rtn{nbits} codes")
    assert_same(bits(y), orc.rtn_dequantize(pe, se, head_dim, nbits), f"rtn{nbits} dequant")


@pytest.mark.parametrize("nbits", [4, 2])
def test_rtn_worked_example_on_gpu(nbits):
    g = read_sections("rtn_worked_example.txt")
    x = _bf16(floats_to_bf16_bits(g[f"int{nbits}.input"]))
    p, s = kvq.kvq_rtn_quantize(x, nbits, 16)
    y = kvq.kvq_rtn_dequantize(p, s, nbits, 16)
    torch.cuda.synchronize()
    assert_same(bits(s), np.array([int(t, 16) for t in g[f"int{nbits}.scales"]], np.uint16), "scales")
    assert_same(p.cpu().numpy(), np.array([int(t, 16) for t in g[f"int{nbits}.packed"]], np.uint8), "codes")
    assert_same(bits(y), floats_to_bf16_bits(g[f"int{nbits}.dequant"]), "dequant")


@pytest.mark.parametrize("nbits", [4, 2])
def test_rtn_workload_inputs(orc, nbits):
    check(orc, inputs.single_k("cuda"), nbits, 128)
    check(orc, inputs.layer_kv(0, device="cuda"), nbits, 128)
    check(orc, inputs.rollout_chunk(3, 7, device="cuda"), nbits, 128)


@pytest.mark.parametrize("nbits", [4, 2])
def test_rtn_every_bf16_value_and_ties(orc, nbits):
    """Blocks whose scale is exactly 1 (amax = qmax): every bf16 in [-qmax, qmax] is
    rounded by the kernel's corrected quotient and magic-number rounding, ties included;
    plus every positive bf16 amax as a block maximum."""
    qmax = (1 << (nbits - 1)) - 1
    u = np.arange(0, 1 << 16, dtype=np.uint32).astype(np.uint16)
    f = torch.from_numpy(u.view(np.int16)).view(torch.bfloat16).float().numpy()
    vals = u[np.isfinite(f) & (np.abs(f) <= qmax)]
    vals = np.concatenate([vals, np.zeros((-vals.size) % 15, np.uint16)]).reshape(-1, 15)
    top = floats_to_bf16_bits([float(qmax)])[0]
    blocks = np.concatenate([np.full((vals.shape[0], 1), top, np.uint16), vals], 1)
    amaxes = u[np.isfinite(f) & (f > 0)]
    ablocks = np.zeros((amaxes.size, 16), np.uint16)
    ablocks[:, 0] = amaxes
    ablocks[:, 1] = amaxes ^ 0x8000
    ablocks[:, 2:] = np.where(amaxes >= 7, amaxes - 7, 0).astype(np.uint16)[:, None]
    check(orc, _bf16(np.concatenate([blocks, ablocks]).reshape(-1)), nbits, 16)


@pytest.mark.parametrize("nbits", [4, 2])
def test_rtn_extremes_and_ragged(orc, nbits):
    rng = np.random.default_rng(2)
    for scale in (1e-38, 1e-40, 2.0 ** -120, 1e-30, 1e30, 5e37):  # tiny scales take the IEEE-division path
        x = torch.from_numpy(rng.standard_normal(128 * 9) * scale).to(torch.bfloat16).cuda()
        check(orc, x, nbits, 128)
    for D, rows in ((16, 1), (48, 7), (144, 5)):
        check(orc, inputs.normal((rows, D), seed=D + rows, device="cuda"), nbits, D)
    z = torch.zeros(128 * 3, dtype=torch.bfloat16, device="cuda")
    z[::5] = -0.0
    check(orc, z, nbits, 128)


@pytest.mark.parametrize("nbits", [4, 2])
def test_rtn_narrow_path_for_offset_buffers(orc, nbits):
    """Codes aligned to 2*bits bytes and scales to 2 bytes, but not to 4*bits and 4: the
    launch falls back to one block per thread; the results must not change. An odd block
    count also leaves the two-block path's last block alone."""
    x = inputs.normal((21, 16), seed=5, device="cuda")
    n = x.numel()
    pbuf = torch.zeros(n * nbits // 8 + 2 * nbits, dtype=torch.uint8, device="cuda")
    sbuf = torch.zeros(n // 16 + 1, dtype=torch.bfloat16, device="cuda")
    p_off, s_off = pbuf[2 * nbits:], sbuf[1:]
    assert p_off.data_ptr() % (4 * nbits) != 0 and s_off.data_ptr() % 4 != 0
    p, s = kvq.kvq_rtn_quantize(x, nbits, 16, packed=p_off, scales=s_off)
    ybuf = torch.zeros(n + 16, dtype=torch.bfloat16, device="cuda")
    y = kvq.kvq_rtn_dequantize(p, s, nbits, 16, y=ybuf[16:])
    torch.cuda.synchronize()
    pe, se = orc.rtn_quantize(bits(x), 16, nbits)
    assert_same(p.cpu().numpy(), pe, "codes")
    assert_same(bits(s), se, "scales")
    assert_same(bits(y), orc.rtn_dequantize(pe, se, 16, nbits), "dequant")
    # the wide path on aligned buffers agrees
    check(orc, x, nbits, 16)


def test_rtn_k2_v4_batches(orc):
    """RTN_K2_V4: keys with 2 bits, values with 4, one batched call per kind."""
    ks = [inputs.layer_kv(0, heads=2, tokens=100, device="cuda"), inputs.cache_kv(1, 0, heads=2, tokens=100, device="cuda")]
    vs = [inputs.layer_kv(1, heads=2, tokens=100, device="cuda"), inputs.cache_kv(1, 1, heads=2, tokens=100, device="cuda")]
    for xs, nbits in ((ks, 2), (vs, 4)):
        p, s = kvq.kvq_rtn_quantize_batch(xs, nbits, 128)
        ys = kvq.kvq_rtn_dequantize_batch(p, s, nbits, 128)
        torch.cuda.synchronize()
        for i, x in enumerate(xs):
            pe, se = orc.rtn_quantize(bits(x), 128, nbits)
            assert_same(p[i].cpu().numpy(), pe, f"codes t{i}")
            assert_same(bits(s[i]), se, f"scales t{i}")
            assert_same(bits(ys[i]), orc.rtn_dequantize(pe, se, 128, nbits), f"dequant t{i}")


def test_rtn_rejects_bad_bits():
    x = torch.zeros(128, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(kvq.KvqError) as e:
        kvq.kvq_rtn_quantize(x, 3, 128)
    assert e.value.status == 1
