"""Parity at the workloads' full sizes, in the launch configuration the benchmark times.

Where the oracle can redo a whole tensor in seconds it does; elsewhere each output is
checked through properties that hold at any size (the amax against torch's max |x| and
against the oracle's amax of the chunk) and through thousands of sampled blocks that
the oracle re-quantizes and dequantizes one by one under that amax."""
import numpy as np
import pytest
import torch

import nvfp4_kv_cache_kvq_b200 as kvq
from gpu_helpers import assert_same, check_full, check_sampled
from nvfp4_kv_cache_kvq_b200 import inputs
from nvfp4_kv_cache_kvq_b200.inputs import bits

pytestmark = pytest.mark.gpu


def _sample_blocks(nb, n, seed):
    g = torch.Generator().manual_seed(seed)
    idx = torch.randint(0, nb, (min(n, nb),), generator=g)
    return torch.cat([idx, torch.tensor([0, nb - 1])])


@pytest.fixture(scope="module")
def wan_cache_inputs():
    """30 layers x {K, V} of [1, 24, 32760, 128] (12 GB of bf16), generated once for the
    three rules."""
    layers, heads, tokens, D = 30, 24, 32760, 128
    T = 2 * layers
    x = torch.empty((T, heads * tokens * D), dtype=torch.bfloat16, device="cuda")
    for t in range(T):
        x[t] = inputs.cache_kv(t // 2, t % 2, device="cuda").reshape(-1)
    yield x
    del x
    torch.cuda.empty_cache()


@pytest.mark.parametrize("rule", ["mse", "static_6", "static_4"])
def test_full_wan_cache(orc, wan_cache_inputs, rule):
    """30 layers x {K, V} of [1, 24, 32760, 128]: quantize all 60 tensors, then
    dequantize layer by layer into one reused bf16 buffer (the benchmark's order). Layer 0
    whole against the oracle; every other layer on 1024 sampled blocks per tensor."""
    layers, heads, tokens, D = 30, 24, 32760, 128
    T = 2 * layers
    n = heads * tokens * D
    x = wan_cache_inputs
    p = torch.empty((T, n // 2), dtype=torch.uint8, device="cuda")
    s = torch.empty((T, n // 16), dtype=torch.uint8, device="cuda")
    a = torch.empty((T, 1), dtype=torch.float32, device="cuda")
    y = torch.empty((2, n), dtype=torch.bfloat16, device="cuda")
    for t in range(T):
        kvq.kvq_quantize(x[t], D, rule, amax_out=a[t], packed=p[t], scales=s[t])
    for l in range(layers):
        for kv in (0, 1):
            t = 2 * l + kv
            kvq.kvq_dequantize(p[t], s[t], a[t], D, y=y[kv])
        torch.cuda.synchronize()
        for kv in (0, 1):
            t = 2 * l + kv
            if l == 0:  # the whole first layer against the oracle
                xb = bits(x[t])
                pe, se, ae = orc.quantize(xb, D, rule)
                assert float(a[t, 0]) == ae
                assert_same(s[t].cpu().numpy(), se, "scales")
                assert_same(p[t].cpu().numpy(), pe, "packed")
                assert_same(bits(y[kv]), orc.dequantize(pe, se, ae, D), "dequant")
            else:
                check_sampled(orc, x[t], p[t], s[t], float(a[t, 0]), y[kv], rule, n_samples=1024, seed=t)


def test_full_rollout(orc):
    """30 layers x {K, V}, 12 heads, 60 frames of 1560 tokens, rule mse, through
    kvq_append_batch and kvq_dequantize_cache_batch exactly as the benchmark runs them.
    Every append: each chunk amax against the oracle's amax of the chunk, and sampled
    blocks of every tensor. Frames 1, 30 and 60: layer 0's whole prefix against the
    oracle's cache, and sampled blocks of every other layer's prefix, the expected
    values computed by the oracle from the input chunks and the oracle's chunk amax."""
    layers, heads, tokens, frames, D = 30, 12, 1560, 60, 128
    T, rpc = 2 * layers, heads * tokens
    chunk = rpc * D
    bpc = chunk // 16
    caches = kvq.allocate_caches(layers, heads, frames * tokens, D, tokens)
    ocs = [orc.Cache(frames * rpc, rpc, D) for _ in range(2)]  # layer 0 K and V in full
    yk = torch.empty(frames * chunk, dtype=torch.bfloat16, device="cuda")
    yv = torch.empty(frames * chunk, dtype=torch.bfloat16, device="cuda")
    xs_all = torch.empty((frames, T, chunk), dtype=torch.bfloat16, device="cuda")
    amax_ref = np.zeros((frames, T), np.float32)
    for f in range(frames):
        for t in range(T):
            xs_all[f, t] = inputs.rollout_chunk(f, t, heads=heads, tokens=tokens, device="cuda").reshape(-1)
        kvq.kvq_append_batch(caches, [f * rpc] * T, [xs_all[f, t] for t in range(T)], "mse")
        torch.cuda.synchronize()
        for t in range(T):
            c = caches[t]
            xb = bits(xs_all[f, t])
            amax_ref[f, t] = orc.amax(xb)
            assert float(c.amax[f]) == amax_ref[f, t], (f, t)
            if t < 2:
                assert ocs[t].append(f * rpc, xb, "mse") == 0
            idx = _sample_blocks(bpc, 256, f * 100 + t)
            pe, se, _ = orc.quantize(xb.reshape(-1, 16)[idx.numpy()].reshape(-1), 16, "mse",
                                     amax_in=float(amax_ref[f, t]))
            gidx = (idx + f * bpc).cuda()
            assert_same(c.scales[gidx].cpu().numpy(), se, f"scales f{f} t{t}")
            assert_same(c.packed.view(-1, 8)[gidx].cpu().numpy(), pe, f"packed f{f} t{t}")
        rows = (f + 1) * rpc
        check = f in (0, 29, frames - 1)
        for l in range(layers):
            kvq.kvq_dequantize_cache_batch(caches[2 * l:2 * l + 2], 0, rows, [yk[:rows * D], yv[:rows * D]])
            if not check:
                continue
            torch.cuda.synchronize()
            for kv, yt in ((0, yk), (1, yv)):
                t = 2 * l + kv
                if l == 0:
                    assert_same(caches[t].packed[:rows * D // 2].cpu().numpy(), ocs[kv].packed[:rows * D // 2],
                                "packed prefix")
                    assert_same(bits(yt[:rows * D]), ocs[kv].dequantize(0, rows), f"dequant prefix f{f}")
                    continue
                idx = _sample_blocks(rows * D // 16, 512, l * 7 + kv)
                fr = (idx // bpc).numpy()
                off = (idx % bpc).cuda()
                xb = bits(xs_all[:f + 1, t].reshape(f + 1, bpc, 16)[torch.from_numpy(fr).cuda(), off])
                want = []
                for i in range(idx.numel()):
                    pe, se, _ = orc.quantize(xb[16 * i:16 * i + 16], 16, "mse", amax_in=float(amax_ref[fr[i], t]))
                    want.append(orc.dequantize(pe, se, float(amax_ref[fr[i], t]), 16))
                assert_same(bits(yt.view(-1, 16)[idx.cuda()]), np.concatenate(want), f"sampled dequant f{f} l{l}")


@pytest.mark.parametrize("rule", ["static_6", "mse"])
def test_sweep(orc, rule):
    """[T, 128] N(0, 1): T = 2^10 .. 2^20 in full, 2^22 .. 2^26 by sampling."""
    for e in range(10, 27, 2):
        T = 1 << e
        x = inputs.sweep(T, device="cuda")
        if e <= 20:
            check_full(orc, x, rule, 128)
        else:
            p, s, a = kvq.kvq_quantize(x, 128, rule)
            y = kvq.kvq_dequantize(p, s, a, 128)
            torch.cuda.synchronize()
            check_sampled(orc, x, p, s, float(a[0]), y, rule, n_samples=4096, seed=e)
            del p, s, a, y
        del x
        torch.cuda.empty_cache()
