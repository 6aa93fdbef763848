"""The C ABI inside CUDA graphs, and a packed cache saved and restored mid-rollout.

A graph replay re-runs the captured launches on whatever the static buffers hold, so each
replay is checked against the oracle on fresh inputs. A checkpoint is the cache's three
byte buffers (codes, scales, per-chunk amax): restoring them into a fresh cache and
continuing the rollout must give the same bytes and the same dequantized prefix as the
uninterrupted run."""
import numpy as np
import pytest
import torch

import nvfp4_kv_cache_kvq_b200 as kvq
from gpu_helpers import assert_same
from nvfp4_kv_cache_kvq_b200 import inputs
from nvfp4_kv_cache_kvq_b200.inputs import bits

pytestmark = pytest.mark.gpu


def test_append_and_read_captured_in_a_cuda_graph(orc):
    heads, tokens, D, frames = 2, 40, 128, 3
    rpc = heads * tokens
    caches = kvq.allocate_caches(1, heads, frames * tokens, D, tokens)
    x_static = [torch.empty((tokens, heads, D), dtype=torch.bfloat16, device="cuda") for _ in caches]
    y_static = [torch.empty(frames * rpc * D, dtype=torch.bfloat16, device="cuda") for _ in caches]
    graphs = []
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):  # warm-up outside capture
        kvq.kvq_append_batch(caches, [0, 0], x_static, "mse")
        kvq.kvq_dequantize_cache_batch(caches, 0, rpc, [y[:rpc * D] for y in y_static])
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    for f in range(frames):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            kvq.kvq_append_batch(caches, [f * rpc] * 2, x_static, "mse")
            kvq.kvq_dequantize_cache_batch(caches, 0, (f + 1) * rpc, [y[:(f + 1) * rpc * D] for y in y_static])
        graphs.append(g)
    ocs = [orc.Cache(frames * rpc, rpc, D) for _ in caches]
    for replay in range(2):
        for f in range(frames):
            for t in range(2):
                x_static[t].copy_(inputs.rollout_chunk(f + 10 * replay, t, heads=heads, tokens=tokens, device="cuda"))
                assert ocs[t].append(f * rpc, bits(x_static[t]), "mse") == 0
            graphs[f].replay()
            torch.cuda.synchronize()
            for t in range(2):
                assert_same(bits(y_static[t][:(f + 1) * rpc * D]), ocs[t].dequantize(0, (f + 1) * rpc),
                            f"graph replay {replay} frame {f} tensor {t}")


def test_cache_checkpoint_and_resume_is_bit_identical():
    heads, tokens, D, frames, cut = 3, 50, 128, 6, 3
    rpc = heads * tokens
    xs = [[inputs.rollout_chunk(f, t, heads=heads, tokens=tokens, device="cuda") for t in range(4)]
          for f in range(frames)]
    a = kvq.allocate_caches(2, heads, frames * tokens, D, tokens)
    for f in range(cut):
        kvq.kvq_append_batch(a, [f * rpc] * 4, xs[f], "mse")
    torch.cuda.synchronize()
    saved = [(c.packed.cpu().numpy().copy(), c.scales.cpu().numpy().copy(), c.amax.cpu().numpy().copy()) for c in a]
    for f in range(cut, frames):
        kvq.kvq_append_batch(a, [f * rpc] * 4, xs[f], "mse")
    b = kvq.allocate_caches(2, heads, frames * tokens, D, tokens)
    for c, (p, s, m) in zip(b, saved):
        c.packed.copy_(torch.from_numpy(p))
        c.scales.copy_(torch.from_numpy(s))
        c.amax.copy_(torch.from_numpy(m))
    for f in range(cut, frames):
        kvq.kvq_append_batch(b, [f * rpc] * 4, xs[f], "mse")
    ya = kvq.kvq_dequantize_cache_batch(a, 0, frames * rpc)
    yb = kvq.kvq_dequantize_cache_batch(b, 0, frames * rpc)
    torch.cuda.synchronize()
    for ca, cb, y1, y2 in zip(a, b, ya, yb):
        assert torch.equal(ca.packed, cb.packed) and torch.equal(ca.scales, cb.scales)
        assert torch.equal(ca.amax, cb.amax)
        assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))
