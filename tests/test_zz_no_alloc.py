"""kvq_attention_noalloc: attention for callers that cannot allocate device memory (a
plugin inside a framework that owns the GPU's memory through its own pool and budget, or
a latency-critical loop that cannot take cudaMalloc's implicit synchronization). It
uses the library's built-in 32 MiB scratch instead of a caller workspace. Checked
through the C ABI against kvq_attention with the recommended workspace, on two calls in
a row (the second sees the first call's leftovers in the shared scratch). Both calls make
the same key split, so the outputs must be identical: tighter than the parity tolerance
of the attention tests. This file is collected last on purpose."""
import pytest
import torch

import nvfp4_kv_cache_kvq_b200 as kvq
from nvfp4_kv_cache_kvq_b200 import inputs

pytestmark = pytest.mark.gpu
D = 128


def _caches(heads, n_keys, tokens_per_chunk, seed):
    rpc = tokens_per_chunk * heads
    n_chunks = -(-n_keys // tokens_per_chunk)
    caches = [kvq.KVCache(n_chunks * rpc, rpc, D) for _ in range(2)]
    for c in range(n_chunks):
        toks = min(tokens_per_chunk, n_keys - c * tokens_per_chunk)
        for t in range(2):
            kvq.kvq_append(caches[t], c * rpc, inputs.student_t((toks, heads, D), 4, seed + 2 * c + t, "cuda"), "mse")
    return caches


def test_noalloc_matches_attention_twice_in_a_row():
    heads, n_q, n_keys = 4, 600, 5000
    need = kvq.kvq_attention_workspace_bytes(n_q, heads, n_keys)
    assert 0 < need <= 32 << 20  # the shape splits its keys, so the scratch is used
    caches = _caches(heads, n_keys, 500, 7)
    for call in range(2):
        q = inputs.normal((n_q, heads, D), 100 + call, "cuda")
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        got = kvq.kvq_attention_noalloc(q, caches[0], caches[1], n_keys, status=status)
        ref_status = torch.zeros(1, dtype=torch.int32, device="cuda")
        ref = kvq.kvq_attention(q, caches[0], caches[1], n_keys, status=ref_status)
        torch.cuda.synchronize()
        assert int(status.item()) == 0 and int(ref_status.item()) == 0
        assert torch.isfinite(got.float()).all()
        assert torch.equal(got.view(torch.int16), ref.view(torch.int16)), f"call {call}"


def test_noalloc_rejects_sizes_beyond_its_scratch():
    # 4096 queries x 32 heads over 93,600 keys split their keys at least in two: over
    # 100 MB of partials, beyond the 32 MiB built in, so the call is refused up front
    n_q, heads, n_keys = 4096, 32, 93600
    assert kvq.kvq_attention_workspace_bytes(n_q, heads, n_keys) > 32 << 20
    caches = _caches(heads, 16, 16, 3)
    q = torch.zeros((n_q, heads, D), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(kvq.KvqError) as e:
        kvq.kvq_attention_noalloc(q, caches[0], caches[1], n_keys)
    assert e.value.status == 4 and "scratch" in str(e.value)
