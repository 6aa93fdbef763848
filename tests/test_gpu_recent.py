"""Bit-exact parity of the RECENT cache policy (RTN_INT4 RECENT2 of the Self-Forcing
study) through the C ABI against the oracle, read back after every append."""
import numpy as np
import pytest
import torch

import nvfp4_kv_cache_kvq_b200 as kvq
from gpu_helpers import assert_same
from nvfp4_kv_cache_kvq_b200 import inputs
from nvfp4_kv_cache_kvq_b200.inputs import bits

pytestmark = pytest.mark.gpu
D = 128


@pytest.mark.parametrize("R,nbits,n_blocks,rows,n_caches", [
    (2, 4, 7, 24, 3),    # the study's RECENT2 with an INT4 prefix
    (1, 4, 4, 16, 1),
    (3, 2, 6, 40, 2),
    (2, 4, 2, 8, 2),     # never evicts
    (2, 4, 70, 12, 65),  # more caches than one launch batch
])
def test_recent_append_and_read_match_oracle(orc, R, nbits, n_blocks, rows, n_caches):
    caches = [kvq.RecentCache(n_blocks, rows, D, nbits, R) for _ in range(n_caches)]
    ocs = [orc.RecentCache(rows, D, nbits, R) for _ in range(n_caches)]
    for b in range(n_blocks):
        xs = [inputs.student_t((rows, D), 4, 1000 * i + b, "cuda") for i in range(n_caches)]
        kvq.kvq_recent_append_batch(caches, b, xs)
        for oc, x in zip(ocs, xs):
            oc.append(bits(x))
        if b < 3 or b == n_blocks - 1 or n_caches <= 3:
            ys = kvq.kvq_recent_read_batch(caches, b + 1)
            torch.cuda.synchronize()
            for y, oc in zip(ys, ocs):
                assert_same(bits(y), oc.read(), f"recent read after block {b}")


def test_recent_rollout_shape(orc):
    """One rollout-shaped cache (1560 tokens x 12 heads per frame, RECENT2 over INT4),
    12 frames: the GPU read equals the oracle's after the last append."""
    rows, frames = 1560 * 12, 12
    c = kvq.RecentCache(frames, rows, D, 4, 2)
    oc = orc.RecentCache(rows, D, 4, 2)
    for f in range(frames):
        x = inputs.rollout_chunk(f, 0, device="cuda").reshape(-1, D)
        kvq.kvq_recent_append_batch([c], f, [x])
        oc.append(bits(x))
    y = kvq.kvq_recent_read_batch([c], frames)[0]
    torch.cuda.synchronize()
    assert_same(bits(y), oc.read(), "recent rollout read")


def test_recent_errors():
    c = kvq.RecentCache(2, 8, D, 4, 2)
    x = torch.zeros((8, D), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(kvq.KvqError):
        kvq.kvq_recent_append_batch([c], 2, [x])  # past capacity
    with pytest.raises(kvq.KvqError):
        kvq.kvq_recent_read_batch([c], 3)
    with pytest.raises(kvq.KvqError):
        kvq.kvq_recent_append_batch([c, kvq.RecentCache(2, 8, D, 2, 2)], 0, [x, x])  # mixed bits
