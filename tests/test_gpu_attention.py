"""Parity of the fused consumer kvq_attention (softmax attention reading K and V from
their NVFP4 caches) against the fp64 oracle attention over the oracle's own dequantized
cache.

Tolerance, derived from the kernel's arithmetic: Q K^T is exact products summed in fp32;
P = exp2(s - m) is rounded to bf16 (relative error <= 2^-9 per element) before P V, whose
sums are fp32; the output O / l is rounded to bf16 (<= 2^-9 relative). The P rounding moves
the output by at most 2^-9 * sum_i p_i |v_i| / l, i.e. 2^-9 times the attention of |V|,
which the oracle computes. The bound used, 2^-8 * (attn(|V|) + |out|) + 2^-20, doubles both
terms to absorb the fp32 accumulation and exp2 errors (below 1e-4 relative at these
magnitudes). With a single key the result is exact: p = 1, so out is that key's V row,
value for value as the oracle dequantizes it."""
import numpy as np
import pytest
import torch

import nvfp4_kv_cache_kvq_b200 as kvq
from gpu_helpers import assert_same
from nvfp4_kv_cache_kvq_b200 import inputs
from nvfp4_kv_cache_kvq_b200.inputs import bits

pytestmark = pytest.mark.gpu
D = 128


def _filled_caches(orc, heads, n_tokens, tokens_per_chunk, rule, seed):
    """A K and a V cache of n_tokens tokens appended chunk by chunk on the GPU and in the
    oracle from the same inputs; returns (gpu caches, oracle caches)."""
    rpc = tokens_per_chunk * heads
    n_chunks = -(-n_tokens // tokens_per_chunk)
    caches = [kvq.KVCache(n_chunks * rpc, rpc, D) for _ in range(2)]
    ocs = [orc.Cache(n_chunks * rpc, rpc, D) for _ in range(2)]
    for c in range(n_chunks):
        toks = min(tokens_per_chunk, n_tokens - c * tokens_per_chunk)
        for t in range(2):
            x = inputs.student_t((toks, heads, D), 4, seed + 2 * c + t, "cuda")
            kvq.kvq_append(caches[t], c * rpc, x, rule)
            assert ocs[t].append(c * rpc, bits(x), rule) == 0
    torch.cuda.synchronize()
    for t in range(2):
        assert_same(caches[t].packed.cpu().numpy(), ocs[t].packed, "packed cache")
        assert_same(caches[t].scales.cpu().numpy(), ocs[t].scales, "cache scales")
    return caches, ocs


def _abs_bits(b: np.ndarray) -> np.ndarray:
    return (b & 0x7FFF).astype(np.uint16)


def _check_close(orc, got: torch.Tensor, qb, kb, vb, n_q, n_keys, heads, scale):
    want = orc.attention(qb, kb, vb, n_q, n_keys, heads, D, scale)
    mag = orc.attention(qb, kb, _abs_bits(vb), n_q, n_keys, heads, D, scale)
    g = got.float().cpu().numpy().astype(np.float64).reshape(want.shape)
    tol = 2.0 ** -8 * (mag + np.abs(want)) + 2.0 ** -20
    err = np.abs(g - want)
    bad = np.argwhere(err > tol)
    assert bad.size == 0, (f"{len(bad)} of {err.size} outside tolerance; first {bad[:4].tolist()}: "
                           f"got {g[tuple(bad[0])]} want {want[tuple(bad[0])]} tol {tol[tuple(bad[0])]}")
    assert np.isfinite(g).all()


@pytest.mark.parametrize("n_q,heads,tokens_per_chunk", [(1, 1, 1), (130, 3, 7), (256, 2, 64), (300, 2, 5)])
def test_single_key_returns_v_row_exactly(orc, n_q, heads, tokens_per_chunk):
    caches, ocs = _filled_caches(orc, heads, 2 * tokens_per_chunk, tokens_per_chunk, "mse", 11)
    q = inputs.normal((n_q, heads, D), 5, "cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = kvq.kvq_attention(q, caches[0], caches[1], 1, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    v0 = ocs[1].dequantize(0, heads).reshape(heads, D)  # token 0, every head
    want = np.broadcast_to(v0, (n_q, heads, D)).reshape(-1)
    # equal values; a -0 of V may come out +0 (the MMA adds the masked keys' +0 products)
    got = bits(out)
    got_f = (got.astype(np.uint32) << 16).view(np.float32)
    want_f = (want.astype(np.uint32) << 16).view(np.float32)
    bad = np.nonzero(got_f != want_f)[0]
    assert bad.size == 0, (f"{bad.size} of {got.size} differ; first at {bad[:8].tolist()}: "
                           f"got {got[bad[:8]].tolist()} want {want[bad[:8]].tolist()}")


def _workspace(split):
    # "auto": the recommended workspace (keys split to fill the GPU); "none": no split
    return None if split == "auto" else torch.empty(0, dtype=torch.uint8, device="cuda")


@pytest.mark.parametrize("split", ["auto", "none"])
@pytest.mark.parametrize("n_q,heads,n_keys,tokens_per_chunk,rule", [
    (1, 1, 1, 1, "static_6"),
    (130, 3, 200, 50, "mse"),       # ragged query and key tiles, chunks inside a tile
    (128, 2, 384, 128, "static_6"),  # exact tiles
    (257, 2, 129, 64, "static_4"),   # one key past a tile; a second query pair
    (64, 4, 1000, 100, "mse"),
    (600, 1, 2000, 300, "mse"),      # three query pairs, the last with one partial tile
    # CTA pairs (cta_group::2) take these: 2 x 15/16 x ceil(n_q / 512) < ceil(n_q / 256)
    (400, 2, 300, 100, "mse"),       # one pair; CTA 1's second slot holds 16 rows
    (1024, 1, 385, 64, "static_6"),  # two full pairs, a partial last key tile
    # at most 128 rows: the CTA's two slots split its key range (dual); with two key
    # ranges of 2 and 3 tiles, the second range's slots take 2 and 1, the last ragged
    (100, 2, 5 * 128 - 7, 100, "static_4"),
])
def test_attention_matches_oracle(orc, n_q, heads, n_keys, tokens_per_chunk, rule, split):
    caches, ocs = _filled_caches(orc, heads, n_keys, tokens_per_chunk, rule, 100)
    q = inputs.normal((n_q, heads, D), 7, "cuda")
    scale = D ** -0.5
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = kvq.kvq_attention(q, caches[0], caches[1], n_keys, scale, workspace=_workspace(split), status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    kb, vb = ocs[0].dequantize(0, n_keys * heads), ocs[1].dequantize(0, n_keys * heads)
    _check_close(orc, out, bits(q), kb, vb, n_q, n_keys, heads, scale)


@pytest.mark.parametrize("n_q,heads,n_keys,tokens_per_chunk,rule", [
    # one pair unit and a 24-row dual part: the pair launch's 61 key ranges hold 4 or 5
    # tiles, the dual CTAs' 50 ranges 6 or 7 (slots of 3 and 3, or 4 and 3)
    (536, 1, 301 * 128 - 5, 1000, "mse"),
    # two pair units per head over 17 key ranges of 5 or 6 tiles; a 100-row dual part
    # over 50 ranges of 2 tiles (one per slot)
    (1124, 2, 100 * 128, 128, "static_6"),
])
def test_pairs_then_dual_with_ragged_key_ranges(orc, n_q, heads, n_keys, tokens_per_chunk, rule):
    """A pair part followed by a dual part, both over key ranges of unequal length."""
    assert kvq.kvq_attention_launches(n_q, heads, n_keys) == 4
    caches, ocs = _filled_caches(orc, heads, n_keys, tokens_per_chunk, rule, 700)
    q = inputs.normal((n_q, heads, D), 13, "cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = kvq.kvq_attention(q, caches[0], caches[1], n_keys, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    kb, vb = ocs[0].dequantize(0, n_keys * heads), ocs[1].dequantize(0, n_keys * heads)
    _check_close(orc, out, bits(q), kb, vb, n_q, n_keys, heads, D ** -0.5)


def test_attention_many_key_splits(orc):
    """One query tile of one head over 64 key tiles: the split heuristic spreads the keys
    over the most units (up to 64), so the combine merges many partials."""
    heads, n_keys, n_q = 1, 64 * 128 - 3, 100
    assert kvq.kvq_attention_workspace_bytes(n_q, heads, n_keys) >= 32 * n_q * heads * (128 * 4 + 8)
    caches, ocs = _filled_caches(orc, heads, n_keys, 1000, "mse", 500)
    q = inputs.normal((n_q, heads, D), 11, "cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = kvq.kvq_attention(q, caches[0], caches[1], n_keys, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    kb, vb = ocs[0].dequantize(0, n_keys * heads), ocs[1].dequantize(0, n_keys * heads)
    _check_close(orc, out, bits(q), kb, vb, n_q, n_keys, heads, D ** -0.5)


def test_attention_peaked_scores(orc):
    """Large scores: the running max moves between key tiles, so O is rescaled."""
    heads, n_keys, n_q = 2, 640, 128
    caches, ocs = _filled_caches(orc, heads, n_keys, 128, "mse", 300)
    q = (inputs.normal((n_q, heads, D), 9, "cuda").float() * 4).to(torch.bfloat16)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = kvq.kvq_attention(q, caches[0], caches[1], n_keys, 1.0, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    kb, vb = ocs[0].dequantize(0, n_keys * heads), ocs[1].dequantize(0, n_keys * heads)
    _check_close(orc, out, bits(q), kb, vb, n_q, n_keys, heads, 1.0)


def test_workspace_size_and_split_agree():
    """The recommended workspace is 0 exactly when no split is used, and a split result
    agrees with the unsplit one (both are checked against the oracle above). 1560 queries
    over 732 key tiles split the keys of every query row at least in two, in 256-byte
    aligned regions (one per launch part)."""
    assert kvq.kvq_attention_workspace_bytes(1, 1, 1) == 0
    b = kvq.kvq_attention_workspace_bytes(1560, 12, 93600)
    assert b >= 2 * 1560 * 12 * (128 * 4 + 8) and b % 256 == 0


@pytest.mark.parametrize("log2_scale", [-133, -125, -121, -119, -118, -100, -40, 0, 40, 100, 120])
def test_attention_dequantizes_like_the_cache_reader(log2_scale):
    """The K/V tiles the attention kernel dequantizes on chip are the bf16 values
    kvq_dequantize_cache writes, bit for bit, whatever the chunk amax: with one key and
    zero queries, softmax gives p = 1 and the output is that key's V row exactly. The
    scales 2^-133 .. 2^120 cover amax whose global scale amax / 2688 is subnormal (the
    kernel then divides) and the normal range (it uses a correction step). At 2^-133
    every value dequantizes to a signed zero."""
    heads, n_q = 4, 3
    x = (inputs.normal((1, heads, D), 1000 + log2_scale, "cuda").double() * 2.0 ** log2_scale).to(torch.bfloat16)
    caches = [kvq.KVCache(heads, heads, D) for _ in range(2)]
    for c in caches:
        kvq.kvq_append(c, 0, x, "mse")
    q = torch.zeros((n_q, heads, D), dtype=torch.bfloat16, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = kvq.kvq_attention(q, caches[0], caches[1], 1, status=status)
    v = kvq.kvq_dequantize_cache(caches[1], 0, heads).view(1, heads, D)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    # compared as values: equal bf16 values have equal bits, except -0, which the sum
    # P V turns into +0
    want = v.expand(n_q, heads, D).float()
    assert torch.equal(out.float(), want)


def test_attention_launch_count():
    """The launch plan as kvq_attention_launches reports it: 1560 queries run as CTA pairs
    over 1536 rows and single CTAs over the last 24, each part splitting its keys (two
    attention launches, two combines); 2048 queries are all pairs; one query over one key
    tile is a single unsplit launch."""
    assert kvq.kvq_attention_launches(0, 12, 100) == 0
    assert kvq.kvq_attention_launches(1, 1, 1) == 1
    assert kvq.kvq_attention_launches(1560, 12, 93600) == 4
    assert kvq.kvq_attention_launches(2048, 12, 93600) == 2


def test_attention_rollout_shape_sampled(orc):
    """The rollout's attention at full size -- one frame of 1560 queries x 12 heads over a
    60-frame cache (93,600 keys) appended frame by frame with the mse rule -- checked on a
    sample of query rows of the pair part and on every row of the 24-row remainder that
    runs on single CTAs (the oracle computes those rows only)."""
    heads, tpc, frames = 12, inputs.TOKENS_PER_FRAME, 60
    rpc = tpc * heads
    caches = [kvq.KVCache(frames * rpc, rpc, D) for _ in range(2)]
    ocs = [orc.Cache(frames * rpc, rpc, D) for _ in range(2)]
    for step in range(frames):
        for t in range(2):
            x = inputs.rollout_chunk(step, t, heads, device="cuda")
            kvq.kvq_append(caches[t], step * rpc, x, "mse")
            assert ocs[t].append(step * rpc, bits(x), "mse") == 0
    q = inputs.queries(frames - 1, heads, device="cuda")
    n_keys = frames * tpc
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = kvq.kvq_attention(q, caches[0], caches[1], n_keys, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    rows = torch.tensor([0, 1, 127, 128, 777, 1400, 1535] + list(range(1536, 1560)))
    kb, vb = ocs[0].dequantize(0, n_keys * heads), ocs[1].dequantize(0, n_keys * heads)
    _check_close(orc, out[rows.cuda()], bits(q[rows.cuda()]), kb, vb, len(rows), n_keys, heads, D ** -0.5)


def test_attention_argument_errors():
    c = kvq.KVCache(64, 16, D)
    q = torch.zeros((4, 2, D), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(kvq.KvqError):  # rows_per_chunk 16 is not a multiple of 3 heads
        kvq.kvq_attention(torch.zeros((4, 3, D), dtype=torch.bfloat16, device="cuda"), c, c, 4)
    with pytest.raises(kvq.KvqError):  # 33 keys x 2 heads > 64 rows
        kvq.kvq_attention(q, c, c, 33)
    with pytest.raises(kvq.KvqError):  # no keys
        kvq.kvq_attention(q, c, c, 0)
    c64 = kvq.KVCache(64, 16, 64)
    with pytest.raises(kvq.KvqError):  # head_dim 64 unsupported
        kvq.kvq_attention(torch.zeros((4, 2, 64), dtype=torch.bfloat16, device="cuda"), c64, c64, 4)


@pytest.mark.parametrize("n_q,heads,n_tokens", [(100, 2, 700), (1100, 2, 900)])
def test_wait_that_gives_up_sets_status_and_the_next_call_is_exact(orc, n_q, heads, n_tokens):
    """With the test hook the MMA warp first waits on an mbarrier nothing arrives on and
    every wait gives up after 1 ms: status is 1 and the binding's check raises
    KVQ_ERR_TIMEOUT. The call drains and frees its tensor memory, which the next call on
    the same stream shows: status 0 and the oracle's result. 100 queries run on single
    CTAs, 1100 on CTA pairs plus a remainder."""
    caches, ocs = _filled_caches(orc, heads, n_tokens, 64, "mse", 23)
    q = inputs.normal((n_q, heads, D), 29, "cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    try:
        kvq.testing_set_attention_wait(1_000_000)
        kvq.kvq_attention(q, caches[0], caches[1], n_tokens, status=status)
        torch.cuda.synchronize()
        assert int(status.item()) == 1
        with pytest.raises(kvq.KvqError) as e:
            kvq.kvq_attention(q, caches[0], caches[1], n_tokens, check=True)
        assert e.value.status == 6
    finally:
        kvq.testing_set_attention_wait(0)
    status.zero_()
    out = kvq.kvq_attention(q, caches[0], caches[1], n_tokens, status=status, check=True)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    kb = ocs[0].dequantize(0, n_tokens * heads)
    vb = ocs[1].dequantize(0, n_tokens * heads)
    _check_close(orc, out, bits(q), kb, vb, n_q, n_tokens, heads, D ** -0.5)


@pytest.mark.parametrize("fraction", [0.5, 0.1])
def test_smaller_workspace_than_recommended(orc, fraction):
    """A workspace smaller than recommended (but not empty) makes the launch plan shrink:
    fewer key splits for the part with the most partials, then no dual mode, offsets
    recomputed. 600 queries x 4 heads run a pair part and a remainder part; the result
    stays within the oracle's bound."""
    n_q, heads, n_tokens = 600, 4, 5000
    caches, ocs = _filled_caches(orc, heads, n_tokens, 500, "mse", 31)
    q = inputs.normal((n_q, heads, D), 37, "cuda")
    need = kvq.kvq_attention_workspace_bytes(n_q, heads, n_tokens)
    assert need > 0 and kvq.kvq_attention_launches(n_q, heads, n_tokens) >= 3
    ws = torch.empty(int(need * fraction) // 256 * 256, dtype=torch.uint8, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = kvq.kvq_attention(q, caches[0], caches[1], n_tokens, workspace=ws, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    kb = ocs[0].dequantize(0, n_tokens * heads)
    vb = ocs[1].dequantize(0, n_tokens * heads)
    _check_close(orc, out, bits(q), kb, vb, n_q, n_tokens, heads, D ** -0.5)
