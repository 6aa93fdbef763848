"""A model of the one-launch quantizer's schedule, checked for progress on the CPU.

The kernel deals the tiles of all tensors (tensor-major) round-robin to G resident CTAs.
In each CTA an amax warp takes its tiles' amax parts in order, never more than W tiles
ahead of the position its own quantize warps have published (0 before the first tile),
and the quantize warps take the same tiles in order, each once every amax tile of its
tensor is in. The model runs those two steps per CTA under random interleavings and
asserts that every run finishes for the window the host chooses (one tensor and one and a
half grids) and for the smallest window the progress argument needs (one tensor), and that
a window below that can stall (so the model can fail)."""
import random

import pytest


def _run(G, N, T, W, rng, max_steps=1_000_000):
    M = N * T
    seq = [list(range(b, M, G)) for b in range(G)]
    a_idx = [0] * G  # next amax tile (index into seq[b])
    q_idx = [0] * G  # next quantize tile
    q_pos = [0] * G  # published quantize position; None once the CTA has no more tiles
    folded = [0] * N
    for _ in range(max_steps):
        enabled = []
        for b in range(G):
            if a_idx[b] < len(seq[b]):
                a = seq[b][a_idx[b]]
                if q_pos[b] is None or a <= q_pos[b] + W:
                    enabled.append(("a", b))
            if q_idx[b] < len(seq[b]):
                q = seq[b][q_idx[b]]
                # a step either publishes the position or quantizes a tile whose tensor
                # is complete; a wait that changes nothing is not a step
                if q_pos[b] != q or folded[q // T] == T:
                    enabled.append(("q", b))
        if not enabled:
            return all(x == T for x in folded) and all(q_idx[b] == len(seq[b]) for b in range(G))
        kind, b = rng.choice(enabled)
        if kind == "a":
            folded[seq[b][a_idx[b]] // T] += 1
            a_idx[b] += 1
        else:
            q = seq[b][q_idx[b]]
            q_pos[b] = q  # published before the wait, as the quantize leader does
            if folded[q // T] == T:  # the tensor's amax is complete: the tile is quantized
                q_idx[b] += 1
                if q_idx[b] == len(seq[b]):
                    q_pos[b] = None
            # else: waiting; the published position stays
    raise AssertionError("no progress decision within the step budget")


CASES = [(1, 1, 1), (1, 3, 4), (3, 1, 7), (4, 5, 3), (7, 2, 11), (8, 6, 5), (16, 3, 40), (5, 9, 2)]


@pytest.mark.parametrize("G,N,T", CASES)
def test_host_window_always_finishes(G, N, T):
    rng = random.Random(1000 * G + 10 * N + T)
    W = T + G + G // 2
    for _ in range(60):
        assert _run(G, N, T, W, rng)


@pytest.mark.parametrize("G,N,T", CASES)
def test_one_tensor_window_always_finishes(G, N, T):
    rng = random.Random(7 + 1000 * G + 10 * N + T)
    for _ in range(60):
        assert _run(G, N, T, T, rng)


def test_a_window_below_one_tensor_can_stall():
    # one CTA, one tensor of three tiles, window 0: the amax warp may take tile 0 only
    # until the quantize warps move, and they wait for all three tiles
    assert not _run(1, 1, 3, 0, random.Random(1))
    stalled = sum(not _run(4, 2, 9, 2, random.Random(s)) for s in range(40))
    assert stalled > 0
