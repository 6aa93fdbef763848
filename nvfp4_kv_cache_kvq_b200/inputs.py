"""Seeded synthetic K/V inputs shaped like the Wan / Self-Forcing KV caches.

This module only draws random numbers and lays them out; it holds none of the
quantization arithmetic. The tests, the benchmark and the CPU oracle's callers all take
their inputs from here, so the GPU path and the oracle always see the same bytes.

Workloads (K/V shapes of a Wan-style causal video DiT: 1560 tokens per latent frame,
head_dim 128; the Self-Forcing study, "KV Cache Quantization for Self-Forcing Video
Generation", runs a Wan2.1 stack, Table 2):

* ``single``  -- one K tensor [4096, 128], N(0, 1), seed 0.
* ``layer``   -- one layer's K and V [1, 24, 4680, 128], Student-t(3) with 4 outlier
  channels per head scaled x20; seeds 0 (K) and 1 (V).
* ``cache``   -- 30 layers x {K, V} of [1, 24, 32760, 128], N(0, 1) with 1% of the
  tokens (all heads and channels of those tokens) scaled x10; seed 1000*layer + kv.
* ``rollout`` -- per step, 30 layers x {K, V} chunks of [1560, 12, 128] (token-major),
  Student-t(4); seed step*60 + tensor.
* ``sweep``   -- [T, 128] N(0, 1) for T = 2^10 .. 2^26; seed T.
* ``queries`` -- attention queries of one frame [1560, 12, 128] (token-major), N(0, 1);
  seed 1_000_000 + step (the pages give no query statistics; N(0, 1) is the plainest).

Everything is drawn in fp32 with ``torch.Generator`` and rounded to bf16 by torch.
Student-t(nu) for integer nu is drawn as Z / sqrt(chi2_nu / nu), with chi2_nu the sum
of nu squared standard normals.
"""
from __future__ import annotations

import torch

HEAD_DIM = 128
TOKENS_PER_FRAME = 1560


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def normal(shape, seed: int, device="cpu") -> torch.Tensor:
    g = _gen(seed, device)
    return torch.randn(shape, generator=g, device=device, dtype=torch.float32).to(torch.bfloat16)


def _student_t_f32(shape, nu: int, g: torch.Generator, device) -> torch.Tensor:
    z = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    chi2 = torch.zeros(shape, device=device, dtype=torch.float32)
    for _ in range(nu):
        w = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
        chi2.add_(w * w)
    return z / torch.sqrt(chi2 / nu)


def student_t(shape, nu: int, seed: int, device="cpu") -> torch.Tensor:
    return _student_t_f32(shape, nu, _gen(seed, device), device).to(torch.bfloat16)


def single_k(device="cpu") -> torch.Tensor:
    """bf16 [4096, 128], N(0, 1), seed 0."""
    return normal((4096, HEAD_DIM), 0, device)


def layer_kv(kv: int, heads: int = 24, tokens: int = 3 * TOKENS_PER_FRAME, device="cpu") -> torch.Tensor:
    """bf16 [1, heads, tokens, 128], Student-t(3); per head 4 channels scaled x20."""
    x = _student_t_f32((1, heads, tokens, HEAD_DIM), 3, _gen(kv, device), device)
    gc = torch.Generator(device="cpu")
    gc.manual_seed(10_000 + kv)
    for h in range(heads):
        ch = torch.randperm(HEAD_DIM, generator=gc)[:4].to(device)
        x[0, h, :, ch] *= 20.0
    return x.to(torch.bfloat16)


def cache_kv(layer: int, kv: int, heads: int = 24, tokens: int = 21 * TOKENS_PER_FRAME,
             device="cpu") -> torch.Tensor:
    """bf16 [1, heads, tokens, 128], N(0, 1); 1% of tokens scaled x10."""
    seed = 1000 * layer + kv
    g = _gen(seed, device)
    x = torch.randn((1, heads, tokens, HEAD_DIM), generator=g, device=device, dtype=torch.float32)
    gc = torch.Generator(device="cpu")
    gc.manual_seed(seed)
    n_out = max(1, tokens // 100)
    idx = torch.randperm(tokens, generator=gc)[:n_out].to(device)
    x[:, :, idx, :] *= 10.0
    return x.to(torch.bfloat16)


def rollout_chunk(step: int, tensor: int, heads: int = 12, tokens: int = TOKENS_PER_FRAME,
                  device="cpu") -> torch.Tensor:
    """bf16 [tokens, heads, 128] (token-major), Student-t(4), seed step*60 + tensor."""
    return student_t((tokens, heads, HEAD_DIM), 4, step * 60 + tensor, device)


def queries(step: int, heads: int = 12, tokens: int = TOKENS_PER_FRAME, device="cpu") -> torch.Tensor:
    """bf16 [tokens, heads, 128] (token-major), N(0, 1), seed 1_000_000 + step."""
    return normal((tokens, heads, HEAD_DIM), 1_000_000 + step, device)


def sweep(tokens: int, device="cpu") -> torch.Tensor:
    """bf16 [tokens, 128], N(0, 1), seed = tokens."""
    return normal((tokens, HEAD_DIM), tokens, device)


def scale_codes(rows: int, cols: int, seed: int, device="cpu") -> torch.Tensor:
    """uint8 [rows * cols] e4m3 scale codes, uniform over 0x30 .. 0x6F (block scales
    2^-3 .. 2^4 times the tensor's global scale), seed `seed`."""
    g = _gen(seed, device)
    return torch.randint(0x30, 0x70, (rows * cols,), generator=g, device=device, dtype=torch.int32).to(torch.uint8)


def bits(x: torch.Tensor):
    """The bf16 bit patterns of a tensor as a flat numpy uint16 array (host copy)."""
    return x.detach().contiguous().view(torch.int16).cpu().numpy().view("uint16").reshape(-1)
