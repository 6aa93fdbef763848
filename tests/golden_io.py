"""Reader for the hand-worked fixtures under tests/golden/."""
import os

import numpy as np
import torch

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def read_sections(name: str) -> dict:
    """Parse 'key: v v v' / 'key:' + following lines into {key: [tokens]}."""
    out, key = {}, None
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            if ":" in line:
                key, rest = line.split(":", 1)
                key = key.strip()
                out[key] = rest.split()
            else:
                out[key].extend(line.split())
    return out


def floats_to_bf16_bits(vals) -> np.ndarray:
    """Exact bf16 bit patterns of decimal literals (asserts each is representable)."""
    f = torch.tensor([float(v) for v in vals], dtype=torch.float64)
    b = f.to(torch.bfloat16)
    assert torch.equal(b.to(torch.float64), f), "golden literal not representable in bf16"
    return b.view(torch.int16).numpy().view(np.uint16).copy()


def hex_bytes(tokens) -> np.ndarray:
    return np.array([int(t, 16) for t in tokens], dtype=np.uint8)


def round_to_bf16_bits(vals) -> np.ndarray:
    """bf16 bit patterns of arbitrary values, rounded to nearest even by torch."""
    f = torch.as_tensor(np.asarray(vals, dtype=np.float64))
    return f.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16).copy()
