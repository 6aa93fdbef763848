"""CPU oracle for blockwise NVFP4 KV-cache quantization -- TEST INFRASTRUCTURE ONLY.

The arithmetic lives in ``kvq_oracle.c`` (plain C, one IEEE binary32 operation at a
time). This module builds that file with gcc and marshals numpy arrays to it. Only the
tests, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg may import it;
the CUDA library and its Python binding never do, and nothing here imports them.

bf16 tensors cross this boundary as ``numpy.uint16`` arrays of their bit patterns.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kvq_oracle.c")
_LIB_PATH = os.path.join(_HERE, "_build", "libkvq_oracle.so")

RULE_STATIC_6, RULE_STATIC_4, RULE_MSE = 0, 1, 2
RULES = {"static_6": RULE_STATIC_6, "static_4": RULE_STATIC_4, "mse": RULE_MSE}
BLOCK = 16

_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (no fast-math, no FP contraction)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        os.makedirs(os.path.dirname(_LIB_PATH), exist_ok=True)
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared", "-pthread",
             "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is not None:
        return _lib
    lib = ctypes.CDLL(build())
    P, I64, I32, F32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_float
    lib.orc_e2m1_encode.argtypes, lib.orc_e2m1_encode.restype = [F32], ctypes.c_uint8
    lib.orc_e2m1_decode.argtypes, lib.orc_e2m1_decode.restype = [ctypes.c_uint8], ctypes.c_double
    lib.orc_e4m3_encode.argtypes, lib.orc_e4m3_encode.restype = [F32], ctypes.c_uint8
    lib.orc_e4m3_decode.argtypes, lib.orc_e4m3_decode.restype = [ctypes.c_uint8], ctypes.c_double
    lib.orc_bf16_rne.argtypes, lib.orc_bf16_rne.restype = [F32], ctypes.c_uint16
    lib.orc_amax.argtypes, lib.orc_amax.restype = [P, I64, I32], F32
    lib.orc_quantize.argtypes = [P, I64, I32, I32, P, P, P, P, I32]
    lib.orc_quantize_block_detail.argtypes = [P, F32, I32, P, P, P, P]
    lib.orc_dequantize.argtypes = [P, P, F32, I64, I32, P, I32]
    lib.orc_append.argtypes = [P, P, P, I64, I64, I32, I64, P, I64, I32, I32]
    lib.orc_dequantize_cache.argtypes = [P, P, P, I64, I64, I32, I64, I64, P, I32]
    lib.orc_cache_bytes.argtypes = [I32, I32, I64, I32, I64, P]
    lib.orc_rtn_quantize.argtypes = [P, I64, I32, I32, P, P]
    lib.orc_rtn_dequantize.argtypes = [P, P, I64, I32, I32, P]
    lib.orc_scales_to_blocked.argtypes = [P, I64, I32, P]
    lib.orc_scales_from_blocked.argtypes = [P, I64, I32, P]
    for f in ("orc_quantize", "orc_quantize_block_detail", "orc_dequantize", "orc_append",
              "orc_dequantize_cache", "orc_cache_bytes", "orc_rtn_quantize", "orc_rtn_dequantize",
              "orc_scales_to_blocked", "orc_scales_from_blocked"):
        getattr(lib, f).restype = ctypes.c_int
    _lib = lib
    return lib


def default_threads() -> int:
    return os.cpu_count() or 1


def _ptr(a: np.ndarray) -> int:
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data


def _rule(rule) -> int:
    return RULES[rule] if isinstance(rule, str) else int(rule)


# ---- scalar formats -------------------------------------------------------------

def e2m1_encode(v: float) -> int:
    return int(_load().orc_e2m1_encode(float(v)))


def e2m1_decode(nibble: int) -> float:
    return float(_load().orc_e2m1_decode(int(nibble)))


def e4m3_encode(r: float) -> int:
    return int(_load().orc_e4m3_encode(float(r)))


def e4m3_decode(code: int) -> float:
    return float(_load().orc_e4m3_decode(int(code)))


def bf16_rne(f: float) -> int:
    return int(_load().orc_bf16_rne(float(f)))


# ---- tensors --------------------------------------------------------------------

def amax(x_bits: np.ndarray, threads: int | None = None) -> float:
    x_bits = np.ascontiguousarray(x_bits, dtype=np.uint16).reshape(-1)
    return float(_load().orc_amax(_ptr(x_bits), x_bits.size, threads or default_threads()))


def quantize(x_bits: np.ndarray, head_dim: int, rule, amax_in: float | None = None,
             threads: int | None = None):
    """Returns (packed uint8[n/2], scales uint8[n/16], amax float)."""
    x_bits = np.ascontiguousarray(x_bits, dtype=np.uint16).reshape(-1)
    n = x_bits.size
    packed = np.zeros(n // 2, np.uint8)
    scales = np.zeros(n // BLOCK, np.uint8)
    amax_out = np.zeros(1, np.float32)
    ain = None if amax_in is None else np.array([amax_in], np.float32)
    rc = _load().orc_quantize(_ptr(x_bits), n, head_dim, _rule(rule), None if ain is None else _ptr(ain),
                              _ptr(amax_out), _ptr(packed), _ptr(scales), threads or default_threads())
    if rc != 0:
        raise ValueError(f"oracle quantize: status {rc}")
    return packed, scales, float(amax_out[0])


def quantize_block_detail(x16_bits: np.ndarray, amax_t: float, rule):
    """One block: (scale code, packed[8], err6, err4); errors only for rule mse."""
    x16 = np.ascontiguousarray(x16_bits, dtype=np.uint16).reshape(-1)
    assert x16.size == BLOCK
    sc = np.zeros(1, np.uint8)
    pk = np.zeros(8, np.uint8)
    e6 = np.full(1, np.nan, np.float32)
    e4 = np.full(1, np.nan, np.float32)
    rc = _load().orc_quantize_block_detail(_ptr(x16), float(amax_t), _rule(rule), _ptr(sc), _ptr(pk),
                                           _ptr(e6), _ptr(e4))
    if rc != 0:
        raise ValueError(f"oracle block: status {rc}")
    return int(sc[0]), pk, float(e6[0]), float(e4[0])


def dequantize(packed: np.ndarray, scales: np.ndarray, amax_t: float, head_dim: int,
               threads: int | None = None) -> np.ndarray:
    """Returns the bf16 bit patterns (uint16[n])."""
    packed = np.ascontiguousarray(packed, dtype=np.uint8).reshape(-1)
    scales = np.ascontiguousarray(scales, dtype=np.uint8).reshape(-1)
    n = packed.size * 2
    y = np.zeros(n, np.uint16)
    rc = _load().orc_dequantize(_ptr(packed), _ptr(scales), float(amax_t), n, head_dim, _ptr(y),
                                threads or default_threads())
    if rc != 0:
        raise ValueError(f"oracle dequantize: status {rc}")
    return y


class Cache:
    """Host-side packed cache for one (layer, K or V) tensor, token-major rows."""

    def __init__(self, capacity_rows: int, rows_per_chunk: int, head_dim: int):
        self.capacity_rows, self.rows_per_chunk, self.head_dim = capacity_rows, rows_per_chunk, head_dim
        n = capacity_rows * head_dim
        self.packed = np.zeros(n // 2, np.uint8)
        self.scales = np.zeros(n // BLOCK, np.uint8)
        self.amax = np.zeros(-(-capacity_rows // rows_per_chunk), np.float32)

    def append(self, row_offset: int, x_bits: np.ndarray, rule, threads: int | None = None) -> int:
        x_bits = np.ascontiguousarray(x_bits, dtype=np.uint16).reshape(-1)
        n_rows = x_bits.size // self.head_dim
        return _load().orc_append(_ptr(self.packed), _ptr(self.scales), _ptr(self.amax), self.capacity_rows,
                                  self.rows_per_chunk, self.head_dim, row_offset, _ptr(x_bits), n_rows,
                                  _rule(rule), threads or default_threads())

    def dequantize(self, row_begin: int, row_end: int, threads: int | None = None) -> np.ndarray:
        y = np.zeros(max(row_end - row_begin, 0) * self.head_dim, np.uint16)
        rc = _load().orc_dequantize_cache(_ptr(self.packed), _ptr(self.scales), _ptr(self.amax),
                                          self.capacity_rows, self.rows_per_chunk, self.head_dim, row_begin,
                                          row_end, _ptr(y) if y.size else None, threads or default_threads())
        if rc != 0:
            raise ValueError(f"oracle dequantize_cache: status {rc}")
        return y


def cache_bytes(layers: int, heads: int, capacity_tokens: int, head_dim: int, tokens_per_chunk: int):
    """(packed bytes, scale bytes, amax bytes) for layers x {K, V}."""
    out = np.zeros(3, np.uint64)
    rc = _load().orc_cache_bytes(layers, heads, capacity_tokens, head_dim, tokens_per_chunk, _ptr(out))
    if rc != 0:
        raise ValueError(f"oracle cache_bytes: status {rc}")
    return int(out[0]), int(out[1]), int(out[2])


# ---- RTN integer codecs -----------------------------------------------------------

def rtn_quantize(x_bits: np.ndarray, head_dim: int, bits: int):
    """Returns (packed uint8[n*bits/8], scales as bf16 bit patterns uint16[n/16])."""
    x_bits = np.ascontiguousarray(x_bits, dtype=np.uint16).reshape(-1)
    n = x_bits.size
    packed = np.zeros(n * bits // 8, np.uint8)
    scales = np.zeros(n // BLOCK, np.uint16)
    rc = _load().orc_rtn_quantize(_ptr(x_bits), n, head_dim, bits, _ptr(packed), _ptr(scales))
    if rc != 0:
        raise ValueError(f"oracle rtn_quantize: status {rc}")
    return packed, scales


def rtn_dequantize(packed: np.ndarray, scales: np.ndarray, head_dim: int, bits: int) -> np.ndarray:
    packed = np.ascontiguousarray(packed, dtype=np.uint8).reshape(-1)
    scales = np.ascontiguousarray(scales, dtype=np.uint16).reshape(-1)
    n = packed.size * 8 // bits
    y = np.zeros(n, np.uint16)
    rc = _load().orc_rtn_dequantize(_ptr(packed), _ptr(scales), n, head_dim, bits, _ptr(y))
    if rc != 0:
        raise ValueError(f"oracle rtn_dequantize: status {rc}")
    return y


# ---- RECENT cache policy ---------------------------------------------------------------

class RecentCache:
    """The RTN_INT4 RECENT2 cache policy of the Self-Forcing study (appendix Table 3),
    step by step: the newest `recent_blocks` frame-blocks are kept as bf16 state; when a
    block is appended, the block falling out of that window is RTN-quantized (bits) into
    the prefix; a read dequantizes the prefix and appends the bf16 tail."""

    def __init__(self, rows_per_block: int, head_dim: int, bits: int = 4, recent_blocks: int = 2):
        self.rows_per_block, self.head_dim, self.bits, self.recent_blocks = rows_per_block, head_dim, bits, recent_blocks
        self.prefix = []  # (packed, scales) of quantized blocks 0, 1, ...
        self.recent = []  # bf16 bit patterns of the newest blocks, oldest first

    def append(self, x_bits: np.ndarray):
        x_bits = np.ascontiguousarray(x_bits, dtype=np.uint16).reshape(-1)
        assert x_bits.size == self.rows_per_block * self.head_dim
        self.recent.append(x_bits.copy())
        if len(self.recent) > self.recent_blocks:
            self.prefix.append(rtn_quantize(self.recent.pop(0), self.head_dim, self.bits))

    def read(self) -> np.ndarray:
        parts = [rtn_dequantize(p, s, self.head_dim, self.bits) for p, s in self.prefix] + list(self.recent)
        return np.concatenate(parts) if parts else np.zeros(0, np.uint16)


# ---- blocked scale layout ----------------------------------------------------------

def blocked_bytes(rows: int, cols: int) -> int:
    return -(-rows // 128) * 128 * -(-cols // 4) * 4


def scales_to_blocked(scales: np.ndarray, rows: int, cols: int) -> np.ndarray:
    scales = np.ascontiguousarray(scales, dtype=np.uint8).reshape(-1)
    out = np.zeros(blocked_bytes(rows, cols), np.uint8)
    if _load().orc_scales_to_blocked(_ptr(scales), rows, cols, _ptr(out)) != 0:
        raise ValueError("oracle scales_to_blocked: bad shape")
    return out


def scales_from_blocked(blocked: np.ndarray, rows: int, cols: int) -> np.ndarray:
    blocked = np.ascontiguousarray(blocked, dtype=np.uint8).reshape(-1)
    out = np.zeros(rows * cols, np.uint8)
    if _load().orc_scales_from_blocked(_ptr(blocked), rows, cols, _ptr(out)) != 0:
        raise ValueError("oracle scales_from_blocked: bad shape")
    return out


# ---- attention over a dequantized cache ---------------------------------------------

def attention(q_bits: np.ndarray, k_bits: np.ndarray, v_bits: np.ndarray, n_queries: int, n_keys: int,
              heads: int, head_dim: int, scale: float) -> np.ndarray:
    """softmax(Q K^T * scale) V per head, in fp64, on bf16 inputs given as bit patterns:
    q [n_queries, heads, head_dim], k and v [n_keys, heads, head_dim] (token-major, the
    cache's row order). Returns fp64 [n_queries, heads, head_dim]. This is the consumer
    the pages place after dequantization (the Self-Forcing study, appendix Table 3:
    the active cache is turned back into dense BF16 and then attended over)."""
    def f64(b, rows):
        u = (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)
        return u.astype(np.float64).reshape(rows, heads, head_dim)
    q, k, v = f64(q_bits, n_queries), f64(k_bits, n_keys), f64(v_bits, n_keys)
    out = np.empty((n_queries, heads, head_dim))
    for h in range(heads):
        s = q[:, h, :] @ k[:, h, :].T * scale
        s -= s.max(axis=1, keepdims=True)
        p = np.exp(s)
        out[:, h, :] = (p @ v[:, h, :]) / p.sum(axis=1, keepdims=True)
    return out
