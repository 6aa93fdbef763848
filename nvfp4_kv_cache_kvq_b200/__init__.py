"""nvfp4_kv_cache_kvq_b200 -- blockwise NVFP4 KV-cache quantization for B200.

Thin Python binding of ``libkvq.so`` (C ABI in ``include/kvq.h``). The functions here
carry the C names and only marshal arguments: torch tensors become device pointers,
the current torch CUDA stream becomes the ``cudaStream_t``, and missing outputs are
allocated with torch. Every step of the computation runs in the library's CUDA kernels;
there is no other code path. Loading fails loudly when the library cannot be built or
loaded.
"""
from __future__ import annotations

import ctypes
import os

import torch

from . import build as _build

BLOCK = 16
RULES = {"static_6": 0, "static_4": 1, "mse": 2}
STATUS = {0: "KVQ_OK", 1: "KVQ_ERR_INVALID_ARG", 2: "KVQ_ERR_MISALIGNED", 3: "KVQ_ERR_UNSUPPORTED",
          4: "KVQ_ERR_CAPACITY", 5: "KVQ_ERR_CUDA", 6: "KVQ_ERR_TIMEOUT"}
MAX_BATCH = 64

_lib = None


class KvqError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS.get(status, status)}: {message}")
        self.status = status


class _RecentCache(ctypes.Structure):
    _fields_ = [("packed", ctypes.c_void_p), ("scales", ctypes.c_void_p), ("recent", ctypes.c_void_p),
                ("capacity_blocks", ctypes.c_int64), ("rows_per_block", ctypes.c_int64), ("head_dim", ctypes.c_int32),
                ("bits", ctypes.c_int32), ("recent_blocks", ctypes.c_int32)]


class _Cache(ctypes.Structure):
    _fields_ = [("packed", ctypes.c_void_p), ("scales", ctypes.c_void_p), ("amax", ctypes.c_void_p),
                ("capacity_rows", ctypes.c_int64), ("rows_per_chunk", ctypes.c_int64),
                ("head_dim", ctypes.c_int32)]


def library_path() -> str:
    return _build.LIB


def load() -> ctypes.CDLL:
    """Build (if stale) and load libkvq.so. Raises if either step fails."""
    global _lib
    if _lib is not None:
        return _lib
    path = _build.build()
    lib = ctypes.CDLL(path)
    P, I64, I32, U64P = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.POINTER(ctypes.c_uint64)
    CP = ctypes.POINTER(_Cache)
    sig = {
        "kvq_quantize": [P, I64, I32, I32, P, P, P, P, P],
        "kvq_quantize_batch": [ctypes.POINTER(P), I32, I64, I32, I32, ctypes.POINTER(P), ctypes.POINTER(P),
                               ctypes.POINTER(P), ctypes.POINTER(P), P],
        "kvq_dequantize_batch": [ctypes.POINTER(P), ctypes.POINTER(P), ctypes.POINTER(P), I32, I64, I32,
                                 ctypes.POINTER(P), P],
        "kvq_quantize_dequantize": [P, I64, I32, I32, P, P, P, P, P, P],
        "kvq_dequantize": [P, P, P, I64, I32, P, P],
        "kvq_rtn_quantize": [P, I64, I32, I32, P, P, P],
        "kvq_rtn_dequantize": [P, P, I64, I32, I32, P, P],
        "kvq_rtn_quantize_batch": [ctypes.POINTER(P), I32, I64, I32, I32, ctypes.POINTER(P), ctypes.POINTER(P), P],
        "kvq_rtn_dequantize_batch": [ctypes.POINTER(P), ctypes.POINTER(P), I32, I64, I32, I32, ctypes.POINTER(P), P],
        "kvq_append": [CP, I64, P, I64, I32, P],
        "kvq_append_batch": [CP, ctypes.POINTER(I64), ctypes.POINTER(P), I32, I64, I32, P],
        "kvq_dequantize_cache": [CP, I64, I64, P, P],
        "kvq_dequantize_cache_batch": [CP, ctypes.POINTER(P), I32, I64, I64, P],
        "kvq_attention": [P, I32, I32, CP, CP, I64, ctypes.c_float, P, P, ctypes.c_uint64, P, P],
        "kvq_attention_workspace_bytes": [I32, I32, I64, U64P],
        "kvq_attention_launches": [I32, I32, I64, ctypes.POINTER(ctypes.c_int32)],
        "kvq_quantize_launches": [I32, I64, I32, I32, ctypes.POINTER(ctypes.c_int32)],
        "kvq_attention_noalloc": [P, I32, I32, CP, CP, I64, ctypes.c_float, P, P, P],
        "kvq_recent_append_batch": [ctypes.POINTER(_RecentCache), I32, I64, ctypes.POINTER(P), P],
        "kvq_recent_read_batch": [ctypes.POINTER(_RecentCache), I32, I64, ctypes.POINTER(P), P],
        "kvq_cache_bytes": [I32, I32, I64, I32, I64, U64P, U64P, U64P],
        "kvq_scales_to_blocked": [P, I64, I32, P, P],
        "kvq_scales_from_blocked": [P, I64, I32, P, P],
        "kvq_blocked_scale_bytes": [I64, I32, U64P],
    }
    for name, args in sig.items():
        fn = getattr(lib, name)
        fn.argtypes, fn.restype = args, ctypes.c_int
    lib.kvq_status_string.argtypes, lib.kvq_status_string.restype = [ctypes.c_int], ctypes.c_char_p
    lib.kvq_last_error.argtypes, lib.kvq_last_error.restype = [], ctypes.c_char_p
    lib.kvq_version.argtypes, lib.kvq_version.restype = [], ctypes.c_char_p
    lib.kvq_device_status.argtypes, lib.kvq_device_status.restype = [I32], ctypes.c_int
    lib.kvq_testing_set_fused_wait.argtypes = [ctypes.c_uint32, ctypes.c_uint64]
    lib.kvq_testing_set_fused_wait.restype = None
    lib.kvq_testing_set_attention_wait.argtypes, lib.kvq_testing_set_attention_wait.restype = [ctypes.c_uint64], None
    _lib = lib
    return lib


def _check(status: int):
    if status != 0:
        raise KvqError(status, load().kvq_last_error().decode())


def _rule(rule) -> int:
    return RULES[rule] if isinstance(rule, str) else int(rule)


def _stream(stream, device) -> int:
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return int(stream.cuda_stream) if hasattr(stream, "cuda_stream") else int(stream)


def _dev(t: torch.Tensor, what: str) -> int:
    if not t.is_cuda:
        raise ValueError(f"{what} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{what} must be contiguous")
    return t.data_ptr()


def kvq_status_string(status: int) -> str:
    return load().kvq_status_string(int(status)).decode()


def kvq_version() -> str:
    return load().kvq_version().decode()


def kvq_quantize_launches(n_tensors: int, n_elems: int, head_dim: int = 128, amax_given: bool = False) -> int:
    """Kernels one quantize or append call launches (host only)."""
    out = ctypes.c_int32()
    _check(load().kvq_quantize_launches(int(n_tensors), int(n_elems), int(head_dim), 1 if amax_given else 0,
                                        ctypes.byref(out)))
    return out.value


def kvq_device_status(clear: bool = True) -> None:
    """Raise KvqError(KVQ_ERR_TIMEOUT) if a bounded wait inside one of the library's
    kernels gave up on the current device since the last clearing call (the word is
    cleared when ``clear``). Synchronize the streams of interest first."""
    _check(load().kvq_device_status(1 if clear else 0))


def testing_set_attention_wait(wait_ns: int = 0) -> None:
    """Test hook (kvq_testing.h): the bound of the attention kernel's data-path waits on
    the current device (0 restores 1 s)."""
    load().kvq_testing_set_attention_wait(int(wait_ns))


def testing_set_fused_wait(extra_a_tiles: int, wait_ns: int = 0) -> None:
    """Test hook (kvq_testing.h): make the one-launch quantize of this thread wait for
    amax tiles that never come, with the given bound. (0, 0) restores normal operation."""
    load().kvq_testing_set_fused_wait(int(extra_a_tiles), int(wait_ns))


def kvq_quantize(x: torch.Tensor, head_dim: int | None = None, rule="static_6", amax_in: torch.Tensor | None = None,
                 amax_out: torch.Tensor | None = None, packed: torch.Tensor | None = None,
                 scales: torch.Tensor | None = None, stream=None):
    """Quantize a bf16 tensor. Returns (packed uint8[n/2], scales uint8[n/16], amax float32[1])."""
    if x.dtype != torch.bfloat16:
        raise TypeError("x must be bfloat16")
    n = x.numel()
    head_dim = int(head_dim or x.shape[-1])
    dev = x.device
    if packed is None:
        packed = torch.empty(n // 2, dtype=torch.uint8, device=dev)
    if scales is None:
        scales = torch.empty(n // BLOCK, dtype=torch.uint8, device=dev)
    if amax_out is None and amax_in is None:
        amax_out = torch.empty(1, dtype=torch.float32, device=dev)
    _check(load().kvq_quantize(_dev(x, "x"), n, head_dim, _rule(rule),
                               None if amax_in is None else _dev(amax_in, "amax_in"),
                               None if amax_out is None else _dev(amax_out, "amax_out"),
                               _dev(packed, "packed"), _dev(scales, "scales"), _stream(stream, dev)))
    return packed, scales, (amax_out if amax_out is not None else amax_in)


def kvq_dequantize(packed: torch.Tensor, scales: torch.Tensor, amax: torch.Tensor, head_dim: int,
                   y: torch.Tensor | None = None, shape=None, stream=None) -> torch.Tensor:
    """Dequantize to bf16. ``shape`` (default flat) applies when y is allocated here."""
    n = packed.numel() * 2
    dev = packed.device
    if y is None:
        y = torch.empty(shape if shape is not None else (n,), dtype=torch.bfloat16, device=dev)
    if y.dtype != torch.bfloat16 or y.numel() != n:
        raise ValueError("y must be bfloat16 with 2 * packed.numel() elements")
    _check(load().kvq_dequantize(_dev(packed, "packed"), _dev(scales, "scales"), _dev(amax, "amax"), n,
                                 int(head_dim), _dev(y, "y"), _stream(stream, dev)))
    return y


def _ptrs(ts, what):
    return (ctypes.c_void_p * len(ts))(*[_dev(t, what) for t in ts])


def kvq_quantize_batch(xs, head_dim: int | None = None, rule="static_6", amax_in=None, amax_out=None,
                       packed=None, scales=None, stream=None):
    """Quantize equally sized bf16 tensors in one set of launches, each with its own amax.
    Returns (packed list, scales list, amax list)."""
    n = len(xs)
    if n == 0:
        return [], [], []
    if any(x.dtype != torch.bfloat16 or x.numel() != xs[0].numel() for x in xs):
        raise ValueError("xs must be bfloat16 tensors of one size")
    numel = xs[0].numel()
    head_dim = int(head_dim or xs[0].shape[-1])
    dev = xs[0].device
    packed = packed or [torch.empty(numel // 2, dtype=torch.uint8, device=dev) for _ in xs]
    scales = scales or [torch.empty(numel // BLOCK, dtype=torch.uint8, device=dev) for _ in xs]
    if amax_in is None and amax_out is None:
        amax_out = [torch.empty(1, dtype=torch.float32, device=dev) for _ in xs]
    _check(load().kvq_quantize_batch(_ptrs(xs, "x"), n, numel, head_dim, _rule(rule),
                                     None if amax_in is None else _ptrs(amax_in, "amax_in"),
                                     None if amax_out is None else _ptrs(amax_out, "amax_out"),
                                     _ptrs(packed, "packed"), _ptrs(scales, "scales"), _stream(stream, dev)))
    return packed, scales, (amax_out if amax_out is not None else amax_in)


def kvq_dequantize_batch(packed, scales, amax, head_dim: int, ys=None, stream=None):
    """Dequantize equally sized tensors in one set of launches. Returns the bf16 list."""
    n = len(packed)
    if n == 0:
        return []
    numel = packed[0].numel() * 2
    dev = packed[0].device
    ys = ys or [torch.empty(numel, dtype=torch.bfloat16, device=dev) for _ in packed]
    _check(load().kvq_dequantize_batch(_ptrs(packed, "packed"), _ptrs(scales, "scales"), _ptrs(amax, "amax"), n,
                                       numel, int(head_dim), _ptrs(ys, "y"), _stream(stream, dev)))
    return ys


def kvq_quantize_dequantize(x: torch.Tensor, head_dim: int | None = None, rule="static_6",
                            amax_in: torch.Tensor | None = None, amax_out: torch.Tensor | None = None,
                            packed: torch.Tensor | None = None, scales: torch.Tensor | None = None,
                            y: torch.Tensor | None = None, codes: bool = True, stream=None):
    """Fused round trip: returns (y, packed, scales, amax); with codes=False only y (and
    amax) are written and packed/scales are None."""
    if x.dtype != torch.bfloat16:
        raise TypeError("x must be bfloat16")
    n = x.numel()
    head_dim = int(head_dim or x.shape[-1])
    dev = x.device
    if codes:
        packed = packed if packed is not None else torch.empty(n // 2, dtype=torch.uint8, device=dev)
        scales = scales if scales is not None else torch.empty(n // BLOCK, dtype=torch.uint8, device=dev)
    else:
        packed = scales = None
    if y is None:
        y = torch.empty_like(x)
    if amax_out is None and amax_in is None:
        amax_out = torch.empty(1, dtype=torch.float32, device=dev)
    _check(load().kvq_quantize_dequantize(_dev(x, "x"), n, head_dim, _rule(rule),
                                          None if amax_in is None else _dev(amax_in, "amax_in"),
                                          None if amax_out is None else _dev(amax_out, "amax_out"),
                                          None if packed is None else _dev(packed, "packed"),
                                          None if scales is None else _dev(scales, "scales"), _dev(y, "y"),
                                          _stream(stream, dev)))
    return y, packed, scales, (amax_out if amax_out is not None else amax_in)


def kvq_rtn_quantize(x: torch.Tensor, bits: int, head_dim: int | None = None, packed: torch.Tensor | None = None,
                     scales: torch.Tensor | None = None, stream=None):
    """RTN INT4 / INT2 of a bf16 tensor. Returns (packed uint8[n*bits/8], scales bf16[n/16])."""
    if x.dtype != torch.bfloat16:
        raise TypeError("x must be bfloat16")
    n, dev = x.numel(), x.device
    head_dim = int(head_dim or x.shape[-1])
    packed = packed if packed is not None else torch.empty(n * bits // 8, dtype=torch.uint8, device=dev)
    scales = scales if scales is not None else torch.empty(n // BLOCK, dtype=torch.bfloat16, device=dev)
    _check(load().kvq_rtn_quantize(_dev(x, "x"), n, head_dim, int(bits), _dev(packed, "packed"),
                                   _dev(scales, "scales"), _stream(stream, dev)))
    return packed, scales


def kvq_rtn_dequantize(packed: torch.Tensor, scales: torch.Tensor, bits: int, head_dim: int,
                       y: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    n = packed.numel() * 8 // int(bits)
    dev = packed.device
    y = y if y is not None else torch.empty(n, dtype=torch.bfloat16, device=dev)
    _check(load().kvq_rtn_dequantize(_dev(packed, "packed"), _dev(scales, "scales"), n, int(head_dim), int(bits),
                                     _dev(y, "y"), _stream(stream, dev)))
    return y


def kvq_rtn_quantize_batch(xs, bits: int, head_dim: int | None = None, packed=None, scales=None, stream=None):
    n = len(xs)
    if n == 0:
        return [], []
    numel, dev = xs[0].numel(), xs[0].device
    head_dim = int(head_dim or xs[0].shape[-1])
    packed = packed or [torch.empty(numel * bits // 8, dtype=torch.uint8, device=dev) for _ in xs]
    scales = scales or [torch.empty(numel // BLOCK, dtype=torch.bfloat16, device=dev) for _ in xs]
    _check(load().kvq_rtn_quantize_batch(_ptrs(xs, "x"), n, numel, head_dim, int(bits), _ptrs(packed, "packed"),
                                         _ptrs(scales, "scales"), _stream(stream, dev)))
    return packed, scales


def kvq_rtn_dequantize_batch(packed, scales, bits: int, head_dim: int, ys=None, stream=None):
    n = len(packed)
    if n == 0:
        return []
    numel, dev = packed[0].numel() * 8 // int(bits), packed[0].device
    ys = ys or [torch.empty(numel, dtype=torch.bfloat16, device=dev) for _ in packed]
    _check(load().kvq_rtn_dequantize_batch(_ptrs(packed, "packed"), _ptrs(scales, "scales"), n, numel,
                                           int(head_dim), int(bits), _ptrs(ys, "y"), _stream(stream, dev)))
    return ys


class KVCache:
    """A packed K or V cache of one layer (token-major rows of head_dim), backed by torch
    device tensors. ``rows_per_chunk`` is the rows of one append (tokens x heads)."""

    def __init__(self, capacity_rows: int, rows_per_chunk: int, head_dim: int, device="cuda",
                 packed: torch.Tensor | None = None, scales: torch.Tensor | None = None,
                 amax: torch.Tensor | None = None):
        self.capacity_rows, self.rows_per_chunk, self.head_dim = int(capacity_rows), int(rows_per_chunk), int(head_dim)
        n = self.capacity_rows * self.head_dim
        n_chunks = -(-self.capacity_rows // self.rows_per_chunk)
        self.packed = packed if packed is not None else torch.zeros(n // 2, dtype=torch.uint8, device=device)
        self.scales = scales if scales is not None else torch.zeros(n // BLOCK, dtype=torch.uint8, device=device)
        self.amax = amax if amax is not None else torch.zeros(n_chunks, dtype=torch.float32, device=device)
        self.device = self.packed.device

    def struct(self) -> _Cache:
        return _Cache(_dev(self.packed, "packed"), _dev(self.scales, "scales"), _dev(self.amax, "amax"),
                      self.capacity_rows, self.rows_per_chunk, self.head_dim)


def allocate_caches(layers: int, heads: int, capacity_tokens: int, head_dim: int, tokens_per_chunk: int,
                    device="cuda") -> list[KVCache]:
    """2 * layers caches (layer l: K = 2l, V = 2l + 1) carved from three device buffers
    sized by kvq_cache_bytes."""
    pb, sb, ab = kvq_cache_bytes(layers, heads, capacity_tokens, head_dim, tokens_per_chunk)
    t = 2 * layers
    packed = torch.zeros(pb, dtype=torch.uint8, device=device)
    scales = torch.zeros(sb, dtype=torch.uint8, device=device)
    amax = torch.zeros(ab // 4, dtype=torch.float32, device=device)
    rows = capacity_tokens * heads
    out = []
    for i in range(t):
        out.append(KVCache(rows, tokens_per_chunk * heads, head_dim, device,
                           packed[i * (pb // t):(i + 1) * (pb // t)], scales[i * (sb // t):(i + 1) * (sb // t)],
                           amax[i * (ab // 4 // t):(i + 1) * (ab // 4 // t)]))
    return out


def kvq_append(cache: KVCache, row_offset: int, x: torch.Tensor, rule="static_6", stream=None):
    """Quantize-on-write of x (bf16, n_rows x head_dim) at row_offset of the cache."""
    c = cache.struct()
    _check(load().kvq_append(ctypes.byref(c), int(row_offset), _dev(x, "x"), x.numel() // cache.head_dim,
                             _rule(rule), _stream(stream, cache.device)))


def kvq_append_batch(caches, row_offsets, xs, rule="static_6", stream=None):
    """One append per cache (same row count), in one set of launches."""
    n = len(caches)
    if not (len(row_offsets) == len(xs) == n):
        raise ValueError("caches, row_offsets and xs differ in length")
    if n == 0:
        return
    arr = (_Cache * n)(*[c.struct() for c in caches])
    offs = (ctypes.c_int64 * n)(*[int(o) for o in row_offsets])
    ptrs = (ctypes.c_void_p * n)(*[_dev(x, "x") for x in xs])
    n_rows = xs[0].numel() // caches[0].head_dim
    if any(x.numel() != xs[0].numel() for x in xs):
        raise ValueError("all appended tensors must have the same size")
    _check(load().kvq_append_batch(arr, offs, ptrs, n, n_rows, _rule(rule), _stream(stream, caches[0].device)))


def kvq_dequantize_cache(cache: KVCache, row_begin: int, row_end: int, y: torch.Tensor | None = None,
                         stream=None) -> torch.Tensor:
    if y is None:
        y = torch.empty((row_end - row_begin) * cache.head_dim, dtype=torch.bfloat16, device=cache.device)
    c = cache.struct()
    _check(load().kvq_dequantize_cache(ctypes.byref(c), int(row_begin), int(row_end), _dev(y, "y"),
                                       _stream(stream, cache.device)))
    return y


def kvq_dequantize_cache_batch(caches, row_begin: int, row_end: int, ys=None, stream=None):
    n = len(caches)
    if n == 0:
        return []
    if ys is None:
        ys = [torch.empty((row_end - row_begin) * c.head_dim, dtype=torch.bfloat16, device=c.device) for c in caches]
    arr = (_Cache * n)(*[c.struct() for c in caches])
    ptrs = (ctypes.c_void_p * n)(*[_dev(y, "y") for y in ys])
    _check(load().kvq_dequantize_cache_batch(arr, ptrs, n, int(row_begin), int(row_end),
                                             _stream(stream, caches[0].device)))
    return ys


def kvq_attention_workspace_bytes(n_queries: int, heads: int, n_keys: int) -> int:
    """Workspace bytes that let kvq_attention split the keys as it would on this device."""
    b = ctypes.c_uint64()
    _check(load().kvq_attention_workspace_bytes(int(n_queries), int(heads), int(n_keys), ctypes.byref(b)))
    return b.value


def kvq_attention_launches(n_queries: int, heads: int, n_keys: int) -> int:
    """Kernels one kvq_attention call of these sizes launches with the recommended workspace."""
    n = ctypes.c_int32()
    _check(load().kvq_attention_launches(int(n_queries), int(heads), int(n_keys), ctypes.byref(n)))
    return n.value


def kvq_attention(q: torch.Tensor, k_cache: KVCache, v_cache: KVCache, n_keys: int,
                  softmax_scale: float | None = None, out: torch.Tensor | None = None,
                  workspace: torch.Tensor | None = None, status: torch.Tensor | None = None,
                  stream=None, check: bool = False) -> torch.Tensor:
    """softmax(scale * Q K^T) V per head over cache tokens [0, n_keys), K and V read from
    their packed caches. q: bf16 [n_queries, heads, 128]; returns bf16 of q's shape.
    ``workspace`` (uint8, device) holds key-split partials; None allocates the size
    kvq_attention_workspace_bytes recommends, an empty tensor forbids splitting.
    ``status`` (int32, one element, device) is set to 1 if an on-chip wait timed out; the
    output is then invalid. The call stays asynchronous and does not read ``status``
    unless ``check`` is set: then it synchronizes the stream and raises
    KvqError(KVQ_ERR_TIMEOUT) when the status is nonzero."""
    if q.dim() != 3:
        raise ValueError("q must be [n_queries, heads, head_dim]")
    n_q, heads, d = q.shape
    if softmax_scale is None:
        softmax_scale = d ** -0.5
    if out is None:
        out = torch.empty_like(q)
    if workspace is None:
        workspace = torch.empty(kvq_attention_workspace_bytes(n_q, heads, n_keys), dtype=torch.uint8,
                                device=q.device)
    if status is None:
        status = torch.zeros(1, dtype=torch.int32, device=q.device)
    ws_ptr = _dev(workspace, "workspace") if workspace.numel() else None
    kc, vc = k_cache.struct(), v_cache.struct()
    _check(load().kvq_attention(_dev(q, "q"), n_q, heads, ctypes.byref(kc), ctypes.byref(vc), int(n_keys),
                                float(softmax_scale), _dev(out, "out"), ws_ptr, workspace.numel(),
                                _dev(status, "status"), _stream(stream, q.device)))
    if check:
        _check_status(status, stream, q.device)
    return out


def _check_status(status: torch.Tensor, stream, device):
    s = stream if stream is not None else torch.cuda.current_stream(device)
    if hasattr(s, "synchronize"):
        s.synchronize()
    else:
        torch.cuda.synchronize(device)
    if int(status.item()) != 0:
        raise KvqError(6, "an on-chip wait of the attention kernel gave up; the output is invalid")


def kvq_attention_noalloc(q: torch.Tensor, k_cache: KVCache, v_cache: KVCache, n_keys: int,
                          softmax_scale: float | None = None, out: torch.Tensor | None = None,
                          status: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """kvq_attention for callers that cannot allocate device memory for a workspace: the
    key-split partials use the library's built-in 32 MiB scratch (sizes needing more are
    rejected). ``out`` and ``status`` are still the caller's; pass them to allocate
    nothing here either."""
    if q.dim() != 3:
        raise ValueError("q must be [n_queries, heads, head_dim]")
    n_q, heads, d = q.shape
    if softmax_scale is None:
        softmax_scale = d ** -0.5
    if out is None:
        out = torch.empty_like(q)
    if status is None:
        status = torch.zeros(1, dtype=torch.int32, device=q.device)
    kc, vc = k_cache.struct(), v_cache.struct()
    _check(load().kvq_attention_noalloc(_dev(q, "q"), n_q, heads, ctypes.byref(kc), ctypes.byref(vc), int(n_keys),
                                        float(softmax_scale), _dev(out, "out"), _dev(status, "status"),
                                        _stream(stream, q.device)))
    return out


class RecentCache:
    """A K or V cache under the RECENT policy (RTN_INT4 RECENT2 of the Self-Forcing study):
    the newest ``recent_blocks`` frame-blocks in a bf16 ring, older blocks RTN-quantized
    (``bits``) in the prefix. A frame-block is ``rows_per_block`` rows of ``head_dim``."""

    def __init__(self, capacity_blocks: int, rows_per_block: int, head_dim: int = 128, bits: int = 4,
                 recent_blocks: int = 2, device="cuda"):
        self.capacity_blocks, self.rows_per_block, self.head_dim = int(capacity_blocks), int(rows_per_block), int(head_dim)
        self.bits, self.recent_blocks = int(bits), int(recent_blocks)
        elems = self.rows_per_block * self.head_dim
        self.packed = torch.zeros(self.capacity_blocks * elems * self.bits // 8, dtype=torch.uint8, device=device)
        self.scales = torch.zeros(self.capacity_blocks * elems // BLOCK, dtype=torch.bfloat16, device=device)
        self.recent = torch.zeros(self.recent_blocks * elems, dtype=torch.bfloat16, device=device)
        self.device = self.packed.device

    def struct(self) -> _RecentCache:
        return _RecentCache(_dev(self.packed, "packed"), _dev(self.scales, "scales"), _dev(self.recent, "recent"),
                            self.capacity_blocks, self.rows_per_block, self.head_dim, self.bits, self.recent_blocks)


def kvq_recent_append_batch(caches, block: int, xs, stream=None):
    """Quantize-on-write of frame-block ``block`` (bf16, rows_per_block x head_dim each)."""
    n = len(caches)
    if len(xs) != n:
        raise ValueError("caches and xs differ in length")
    if n == 0:
        return
    arr = (_RecentCache * n)(*[c.struct() for c in caches])
    ptrs = (ctypes.c_void_p * n)(*[_dev(x, "x") for x in xs])
    _check(load().kvq_recent_append_batch(arr, n, int(block), ptrs, _stream(stream, caches[0].device)))


def kvq_recent_read_batch(caches, n_blocks: int, ys=None, stream=None):
    """The first n_blocks frame-blocks of each cache as bf16 (prefix dequantized, tail copied)."""
    n = len(caches)
    if n == 0:
        return []
    if ys is None:
        ys = [torch.empty(n_blocks * c.rows_per_block * c.head_dim, dtype=torch.bfloat16, device=c.device)
              for c in caches]
    arr = (_RecentCache * n)(*[c.struct() for c in caches])
    ptrs = (ctypes.c_void_p * n)(*[_dev(y, "y") for y in ys])
    _check(load().kvq_recent_read_batch(arr, n, int(n_blocks), ptrs, _stream(stream, caches[0].device)))
    return ys


def kvq_cache_bytes(layers: int, heads: int, capacity_tokens: int, head_dim: int, tokens_per_chunk: int):
    """(packed bytes, scale bytes, amax bytes) of layers x {K, V}; host only."""
    p, s, a = ctypes.c_uint64(), ctypes.c_uint64(), ctypes.c_uint64()
    _check(load().kvq_cache_bytes(int(layers), int(heads), int(capacity_tokens), int(head_dim),
                                  int(tokens_per_chunk), ctypes.byref(p), ctypes.byref(s), ctypes.byref(a)))
    return p.value, s.value, a.value


def kvq_blocked_scale_bytes(rows: int, cols: int) -> int:
    b = ctypes.c_uint64()
    _check(load().kvq_blocked_scale_bytes(int(rows), int(cols), ctypes.byref(b)))
    return b.value


def kvq_scales_to_blocked(scales: torch.Tensor, rows: int, cols: int, blocked: torch.Tensor | None = None,
                          stream=None) -> torch.Tensor:
    """Row-major [rows, cols] one-byte scales -> the blocked 128 x 4 tile layout."""
    if blocked is None:
        blocked = torch.empty(kvq_blocked_scale_bytes(rows, cols), dtype=torch.uint8, device=scales.device)
    _check(load().kvq_scales_to_blocked(_dev(scales, "scales"), int(rows), int(cols), _dev(blocked, "blocked"),
                                        _stream(stream, scales.device)))
    return blocked


def kvq_scales_from_blocked(blocked: torch.Tensor, rows: int, cols: int, scales: torch.Tensor | None = None,
                            stream=None) -> torch.Tensor:
    if scales is None:
        scales = torch.empty(rows * cols, dtype=torch.uint8, device=blocked.device)
    _check(load().kvq_scales_from_blocked(_dev(blocked, "blocked"), int(rows), int(cols), _dev(scales, "scales"),
                                          _stream(stream, blocked.device)))
    return scales


def loaded_library() -> str | None:
    """Path of the loaded libkvq.so, or None before the first call."""
    return _build.LIB if _lib is not None else None


__all__ = [n for n in dir() if n.startswith("kvq_")] + ["KVCache", "allocate_caches", "KvqError", "load"]
