"""The C ABI without a GPU: the library builds for sm_100a, loads, exports every
function include/kvq.h declares, and rejects bad arguments on the host (before any CUDA
call). No kernel runs here."""
import ctypes
import os
import re
import subprocess

import pytest

import nvfp4_kv_cache_kvq_b200 as kvq

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADERS = [os.path.join(ROOT, "include", h) for h in sorted(os.listdir(os.path.join(ROOT, "include")))
           if h.endswith(".h")]


def declared_functions():
    names = set()
    for h in HEADERS:
        src = re.sub(r"/\*.*?\*/", "", open(h).read(), flags=re.S)
        names |= set(re.findall(r"^\s*(?:const\s+)?\w+\s*\**\s*(kvq_\w+)\s*\(", src, flags=re.M))
    return sorted(names)


def test_header_declares_the_boundary():
    names = declared_functions()
    for must in ("kvq_quantize", "kvq_dequantize", "kvq_quantize_batch", "kvq_dequantize_batch",
                 "kvq_quantize_dequantize", "kvq_append", "kvq_append_batch", "kvq_dequantize_cache",
                 "kvq_dequantize_cache_batch", "kvq_cache_bytes", "kvq_status_string", "kvq_last_error",
                 "kvq_device_status", "kvq_testing_set_fused_wait"):
        assert must in names


def test_library_exports_every_declared_symbol():
    lib = kvq.load()
    out = subprocess.check_output(["nm", "-D", "--defined-only", kvq.library_path()], text=True)
    exported = {line.split()[-1] for line in out.splitlines() if line.strip()}
    for name in declared_functions():
        assert name in exported, name
        assert getattr(lib, name) is not None


def test_library_is_built_for_sm100a_only():
    from nvfp4_kv_cache_kvq_b200 import build

    flags = " ".join(build.NVCC_FLAGS)
    assert "arch=compute_100a,code=sm_100a" in flags
    assert flags.count("-gencode") == 1 and "-fmad=false" in flags


def test_host_only_calls():
    assert kvq.kvq_status_string(0) == "KVQ_OK"
    assert kvq.kvq_status_string(4) == "KVQ_ERR_CAPACITY"
    assert kvq.kvq_status_string(6) == "KVQ_ERR_TIMEOUT"
    assert kvq.kvq_version().count(".") == 2
    p, s, a = kvq.kvq_cache_bytes(30, 12, 93600, 128, 1560)
    elems = 60 * 93600 * 12 * 128
    assert (p, s, a) == (elems // 2, elems // 16, 60 * 60 * 4)
    with pytest.raises(kvq.KvqError) as e:
        kvq.kvq_cache_bytes(30, 12, 93600, 100, 1560)
    assert e.value.status == 1


def test_quantize_launch_plan():
    """The launch plan kvq_quantize_launches reports (host only): a batch of two or more
    tensors of up to 2^21 blocks takes the slot fill and one amax + quantize launch; a
    single tensor, or a larger one, the fill, the amax pass and the quantize pass; a given
    amax, the quantize pass alone; each group of 64 tensors is planned on its own."""
    big = (1 << 21) * 16  # elements of the largest one-launch tensor
    assert kvq.kvq_quantize_launches(1, 4096 * 128) == 3
    assert kvq.kvq_quantize_launches(2, 4096 * 128) == 2
    assert kvq.kvq_quantize_launches(60, 1560 * 12 * 128) == 2
    assert kvq.kvq_quantize_launches(2, big) == 2
    assert kvq.kvq_quantize_launches(2, big + 128) == 3
    assert kvq.kvq_quantize_launches(64, 128) == 2
    assert kvq.kvq_quantize_launches(65, 128) == 2 + 3  # 64, then a single tensor
    assert kvq.kvq_quantize_launches(66, 128) == 2 + 2
    assert kvq.kvq_quantize_launches(130, 128, amax_given=True) == 3
    assert kvq.kvq_quantize_launches(0, 128) == 0
    assert kvq.kvq_quantize_launches(2, 0) == 0


def _fake(addr):
    return ctypes.c_void_p(addr)


def test_invalid_arguments_rejected_before_any_launch():
    lib = kvq.load()
    A = 1 << 40  # never dereferenced: every call below fails validation first
    # head_dim not a multiple of 16
    assert lib.kvq_quantize(_fake(A), 96, 12, 0, None, _fake(A), _fake(A), _fake(A), None) == 1
    # n_elems not a multiple of head_dim
    assert lib.kvq_quantize(_fake(A), 100, 16, 0, None, _fake(A), _fake(A), _fake(A), None) == 1
    # unknown rule
    assert lib.kvq_quantize(_fake(A), 128, 128, 7, None, _fake(A), _fake(A), _fake(A), None) == 1
    # no amax destination
    assert lib.kvq_quantize(_fake(A), 128, 128, 0, None, None, _fake(A), _fake(A), None) == 1
    assert b"both null" in lib.kvq_last_error()
    # misaligned x / packed / y
    assert lib.kvq_quantize(_fake(A + 16), 128, 128, 0, None, _fake(A), _fake(A), _fake(A), None) == 2
    assert lib.kvq_quantize(_fake(A), 128, 128, 0, None, _fake(A), _fake(A + 4), _fake(A), None) == 2
    assert lib.kvq_dequantize(_fake(A), _fake(A), _fake(A), 128, 128, _fake(A + 2), None) == 2
    # too large
    assert lib.kvq_quantize(_fake(A), (1 << 37), 128, 0, None, _fake(A), _fake(A), _fake(A), None) == 3
    # round trip: packed and scales must come together; y alignment
    assert lib.kvq_quantize_dequantize(_fake(A), 128, 128, 0, None, _fake(A), _fake(A), None, _fake(A), None) == 1
    assert lib.kvq_quantize_dequantize(_fake(A), 128, 128, 0, None, _fake(A), None, None, _fake(A + 16), None) == 2
    # batch: amax_in given for some tensors only
    xs = (ctypes.c_void_p * 2)(A, A)
    ain = (ctypes.c_void_p * 2)(A, None)
    outs = (ctypes.c_void_p * 2)(A, A)
    assert lib.kvq_quantize_batch(xs, 2, 128, 128, 0, ain, None, outs, outs, None) == 1
    assert lib.kvq_quantize_batch(xs, -1, 128, 128, 0, None, outs, outs, outs, None) == 1
    # computed amax: two tensors may not share one amax output (the slot is the launch's
    # synchronisation word)
    assert lib.kvq_quantize_batch(xs, 2, 128, 128, 2, None, outs, outs, outs, None) == 1
    assert b"share one amax output" in lib.kvq_last_error()


def _cache(capacity_rows=64, rows_per_chunk=16, head_dim=128, base=1 << 40):
    return kvq._Cache(base, base, base, capacity_rows, rows_per_chunk, head_dim)


def test_append_capacity_and_alignment_checked_on_host():
    lib = kvq.load()
    c = _cache()
    x = _fake(1 << 41)
    assert lib.kvq_append(ctypes.byref(c), 8, x, 16, 0, None) == 1      # not chunk aligned
    assert lib.kvq_append(ctypes.byref(c), 0, x, 17, 0, None) == 1      # more rows than a chunk
    assert lib.kvq_append(ctypes.byref(c), 64, x, 16, 0, None) == 4     # past capacity
    assert lib.kvq_append(ctypes.byref(c), 48, x, 16, 3, None) == 1     # bad rule
    assert lib.kvq_append(ctypes.byref(c), 48, _fake((1 << 41) + 8), 16, 0, None) == 2
    bad = _cache(head_dim=24)
    assert lib.kvq_append(ctypes.byref(bad), 0, x, 16, 0, None) == 1
    y = _fake(1 << 42)
    assert lib.kvq_dequantize_cache(ctypes.byref(c), 0, 65, y, None) == 4
    assert lib.kvq_dequantize_cache(ctypes.byref(c), 10, 5, y, None) == 1


def test_append_batch_rejects_a_shared_chunk_amax():
    lib = kvq.load()
    arr = (kvq._Cache * 2)(_cache(), _cache())
    offs = (ctypes.c_int64 * 2)(16, 16)  # same caches' buffers, same chunk: one amax slot
    ptrs = (ctypes.c_void_p * 2)(1 << 41, 1 << 42)
    assert lib.kvq_append_batch(arr, offs, ptrs, 2, 16, 2, None) == 1
    assert b"share one amax output" in lib.kvq_last_error()


def test_batch_rejects_mixed_head_dims():
    lib = kvq.load()
    arr = (kvq._Cache * 2)(_cache(), _cache(head_dim=64))
    offs = (ctypes.c_int64 * 2)(0, 0)
    ptrs = (ctypes.c_void_p * 2)(1 << 41, 1 << 41)
    assert lib.kvq_append_batch(arr, offs, ptrs, 2, 16, 0, None) == 1
    ys = (ctypes.c_void_p * 2)(1 << 42, 1 << 42)
    assert lib.kvq_dequantize_cache_batch(arr, ys, 2, 0, 16, None) == 1
