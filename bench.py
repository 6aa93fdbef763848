#!/usr/bin/env python3
"""Benchmark of the NVFP4 KV-cache path on B200: GB/s of algorithmic bytes moved, the
fraction of the HBM roofline, and tokens/s.

Default workload (``--workload rollout``): a self-forcing video rollout on a Wan-shaped
cache -- 30 layers x {K, V}, 12 heads, head_dim 128, 1560 tokens per frame, capacity 60
frames. One bench step is the whole 60-frame rollout: every frame appends 1560 new
tokens per layer through kvq_append_batch (quantize-on-write, rule mse) and then
dequantizes every layer's K and V prefix into one reused bf16 buffer through
kvq_dequantize_cache_batch. This one workload runs every stage of the path: cache
sizing, per-chunk amax, block scales, e2m1 packing, and dequantization.

Other workloads: ``single`` ([4096,128], static_6), ``layer`` (one layer's K and V of
[1,24,4680,128], mse), ``cache`` (30 layers x {K,V} of [1,24,32760,128]; quantize all,
dequantize per layer), ``sweep`` ([T,128], --tokens), ``roundtrip`` ([T,128] through the
fused quantize + dequantize kernel), ``rtn`` ([T,128] through the RTN INT4 / INT2 codec,
--bits).

Timing: each bench step is captured as CUDA graphs (one per segment: an append, a
layer loop of reads, ...), replayed with CUDA events between segments on the launching
stream; W warm-up steps, then K timed steps between a barrier and a device synchronize;
the step time is the max over ranks. Workloads smaller than L2 flush it (a 256 MB
write) between timed steps, outside the events.

``--impl reference`` times the CPU oracle (the plain C restatement of the method) on a
bounded sample of the same workload, on this host's cores.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "NVFP4 KV quant+dequant GB/s (bytes moved) and % of B200 HBM peak; tokens/s"
B_QUANT = 2.5625   # bf16 read + 0.5 B codes + 1/16 B scale written, per element
B_AMAX = 2.0       # bf16 read, per element
B_DEQUANT = 2.5625  # 0.5625 B read + bf16 written, per element
L2_BYTES = 126 * 2 ** 20


# The sources each traffic entry's counters depend on: an entry stays valid across edits of
# other kernels and of comments, not across code changes of its own kernel.
TRAFFIC_SOURCES = {
    "codec": ("nvfp4_kv_cache_kvq_b200/csrc/kvq.cu", "nvfp4_kv_cache_kvq_b200/csrc/kvq_device.cuh",
              "nvfp4_kv_cache_kvq_b200/csrc/kvq_common.h"),
    "attention": ("nvfp4_kv_cache_kvq_b200/csrc/kvq_attention.cu", "nvfp4_kv_cache_kvq_b200/csrc/kvq_device.cuh",
                  "nvfp4_kv_cache_kvq_b200/csrc/kvq_common.h"),
    "rtn": ("nvfp4_kv_cache_kvq_b200/csrc/kvq_rtn.cu", "nvfp4_kv_cache_kvq_b200/csrc/kvq_device.cuh",
            "nvfp4_kv_cache_kvq_b200/csrc/kvq_common.h"),
    "layout": ("nvfp4_kv_cache_kvq_b200/csrc/kvq_layout.cu", "nvfp4_kv_cache_kvq_b200/csrc/kvq_device.cuh",
               "nvfp4_kv_cache_kvq_b200/csrc/kvq_common.h"),
}


def kernel_source_sha256(group: str) -> str:
    """SHA-256 of the code of one group of kernel sources, comments and whitespace left out."""
    import hashlib
    import re

    h = hashlib.sha256()
    for rel in TRAFFIC_SOURCES[group]:
        with open(os.path.join(ROOT, rel)) as f:
            src = f.read()
        src = re.sub(r"/\*.*?\*/", " ", src, flags=re.S)  # block comments
        src = re.sub(r"//[^\n]*", " ", src)                # line comments (no source line has // in a string)
        h.update(" ".join(src.split()).encode())
    return h.hexdigest()


def _traffic_entry(kind: str):
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            k = json.load(f).get("kernels", {}).get(kind)
    except Exception:
        return None
    if k is None or k.get("sources") not in TRAFFIC_SOURCES:
        return None
    return k if k.get("source_sha256") == kernel_source_sha256(k["sources"]) else None


def measured_traffic(kind: str):
    """DRAM bytes per element of a kernel kind from the committed ncu summary
    (profiles/traffic.json), or None when the kernels changed since that capture."""
    k = _traffic_entry(kind)
    return None if k is None or "dram_bytes_per_elem" not in k else float(k["dram_bytes_per_elem"])


def measured_launch_traffic(kind: str, shape: str):
    """DRAM bytes of one launch of a kernel kind captured on exactly `shape`, or None."""
    k = _traffic_entry(kind)
    if k is None or k.get("shape") != shape:
        return None
    return float(k["dram_bytes_per_launch"])


REL_MSE_BOUND = 2e-2  # relative MSE bound on N(0,1)-like inputs the method is held to


def rel_mse(xs, ys, step: int = 1 << 26) -> float:
    """sum (y - x)^2 / sum x^2 in fp64 over pairs of bf16 tensors (the library's outputs
    against its inputs, read back after the timed region)."""
    num = den = 0.0  # summed over passes of `step` elements (fp64 temporaries of 8 step bytes)
    for x, y in zip(xs, ys):
        xr, yr = x.reshape(-1), y.reshape(-1)
        for i in range(0, xr.numel(), step):
            xf, yf = xr[i:i + step].double(), yr[i:i + step].double()
            num += float(((yf - xf) ** 2).sum())
            den += float((xf ** 2).sum())
    return num / den if den else 0.0


def footprint(packed: int, scales: int, amax: int, elems: int, transient_bf16: int = 0) -> dict:
    """Bytes of the quantized form against the bf16 it stands for."""
    q = packed + scales + amax
    return {"quantized_bytes": q, "bf16_bytes": 2 * elems, "ratio": 2 * elems / q if q else None,
            "transient_bf16_bytes": transient_bf16}


_CUDART = None


def memcpy2d_to_host(dst: int, dpitch: int, src: int, spitch: int, width: int, height: int, stream) -> None:
    """cudaMemcpy2DAsync device -> pinned host on `stream` (height rows of width bytes)."""
    global _CUDART
    if _CUDART is None:
        import ctypes
        import ctypes.util
        import glob

        paths = glob.glob(os.path.join(os.path.dirname(torch.__file__), "..", "nvidia", "cuda_runtime", "lib",
                                       "libcudart.so*")) + [ctypes.util.find_library("cudart")]
        for path in paths:
            if path:
                try:
                    _CUDART = ctypes.CDLL(path)
                    break
                except OSError:
                    pass
        if _CUDART is None:
            raise RuntimeError("libcudart not found")
        f = _CUDART.cudaMemcpy2DAsync
        f.argtypes = [ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_size_t,
                      ctypes.c_size_t, ctypes.c_int, ctypes.c_void_p]
        f.restype = ctypes.c_int
    rc = _CUDART.cudaMemcpy2DAsync(dst, dpitch, src, spitch, width, height, 2, stream.cuda_stream)
    if rc != 0:
        raise RuntimeError(f"cudaMemcpy2DAsync failed: {rc}")


def tensor_peak():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["bf16_tflops_sustained"]), "measured (MEASURED_PEAKS.json bf16_tflops_sustained)"
    except Exception:
        return 1400.0, "fallback (sustained dense bf16)"


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


# ---------------------------------------------------------------------------- clocks

class ClockSampler:
    """Samples SM clock, power and clock-event reasons through NVML every 100 ms."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
               0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
               0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}

    def __init__(self, device_index: int):
        self.samples, self.reasons, self.ok = [], set(), False
        self._stop = threading.Event()
        try:
            import pynvml

            pynvml.nvmlInit()
            p = torch.cuda.get_device_properties(device_index)
            bus = f"{p.pci_domain_id:08x}:{p.pci_bus_id:02x}:{p.pci_device_id:02x}.0"
            self.h = pynvml.nvmlDeviceGetHandleByPciBusId(bus.encode())
            self.nv = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # no NVML: report that, keep running
            self.err = str(e)

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                mhz = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                self.samples.append(mhz)
                for bit, name in self.REASONS.items():
                    if r & bit and bit != 0x1:
                        self.reasons.add(name)
            except Exception:
                pass
            self._stop.wait(0.1)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "note": f"NVML unavailable: {self.err}"}
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None, "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# ---------------------------------------------------------------------------- workloads

class Segment:
    """A unit of GPU work captured as one CUDA graph; `kind` groups segments for the
    per-kernel timing, `launches` counts the library's kernels it runs."""

    def __init__(self, kind, fn, launches, bytes_alg, h2d=None):
        self.kind, self.fn, self.launches, self.bytes_alg, self.h2d = kind, fn, launches, bytes_alg, h2d
        self.graph = None


class Rollout:
    name = "rollout"

    def __init__(self, args, rank):
        self.layers, self.heads, self.tokens, self.frames, self.D = 30, 12, 1560, 60, 128
        if args.small:
            self.layers, self.heads, self.tokens, self.frames = 2, 2, 120, 6
        if args.frames:  # fewer frames of the same shape (profiling)
            self.frames = args.frames
        self.rule = args.rule or "mse"
        self.rank = rank
        self.rpc = self.tokens * self.heads
        self.chunk_elems = self.rpc * self.D
        self.config = {
            "workload": f"rollout append+dequant: {self.layers} layers x {{K,V}}, {self.heads} heads, "
                        f"{self.tokens} tokens/frame x {self.frames} frames, head_dim {self.D}, Student-t(4), "
                        f"rule {self.rule}",
            "model": "Wan-shaped self-forcing KV cache (synthetic)",
            "global_batch": 1, "seq_len": self.tokens * self.frames, "parallelism": "replica per GPU",
            "l2": "inputs larger than L2 (per-step appends and the growing cache exceed 126 MB)",
        }

    def setup(self, kvq, inputs, dev):
        T = 2 * self.layers
        self.caches = kvq.allocate_caches(self.layers, self.heads, self.frames * self.tokens, self.D, self.tokens, dev)
        self.sizes = kvq.kvq_cache_bytes(self.layers, self.heads, self.frames * self.tokens, self.D, self.tokens)
        self.x = torch.empty((self.frames, T, self.chunk_elems), dtype=torch.bfloat16, device=dev)
        for f in range(self.frames):
            for t in range(T):
                self.x[f, t] = inputs.rollout_chunk(f + self.frames * self.rank, t, heads=self.heads,
                                                    tokens=self.tokens, device=dev).reshape(-1)
        cap = self.frames * self.chunk_elems
        self.yk = torch.empty(cap, dtype=torch.bfloat16, device=dev)
        self.yv = torch.empty(cap, dtype=torch.bfloat16, device=dev)
        self.kvq = kvq

    def segments(self):
        kvq, T, segs = self.kvq, 2 * self.layers, []
        for f in range(self.frames):
            xs = [self.x[f, t] for t in range(T)]

            def app(f=f, xs=xs):
                kvq.kvq_append_batch(self.caches, [f * self.rpc] * T, xs, self.rule)
            segs.append(Segment("append", app, kvq.kvq_quantize_launches(T, self.chunk_elems, self.D),
                                T * self.chunk_elems * (B_AMAX + B_QUANT), h2d=(self.x[f],)))
            rows = (f + 1) * self.rpc

            def deq(rows=rows):
                for l in range(self.layers):
                    kvq.kvq_dequantize_cache_batch(self.caches[2 * l:2 * l + 2], 0, rows,
                                                   [self.yk[:rows * self.D], self.yv[:rows * self.D]])
            segs.append(Segment("dequant", deq, self.layers, T * rows * self.D * B_DEQUANT))
        return segs

    def _bases(self):
        c0 = self.caches[0]
        # the three backing buffers of every cache (allocate_caches carves them contiguously)
        return [t._base if t._base is not None else t for t in (c0.packed, c0.scales, c0.amax)]

    def d2h(self):
        """Copied back at the end of the step: the chunk amax of every cache (the packed
        codes and scales go back frame by frame, see d2h_per_segment)."""
        return [self._bases()[2]]

    def d2h_per_segment(self, n_segs):
        """After frame f's append, its packed rows and scales are final in every cache:
        one 2D copy per buffer (a row per cache) sends them back while later frames run."""
        packed, scales, _ = self._bases()
        T = 2 * self.layers
        self.packed_h = torch.empty(packed.shape, dtype=packed.dtype, pin_memory=True)
        self.scales_h = torch.empty(scales.shape, dtype=scales.dtype, pin_memory=True)
        after = [None] * n_segs
        pb, sb = self.chunk_elems // 2, self.chunk_elems // 16  # bytes of one frame in one cache
        p_pitch, s_pitch = packed.numel() // T, scales.numel() // T

        def make(f):
            def go(stream):
                memcpy2d_to_host(self.packed_h.data_ptr() + f * pb, p_pitch, packed.data_ptr() + f * pb, p_pitch,
                                 pb, T, stream)
                memcpy2d_to_host(self.scales_h.data_ptr() + f * sb, s_pitch, scales.data_ptr() + f * sb, s_pitch,
                                 sb, T, stream)
            return go
        for f in range(self.frames):
            after[2 * f] = make(f)  # segment 2f is frame f's append
        return after, self.frames * T * (pb + sb)

    def tokens_per_step(self):
        return self.tokens * self.frames

    def rel_mse(self):
        """Layer 0's K and V over the whole rollout: the cache read back against the frames
        appended into it."""
        rows = self.frames * self.rpc
        ys = self.kvq.kvq_dequantize_cache_batch(self.caches[0:2], 0, rows)
        torch.cuda.synchronize()
        xs = [self.x[:, t].reshape(-1) for t in range(2)]
        return {"value": rel_mse(xs, ys), "bound": REL_MSE_BOUND,
                "what": "layer 0 K and V, all frames, fp64: sum (y - x)^2 / sum x^2"}

    def footprint(self):
        """The full cache after the rollout (every layer's K and V) against its bf16 size, and
        the bf16 buffers the per-layer reads reuse."""
        pb, sb, ab = self.sizes
        elems = 2 * self.layers * self.frames * self.chunk_elems
        return footprint(pb, sb, ab, elems, 2 * self.yk.numel() * 2)

    def extra_rates(self, kind_ms):
        """Appended tokens/s of the append kernels, and prefix tokens/s of the reads
        (every layer, K and V, all heads of a token counted once)."""
        prefix_tokens = self.tokens * self.frames * (self.frames + 1) // 2
        return {"append_tokens_per_s": self.tokens * self.frames / (kind_ms["append"] * 1e-3),
                "dequant_prefix_tokens_per_s": prefix_tokens / (kind_ms["dequant"] * 1e-3)}

    def oracle_sample(self, orc, inputs, budget_s):
        """Layer 0's K and V through the rollout until the time budget is spent."""
        caches = [orc.Cache(self.frames * self.rpc, self.rpc, self.D) for _ in range(2)]
        spent, nbytes, f = 0.0, 0.0, 0
        while f < self.frames and spent < budget_s:
            for t in range(2):
                xb = inputs.bits(inputs.rollout_chunk(f, t, heads=self.heads, tokens=self.tokens))
                t1 = time.perf_counter()
                caches[t].append(f * self.rpc, xb, self.rule)
                caches[t].dequantize(0, (f + 1) * self.rpc)
                spent += time.perf_counter() - t1
                nbytes += self.chunk_elems * (B_AMAX + B_QUANT) + (f + 1) * self.chunk_elems * B_DEQUANT
            f += 1
        return nbytes, spent, f"layer 0 K and V (2 of {2 * self.layers} tensors), frames 1..{f} of the rollout"


class Layer:
    name = "layer"

    def __init__(self, args, rank):
        self.heads, self.tokens, self.D = 24, 4680, 128
        if args.small:
            self.heads, self.tokens = 2, 300
        self.rule = args.rule or "mse"
        self.rank = rank
        self.n = self.heads * self.tokens * self.D
        self.config = {"workload": f"layer K and V quantize+dequantize: [1,{self.heads},{self.tokens},{self.D}] "
                                   f"Student-t(3) with 4 outlier channels/head x20, rule {self.rule}",
                       "model": "Wan-shaped attention layer (synthetic)", "global_batch": 1,
                       "seq_len": self.tokens, "parallelism": "replica per GPU",
                       "l2": "flushed between timed steps (256 MB write)"}
        self.flush = True

    def setup(self, kvq, inputs, dev):
        self.x = [inputs.layer_kv(2 * self.rank + kv, heads=self.heads, tokens=self.tokens, device=dev)
                  for kv in (0, 1)]
        self.allocate(kvq, dev)

    def allocate(self, kvq, dev):
        """Outputs for every input tensor in self.x."""
        m = len(self.x)
        self.p = [torch.empty(self.n // 2, dtype=torch.uint8, device=dev) for _ in range(m)]
        self.s = [torch.empty(self.n // 16, dtype=torch.uint8, device=dev) for _ in range(m)]
        self.a = [torch.empty(1, dtype=torch.float32, device=dev) for _ in range(m)]
        self.y = [torch.empty(self.n, dtype=torch.bfloat16, device=dev) for _ in range(m)]
        self.kvq = kvq

    def segments(self):
        kvq, m = self.kvq, len(self.x)

        def q():
            kvq.kvq_quantize_batch(self.x, self.D, self.rule, amax_out=self.a[:m], packed=self.p[:m],
                                   scales=self.s[:m])

        def d():
            kvq.kvq_dequantize_batch(self.p[:m], self.s[:m], self.a[:m], self.D, ys=self.y[:m])
        return [Segment("quantize", q, kvq.kvq_quantize_launches(m, self.n, self.D), m * self.n * (B_AMAX + B_QUANT),
                        h2d=tuple(self.x)),
                Segment("dequant", d, 1, m * self.n * B_DEQUANT)]

    def d2h(self):
        m = len(self.x)
        return self.p[:m] + self.s[:m] + self.a[:m] + self.y[:m]

    def rel_mse(self):
        m = len(self.x)
        return {"value": rel_mse(self.x, self.y[:m]), "bound": REL_MSE_BOUND,
                "what": f"{m} tensor(s), fp64: sum (y - x)^2 / sum x^2"}

    def footprint(self):
        m = len(self.x)
        return footprint(m * self.n // 2, m * self.n // 16, 4 * m, m * self.n)

    def tokens_per_step(self):
        return self.tokens

    def oracle_sample(self, orc, inputs, budget_s):
        nbytes, spent, done = 0.0, 0.0, 0
        for kv in (0, 1):
            xb = inputs.bits(inputs.layer_kv(kv, heads=self.heads, tokens=self.tokens))
            t1 = time.perf_counter()
            p, s, a = orc.quantize(xb, self.D, self.rule)
            orc.dequantize(p, s, a, self.D)
            spent += time.perf_counter() - t1
            nbytes += self.n * (B_AMAX + B_QUANT + B_DEQUANT)
            done += 1
            if spent > budget_s:
                break
        return nbytes, spent, f"{done} of 2 tensors (K, V), full size"


class Cache:
    name = "cache"

    def __init__(self, args, rank):
        self.layers, self.heads, self.tokens, self.D = 30, 24, 32760, 128
        if args.small:
            self.layers, self.heads, self.tokens = 2, 2, 2000
        self.rule = args.rule or "mse"
        self.rank = rank
        self.n = self.heads * self.tokens * self.D
        self.config = {"workload": f"full cache quantize then per-layer dequantize: {self.layers} layers x {{K,V}} x "
                                   f"[1,{self.heads},{self.tokens},{self.D}], N(0,1) + 1% tokens x10, rule {self.rule}",
                       "model": "Wan-shaped KV cache (synthetic)", "global_batch": 1, "seq_len": self.tokens,
                       "parallelism": "replica per GPU", "l2": "inputs larger than L2"}

    def setup(self, kvq, inputs, dev):
        T = 2 * self.layers
        self.x = torch.empty((T, self.n), dtype=torch.bfloat16, device=dev)
        for t in range(T):
            self.x[t] = inputs.cache_kv(t // 2 + self.layers * self.rank, t % 2, heads=self.heads,
                                        tokens=self.tokens, device=dev).reshape(-1)
        self.p = torch.empty((T, self.n // 2), dtype=torch.uint8, device=dev)
        self.s = torch.empty((T, self.n // 16), dtype=torch.uint8, device=dev)
        self.a = torch.empty((T, 1), dtype=torch.float32, device=dev)
        self.y = torch.empty((2, self.n), dtype=torch.bfloat16, device=dev)
        self.kvq = kvq

    def segments(self):
        kvq, T = self.kvq, 2 * self.layers

        def q():
            kvq.kvq_quantize_batch(list(self.x), self.D, self.rule, amax_out=list(self.a), packed=list(self.p),
                                   scales=list(self.s))

        def d():
            for l in range(self.layers):
                kvq.kvq_dequantize_batch([self.p[2 * l], self.p[2 * l + 1]], [self.s[2 * l], self.s[2 * l + 1]],
                                         [self.a[2 * l], self.a[2 * l + 1]], self.D, ys=[self.y[0], self.y[1]])
        return [Segment("quantize", q, kvq.kvq_quantize_launches(T, self.n, self.D), T * self.n * (B_AMAX + B_QUANT),
                        h2d=(self.x,)),
                Segment("dequant", d, self.layers, T * self.n * B_DEQUANT)]

    def d2h(self):
        return [self.p, self.s, self.a]

    def rel_mse(self):
        """The last layer's K and V (the pair the step dequantized last)."""
        T = 2 * self.layers
        return {"value": rel_mse([self.x[T - 2], self.x[T - 1]], [self.y[0], self.y[1]]), "bound": REL_MSE_BOUND,
                "what": f"layer {self.layers - 1} K and V, fp64: sum (y - x)^2 / sum x^2"}

    def footprint(self):
        T = 2 * self.layers
        return footprint(T * self.n // 2, T * self.n // 16, 4 * T, T * self.n, 2 * self.n * 2)

    def tokens_per_step(self):
        return self.tokens

    def oracle_sample(self, orc, inputs, budget_s):
        spent, nbytes, done = 0.0, 0.0, 0
        for t in range(2 * self.layers):
            xb = inputs.bits(inputs.cache_kv(t // 2, t % 2, heads=self.heads, tokens=self.tokens))
            t1 = time.perf_counter()
            p, s, a = orc.quantize(xb, self.D, self.rule)
            orc.dequantize(p, s, a, self.D)
            spent += time.perf_counter() - t1
            nbytes += self.n * (B_AMAX + B_QUANT + B_DEQUANT)
            done += 1
            if spent > budget_s:
                break
        return nbytes, spent, f"{done} of {2 * self.layers} tensors, full size"


class Single(Layer):
    name = "single"

    def __init__(self, args, rank):
        self.heads, self.tokens, self.D = 1, 4096, 128
        self.rule = args.rule or "static_6"
        self.rank = rank
        self.n = self.tokens * self.D
        self.config = {"workload": f"single K quantize+dequantize: [4096,128] N(0,1), rule {self.rule}",
                       "model": "one K tensor (synthetic)", "global_batch": 1, "seq_len": 4096,
                       "parallelism": "replica per GPU", "l2": "flushed between timed steps (256 MB write)"}
        self.flush = True

    def setup(self, kvq, inputs, dev):
        self.x = [inputs.normal((self.tokens, self.D), seed=self.rank, device=dev)]
        self.allocate(kvq, dev)

    def oracle_sample(self, orc, inputs, budget_s):
        t0, nbytes, reps = time.perf_counter(), 0.0, 0
        xb = inputs.bits(inputs.single_k())
        t0 = time.perf_counter()
        while reps < 2 or time.perf_counter() - t0 < min(budget_s, 5.0):
            p, s, a = orc.quantize(xb, self.D, self.rule)
            orc.dequantize(p, s, a, self.D)
            nbytes += self.n * (B_AMAX + B_QUANT + B_DEQUANT)
            reps += 1
        return nbytes, time.perf_counter() - t0, f"[4096,128] K, {reps} repetitions"


class Sweep(Layer):
    name = "sweep"

    def __init__(self, args, rank):
        self.heads, self.tokens, self.D = 1, args.tokens, 128
        self.rule = args.rule or "static_6"
        self.rank = rank
        self.n = self.tokens * self.D
        self.flush = self.n * 2 * 2 < L2_BYTES * 4
        self.config = {"workload": f"sweep quantize+dequantize: [{self.tokens},128] N(0,1), rule {self.rule}",
                       "model": "bandwidth sweep (synthetic)", "global_batch": 1, "seq_len": self.tokens,
                       "parallelism": "replica per GPU",
                       "l2": "flushed between timed steps (256 MB write)" if self.flush else "inputs larger than L2"}

    def setup(self, kvq, inputs, dev):
        self.x = [inputs.sweep(self.tokens, device=dev)]
        self.allocate(kvq, dev)

    def segments(self):
        """quantize (amax + codes), quantize again with amax_in (codes only: the same
        bytes, timed on their own), dequantize."""
        segs = Layer.segments(self)
        kvq = self.kvq

        def q_in():
            kvq.kvq_quantize_batch(self.x, self.D, self.rule, amax_in=self.a[:1], packed=self.p[:1], scales=self.s[:1])
        segs.insert(1, Segment("quantize_amax_in", q_in, 1, self.n * B_QUANT))
        return segs

    def oracle_sample(self, orc, inputs, budget_s):
        nbytes, reps = 0.0, 0
        m = min(self.tokens, 1 << 18)
        xb = inputs.bits(inputs.sweep(self.tokens)[:m])
        t0 = time.perf_counter()
        while reps < 1 or time.perf_counter() - t0 < min(budget_s, 5.0):
            p, s, a = orc.quantize(xb, self.D, self.rule)
            orc.dequantize(p, s, a, self.D)
            nbytes += m * self.D * (B_AMAX + B_QUANT + B_DEQUANT)
            reps += 1
        return nbytes, time.perf_counter() - t0, f"first {m} of {self.tokens} rows, {reps} repetitions"


class RoundTrip(Sweep):
    """The fused round trip (quantize + bf16 reconstruction in one pass) on [T, 128]."""
    name = "roundtrip"

    def __init__(self, args, rank):
        Sweep.__init__(self, args, rank)
        self.config["workload"] = (f"fused quantize+dequantize (one pass, codes and bf16 written): "
                                   f"[{self.tokens},128] N(0,1), rule {self.rule}")

    def segments(self):
        kvq = self.kvq

        def rt():
            kvq.kvq_quantize_dequantize(self.x[0], self.D, self.rule, amax_out=self.a[0], packed=self.p[0],
                                        scales=self.s[0], y=self.y[0])
        return [Segment("roundtrip", rt, kvq.kvq_quantize_launches(1, self.n, self.D), self.n * (B_AMAX + B_QUANT + 2.0),
                        h2d=(self.x[0],))]

    def d2h(self):
        return [self.p[0], self.s[0], self.a[0], self.y[0]]


class Rtn(Sweep):
    """The RTN integer codec (INT4 / INT2, bf16 scale per 16 values) on [T, 128]:
    quantize then dequantize."""
    name = "rtn"

    def __init__(self, args, rank):
        Sweep.__init__(self, args, rank)
        self.bits = args.bits
        self.config["workload"] = f"RTN INT{self.bits} quantize+dequantize: [{self.tokens},128] N(0,1)"

    def setup(self, kvq, inputs, dev):
        Sweep.setup(self, kvq, inputs, dev)
        self.p = [torch.empty(self.n * self.bits // 8, dtype=torch.uint8, device=dev)]
        self.s = [torch.empty(self.n // 16, dtype=torch.bfloat16, device=dev)]

    def segments(self):
        kvq, bq = self.kvq, 2.0 + self.bits / 8 + 2.0 / 16

        def q():
            kvq.kvq_rtn_quantize(self.x[0], self.bits, self.D, packed=self.p[0], scales=self.s[0])

        def d():
            kvq.kvq_rtn_dequantize(self.p[0], self.s[0], self.bits, self.D, y=self.y[0])
        return [Segment("rtn_quantize", q, 1, self.n * bq, h2d=(self.x[0],)),
                Segment("rtn_dequantize", d, 1, self.n * bq)]

    def d2h(self):
        return [self.p[0], self.s[0], self.y[0]]

    def footprint(self):  # packed codes and one bf16 scale per 16 values
        return footprint(self.n * self.bits // 8, self.n // 16 * 2, 0, self.n)

    def oracle_sample(self, orc, inputs, budget_s):
        m = min(self.tokens, 1 << 16)
        xb = inputs.bits(inputs.sweep(self.tokens)[:m])
        t0, nbytes, reps = time.perf_counter(), 0.0, 0
        while reps < 1 or time.perf_counter() - t0 < min(budget_s, 5.0):
            p, s = orc.rtn_quantize(xb, self.D, self.bits)
            orc.rtn_dequantize(p, s, self.D, self.bits)
            nbytes += 2 * m * self.D * (2.0 + self.bits / 8 + 2.0 / 16)
            reps += 1
        return nbytes, time.perf_counter() - t0, f"first {m} of {self.tokens} rows, {reps} repetitions"


class Layout:
    """The blocked scale layout (the 128 x 4 tiles block-scaled MMA operands read) of the
    scales of a [T, 128] tensor: scales [T, 8] (seeded e4m3 codes; the conversion is a
    permutation, so its cost does not depend on them) -> blocked and back."""
    name = "layout"

    def __init__(self, args, rank):
        self.tokens, self.cols, self.D = args.tokens, 8, 128
        self.rank = rank
        self.n = self.tokens * self.cols  # scale bytes
        self.flush = 3 * self.n < L2_BYTES * 4
        self.config = {"workload": f"blocked scale layout: the [{self.tokens},8] e4m3 scales of a "
                                   f"[{self.tokens},128] tensor, to blocked and back",
                       "model": "scale layout conversion (synthetic)", "global_batch": 1, "seq_len": self.tokens,
                       "parallelism": "replica per GPU",
                       "l2": "flushed between timed steps (256 MB write)" if self.flush else "inputs larger than L2"}

    def setup(self, kvq, inputs, dev):
        self.kvq = kvq
        self.s = inputs.scale_codes(self.tokens, self.cols, self.tokens, device=dev)
        self.nb = kvq.kvq_blocked_scale_bytes(self.tokens, self.cols)
        self.b = torch.empty(self.nb, dtype=torch.uint8, device=dev)
        self.back = torch.empty_like(self.s)

    def segments(self):
        kvq, byts = self.kvq, float(self.n + self.nb)

        def to():
            kvq.kvq_scales_to_blocked(self.s, self.tokens, self.cols, blocked=self.b)

        def back():
            kvq.kvq_scales_from_blocked(self.b, self.tokens, self.cols, scales=self.back)
        return [Segment("to_blocked", to, 1, byts, h2d=(self.s,)), Segment("from_blocked", back, 1, byts)]

    def d2h(self):
        return [self.back]

    def tokens_per_step(self):
        return self.tokens

    def oracle_sample(self, orc, inputs, budget_s):
        m = min(self.tokens, 1 << 18)
        sc = inputs.scale_codes(m, self.cols, self.tokens).numpy()
        t0, nbytes, reps = time.perf_counter(), 0.0, 0
        while reps < 1 or time.perf_counter() - t0 < min(budget_s, 5.0):
            b = orc.scales_to_blocked(sc, m, self.cols)
            orc.scales_from_blocked(b, m, self.cols)
            nbytes += 2.0 * (m * self.cols + orc.blocked_bytes(m, self.cols))
            reps += 1
        return nbytes, time.perf_counter() - t0, f"scales of the first {m} of {self.tokens} rows, {reps} repetitions"


class Recent:
    """The rollout under the RECENT2 cache policy of the Self-Forcing study (RTN_INT4
    RECENT2): every frame appends 1560 tokens per layer to 30 layers x {K, V} through
    kvq_recent_append_batch (the frame leaving the two-frame bf16 window is RTN
    INT4-quantized into the prefix) and reads every layer's whole cache back through
    kvq_recent_read_batch (prefix dequantized, bf16 tail copied)."""
    name = "recent"

    def __init__(self, args, rank):
        self.layers, self.heads, self.tokens, self.frames, self.D, self.R, self.bits = 30, 12, 1560, 60, 128, 2, 4
        if args.small:
            self.layers, self.heads, self.tokens, self.frames = 2, 2, 120, 6
        self.rank = rank
        self.rpc = self.tokens * self.heads
        self.chunk_elems = self.rpc * self.D
        self.config = {
            "workload": f"rollout with the RECENT2 policy (RTN INT4 prefix, newest {self.R} frames bf16): "
                        f"{self.layers} layers x {{K,V}}, {self.heads} heads, {self.tokens} tokens/frame x "
                        f"{self.frames} frames, head_dim {self.D}, Student-t(4)",
            "model": "Wan-shaped self-forcing KV cache (synthetic)", "global_batch": 1,
            "seq_len": self.tokens * self.frames, "parallelism": "replica per GPU",
            "l2": "inputs larger than L2 (per-step appends and the growing cache exceed 126 MB)",
        }

    def setup(self, kvq, inputs, dev):
        T = 2 * self.layers
        self.caches = [kvq.RecentCache(self.frames, self.rpc, self.D, self.bits, self.R, dev) for _ in range(T)]
        self.x = torch.empty((self.frames, T, self.chunk_elems), dtype=torch.bfloat16, device=dev)
        for f in range(self.frames):
            for t in range(T):
                self.x[f, t] = inputs.rollout_chunk(f + self.frames * self.rank, t, heads=self.heads,
                                                    tokens=self.tokens, device=dev).reshape(-1)
        cap = self.frames * self.chunk_elems
        self.yk = torch.empty(cap, dtype=torch.bfloat16, device=dev)
        self.yv = torch.empty(cap, dtype=torch.bfloat16, device=dev)
        self.kvq = kvq

    def segments(self):
        kvq, T, segs = self.kvq, 2 * self.layers, []
        bq = 2.0 + self.bits / 8 + 2.0 / 16  # RTN quantize: bf16 read, codes + bf16 scale written
        for f in range(self.frames):
            xs = [self.x[f, t] for t in range(T)]
            evict = f >= self.R

            def app(f=f, xs=xs):
                kvq.kvq_recent_append_batch(self.caches, f, xs)
            # RTN quantize of the evicted frame (once the window is full) + the bf16 copy
            segs.append(Segment("recent_append", app, math.ceil(T / kvq.MAX_BATCH) * (2 if evict else 1),
                                T * self.chunk_elems * ((bq if evict else 0.0) + 4.0), h2d=(self.x[f],)))
            n = f + 1
            r = min(self.R, n)
            prefix = n - r

            def rd(n=n):
                for l in range(self.layers):
                    kvq.kvq_recent_read_batch(self.caches[2 * l:2 * l + 2], n,
                                              [self.yk[:n * self.chunk_elems], self.yv[:n * self.chunk_elems]])
            segs.append(Segment("recent_read", rd, self.layers * ((1 if prefix else 0) + 1),
                                T * self.chunk_elems * (prefix * bq + r * 4.0)))
        return segs

    def d2h(self):
        return [self.caches[0].packed, self.caches[0].scales, self.caches[0].recent]

    def tokens_per_step(self):
        return self.tokens * self.frames

    def oracle_sample(self, orc, inputs, budget_s):
        """Layer 0's K and V through the rollout until the time budget is spent."""
        caches = [orc.RecentCache(self.rpc, self.D, self.bits, self.R) for _ in range(2)]
        bq = 2.0 + self.bits / 8 + 2.0 / 16
        spent, nbytes, f = 0.0, 0.0, 0
        while f < self.frames and spent < budget_s:
            for t in range(2):
                xb = inputs.bits(inputs.rollout_chunk(f, t, heads=self.heads, tokens=self.tokens))
                t1 = time.perf_counter()
                caches[t].append(xb)
                caches[t].read()
                spent += time.perf_counter() - t1
                n = f + 1
                r = min(self.R, n)
                nbytes += self.chunk_elems * ((bq if f >= self.R else 0.0) + 4.0 + (n - r) * bq + r * 4.0)
            f += 1
        return nbytes, spent, f"layer 0 K and V (2 of {2 * self.layers} tensors), frames 1..{f} of the rollout"


class Attention:
    """The rollout's attention at its last frame, reading the packed cache directly: for
    every layer, one frame of 1560 queries x 12 heads attends to that layer's 60-frame
    K/V cache (93,600 tokens) through kvq_attention. The same work done unfused --
    kvq_dequantize_cache_batch into bf16 buffers, then torch's scaled_dot_product_attention
    -- is timed beside it (``unfused``), with the bf16 bytes it has to hold."""
    name = "attention"

    def __init__(self, args, rank):
        self.layers, self.heads, self.tokens, self.frames, self.D = 30, 12, 1560, 60, 128
        if args.small:
            self.layers, self.heads, self.tokens, self.frames = 2, 2, 120, 6
        if args.layers:
            self.layers = args.layers
        self.rule = args.rule or "mse"
        self.rank = rank
        self.rpc = self.tokens * self.heads
        self.n_keys = self.tokens * self.frames
        self.flops_layer = 4.0 * self.tokens * self.n_keys * self.heads * self.D
        self.launch_shape = f"{self.tokens} queries x {self.heads} heads x {self.n_keys} keys"
        # packed K and V (codes + scales) read once, queries read, output written
        self.bytes_layer = 2 * self.n_keys * self.heads * self.D * 0.5625 + 2 * self.rpc * self.D * 2.0
        self.config = {
            "workload": f"fused NVFP4-cache attention: {self.layers} layers, {self.tokens} queries x {self.heads} "
                        f"heads over a {self.frames}-frame cache ({self.n_keys} tokens), head_dim {self.D}, "
                        f"Student-t(4) K/V appended with rule {self.rule}, N(0,1) queries",
            "model": "Wan-shaped self-forcing KV cache (synthetic)", "global_batch": 1, "seq_len": self.n_keys,
            "parallelism": "replica per GPU", "l2": "inputs larger than L2 (each layer's packed cache is 162 MB)",
        }

    def setup(self, kvq, inputs, dev):
        T = 2 * self.layers
        self.caches = kvq.allocate_caches(self.layers, self.heads, self.n_keys, self.D, self.tokens, dev)
        for f in range(self.frames):
            xs = [inputs.rollout_chunk(f + self.frames * self.rank, t, heads=self.heads, tokens=self.tokens,
                                       device=dev) for t in range(T)]
            kvq.kvq_append_batch(self.caches, [f * self.rpc] * T, xs, self.rule)
        self.q = torch.stack([inputs.queries(l + self.layers * self.rank, heads=self.heads, tokens=self.tokens,
                                             device=dev) for l in range(self.layers)])
        self.o = torch.empty_like(self.q)
        self.ws = torch.empty(kvq.kvq_attention_workspace_bytes(self.tokens, self.heads, self.n_keys),
                              dtype=torch.uint8, device=dev)
        self.status = torch.zeros(1, dtype=torch.int32, device=dev)
        self.kvq = kvq
        torch.cuda.synchronize()

    def segments(self):
        kvq = self.kvq

        def attn():
            for l in range(self.layers):
                kvq.kvq_attention(self.q[l], self.caches[2 * l], self.caches[2 * l + 1], self.n_keys,
                                  out=self.o[l], workspace=self.ws, status=self.status)
        # one or two attention launches per layer, each followed by a combine when it splits keys
        launches = self.layers * kvq.kvq_attention_launches(self.tokens, self.heads, self.n_keys)
        seg = Segment("attention", attn, launches, self.layers * self.bytes_layer, h2d=(self.q,))
        seg.flops = self.layers * self.flops_layer
        return [seg]

    def d2h(self):
        return [self.o]

    def tokens_per_step(self):
        return self.tokens * self.layers

    def check(self):
        if int(self.status.item()) != 0:
            raise RuntimeError("kvq_attention reported an on-chip wait timeout")

    def unfused(self, steps):
        """Dequantize each layer's K and V to bf16, then torch's SDPA, timed with events."""
        import torch.nn.functional as F

        kvq, H, D = self.kvq, self.heads, self.D
        rows = self.n_keys * H
        yk = torch.empty(rows * D, dtype=torch.bfloat16, device=self.q.device)
        yv = torch.empty_like(yk)

        def layer(l):
            kvq.kvq_dequantize_cache_batch(self.caches[2 * l:2 * l + 2], 0, rows, [yk, yv])
            k = yk.view(1, self.n_keys, H, D).transpose(1, 2)
            v = yv.view(1, self.n_keys, H, D).transpose(1, 2)
            q = self.q[l].unsqueeze(0).transpose(1, 2)
            return F.scaled_dot_product_attention(q, k, v).transpose(1, 2)

        for l in range(self.layers):
            out = layer(l)
        torch.cuda.synchronize()
        diff = float((out[0].float() - self.o[self.layers - 1].float()).abs().max())
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ms = []
        for _ in range(steps):
            e0.record()
            for l in range(self.layers):
                layer(l)
            e1.record()
            torch.cuda.synchronize()
            ms.append(e0.elapsed_time(e1))
        return {"ms_per_step": sum(ms) / len(ms), "what": "kvq_dequantize_cache_batch + torch SDPA per layer",
                "transient_bf16_bytes": 2 * rows * D * 2, "max_abs_diff_vs_fused": diff}

    def oracle_sample(self, orc, inputs, budget_s):
        """Layer 0: the oracle appends the cache (untimed), then dequantizes K and V and
        computes query rows' attention in fp64 (timed), doubling the rows per batch until
        the time budget is spent. The bytes credited are the whole dequantization of K and
        V (read 0.5625, write 2 B per element, as the timed region does it in full) plus
        the layer's algorithmic attention bytes scaled by the share of query rows done."""
        caches = [orc.Cache(self.frames * self.rpc, self.rpc, self.D) for _ in range(2)]
        for f in range(self.frames):
            for t in range(2):
                caches[t].append(f * self.rpc, inputs.bits(inputs.rollout_chunk(f, t, heads=self.heads,
                                                                                tokens=self.tokens)), self.rule)
        qb = inputs.bits(inputs.queries(0, heads=self.heads, tokens=self.tokens)).reshape(self.tokens, -1)
        t0 = time.perf_counter()
        kb, vb = caches[0].dequantize(0, self.n_keys * self.heads), caches[1].dequantize(0, self.n_keys * self.heads)
        rows, m = 0, 4
        while rows < self.tokens:
            m = min(m, self.tokens - rows)
            orc.attention(qb[rows:rows + m].reshape(-1), kb, vb, m, self.n_keys, self.heads, self.D, self.D ** -0.5)
            rows += m
            if time.perf_counter() - t0 >= budget_s:
                break
            m *= 2
        dt = time.perf_counter() - t0
        deq_bytes = 2 * self.n_keys * self.heads * self.D * B_DEQUANT
        return (deq_bytes + self.bytes_layer * rows / self.tokens, dt,
                f"layer 0: K and V dequantized in full, then {rows} of {self.tokens} query rows")


WORKLOADS = {c.name: c for c in (Rollout, Layer, Cache, Single, Sweep, RoundTrip, Rtn, Attention, Recent, Layout)}


# ---------------------------------------------------------------------------- runner

def dist_setup(backend: str = "nccl"):
    """One process per GPU (torchrun's RANK / LOCAL_RANK / WORLD_SIZE). The process
    group only carries the barrier around the timed region and the max of the step
    times: the workload itself has no exchange (every rank is an independent replica)."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if backend == "nccl":
        torch.cuda.set_device(local if world > 1 else 0)
    if world > 1:
        import datetime

        import torch.distributed as dist

        kw = {"device_id": torch.device("cuda", local)} if backend == "nccl" else {}
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120), **kw)
    return world, rank, local


def _reduce_device():
    import torch.distributed as dist

    return torch.device("cuda", torch.cuda.current_device()) if dist.get_backend() == "nccl" else torch.device("cpu")


def barrier(world):
    if world > 1:
        import torch.distributed as dist

        dist.barrier()


def max_over_ranks(v: float, world: int) -> float:
    if world == 1:
        return v
    import torch.distributed as dist

    t = torch.tensor([v], dtype=torch.float64, device=_reduce_device())
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_gbs(world: int, bytes_per_rank_step: float, max_ms_per_step: float) -> float:
    """Whole-job GB/s: every rank processed bytes_per_rank_step per step; the step time
    is the slowest rank's."""
    return world * bytes_per_rank_step / (max_ms_per_step * 1e-3) / 1e9


def cpu_baseline(wl, budget_s):
    import oracle
    from nvfp4_kv_cache_kvq_b200 import inputs

    oracle.build()
    nbytes, dt, sample = wl.oracle_sample(oracle, inputs, budget_s)
    return {"value": nbytes / dt / 1e9, "unit": "GB/s", "cores": oracle.default_threads(), "kind": "oracle",
            "sample": sample, "seconds": round(dt, 3)}


def run_reference(args, wl, world, rank):
    """The CPU oracle, as it stands, on a bounded sample of the workload per step."""
    if rank != 0:
        return
    import oracle
    from nvfp4_kv_cache_kvq_b200 import inputs

    oracle.build()
    per_step = []
    sample = ""
    for i in range(args.warmup + args.steps):
        nbytes, dt, sample = wl.oracle_sample(oracle, inputs, args.ref_step_s)
        if i >= args.warmup:
            per_step.append((nbytes, dt))
    tot_b = sum(b for b, _ in per_step)
    tot_t = sum(t for _, t in per_step)
    value = tot_b / tot_t / 1e9
    line = {"metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": 1e3 * tot_t / len(per_step), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic", "config": wl.config,
            "impl": "reference",
            "cpu_baseline": {"value": value, "unit": "GB/s", "cores": oracle.default_threads(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def capture(segs, use_graphs):
    if not use_graphs:
        return
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        for seg in segs:  # one eager run first: builds the library and settles its queries
            seg.fn()
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    for seg in segs:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            seg.fn()
        seg.graph = g
    torch.cuda.synchronize()


def run_step(segs, events, e2e=None):
    """One bench step on the current stream; events[i] is recorded before segment i and
    events[-1] after the last. With e2e, every segment's inputs are copied in from pinned
    host memory on a copy stream that starts with the step and runs ahead of the compute
    (each segment waits only for its own inputs), and the step's outputs are copied back
    at the end, all inside the timed interval."""
    main = torch.cuda.current_stream()
    events[0].record()
    ready = [None] * len(segs)
    if e2e is not None:
        cs = e2e["stream"]
        cs.wait_event(events[0])
        with torch.cuda.stream(cs):
            for i, seg in enumerate(segs):
                if seg.h2d is None:
                    continue
                for dst, src in zip(seg.h2d, e2e["h2d"][i]):
                    dst.copy_(src, non_blocking=True)
                ready[i] = torch.cuda.Event()
                ready[i].record(cs)
    per_seg = e2e.get("d2h_after") if e2e is not None else None
    for i, seg in enumerate(segs):
        if i > 0:
            events[i].record()
        if ready[i] is not None:
            main.wait_event(ready[i])
        if seg.graph is not None:
            seg.graph.replay()
        else:
            seg.fn()
        if per_seg is not None and per_seg[i] is not None:
            # this segment's final outputs go back on their own stream while the next
            # segments compute
            done = torch.cuda.Event()
            done.record(main)
            e2e["d2h_stream"].wait_event(done)
            per_seg[i](e2e["d2h_stream"])
    if e2e is not None:
        with torch.cuda.stream(e2e["d2h_stream"]):
            e2e["d2h_stream"].wait_stream(main)
            for dst, src in zip(e2e["d2h_dst"], e2e["d2h_src"]):
                dst.copy_(src, non_blocking=True)
        main.wait_stream(e2e["d2h_stream"])
    events[-1].record()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default="rollout")
    ap.add_argument("--rule", choices=("static_6", "static_4", "mse"), default=None)
    ap.add_argument("--tokens", type=int, default=1 << 24, help="rows of the sweep workload")
    ap.add_argument("--bits", type=int, choices=(2, 4), default=4, help="bits of the rtn workload")
    ap.add_argument("--small", action="store_true", help="a reduced shape of the workload (for tests)")
    ap.add_argument("--layers", type=int, default=None, help="layers of the attention workload (profiling)")
    ap.add_argument("--frames", type=int, default=None, help="frames of the rollout workload (profiling)")
    ap.add_argument("--no-graphs", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget-s", type=float, default=15.0)
    ap.add_argument("--ref-step-s", type=float, default=8.0)
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "ours":
        print("warning: fewer than 3 warm-up steps", file=sys.stderr)

    if args.impl == "reference":
        # the oracle runs on rank 0's host cores; other ranks exit without work
        world, rank = int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0"))
        run_reference(args, WORKLOADS[args.workload](args, rank), world, rank)
        return
    world, rank, _ = dist_setup()
    wl = WORKLOADS[args.workload](args, rank)

    import nvfp4_kv_cache_kvq_b200 as kvq
    from nvfp4_kv_cache_kvq_b200 import inputs

    kvq.load()
    dev = torch.device("cuda", torch.cuda.current_device())
    wl.setup(kvq, inputs, dev)
    segs = wl.segments()
    capture(segs, not args.no_graphs)
    flush_buf = torch.empty(256 * 2 ** 20, dtype=torch.uint8, device=dev) if getattr(wl, "flush", False) else None

    events = [torch.cuda.Event(enable_timing=True) for _ in range(len(segs) + 1)]
    for _ in range(args.warmup):
        run_step(segs, events)
    torch.cuda.synchronize()

    kinds = sorted({s.kind for s in segs})
    kind_ms = {k: 0.0 for k in kinds}
    step_ms = []
    barrier(world)
    torch.cuda.synchronize()
    sampler = ClockSampler(dev.index)
    with sampler:
        for _ in range(args.steps):
            if flush_buf is not None:
                flush_buf.zero_()
            run_step(segs, events)
            torch.cuda.synchronize()
            for i, seg in enumerate(segs):
                kind_ms[seg.kind] += events[i].elapsed_time(events[i + 1])
            step_ms.append(events[0].elapsed_time(events[-1]))
    torch.cuda.synchronize()
    barrier(world)
    mean_ms = max_over_ranks(sum(step_ms) / len(step_ms), world)

    bytes_step = sum(s.bytes_alg for s in segs)
    value = aggregate_gbs(world, bytes_step, mean_ms)
    peak, peak_src = peaks()
    kind_bytes = {k: sum(s.bytes_alg for s in segs if s.kind == k) for k in kinds}
    kind_launch = {k: sum(s.launches for s in segs if s.kind == k) for k in kinds}
    dom = max(kinds, key=lambda k: kind_ms[k])
    dom_ms = kind_ms[dom] / args.steps
    achieved = kind_bytes[dom] / (dom_ms * 1e-3) / 1e9
    dom_flops = sum(getattr(s, "flops", 0.0) for s in segs if s.kind == dom)
    if dom_flops:
        # a contraction: against the measured dense bf16 GEMM peak (sustained: the kernel
        # runs back to back for the whole timed region)
        tflops = dom_flops / (dom_ms * 1e-3) / 1e12
        tpeak, tsrc = tensor_peak()
        roofline = {"bound": "tensor", "kernel": dom, "achieved": tflops, "peak": tpeak, "unit": "TFLOP/s",
                    "frac": tflops / tpeak, "peak_source": tsrc,
                    "traffic": measured_launch_traffic(dom, getattr(wl, "launch_shape", "")),
                    "flops_per_step": dom_flops, "launches_per_step": kind_launch[dom],
                    "ms_per_step": dom_ms, "hbm_GB_s": achieved}
    else:
        per_elem = {"dequant": B_DEQUANT, "append": B_AMAX + B_QUANT, "quantize": B_AMAX + B_QUANT,
                    "quantize_amax_in": B_QUANT,
                    "roundtrip": B_AMAX + B_QUANT + 2.0, "rtn_quantize": 2.0 + args.bits / 8 + 2.0 / 16,
                    "rtn_dequantize": 2.0 + args.bits / 8 + 2.0 / 16,
                    "to_blocked": 2.0, "from_blocked": 2.0}.get(dom)  # layout: per scale byte
        # the RTN codecs' traffic depends on the bit width: their entries carry it; a
        # quantize with its own amax runs in one launch (plus the slot fill) up to 2^21
        # blocks per tensor, else as two passes
        key = dom
        if dom.startswith("rtn_"):
            key = f"{dom}_int{args.bits}"
        elif dom == "quantize" and kind_launch[dom] == 2 * sum(1 for s_ in segs if s_.kind == dom):
            key = "quantize_one_launch"
        tb = measured_traffic(key) if per_elem else None
        elems_per_launch = kind_bytes[dom] / per_elem / kind_launch[dom] if per_elem else None
        roofline = {"bound": "hbm", "kernel": dom, "achieved": achieved, "peak": peak, "unit": "GB/s",
                    "frac": achieved / peak, "peak_source": f"{peak_src} (MEASURED_PEAKS.json hbm_gbs)",
                    "traffic": None if tb is None else tb * elems_per_launch,
                    "alg_bytes_per_launch": kind_bytes[dom] / kind_launch[dom],
                    "launches_per_step": kind_launch[dom], "ms_per_step": dom_ms}
    per_kind = {k: {"ms_per_step": kind_ms[k] / args.steps,
                    "GB_s": kind_bytes[k] / (kind_ms[k] / args.steps * 1e-3) / 1e9 if kind_ms[k] else None,
                    "launches_per_step": kind_launch[k]} for k in kinds}

    line = {"metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": mean_ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f32", "data": "synthetic", "config": wl.config,
            "hbm_frac": value / world / peak, "tokens_per_s": world * wl.tokens_per_step() / (mean_ms * 1e-3),
            "roofline": roofline, "kernels": per_kind, "gpu_launches": sum(s.launches for s in segs) * args.steps,
            "clocks": sampler.summary(), "graphs": not args.no_graphs}

    if hasattr(wl, "extra_rates"):
        line.update(wl.extra_rates({k: kind_ms[k] / args.steps for k in kinds}))
    if hasattr(wl, "rel_mse"):
        line["rel_mse"] = wl.rel_mse()
    if hasattr(wl, "footprint"):
        line["footprint"] = wl.footprint()
    if hasattr(wl, "check"):
        wl.check()
    if hasattr(wl, "unfused"):
        line["unfused"] = wl.unfused(args.steps)
    if not args.no_e2e:
        line["e2e"] = run_e2e(args, wl, segs, bytes_step, world)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(wl, args.cpu_budget_s)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist

        for s in segs:
            s.graph = None
        dist.destroy_process_group()


def run_e2e(args, wl, segs, bytes_step, world):
    """The same steps with every segment's inputs copied in from pinned host memory (on a
    copy stream overlapping the compute) and the step's outputs copied back, inside the
    timed region."""
    h2d, h2d_bytes = [], 0
    for seg in segs:
        if seg.h2d is None:
            h2d.append(None)
            continue
        srcs = []
        for t in seg.h2d:
            host = torch.empty(t.shape, dtype=t.dtype, pin_memory=True)
            host.copy_(t)
            srcs.append(host)
            h2d_bytes += t.numel() * t.element_size()
        h2d.append(srcs)
    d2h_src = wl.d2h()
    d2h_dst = [torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in d2h_src]
    d2h_bytes = sum(t.numel() * t.element_size() for t in d2h_src)
    e2e = {"h2d": h2d, "d2h_src": d2h_src, "d2h_dst": d2h_dst, "stream": torch.cuda.Stream(),
           "d2h_stream": torch.cuda.Stream()}
    if hasattr(wl, "d2h_per_segment"):
        # outputs that are final after a segment are copied back right after it
        after, more_bytes = wl.d2h_per_segment(len(segs))
        e2e["d2h_after"] = after
        d2h_bytes += more_bytes
    events = [torch.cuda.Event(enable_timing=True) for _ in range(len(segs) + 1)]
    run_step(segs, events, e2e)
    torch.cuda.synchronize()
    steps = max(1, min(args.steps, 3))
    ms = []
    for _ in range(steps):
        run_step(segs, events, e2e)
        torch.cuda.synchronize()
        ms.append(events[0].elapsed_time(events[-1]))
    mean_ms = max_over_ranks(sum(ms) / len(ms), world)
    return {"value": aggregate_gbs(world, bytes_step, mean_ms), "unit": "GB/s", "ms_per_step": mean_ms,
            "h2d_bytes_per_step": h2d_bytes, "d2h_bytes_per_step": d2h_bytes, "steps": steps}


if __name__ == "__main__":
    main()
