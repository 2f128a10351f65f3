#!/usr/bin/env python
"""Benchmark of the paged-KV-cache attention hot path on B200.

One step = one pass of the hot path over one batch of synthetic inputs that
already sit in HBM.  The default workload is the Llama-2-7B-shaped MHA decode
step: the cache append of the 64 new K/V rows (random slot mapping) followed
by decode attention of 64 sequences (32/32 heads, head_dim 128, bf16, page
16, contexts uniform in [512, 4096]), split-KV partitions and their merge
included.  ``--workload`` selects the other workloads (GQA decode, long
context bf16/INT8, chunked prefill with a shared prefix, tiny fp32 decode), and
``kv_cache_write_full`` the cache append at bandwidth scale (every cached token of
the Llama-2-7B-shaped batch written through a random slot permutation).

Prints ONE JSON line (rank 0).  ``value`` is whole-job throughput: algorithmic
bytes (decode, cache append) or flops (prefill) of all ranks' steps divided by the device
time of the timed steps (CUDA events on the launching stream, max over ranks).
``e2e`` repeats the measurement through the public API from pinned host
buffers, with the per-step host->device copies of the step's inputs and the
device->host copy of its output inside the timed region.  ``roofline`` is for
the dominant kernel (the decode or prefill call), timed with CUDA events
around that call inside the timed steps.  ``cpu_baseline`` times the fp64
oracle on the host cores (rank 0, N = 1 only).

``--impl reference`` times the fp64 CPU oracle (the reference arm here) on a
bounded sample of the same workload and prints the same line shape.

Multi-GPU (torchrun): each rank runs an independent replica of the workload
(the decode and prefill paths shard over sequences with no exchange step), so
scaling is weak and there is no data-path collective; ranks only meet at the
barriers around the timed region and in the max/sum of the timings.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "paged decode attention HBM GB/s (% of 8 TB/s), tokens/s; prefill TFLOP/s"
L2_BYTES = 126 * 2 ** 20
FLUSH_BYTES = 256 * 2 ** 20        # written between timed steps (outside the events) to empty L2
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

# DRAM traffic per launch of the dominant kernel from an ncu capture
# (dram__bytes_read.sum + dram__bytes_write.sum), keyed by workload, with the
# hash of the kernel sources it was taken on; reported only while they match.
TRAFFIC = {
    # decode_mma_kernel: 1204.69 MB per launch at batch 32 (the capture-size case, same partitions
    # as the bench launch), 1.0034 x its algorithmic bytes; scaled to batch 64 (2346.50 MB)
    "llama2_7b_mha_decode": {"bytes": 2354590000, "kernel_sha": "d9cce3085c6f990f"},
    # decode_mma_kernel (GQA, 8 query heads per KV head): 693.36 MB per launch at batch 64 (same
    # partitions as the bench launch), 1.0067 x its algorithmic bytes; scaled to batch 128 (1396.15 MB)
    "llama2_70b_gqa_decode": {"bytes": 1405480000, "kernel_sha": "d9cce3085c6f990f"},
    # decode_mma_kernel (int8 codes + fp16 scales): the bench launch itself, 1098.45 MB (1.0072 x its
    # algorithmic bytes, split partials included)
    "long_ctx_split_kv_int8": {"bytes": 1098450000, "kernel_sha": "d9cce3085c6f990f"},
    # prefill_tc_kernel: 54.76 MB read + 3.63 MB written per launch, full workload, cold L2
    "chunked_prefill_shared_prefix": {"bytes": 58394112, "kernel_sha": "19f948ac33e1e7cf"},
    # kv_scatter_kernel: 1120.62 MB per launch at a source batch of 16 (35 476 rows; ~43 MB of the
    # writes still in L2 at the end), scaled to the 143 153-row launch by rows
    "kv_cache_write_full": {"bytes": 4521850000, "kernel_sha": "d05e87c4610560d2"},
}
KERNEL_SOURCES = {
    "decode": ["paged_kv_cache_380_b200/csrc/decode.cu", "paged_kv_cache_380_b200/csrc/pkv_ptx.cuh",
               "paged_kv_cache_380_b200/csrc/pkv_common.cuh", "paged_kv_cache_380_b200/csrc/api.cu"],
    "prefill": ["paged_kv_cache_380_b200/csrc/prefill.cu", "paged_kv_cache_380_b200/csrc/pkv_ptx.cuh",
                "paged_kv_cache_380_b200/csrc/pkv_common.cuh"],
    "scatter": ["paged_kv_cache_380_b200/csrc/scatter.cu", "paged_kv_cache_380_b200/csrc/pkv_common.cuh"],
}


def kernel_sha(kind: str) -> str:
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES[kind]:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ---- distributed plumbing (host logic; tested on CPU with gloo) ------------------

def dist_env():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def aggregate(elapsed_ms: float, units: float, work: float, group=None):
    """Max of the timed region over ranks and sums of units/work over ranks."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return elapsed_ms, units, work
    dev = "cuda" if dist.get_backend(group) == "nccl" else "cpu"
    t = torch.tensor([elapsed_ms], dtype=torch.float64, device=dev)
    s = torch.tensor([units, work], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    dist.all_reduce(s, op=dist.ReduceOp.SUM, group=group)
    return float(t.item()), float(s[0].item()), float(s[1].item())


def barrier():
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        dist.barrier()


# ---- clock sampling during the timed region (NVML reads only) ---------------------

REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
           0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
           0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}


class ClockSampler:
    """Polls the SM clock and clock-event reasons of this process's GPU every
    few milliseconds in a background thread (read-only NVML queries)."""

    def __init__(self, torch_device: int, period_s: float = 0.005):
        self.samples = []
        self.period = period_s
        self._stop = threading.Event()
        self._thread = None
        self.max_mhz = None
        self.handle = None
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            props = torch.cuda.get_device_properties(torch_device)
            bus = "%08X:%02X:%02X.0" % (props.pci_domain_id, props.pci_bus_id, props.pci_device_id)
            self.handle = pynvml.nvmlDeviceGetHandleByPciBusId(bus)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.handle, pynvml.NVML_CLOCK_SM)
            self._nvml = pynvml
        except Exception as e:  # pragma: no cover - reported, not fatal
            self.error = repr(e)

    def _run(self):
        nv = self._nvml
        while not self._stop.is_set():
            try:
                mhz = nv.nvmlDeviceGetClockInfo(self.handle, nv.NVML_CLOCK_SM)
                try:
                    reasons = nv.nvmlDeviceGetCurrentClocksEventReasons(self.handle)
                except AttributeError:
                    reasons = nv.nvmlDeviceGetCurrentClocksThrottleReasons(self.handle)
                self.samples.append((time.perf_counter(), mhz, reasons))
            except Exception:
                pass
            time.sleep(self.period)

    def start(self):
        if self.handle is not None:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
            time.sleep(0.05)

    def stop(self):
        self._stop.set()
        if self._thread:
            self._thread.join()

    def summary(self, t0: float, t1: float):
        if self.handle is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "error": getattr(self, "error", "")}
        inside = [s for s in self.samples if t0 <= s[0] <= t1]
        if not inside and self.samples:        # very short region: nearest samples around it
            inside = sorted(self.samples, key=lambda s: min(abs(s[0] - t0), abs(s[0] - t1)))[:3]
        mask = 0
        for s in inside:
            mask |= s[2]
        names = [n for bit, n in REASONS.items() if mask & bit and n != "gpu_idle"]
        return {"sm_mhz": statistics.median(s[1] for s in inside) if inside else None,
                "sm_max_mhz": self.max_mhz, "reasons": names, "samples": len(inside)}


# ---- workloads -----------------------------------------------------------------------

class L2Flush:
    """Empties L2 between timed steps: writes a buffer larger than L2, then reads
    another one, so that L2 ends up holding clean lines of the second buffer and
    the next step neither hits on its own data nor pays for write-backs of the
    flush."""

    def __init__(self):
        import torch
        self.wr = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device="cuda")
        # float32, so that the sum reads it in place (an int32 sum would first widen a copy)
        self.rd = torch.zeros(FLUSH_BYTES // 4, dtype=torch.float32, device="cuda")

    def __call__(self):
        self.wr.fill_(1)
        self.sink = self.rd.sum()

def dev(a, tag):
    import numpy as np
    import torch
    a = np.ascontiguousarray(a)
    if tag == "bf16":
        return torch.from_numpy(a.view(np.int16)).cuda().view(torch.bfloat16)
    if tag == "f16":
        return torch.from_numpy(a.view(np.float16)).cuda()
    return torch.from_numpy(a).cuda()


class DecodeStep:
    """Cache append of the new rows (when the workload has them) + decode."""

    kind = "decode"

    def __init__(self, case, int8: bool = False, window: int = 0):
        import numpy as np
        import torch
        from paged_kv_cache_380_b200 import ops
        self.case, self.int8, self.window = case, int8, window
        tag = case.dtype
        B, Hq, D = case.q.shape
        P, ps, Hkv, _ = case.k_pages.shape
        self.q = dev(case.q, tag)
        self.bt = dev(case.block_tables, "i32")
        self.cl = dev(case.context_lens, "i32")
        self.out = torch.empty_like(self.q)
        if int8:
            kb, vb = dev(case.k_pages, tag), dev(case.v_pages, tag)
            self.kp = torch.empty(kb.shape, dtype=torch.int8, device="cuda")
            self.vp = torch.empty_like(self.kp)
            self.ks = torch.empty(kb.shape[:3], dtype=torch.float16, device="cuda")
            self.vs = torch.empty_like(self.ks)
            ident = torch.arange(P * ps, dtype=torch.int64, device="cuda")
            ops.kv_cache_write_quant(kb.view(P * ps, Hkv, D), vb.view(P * ps, Hkv, D), ident, self.kp, self.vp,
                                     self.ks, self.vs)
            del kb, vb
            torch.cuda.synchronize()
            elem, scale_bytes = 1, 2
        else:
            self.kp, self.vp = dev(case.k_pages, tag), dev(case.v_pages, tag)
            self.ks = self.vs = None
            elem, scale_bytes = (4 if tag == "f32" else 2), 0
        self.has_new = case.k_new is not None and not int8
        if self.has_new:
            self.k_new, self.v_new = dev(case.k_new, tag), dev(case.v_new, tag)
            self.slots = dev(case.slot_mapping, "i64")
        kvdt = torch.int8 if int8 else self.kp.dtype
        self.splits, self.split_tokens = ops.decode_plan(B, Hq, Hkv, D, ps, case.max_pages_per_seq, kvdt)
        need = ops.decode_workspace_size(B, Hq, Hkv, D, ps, case.max_pages_per_seq, kvdt)
        self.ws = torch.empty(max(need, 1), dtype=torch.uint8, device="cuda")
        qelem = 4 if tag == "f32" else 2
        ctx = case.context_lens.astype(np.int64)
        if window > 0:
            ctx = np.minimum(ctx, window)                      # keys a windowed query reads
        pages = int(np.sum((ctx + ps - 1) // ps))
        # algorithmic bytes: every attended K/V element read once (+ its scale for INT8),
        # q read, out written, block-table entries and context lengths read
        self.decode_bytes = (int(ctx.sum()) * Hkv * (2 * D * elem + 2 * scale_bytes)
                             + 2 * B * Hq * D * qelem + pages * 4 + B * 4)
        self.write_bytes = 0
        if self.has_new:
            T = case.k_new.shape[0]
            self.write_bytes = 2 * 2 * T * Hkv * D * elem + T * 8
        self.work = self.decode_bytes + self.write_bytes       # bytes per step
        self.units = B                                          # sequences advanced one token
        self.launches = (1 if self.has_new else 0) + 1 + (1 if self.splits > 1 else 0)
        self.flush = L2Flush()

    def before_step(self):
        self.flush()                               # outside the per-step events

    def run(self, ev=None):
        from paged_kv_cache_380_b200 import ops
        if self.has_new:
            ops.kv_cache_write(self.k_new, self.v_new, self.slots, self.kp, self.vp)
        if ev is not None:
            ev[0].record()
        ops.paged_attention_decode(self.q, self.kp, self.vp, self.bt, self.cl, self.case.scale, self.out,
                                   k_scales=self.ks, v_scales=self.vs, workspace=self.ws, window=self.window)
        if ev is not None:
            ev[1].record()

    def host_io(self):
        """Pinned host copies of the per-step inputs and the output buffer."""
        import torch
        ins = [self.q, self.bt, self.cl] + ([self.k_new, self.v_new, self.slots] if self.has_new else [])
        hosts = [t.cpu().pin_memory() for t in ins]
        out_h = torch.empty(self.out.shape, dtype=self.out.dtype).pin_memory()
        return list(zip(hosts, ins)), out_h

    def config(self):
        c = self.case
        B, Hq, D = c.q.shape
        return {"workload": c.name + ("_int8" if self.int8 else ""), "batch": B, "num_q_heads": Hq,
                "num_kv_heads": c.num_kv_heads, "head_dim": D, "page_size": c.page_size,
                "kv_dtype": "i8" if self.int8 else c.dtype, "mean_context": float(c.context_lens.mean()),
                "window": self.window,
                "num_pages": c.num_pages, "splits": self.splits, "split_tokens": self.split_tokens,
                "new_tokens_written": int(c.k_new.shape[0]) if self.has_new else 0,
                "l2": ("L2 flushed between steps (256 MiB write + 256 MiB read outside the events); %.2f GB read "
                       "per step"
                       % (self.work / 1e9))}


class PrefillStep:
    """Cache append of the chunk's K/V, then causal chunked prefill."""

    kind = "prefill"

    def __init__(self, case, window: int = 0):
        import numpy as np
        import torch
        self.case, self.window = case, window
        tag = case.dtype
        self.q = dev(case.q, tag)
        self.kp, self.vp = dev(case.k_pages, tag), dev(case.v_pages, tag)
        self.bt, self.qs, self.cl = dev(case.block_tables, "i32"), dev(case.q_start, "i32"), dev(case.context_lens, "i32")
        self.k_new, self.v_new, self.slots = dev(case.k_new, tag), dev(case.v_new, tag), dev(case.slot_mapping, "i64")
        self.out = torch.empty_like(self.q)
        self.max_q = int(np.max(np.diff(case.q_start)))
        Hq, D = case.num_q_heads, case.head_dim
        n = np.diff(case.q_start).astype(np.int64)
        ctx = case.context_lens.astype(np.int64)
        # keys attended per (row, head): ctx - n + r + 1 for r < n (at most `window` of them)
        if window > 0:
            keys = int(sum(np.minimum(np.arange(c - k + 1, c + 1), window).sum() for k, c in zip(n, ctx)))
        else:
            keys = int(np.sum(n * (ctx - n) + n * (n + 1) // 2))
        self.work = 4.0 * D * Hq * keys           # flops per step (QK^T and PV, 2 flops per MAC)
        self.units = int(n.sum())                  # query rows processed
        self.launches = 2
        self.flush = L2Flush()

    def before_step(self):
        self.flush()                               # outside the per-step events

    def run(self, ev=None):
        from paged_kv_cache_380_b200 import ops
        ops.kv_cache_write(self.k_new, self.v_new, self.slots, self.kp, self.vp)
        if ev is not None:
            ev[0].record()
        ops.paged_attention_prefill(self.q, self.kp, self.vp, self.bt, self.qs, self.cl, True, self.case.scale,
                                    self.out, max_q_len=self.max_q, window=self.window)
        if ev is not None:
            ev[1].record()

    def host_io(self):
        import torch
        ins = [self.q, self.bt, self.qs, self.cl, self.k_new, self.v_new, self.slots]
        hosts = [t.cpu().pin_memory() for t in ins]
        out_h = torch.empty(self.out.shape, dtype=self.out.dtype).pin_memory()
        return list(zip(hosts, ins)), out_h

    def config(self):
        c = self.case
        return {"workload": c.name, "num_seqs": c.batch, "chunk": int(np.diff(c.q_start)[0]) if c.batch else 0,
                "context": int(c.context_lens[0]), "shared_prefix_pages": c.meta.get("shared_pages"),
                "num_q_heads": c.num_q_heads, "num_kv_heads": c.num_kv_heads, "head_dim": c.head_dim,
                "page_size": c.page_size, "window": self.window,
                "l2": "L2 flushed between steps (256 MiB write + 256 MiB read outside the events)"}


class ScatterStep:
    """The cache append at bandwidth scale: every cached token of the Llama-2-7B-shaped
    decode batch (143 k rows of K and of V, 8 KiB each) is written again through a
    seeded random permutation of the pool's slots.  Bytes per step: the K and V rows
    read and written, plus the slots."""

    kind = "scatter"

    def __init__(self, case):
        import torch
        from paged_kv_cache_380_b200 import workloads as W
        self.case = case
        tag = case.dtype
        self.src, self.dst = W.full_cache_scatter(case)
        self.kp, self.vp = dev(case.k_pages, tag), dev(case.v_pages, tag)
        Hkv, D = case.num_kv_heads, case.head_dim
        src = torch.as_tensor(self.src, device="cuda")
        self.k_new = self.kp.view(-1, Hkv, D)[src].clone()     # the cached rows, in sequence order
        self.v_new = self.vp.view(-1, Hkv, D)[src].clone()
        self.slots = dev(self.dst, "i64")
        T = int(self.src.shape[0])
        self.row_bytes = Hkv * D * self.kp.element_size()
        self.work = 2 * 2 * T * self.row_bytes + 8 * T          # bytes per step
        self.units = T
        self.launches = 1
        # the step's result read back end to end: the first destination row of K
        self.out = self.kp.view(-1, Hkv * D)[int(self.dst[0])]
        self.flush = L2Flush()

    def before_step(self):
        self.flush()                               # outside the per-step events

    def run(self, ev=None):
        from paged_kv_cache_380_b200 import ops
        if ev is not None:
            ev[0].record()
        ops.kv_cache_write(self.k_new, self.v_new, self.slots, self.kp, self.vp)
        if ev is not None:
            ev[1].record()

    def host_io(self):
        import torch
        ins = [self.k_new, self.v_new, self.slots]
        hosts = [t.cpu().pin_memory() for t in ins]
        out_h = torch.empty(self.out.shape, dtype=self.out.dtype).pin_memory()
        return list(zip(hosts, ins)), out_h

    def config(self):
        c = self.case
        return {"workload": "kv_cache_write_full", "rows": self.units, "row_bytes": self.row_bytes,
                "num_kv_heads": c.num_kv_heads, "head_dim": c.head_dim, "page_size": c.page_size,
                "slots": "seeded random permutation of the pool's slots",
                "l2": "L2 flushed between steps (256 MiB write + 256 MiB read outside the events); 4.7 GB moved "
                      "per step"}


def make_step(name: str, batch: int = 0, graph: bool = False, window: int = 0):
    from paged_kv_cache_380_b200 import workloads as W
    if name == "kv_cache_write_full":
        return ScatterStep(W.llama2_7b_mha_decode(**({"batch": batch} if batch else {})))
    if name == "long_ctx_split_kv_int8":
        step = DecodeStep(W.long_ctx_split_kv(**({"batch": batch} if batch else {})), int8=True, window=window)
        return GraphStep(step) if graph else step
    case = W.WORKLOADS[name](**({"batch": batch} if batch else {}))
    if graph and case.kind == "decode":
        return GraphStep(DecodeStep(case, window=window))
    return PrefillStep(case, window) if case.kind == "prefill" else DecodeStep(case, window=window)


class GraphStep:
    """A DecodeStep replayed as one captured CUDA graph (append + decode + merge)."""

    def __init__(self, inner):
        from paged_kv_cache_380_b200.graph import DecodeStepGraph
        self.inner = inner
        for k in ("case", "kind", "int8", "window", "has_new", "decode_bytes", "write_bytes", "work", "units",
                  "launches", "splits", "split_tokens"):
            setattr(self, k, getattr(inner, k))
        kw = dict(k_scales=inner.ks, v_scales=inner.vs)
        if inner.has_new:
            kw.update(k_new=inner.k_new, v_new=inner.v_new, slot_mapping=inner.slots)
        self.g = DecodeStepGraph(inner.q, inner.kp, inner.vp, inner.bt, inner.cl, inner.case.scale, out=inner.out, **kw)
        self.out = inner.out

    def before_step(self):
        self.inner.before_step()

    def run(self, ev=None):
        if ev is not None:
            ev[0].record()
        self.g.replay()
        if ev is not None:
            ev[1].record()

    def host_io(self):
        return self.inner.host_io()

    def config(self):
        return dict(self.inner.config(), cuda_graph=True)


# ---- the GPU arm ------------------------------------------------------------------------

def time_steps(step, K, events=True):
    """Run K steps, per-step CUDA events; returns (total_ms, dominant_ms_list)."""
    import torch
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    dom = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    for i in range(K):
        if hasattr(step, "before_step"):
            step.before_step()
        starts[i].record()
        step.run(dom[i] if events else None)
        ends[i].record()
    torch.cuda.synchronize()
    total = sum(s.elapsed_time(e) for s, e in zip(starts, ends))
    dom_ms = [a.elapsed_time(b) for a, b in dom] if events else []
    return total, dom_ms


def time_e2e(step, K):
    import torch
    pairs, out_h = step.host_io()
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    h2d = sum(h.numel() * h.element_size() for h, _ in pairs)
    d2h = out_h.numel() * out_h.element_size()
    for i in range(K):
        if hasattr(step, "before_step"):
            step.before_step()
        starts[i].record()
        for h, d in pairs:
            d.copy_(h, non_blocking=True)
        step.run()
        out_h.copy_(step.out, non_blocking=True)
        ends[i].record()
    torch.cuda.synchronize()
    return sum(s.elapsed_time(e) for s, e in zip(starts, ends)), h2d, d2h


def _oracle_scatter_rate(case, src, dst, n_rows):
    """The oracle's row copy of the first n_rows of a full-cache scatter into host copies of
    the pools; returns (bytes per second, seconds)."""
    import oracle
    Hkv, D = case.num_kv_heads, case.head_dim
    k_rows = case.k_pages.reshape(-1, Hkv, D)[src[:n_rows]]
    v_rows = case.v_pages.reshape(-1, Hkv, D)[src[:n_rows]]
    kp, vp = case.k_pages.copy(), case.v_pages.copy()
    t0 = time.perf_counter()
    oracle.kv_cache_write(k_rows, v_rows, dst[:n_rows], kp, vp)
    dt = max(time.perf_counter() - t0, 1e-9)
    return (2 * 2 * n_rows * k_rows[0].nbytes + 8 * n_rows) / dt, dt


def cpu_baseline(step, budget_s: float = 20.0):
    """The fp64 oracle on the host cores over a bounded sample of the workload."""
    import oracle
    c = step.case
    threads = oracle.max_threads()
    if step.kind == "scatter":
        T = step.units
        rate, dt = _oracle_scatter_rate(c, step.src, step.dst, T)
        return {"value": rate / 1e9, "unit": "GB/s", "cores": threads, "kind": "oracle",
                "sample": f"all {T} rows of the scatter, one row copy each ({dt:.2f} s)", "seconds": dt}
    if step.kind == "decode":
        B, Hq = c.batch, c.num_q_heads
        eff = c.context_lens.astype(np.int64)
        if getattr(step, "window", 0) > 0:
            eff = np.minimum(eff, step.window)                 # keys a windowed query reads
        _oracle_inputs(step)                                   # untimed: the appended / quantised pool

        def sample(n_threads, seconds):
            # the first S sequences (all heads), S grown until the run takes about `seconds`
            oracle.set_threads(n_threads)
            try:
                S, dt, reps = 1, 0.0, 1
                for _ in range(5):
                    t0 = time.perf_counter()
                    _run_oracle_decode(step, np.arange(S * Hq))
                    dt = time.perf_counter() - t0
                    if dt >= seconds / 2 or S == B:
                        break
                    S = int(min(B, max(S + 1, S * seconds / max(dt, 1e-3))))
                if dt < seconds / 2:                           # the whole batch is quicker: repeat it
                    reps = int(min(20, np.ceil(seconds / 2 / max(dt, 1e-3))))
                    t0 = time.perf_counter()
                    for _ in range(reps):
                        _run_oracle_decode(step, np.arange(S * Hq))
                    dt = time.perf_counter() - t0
            finally:
                oracle.set_threads(threads)
            work = reps * step.decode_bytes * eff[:S].sum() / eff.sum()
            return work / dt / 1e9, (S if reps == 1 else f"{S} (x{reps})"), dt

        v, S, dt = sample(threads, budget_s / 2)
        v1, S1, dt1 = sample(1, budget_s / 4)
        return {"value": v, "unit": "GB/s", "cores": threads, "kind": "oracle",
                "sample": f"decode of the first {S} of {B} sequences, all {Hq} heads, fp64 ({dt:.1f} s)",
                "seconds": dt,
                "single_thread": {"value": v1, "unit": "GB/s", "cores": 1,
                                  "sample": f"decode of the first {S1} of {B} sequences, all heads, fp64, "
                                            f"one thread ({dt1:.1f} s)"}}
    T = c.q.shape[0]
    Hq = c.num_q_heads
    rng = np.random.default_rng(0)
    _oracle_inputs(step)

    def sample(n_threads, seconds):
        # random (row, head) items, their number grown until the run takes about `seconds`
        oracle.set_threads(n_threads)
        try:
            n, dt, reps = 64, 0.0, 1
            for _ in range(5):
                items = rng.choice(T * Hq, n, replace=False)
                t0 = time.perf_counter()
                _run_oracle_prefill(step, items)
                dt = time.perf_counter() - t0
                if dt >= seconds / 2 or n == T * Hq:
                    break
                n = int(min(T * Hq, max(n + 1, n * seconds / max(dt, 1e-3))))
            if dt < seconds / 2:                               # every item is quicker: repeat them
                reps = int(min(20, np.ceil(seconds / 2 / max(dt, 1e-3))))
                t0 = time.perf_counter()
                for _ in range(reps):
                    _run_oracle_prefill(step, items)
                dt = time.perf_counter() - t0
        finally:
            oracle.set_threads(threads)
        # items are drawn uniformly, so their share of the flops is their share of the items
        return reps * step.work * n / (T * Hq) / dt / 1e12, (n if reps == 1 else f"{n} (x{reps})"), dt

    v, n, dt = sample(threads, budget_s / 2)
    v1, n1, dt1 = sample(1, budget_s / 4)
    return {"value": v, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
            "sample": f"prefill of {n} random (row, head) items of {T * Hq}, fp64 ({dt:.1f} s)", "seconds": dt,
            "single_thread": {"value": v1, "unit": "TFLOP/s", "cores": 1,
                              "sample": f"prefill of {n1} random (row, head) items, fp64, one thread "
                                        f"({dt1:.1f} s)"}}


def _oracle_inputs(step):
    """The pool the oracle reads (after the step's cache append, or quantised for INT8),
    built once per step object outside any timed region."""
    import oracle
    if hasattr(step, "_oracle_kv"):
        return step._oracle_kv
    c = step.case
    if getattr(step, "int8", False):
        kq, ks = oracle.quantize_int8(c.k_pages, c.dtype)
        vq, vs = oracle.quantize_int8(c.v_pages, c.dtype)
        step._oracle_kv = (kq, vq, "i8", ks, vs)
    else:
        k, v = c.k_pages, c.v_pages
        if c.k_new is not None and c.slot_mapping is not None and len(c.slot_mapping):
            k, v = k.copy(), v.copy()
            oracle.kv_cache_write(c.k_new, c.v_new, c.slot_mapping, k, v)
        step._oracle_kv = (k, v, c.dtype, None, None)
    return step._oracle_kv


def _run_oracle_decode(step, items):
    import oracle
    c = step.case
    k, v, kv_tag, ks, vs = _oracle_inputs(step)
    return oracle.decode(c.q, c.dtype, k, v, kv_tag, c.block_tables, c.context_lens, c.scale,
                         k_scales=ks, v_scales=vs, items=items, window=getattr(step, "window", 0))


def _run_oracle_prefill(step, items):
    import oracle
    c = step.case
    k, v, kv_tag, _, _ = _oracle_inputs(step)
    return oracle.prefill(c.q, c.dtype, k, v, kv_tag, c.block_tables, c.q_start, c.context_lens, True,
                          c.scale, items=items, window=getattr(step, "window", 0))


def run_ours(args):
    import torch
    import torch.distributed as dist
    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    from paged_kv_cache_380_b200 import ops
    ops.load()
    step = make_step(args.workload, args.batch, args.graph, args.window)
    K, W = args.steps, max(3, args.warmup)
    for _ in range(W):
        if hasattr(step, "before_step"):
            step.before_step()
        step.run()
    torch.cuda.synchronize()
    code, detail = ops.device_status()
    if code != 0:
        raise RuntimeError(f"device status after warm-up: {ops.error_string(code)} ({detail})")

    sampler = ClockSampler(local)
    sampler.start()
    barrier()
    torch.cuda.synchronize()
    t_wall0 = time.perf_counter()
    total_ms, dom_ms = time_steps(step, K)
    torch.cuda.synchronize()
    t_wall1 = time.perf_counter()
    barrier()
    sampler.stop()
    clocks = sampler.summary(t_wall0, t_wall1)

    elapsed, units, work = aggregate(total_ms, step.units * K, step.work * K)

    # end to end from pinned host buffers (same metric)
    barrier()
    torch.cuda.synchronize()
    e2e_ms, h2d, d2h = time_e2e(step, K)
    e2e_ms, _, _ = aggregate(e2e_ms, 0, 0)
    barrier()
    code, detail = ops.device_status()
    if code != 0:
        raise RuntimeError(f"device status after timing: {ops.error_string(code)} ({detail})")

    peaks, peak_src = load_peaks()
    hbm = step.kind in ("decode", "scatter")
    scale_div = 1e9 if hbm else 1e12
    unit = "GB/s" if hbm else "TFLOP/s"
    value = work / (elapsed / 1e3) / scale_div
    dom_avg_ms = statistics.mean(dom_ms)
    if hbm:
        dom_work = step.decode_bytes if step.kind == "decode" else step.work
        peak = peaks["hbm_gbs"]
        achieved = dom_work / (dom_avg_ms / 1e3) / 1e9
        bound, runit = "hbm", "GB/s"
    else:
        dom_work = step.work
        peak = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
        achieved = dom_work / (dom_avg_ms / 1e3) / 1e12
        bound, runit = "tensor", "TFLOP/s"
    # the ncu figures belong to the bench launch of each workload: not to other batch sizes,
    # a local window or the graph replay
    tr = TRAFFIC.get(config_key(args.workload)) if not (args.batch or args.window or args.graph) else None
    traffic = tr["bytes"] if tr and tr["kernel_sha"] == kernel_sha(step.kind) else None
    line = {
        "metric": METRIC, "value": round(value, 3), "unit": unit, "n_gpus": world, "steps": K, "warmup": W,
        "ms_per_step": round(elapsed / K, 5), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": ("u8" if step.kind == "scatter" else "i8" if getattr(step, "int8", False)
                  else step.case.dtype),
        "data": "synthetic (seeded N(0,1) inputs, shuffled physical pages)",
        "config": dict(step.config(), parallelism=f"replicas{world}" if world > 1 else "single-gpu"),
        "impl": "ours",
        "extra": ({"tokens_per_s": round(units / (elapsed / 1e3), 1),
                   "pct_of_8TBps": round(100 * value / 8000.0, 2)} if step.kind == "decode"
                  else {"rows_per_s": round(units / (elapsed / 1e3), 1),
                        "pct_of_8TBps": round(100 * value / 8000.0, 2)} if step.kind == "scatter"
                  else {"rows_per_s": round(units / (elapsed / 1e3), 1)}),
        "roofline": {"bound": bound, "achieved": round(achieved, 3), "peak": peak, "unit": runit,
                     "frac": round(achieved / peak, 4), "traffic": traffic,
                     "kernel": ("graph replay (append + decode + merge)" if args.graph else
                                "decode call (main kernel + split-KV merge)" if step.kind == "decode"
                                else "cache append (scatter kernel)" if step.kind == "scatter"
                                else "prefill kernel"),
                     "kernel_ms": round(dom_avg_ms, 5), "peak_source": f"{peak_src} (MEASURED_PEAKS.json)"
                     if peak_src == "measured" else "fallback",
                     **({"peak_kind": "measured HBM copy rate (read + write stream); a read-mostly kernel "
                                      "can exceed it, so frac is a fraction of the copy rate",
                         "frac_of_8TBps": round(achieved / 8000.0, 4)} if hbm else
                        {"peak_kind": "measured cuBLAS bf16 GEMM rate (burst)"})},
        "e2e": {"value": round(work / (e2e_ms / 1e3) / scale_div, 3), "unit": unit,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": round(e2e_ms / K, 5)},
        "gpu_launches": step.launches * K,
        "clocks": clocks,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(step, args.cpu_seconds)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


def config_key(name):
    return name


def run_reference(args):
    """The fp64 CPU oracle as the reference arm (rank 0 only)."""
    rank, world, _ = dist_env()
    if rank != 0:
        return
    import oracle
    from paged_kv_cache_380_b200 import workloads as W
    name = args.workload
    if name == "kv_cache_write_full":
        case = W.llama2_7b_mha_decode()
        src, dst = W.full_cache_scatter(case)
        Wm, K = max(3, args.warmup), args.steps
        for _ in range(Wm):
            _oracle_scatter_rate(case, src, dst, src.shape[0])
        total = 0.0
        nbytes = 2 * 2 * int(src.shape[0]) * case.num_kv_heads * case.head_dim * 2 + 8 * int(src.shape[0])
        for _ in range(K):
            total += _oracle_scatter_rate(case, src, dst, src.shape[0])[1]
        value = nbytes * K / total / 1e9
        sample = f"all {src.shape[0]} rows per step (row copies into host copies of the pools)"
        print(json.dumps({"metric": METRIC, "value": round(value, 6), "unit": "GB/s", "n_gpus": world, "steps": K,
                          "warmup": Wm, "ms_per_step": round(total / K * 1e3, 3), "higher_is_better": True,
                          "scaling": "weak", "vs_baseline": None, "dtype": "u8",
                          "data": "synthetic (seeded N(0,1) inputs, shuffled physical pages)",
                          "config": {"workload": name, "parallelism": "host cores"}, "impl": "reference",
                          "cpu_baseline": {"value": round(value, 6), "unit": "GB/s", "cores": oracle.max_threads(),
                                           "kind": "oracle", "sample": sample},
                          "e2e": {"value": round(value, 6), "unit": "GB/s", "h2d_bytes_per_step": 0,
                                  "d2h_bytes_per_step": 0}}), flush=True)
        return
    int8 = name == "long_ctx_split_kv_int8"
    case = W.long_ctx_split_kv() if int8 else W.WORKLOADS[name]()

    class HostStep:
        pass
    step = HostStep()
    step.case, step.int8, step.kind = case, int8, case.kind
    step.has_new = case.k_new is not None and not int8
    K, Wm = args.steps, max(3, args.warmup)
    if case.kind == "decode":
        S = max(1, min(case.batch, args.ref_seqs))
        items = np.arange(S * case.num_q_heads)
        Hkv, D = case.num_kv_heads, case.head_dim
        elem = 1 if int8 else (4 if case.dtype == "f32" else 2)
        ctx = case.context_lens[:S].astype(np.int64)
        work = int(ctx.sum()) * Hkv * (2 * D * elem + (4 if int8 else 0)) + 2 * S * case.num_q_heads * D * 2
        fn = lambda: _run_oracle_decode(step, items)  # noqa: E731
        div, unit, units = 1e9, "GB/s", S
        sample = f"decode of the first {S} of {case.batch} sequences (all heads) per step"
    else:
        T, Hq = case.q.shape[0], case.num_q_heads
        n = min(T * Hq, args.ref_items)
        items = np.random.default_rng(0).choice(T * Hq, n, replace=False)
        nn = np.diff(case.q_start).astype(np.int64)
        ctx = case.context_lens.astype(np.int64)
        keys = int(np.sum(nn * (ctx - nn) + nn * (nn + 1) // 2))
        work = 4.0 * case.head_dim * Hq * keys * n / (T * Hq)
        fn = lambda: _run_oracle_prefill(step, items)  # noqa: E731
        div, unit, units = 1e12, "TFLOP/s", n
        sample = f"prefill of {n} random (row, head) items per step"
    for _ in range(Wm):
        fn()
    t0 = time.perf_counter()
    for _ in range(K):
        fn()
    dt = time.perf_counter() - t0
    value = work * K / dt / div
    line = {"metric": METRIC, "value": round(value, 6), "unit": unit, "n_gpus": world, "steps": K, "warmup": Wm,
            "ms_per_step": round(dt / K * 1e3, 3), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded N(0,1) inputs, shuffled physical pages)",
            "config": {"workload": name, "parallelism": "host cores"}, "impl": "reference",
            "cpu_baseline": {"value": round(value, 6), "unit": unit, "cores": oracle.max_threads(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": round(value, 6), "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="llama2_7b_mha_decode",
                    choices=["tiny_decode_f32", "llama2_7b_mha_decode", "llama2_70b_gqa_decode",
                             "long_ctx_split_kv", "long_ctx_split_kv_int8", "chunked_prefill_shared_prefix",
                             "kv_cache_write_full"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--graph", action="store_true",
                    help="decode workloads: replay the step as one captured CUDA graph")
    ap.add_argument("--batch", type=int, default=0,
                    help="override the batch size of a decode workload (or of kv_cache_write_full's source batch)")
    ap.add_argument("--window", type=int, default=0, help="local attention: attend only the last W keys")
    ap.add_argument("--cpu-seconds", type=float, default=20.0, help="CPU-baseline sample budget")
    ap.add_argument("--ref-seqs", type=int, default=4, help="reference arm: sequences per step (decode)")
    ap.add_argument("--ref-items", type=int, default=512, help="reference arm: (row, head) items per step")
    args = ap.parse_args(argv)
    rank, world, _ = dist_env()
    if args.gpus != world and world > 1:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE {world}")
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
