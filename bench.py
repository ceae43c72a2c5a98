#!/usr/bin/env python3
"""Benchmark of the paged decode step on B200: cache write + decode attention.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME]
    python bench.py --impl reference ...        # the fp64 CPU oracle, same workload

One step = the whole hot path over one seeded synthetic decode batch:
pa_reshape_and_cache (one new token per sequence), then pa_decode, or
pa_decode_split + pa_reduce for the long-context workload (the default, the
largest single-GPU one).  Inputs are resident in HBM when timing starts; the
K/V bytes each step reads exceed the 126 MB L2, so no flush is needed
between steps.  Timing: regions of exactly K steps, each bracketed by a
barrier and a device synchronise on both sides and timed with CUDA events,
repeated until --min-timed-s is covered; the value uses the median region.
Each kernel is also timed alone, per launch, with L2 flushed before every
launch (the roofline figure).  Multi-GPU runs are independent replicas (one
batch per GPU, no collective on the data path); times are the max over ranks.

Rank 0 prints ONE JSON line.
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
from pathlib import Path

import torch

ROOT = Path(__file__).resolve().parent
sys.path.insert(0, str(ROOT))

from paged_kv_cache_444_b200 import workloads  # noqa: E402

MAIN_CONFIG = "long_context_split"
METRIC = "paged decode attn achieved HBM GB/s & % of peak; decode tokens/s (1 B200)"
FALLBACK_HBM_GBS = 6650.0


# ---------------------------------------------------------------------------
# distributed plumbing
# ---------------------------------------------------------------------------
def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def init_dist(world: int, backend: str):
    if world > 1:
        import datetime
        import torch.distributed as dist
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))


def barrier(world: int, device=None):
    if world > 1:
        import torch.distributed as dist
        if device is not None and dist.get_backend() == "nccl":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


def max_over_ranks(value: float, world: int, device) -> float:
    if world == 1:
        return value
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(value: float, world: int, device) -> float:
    if world == 1:
        return value
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


# ---------------------------------------------------------------------------
# clocks during the timed region (NVML reads only; nothing is changed)
# ---------------------------------------------------------------------------
class ClockSampler:
    REASONS = {  # NVML clocks-event-reason bits
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
        0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
        0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
        0x100: "display_clock_setting"}

    def __init__(self, device_index: int, interval_s: float = 0.01):
        self.samples: list[tuple[int, int]] = []
        self.max_mhz = None
        self._stop = threading.Event()
        self._thread = None
        self.error = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(self._physical_index(device_index))
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception as e:  # pragma: no cover - depends on the box
            self._nv = None
            self.error = repr(e)
        self.interval = interval_s

    @staticmethod
    def _physical_index(i: int) -> int:
        vis = os.environ.get("CUDA_VISIBLE_DEVICES")
        if vis:
            try:
                return int(vis.split(",")[i])
            except (ValueError, IndexError):
                return i
        return i

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                mhz = nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM)
                reasons = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                self.samples.append((mhz, reasons))
            except Exception as e:  # pragma: no cover
                self.error = repr(e)
                return
            time.sleep(self.interval)

    def __enter__(self):
        if self._nv is not None:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self._thread:
            self._thread.join()

    def summary(self) -> dict:
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [],
                    "samples": 0, "error": self.error}
        mhz = [m for m, _ in self.samples]
        bits = 0
        for _, r in self.samples:
            bits |= r
        reasons = [name for b, name in self.REASONS.items() if bits & b and b != 0x1]
        return {"sm_mhz": statistics.median(mhz), "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(mhz)}


# ---------------------------------------------------------------------------
# the step, its kernels, and how they are timed
# ---------------------------------------------------------------------------
L2_BYTES = 126 * 1024 * 1024


class L2Flush:
    """Reads a buffer of twice the L2 size, so that the next launch starts
    with none of its inputs in L2.  Runs between timed launches, untimed.  A
    read leaves L2 holding clean lines; a write flush would leave ~126 MB of
    dirty lines whose write-back to HBM lands inside the next timed launch."""

    def __init__(self, device):
        self.buf = torch.zeros(2 * L2_BYTES // 4, dtype=torch.float32, device=device)
        self.out = torch.zeros((), dtype=torch.float32, device=device)

    def __call__(self):
        torch.sum(self.buf, dim=0, out=self.out)


def stats_ms(times) -> dict:
    """Mean, median and p10 / p90 (nearest rank) of a list of times in ms."""
    xs = sorted(float(t) for t in times)
    pick = lambda f: xs[min(len(xs) - 1, max(0, int(round(f * (len(xs) - 1)))))]
    return {"n": len(xs), "mean": statistics.fmean(xs), "median": statistics.median(xs),
            "p10": pick(0.1), "p90": pick(0.9)}


def launch_times(fn, reps: int, warmup: int, flush=None) -> list[float]:
    """CUDA-event time (ms) of each of `reps` launches of fn() on the current
    stream (the stream the binding launches on), each bracketed by its own
    pair of events; with `flush`, L2 is flushed before every launch, outside
    the events."""
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(reps)]
    for a, b in evs:
        if flush is not None:
            flush()
        a.record()
        fn()
        b.record()
    torch.cuda.synchronize()
    return [a.elapsed_time(b) for a, b in evs]


def loop_ms(fn, reps: int, warmup: int) -> float:
    """Average time (ms) of `reps` back-to-back launches of fn(): events at
    the two ends only, so consecutive launches overlap as they would in use."""
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(reps):
        fn()
    b.record()
    torch.cuda.synchronize()
    return a.elapsed_time(b) / reps


def kernel_stats(fn, nbytes: int, reps: int, warmup: int, flush) -> dict:
    """One kernel (or fixed group of kernels) timed alone: per-launch times
    with L2 flushed before each, and the back-to-back average; GB/s from the
    algorithmic bytes over the mean flushed launch time."""
    t = stats_ms(launch_times(fn, reps, warmup, flush))
    b2b = loop_ms(fn, reps, warmup)
    return {"ms": {k: (round(v, 5) if k != "n" else v) for k, v in t.items()},
            "ms_back_to_back": round(b2b, 5), "algorithmic_bytes": int(nbytes),
            "gbs": round(nbytes / (t["mean"] / 1e3) / 1e9, 1),
            "gbs_median": round(nbytes / (t["median"] / 1e3) / 1e9, 1),
            "gbs_back_to_back": round(nbytes / (b2b / 1e3) / 1e9, 1)}


class Step:
    """One decode step over a seeded batch: pa_reshape_and_cache, then
    pa_decode, or pa_decode_split + pa_reduce for the split workload."""

    def __init__(self, batch: workloads.DecodeBatch):
        from paged_kv_cache_444_b200 import SplitWorkspace
        self.b = batch
        cfg = batch.cfg
        self.cfg = cfg
        self.out = torch.empty_like(batch.query)
        self.ps = cfg.partition_size
        self.ws = None
        if self.ps:
            P = (batch.block_tables.shape[1] * cfg.block_size + self.ps - 1) // self.ps
            self.ws = SplitWorkspace(cfg.num_seqs, cfg.num_heads, cfg.head_dim, P,
                                     batch.query.device)
        self.launches = 3 if self.ps else 2
        from paged_kv_cache_444_b200 import DecodePlan
        self.plan = DecodePlan(batch.query, batch.key, batch.value, batch.key_cache,
                               batch.value_cache, batch.slot_mapping, batch.block_tables,
                               batch.context_lens, cfg.scale, out=self.out,
                               partition_size=self.ps, workspace=self.ws)

    def run(self):
        self.plan.run()   # validated once; the timed path

    def kernels(self, ctx) -> list:
        """(name, launch, algorithmic bytes) of each kernel of the step, and of
        the attention as a whole when it takes two kernels."""
        from paged_kv_cache_444_b200 import (pa_decode, pa_decode_split, pa_reduce,
                                             pa_reshape_and_cache)
        b, cfg, w = self.b, self.cfg, self.ws
        by = workloads.algorithmic_bytes(cfg, ctx)
        write = lambda: pa_reshape_and_cache(b.key, b.value, b.key_cache, b.value_cache,
                                             b.slot_mapping)
        ks = [("pa_reshape_and_cache", write, by["write"])]
        if self.ps:
            split = lambda: pa_decode_split(w.tmp_out, w.max_logits, w.exp_sums, b.query,
                                            b.key_cache, b.value_cache, b.block_tables,
                                            b.context_lens, cfg.scale, self.ps)
            reduce = lambda: pa_reduce(self.out, w.tmp_out, w.max_logits, w.exp_sums,
                                       b.context_lens, self.ps)

            def both():
                split()
                reduce()
            parts = sum(-(-int(c) // self.ps) for c in ctx) * cfg.num_heads
            reduce_bytes = parts * (cfg.head_dim + 2) * 4 + by["out"] + by["context_lens"]
            ks += [("pa_decode_split", split, attention_kernel_bytes(cfg, ctx, True)),
                   ("pa_reduce", reduce, reduce_bytes),
                   ("pa_decode_split+pa_reduce", both, by["attention"])]
        else:
            ks.append(("pa_decode", lambda: pa_decode(self.out, b.query, b.key_cache,
                                                      b.value_cache, b.block_tables,
                                                      b.context_lens, cfg.scale),
                       by["attention"]))
        return ks


def time_regions(run, steps: int, warmup: int, world: int, device, min_total_s: float,
                 max_regions: int = 400) -> list[float]:
    """Warm up, then time regions of exactly `steps` back-to-back runs, each
    bracketed by a barrier and a device synchronise on both sides and timed
    with CUDA events at its two ends; as many regions as make up min_total_s
    (at least one).  Returns each region's ms per step, max over ranks."""
    for _ in range(warmup):
        run()
    torch.cuda.synchronize()

    def region() -> float:
        barrier(world, device)
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(steps):
            run()
        b.record()
        torch.cuda.synchronize()
        barrier(world, device)
        return a.elapsed_time(b) / steps

    first = max_over_ranks(region(), world, device)
    n = max(1, min(max_regions, math.ceil(min_total_s * 1e3 / max(1e-6, first * steps))))
    times = [region() for _ in range(n - 1)]
    if world > 1 and times:
        import torch.distributed as dist
        t = torch.tensor(times, dtype=torch.float64, device=device)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        times = t.tolist()
    return [first] + times


SPLIT_PARTITION = 512  # tokens per partition of the split forms timed on single-pass batches


def shared_prefix_stats(batch, warmup: int, flush, reps: int = 100) -> dict:
    """pa_decode_shared_prefix timed alone on a batch with prefix groups: the
    same attention as pa_decode, reading each shared page once per group.
    Algorithmic bytes count the unique K/V bytes."""
    from paged_kv_cache_444_b200 import pa_decode_shared_prefix
    cfg = batch.cfg
    out = torch.empty_like(batch.query)
    sizes = (batch.group_starts[1:] - batch.group_starts[:-1]).tolist()

    def run():
        pa_decode_shared_prefix(out, batch.query, batch.key_cache, batch.value_cache,
                                batch.block_tables, batch.context_lens, batch.group_starts,
                                batch.prefix_blocks, cfg.scale, max(sizes))
    unique = workloads.unique_kv_bytes(cfg, batch.block_tables.cpu().tolist(),
                                       batch.context_lens.cpu().tolist())
    by = workloads.algorithmic_bytes(cfg, batch.context_lens.cpu().tolist())
    nbytes = unique + by["block_table"] + by["query"] + by["out"] + by["context_lens"]
    r = kernel_stats(run, nbytes, reps, warmup, flush)
    r["kernel"] = "pa_decode_shared_prefix"
    return r


def fp8_stats(batch, warmup: int, flush, reps: int = 100,
              partition_size: int | None = None) -> dict | None:
    """pa_decode_fp8 (pa_decode_split_fp8 + pa_reduce for the split workload,
    or when a partition size is given) timed alone on the same batch with its
    caches held as E4M3 codes (x * 64 quantised by torch, scale 1/64); None
    where the fp8 path is not built (head_dim != 128).  Algorithmic bytes
    count K/V at one byte per element."""
    from paged_kv_cache_444_b200 import (SplitWorkspace, pa_decode_fp8, pa_decode_split_fp8,
                                         pa_reduce)
    cfg = batch.cfg
    if cfg.head_dim != 128:
        return None
    q8 = lambda t: (t.float() * 64.0).clamp(-448, 448).to(torch.float8_e4m3fn).view(torch.uint8)
    kc, vc = q8(batch.key_cache), q8(batch.value_cache)
    out = torch.empty_like(batch.query)
    ctx = batch.context_lens.cpu().tolist()
    by = workloads.algorithmic_bytes(cfg, ctx)
    nbytes = by["kv"] // 2 + by["block_table"] + by["query"] + by["out"] + by["context_lens"]
    ps = cfg.partition_size if partition_size is None else partition_size
    if ps:
        P = (batch.block_tables.shape[1] * cfg.block_size + ps - 1) // ps
        ws = SplitWorkspace(cfg.num_seqs, cfg.num_heads, cfg.head_dim, P, batch.query.device)

        def run():
            pa_decode_split_fp8(ws.tmp_out, ws.max_logits, ws.exp_sums, batch.query, kc, vc,
                                batch.block_tables, batch.context_lens, cfg.scale, 1.0 / 64,
                                1.0 / 64, ps)
            pa_reduce(out, ws.tmp_out, ws.max_logits, ws.exp_sums, batch.context_lens, ps)
        kernel = "pa_decode_split_fp8+pa_reduce"
    else:
        def run():
            pa_decode_fp8(out, batch.query, kc, vc, batch.block_tables, batch.context_lens,
                          cfg.scale, 1.0 / 64, 1.0 / 64)
        kernel = "pa_decode_fp8"
    r = kernel_stats(run, nbytes, reps, warmup, flush)
    r["kernel"] = kernel
    if ps:
        r["partition_size"] = ps
    del kc, vc
    return r


def split_variants(batch, warmup: int, flush, reps: int, fp8: bool) -> dict:
    """pa_decode_split + pa_reduce (and its fp8 form) with 512-token
    partitions on a single-pass batch: the same attention cut into
    equal-sized items."""
    from paged_kv_cache_444_b200 import SplitWorkspace, pa_decode_split, pa_reduce
    cfg = batch.cfg
    ps = SPLIT_PARTITION
    P = (batch.block_tables.shape[1] * cfg.block_size + ps - 1) // ps
    ws = SplitWorkspace(cfg.num_seqs, cfg.num_heads, cfg.head_dim, P, batch.query.device)
    out = torch.empty_like(batch.query)

    def run():
        pa_decode_split(ws.tmp_out, ws.max_logits, ws.exp_sums, batch.query, batch.key_cache,
                        batch.value_cache, batch.block_tables, batch.context_lens, cfg.scale, ps)
        pa_reduce(out, ws.tmp_out, ws.max_logits, ws.exp_sums, batch.context_lens, ps)
    nbytes = workloads.algorithmic_bytes(cfg, batch.context_lens.cpu().tolist())["attention"]
    r = {"pa_decode_split+pa_reduce": kernel_stats(run, nbytes, reps, warmup, flush)}
    if fp8:
        r["fp8"] = fp8_stats(batch, warmup, flush, reps, partition_size=ps)
    return r


def prefill_measure(device, warmup: int, reps: int = 100, peak_tflops: float = 0.0,
                    peak_kind: str = "", flush=None) -> dict:
    """Chunked prefill on a Llama-3-8B-shaped GQA layer: 8 sequences each
    bringing a 512-token chunk at the end of a context drawn U[512, 4096]
    (32/8 heads, d=128, bf16, 16-token blocks).  Compute-bound: reported in
    TFLOP/s against the measured dense bf16 peak, with the CPU oracle's
    count of flops: 4 * D * H * sum over queries of (position + 1)."""
    from paged_kv_cache_444_b200 import pa_prefill
    pb = workloads.make_prefill_batch(device=device)
    b, cfg, chunk, query, starts = pb.cache, pb.cache.cfg, pb.chunk, pb.query, pb.query_starts
    T = query.shape[0]
    out = torch.empty_like(query)

    def run():
        pa_prefill(out, query, b.key_cache, b.value_cache, b.block_tables, b.context_lens,
                   starts, cfg.scale, chunk)
    t = stats_ms(launch_times(run, reps, warmup, flush))
    b2b = loop_ms(run, reps, warmup)
    ms = t["mean"]
    ctx = b.context_lens.cpu().tolist()
    pairs = sum(sum(c - chunk + i + 1 for i in range(chunk)) for c in ctx)
    flops = 4 * cfg.head_dim * cfg.num_heads * pairs
    tf = flops / (ms / 1e3) / 1e12
    return {"workload": "chunked_prefill_gqa: 8 seqs x 512-token chunks at ctx U[512,4096], "
                        "32/8 heads, d=128, bf16", "kernel": "pa_prefill",
            "ms": round(ms, 5), "ms_stats": {k: (round(v, 5) if k != "n" else v)
                                             for k, v in t.items()},
            "ms_back_to_back": round(b2b, 5), "tflops": round(tf, 1),
            "tflops_back_to_back": round(flops / (b2b / 1e3) / 1e12, 1),
            "query_tokens_per_s": round(T / (ms / 1e3), 1),
            "roofline": {"bound": "tensor", "achieved": round(tf, 1), "peak": peak_tflops,
                         "unit": "TFLOP/s", "frac": round(tf / peak_tflops, 4) if peak_tflops else None,
                         "peak_kind": peak_kind, "algorithmic_flops": flops,
                         "timing": "mean of per-launch CUDA-event times, L2 flushed before each"}}


def graph_steps(step: Step, steps: int, warmup: int) -> float | None:
    """The same step captured once in a CUDA graph and replayed `steps` times
    (ms per step), or None if capture is not possible here."""
    try:
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            for _ in range(3):
                step.run()
        torch.cuda.current_stream().wait_stream(s)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            step.run()
        for _ in range(warmup):
            g.replay()
        torch.cuda.synchronize()
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        start.record()
        for _ in range(steps):
            g.replay()
        end.record()
        torch.cuda.synchronize()
        del g
        return start.elapsed_time(end) / steps
    except Exception as e:  # pragma: no cover - depends on the box
        print(f"graph capture unavailable: {e!r}", file=sys.stderr)
        return None


class _Null:
    def __enter__(self):
        return self

    def __exit__(self, *a):
        return False


def parse_cpulist(spec: str) -> set[int]:
    """The CPUs of a sysfs cpulist such as "0-15,32-47" (an empty list: none)."""
    cpus: set[int] = set()
    for part in spec.strip().split(","):
        if not part:
            continue
        lo, _, hi = part.partition("-")
        cpus.update(range(int(lo), int(hi or lo) + 1))
    return cpus


def bind_to_gpu_local_cpus(device_index: int) -> str:
    """Restrict this process to the CPUs on the GPU's own NUMA node, before any
    pinned host buffer is allocated, so that the staging memory of the
    host-buffer step is first touched (and so placed) on that node and the PCIe
    copies do not cross the socket link.  Reads sysfs only; changes nothing
    outside this process.  Returns a short description for the JSON line."""
    try:
        p = torch.cuda.get_device_properties(device_index)
        dev = Path("/sys/bus/pci/devices") / (
            f"{p.pci_domain_id:04x}:{p.pci_bus_id:02x}:{p.pci_device_id:02x}.0")
        cpus = parse_cpulist((dev / "local_cpulist").read_text())
        node = (dev / "numa_node").read_text().strip()
        cpus &= os.sched_getaffinity(0)
        if not cpus:
            return "unbound (no GPU-local CPU available to this process)"
        os.sched_setaffinity(0, cpus)
        return f"{len(cpus)} GPU-local CPUs (NUMA node {node})"
    except Exception as e:  # pragma: no cover - depends on the box
        return f"unbound ({type(e).__name__})"


def e2e_regions(step: Step, steps: int, warmup: int, world: int, device, min_total_s: float):
    """The same step through the C ABI from host buffers (pa_decode_step_host):
    every step copies its inputs in from pinned host memory, writes the cache,
    attends, and copies the output back, all inside the timing.  Regions of
    exactly `steps` steps as for the device-resident step."""
    from paged_kv_cache_444_b200 import HostStep
    b, cfg = step.b, step.cfg
    hs = HostStep(b.key_cache, b.value_cache, cfg.num_seqs, cfg.num_heads,
                  b.block_tables.shape[1], cfg.scale, step.ps, cfg.torch_dtype)
    for n in ("query", "key", "value", "slot_mapping", "block_tables", "context_lens"):
        getattr(hs, n).copy_(getattr(b, n).cpu())
    regions = time_regions(hs.run, steps, warmup, world, device, min_total_s)
    return regions, hs.h2d_bytes, hs.d2h_bytes


# ---------------------------------------------------------------------------
# byte accounting and peaks
# ---------------------------------------------------------------------------
def measured_peak():
    p = ROOT / "MEASURED_PEAKS.json"
    if p.exists():
        try:
            d = json.loads(p.read_text())
            return float(d["hbm_gbs"]), "measured"
        except Exception:
            pass
    return FALLBACK_HBM_GBS, "fallback"


def measured_tensor_peak():
    """Dense bf16 TFLOP/s: the burst figure (a kernel timed alone)."""
    p = ROOT / "MEASURED_PEAKS.json"
    if p.exists():
        try:
            return float(json.loads(p.read_text())["bf16_tflops"]), "measured (burst)"
        except Exception:
            pass
    return 1590.0, "fallback (burst)"


def attention_kernel_bytes(cfg, context_lens, split: bool) -> int:
    a = workloads.algorithmic_bytes(cfg, context_lens)
    return a["kv"] + a["block_table"] + a["query"] + a["context_lens"] + (0 if split else a["out"])


# ---------------------------------------------------------------------------
# CPU baseline: the oracle on a bounded sample of the same workload
# ---------------------------------------------------------------------------
def _compact_host(cfg, context_lens, block_tables, seqs, gen_values: bool, batch=None):
    """Host inputs for sequences `seqs` with their blocks renumbered 0..n-1."""
    import numpy as np
    bs = cfg.block_size
    used, bt_new = {}, []
    for s in seqs:
        c = int(context_lens[s])
        row = []
        for j in range((c + bs - 1) // bs):
            b = int(block_tables[s][j])
            row.append(used.setdefault(b, len(used)))
        bt_new.append(row)
    MB = max(1, max(len(r) for r in bt_new))
    bt = np.full((len(seqs), MB), -1, dtype=np.int32)
    for i, r in enumerate(bt_new):
        bt[i, :len(r)] = r
    n = len(used)
    shape = (n, bs, cfg.num_kv_heads, cfg.head_dim)
    if gen_values:
        g = torch.Generator().manual_seed(cfg.seed + 99)
        mk = lambda sh: torch.randn(sh, generator=g).to(cfg.torch_dtype)
        kc, vc = mk(shape), mk(shape)
        q = mk((len(seqs), cfg.num_heads, cfg.head_dim))
        key = mk((len(seqs), cfg.num_kv_heads, cfg.head_dim))
        value = mk((len(seqs), cfg.num_kv_heads, cfg.head_dim))
    else:
        ids = torch.tensor(list(used), dtype=torch.long, device=batch.key_cache.device)
        kc = batch.key_cache.index_select(0, ids).cpu()
        vc = batch.value_cache.index_select(0, ids).cpu()
        idx = torch.tensor(seqs, dtype=torch.long, device=batch.query.device)
        q, key, value = (batch.query[idx].cpu(), batch.key[idx].cpu(), batch.value[idx].cpu())
    to_bits = lambda t: t.contiguous().view(torch.int16).numpy().view(np.uint16)
    slots = []
    for i, s in enumerate(seqs):
        c = int(context_lens[s])
        slots.append(-1 if c == 0 else int(bt[i, (c - 1) // bs]) * bs + (c - 1) % bs)
    return dict(kc=to_bits(kc), vc=to_bits(vc), q=to_bits(q), key=to_bits(key),
                value=to_bits(value), bt=bt, slots=np.array(slots, dtype=np.int64),
                ctx=np.array([int(context_lens[s]) for s in seqs], dtype=np.int32), nblocks=n)


def oracle_sample_run(cfg, host) -> float:
    """One oracle step (write + decode) on a compact host sample; seconds."""
    import oracle
    orc = oracle.load()
    code = oracle.BF16 if cfg.dtype == "bf16" else oracle.F16
    kc, vc = host["kc"].copy(), host["vc"].copy()
    t0 = time.perf_counter()
    orc.reshape_and_cache(host["key"], host["value"], kc, vc, host["slots"], host["nblocks"],
                          cfg.block_size)
    orc.decode(host["q"], kc, vc, host["bt"], host["ctx"], cfg.scale, code)
    return time.perf_counter() - t0


def pick_sample(cfg, context_lens, budget_s: float, probe_s_per_token: float | None = None):
    """Sequences (in order) whose oracle work fits in about budget_s."""
    S = len(context_lens)
    order = list(range(S))
    if probe_s_per_token is None:
        return order
    seqs, acc = [], 0.0
    for s in order:
        est = int(context_lens[s]) * probe_s_per_token
        if seqs and acc + est > budget_s:
            break
        seqs.append(s)
        acc += est
    return seqs


def cpu_baseline(cfg, context_lens, block_tables, batch, budget_s: float = 12.0) -> dict:
    # calibrate on the shortest sequence, then fill the budget
    shortest = min(range(len(context_lens)), key=lambda s: int(context_lens[s]))
    probe = _compact_host(cfg, context_lens, block_tables, [shortest], batch is None, batch)
    t = oracle_sample_run(cfg, probe)
    per_tok = t / max(1, int(context_lens[shortest]))
    seqs = pick_sample(cfg, context_lens, budget_s, per_tok)
    host = _compact_host(cfg, context_lens, block_tables, seqs, batch is None, batch)
    secs = oracle_sample_run(cfg, host)
    sub_ctx = [int(context_lens[s]) for s in seqs]
    sub_cfg = cfg.scaled(num_seqs=len(seqs))
    by = workloads.algorithmic_bytes(sub_cfg, sub_ctx)["step"]
    return {"value": round(by / secs / 1e9, 4), "unit": "GB/s", "cores": 1, "kind": "oracle",
            "seconds": round(secs, 3), "host": host_description(),
            "sample": f"{len(seqs)} of {cfg.num_seqs} sequences of {cfg.name} "
                      f"({sum(sub_ctx)} context tokens, all {cfg.num_heads} heads): oracle "
                      f"cache write + fp64 decode, single thread"}


def host_description() -> dict:
    """The host the CPU baseline ran on: its CPU model (/proc/cpuinfo), the
    logical CPUs the OS reports, and how many the oracle used (one)."""
    model = None
    try:
        for line in Path("/proc/cpuinfo").read_text().splitlines():
            if line.startswith("model name"):
                model = line.split(":", 1)[1].strip()
                break
    except OSError:
        pass
    return {"cpu_model": model, "os_cpu_count": os.cpu_count(), "cores_used": 1}


# ---------------------------------------------------------------------------
# arms
# ---------------------------------------------------------------------------
def run_native(args, world, rank, local):
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    host_cpus = bind_to_gpu_local_cpus(local)
    init_dist(world, "nccl")
    from paged_kv_cache_444_b200 import load
    load()
    peak, peak_kind = measured_peak()
    flush = L2Flush(device)

    def bench_config(name, steps, min_total_s, clocks=None):
        cfg = workloads.CONFIGS[name]
        cfg = cfg.scaled(seed=cfg.seed + 1000 * rank)
        if name == args.config and (args.num_seqs or args.num_blocks):
            # a smaller batch of the same workload (profiling captures only)
            cfg = cfg.scaled(num_seqs=args.num_seqs or cfg.num_seqs,
                             num_blocks=args.num_blocks or cfg.num_blocks,
                             name=f"{cfg.name}[seqs={args.num_seqs or cfg.num_seqs}]")
        batch = workloads.make_batch(cfg, device)
        step = Step(batch)
        ctx = batch.context_lens.cpu().tolist()
        by = workloads.algorithmic_bytes(cfg, ctx)
        with (clocks if clocks is not None else _Null()):
            regions = time_regions(step.run, steps, args.warmup, world, device, min_total_s)
        st = stats_ms(regions)
        total_bytes = sum_over_ranks(by["step"], world, device)
        kernels = {}
        for kname, fn, nbytes in step.kernels(ctx):
            k = kernel_stats(fn, nbytes, args.kernel_reps, args.warmup, flush)
            k["frac_of_peak"] = round(k["gbs"] / peak, 4)
            kernels[kname] = k
        attn = "pa_decode_split+pa_reduce" if step.ps else "pa_decode"
        res = {
            "regions": regions, "stats": st, "ms_per_step": st["median"],
            "value": total_bytes / (st["median"] / 1e3) / 1e9,
            "bytes": by, "kernels": kernels, "attention_kernel": attn,
            "dominant": "pa_decode_split" if step.ps else "pa_decode",
            "tokens_per_s": sum_over_ranks(cfg.num_seqs, world, device) / (st["median"] / 1e3),
            "graph_ms_per_step": graph_steps(step, steps, args.warmup) if args.graph else None,
            "shared_prefix": (shared_prefix_stats(batch, args.warmup, flush, args.kernel_reps)
                              if batch.group_starts is not None else None),
            "fp8": fp8_stats(batch, args.warmup, flush, args.kernel_reps) if args.fp8 else None,
            # batches of few, unequal items: the split form of each kernel too
            "split512": (split_variants(batch, args.warmup, flush, args.kernel_reps, args.fp8)
                         if batch.group_starts is not None else None),
            "context_tokens": int(sum(ctx)), "name": name,
        }
        for key in ("shared_prefix",):
            if res[key]:
                res[key]["frac_of_peak"] = round(res[key]["gbs"] / peak, 4)
                res[key]["speedup_vs_pa_decode"] = round(
                    kernels["pa_decode"]["ms"]["mean"] / res[key]["ms"]["mean"], 3)
        if res["fp8"]:
            res["fp8"]["frac_of_peak"] = round(res["fp8"]["gbs"] / peak, 4)
            res["fp8"]["speedup_vs_16bit"] = round(
                kernels[attn]["ms"]["mean"] / res["fp8"]["ms"]["mean"], 3)
        if res["split512"]:
            for v in (res["split512"]["pa_decode_split+pa_reduce"], res["split512"].get("fp8")):
                if v:
                    v["frac_of_peak"] = round(v["gbs"] / peak, 4)
        return cfg, batch, step, res

    results = {}
    clocks = ClockSampler(local)
    cfg, batch, step, main = bench_config(args.config, args.steps, args.min_timed_s, clocks)
    e2e_reg, h2d, d2h = e2e_regions(step, args.steps, args.warmup, world, device,
                                    args.min_timed_s)
    e2e_st = stats_ms(e2e_reg)
    total_bytes = sum_over_ranks(main["bytes"]["step"], world, device)
    ctx_main = batch.context_lens.cpu().tolist()
    bt_main = batch.block_tables.cpu().tolist()

    results[args.config] = main
    if not args.only_main:
        for name in workloads.CONFIG_ORDER:
            if name == args.config:
                continue
            _, b2, s2, r = bench_config(name, args.config_steps, args.config_min_timed_s)
            results[name] = r
            del b2, s2
            torch.cuda.empty_cache()

    kname = main["dominant"]
    kmain = main["kernels"][kname]
    roof = {"bound": "hbm", "kernel": kname,
            "achieved": kmain["gbs"], "peak": peak, "unit": "GB/s",
            "frac": round(kmain["gbs"] / peak, 4), "peak_kind": peak_kind,
            "algorithmic_bytes_per_launch": kmain["algorithmic_bytes"],
            "timing": f"mean of {kmain['ms']['n']} per-launch CUDA-event times of the kernel "
                      f"alone, L2 flushed before each launch",
            "launch_ms": kmain["ms"],
            "traffic": recorded_traffic(args.config, kname, sum(ctx_main))}
    st = main["stats"]
    line = {
        "metric": METRIC,
        "value": round(main["value"], 2),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(main["ms_per_step"], 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": cfg.dtype,
        "data": "synthetic (seeded N(0,1) K/V/Q, seeded random block placement)",
        "config": {"workload": cfg.name, "description": cfg.description,
                   "num_seqs": cfg.num_seqs, "num_heads": cfg.num_heads,
                   "num_kv_heads": cfg.num_kv_heads, "head_dim": cfg.head_dim,
                   "block_size": cfg.block_size, "num_blocks": cfg.num_blocks,
                   "partition_size": cfg.partition_size or None,
                   "context_tokens": int(sum(ctx_main)),
                   "l2": "inputs larger than L2 (K/V read per step >> 126 MB), no flush between "
                         "steps; kernels timed alone are L2-flushed before each launch",
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU"},
        "timing": {"regions": len(main["regions"]), "steps_per_region": args.steps,
                   "ms_per_step_median": round(st["median"], 5),
                   "ms_per_step_p10": round(st["p10"], 5), "ms_per_step_p90": round(st["p90"], 5),
                   "ms_per_step_mean": round(st["mean"], 5),
                   "first_region_ms_per_step": round(main["regions"][0], 5),
                   "timed_s": round(sum(main["regions"]) * args.steps / 1e3, 3),
                   "value_is": "step bytes / median over regions of the region's ms per step"},
        "decode_tokens_per_s": round(main["tokens_per_s"], 1),
        "graph_ms_per_step": (round(main["graph_ms_per_step"], 5)
                              if main["graph_ms_per_step"] else None),
        "kernels": main["kernels"],
        "roofline": roof,
        "gpu_launches": step.launches * args.steps * len(main["regions"]),
        "e2e": {"value": round(total_bytes / (e2e_st["median"] / 1e3) / 1e9, 2), "unit": "GB/s",
                "ms_per_step": round(e2e_st["median"], 5),
                "ms_per_step_p10": round(e2e_st["p10"], 5),
                "ms_per_step_p90": round(e2e_st["p90"], 5),
                "steps": args.steps * len(e2e_reg), "regions": len(e2e_reg),
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "frac_of_resident_step": round(main["ms_per_step"] / e2e_st["median"], 4),
                "api": "pa_decode_step_host (C ABI, pinned host buffers in and out)",
                "host_cpus": host_cpus},
        "clocks": clocks.summary(),
    }
    line["per_config"] = {n: config_entry(r, peak) for n, r in results.items()}
    if args.prefill and not args.only_main:
        tp, tk = measured_tensor_peak()
        line["prefill"] = prefill_measure(device, args.warmup, reps=args.prefill_reps,
                                          peak_tflops=tp, peak_kind=tk, flush=flush)
    if world == 1 and rank == 0 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(cfg, ctx_main, bt_main, batch,
                                            budget_s=args.cpu_budget)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def config_entry(r: dict, peak: float) -> dict:
    """The per-workload summary of the JSON line."""
    attn = r["kernels"][r["attention_kernel"]]
    e = {"ms_per_step": round(r["ms_per_step"], 5), "step_gbs": round(r["value"], 1),
         "ms_per_step_p10": round(r["stats"]["p10"], 5),
         "ms_per_step_p90": round(r["stats"]["p90"], 5),
         "attention_kernel": r["attention_kernel"], "attention_gbs": attn["gbs"],
         "attention_frac_of_peak": round(attn["gbs"] / peak, 4),
         "kernel": r["dominant"], "kernel_gbs": r["kernels"][r["dominant"]]["gbs"],
         "kernel_frac_of_peak": r["kernels"][r["dominant"]]["frac_of_peak"],
         "kernel_traffic": recorded_traffic(r.get("name", ""), r["dominant"],
                                            r["context_tokens"]),
         "decode_tokens_per_s": round(r["tokens_per_s"], 1),
         "graph_ms_per_step": (round(r["graph_ms_per_step"], 5)
                               if r["graph_ms_per_step"] else None),
         "kernels": {k: {"ms_mean": v["ms"]["mean"], "ms_median": v["ms"]["median"],
                         "ms_p10": v["ms"]["p10"], "ms_p90": v["ms"]["p90"],
                         "ms_back_to_back": v["ms_back_to_back"], "gbs": v["gbs"],
                         "frac_of_peak": v["frac_of_peak"]}
                     for k, v in r["kernels"].items()}}
    if r["shared_prefix"]:
        e["pa_decode_shared_prefix"] = r["shared_prefix"]
    if r["fp8"]:
        e["fp8"] = r["fp8"]
    if r["split512"]:
        e["split512"] = r["split512"]
    return e


def recorded_traffic(config: str, kernel: str, context_tokens: int):
    """DRAM bytes per launch of `kernel` on `config` from the committed ncu
    capture (profiles/traffic.json), or None if there is none or the kernel
    sources changed since it was taken."""
    tp = ROOT / "profiles" / "traffic.json"
    if not tp.exists():
        return None
    try:
        t = json.loads(tp.read_text()).get(config, {}).get(kernel)
    except Exception:
        return None
    if not t or t.get("source_sha") != kernel_source_digest():
        return None
    if t.get("bytes_per_launch"):
        return int(t["bytes_per_launch"])
    if t.get("bytes_per_context_token"):
        return int(t["bytes_per_context_token"] * context_tokens)
    return None


# sources off the 16-bit decode path whose traffic profiles/traffic.json
# records: the chunked-prefill kernel, its tensor-core helpers, the
# shared-prefix kernel and the fp8 page steps
OFF_DECODE_PATH = ("pa_prefill.cuh", "pa_umma.cuh", "pa_shared_prefix.cuh", "pa_decode_fp8.cuh")


def kernel_source_digest(csrc: Path | None = None) -> str:
    """Hash of the decode path's code: every csrc file but those off the
    path, with the marked host-side regions of pa_api.cu that serve other
    kernels ("// >>> ..." to "// <<< ...") left out, then comments, trailing
    blanks and empty lines removed, so that an edit of comments alone keeps
    the hash (and the traffic captured for the code)."""
    import hashlib
    import re
    h = hashlib.sha256()
    for p in sorted((csrc or ROOT / "paged_kv_cache_444_b200" / "csrc").glob("*")):
        if p.name in OFF_DECODE_PATH:
            continue
        data = p.read_bytes()
        if p.name == "pa_api.cu":
            data = re.sub(rb"\n// >>> .*?\n// <<< [^\n]*", b"", data, flags=re.S)
        data = re.sub(rb"/\*.*?\*/", b"", data, flags=re.S)
        data = re.sub(rb"//[^\n]*", b"", data)
        data = re.sub(rb"[ \t]+\n", b"\n", data)
        data = re.sub(rb"\n\s*\n", b"\n", data)
        h.update(p.name.encode() + b"\0" + data)
    return h.hexdigest()[:16]


PROFILE_KERNELS = ("pa_reshape_and_cache", "pa_decode", "pa_decode_split", "pa_reduce",
                   "pa_decode_shared_prefix", "pa_decode_fp8", "pa_decode_split_fp8", "pa_prefill")


def run_profile(args, local):
    """Launch one kernel alone, --warmup + --steps times, on the --config
    workload (pa_prefill: its chunked-prefill layer), for profiler captures:
    nothing else of the library runs.  Prints the mean CUDA-event time of the
    --steps launches as a short JSON object (not a bench line)."""
    from paged_kv_cache_444_b200 import (SplitWorkspace, load, pa_decode_fp8,
                                         pa_decode_shared_prefix, pa_decode_split,
                                         pa_decode_split_fp8, pa_prefill, pa_reduce)
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    load()
    name = args.profile
    if name == "pa_prefill":
        pb = workloads.make_prefill_batch(device=device)
        b = pb.cache

        out = torch.empty_like(pb.query)

        def run():
            pa_prefill(out, pb.query, b.key_cache, b.value_cache, b.block_tables,
                       b.context_lens, pb.query_starts, b.cfg.scale, pb.chunk)
        cfg = b.cfg
    else:
        cfg = workloads.CONFIGS[args.config]
        if args.num_seqs or args.num_blocks:
            cfg = cfg.scaled(num_seqs=args.num_seqs or cfg.num_seqs,
                             num_blocks=args.num_blocks or cfg.num_blocks)
        b = workloads.make_batch(cfg, device)
        step = Step(b)
        ps = cfg.partition_size or SPLIT_PARTITION
        P = (b.block_tables.shape[1] * cfg.block_size + ps - 1) // ps
        ws = SplitWorkspace(cfg.num_seqs, cfg.num_heads, cfg.head_dim, P, device)
        out = torch.empty_like(b.query)
        sizes = ((b.group_starts[1:] - b.group_starts[:-1]).tolist()
                 if b.group_starts is not None else None)
        if name in ("pa_decode_fp8", "pa_decode_split_fp8"):
            q8 = lambda t: (t.float() * 64.0).clamp(-448, 448).to(torch.float8_e4m3fn) \
                .view(torch.uint8)
            kc8, vc8 = q8(b.key_cache), q8(b.value_cache)
        if name == "pa_decode_shared_prefix" and sizes is None:
            raise SystemExit(f"--profile {name} needs a workload with prefix groups")
        step_kernels = dict((n, fn) for n, fn, _ in step.kernels([]))
        launches = {
            "pa_reshape_and_cache": step_kernels["pa_reshape_and_cache"],
            "pa_decode": step_kernels.get("pa_decode"),
            "pa_decode_split": lambda: pa_decode_split(
                ws.tmp_out, ws.max_logits, ws.exp_sums, b.query, b.key_cache, b.value_cache,
                b.block_tables, b.context_lens, cfg.scale, ps),
            "pa_reduce": lambda: pa_reduce(out, ws.tmp_out, ws.max_logits, ws.exp_sums,
                                           b.context_lens, ps),
            "pa_decode_shared_prefix": lambda: pa_decode_shared_prefix(
                out, b.query, b.key_cache, b.value_cache, b.block_tables, b.context_lens,
                b.group_starts, b.prefix_blocks, cfg.scale, max(sizes)),
            "pa_decode_fp8": lambda: pa_decode_fp8(
                out, b.query, kc8, vc8, b.block_tables, b.context_lens, cfg.scale, 1 / 64, 1 / 64),
            "pa_decode_split_fp8": lambda: pa_decode_split_fp8(
                ws.tmp_out, ws.max_logits, ws.exp_sums, b.query, kc8, vc8, b.block_tables,
                b.context_lens, cfg.scale, 1 / 64, 1 / 64, ps),
        }
        if name == "pa_decode" and step.ps:
            raise SystemExit("--profile pa_decode: use a single-pass workload")
        if name == "pa_reduce":
            launches["pa_decode_split"]()      # partials for the merge to read
        run = launches[name]
    for _ in range(args.warmup):
        run()
    torch.cuda.synchronize()
    a, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(args.steps):
        run()
    e.record()
    torch.cuda.synchronize()
    print(json.dumps({"profile": name, "workload": cfg.name, "launches": args.steps,
                      "ms_per_launch": round(a.elapsed_time(e) / args.steps, 5)}))


def run_reference(args, world, rank, local):
    """The oracle (fp64, one CPU thread) as the reference arm: each step is a
    bounded sample of the same workload."""
    if world > 1:
        init_dist(world, "gloo")
        if rank != 0:
            import torch.distributed as dist
            dist.barrier()
            dist.destroy_process_group()
            return
    cfg = workloads.CONFIGS[args.config]
    gen = torch.Generator().manual_seed(cfg.seed)
    ctx = workloads.draw_context_lens(cfg, gen)
    bt = workloads.build_block_tables(cfg, ctx, gen)
    ctx_l, bt_l = ctx.tolist(), bt.tolist()
    probe = _compact_host(cfg, ctx_l, bt_l, [0], True)
    per_tok = oracle_sample_run(cfg, probe) / max(1, ctx_l[0])
    budget = max(0.5, args.cpu_budget / max(1, args.steps + args.warmup))
    seqs = pick_sample(cfg, ctx_l, budget, per_tok)
    host = _compact_host(cfg, ctx_l, bt_l, seqs, True)
    for _ in range(args.warmup):
        oracle_sample_run(cfg, host)
    times = [oracle_sample_run(cfg, host) for _ in range(args.steps)]
    secs = sum(times) / len(times)
    sub_ctx = [ctx_l[s] for s in seqs]
    by = workloads.algorithmic_bytes(cfg.scaled(num_seqs=len(seqs)), sub_ctx)["step"]
    value = by / secs / 1e9
    sample = (f"{len(seqs)} of {cfg.num_seqs} sequences of {cfg.name} per step "
              f"({sum(sub_ctx)} context tokens, all {cfg.num_heads} heads)")
    line = {
        "metric": METRIC, "impl": "reference", "value": round(value, 4), "unit": "GB/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(secs * 1e3, 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": cfg.name, "description": cfg.description},
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": 1, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20,
                    help="steps per timed region (each region is exactly this many steps)")
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["native", "reference"], default="native")
    ap.add_argument("--config", default=MAIN_CONFIG, choices=list(workloads.CONFIGS))
    ap.add_argument("--min-timed-s", type=float, default=1.0,
                    help="regions of --steps steps are repeated until this much is timed")
    ap.add_argument("--config-steps", type=int, default=20,
                    help="steps per timed region for each of the other workloads")
    ap.add_argument("--config-min-timed-s", type=float, default=0.25)
    ap.add_argument("--kernel-reps", type=int, default=100,
                    help="launches of each kernel timed alone (L2 flushed before each)")
    ap.add_argument("--only-main", action="store_true", help="skip the per-workload table")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=12.0,
                    help="seconds of oracle work for the CPU baseline")
    ap.add_argument("--graph", action=argparse.BooleanOptionalAction, default=True,
                    help="also time the step replayed from a CUDA graph")
    ap.add_argument("--fp8", action=argparse.BooleanOptionalAction, default=True,
                    help="also time the fp8 decode on each batch (E4M3 copy of its caches)")
    ap.add_argument("--prefill", action=argparse.BooleanOptionalAction, default=True,
                    help="also time pa_prefill on a chunked-prefill GQA layer")
    ap.add_argument("--only-prefill", action="store_true",
                    help="time only pa_prefill (its own JSON object; for profiling captures)")
    ap.add_argument("--prefill-reps", type=int, default=100)
    ap.add_argument("--profile", choices=PROFILE_KERNELS, default=None,
                    help="launch only this kernel (--warmup + --steps times) on the --config "
                         "workload, for profiler captures; prints its mean time, no bench line")
    ap.add_argument("--num-seqs", type=int, default=0,
                    help="override the workload's batch size (small profiling captures)")
    ap.add_argument("--num-blocks", type=int, default=0,
                    help="override the workload's block pool size (small profiling captures)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    world, rank, local = dist_env()
    if world != args.gpus and world == 1 and args.gpus > 1:
        ap.error("--gpus N > 1 must be launched with torch.distributed.run (one rank per GPU)")
    if args.impl == "reference":
        run_reference(args, world, rank, local)
    elif args.profile:
        run_profile(args, local)
    elif args.only_prefill:
        import torch
        device = torch.device("cuda", local)
        torch.cuda.set_device(device)
        tp, tk = measured_tensor_peak()
        print(json.dumps(prefill_measure(device, args.warmup, reps=args.prefill_reps,
                                         peak_tflops=tp, peak_kind=tk, flush=L2Flush(device))))
    else:
        run_native(args, world, rank, local)


if __name__ == "__main__":
    main()
