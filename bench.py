#!/usr/bin/env python3
"""Benchmark of the paged decode step on B200: cache write + decode attention.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME]
    python bench.py --impl reference ...        # the fp64 CPU oracle, same workload

One step = the whole hot path over one seeded synthetic decode batch:
pa_reshape_and_cache (one new token per sequence), then pa_decode, or
pa_decode_split + pa_reduce for the long-context workload.  Inputs are
resident in HBM when the timed region starts; the K/V bytes each step reads
exceed the 126 MB L2, so no flush is needed between steps.  Multi-GPU runs
are independent replicas (one batch per GPU, no collective on the data
path); timing is the max over ranks of the CUDA-event time.

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

MAIN_CONFIG = "mha_llama2_7b"
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
# the step, with CUDA events around each kernel
# ---------------------------------------------------------------------------
class Step:
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

    def run(self, ev=None):
        """One step; ev = list of launches+1 CUDA events to record between kernels."""
        from paged_kv_cache_444_b200 import (pa_decode, pa_decode_split, pa_reduce,
                                             pa_reshape_and_cache)
        b, cfg = self.b, self.cfg
        if not ev:
            self.plan.run()   # validated once; the timed path
            return
        if ev:
            ev[0].record()
        pa_reshape_and_cache(b.key, b.value, b.key_cache, b.value_cache, b.slot_mapping)
        if ev:
            ev[1].record()
        if self.ps:
            w = self.ws
            pa_decode_split(w.tmp_out, w.max_logits, w.exp_sums, b.query, b.key_cache,
                            b.value_cache, b.block_tables, b.context_lens, cfg.scale, self.ps)
            if ev:
                ev[2].record()
            pa_reduce(self.out, w.tmp_out, w.max_logits, w.exp_sums, b.context_lens, self.ps)
            if ev:
                ev[3].record()
        else:
            pa_decode(self.out, b.query, b.key_cache, b.value_cache, b.block_tables,
                      b.context_lens, cfg.scale)
            if ev:
                ev[2].record()


def time_steps(step: Step, steps: int, warmup: int, world: int, device, clocks=None,
               kernel_steps: int = 200):
    """Warm up, then time `steps` steps back to back (CUDA events at the two
    ends only, so consecutive launches may overlap as they would in use), then
    time `kernel_steps` more with an event between every two kernels for the
    per-kernel durations.  Returns (ms per step, [ms per kernel])."""
    for _ in range(warmup):
        step.run()
    torch.cuda.synchronize()
    barrier(world, device)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ctx = clocks if clocks is not None else _Null()
    with ctx:
        torch.cuda.synchronize()
        start.record()
        for _ in range(steps):
            step.run()
        end.record()
        torch.cuda.synchronize()
    barrier(world, device)
    ms = start.elapsed_time(end) / steps
    ks = max(1, min(steps, kernel_steps))
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(step.launches + 1)]
           for _ in range(ks)]
    for k in range(ks):
        step.run(evs[k])
    torch.cuda.synchronize()
    per_kernel = [sum(e[i].elapsed_time(e[i + 1]) for e in evs) / ks
                  for i in range(step.launches)]
    return ms, per_kernel


def shared_prefix_kernel_ms(batch, warmup: int, reps: int = 100) -> float:
    """CUDA-event time of pa_decode_shared_prefix on a batch with prefix groups
    (the same attention as pa_decode, reading each shared page once per group)."""
    from paged_kv_cache_444_b200 import pa_decode_shared_prefix
    cfg = batch.cfg
    out = torch.empty_like(batch.query)
    sizes = (batch.group_starts[1:] - batch.group_starts[:-1]).tolist()

    def run():
        pa_decode_shared_prefix(out, batch.query, batch.key_cache, batch.value_cache,
                                batch.block_tables, batch.context_lens, batch.group_starts,
                                batch.prefix_blocks, cfg.scale, max(sizes))
    for _ in range(warmup):
        run()
    torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record()
    for _ in range(reps):
        run()
    end.record()
    torch.cuda.synchronize()
    return start.elapsed_time(end) / reps


def fp8_decode_ms(batch, warmup: int, reps: int = 100) -> float | None:
    """CUDA-event time of pa_decode_fp8 on the same batch with its caches held
    as E4M3 codes (x * 64 quantised by torch, scale 1/64); None where the
    fp8 path is not built (head_dim != 128) or the batch uses the split path."""
    from paged_kv_cache_444_b200 import pa_decode_fp8
    cfg = batch.cfg
    if cfg.head_dim != 128 or cfg.partition_size:
        return None
    q8 = lambda t: (t.float() * 64.0).clamp(-448, 448).to(torch.float8_e4m3fn).view(torch.uint8)
    kc, vc = q8(batch.key_cache), q8(batch.value_cache)
    out = torch.empty_like(batch.query)

    def run():
        pa_decode_fp8(out, batch.query, kc, vc, batch.block_tables, batch.context_lens,
                      cfg.scale, 1.0 / 64, 1.0 / 64)
    for _ in range(warmup):
        run()
    torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record()
    for _ in range(reps):
        run()
    end.record()
    torch.cuda.synchronize()
    del kc, vc
    return start.elapsed_time(end) / reps


def prefill_measure(device, warmup: int, reps: int = 20, peak_tflops: float = 0.0,
                    peak_kind: str = "") -> dict:
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
    for _ in range(warmup):
        run()
    torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record()
    for _ in range(reps):
        run()
    end.record()
    torch.cuda.synchronize()
    ms = start.elapsed_time(end) / reps
    ctx = b.context_lens.cpu().tolist()
    pairs = sum(sum(c - chunk + i + 1 for i in range(chunk)) for c in ctx)
    flops = 4 * cfg.head_dim * cfg.num_heads * pairs
    tf = flops / (ms / 1e3) / 1e12
    return {"workload": "chunked_prefill_gqa: 8 seqs x 512-token chunks at ctx U[512,4096], "
                        "32/8 heads, d=128, bf16", "kernel": "pa_prefill",
            "ms": round(ms, 5), "tflops": round(tf, 1),
            "query_tokens_per_s": round(T / (ms / 1e3), 1),
            "roofline": {"bound": "tensor", "achieved": round(tf, 1), "peak": peak_tflops,
                         "unit": "TFLOP/s", "frac": round(tf / peak_tflops, 4) if peak_tflops else None,
                         "peak_kind": peak_kind, "algorithmic_flops": flops}}


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


def e2e_steps(step: Step, steps: int, warmup: int, world: int, device):
    """The same step through the C ABI from host buffers (pa_decode_step_host):
    every step copies its inputs in from pinned host memory, writes the cache,
    attends, and copies the output back, all inside the timing."""
    from paged_kv_cache_444_b200 import HostStep
    b, cfg = step.b, step.cfg
    hs = HostStep(b.key_cache, b.value_cache, cfg.num_seqs, cfg.num_heads,
                  b.block_tables.shape[1], cfg.scale, step.ps, cfg.torch_dtype)
    for n in ("query", "key", "value", "slot_mapping", "block_tables", "context_lens"):
        getattr(hs, n).copy_(getattr(b, n).cpu())
    for _ in range(warmup):
        hs.run()
    torch.cuda.synchronize()
    barrier(world, device)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record()
    for _ in range(steps):
        hs.run()
    end.record()
    torch.cuda.synchronize()
    barrier(world, device)
    return start.elapsed_time(end) / steps, hs.h2d_bytes, hs.d2h_bytes


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
            "seconds": round(secs, 3),
            "sample": f"{len(seqs)} of {cfg.num_seqs} sequences of {cfg.name} "
                      f"({sum(sub_ctx)} context tokens, all {cfg.num_heads} heads): oracle "
                      f"cache write + fp64 decode, single thread"}


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

    def bench_config(name, steps, warmup, clocks=None):
        cfg = workloads.CONFIGS[name]
        cfg = cfg.scaled(seed=cfg.seed + 1000 * rank)
        if name == args.config and (args.num_seqs or args.num_blocks):
            # a smaller batch of the same workload (profiling captures only)
            cfg = cfg.scaled(num_seqs=args.num_seqs or cfg.num_seqs,
                             num_blocks=args.num_blocks or cfg.num_blocks,
                             name=f"{cfg.name}[seqs={args.num_seqs or cfg.num_seqs}]")
        batch = workloads.make_batch(cfg, device)
        step = Step(batch)
        ms, per_kernel = time_steps(step, steps, warmup, world, device, clocks)
        ms_max = max_over_ranks(ms, world, device)
        gms = graph_steps(step, steps, warmup) if args.graph else None
        shared_ms = shared_prefix_kernel_ms(batch, warmup) if batch.group_starts is not None \
            else None
        f8_ms = fp8_decode_ms(batch, warmup) if args.fp8 else None
        ctx = batch.context_lens.cpu().tolist()
        by = workloads.algorithmic_bytes(cfg, ctx)
        attn_ms = per_kernel[1] + (per_kernel[2] if step.ps else 0.0)
        kern_ms = per_kernel[1]
        kern_bytes = attention_kernel_bytes(cfg, ctx, bool(step.ps))
        total_bytes = sum_over_ranks(by["step"], world, device)
        res = {
            "ms_per_step": ms_max,
            "value": total_bytes / (ms_max / 1e3) / 1e9,
            "per_kernel_ms": per_kernel,
            "attention_ms": attn_ms,
            "attention_gbs": (by["attention"]) / (attn_ms / 1e3) / 1e9,
            "kernel_gbs": kern_bytes / (kern_ms / 1e3) / 1e9,
            "kernel_bytes": kern_bytes,
            "bytes": by,
            "tokens_per_s": sum_over_ranks(cfg.num_seqs, world, device) / (ms_max / 1e3),
            "graph_ms_per_step": gms,
            "shared_prefix_kernel_ms": shared_ms,
            "unique_kv_bytes": (workloads.unique_kv_bytes(cfg, batch.block_tables.cpu().tolist(),
                                                          batch.context_lens.cpu().tolist())
                                if shared_ms else None),
            "fp8_ms": f8_ms,
            "kernel": "pa_decode_split" if step.ps else "pa_decode",
            "context_tokens": int(sum(ctx)),
        }
        return cfg, batch, step, res

    results = {}
    clocks = ClockSampler(local)
    cfg, batch, step, main = bench_config(args.config, args.steps, args.warmup, clocks)
    e2e_ms, h2d, d2h = e2e_steps(step, max(3, args.steps // 4), args.warmup, world, device)
    e2e_ms = max_over_ranks(e2e_ms, world, device)
    total_bytes = sum_over_ranks(main["bytes"]["step"], world, device)
    ctx_main = batch.context_lens.cpu().tolist()
    bt_main = batch.block_tables.cpu().tolist()

    if not args.only_main:
        for name in workloads.CONFIG_ORDER:
            if name == args.config:
                results[name] = main
                continue
            _, b2, s2, r = bench_config(name, args.config_steps, args.warmup)
            results[name] = r
            del b2, s2
            torch.cuda.empty_cache()

    kname = "pa_decode_split" if step.ps else "pa_decode"
    roof = {"bound": "hbm", "kernel": kname,
            "achieved": round(main["kernel_gbs"], 1), "peak": peak, "unit": "GB/s",
            "frac": round(main["kernel_gbs"] / peak, 4), "peak_kind": peak_kind,
            "algorithmic_bytes_per_launch": main["kernel_bytes"],
            "traffic": None}
    roof["traffic"] = recorded_traffic(args.config, kname, sum(ctx_main))

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
                   "l2": "inputs larger than L2 (K/V read per step >> 126 MB), no flush",
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU"},
        "decode_tokens_per_s": round(main["tokens_per_s"], 1),
        "graph_ms_per_step": (round(main["graph_ms_per_step"], 5)
                              if main["graph_ms_per_step"] else None),
        "attention_gbs": round(main["attention_gbs"], 1),
        "per_kernel_ms": {n: round(v, 5) for n, v in zip(
            ["pa_reshape_and_cache", kname] + (["pa_reduce"] if step.ps else []),
            main["per_kernel_ms"])},
        "roofline": roof,
        "gpu_launches": step.launches * args.steps,
        "e2e": {"value": round(total_bytes / (e2e_ms / 1e3) / 1e9, 2), "unit": "GB/s",
                "ms_per_step": round(e2e_ms, 5), "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h,
                "api": "pa_decode_step_host (C ABI, pinned host buffers in and out)",
                "host_cpus": host_cpus},
        "clocks": clocks.summary(),
    }
    if results:
        line["per_config"] = {
            n: {"ms_per_step": round(r["ms_per_step"], 5), "step_gbs": round(r["value"], 1),
                "attention_gbs": round(r["attention_gbs"], 1),
                "kernel_gbs": round(r["kernel_gbs"], 1),
                "kernel_frac_of_peak": round(r["kernel_gbs"] / peak, 4),
                "kernel_traffic": recorded_traffic(n, r["kernel"], r["context_tokens"]),
                "kernel_algorithmic_bytes": r["kernel_bytes"],
                "attention_frac_of_peak": round(r["attention_gbs"] / peak, 4),
                "decode_tokens_per_s": round(r["tokens_per_s"], 1),
                "graph_ms_per_step": (round(r["graph_ms_per_step"], 5)
                                      if r["graph_ms_per_step"] else None),
                "per_kernel_ms": [round(x, 5) for x in r["per_kernel_ms"]],
                **({"pa_decode_shared_prefix_ms": round(r["shared_prefix_kernel_ms"], 5),
                    # the shared-prefix kernel reads each shared page once:
                    # its rate on the unique K/V bytes, against the copy peak
                    "pa_decode_shared_prefix_unique_gbs": round(
                        r["unique_kv_bytes"] / (r["shared_prefix_kernel_ms"] / 1e3) / 1e9, 1),
                    "pa_decode_shared_prefix_unique_frac_of_peak": round(
                        r["unique_kv_bytes"] / (r["shared_prefix_kernel_ms"] / 1e3) / 1e9 / peak,
                        4)}
                   if r["shared_prefix_kernel_ms"] else {}),
                **(fp8_entry(r, peak) if r["fp8_ms"] else {})}
            for n, r in results.items()}
    if args.prefill and not args.only_main:
        tp, tk = measured_tensor_peak()
        line["prefill"] = prefill_measure(device, args.warmup, reps=args.prefill_reps,
                                          peak_tflops=tp, peak_kind=tk)
    if world == 1 and rank == 0 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(cfg, ctx_main, bt_main, batch,
                                            budget_s=args.cpu_budget)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def fp8_entry(r: dict, peak: float) -> dict:
    """pa_decode_fp8 on the same batch: time, algorithmic GB/s (K/V at one
    byte per element) and the speed-up over the 16-bit decode kernel."""
    by = r["bytes"]
    fp8_bytes = by["kv"] // 2 + by["block_table"] + by["query"] + by["out"] + by["context_lens"]
    gbs = fp8_bytes / (r["fp8_ms"] / 1e3) / 1e9
    return {"pa_decode_fp8": {"ms": round(r["fp8_ms"], 5), "gbs": round(gbs, 1),
                              "frac_of_peak": round(gbs / peak, 4),
                              "speedup_vs_16bit_kernel": round(r["per_kernel_ms"][1] /
                                                               r["fp8_ms"], 3)}}


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
    """Hash of the decode path's sources: every csrc file but those off the
    path, with the marked host-side regions of pa_api.cu that serve other
    kernels ("// >>> ..." to "// <<< ...") left out."""
    import hashlib
    import re
    h = hashlib.sha256()
    for p in sorted((csrc or ROOT / "paged_kv_cache_444_b200" / "csrc").glob("*")):
        if p.name in OFF_DECODE_PATH:
            continue
        data = p.read_bytes()
        if p.name == "pa_api.cu":
            data = re.sub(rb"\n// >>> .*?\n// <<< [^\n]*", b"", data, flags=re.S)
        h.update(data)
    return h.hexdigest()[:16]


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
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["native", "reference"], default="native")
    ap.add_argument("--config", default=MAIN_CONFIG, choices=list(workloads.CONFIGS))
    ap.add_argument("--config-steps", type=int, default=300,
                    help="timed steps for each of the other workloads")
    ap.add_argument("--only-main", action="store_true", help="skip the per-workload table")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=12.0,
                    help="seconds of oracle work for the CPU baseline")
    ap.add_argument("--graph", action=argparse.BooleanOptionalAction, default=True,
                    help="also time the step replayed from a CUDA graph")
    ap.add_argument("--fp8", action=argparse.BooleanOptionalAction, default=True,
                    help="also time pa_decode_fp8 on each batch (E4M3 copy of its caches)")
    ap.add_argument("--prefill", action=argparse.BooleanOptionalAction, default=True,
                    help="also time pa_prefill on a chunked-prefill GQA layer")
    ap.add_argument("--only-prefill", action="store_true",
                    help="time only pa_prefill (its own JSON object; for profiling captures)")
    ap.add_argument("--prefill-reps", type=int, default=20)
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
    elif args.only_prefill:
        import torch
        device = torch.device("cuda", local)
        torch.cuda.set_device(device)
        tp, tk = measured_tensor_peak()
        print(json.dumps(prefill_measure(device, args.warmup, reps=args.prefill_reps,
                                         peak_tflops=tp, peak_kind=tk)))
    else:
        run_native(args, world, rank, local)


if __name__ == "__main__":
    main()
