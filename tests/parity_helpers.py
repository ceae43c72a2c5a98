"""Shared plumbing of the GPU parity tests: move a seeded batch between the
CUDA path (through the C-ABI binding) and the fp64 oracle (on host copies
taken BEFORE the GPU touches anything).  No attention arithmetic here."""
from __future__ import annotations

import numpy as np
import torch

import oracle as oracle_mod
from paged_kv_cache_444_b200 import workloads

TOL = {"f16": 2e-3, "bf16": 8e-3}   # max-abs vs the fp64 oracle


def bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def ocode(cfg: workloads.DecodeConfig) -> int:
    return oracle_mod.BF16 if cfg.dtype == "bf16" else oracle_mod.F16


class HostCopy:
    """Host snapshot of a batch (16-bit data as uint16 bits)."""

    def __init__(self, batch: workloads.DecodeBatch):
        self.cfg = batch.cfg
        self.context_lens = batch.context_lens.cpu().numpy().astype(np.int32)
        self.block_tables = batch.block_tables.cpu().numpy().astype(np.int32)
        self.slot_mapping = batch.slot_mapping.cpu().numpy().astype(np.int64)
        self.key_cache = bits(batch.key_cache)
        self.value_cache = bits(batch.value_cache)
        self.query = bits(batch.query)
        self.key = bits(batch.key)
        self.value = bits(batch.value)


def oracle_step(orc, host: HostCopy, write: bool = True):
    """Oracle cache write (on copies) then oracle decode; returns
    (out float64 [S,H,D], key_cache_after, value_cache_after)."""
    cfg = host.cfg
    kc = host.key_cache.copy()
    vc = host.value_cache.copy()
    if write:
        rc = orc.reshape_and_cache(host.key, host.value, kc, vc, host.slot_mapping,
                                   cfg.num_blocks, cfg.block_size)
        assert rc == oracle_mod.OK
    out = orc.decode(host.query, kc, vc, host.block_tables, host.context_lens, cfg.scale,
                     ocode(cfg))
    return out, kc, vc


def gpu_step(batch: workloads.DecodeBatch, write: bool = True, partition_size: int = 0,
             max_partitions: int | None = None, shared_prefix: bool = False,
             max_group_size: int | None = None):
    """The CUDA path: pa_reshape_and_cache, then pa_decode, pa_decode_split +
    pa_reduce, or pa_decode_shared_prefix.  Returns (out, partials or None)."""
    from paged_kv_cache_444_b200 import (SplitWorkspace, pa_decode, pa_decode_shared_prefix,
                                         pa_decode_split, pa_reduce, pa_reshape_and_cache)
    cfg = batch.cfg
    if write:
        pa_reshape_and_cache(batch.key, batch.value, batch.key_cache, batch.value_cache,
                             batch.slot_mapping)
    out = torch.full_like(batch.query, float("nan"))
    parts = None
    if shared_prefix:
        sizes = (batch.group_starts[1:] - batch.group_starts[:-1]).tolist()
        pa_decode_shared_prefix(out, batch.query, batch.key_cache, batch.value_cache,
                                batch.block_tables, batch.context_lens, batch.group_starts,
                                batch.prefix_blocks, cfg.scale, max_group_size or max(sizes))
    elif partition_size:
        P = max_partitions or (batch.block_tables.shape[1] * cfg.block_size + partition_size - 1) \
            // partition_size
        ws = SplitWorkspace(cfg.num_seqs, cfg.num_heads, cfg.head_dim, P, batch.query.device)
        ws.tmp_out.fill_(float("nan"))
        ws.max_logits.fill_(float("nan"))
        ws.exp_sums.fill_(float("nan"))
        pa_decode_split(ws.tmp_out, ws.max_logits, ws.exp_sums, batch.query,
                        batch.key_cache, batch.value_cache, batch.block_tables,
                        batch.context_lens, cfg.scale, partition_size)
        pa_reduce(out, ws.tmp_out, ws.max_logits, ws.exp_sums, batch.context_lens,
                  partition_size)
        parts = ws
    else:
        pa_decode(out, batch.query, batch.key_cache, batch.value_cache, batch.block_tables,
                  batch.context_lens, cfg.scale)
    torch.cuda.synchronize()
    return out, parts


def poison_past_context(batch: workloads.DecodeBatch, key_cache=None, value_cache=None,
                        fill=float("nan")) -> int:
    """Fill the cache rows past each sequence's context in its last block with
    `fill` (NaN, or an E4M3 NaN code for fp8 caches).  Those rows were never
    written: the oracle never reads them, and the kernels must not let a
    probability of 0 times a NaN reach the output.  Returns the rows filled."""
    cfg = batch.cfg
    kc = batch.key_cache if key_cache is None else key_cache
    vc = batch.value_cache if value_cache is None else value_cache
    bt = batch.block_tables.cpu().numpy()
    n = 0
    for s, c in enumerate(batch.context_lens.cpu().tolist()):
        if c % cfg.block_size:
            blk = int(bt[s, (c - 1) // cfg.block_size])
            kc[blk, c % cfg.block_size:] = fill
            vc[blk, c % cfg.block_size:] = fill
            n += cfg.block_size - c % cfg.block_size
    return n


def to_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def max_err(gpu_out: torch.Tensor, ref: np.ndarray) -> float:
    return float(np.max(np.abs(to_f64(gpu_out) - ref))) if ref.size else 0.0


# (workload, kernel, max|gpu - oracle|, max|gpu - round_to_dtype(oracle)|, tolerance)
# of the full-size checks, printed in pytest's terminal summary and, when
# PA_PARITY_REPORT names a file, written there as JSON lines.
PARITY_REPORT: list[dict] = []


def report_parity(orc, workload: str, kernel: str, gpu_out: torch.Tensor, ref: np.ndarray,
                  dtype_code: int, tol: float) -> float:
    """Record the error of gpu_out against the fp64 oracle and against the
    oracle rounded to the output dtype (nearest even); returns the first."""
    import json
    import os
    g = to_f64(gpu_out)
    err = float(np.max(np.abs(g - ref))) if ref.size else 0.0
    rounded = orc.decode_bits(orc.round_to_dtype(ref, dtype_code), dtype_code)
    err_r = float(np.max(np.abs(g - rounded))) if ref.size else 0.0
    row = {"workload": workload, "kernel": kernel, "max_abs_vs_oracle": err,
           "max_abs_vs_rounded_oracle": err_r, "tolerance": tol, "outputs": int(ref.size)}
    PARITY_REPORT.append(row)
    path = os.environ.get("PA_PARITY_REPORT")
    if path:
        with open(path, "a", encoding="utf-8") as f:
            f.write(json.dumps(row) + "\n")
    return err


# E4M3 caches for the fp8 tests: one scale per cache tensor
K_SCALE, V_SCALE = 1.0 / 64, 1.0 / 32


def grow_logits(batch: workloads.DecodeBatch, step: float = 7.0, every: int = 64,
                max_steps: int = 1 << 30) -> float:
    """Rewrite the key cache so that, for every sequence and KV head, the
    logit of the group's first query head climbs by about `step` (natural
    units; 7 is 10 log2 units) every `every` tokens: key row j becomes a
    quarter of its random self plus c_j times that query's unit vector, with
    c_j * |q| * scale = step * min(j // every, max_steps) (a cap keeps E4M3
    codes of the rows below saturation).  The running maximum then jumps
    past any slack of 2^8 several times along each sequence.  A block that
    several sequences share keeps the last one's rewrite (the cache stays one
    consistent input for both sides).  Returns the largest climb (natural
    units) planned for one (sequence, head)."""
    cfg = batch.cfg
    G = cfg.num_heads // cfg.num_kv_heads
    kc = batch.key_cache.float()
    bt = batch.block_tables.cpu()
    cl = batch.context_lens.cpu().tolist()
    dev = kc.device
    top = 0.0
    for s, n in enumerate(cl):
        if n <= 0:
            continue
        j = torch.arange(n)
        blocks = bt[s, j // cfg.block_size].to(dev)
        rows = (j % cfg.block_size).to(dev)
        for h in range(cfg.num_kv_heads):
            q = batch.query[s, h * G].float()
            qn = float(q.norm())
            if qn == 0.0:
                continue
            k = torch.clamp(j // every, max=max_steps).to(torch.float32)
            c = (step * k / (qn * cfg.scale)).to(dev)
            kc[blocks, rows, h] = 0.25 * kc[blocks, rows, h] + c[:, None] * (q / qn)[None, :]
            top = max(top, step * min((n - 1) // every, max_steps))
    batch.key_cache.copy_(kc.to(batch.key_cache.dtype))
    return top


def fp8_batch(cfg: workloads.DecodeConfig, dev, prepare=None):
    """A seeded batch whose caches are also held as E4M3 codes (torch's
    float8_e4m3fn cast of x / scale, saturated to +-448).  `prepare(batch)`,
    if given, edits the 16-bit batch before the codes are taken."""
    b = workloads.make_batch(cfg, dev)
    if prepare is not None:
        prepare(b)
    q8 = lambda t, s: (t.float() * (1.0 / s)).clamp(-448, 448).to(torch.float8_e4m3fn) \
        .view(torch.uint8)
    kc = q8(b.key_cache, K_SCALE).contiguous()
    vc = q8(b.value_cache, V_SCALE).contiguous()
    return b, kc, vc


def fp8_oracle(orc, b: workloads.DecodeBatch, kc: torch.Tensor, vc: torch.Tensor):
    """Oracle quantising write (on host copies of the E4M3 caches) then the
    oracle's fp8 decode; returns (out float64, key codes after, value codes after)."""
    cfg = b.cfg
    kh = kc.cpu().numpy().copy()
    vh = vc.cpu().numpy().copy()
    assert orc.reshape_and_cache_fp8(bits(b.key), bits(b.value), kh, vh,
                                     b.slot_mapping.cpu().numpy(), cfg.num_blocks,
                                     cfg.block_size, K_SCALE, V_SCALE, ocode(cfg)) == 0
    ref = orc.decode_fp8(bits(b.query), kh, vh, b.block_tables.cpu().numpy(),
                         b.context_lens.cpu().numpy(), cfg.scale, K_SCALE, V_SCALE, ocode(cfg))
    return ref, kh, vh
