"""The five decode workloads at full size, in the launch configurations the
benchmark times (GPU): the step (cache write + pa_decode, or pa_decode_split
+ pa_reduce), pa_decode_shared_prefix on the beam batch with the groups the
benchmark passes, and pa_decode_fp8 / pa_decode_split_fp8 on the E4M3 copies
of the caches the benchmark makes.

The oracle checks every output of a sample of sequences (chosen to include
the longest and shortest), computed from host copies of those sequences'
blocks taken before the GPU step; the cache write is checked bit for bit on
the sampled rows and, over the whole pool, by the property that nothing but
the mapped slots changed.  Each check records its error against the oracle
and against the oracle rounded to the output dtype (terminal summary)."""
import numpy as np
import pytest
import torch

import oracle as oracle_mod
from paged_kv_cache_444_b200 import (SplitWorkspace, decode_step, pa_check_error, pa_decode_fp8,
                                     pa_decode_shared_prefix, pa_decode_split_fp8, pa_reduce,
                                     pa_reshape_and_cache, workloads)
from parity_helpers import TOL, bits, ocode, report_parity, to_f64

pytestmark = pytest.mark.gpu

# the benchmark's fp8 copies of a cache: x * 64 quantised by torch, scale 1/64
FP8_SCALE = 1.0 / 64


def _fp8(t):
    return (t.float() * (1.0 / FP8_SCALE)).clamp(-448, 448).to(torch.float8_e4m3fn) \
        .view(torch.uint8).contiguous()


def _sample(batch, k):
    ctx = batch.context_lens.cpu()
    order = torch.argsort(ctx, descending=True).tolist()
    picks = [order[0], order[-1]] + [order[len(order) // 2]]
    picks += list(range(0, batch.cfg.num_seqs, max(1, batch.cfg.num_seqs // k)))[:k]
    return sorted(set(picks))[:max(k, 3)]


def _compact(batch, seqs, key_cache=None, value_cache=None):
    """Host snapshot of sequences `seqs` only: their blocks renumbered
    0..n-1 (a permutation of physical ids, which leaves the result unchanged).
    Caches default to the batch's 16-bit ones (as uint16 bits); fp8 caches
    are passed as uint8 tensors and copied as they are."""
    cfg = batch.cfg
    bs = cfg.block_size
    kc_src = batch.key_cache if key_cache is None else key_cache
    vc_src = batch.value_cache if value_cache is None else value_cache
    host = (lambda t: t.cpu().numpy().copy()) if kc_src.dtype == torch.uint8 else bits
    bt = batch.block_tables[seqs].cpu().numpy()
    ctx = batch.context_lens[seqs].cpu().numpy().astype(np.int32)
    used = sorted({int(bt[i, j]) for i in range(len(seqs))
                   for j in range((int(ctx[i]) + bs - 1) // bs)})
    remap = {b: n for n, b in enumerate(used)}
    bt_new = np.full_like(bt, -1)
    for i in range(len(seqs)):
        for j in range((int(ctx[i]) + bs - 1) // bs):
            bt_new[i, j] = remap[int(bt[i, j])]
    ids = torch.tensor(used, dtype=torch.long, device=kc_src.device)
    slots = batch.slot_mapping[seqs].cpu().numpy()
    slots_new = np.array([remap[int(s) // bs] * bs + int(s) % bs if s >= 0 else -1
                          for s in slots], dtype=np.int64)
    return dict(kc=host(kc_src.index_select(0, ids)), vc=host(vc_src.index_select(0, ids)),
                bt=bt_new.astype(np.int32), ctx=ctx, q=bits(batch.query[seqs]),
                key=bits(batch.key[seqs]), value=bits(batch.value[seqs]), slots=slots_new,
                used=used, ids=ids)


def _oracle_written(orc, cfg, snap):
    """The oracle's own cache write on the snapshot, then its decode."""
    kc, vc = snap["kc"].copy(), snap["vc"].copy()
    assert orc.reshape_and_cache(snap["key"], snap["value"], kc, vc, snap["slots"],
                                 len(snap["used"]), cfg.block_size) == oracle_mod.OK
    ref = orc.decode(snap["q"], kc, vc, snap["bt"], snap["ctx"], cfg.scale, ocode(cfg))
    return ref, kc, vc


@pytest.mark.parametrize("name", workloads.CONFIG_ORDER)
def test_full_size_workload(name, cuda_device, oracle_lib):
    cfg = workloads.CONFIGS[name]
    batch = workloads.make_batch(cfg, cuda_device)
    seqs = _sample(batch, 2 if name == "long_context_split" else 4)
    snap = _compact(batch, seqs)
    kc_before = batch.key_cache.clone()

    out = decode_step(batch.query, batch.key, batch.value, batch.key_cache, batch.value_cache,
                      batch.slot_mapping, batch.block_tables, batch.context_lens, cfg.scale,
                      partition_size=cfg.partition_size)
    torch.cuda.synchronize()
    pa_check_error()

    ref, kc, vc = _oracle_written(oracle_lib, cfg, snap)
    assert np.isfinite(to_f64(out)).all()
    kernel = "pa_decode_split+pa_reduce" if cfg.partition_size else "pa_decode"
    err = report_parity(oracle_lib, name, kernel, out[seqs], ref, ocode(cfg), TOL[cfg.dtype])
    assert err <= TOL[cfg.dtype], f"{name}: max-abs {err:.3e}"

    # write: sampled blocks bit-exact, and nothing else in the pool changed
    ids = snap["ids"]
    assert np.array_equal(bits(batch.key_cache.index_select(0, ids)), kc)
    assert np.array_equal(bits(batch.value_cache.index_select(0, ids)), vc)
    flat_before = kc_before.view(-1, cfg.num_kv_heads, cfg.head_dim)
    flat_after = batch.key_cache.view(-1, cfg.num_kv_heads, cfg.head_dim)
    written = batch.slot_mapping[batch.slot_mapping >= 0]
    flat_before[written] = batch.key[batch.slot_mapping >= 0]
    assert torch.equal(flat_before, flat_after)


def test_full_size_shared_prefix_beam(cuda_device, oracle_lib):
    """pa_decode_shared_prefix on the full beam batch (64 sequences in groups
    of 4 sharing 32 blocks), with the group arrays and max group size the
    benchmark passes, after the step's cache write."""
    cfg = workloads.CONFIGS["shared_prefix_beam"]
    batch = workloads.make_batch(cfg, cuda_device)
    # two whole groups (members share their prefix) plus the longest and shortest
    seqs = sorted(set(_sample(batch, 4)) | {0, 1, 2, 3, 60, 61, 62, 63})
    snap = _compact(batch, seqs)
    pa_reshape_and_cache(batch.key, batch.value, batch.key_cache, batch.value_cache,
                         batch.slot_mapping)
    sizes = (batch.group_starts[1:] - batch.group_starts[:-1]).tolist()
    out = torch.full_like(batch.query, float("nan"))
    pa_decode_shared_prefix(out, batch.query, batch.key_cache, batch.value_cache,
                            batch.block_tables, batch.context_lens, batch.group_starts,
                            batch.prefix_blocks, cfg.scale, max(sizes))
    kernel = "pa_decode_shared_prefix"
    torch.cuda.synchronize()
    pa_check_error()
    ref, _, _ = _oracle_written(oracle_lib, cfg, snap)
    assert np.isfinite(to_f64(out)).all()
    err = report_parity(oracle_lib, cfg.name, kernel, out[seqs], ref, ocode(cfg),
                        TOL[cfg.dtype])
    assert err <= TOL[cfg.dtype], f"max-abs {err:.3e}"


@pytest.mark.parametrize("name,ps", [("mha_llama2_7b", 0), ("gqa_llama3_8b", 0),
                                     ("shared_prefix_beam", 0), ("shared_prefix_beam", 512),
                                     ("long_context_split", 512)])
def test_full_size_fp8(name, ps, cuda_device, oracle_lib):
    """pa_decode_fp8, or pa_decode_split_fp8 + pa_reduce with 512-token
    partitions, on the E4M3 copies of the full-size caches the benchmark
    times, after the step's 16-bit write."""
    cfg = workloads.CONFIGS[name]
    batch = workloads.make_batch(cfg, cuda_device)
    pa_reshape_and_cache(batch.key, batch.value, batch.key_cache, batch.value_cache,
                         batch.slot_mapping)
    kc8, vc8 = _fp8(batch.key_cache), _fp8(batch.value_cache)
    seqs = _sample(batch, 2 if cfg.partition_size else 4)
    snap = _compact(batch, seqs, kc8, vc8)
    out = torch.full_like(batch.query, float("nan"))
    if ps:
        ws = SplitWorkspace(cfg.num_seqs, cfg.num_heads, cfg.head_dim,
                            (batch.block_tables.shape[1] * cfg.block_size + ps - 1) // ps,
                            cuda_device)
        pa_decode_split_fp8(ws.tmp_out, ws.max_logits, ws.exp_sums, batch.query, kc8, vc8,
                            batch.block_tables, batch.context_lens, cfg.scale, FP8_SCALE,
                            FP8_SCALE, ps)
        pa_reduce(out, ws.tmp_out, ws.max_logits, ws.exp_sums, batch.context_lens, ps)
        kernel = "pa_decode_split_fp8+pa_reduce"
    else:
        pa_decode_fp8(out, batch.query, kc8, vc8, batch.block_tables, batch.context_lens,
                      cfg.scale, FP8_SCALE, FP8_SCALE)
        kernel = "pa_decode_fp8"
    torch.cuda.synchronize()
    pa_check_error()
    ref = oracle_lib.decode_fp8(snap["q"], snap["kc"], snap["vc"], snap["bt"], snap["ctx"],
                                cfg.scale, FP8_SCALE, FP8_SCALE, ocode(cfg))
    assert np.isfinite(to_f64(out)).all()
    err = report_parity(oracle_lib, name, kernel, out[seqs], ref, ocode(cfg), TOL[cfg.dtype])
    assert err <= TOL[cfg.dtype], f"{name} fp8: max-abs {err:.3e}"
