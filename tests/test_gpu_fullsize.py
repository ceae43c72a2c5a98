"""The five decode workloads at full size, in the launch configuration the
benchmark times (GPU).  The oracle checks every output of a sample of
sequences (chosen to include the longest and shortest), computed from host
copies of those sequences' blocks taken before the GPU step; the cache write
is checked bit for bit on the sampled rows and, over the whole pool, by the
property that nothing but the mapped slots changed."""
import numpy as np
import pytest
import torch

import oracle as oracle_mod
from paged_kv_cache_444_b200 import decode_step, pa_check_error, workloads
from parity_helpers import TOL, bits, max_err, ocode, to_f64

pytestmark = pytest.mark.gpu


def _sample(batch, k):
    ctx = batch.context_lens.cpu()
    order = torch.argsort(ctx, descending=True).tolist()
    picks = [order[0], order[-1]] + [order[len(order) // 2]]
    picks += list(range(0, batch.cfg.num_seqs, max(1, batch.cfg.num_seqs // k)))[:k]
    return sorted(set(picks))[:max(k, 3)]


def _compact(batch, seqs):
    """Host snapshot of sequences `seqs` only: their blocks renumbered
    0..n-1 (a permutation of physical ids, which leaves the result unchanged)."""
    cfg = batch.cfg
    bs = cfg.block_size
    bt = batch.block_tables[seqs].cpu().numpy()
    ctx = batch.context_lens[seqs].cpu().numpy().astype(np.int32)
    used = sorted({int(bt[i, j]) for i in range(len(seqs))
                   for j in range((int(ctx[i]) + bs - 1) // bs)})
    remap = {b: n for n, b in enumerate(used)}
    bt_new = np.full_like(bt, -1)
    for i in range(len(seqs)):
        for j in range((int(ctx[i]) + bs - 1) // bs):
            bt_new[i, j] = remap[int(bt[i, j])]
    ids = torch.tensor(used, dtype=torch.long, device=batch.key_cache.device)
    slots = batch.slot_mapping[seqs].cpu().numpy()
    slots_new = np.array([remap[int(s) // bs] * bs + int(s) % bs if s >= 0 else -1
                          for s in slots], dtype=np.int64)
    return dict(kc=bits(batch.key_cache.index_select(0, ids)),
                vc=bits(batch.value_cache.index_select(0, ids)),
                bt=bt_new.astype(np.int32), ctx=ctx, q=bits(batch.query[seqs]),
                key=bits(batch.key[seqs]), value=bits(batch.value[seqs]), slots=slots_new,
                used=used)


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

    # oracle: its own write on the host snapshot, then attention
    kc, vc = snap["kc"].copy(), snap["vc"].copy()
    assert oracle_lib.reshape_and_cache(snap["key"], snap["value"], kc, vc, snap["slots"],
                                        len(snap["used"]), cfg.block_size) == oracle_mod.OK
    ref = oracle_lib.decode(snap["q"], kc, vc, snap["bt"], snap["ctx"], cfg.scale, ocode(cfg))
    err = max_err(out[seqs], ref)
    assert np.isfinite(to_f64(out)).all()
    assert err <= TOL[cfg.dtype], f"{name}: max-abs {err:.3e}"

    # write: sampled blocks bit-exact, and nothing else in the pool changed
    ids = torch.tensor(snap["used"], dtype=torch.long, device=cuda_device)
    assert np.array_equal(bits(batch.key_cache.index_select(0, ids)), kc)
    assert np.array_equal(bits(batch.value_cache.index_select(0, ids)), vc)
    flat_before = kc_before.view(-1, cfg.num_kv_heads, cfg.head_dim)
    flat_after = batch.key_cache.view(-1, cfg.num_kv_heads, cfg.head_dim)
    written = batch.slot_mapping[batch.slot_mapping >= 0]
    flat_before[written] = batch.key[batch.slot_mapping >= 0]
    assert torch.equal(flat_before, flat_after)
