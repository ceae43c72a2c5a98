"""The seeded input generators (CPU): the index structure every parity test and
the benchmark draw from.  Checked for each of the five workloads without
allocating their caches: context lengths inside the recipe's range, block
tables that hand each sequence distinct in-range physical blocks (members of
a sharing group share exactly their group's prefix ids), and the written
slot at each sequence's newest position."""
import numpy as np
import pytest
import torch

from paged_kv_cache_444_b200 import workloads

C = workloads.CONFIGS


def _index_structure(cfg):
    gen = torch.Generator(device="cpu")
    gen.manual_seed(cfg.seed)
    ctx = workloads.draw_context_lens(cfg, gen)
    bt = workloads.build_block_tables(cfg, ctx, gen)
    slots = workloads.slot_of_last_token(bt, ctx, cfg.block_size)
    return ctx.numpy(), bt.numpy(), slots.numpy()


@pytest.mark.parametrize("name", workloads.CONFIG_ORDER)
def test_context_lengths_follow_the_recipe(name):
    cfg = C[name]
    ctx, _, _ = _index_structure(cfg)
    assert ctx.shape == (cfg.num_seqs,) and ctx.dtype == np.int32
    kind = cfg.ctx[0]
    if kind == "fixed":
        assert ctx.tolist() == list(cfg.ctx[1])
    elif kind == "uniform":
        assert ctx.min() >= cfg.ctx[1] and ctx.max() <= cfg.ctx[2]
    else:  # lognormal, clamped
        assert ctx.min() >= cfg.ctx[3] and ctx.max() <= cfg.ctx[4]


@pytest.mark.parametrize("name", workloads.CONFIG_ORDER)
def test_block_tables_are_distinct_in_range_blocks(name):
    cfg = C[name]
    ctx, bt, _ = _index_structure(cfg)
    need = (ctx.astype(np.int64) + cfg.block_size - 1) // cfg.block_size
    owner = {}
    for s in range(cfg.num_seqs):
        row = bt[s]
        used = row[:need[s]]
        assert (used >= 0).all() and (used < cfg.num_blocks).all()
        assert (row[max(need[s], cfg.shared_prefix_blocks):] == -1).all()
        shared = cfg.shared_prefix_blocks
        for i, b in enumerate(used.tolist()):
            key = ("prefix", s // cfg.share_group, i) if i < shared else ("own", s, i)
            assert owner.setdefault(b, key) == key, f"block {b} handed out twice"


def test_shared_prefix_groups_share_exactly_their_prefix():
    cfg = C["shared_prefix_beam"]
    _, bt, _ = _index_structure(cfg)
    p = cfg.shared_prefix_blocks
    for g in range(0, cfg.num_seqs, cfg.share_group):
        members = bt[g:g + cfg.share_group]
        assert (members[:, :p] == members[0, :p]).all()
        if g + cfg.share_group < cfg.num_seqs:
            assert not set(members[0, :p].tolist()) & set(bt[g + cfg.share_group, :p].tolist())


@pytest.mark.parametrize("name", workloads.CONFIG_ORDER)
def test_written_slot_is_the_newest_position(name, oracle_lib):
    """The generator's slot of position ctx-1 equals the oracle's slot (whose
    arithmetic is pinned to the pages' worked example of tokens 1..9)."""
    cfg = C[name]
    ctx, bt, slots = _index_structure(cfg)
    for s in range(cfg.num_seqs):
        pos = int(ctx[s]) - 1
        assert slots[s] == oracle_lib.slot(np.ascontiguousarray(bt[s]), pos, cfg.block_size)


def test_batches_are_reproducible_bit_for_bit():
    a = workloads.make_batch(C["tiny"])
    b = workloads.make_batch(C["tiny"])
    for n in ("context_lens", "block_tables", "slot_mapping", "key_cache", "value_cache",
              "query", "key", "value"):
        assert torch.equal(getattr(a, n), getattr(b, n)), n


def test_algorithmic_bytes_of_the_tiny_batch():
    """Counted by hand for the tiny batch (4 sequences, contexts 1, 9, 16, 37,
    4/4 heads, d = 64, fp16): K+V 2*(63 tokens*4 heads*64*2 B), block-table
    entries 1+1+1+3 ints, q and out 4*4*64*2 B each, 4 context lengths."""
    cfg = C["tiny"]
    a = workloads.algorithmic_bytes(cfg, [1, 9, 16, 37])
    assert a["kv"] == 2 * 63 * 4 * 64 * 2
    assert a["block_table"] == 6 * 4
    assert a["query"] == a["out"] == 4 * 4 * 64 * 2
    assert a["context_lens"] == 16
    assert a["attention"] == 64512 + 24 + 2048 + 2048 + 16
