"""CUDA path vs the fp64 oracle, element by element, on seeded batches small
enough for the oracle to finish in seconds but spanning many pages, warps and
ragged tails (GPU).  Tolerances: max-abs 2e-3 (fp16), 8e-3 (bf16); the cache
write is compared bit for bit over the whole buffer."""
import numpy as np
import pytest
import torch

from paged_kv_cache_444_b200 import PagedAttentionError, pa_check_error, workloads
from parity_helpers import (TOL, HostCopy, bits, gpu_step, grow_logits, max_err, oracle_step,
                            poison_past_context, to_f64)

pytestmark = pytest.mark.gpu

C = workloads.CONFIGS

# Scaled-down versions of the five workloads (same dtype / head layout).
SMALL = {
    "tiny": C["tiny"],
    "mha_small": C["mha_llama2_7b"].scaled(name="mha_small", num_seqs=6, num_heads=8,
                                             num_kv_heads=8, num_blocks=256,
                                             ctx=("uniform", 1, 300), seed=11),
    "gqa_small": C["gqa_llama3_8b"].scaled(name="gqa_small", num_seqs=8, num_heads=32,
                                             num_kv_heads=8, num_blocks=512,
                                             ctx=("uniform", 1, 700), seed=12),
    "long_small": C["long_context_split"].scaled(name="long_small", num_seqs=2, num_heads=8,
                                                   num_kv_heads=2, num_blocks=512,
                                                   ctx=("uniform", 1500, 3000), seed=13),
    "shared_small": C["shared_prefix_beam"].scaled(name="shared_small", num_seqs=8,
                                                     num_heads=8, num_kv_heads=2,
                                                     num_blocks=256, shared_prefix_blocks=4,
                                                     ctx=("lognormal", 150.0, 0.6, 65, 400),
                                                     seed=14),
    # other head layouts the kernels are built for
    "d64_gqa2": C["tiny"].scaled(name="d64_gqa2", num_seqs=5, num_heads=8, num_kv_heads=4,
                                 dtype="bf16", num_blocks=128, ctx=("uniform", 1, 200), seed=15),
    "gqa3_f16": C["gqa_llama3_8b"].scaled(name="gqa3_f16", num_seqs=4, num_heads=12,
                                            num_kv_heads=4, dtype="f16", num_blocks=128,
                                            ctx=("uniform", 1, 300), seed=16),
    "gqa8": C["gqa_llama3_8b"].scaled(name="gqa8", num_seqs=3, num_heads=16, num_kv_heads=2,
                                        num_blocks=128, ctx=("uniform", 30, 400), seed=17),
    "gqa16_two_rows": C["gqa_llama3_8b"].scaled(name="gqa16_two_rows", num_seqs=3,
                                                  num_heads=32, num_kv_heads=2, num_blocks=128,
                                                  ctx=("uniform", 30, 400), seed=18),
    "gqa16_d64_f16": C["tiny"].scaled(name="gqa16_d64_f16", num_seqs=3, num_heads=32,
                                        num_kv_heads=2, num_blocks=128,
                                        ctx=("uniform", 1, 300), seed=19),
    "mha_bf16": C["mha_llama2_7b"].scaled(name="mha_bf16", num_seqs=4, num_heads=4,
                                            num_kv_heads=4, dtype="bf16", num_blocks=128,
                                            ctx=("uniform", 1, 400), seed=20),
}


@pytest.fixture(scope="module")
def dev(cuda_device):
    from paged_kv_cache_444_b200 import load
    load()
    return cuda_device


def _check_close(gpu_out, ref, cfg, what):
    err = max_err(gpu_out, ref)
    assert np.isfinite(to_f64(gpu_out)).all(), f"{what}: non-finite output"
    assert err <= TOL[cfg.dtype], f"{what}: max-abs error {err:.3e} > {TOL[cfg.dtype]}"
    return err


@pytest.mark.parametrize("name", list(SMALL))
def test_decode_matches_oracle(name, dev, oracle_lib):
    cfg = SMALL[name]
    batch = workloads.make_batch(cfg, dev)
    host = HostCopy(batch)
    ref, kc_ref, vc_ref = oracle_step(oracle_lib, host)
    out, _ = gpu_step(batch)
    pa_check_error()
    # cache write: bit-exact over the whole buffers
    assert np.array_equal(bits(batch.key_cache), kc_ref)
    assert np.array_equal(bits(batch.value_cache), vc_ref)
    _check_close(out, ref, cfg, name)


@pytest.mark.parametrize("name", ["long_small", "gqa_small", "mha_small", "d64_gqa2",
                                  "gqa16_two_rows"])
@pytest.mark.parametrize("ps", [16, 64, 512])
def test_split_matches_oracle(name, ps, dev, oracle_lib):
    cfg = SMALL[name]
    batch = workloads.make_batch(cfg, dev)
    host = HostCopy(batch)
    ref, kc_ref, vc_ref = oracle_step(oracle_lib, host)
    out, ws = gpu_step(batch, partition_size=ps)
    pa_check_error()
    _check_close(out, ref, cfg, f"{name} split {ps}")
    _check_partials(oracle_lib, host, kc_ref, vc_ref, cfg, ws, ps)


def _check_partials(oracle_lib, host, kc_ref, vc_ref, cfg, ws, ps):
    """The partial statistics of a split launch against the oracle's
    partitions: exactly the partitions p < ceil(ctx/P) are written."""
    P = ws.max_partitions
    acc, pmax, psum = oracle_lib.decode_partitioned(host.query, kc_ref, vc_ref,
                                                    host.block_tables, host.context_lens,
                                                    cfg.scale, 1 if cfg.dtype == "bf16" else 0,
                                                    ps, P)
    gm = ws.max_logits.cpu().numpy().astype(np.float64)
    gs = ws.exp_sums.cpu().numpy().astype(np.float64)
    ga = ws.tmp_out.cpu().numpy().astype(np.float64)
    valid = ~np.isnan(pmax)
    assert np.array_equal(valid, ~np.isnan(gm)), "partitions written differ from ceil(ctx/P)"
    assert np.max(np.abs(gm[valid] - pmax[valid])) <= 1e-4
    rel = np.abs(gs[valid] - psum[valid]) / psum[valid]
    assert np.max(rel) <= 1e-2
    na = acc / psum[..., None]
    ng = ga / gs[..., None]
    assert np.nanmax(np.abs(na - ng)[valid]) <= TOL[cfg.dtype]


@pytest.mark.parametrize("ps", [0, 256])
@pytest.mark.parametrize("name", ["mha_small", "gqa_small", "gqa8", "mha_bf16", "gqa16_two_rows"])
def test_growing_logits_force_the_rescale(name, ps, dev, oracle_lib):
    """Logits that climb by about 10 log2 units every 4 pages: the running
    maximum outgrows the page step's slack again and again, so O and l are
    rescaled mid-sequence and the published partials are restated against
    the true maximum.  Output (and the split's partials) against the oracle."""
    cfg = SMALL[name]
    batch = workloads.make_batch(cfg, dev)
    assert grow_logits(batch) >= 14.0  # at least two climbs past the slack
    host = HostCopy(batch)
    ref, kc_ref, vc_ref = oracle_step(oracle_lib, host)
    out, ws = gpu_step(batch, partition_size=ps)
    pa_check_error()
    _check_close(out, ref, cfg, f"{name} growing logits, split {ps}")
    if ps:
        _check_partials(oracle_lib, host, kc_ref, vc_ref, cfg, ws, ps)


def test_split_over_full_grid_for_many_sequences(dev, oracle_lib):
    """300 sequences on a short table: the grid over every possible partition
    stays far below 64 waves, so the split launch gives each its own CTA;
    partials and merged output against the oracle."""
    cfg = SMALL["mha_small"].scaled(num_seqs=300, num_heads=2, num_kv_heads=2, num_blocks=2048,
                                    ctx=("uniform", 0, 90), seed=23)
    batch = workloads.make_batch(cfg, dev)
    host = HostCopy(batch)
    ref, kc_ref, vc_ref = oracle_step(oracle_lib, host)
    out, ws = gpu_step(batch, partition_size=32)
    pa_check_error()
    _check_close(out, ref, cfg, "split, 300 sequences")
    _check_partials(oracle_lib, host, kc_ref, vc_ref, cfg, ws, 32)


def test_split_single_partition_equals_single_pass(dev):
    cfg = SMALL["gqa_small"]
    batch = workloads.make_batch(cfg, dev)
    one, _ = gpu_step(batch)
    batch2 = workloads.make_batch(cfg, dev)
    big = 16 * batch.block_tables.shape[1]
    two, _ = gpu_step(batch2, partition_size=big)
    assert (to_f64(one) - to_f64(two)).__abs__().max() <= 2 * TOL[cfg.dtype]


@pytest.mark.parametrize("name", ["tiny", "gqa_small", "mha_bf16"])
def test_context_len_one_returns_v_exactly(name, dev):
    cfg = SMALL[name]
    batch = workloads.make_batch(cfg, dev)
    batch.context_lens.fill_(1)
    out, _ = gpu_step(batch, write=False)
    G = cfg.group_size
    bt0 = batch.block_tables[:, 0].long()
    v0 = batch.value_cache[bt0, 0]                     # [S, Hk, D]
    want = v0.repeat_interleave(G, dim=1)
    assert torch.equal(out, want)


def test_permutation_invariance_bitwise(dev):
    cfg = SMALL["gqa_small"]
    batch = workloads.make_batch(cfg, dev)
    base, _ = gpu_step(batch, write=False)
    g = torch.Generator().manual_seed(5)
    pi = torch.randperm(cfg.num_blocks, generator=g).to(dev)
    kc = torch.empty_like(batch.key_cache)
    vc = torch.empty_like(batch.value_cache)
    kc[pi] = batch.key_cache
    vc[pi] = batch.value_cache
    bt = torch.where(batch.block_tables >= 0, pi[batch.block_tables.clamp(min=0).long()],
                     torch.full_like(batch.block_tables, -1)).to(torch.int32)
    batch.key_cache, batch.value_cache, batch.block_tables = kc, vc, bt
    moved, _ = gpu_step(batch, write=False)
    assert torch.equal(base, moved)


def test_shared_prefix_equals_private_copies_bitwise(dev):
    cfg = SMALL["shared_small"]
    batch = workloads.make_batch(cfg, dev)
    shared, _ = gpu_step(batch, write=False)
    bt = batch.block_tables.clone()
    used = set(int(x) for x in bt.flatten().tolist() if x >= 0)
    free = [b for b in range(cfg.num_blocks) if b not in used]
    for s in range(cfg.num_seqs):
        if s % cfg.share_group == 0:
            continue
        for i in range(cfg.shared_prefix_blocks):
            nb = free.pop()
            batch.key_cache[nb] = batch.key_cache[int(bt[s, i])]
            batch.value_cache[nb] = batch.value_cache[int(bt[s, i])]
            bt[s, i] = nb
    batch.block_tables = bt
    private, _ = gpu_step(batch, write=False)
    assert torch.equal(shared, private)


def test_zero_and_ragged_context_lengths(dev, oracle_lib):
    cfg = SMALL["gqa_small"].scaled(ctx=("fixed", (0, 1, 15, 16, 17, 31, 32, 33)), num_seqs=8)
    batch = workloads.make_batch(cfg, dev)
    host = HostCopy(batch)
    ref, _, _ = oracle_step(oracle_lib, host)
    out, _ = gpu_step(batch)
    assert (to_f64(out[0]) == 0).all()
    _check_close(out, ref, cfg, "ragged")
    b2 = workloads.make_batch(cfg, dev)
    out2, _ = gpu_step(b2, partition_size=16)
    assert (to_f64(out2[0]) == 0).all()
    _check_close(out2, ref, cfg, "ragged split")


def test_long_sequence_many_pages_per_warp(dev, oracle_lib):
    # > 32 pages per warp exercises the second block-id window
    cfg = SMALL["mha_small"].scaled(num_seqs=2, num_heads=2, num_kv_heads=2, num_blocks=1024,
                                    ctx=("fixed", (3000, 2049)))
    batch = workloads.make_batch(cfg, dev)
    host = HostCopy(batch)
    ref, _, _ = oracle_step(oracle_lib, host)
    out, _ = gpu_step(batch)
    _check_close(out, ref, cfg, "long single pass")


@pytest.mark.parametrize("name,ctx", [
    # long and short items in one launch, with a block table wide enough
    # (> 512 pages) that single-pass decode runs in thread-block clusters:
    # items over 256 pages are spread over the CTAs of their cluster (merged
    # through distributed shared memory), shorter ones stay on one CTA
    ("gqa_small", (1, 40, 4097, 5000, 17000)),
    ("gqa16_two_rows", (17, 9000, 4200)),
    ("d64_gqa2", (5, 12000, 4100)),
    ("mha_bf16", (4300, 1, 8200)),
])
def test_cluster_spread_items_match_oracle(name, ctx, dev, oracle_lib):
    base = SMALL[name]
    need = sum((c + 15) // 16 for c in ctx)
    cfg = base.scaled(num_seqs=len(ctx), ctx=("fixed", ctx), num_blocks=need + 64)
    batch = workloads.make_batch(cfg, dev)
    width = 1100  # table columns past each sequence's pages are never read
    pad = torch.full((cfg.num_seqs, width - batch.block_tables.shape[1]), -1,
                     dtype=torch.int32, device=dev)
    batch.block_tables = torch.cat([batch.block_tables, pad], dim=1).contiguous()
    host = HostCopy(batch)
    ref, _, _ = oracle_step(oracle_lib, host)
    out, _ = gpu_step(batch)
    pa_check_error()
    _check_close(out, ref, cfg, f"{name} spread")


def test_many_sequences_natural_order(dev, oracle_lib):
    # more sequences than the longest-first ordering handles
    cfg = SMALL["mha_small"].scaled(num_seqs=300, num_heads=2, num_kv_heads=2, num_blocks=2048,
                                    ctx=("uniform", 0, 90), seed=21)
    batch = workloads.make_batch(cfg, dev)
    host = HostCopy(batch)
    ref, _, _ = oracle_step(oracle_lib, host)
    out, _ = gpu_step(batch)
    pa_check_error()
    _check_close(out, ref, cfg, "natural order")


NAN_CASES = [(n, m) for n in ("mha_small", "gqa_small", "gqa16_two_rows", "d64_gqa2",
                              "shared_small") for m in ("single", "split64")]
NAN_CASES.append(("shared_small", "shared"))   # the shared-prefix kernel needs its groups


@pytest.mark.parametrize("name,mode", NAN_CASES)
def test_nan_rows_past_context_do_not_leak(name, mode, dev, oracle_lib):
    """Cache rows past a sequence's context (never written) hold NaN: the
    output still matches the oracle, which never reads them."""
    cfg = SMALL[name]
    batch = workloads.make_batch(cfg, dev)
    assert poison_past_context(batch) > 0
    host = HostCopy(batch)
    ref, _, _ = oracle_step(oracle_lib, host)
    out, _ = gpu_step(batch, partition_size=64 if mode == "split64" else 0,
                      shared_prefix=mode == "shared")
    pa_check_error()
    _check_close(out, ref, cfg, f"{name} {mode} with NaN past the context")


def _regroup(batch, starts, prefix):
    """Make sequences [starts[g], starts[g+1]) share their first prefix[g]
    table entries -- the ids of the group's longest member (clamped to its
    block count) -- and attach the group arrays."""
    bt = batch.block_tables.clone()
    ctx = batch.context_lens.tolist()
    prefix = list(prefix)
    for g in range(len(starts) - 1):
        members = list(range(starts[g], starts[g + 1]))
        donor = max(members, key=lambda s: ctx[s])
        prefix[g] = min(prefix[g], (ctx[donor] + 15) // 16)
        for s in members:
            bt[s, :prefix[g]] = bt[donor, :prefix[g]]
    batch.block_tables = bt
    dev = bt.device
    batch.group_starts = torch.tensor(starts, dtype=torch.int32, device=dev)
    batch.prefix_blocks = torch.tensor(prefix, dtype=torch.int32, device=dev)
    return batch


SHARED_CASES = {
    # name: (base config, overrides, group starts, prefix blocks per group)
    "beam4_gqa4": ("shared_small", {}, None, None),
    "mha_16_members": ("mha_small", dict(num_seqs=20, num_heads=2, num_kv_heads=2, num_blocks=600,
                                         ctx=("uniform", 40, 300), seed=41),
                       [0, 16, 20], [2, 1]),
    "gqa8_chunked": ("gqa8", dict(num_seqs=7, num_blocks=300, ctx=("uniform", 1, 400), seed=42),
                     [0, 5, 7], [3, 0]),
    "gqa2_ragged_bf16": ("d64_gqa2", dict(num_seqs=9, num_blocks=400, ctx=("uniform", 1, 600),
                                          seed=43), [0, 1, 4, 9], [1, 5, 2]),
    "short_members": ("gqa_small", dict(num_seqs=4, num_blocks=200,
                                        ctx=("fixed", (20, 300, 5, 0)), seed=44),
                      [0, 4], [8]),
    "long_prefix_spread": ("gqa_small", dict(num_seqs=4, num_blocks=900,
                                             ctx=("fixed", (3000, 2900, 3100, 4000)), seed=45),
                           [0, 4], [150]),
}


@pytest.mark.parametrize("name", ["beam4_gqa4", "gqa8_chunked", "long_prefix_spread"])
def test_shared_prefix_growing_logits(name, dev, oracle_lib):
    """The shared-prefix kernel with key rows whose logits climb by about 10
    log2 units every 4 pages (members sharing a prefix block keep the last
    member's rewrite of it): its page step rescales O mid-sequence, on shared
    and private pages.  Against the oracle."""
    base, over, starts, prefix = SHARED_CASES[name]
    cfg = SMALL[base].scaled(**over) if over else SMALL[base]
    batch = workloads.make_batch(cfg, dev)
    if starts is not None:
        batch = _regroup(batch, starts, prefix)
    assert grow_logits(batch) >= 14.0
    host = HostCopy(batch)
    ref, _, _ = oracle_step(oracle_lib, host)
    out, _ = gpu_step(batch, shared_prefix=True)
    pa_check_error()
    _check_close(out, ref, cfg, f"{name} shared prefix, growing logits")


@pytest.mark.parametrize("name", list(SHARED_CASES))
def test_shared_prefix_matches_oracle(name, dev, oracle_lib):
    base, over, starts, prefix = SHARED_CASES[name]
    cfg = SMALL[base].scaled(**over) if over else SMALL[base]
    batch = workloads.make_batch(cfg, dev)
    if starts is not None:
        batch = _regroup(batch, starts, prefix)
    host = HostCopy(batch)
    ref, kc_ref, vc_ref = oracle_step(oracle_lib, host)
    out, _ = gpu_step(batch, shared_prefix=True)
    pa_check_error()
    assert np.array_equal(bits(batch.key_cache), kc_ref)
    _check_close(out, ref, cfg, f"shared prefix {name}")
    plain, _ = gpu_step(batch, write=False)
    assert np.max(np.abs(to_f64(plain) - to_f64(out))) <= TOL[cfg.dtype]


def test_shared_prefix_reports_bad_groups(dev):
    cfg = SMALL["shared_small"]
    batch = workloads.make_batch(cfg, dev)
    batch.group_starts[1] = batch.group_starts[2] + 1       # not monotone
    gpu_step(batch, write=False, shared_prefix=True, max_group_size=cfg.share_group)
    with pytest.raises(PagedAttentionError) as e:
        pa_check_error()
    assert e.value.detail >> 56 == 6
    batch = _regroup(workloads.make_batch(cfg, dev), [0, 8], [4])
    # one group of 8 members, but room for 4 (one chunk of 16 rows / 4 heads)
    gpu_step(batch, write=False, shared_prefix=True, max_group_size=4)
    with pytest.raises(PagedAttentionError) as e:
        pa_check_error()
    assert e.value.detail >> 56 == 6
    pa_check_error()


@pytest.mark.parametrize("name", ["gqa_small", "tiny"])
def test_copy_blocks_bit_exact(name, dev, oracle_lib):
    cfg = SMALL[name]
    batch = workloads.make_batch(cfg, dev)
    g = torch.Generator().manual_seed(7)
    perm = torch.randperm(cfg.num_blocks, generator=g)
    pairs = torch.stack([perm[:20], perm[20:40]], dim=1).contiguous()  # distinct, disjoint
    kc, vc = bits(batch.key_cache), bits(batch.value_cache)
    assert oracle_lib.copy_blocks(kc, vc, pairs.numpy()) == 0
    from paged_kv_cache_444_b200 import pa_copy_blocks
    pa_copy_blocks(batch.key_cache, batch.value_cache, pairs.to(dev))
    torch.cuda.synchronize()
    pa_check_error()
    assert np.array_equal(bits(batch.key_cache), kc)
    assert np.array_equal(bits(batch.value_cache), vc)
    # an id past the pool is skipped and reported with its pair index
    bad = torch.tensor([[0, 1], [2, cfg.num_blocks]], dtype=torch.int64, device=dev)
    pa_copy_blocks(batch.key_cache, batch.value_cache, bad)
    with pytest.raises(PagedAttentionError) as e:
        pa_check_error()
    assert e.value.detail >> 56 == 2 and e.value.detail & 0xffff == 1


@pytest.mark.parametrize("name,ps", [("gqa_small", 0), ("mha_small", 0), ("long_small", 512)])
def test_host_step_matches_oracle(name, ps, dev, oracle_lib):
    """pa_decode_step_host: inputs in pinned host memory, copied in, written,
    attended and copied back by one C call."""
    from paged_kv_cache_444_b200 import HostStep
    cfg = SMALL[name]
    batch = workloads.make_batch(cfg, dev)
    host = HostCopy(batch)
    ref, kc_ref, _ = oracle_step(oracle_lib, host)
    step = HostStep(batch.key_cache, batch.value_cache, cfg.num_seqs, cfg.num_heads,
                    batch.block_tables.shape[1], cfg.scale, ps, cfg.torch_dtype)
    for name_ in ("query", "key", "value", "slot_mapping", "block_tables", "context_lens"):
        getattr(step, name_).copy_(getattr(batch, name_).cpu())
    step.out.fill_(float("nan"))
    step.run()
    torch.cuda.synchronize()
    pa_check_error()
    assert np.array_equal(bits(batch.key_cache), kc_ref)
    _check_close(step.out, ref, cfg, f"host step {name}")


@pytest.mark.parametrize("name,ps", [("gqa_small", 0), ("long_small", 64)])
def test_host_step_unpacked_inputs_pageable_output(name, ps, dev, oracle_lib):
    """pa_decode_step_host with each input in its own pinned tensor (one copy
    each) and a pageable output (written to the workspace, then copied back),
    run twice in a row on one stream."""
    from paged_kv_cache_444_b200 import HostStep
    cfg = SMALL[name]
    batch = workloads.make_batch(cfg, dev)
    host = HostCopy(batch)
    ref, kc_ref, _ = oracle_step(oracle_lib, host)
    step = HostStep(batch.key_cache, batch.value_cache, cfg.num_seqs, cfg.num_heads,
                    batch.block_tables.shape[1], cfg.scale, ps, cfg.torch_dtype)
    for name_ in ("query", "key", "value", "slot_mapping", "block_tables", "context_lens"):
        setattr(step, name_, getattr(batch, name_).cpu().clone().pin_memory())
    step.out = torch.full(tuple(batch.query.shape), float("nan"), dtype=cfg.torch_dtype)
    assert not step.out.is_pinned()
    for _ in range(2):
        step.run()
    torch.cuda.synchronize()
    pa_check_error()
    assert np.array_equal(bits(batch.key_cache), kc_ref)
    _check_close(step.out, ref, cfg, f"host step {name}, unpacked inputs, pageable output")


@pytest.mark.parametrize("pageable", [("key", "value", "slot_mapping"), ("value",)],
                         ids=["all_rows_pageable", "value_pageable"])
def test_host_step_pageable_new_rows(pageable, dev, oracle_lib):
    """pa_decode_step_host when some of the new rows are in pageable memory:
    the cache write cannot read them from host memory, so all three are copied
    into the workspace first (with every part pinned it reads them directly)."""
    from paged_kv_cache_444_b200 import HostStep
    cfg = SMALL["gqa_small"]
    batch = workloads.make_batch(cfg, dev)
    host = HostCopy(batch)
    ref, kc_ref, _ = oracle_step(oracle_lib, host)
    step = HostStep(batch.key_cache, batch.value_cache, cfg.num_seqs, cfg.num_heads,
                    batch.block_tables.shape[1], cfg.scale, 0, cfg.torch_dtype)
    for name_ in ("query", "key", "value", "slot_mapping", "block_tables", "context_lens"):
        t = getattr(batch, name_).cpu().clone()
        setattr(step, name_, t if name_ in pageable else t.pin_memory())
    step.out.fill_(float("nan"))
    step.run()
    torch.cuda.synchronize()
    pa_check_error()
    assert np.array_equal(bits(batch.key_cache), kc_ref)
    _check_close(step.out, ref, cfg, f"host step, pageable {pageable}")


@pytest.mark.parametrize("name,ps", [("gqa_small", 0), ("long_small", 64), ("tiny", 0)])
def test_plan_replays_from_a_cuda_graph(name, ps, dev, oracle_lib):
    """A DecodePlan run eagerly, and the same plan captured once in a CUDA
    graph and replayed, both match the oracle; replay equals eager bit for bit."""
    from paged_kv_cache_444_b200 import DecodePlan
    cfg = SMALL[name]
    batch = workloads.make_batch(cfg, dev)
    host = HostCopy(batch)
    ref, _, _ = oracle_step(oracle_lib, host)
    plan = DecodePlan(batch.query, batch.key, batch.value, batch.key_cache, batch.value_cache,
                      batch.slot_mapping, batch.block_tables, batch.context_lens, cfg.scale,
                      partition_size=ps)
    eager = plan.run().clone()
    torch.cuda.synchronize()
    _check_close(eager, ref, cfg, f"plan {name}")
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        plan.run()                      # warm-up on the side stream
    torch.cuda.current_stream().wait_stream(s)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        plan.run()
    plan.out.fill_(float("nan"))
    g.replay()
    torch.cuda.synchronize()
    pa_check_error()
    assert torch.equal(plan.out, eager)


def test_write_padding_and_strided_rows(dev, oracle_lib):
    cfg = SMALL["gqa_small"]
    batch = workloads.make_batch(cfg, dev)
    T = cfg.num_seqs
    big = torch.randn((T, 3, cfg.num_kv_heads, cfg.head_dim), device=dev).to(cfg.torch_dtype)
    batch.key = big[:, 0]
    batch.value = big[:, 2]
    batch.slot_mapping[1] = -1
    batch.slot_mapping[5] = -3
    host = HostCopy(batch)
    host.key = bits(batch.key).reshape(T, cfg.num_kv_heads, cfg.head_dim)
    host.value = bits(batch.value).reshape(T, cfg.num_kv_heads, cfg.head_dim)
    kc, vc = host.key_cache.copy(), host.value_cache.copy()
    assert oracle_lib.reshape_and_cache(host.key, host.value, kc, vc, host.slot_mapping,
                                        cfg.num_blocks, cfg.block_size) == 0
    from paged_kv_cache_444_b200 import pa_reshape_and_cache
    pa_reshape_and_cache(batch.key, batch.value, batch.key_cache, batch.value_cache,
                         batch.slot_mapping)
    torch.cuda.synchronize()
    assert np.array_equal(bits(batch.key_cache), kc)
    assert np.array_equal(bits(batch.value_cache), vc)


def test_bounds_checks_report_and_skip(dev):
    cfg = SMALL["gqa_small"]
    pa_check_error()
    batch = workloads.make_batch(cfg, dev)
    # a slot past the end: skipped, reported with its token index
    batch.slot_mapping[3] = cfg.num_blocks * cfg.block_size + 5
    before = batch.key_cache.clone()
    from paged_kv_cache_444_b200 import pa_reshape_and_cache
    pa_reshape_and_cache(batch.key, batch.value, batch.key_cache, batch.value_cache,
                         batch.slot_mapping)
    with pytest.raises(PagedAttentionError) as e:
        pa_check_error()
    assert e.value.detail >> 56 == 1 and e.value.detail & 0xffff == 3
    changed = (batch.key_cache != before).flatten(1).any(1).nonzero().flatten().tolist()
    assert len(changed) <= cfg.num_seqs - 1
    pa_check_error()  # cleared
    # a block id past the pool: read as zeros, reported
    b = workloads.make_batch(cfg, dev)
    b.block_tables[2, 0] = cfg.num_blocks + 7
    out, _ = gpu_step(b, write=False)
    with pytest.raises(PagedAttentionError) as e:
        pa_check_error()
    assert e.value.detail >> 56 == 2
    assert np.isfinite(to_f64(out)).all()
    # a context length beyond the table: clamped, reported
    b = workloads.make_batch(cfg, dev)
    b.context_lens[4] = b.block_tables.shape[1] * cfg.block_size + 100
    b.block_tables[4, :] = b.block_tables[4, 0]   # every entry valid: only the length is wrong
    out, _ = gpu_step(b, write=False)
    with pytest.raises(PagedAttentionError) as e:
        pa_check_error()
    assert e.value.detail >> 56 == 3 and e.value.detail & 0xffff == 4
    # too few partitions for a sequence: reported
    b = workloads.make_batch(cfg, dev)
    gpu_step(b, write=False, partition_size=16, max_partitions=2)
    with pytest.raises(PagedAttentionError) as e:
        pa_check_error()
    assert e.value.detail >> 56 == 4
    pa_check_error()


def test_empty_batch_is_a_no_op(dev):
    from paged_kv_cache_444_b200 import pa_decode
    cfg = SMALL["tiny"]
    b = workloads.make_batch(cfg, dev)
    out = torch.empty((0, cfg.num_heads, cfg.head_dim), dtype=b.query.dtype, device=dev)
    pa_decode(out, b.query[:0], b.key_cache, b.value_cache, b.block_tables[:0],
              b.context_lens[:0], cfg.scale)
    torch.cuda.synchronize()


def test_bounded_wait_gives_up_and_context_stays_usable(dev, oracle_lib):
    """The failure path of every kernel's barrier waits, taken on purpose: a
    kernel waits on a barrier that nothing completes, gives up after the
    bounded wait, records PA_CHECK_WAIT_TIMEOUT and returns.  pa_check_error
    reports it once, and a decode launched afterwards in the same context
    still matches the oracle."""
    from paged_kv_cache_444_b200 import pa_selftest_wait_timeout
    pa_check_error()                                  # start from a clean error word
    pa_selftest_wait_timeout()
    with pytest.raises(PagedAttentionError) as e:
        pa_check_error()
    assert e.value.detail >> 56 == 5                  # PA_CHECK_WAIT_TIMEOUT
    assert pa_check_error() == 0                      # reported once, then cleared
    cfg = SMALL["gqa_small"]
    batch = workloads.make_batch(cfg, dev)
    host = HostCopy(batch)
    ref, kc_ref, _ = oracle_step(oracle_lib, host)
    out, _ = gpu_step(batch)
    pa_check_error()
    assert np.array_equal(bits(batch.key_cache), kc_ref)
    _check_close(out, ref, cfg, "decode after a barrier timeout")


def test_split_persistent_on_a_long_skewed_table(dev, oracle_lib):
    """A 16-bit split launch whose grid over every possible partition would run
    past 64 waves of resident CTAs takes the persistent form, over only the
    partitions that exist: 300 sequences (chunks of three per thread), one of
    4096 tokens among 299 of 0-79, 32-token partitions (a full grid of
    300 x 2 x 128 CTAs, 173 waves of the 444 resident).  Partials and merged
    output against the oracle."""
    rng = np.random.default_rng(444_091)
    ctx = [int(c) for c in rng.integers(0, 80, 300)]
    ctx[137] = 4096
    cfg = SMALL["gqa_small"].scaled(num_seqs=300, num_heads=8, num_kv_heads=2, num_blocks=2048,
                                    ctx=("fixed", tuple(ctx)), seed=91)
    batch = workloads.make_batch(cfg, dev)
    assert cfg.num_seqs * cfg.num_kv_heads * (batch.block_tables.shape[1] * 16 // 32) > 128 * 444
    host = HostCopy(batch)
    ref, kc_ref, vc_ref = oracle_step(oracle_lib, host)
    out, ws = gpu_step(batch, partition_size=32)
    pa_check_error()
    _check_close(out, ref, cfg, "split, persistent, skewed table")
    _check_partials(oracle_lib, host, kc_ref, vc_ref, cfg, ws, 32)
