"""E4M3 (fp8) KV cache on the GPU vs the fp64 oracle (GPU).

The fp8 caches start from seeded N(0,1) values quantised by torch's own
float8_e4m3fn cast (x * 64, so the codes span the E4M3 range, scale 1/64);
the step's new rows are written by pa_reshape_and_cache_fp8 and compared bit
for bit with the oracle's quantising write, then decode is compared with the
oracle's fp8 decode (same tolerances as the 16-bit path, which they inherit
from the 16-bit query and output)."""
import numpy as np
import pytest
import torch

import oracle as oracle_mod
from paged_kv_cache_444_b200 import (SplitWorkspace, pa_check_error, pa_decode_fp8,
                                     pa_decode_split_fp8, pa_reduce, pa_reshape_and_cache_fp8,
                                     workloads)
from parity_helpers import (K_SCALE, V_SCALE, TOL, bits, fp8_batch as _fp8_batch,
                            fp8_oracle as _oracle, grow_logits, ocode, poison_past_context,
                            to_f64)

pytestmark = pytest.mark.gpu

C = workloads.CONFIGS
CASES = {
    "mha_f16": C["mha_llama2_7b"].scaled(num_seqs=5, num_heads=4, num_kv_heads=4, num_blocks=256,
                                         ctx=("uniform", 1, 500), seed=51),
    "gqa_bf16": C["gqa_llama3_8b"].scaled(num_seqs=6, num_blocks=400, ctx=("uniform", 1, 700),
                                          seed=52),
    "gqa_f16": C["shared_prefix_beam"].scaled(num_seqs=4, num_blocks=300, shared_prefix_blocks=0,
                                              share_group=1, ctx=("uniform", 1, 600), seed=53),
    "gqa16_bf16": C["gqa_llama3_8b"].scaled(num_seqs=3, num_heads=32, num_kv_heads=2,
                                            num_blocks=200, ctx=("uniform", 30, 900), seed=54),
    "ragged_bf16": C["gqa_llama3_8b"].scaled(num_seqs=8, num_blocks=100,
                                             ctx=("fixed", (0, 1, 15, 16, 17, 31, 32, 33)),
                                             seed=55),
    # the transposed page step at its widest group (all 8 mma columns live)
    # and at an odd one (3 heads: the second row of some lanes is padding)
    "gqa8_f16": C["mha_llama2_7b"].scaled(num_seqs=5, num_heads=16, num_kv_heads=2,
                                          num_blocks=300, ctx=("uniform", 1, 800), seed=56),
    "gqa3_bf16": C["gqa_llama3_8b"].scaled(num_seqs=5, num_heads=12, num_kv_heads=4,
                                           num_blocks=300, ctx=("uniform", 1, 800), seed=57),
}


@pytest.mark.parametrize("name", list(CASES))
def test_fp8_write_and_decode_match_oracle(name, cuda_device, oracle_lib):
    cfg = CASES[name]
    b, kc, vc = _fp8_batch(cfg, cuda_device)
    ref, kh, vh = _oracle(oracle_lib, b, kc, vc)
    pa_reshape_and_cache_fp8(b.key, b.value, kc, vc, b.slot_mapping, K_SCALE, V_SCALE)
    out = torch.full_like(b.query, float("nan"))
    pa_decode_fp8(out, b.query, kc, vc, b.block_tables, b.context_lens, cfg.scale, K_SCALE,
                  V_SCALE)
    torch.cuda.synchronize()
    pa_check_error()
    assert np.array_equal(kc.cpu().numpy(), kh) and np.array_equal(vc.cpu().numpy(), vh)
    g = to_f64(out)
    assert np.isfinite(g).all()
    err = np.max(np.abs(g - ref))
    assert err <= TOL[cfg.dtype], f"{name}: {err:.3e}"


@pytest.mark.parametrize("ps", [0, 256])
@pytest.mark.parametrize("name", ["mha_f16", "gqa_bf16", "gqa8_f16", "gqa16_bf16"])
def test_fp8_growing_logits_force_the_rescale(name, ps, cuda_device, oracle_lib):
    """Logits that climb by about 10 log2 units every 4 pages (three climbs,
    which keeps the key codes below saturation): the page step rescales O and
    l mid-sequence and restates its partials against the true maximum."""
    cfg = CASES[name]
    top = []
    b, kc, vc = _fp8_batch(cfg, cuda_device,
                           prepare=lambda bb: top.append(grow_logits(bb, max_steps=3)))
    assert top[0] >= 14.0
    ref, _, _ = _oracle(oracle_lib, b, kc, vc)
    pa_reshape_and_cache_fp8(b.key, b.value, kc, vc, b.slot_mapping, K_SCALE, V_SCALE)
    out = torch.full_like(b.query, float("nan"))
    if ps:
        P = (b.block_tables.shape[1] * 16 + ps - 1) // ps
        ws = SplitWorkspace(cfg.num_seqs, cfg.num_heads, cfg.head_dim, P, cuda_device)
        pa_decode_split_fp8(ws.tmp_out, ws.max_logits, ws.exp_sums, b.query, kc, vc,
                            b.block_tables, b.context_lens, cfg.scale, K_SCALE, V_SCALE, ps)
        pa_reduce(out, ws.tmp_out, ws.max_logits, ws.exp_sums, b.context_lens, ps)
    else:
        pa_decode_fp8(out, b.query, kc, vc, b.block_tables, b.context_lens, cfg.scale, K_SCALE,
                      V_SCALE)
    torch.cuda.synchronize()
    pa_check_error()
    g = to_f64(out)
    assert np.isfinite(g).all()
    err = np.max(np.abs(g - ref))
    assert err <= TOL[cfg.dtype], f"{name} growing logits, split {ps}: {err:.3e}"


@pytest.mark.parametrize("name", ["gqa_bf16", "mha_f16", "gqa8_f16", "gqa3_bf16"])
@pytest.mark.parametrize("ps", [16, 256])
def test_fp8_split_matches_oracle(name, ps, cuda_device, oracle_lib):
    cfg = CASES[name]
    b, kc, vc = _fp8_batch(cfg, cuda_device)
    ref, _, _ = _oracle(oracle_lib, b, kc, vc)
    pa_reshape_and_cache_fp8(b.key, b.value, kc, vc, b.slot_mapping, K_SCALE, V_SCALE)
    P = (b.block_tables.shape[1] * 16 + ps - 1) // ps
    ws = SplitWorkspace(cfg.num_seqs, cfg.num_heads, cfg.head_dim, P, cuda_device)
    out = torch.full_like(b.query, float("nan"))
    pa_decode_split_fp8(ws.tmp_out, ws.max_logits, ws.exp_sums, b.query, kc, vc, b.block_tables,
                        b.context_lens, cfg.scale, K_SCALE, V_SCALE, ps)
    pa_reduce(out, ws.tmp_out, ws.max_logits, ws.exp_sums, b.context_lens, ps)
    torch.cuda.synchronize()
    pa_check_error()
    err = np.max(np.abs(to_f64(out) - ref))
    assert err <= TOL[cfg.dtype], f"{name} split {ps}: {err:.3e}"


@pytest.mark.parametrize("name,ps", [("ragged_bf16", 16), ("many_seqs_f16", 32)],
                         ids=["persistent_ragged_with_empty", "full_grid_300_seqs"])
def test_fp8_split_ragged_and_large_batches(name, ps, cuda_device, oracle_lib):
    """The fp8 split launch is persistent (one wave of CTAs over the
    partitions that exist, empty sequences contributing none), on a ragged
    batch and on 300 sequences (chunks of three per thread); both against the
    oracle."""
    cfg = (CASES["ragged_bf16"] if name == "ragged_bf16" else
           C["mha_llama2_7b"].scaled(num_seqs=300, num_heads=2, num_kv_heads=2, num_blocks=2048,
                                     ctx=("uniform", 0, 90), seed=56))
    b, kc, vc = _fp8_batch(cfg, cuda_device)
    ref, _, _ = _oracle(oracle_lib, b, kc, vc)
    pa_reshape_and_cache_fp8(b.key, b.value, kc, vc, b.slot_mapping, K_SCALE, V_SCALE)
    P = (b.block_tables.shape[1] * 16 + ps - 1) // ps
    ws = SplitWorkspace(cfg.num_seqs, cfg.num_heads, cfg.head_dim, P, cuda_device)
    out = torch.full_like(b.query, float("nan"))
    pa_decode_split_fp8(ws.tmp_out, ws.max_logits, ws.exp_sums, b.query, kc, vc, b.block_tables,
                        b.context_lens, cfg.scale, K_SCALE, V_SCALE, ps)
    pa_reduce(out, ws.tmp_out, ws.max_logits, ws.exp_sums, b.context_lens, ps)
    torch.cuda.synchronize()
    pa_check_error()
    g = to_f64(out)
    assert np.isfinite(g).all()
    zero = (b.context_lens == 0).cpu().numpy()
    assert (g[zero] == 0).all()
    err = np.max(np.abs(g - ref))
    assert err <= TOL[cfg.dtype], f"{name} split {ps}: {err:.3e}"


@pytest.mark.parametrize("split", [0, 64])
@pytest.mark.parametrize("name", ["mha_f16", "gqa_bf16", "gqa16_bf16", "gqa8_f16"])
def test_fp8_nan_codes_past_context_do_not_leak(name, split, cuda_device, oracle_lib):
    """E4M3 NaN codes (0x7f) in the never-written rows past each context."""
    cfg = CASES[name]
    b, kc, vc = _fp8_batch(cfg, cuda_device)
    assert poison_past_context(b, kc, vc, fill=0x7F) > 0
    ref, _, _ = _oracle(oracle_lib, b, kc, vc)
    pa_reshape_and_cache_fp8(b.key, b.value, kc, vc, b.slot_mapping, K_SCALE, V_SCALE)
    out = torch.full_like(b.query, float("nan"))
    if split:
        P = (b.block_tables.shape[1] * 16 + split - 1) // split
        ws = SplitWorkspace(cfg.num_seqs, cfg.num_heads, cfg.head_dim, P, cuda_device)
        pa_decode_split_fp8(ws.tmp_out, ws.max_logits, ws.exp_sums, b.query, kc, vc,
                            b.block_tables, b.context_lens, cfg.scale, K_SCALE, V_SCALE, split)
        pa_reduce(out, ws.tmp_out, ws.max_logits, ws.exp_sums, b.context_lens, split)
    else:
        pa_decode_fp8(out, b.query, kc, vc, b.block_tables, b.context_lens, cfg.scale, K_SCALE,
                      V_SCALE)
    torch.cuda.synchronize()
    pa_check_error()
    g = to_f64(out)
    assert np.isfinite(g).all()
    assert np.max(np.abs(g - ref)) <= TOL[cfg.dtype]


@pytest.mark.parametrize("name", ["mha_f16", "gqa_bf16", "gqa3_bf16"])
def test_fp8_context_len_one_is_exact(name, cuda_device):
    # p = 1, and code * 2^-5 is exact in fp32 and in the 16-bit output
    cfg = CASES[name]
    b, kc, vc = _fp8_batch(cfg, cuda_device)
    b.context_lens.fill_(1)
    out = torch.empty_like(b.query)
    pa_decode_fp8(out, b.query, kc, vc, b.block_tables, b.context_lens, cfg.scale, K_SCALE,
                  V_SCALE)
    torch.cuda.synchronize()
    v0 = vc[b.block_tables[:, 0].long(), 0].view(torch.float8_e4m3fn).to(torch.float32) * V_SCALE
    want = v0.to(b.query.dtype).repeat_interleave(cfg.group_size, dim=1)
    assert torch.equal(out, want)


def test_fp8_full_size_gqa_sampled(cuda_device, oracle_lib):
    """The Llama-3-8B GQA batch at full size with an fp8 cache (half the
    bytes of the bf16 one), checked on sampled sequences."""
    cfg = C["gqa_llama3_8b"]
    b, kc, vc = _fp8_batch(cfg, cuda_device)
    seqs = [0, 37, 127]
    # host snapshot of the sampled sequences' blocks before the write
    bt = b.block_tables[seqs].cpu().numpy()
    ctx = b.context_lens[seqs].cpu().numpy().astype(np.int32)
    used = sorted({int(x) for i in range(len(seqs))
                   for x in bt[i, :(int(ctx[i]) + 15) // 16]})
    remap = {blk: n for n, blk in enumerate(used)}
    bt_new = np.full_like(bt, -1)
    for i in range(len(seqs)):
        for j in range((int(ctx[i]) + 15) // 16):
            bt_new[i, j] = remap[int(bt[i, j])]
    ids = torch.tensor(used, dtype=torch.long, device=cuda_device)
    kh = kc.index_select(0, ids).cpu().numpy().copy()
    vh = vc.index_select(0, ids).cpu().numpy().copy()
    slots = b.slot_mapping[seqs].cpu().numpy()
    slots = np.array([remap[int(x) // 16] * 16 + int(x) % 16 for x in slots], dtype=np.int64)
    assert oracle_lib.reshape_and_cache_fp8(bits(b.key[seqs]), bits(b.value[seqs]), kh, vh, slots,
                                            len(used), 16, K_SCALE, V_SCALE, oracle_mod.BF16) == 0
    ref = oracle_lib.decode_fp8(bits(b.query[seqs]), kh, vh, bt_new, ctx, cfg.scale, K_SCALE,
                                V_SCALE, oracle_mod.BF16)
    pa_reshape_and_cache_fp8(b.key, b.value, kc, vc, b.slot_mapping, K_SCALE, V_SCALE)
    out = torch.empty_like(b.query)
    pa_decode_fp8(out, b.query, kc, vc, b.block_tables, b.context_lens, cfg.scale, K_SCALE,
                  V_SCALE)
    torch.cuda.synchronize()
    pa_check_error()
    assert np.array_equal(kc.index_select(0, ids).cpu().numpy(), kh)
    err = np.max(np.abs(to_f64(out[seqs]) - ref))
    assert err <= TOL["bf16"], err


@pytest.mark.parametrize("name,ctx", [
    # a block table wide enough (> 512 pages) that single-pass fp8 decode
    # runs in thread-block clusters: items over 256 pages are spread over the
    # CTAs of their cluster and merged through distributed shared memory,
    # shorter ones stay on one CTA
    ("gqa_bf16", (1, 40, 4097, 5000, 17000)),   # transposed page step, group 4
    ("mha_f16", (4300, 1, 8200)),               # transposed page step, one head
    ("gqa16_bf16", (17, 9000, 4200)),           # 16-row tile, group 16
])
def test_fp8_cluster_spread_items_match_oracle(name, ctx, cuda_device, oracle_lib):
    base = CASES[name]
    need = sum((c + 15) // 16 for c in ctx)
    cfg = base.scaled(num_seqs=len(ctx), ctx=("fixed", ctx), num_blocks=need + 64)
    b, kc, vc = _fp8_batch(cfg, cuda_device)
    width = 1100  # table columns past each sequence's pages are never read
    pad = torch.full((cfg.num_seqs, width - b.block_tables.shape[1]), -1, dtype=torch.int32,
                     device=cuda_device)
    b.block_tables = torch.cat([b.block_tables, pad], dim=1).contiguous()
    ref, _, _ = _oracle(oracle_lib, b, kc, vc)
    pa_reshape_and_cache_fp8(b.key, b.value, kc, vc, b.slot_mapping, K_SCALE, V_SCALE)
    out = torch.full_like(b.query, float("nan"))
    pa_decode_fp8(out, b.query, kc, vc, b.block_tables, b.context_lens, cfg.scale, K_SCALE,
                  V_SCALE)
    torch.cuda.synchronize()
    pa_check_error()
    g = to_f64(out)
    assert np.isfinite(g).all()
    err = np.max(np.abs(g - ref))
    assert err <= TOL[cfg.dtype], f"{name} spread: {err:.3e}"
