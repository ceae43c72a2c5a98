"""Paged (chunked) prefill vs the fp64 oracle (GPU): each sequence's new
query tokens are the last q_len positions of its context and attend
causally over the paged cache.  Tolerances as for decode."""
import numpy as np
import pytest
import torch

from paged_kv_cache_444_b200 import (PagedAttentionError, pa_check_error, pa_prefill,
                                     pa_reshape_and_cache, workloads)
from parity_helpers import TOL, bits, ocode, to_f64

pytestmark = pytest.mark.gpu
C = workloads.CONFIGS

CASES = {
    # name: (base config, overrides, query lengths per sequence)
    "gqa4_bf16": (C["gqa_llama3_8b"], dict(num_seqs=4, num_blocks=300,
                                          ctx=("fixed", (100, 17, 300, 64)), seed=61),
                  (37, 17, 130, 1)),
    "mha_f16": (C["mha_llama2_7b"], dict(num_seqs=3, num_heads=4, num_kv_heads=4,
                                        num_blocks=200, ctx=("fixed", (200, 65, 129)), seed=62),
                (200, 64, 5)),
    "gqa8_f16_d64": (C["tiny"], dict(num_seqs=2, num_heads=16, num_kv_heads=2, num_blocks=100,
                                     ctx=("fixed", (90, 33)), seed=63), (33, 33)),
    "gqa16_bf16": (C["gqa_llama3_8b"], dict(num_seqs=2, num_heads=32, num_kv_heads=2,
                                           num_blocks=100, ctx=("fixed", (50, 700)), seed=64),
                   (9, 300)),
    "gqa3_f16": (C["gqa_llama3_8b"], dict(num_seqs=2, num_heads=12, num_kv_heads=4, dtype="f16",
                                         num_blocks=100, ctx=("fixed", (45, 80)), seed=65),
                 (45, 23)),
}


def _case(name, dev):
    base, over, qlens = CASES[name]
    cfg = base.scaled(**over)
    b = workloads.make_batch(cfg, dev)
    T = sum(qlens)
    g = torch.Generator(device=dev).manual_seed(cfg.seed + 5)
    query = torch.randn((T, cfg.num_heads, cfg.head_dim), generator=g, device=dev).to(
        cfg.torch_dtype)
    starts = torch.tensor(np.concatenate([[0], np.cumsum(qlens)]), dtype=torch.int32, device=dev)
    return cfg, b, query, starts, qlens


@pytest.mark.parametrize("name", list(CASES))
def test_prefill_matches_oracle(name, cuda_device, oracle_lib):
    cfg, b, query, starts, qlens = _case(name, cuda_device)
    # write the step's last token first (any earlier prompt rows are already random cache)
    kc = bits(b.key_cache).copy()
    vc = bits(b.value_cache).copy()
    assert oracle_lib.reshape_and_cache(bits(b.key), bits(b.value), kc, vc,
                                        b.slot_mapping.cpu().numpy(), cfg.num_blocks,
                                        cfg.block_size) == 0
    ref = oracle_lib.prefill(bits(query), kc, vc, b.block_tables.cpu().numpy(),
                             b.context_lens.cpu().numpy(), starts.cpu().numpy(), cfg.scale,
                             ocode(cfg))
    pa_reshape_and_cache(b.key, b.value, b.key_cache, b.value_cache, b.slot_mapping)
    out = torch.full_like(query, float("nan"))
    pa_prefill(out, query, b.key_cache, b.value_cache, b.block_tables, b.context_lens, starts,
               cfg.scale, max(qlens))
    torch.cuda.synchronize()
    pa_check_error()
    g = to_f64(out)
    assert np.isfinite(g).all()
    err = np.max(np.abs(g - ref))
    assert err <= TOL[cfg.dtype], f"{name}: {err:.3e}"


def test_prefill_of_one_token_equals_decode(cuda_device):
    from paged_kv_cache_444_b200 import pa_decode
    cfg = C["gqa_llama3_8b"].scaled(num_seqs=6, num_blocks=400, ctx=("uniform", 1, 900), seed=66)
    b = workloads.make_batch(cfg, cuda_device)
    starts = torch.arange(cfg.num_seqs + 1, dtype=torch.int32, device=cuda_device)
    out_p = torch.empty_like(b.query)
    out_d = torch.empty_like(b.query)
    pa_prefill(out_p, b.query, b.key_cache, b.value_cache, b.block_tables, b.context_lens,
               starts, cfg.scale, 1)
    pa_decode(out_d, b.query, b.key_cache, b.value_cache, b.block_tables, b.context_lens,
              cfg.scale)
    torch.cuda.synchronize()
    assert np.max(np.abs(to_f64(out_p) - to_f64(out_d))) <= TOL[cfg.dtype]


def test_prefill_reports_query_longer_than_context(cuda_device):
    cfg, b, query, starts, qlens = _case("gqa4_bf16", cuda_device)
    b.context_lens[1] = 3                                   # q_len 17 > 3
    out = torch.zeros_like(query)
    pa_prefill(out, query, b.key_cache, b.value_cache, b.block_tables, b.context_lens, starts,
               cfg.scale, max(qlens))
    with pytest.raises(PagedAttentionError) as e:
        pa_check_error()
    assert e.value.detail >> 56 == 7 and e.value.detail & 0xffff == 1
