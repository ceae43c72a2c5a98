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
    # many 128-key blocks per tile: the K/V stage rings wrap several times
    "long_gqa4_bf16": (C["gqa_llama3_8b"], dict(num_seqs=3, num_heads=8, num_kv_heads=2,
                                               num_blocks=500, ctx=("fixed", (3000, 1500, 777)),
                                               seed=67), (512, 200, 777)),
    "long_mha_f16_d64": (C["tiny"], dict(num_seqs=2, num_heads=2, num_kv_heads=2, num_blocks=300,
                                         ctx=("fixed", (2500, 1100)), seed=68), (300, 1100)),
}


def _mixed(seed, n, ctx_hi, q_hi):
    """n contexts U[1, ctx_hi) and query lengths U[0, q_hi] capped by them
    (some sequences bring no query tokens)."""
    rng = np.random.default_rng(seed)
    ctx = [int(c) for c in rng.integers(1, ctx_hi, n)]
    q = [0 if rng.random() < 0.15 else int(min(c, rng.integers(1, q_hi + 1))) for c in ctx]
    return tuple(ctx), tuple(q)


# 40 sequences: the longest-first order ranks units with many equal key counts
# and empty sequences among them
_ctx, _q = _mixed(444_071, 40, 300, 70)
CASES["many_seqs_gqa4_bf16"] = (C["gqa_llama3_8b"], dict(num_seqs=40, num_heads=8,
                                                          num_kv_heads=2, num_blocks=1000,
                                                          ctx=("fixed", _ctx), seed=71), _q)
# more sequences than the longest-first order ranks: the fixed order instead
_ctx, _q = _mixed(444_072, 300, 48, 6)
CASES["fixed_order_300_seqs_f16"] = (C["gqa_llama3_8b"], dict(num_seqs=300, num_heads=4,
                                                               num_kv_heads=2, dtype="f16",
                                                               num_blocks=1200,
                                                               ctx=("fixed", _ctx), seed=72), _q)
# few enough sequences to rank, but too many units x sequences to count: the
# fixed order again, with the sequences checked while the units are counted
_ctx, _q = _mixed(444_073, 100, 500, 300)
CASES["fixed_order_100_seqs_bf16"] = (C["gqa_llama3_8b"], dict(num_seqs=100, num_heads=4,
                                                                num_kv_heads=1, num_blocks=3600,
                                                                ctx=("fixed", _ctx), seed=73), _q)
_units = sum(-(-q // (2 * 32)) for q in _q)                # tile pairs of 2 x 32 tokens
assert _units <= 2048 and _units * 100 > 16384, _units

# a step that mixes decodes with long chunks: 700 sequences (two per thread's
# chunk in the sequence-major order), nearly all bringing one query token, four
# bringing hundreds; the long ones set max_query_len, so most (sequence, pair)
# slots are empty and only the units that exist are walked
_rng = np.random.default_rng(444_074)
_ctx = [int(c) for c in _rng.integers(1, 300, 700)]
_q = [1] * 700
for _i, _n in ((3, 900), (256, 513), (511, 700), (699, 64)):
    _ctx[_i] = _n + int(_rng.integers(0, 400))
    _q[_i] = _n
CASES["mixed_700_seqs_bf16"] = (C["gqa_llama3_8b"], dict(num_seqs=700, num_heads=8,
                                                          num_kv_heads=2, num_blocks=9000,
                                                          ctx=("fixed", tuple(_ctx)), seed=74),
                                 tuple(_q))

# scale 1 instead of 1/sqrt(D): peaked rows whose running maximum jumps by more
# than 2^8 between key blocks, so the output accumulator is rescaled
SCALE = {"peaky_bf16": 1.0, "peaky_f16": 1.0}
CASES["peaky_bf16"] = (C["gqa_llama3_8b"], dict(num_seqs=2, num_heads=8, num_kv_heads=2,
                                                 num_blocks=300, ctx=("fixed", (1200, 640)),
                                                 seed=69), (400, 640))
CASES["peaky_f16"] = (C["gqa_llama3_8b"], dict(num_seqs=2, num_heads=8, num_kv_heads=2,
                                                dtype="f16", num_blocks=300,
                                                ctx=("fixed", (1200, 333)), seed=70), (150, 333))


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


def _poison_past_context(b):
    """Fill every cache row past each sequence's context in its last block
    with NaN (the kernel masks those keys, and must not let 0 * NaN through)."""
    cfg = b.cfg
    bt = b.block_tables.cpu().numpy()
    for s_, c in enumerate(b.context_lens.cpu().tolist()):
        if c % cfg.block_size:
            blk = int(bt[s_, (c - 1) // cfg.block_size])
            b.key_cache[blk, c % cfg.block_size:] = float("nan")
            b.value_cache[blk, c % cfg.block_size:] = float("nan")


# every layout as drawn, and a subset again with NaN in the rows past each context
PREFILL_RUNS = [pytest.param(n, False, id=n) for n in CASES] + [
    pytest.param(n, True, id=f"{n}-nan_past_ctx")
    for n in ("gqa4_bf16", "mha_f16", "gqa3_f16", "long_mha_f16_d64")]


@pytest.mark.parametrize("name,poison", PREFILL_RUNS)
def test_prefill_matches_oracle(name, poison, cuda_device, oracle_lib):
    cfg, b, query, starts, qlens = _case(name, cuda_device)
    scale = SCALE.get(name, cfg.scale)
    if poison:
        _poison_past_context(b)
    # write the step's last token first (any earlier prompt rows are already random cache)
    kc = bits(b.key_cache).copy()
    vc = bits(b.value_cache).copy()
    assert oracle_lib.reshape_and_cache(bits(b.key), bits(b.value), kc, vc,
                                        b.slot_mapping.cpu().numpy(), cfg.num_blocks,
                                        cfg.block_size) == 0
    ref = oracle_lib.prefill(bits(query), kc, vc, b.block_tables.cpu().numpy(),
                             b.context_lens.cpu().numpy(), starts.cpu().numpy(), scale,
                             ocode(cfg))
    pa_reshape_and_cache(b.key, b.value, b.key_cache, b.value_cache, b.slot_mapping)
    out = torch.full_like(query, float("nan"))
    pa_prefill(out, query, b.key_cache, b.value_cache, b.block_tables, b.context_lens, starts,
               scale, max(qlens))
    torch.cuda.synchronize()
    pa_check_error()
    g = to_f64(out)
    assert np.isfinite(g).all()
    bound = TOL[cfg.dtype]
    if name in SCALE:
        # peaked rows give outputs past |4|, where rounding to the 16-bit output
        # alone costs up to half an ulp: 2^-8 |out| (bf16), 2^-11 |out| (fp16)
        bound = bound + (2.0 ** -8 if cfg.dtype == "bf16" else 2.0 ** -11) * np.abs(ref)
    excess = np.max(np.abs(g - ref) - bound)
    assert excess <= 0, f"{name}: error exceeds the bound by {excess:.3e}"


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


def test_prefill_bf16_reports_v_beyond_fp16_range(cuda_device, oracle_lib):
    """bf16 V blocks are rewritten as fp16 in shared memory for the P V
    product; a V value beyond the fp16 range saturates to +-65504 and is
    reported with its sequence (PA_CHECK_VALUE).  The other sequences'
    outputs still match the oracle."""
    cfg, b, query, starts, qlens = _case("gqa4_bf16", cuda_device)
    s_bad = 2
    blk = int(b.block_tables[s_bad, 3])
    b.value_cache[blk, 5, 1, 17] = 1.0e5                     # in context (ctx 300)
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
    with pytest.raises(PagedAttentionError) as e:
        pa_check_error()
    assert e.value.detail >> 56 == 8 and e.value.detail & 0xffff == s_bad
    st = starts.cpu().tolist()
    keep = [t for i in range(len(qlens)) if i != s_bad for t in range(st[i], st[i + 1])]
    g = to_f64(out)
    assert np.max(np.abs(g[keep] - ref[keep])) <= TOL[cfg.dtype]


def test_prefill_reports_invalid_sequence_in_fixed_order(cuda_device):
    """Past 256 sequences the units go out in the fixed order; an invalid
    sequence is still skipped and reported, and the others are written."""
    cfg, b, query, starts, qlens = _case("fixed_order_300_seqs_f16", cuda_device)
    bad = next(i for i, q in enumerate(qlens) if q > 0 and i > 200)
    b.context_lens[bad] = qlens[bad] - 1                    # q_len > context
    out = torch.zeros_like(query)
    pa_prefill(out, query, b.key_cache, b.value_cache, b.block_tables, b.context_lens, starts,
               cfg.scale, max(qlens))
    with pytest.raises(PagedAttentionError) as e:
        pa_check_error()
    assert e.value.detail >> 56 == 7 and e.value.detail & 0xffff == bad


def test_prefill_full_size_sampled(cuda_device, oracle_lib):
    """The chunked-prefill layer bench.py times (8 sequences x 512-token chunks,
    32/8 heads, bf16), in the same launch, checked on samples the oracle
    computes in seconds: the whole chunk of the shortest-context sequence, and
    the last 64 query tokens of the longest (their positions are those of the
    full chunk when they are given as a 64-token chunk of the same context)."""
    pb = workloads.make_prefill_batch(device=cuda_device)
    b, cfg, chunk = pb.cache, pb.cache.cfg, pb.chunk
    out = torch.full_like(pb.query, float("nan"))
    pa_prefill(out, pb.query, b.key_cache, b.value_cache, b.block_tables, b.context_lens,
               pb.query_starts, cfg.scale, chunk)
    torch.cuda.synchronize()
    pa_check_error()
    g = to_f64(out)
    assert np.isfinite(g).all()
    ctx = b.context_lens.cpu().numpy()
    bt = b.block_tables.cpu().numpy()
    for s, t0 in ((int(np.argmin(ctx)), 0), (int(np.argmax(ctx)), chunk - 64)):
        n = (int(ctx[s]) + 15) // 16
        ids = torch.tensor(bt[s, :n], dtype=torch.long, device=cuda_device)
        kc = bits(b.key_cache.index_select(0, ids))
        vc = bits(b.value_cache.index_select(0, ids))
        rows = slice(s * chunk + t0, (s + 1) * chunk)
        ref = oracle_lib.prefill(bits(pb.query[rows]), kc, vc,
                                 np.arange(n, dtype=np.int32)[None, :],
                                 ctx[s:s + 1].astype(np.int32),
                                 np.array([0, chunk - t0], dtype=np.int32), cfg.scale,
                                 ocode(cfg))
        err = np.max(np.abs(g[rows] - ref))
        assert err <= TOL[cfg.dtype], f"seq {s} tokens {t0}..{chunk}: {err:.3e}"
