"""Pins of the fp64 oracle to facts that do not come from the oracle itself.

Every pin takes an ``oracle.Oracle`` so the mutation tests can run the same
checks against deliberately broken copies of the oracle.  Each one names the
fact it rests on: a value printed on a page (golden fixtures with their
citation), a library routine (numpy float16 casts, torch bfloat16 casts,
torch's scaled_dot_product_attention in float64), a closed form, or an
invariant of paging.

Pages:
  "vllm源码剖析" (jsqmd.com)  -- §一.2 cache layout and reshape; §一.3 slot
      mapping worked example; §一.6 page sizing.
  "vLLM PagedAttention 原理与源码深度解析" (toukenai.cn) -- §2.1 KV bytes per
      token; §3.1 block table; §3.3 shared blocks (ref_count); §5.3 attention.
"""
from __future__ import annotations

import math

import numpy as np
import torch
import torch.nn.functional as F

import oracle as oracle_mod
from conftest import read_golden

F16, BF16 = oracle_mod.F16, oracle_mod.BF16


# ---------------------------------------------------------------- helpers --
def _bits(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def _random_case(rng: np.random.Generator, S, H, Hk, D, bs, NB, ctx_list, dtype):
    tdt = torch.bfloat16 if dtype == BF16 else torch.float16
    g = torch.Generator().manual_seed(int(rng.integers(1 << 30)))
    kc = torch.randn((NB, bs, Hk, D), generator=g).to(tdt)
    vc = torch.randn((NB, bs, Hk, D), generator=g).to(tdt)
    q = torch.randn((S, H, D), generator=g).to(tdt)
    MB = max(1, max((c + bs - 1) // bs for c in ctx_list))
    perm = rng.permutation(NB).astype(np.int32)
    bt = np.full((S, MB), -1, dtype=np.int32)
    cur = 0
    for s, c in enumerate(ctx_list):
        nb = (c + bs - 1) // bs
        bt[s, :nb] = perm[cur:cur + nb]
        cur += nb
    assert cur <= NB
    return _bits(q), _bits(kc), _bits(vc), bt, np.asarray(ctx_list, dtype=np.int32)


def _sdpa_reference(q_bits, kc_bits, vc_bits, bt, ctx, scale, dtype):
    """torch's scaled_dot_product_attention (float64, GQA via enable_gqa) on
    K/V gathered out of the block tables with numpy fancy indexing."""
    tdt = torch.bfloat16 if dtype == BF16 else torch.float16
    to64 = lambda b: torch.from_numpy(b.view(np.int16)).view(tdt).to(torch.float64)
    q = to64(q_bits)
    kc = to64(kc_bits)
    vc = to64(vc_bits)
    S, H, D = q.shape
    NB, bs, Hk, _ = kc.shape
    out = torch.zeros((S, H, D), dtype=torch.float64)
    for s in range(S):
        c = int(ctx[s])
        if c == 0:
            continue
        nb = (c + bs - 1) // bs
        k = kc[torch.from_numpy(bt[s, :nb].astype(np.int64))].reshape(nb * bs, Hk, D)[:c]
        v = vc[torch.from_numpy(bt[s, :nb].astype(np.int64))].reshape(nb * bs, Hk, D)[:c]
        o = F.scaled_dot_product_attention(
            q[s][None, :, None, :], k.permute(1, 0, 2)[None], v.permute(1, 0, 2)[None],
            scale=scale, enable_gqa=True)
        out[s] = o[0, :, 0, :]
    return out.numpy()


# ------------------------------------------------------------------- pins --
def pin_f16_decode_all_patterns(orc):
    """binary16 decode equals numpy's float16 -> float64 cast on all 2^16 patterns."""
    bits = np.arange(65536, dtype=np.uint16)
    got = orc.decode_bits(bits, F16)
    want = bits.view(np.float16).astype(np.float64)
    assert np.array_equal(np.isnan(got), np.isnan(want))
    ok = ~np.isnan(want)
    assert np.array_equal(got[ok], want[ok])


def pin_bf16_decode_all_patterns(orc):
    """bfloat16 decode equals torch's bfloat16 -> float64 cast on all 2^16 patterns."""
    bits = np.arange(65536, dtype=np.uint16)
    got = orc.decode_bits(bits, BF16)
    want = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(np.isnan(got), np.isnan(want))
    ok = ~np.isnan(want)
    assert np.array_equal(got[ok], want[ok])


def pin_f16_rounding(orc):
    """double -> binary16 nearest-even equals numpy's float64 -> float16 cast,
    including subnormals, exact ties and the overflow threshold."""
    rng = np.random.default_rng(7)
    xs = list(rng.standard_normal(2000) * np.exp2(rng.integers(-26, 17, 2000)))
    # ties: midpoints between neighbouring binary16 values
    for b in [0x3c00, 0x3c01, 0x0001, 0x0002, 0x03ff, 0x7bfe, 0x4000, 0x1234]:
        lo = float(np.uint16(b).view(np.float16))
        hi = float(np.uint16(b + 1).view(np.float16))
        xs += [(lo + hi) / 2, -(lo + hi) / 2]
    xs += [65504.0, 65519.99, 65520.0, 1e6, -0.0, 0.0, 2.0 ** -25, 2.0 ** -26, 3 * 2.0 ** -26]
    for x in xs:
        with np.errstate(over="ignore"):
            want = int(np.array(x, dtype=np.float64).astype(np.float16).view(np.uint16))
        assert orc.f64_to_f16(x) == want, (x, hex(orc.f64_to_f16(x)), hex(want))


def pin_bf16_rounding(orc):
    """double -> bfloat16 nearest-even equals torch's float32 -> bfloat16 cast
    on float32-representable inputs (one rounding only), ties included."""
    rng = np.random.default_rng(11)
    xs = (rng.standard_normal(2000) * np.exp2(rng.integers(-130, 120, 2000))).astype(np.float32)
    ties = [1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, -(1.0 + 2.0 ** -8), 2.0 ** -133,
            3 * 2.0 ** -134, 3.3895313892515355e38, 3.3961775292304957e38]
    xs = list(xs.astype(np.float64)) + ties
    for x in xs:
        want = int(torch.tensor([x], dtype=torch.float32).to(torch.bfloat16)
                   .view(torch.int16).item()) & 0xffff
        assert orc.f64_to_bf16(float(np.float32(x))) == want, (x, hex(want))


def pin_slot_worked_example(orc):
    """Slots of the page's worked example (block_size 4, tokens 1..9)."""
    rows = read_golden("slot_mapping_example.txt")
    bs = int(rows[0][1])
    table = np.array([0, 1, 2], dtype=np.int32)  # identity: logical block == physical block
    for token, index, block, offset in [tuple(map(int, r)) for r in rows[1:]]:
        assert index == token - 1
        assert orc.slot(table, index, bs) == block * bs + offset
    # a non-identity table moves whole blocks, never offsets
    table = np.array([5, 2, 7], dtype=np.int32)
    for token, index, block, offset in [tuple(map(int, r)) for r in rows[1:]]:
        assert orc.slot(table, index, bs) == int(table[block]) * bs + offset


def pin_kv_bytes_closed_form(orc):
    """512 KB per token and 1 GB per 2048-token sequence (32/32/128 fp16)."""
    for L, Hk, D, e, n, per_tok, per_seq in [tuple(map(int, r)) for r in
                                             read_golden("kv_bytes_closed_form.txt")]:
        assert orc.kv_bytes_per_token(L, Hk, D, e) == per_tok
        assert orc.kv_bytes_per_token(L, Hk, D, e) * n == per_seq


def pin_page_sizing(orc):
    """page_size and num_blocks of the sizing rule, consistent with the
    per-token closed form of the other page."""
    for Hk, D, e, bs, L, avail, page, nblk in [tuple(map(int, r)) for r in
                                               read_golden("page_size_sizing.txt")]:
        assert orc.page_size_bytes(Hk, D, e, bs) == page
        assert orc.num_blocks(avail, page, L) == nblk
        assert page * L // bs == orc.kv_bytes_per_token(L, Hk, D, e)


def pin_write_worked_example(orc):
    """Writing tokens 1..9 of the worked example (block_size 4, 1 KV head,
    head_dim 8) puts token n's row at block (n-1) div 4, offset (n-1) mod 4,
    and nothing else in the cache changes (canary fill)."""
    rows = read_golden("slot_mapping_example.txt")
    bs = int(rows[0][1])
    NB, Hk, D = 3, 1, 8
    canary = np.uint16(0x7e5a)
    kc = np.full((NB, bs, Hk, D), canary, dtype=np.uint16)
    vc = np.full((NB, bs, Hk, D), canary, dtype=np.uint16)
    key = np.arange(9 * Hk * D, dtype=np.uint16).reshape(9, Hk, D) + 1
    value = key + 1000
    table = np.array([0, 1, 2], dtype=np.int32)
    slots = np.array([orc.slot(table, i, bs) for i in range(9)], dtype=np.int64)
    assert orc.reshape_and_cache(key, value, kc, vc, slots, NB, bs) == oracle_mod.OK
    expect_k = np.full_like(kc, canary)
    expect_v = np.full_like(vc, canary)
    for token, index, block, offset in [tuple(map(int, r)) for r in rows[1:]]:
        expect_k[block, offset] = key[index]
        expect_v[block, offset] = value[index]
    assert np.array_equal(kc, expect_k) and np.array_equal(vc, expect_v)


def pin_write_padding_and_strides(orc):
    """Negative slots are skipped, strided key/value rows are honoured, every
    untouched byte keeps its canary value."""
    rng = np.random.default_rng(3)
    NB, bs, Hk, D, T = 6, 4, 2, 16, 7
    big_k = rng.integers(0, 65535, (T, 3 * Hk * D), dtype=np.uint16)
    big_v = rng.integers(0, 65535, (T, 3 * Hk * D), dtype=np.uint16)
    key = big_k[:, :Hk * D].reshape(T, Hk, D)             # row stride 3*Hk*D
    value = big_v[:, Hk * D:2 * Hk * D].reshape(T, Hk, D)
    slots = np.array([0, -1, 23, 5, -7, 12, 17], dtype=np.int64)
    kc = np.full((NB, bs, Hk, D), 0xabcd, dtype=np.uint16)
    vc = np.full((NB, bs, Hk, D), 0xdcba, dtype=np.uint16)
    assert orc.reshape_and_cache(key, value, kc, vc, slots, NB, bs) == oracle_mod.OK
    fk = kc.reshape(NB * bs, Hk, D)
    fv = vc.reshape(NB * bs, Hk, D)
    written = set()
    for t, s in enumerate(slots):
        if s >= 0:
            assert np.array_equal(fk[s], key[t]) and np.array_equal(fv[s], value[t])
            written.add(int(s))
    for s in range(NB * bs):
        if s not in written:
            assert (fk[s] == 0xabcd).all() and (fv[s] == 0xdcba).all()
    bad = np.array([NB * bs], dtype=np.int64)
    assert orc.reshape_and_cache(key[:1], value[:1], kc, vc, bad, NB, bs) == oracle_mod.BAD_SLOT


def pin_bruteforce_sdpa(orc):
    """Paged oracle == torch SDPA (float64) over K/V gathered contiguously, on
    tiny random cases: block sizes 1, 4, 16; MHA and GQA groups 2 and 4;
    ragged lengths that end inside a block."""
    rng = np.random.default_rng(2024)
    cases = [
        (3, 4, 4, 16, 1, 64, [1, 5, 17], F16),
        (4, 8, 2, 32, 4, 40, [3, 4, 9, 40], BF16),
        (2, 8, 4, 64, 16, 8, [37, 16], F16),
        (4, 4, 1, 8, 4, 64, [13, 2, 31, 8], BF16),
    ]
    for S, H, Hk, D, bs, NB, ctx, dt in cases:
        q, kc, vc, bt, cl = _random_case(rng, S, H, Hk, D, bs, NB, ctx, dt)
        scale = 1.0 / math.sqrt(D)
        got = orc.decode(q, kc, vc, bt, cl, scale, dt)
        want = _sdpa_reference(q, kc, vc, bt, cl, scale, dt)
        assert np.max(np.abs(got - want)) <= 1e-12, (S, H, Hk, D, bs)


def pin_permutation_invariance(orc):
    """Relabelling physical blocks by any permutation (moving the cache rows
    with them) leaves the output bit-identical: only the logical order counts."""
    rng = np.random.default_rng(5)
    S, H, Hk, D, bs, NB = 3, 4, 2, 16, 4, 24
    q, kc, vc, bt, cl = _random_case(rng, S, H, Hk, D, bs, NB, [7, 12, 21], F16)
    base = orc.decode(q, kc, vc, bt, cl, 0.25, F16)
    pi = rng.permutation(NB)
    kc2 = np.empty_like(kc)
    vc2 = np.empty_like(vc)
    kc2[pi] = kc
    vc2[pi] = vc
    bt2 = np.where(bt >= 0, pi[np.maximum(bt, 0)], -1).astype(np.int32)
    got = orc.decode(q, kc2, vc2, bt2, cl, 0.25, F16)
    assert np.array_equal(base, got)
    # and the relabelling does change the result when the rows stay put
    bad = orc.decode(q, kc, vc, bt2, cl, 0.25, F16)
    assert not np.array_equal(base, bad)


def pin_shared_prefix_equals_private(orc):
    """Sequences that share prefix blocks (same ids, ref_count > 1) give the
    same output as the same sequences with private copies of the prefix."""
    rng = np.random.default_rng(9)
    Hk, H, D, bs = 2, 4, 16, 4
    NB = 40
    g = torch.Generator().manual_seed(1)
    kc = _bits(torch.randn((NB, bs, Hk, D), generator=g).half())
    vc = _bits(torch.randn((NB, bs, Hk, D), generator=g).half())
    q = _bits(torch.randn((4, H, D), generator=g).half())
    ctx = np.array([13, 10, 15, 9], dtype=np.int32)
    prefix = [3, 17]                      # shared by all four
    tails = [[5, 8], [11], [20, 21], [30]]
    bt = np.full((4, 4), -1, dtype=np.int32)
    for s in range(4):
        row = prefix + tails[s]
        bt[s, :len(row)] = row
    shared = orc.decode(q, kc, vc, bt, ctx, 0.3, F16)
    kc2, vc2, bt2 = kc.copy(), vc.copy(), bt.copy()
    free = [33, 34, 35, 36, 37, 38]
    for s in range(1, 4):
        for i, b in enumerate(prefix):
            nb = free.pop(0)
            kc2[nb] = kc[b]
            vc2[nb] = vc[b]
            bt2[s, i] = nb
    private = orc.decode(q, kc2, vc2, bt2, ctx, 0.3, F16)
    assert np.array_equal(shared, private)
    assert rng is not None


def pin_closed_forms(orc):
    """ctx = 1 returns v exactly; equal keys or scale = 0 give the mean of v;
    constant v returns that constant."""
    rng = np.random.default_rng(13)
    S, H, Hk, D, bs, NB = 2, 4, 2, 16, 4, 16
    q, kc, vc, bt, _ = _random_case(rng, S, H, Hk, D, bs, NB, [1, 11], BF16)
    G = H // Hk
    one = orc.decode(q, kc, vc, bt, np.array([1, 1], np.int32), 0.7, BF16)
    for s in range(S):
        v0 = orc.decode_bits(vc[bt[s, 0], 0], BF16)             # [Hk, D]
        for h in range(H):
            assert np.array_equal(one[s, h], v0[h // G])
    cl = np.array([1, 11], dtype=np.int32)
    # scale = 0 -> uniform weights
    uni = orc.decode(q, kc, vc, bt, cl, 0.0, BF16)
    flat_v = orc.decode_bits(vc, BF16).reshape(NB * bs, Hk, D)
    for s in range(S):
        rows = [int(bt[s, j // bs]) * bs + j % bs for j in range(int(cl[s]))]
        mean = flat_v[rows].mean(axis=0)
        for h in range(H):
            assert np.allclose(uni[s, h], mean[h // G], rtol=0, atol=1e-14)
    # identical keys -> uniform weights whatever the scale
    kc_eq = kc.copy()
    kc_eq[:] = kc[0, 0]
    eq = orc.decode(q, kc_eq, vc, bt, cl, 1.3, BF16)
    assert np.max(np.abs(eq - uni)) <= 1e-14
    # constant values -> that constant
    vc_c = np.full_like(vc, 0x3fc0)                              # bf16 1.5
    c = orc.decode(q, kc, vc_c, bt, cl, 0.9, BF16)
    assert np.max(np.abs(c - 1.5)) <= 1e-14


def pin_context_mask(orc):
    """Rows past ctx in the tail block and block-table entries past
    ceil(ctx / bs) do not change the output; ctx = 0 gives zeros."""
    rng = np.random.default_rng(17)
    S, H, Hk, D, bs, NB = 2, 2, 1, 8, 4, 12
    q, kc, vc, bt, cl = _random_case(rng, S, H, Hk, D, bs, NB, [6, 9], F16)
    base = orc.decode(q, kc, vc, bt, cl, 0.5, F16)
    kc2, vc2 = kc.copy(), vc.copy()
    for s in range(S):
        c = int(cl[s])
        last = int(bt[s, (c - 1) // bs])
        for r in range(c % bs or bs, bs):
            kc2[last, r] = 0x7bff
            vc2[last, r] = 0xfbff
    bt2 = np.concatenate([bt, np.full((S, 3), 1 << 30, np.int32)], axis=1)
    got = orc.decode(q, kc2, vc2, bt2, cl, 0.5, F16)
    assert np.array_equal(base, got)
    zero = orc.decode(q, kc, vc, bt, np.array([0, 9], np.int32), 0.5, F16)
    assert (zero[0] == 0).all() and np.array_equal(zero[1], base[1])


def pin_partition_merge(orc):
    """Log-sum-exp merge of partitions equals the single pass (within 1e-12)
    for several partition sizes; one partition covering everything equals it
    exactly up to the final division."""
    rng = np.random.default_rng(19)
    S, H, Hk, D, bs, NB = 3, 4, 2, 16, 4, 48
    q, kc, vc, bt, cl = _random_case(rng, S, H, Hk, D, bs, NB, [5, 33, 64], BF16)
    single = orc.decode(q, kc, vc, bt, cl, 0.35, BF16)
    for ps in [4, 8, 12, 32, 64]:
        P = (int(cl.max()) + ps - 1) // ps
        acc, pmax, psum = orc.decode_partitioned(q, kc, vc, bt, cl, 0.35, BF16, ps, P)
        merged = orc.lse_merge(acc, pmax, psum, cl, ps)
        assert np.max(np.abs(merged - single)) <= 1e-12, ps
        for s in range(S):
            n = (int(cl[s]) + ps - 1) // ps
            assert np.isfinite(pmax[s, :, :n]).all() and np.isnan(pmax[s, :, n:]).all()
            assert (psum[s, :, :n] >= 1.0).all()          # the max term contributes exp(0)
    acc, pmax, psum = orc.decode_partitioned(q, kc, vc, bt, cl, 0.35, BF16, 64, 1)
    assert np.max(np.abs(acc[:, :, 0] / psum[:, :, 0, None] - single)) <= 1e-14


ALL_PINS = [
    pin_f16_decode_all_patterns,
    pin_bf16_decode_all_patterns,
    pin_f16_rounding,
    pin_bf16_rounding,
    pin_slot_worked_example,
    pin_kv_bytes_closed_form,
    pin_page_sizing,
    pin_write_worked_example,
    pin_write_padding_and_strides,
    pin_bruteforce_sdpa,
    pin_permutation_invariance,
    pin_shared_prefix_equals_private,
    pin_closed_forms,
    pin_context_mask,
    pin_partition_merge,
]
