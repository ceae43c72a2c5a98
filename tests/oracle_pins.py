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


def pin_copy_on_write_blocks(orc):
    """Copy-on-write ("vllm源码分析" 第一讲; "vLLM PagedAttention 原理与源码深度解析"
    §3.3): after copying a shared block to a private one, the private block
    holds the same bytes, the source is untouched, and every other block keeps
    its canary; attention of a sequence re-pointed at the copy is unchanged."""
    rng = np.random.default_rng(23)
    NB, bs, Hk, D = 10, 4, 2, 8
    kc = rng.integers(0, 65535, (NB, bs, Hk, D), dtype=np.uint16)
    vc = rng.integers(0, 65535, (NB, bs, Hk, D), dtype=np.uint16)
    kc = np.where(np.isnan(kc.view(np.float16)), 0x3c00, kc).astype(np.uint16)
    vc = np.where(np.isnan(vc.view(np.float16)), 0x3c00, vc).astype(np.uint16)
    kc = np.where(np.isinf(kc.view(np.float16)), 0x3c00, kc).astype(np.uint16)
    vc = np.where(np.isinf(vc.view(np.float16)), 0x3c00, vc).astype(np.uint16)
    k0, v0 = kc.copy(), vc.copy()
    pairs = np.array([[3, 7], [0, 9]], dtype=np.int64)
    assert orc.copy_blocks(kc, vc, pairs) == oracle_mod.OK
    for b in range(NB):
        src = {7: 3, 9: 0}.get(b, b)
        assert np.array_equal(kc[b], k0[src]) and np.array_equal(vc[b], v0[src])
    # a sequence reading block 3 reads the same values from its private copy 7
    q = rng.integers(0x3000, 0x3c00, (1, Hk, D), dtype=np.uint16)
    bt_shared = np.array([[1, 3]], dtype=np.int32)
    bt_private = np.array([[1, 7]], dtype=np.int32)
    cl = np.array([6], dtype=np.int32)
    a = orc.decode(q, kc, vc, bt_shared, cl, 0.3, F16)
    b = orc.decode(q, kc, vc, bt_private, cl, 0.3, F16)
    assert np.array_equal(a, b)
    bad = np.array([[2, NB]], dtype=np.int64)
    assert orc.copy_blocks(kc, vc, bad) == oracle_mod.BAD_BLOCK


def _e4m3_torch(codes: np.ndarray) -> np.ndarray:
    return torch.from_numpy(np.asarray(codes, dtype=np.uint8)).view(torch.float8_e4m3fn) \
        .to(torch.float64).numpy()


def pin_e4m3_decode_all_codes(orc):
    """E4M3 decode equals torch's float8_e4m3fn -> float64 cast on all 256 codes."""
    codes = np.arange(256, dtype=np.uint8)
    got = np.array([orc.e4m3_to_f64(c) for c in codes])
    want = _e4m3_torch(codes)
    assert np.array_equal(np.isnan(got), np.isnan(want))
    ok = ~np.isnan(want)
    assert np.array_equal(got[ok], want[ok])


def pin_e4m3_rounding(orc):
    """double -> E4M3 nearest-even equals torch's float32 -> float8_e4m3fn cast
    inside +-464 (ties included); beyond, finite values saturate to +-448."""
    rng = np.random.default_rng(29)
    xs = (rng.standard_normal(3000) * np.exp2(rng.integers(-12, 9, 3000))).astype(np.float32)
    xs = xs[np.abs(xs) < 464]
    grid = _e4m3_torch(np.arange(0, 127, dtype=np.uint8))
    ties = (grid[:-1] + grid[1:]) / 2                      # midpoints between neighbours
    xs = np.concatenate([xs.astype(np.float64), ties, -ties])
    want = torch.from_numpy(xs.astype(np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([orc.f64_to_e4m3(float(x)) for x in xs], dtype=np.uint8)
    assert np.array_equal(got, want)
    for x, code in [(464.0, 0x7e), (1e30, 0x7e), (float("inf"), 0x7e), (-500.0, 0xfe),
                    (float("nan"), 0x7f)]:
        assert orc.f64_to_e4m3(x) == code, x


def pin_fp8_write_worked_example(orc):
    """The quantising write puts token n of the worked example (block_size 4)
    at block (n-1) div 4, offset (n-1) mod 4, as E4M3 of x * (1/scale) taken
    in float (torch's float32 product and float8 cast), saturated; nothing
    else changes."""
    rows = read_golden("slot_mapping_example.txt")
    bs = int(rows[0][1])
    NB, Hk, D = 3, 2, 8
    rng = np.random.default_rng(31)
    key_f = (rng.standard_normal((9, Hk, D)) * 3).astype(np.float16)
    val_f = (rng.standard_normal((9, Hk, D)) * 3).astype(np.float16)
    key_f[0, 0, 0] = 1000.0                                 # saturates at 448 * scale
    key, value = key_f.view(np.uint16), val_f.view(np.uint16)
    kc = np.full((NB, bs, Hk, D), 0xaa, dtype=np.uint8)
    vc = np.full((NB, bs, Hk, D), 0x55, dtype=np.uint8)
    table = np.array([0, 1, 2], dtype=np.int32)
    slots = np.array([orc.slot(table, i, bs) for i in range(9)], dtype=np.int64)
    ks, vs = 0.75, 1.5
    assert orc.reshape_and_cache_fp8(key, value, kc, vc, slots, NB, bs, ks, vs, F16) == 0
    inv_k, inv_v = np.float32(1) / np.float32(ks), np.float32(1) / np.float32(vs)

    def q8(x16, inv):
        prod = torch.from_numpy(x16.astype(np.float32)) * torch.tensor(inv)
        prod = prod.clamp(-448, 448)                       # the write saturates
        return prod.to(torch.float8_e4m3fn).view(torch.uint8).numpy()

    ek = np.full_like(kc, 0xaa)
    ev = np.full_like(vc, 0x55)
    for token, index, block, offset in [tuple(map(int, r)) for r in rows[1:]]:
        ek[block, offset] = q8(key_f[index], inv_k)
        ev[block, offset] = q8(val_f[index], inv_v)
    assert np.array_equal(kc, ek) and np.array_equal(vc, ev)
    assert orc.e4m3_to_f64(kc[0, 0, 0, 0]) == 448.0


def pin_fp8_decode_sdpa(orc):
    """Decode over an E4M3 cache == torch SDPA (float64) over the dequantised
    K = code * k_scale, V = code * v_scale, gathered contiguously."""
    rng = np.random.default_rng(37)
    for S, H, Hk, D, bs, ctx, dt in [(3, 8, 2, 32, 4, [5, 13, 1], F16),
                                     (2, 4, 4, 16, 16, [40, 17], BF16)]:
        NB = sum((c + bs - 1) // bs for c in ctx) + 3
        kc = rng.integers(0, 255, (NB, bs, Hk, D), dtype=np.uint8)
        vc = rng.integers(0, 255, (NB, bs, Hk, D), dtype=np.uint8)
        kc[(kc & 0x7f) == 0x7f] = 0x30                      # no NaN codes
        vc[(vc & 0x7f) == 0x7f] = 0x31
        tdt = torch.bfloat16 if dt == BF16 else torch.float16
        q = _bits(torch.randn((S, H, D), generator=torch.Generator().manual_seed(S)).to(tdt))
        perm = rng.permutation(NB).astype(np.int32)
        MB = max((c + bs - 1) // bs for c in ctx)
        bt = np.full((S, MB), -1, dtype=np.int32)
        cur = 0
        for s_, c in enumerate(ctx):
            nb = (c + bs - 1) // bs
            bt[s_, :nb] = perm[cur:cur + nb]
            cur += nb
        cl = np.asarray(ctx, dtype=np.int32)
        ks, vs = 0.02, 0.05
        got = orc.decode_fp8(q, kc, vc, bt, cl, 0.2, ks, vs, dt)
        kd = torch.from_numpy(_e4m3_torch(kc) * ks)
        vd = torch.from_numpy(_e4m3_torch(vc) * vs)
        qd = torch.from_numpy(q.view(np.int16)).view(tdt).to(torch.float64)
        for s_ in range(S):
            nb = (ctx[s_] + bs - 1) // bs
            idx = torch.from_numpy(bt[s_, :nb].astype(np.int64))
            k = kd[idx].reshape(nb * bs, Hk, D)[:ctx[s_]].permute(1, 0, 2)[None]
            v = vd[idx].reshape(nb * bs, Hk, D)[:ctx[s_]].permute(1, 0, 2)[None]
            o = F.scaled_dot_product_attention(qd[s_][None, :, None, :], k, v, scale=0.2,
                                               enable_gqa=True)[0, :, 0, :]
            assert np.max(np.abs(got[s_] - o.numpy())) <= 1e-12


def pin_prefill_causal_sdpa(orc):
    """Chunked prefill: the last q_len positions of each sequence attend
    causally over their context.  Equals torch SDPA (float64) with an
    explicit mask j <= position on contiguously gathered K/V; q_len = 1
    equals decode."""
    rng = np.random.default_rng(41)
    for S, H, Hk, D, bs, ctx, qlen, dt in [(3, 4, 2, 16, 4, [9, 17, 5], [3, 17, 1], F16),
                                           (2, 8, 8, 8, 16, [40, 33], [12, 1], BF16)]:
        NB = sum((c + bs - 1) // bs for c in ctx) + 2
        q, kc, vc, bt, cl = _random_case(rng, S, H, Hk, D, bs, NB, ctx, dt)
        tdt = torch.bfloat16 if dt == BF16 else torch.float16
        T = sum(qlen)
        gq = torch.Generator().manual_seed(T)
        qt = _bits(torch.randn((T, H, D), generator=gq).to(tdt))
        starts = np.concatenate([[0], np.cumsum(qlen)]).astype(np.int32)
        got = orc.prefill(qt, kc, vc, bt, cl, starts, 0.3, dt)
        to64 = lambda b: torch.from_numpy(b.view(np.int16)).view(tdt).to(torch.float64)
        kd, vd, qd = to64(kc), to64(vc), to64(qt)
        for s_ in range(S):
            c, ql = ctx[s_], qlen[s_]
            nb = (c + bs - 1) // bs
            idx = torch.from_numpy(bt[s_, :nb].astype(np.int64))
            k = kd[idx].reshape(nb * bs, Hk, D)[:c].permute(1, 0, 2)[None]
            v = vd[idx].reshape(nb * bs, Hk, D)[:c].permute(1, 0, 2)[None]
            pos = torch.arange(c - ql, c)
            mask = (torch.arange(c)[None, :] <= pos[:, None])[None, None]
            qq = qd[starts[s_]:starts[s_ + 1]].permute(1, 0, 2)[None]
            o = F.scaled_dot_product_attention(qq, k, v, attn_mask=mask, scale=0.3,
                                               enable_gqa=True)[0].permute(1, 0, 2)
            assert np.max(np.abs(got[starts[s_]:starts[s_ + 1]] - o.numpy())) <= 1e-12
        # one query per sequence at its last position is decode
        ones = np.arange(S + 1, dtype=np.int32)
        last = np.stack([qt[starts[i + 1] - 1] for i in range(S)])
        dec = orc.decode(last, kc, vc, bt, cl, 0.3, dt)
        pre = orc.prefill(last, kc, vc, bt, cl, ones, 0.3, dt)
        assert np.array_equal(dec, pre)


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
    pin_copy_on_write_blocks,
    pin_e4m3_decode_all_codes,
    pin_e4m3_rounding,
    pin_fp8_write_worked_example,
    pin_fp8_decode_sdpa,
    pin_prefill_causal_sdpa,
]
