"""Seeded synthetic decode workloads.

The one module that both sides of every parity check read: it draws the
inputs (context lengths, block tables, slot mappings, 16-bit K/V/Q values)
and holds none of the attention arithmetic.  Values are drawn as float32
normals from a seeded ``torch.Generator`` and cast to the cache dtype with
round-to-nearest-even; the cast bits are the ground truth for both sides.

The five workload shapes are the decode batches the pages talk about (a
Llama-2-7B MHA layer, a Llama-3-8B GQA layer, 16-token blocks, shared beam
prefixes); none of the pages measures on a dataset, so none is needed.

Layouts (the pages' own, "vllm源码剖析" §一.2):
  key_cache, value_cache  [num_blocks, block_size, num_kv_heads, head_dim]
  block_tables            [num_seqs, max_blocks_per_seq] int32, unused = -1
  context_lens            [num_seqs] int32 (includes the token written this step)
  query                   [num_seqs, num_heads, head_dim]
  key, value (new token)  [num_seqs, num_kv_heads, head_dim]
  slot_mapping            [num_seqs] int64, slot of position context_lens-1
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field, replace

import torch

DTYPES = {"f16": torch.float16, "bf16": torch.bfloat16}


@dataclass(frozen=True)
class DecodeConfig:
    name: str
    num_seqs: int
    num_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    num_blocks: int
    dtype: str                       # "f16" | "bf16"
    ctx: tuple                       # ("fixed", (..)) | ("uniform", lo, hi) | ("lognormal", mean, sigma, lo, hi)
    seed: int
    partition_size: int = 0          # > 0: long-context split path
    shared_prefix_blocks: int = 0    # > 0: groups share their first blocks
    share_group: int = 1             # sequences per sharing group
    write_new_token: bool = True     # cache write of one token per sequence first
    description: str = ""

    @property
    def group_size(self) -> int:
        return self.num_heads // self.num_kv_heads

    @property
    def torch_dtype(self) -> torch.dtype:
        return DTYPES[self.dtype]

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.head_dim)

    def scaled(self, **changes) -> "DecodeConfig":
        return replace(self, **changes)


CONFIGS: dict[str, DecodeConfig] = {
    "tiny": DecodeConfig(
        name="tiny", num_seqs=4, num_heads=4, num_kv_heads=4, head_dim=64,
        block_size=16, num_blocks=64, dtype="f16", ctx=("fixed", (1, 9, 16, 37)),
        seed=444_001,
        description="4 seqs, ctx {1,9,16,37}, 4/4 heads, d=64, fp16, 64 blocks"),
    "mha_llama2_7b": DecodeConfig(
        name="mha_llama2_7b", num_seqs=32, num_heads=32, num_kv_heads=32, head_dim=128,
        block_size=16, num_blocks=8192, dtype="f16", ctx=("uniform", 256, 2048),
        seed=444_002,
        description="Llama-2-7B-shaped MHA decode layer: 32 seqs, 32/32 heads, d=128, "
                    "fp16, ctx U[256,2048], 8192 blocks"),
    "gqa_llama3_8b": DecodeConfig(
        name="gqa_llama3_8b", num_seqs=128, num_heads=32, num_kv_heads=8, head_dim=128,
        block_size=16, num_blocks=40960, dtype="bf16", ctx=("uniform", 512, 4096),
        seed=444_003,
        description="Llama-3-8B-shaped GQA decode layer: 128 seqs, 32/8 heads, d=128, "
                    "bf16, ctx U[512,4096], 40960 blocks"),
    "long_context_split": DecodeConfig(
        name="long_context_split", num_seqs=8, num_heads=32, num_kv_heads=8, head_dim=128,
        block_size=16, num_blocks=65536, dtype="bf16", ctx=("uniform", 32768, 131072),
        seed=444_004, partition_size=512,
        description="long-context split-K decode: 8 seqs, 32/8 heads, d=128, bf16, "
                    "ctx U[32768,131072], 65536 blocks (~4.3 GB K+V), partition 512"),
    "shared_prefix_beam": DecodeConfig(
        name="shared_prefix_beam", num_seqs=64, num_heads=32, num_kv_heads=8, head_dim=128,
        block_size=16, num_blocks=32768, dtype="f16",
        ctx=("lognormal", 1024.0, 0.6, 513, 8192), seed=444_005,
        shared_prefix_blocks=32, share_group=4,
        description="shared-prefix beam decode: 64 seqs in groups of 4 sharing 32 blocks, "
                    "32/8 heads, d=128, fp16, ctx lognormal mean 1024 in [513,8192]"),
}

# The order of the five workloads as the project states them.
CONFIG_ORDER = ["tiny", "mha_llama2_7b", "gqa_llama3_8b", "long_context_split",
                "shared_prefix_beam"]


def draw_context_lens(cfg: DecodeConfig, gen: torch.Generator) -> torch.Tensor:
    kind = cfg.ctx[0]
    if kind == "fixed":
        vals = torch.tensor(cfg.ctx[1], dtype=torch.int64)
        assert vals.numel() == cfg.num_seqs
    elif kind == "uniform":
        lo, hi = cfg.ctx[1], cfg.ctx[2]
        vals = torch.randint(lo, hi + 1, (cfg.num_seqs,), generator=gen, dtype=torch.int64)
    elif kind == "lognormal":
        mean, sigma, lo, hi = cfg.ctx[1:]
        mu = math.log(mean) - sigma * sigma / 2.0
        z = torch.randn(cfg.num_seqs, generator=gen, dtype=torch.float64)
        vals = torch.exp(mu + sigma * z).round().clamp(lo, hi).to(torch.int64)
    else:
        raise ValueError(f"unknown context-length recipe {cfg.ctx}")
    return vals.to(torch.int32)


def build_block_tables(cfg: DecodeConfig, context_lens: torch.Tensor,
                       gen: torch.Generator) -> torch.Tensor:
    """Physical ids from a seeded permutation of range(num_blocks), handed to
    sequences in order; sharing groups reuse the first shared_prefix_blocks
    ids of their group.  Unused entries are -1."""
    blocks_needed = [(int(c) + cfg.block_size - 1) // cfg.block_size for c in context_lens]
    max_blocks = max(1, max(blocks_needed), cfg.shared_prefix_blocks)
    tables = torch.full((cfg.num_seqs, max_blocks), -1, dtype=torch.int32)
    perm = torch.randperm(cfg.num_blocks, generator=gen).to(torch.int32)
    cursor = 0
    shared: list[int] = []
    for s, nb in enumerate(blocks_needed):
        row: list[int] = []
        if cfg.shared_prefix_blocks > 0:
            # every member's table starts with the group's shared ids (entries
            # past its own context are never read for that member)
            if s % cfg.share_group == 0:
                shared = perm[cursor:cursor + cfg.shared_prefix_blocks].tolist()
                cursor += cfg.shared_prefix_blocks
            row.extend(shared)
            nb = max(0, nb - cfg.shared_prefix_blocks)
        row.extend(perm[cursor:cursor + nb].tolist())
        cursor += nb
        if cursor > cfg.num_blocks:
            raise ValueError(f"{cfg.name}: needs more than {cfg.num_blocks} blocks")
        tables[s, :len(row)] = torch.tensor(row, dtype=torch.int32)
    return tables


def slot_of_last_token(block_tables: torch.Tensor, context_lens: torch.Tensor,
                       block_size: int) -> torch.Tensor:
    """Flat slot of position ctx-1 of every sequence (the token written this
    step); -1 (skip) for an empty sequence."""
    slots = torch.full((block_tables.shape[0],), -1, dtype=torch.int64)
    for s in range(block_tables.shape[0]):
        c = int(context_lens[s])
        if c > 0:
            pos = c - 1
            slots[s] = int(block_tables[s, pos // block_size]) * block_size + pos % block_size
    return slots


def _fill_normal(t: torch.Tensor, gen: torch.Generator, chunk: int = 1 << 27) -> torch.Tensor:
    """Fill a 16-bit tensor with N(0,1) float32 draws cast nearest-even,
    in chunks so a multi-GB cache never needs a full float32 copy."""
    flat = t.view(-1)
    for i in range(0, flat.numel(), chunk):
        n = min(chunk, flat.numel() - i)
        flat[i:i + n] = torch.randn(n, generator=gen, device=t.device,
                                    dtype=torch.float32).to(t.dtype)
    return t


@dataclass
class DecodeBatch:
    cfg: DecodeConfig
    context_lens: torch.Tensor
    block_tables: torch.Tensor
    slot_mapping: torch.Tensor
    key_cache: torch.Tensor
    value_cache: torch.Tensor
    query: torch.Tensor
    key: torch.Tensor
    value: torch.Tensor
    group_starts: torch.Tensor | None = None    # shared-prefix groups (int32 [G+1])
    prefix_blocks: torch.Tensor | None = None   # shared table entries per group (int32 [G])
    meta: dict = field(default_factory=dict)

    @property
    def max_partitions(self) -> int:
        ps = self.cfg.partition_size or 512
        return max(1, (self.block_tables.shape[1] * self.cfg.block_size + ps - 1) // ps)


def make_batch(cfg: DecodeConfig, device: str | torch.device = "cpu") -> DecodeBatch:
    """Draw one decode batch.  Index structure (lengths, tables, slots) always
    comes from a CPU generator; values come from a generator on `device`
    seeded the same way, so the bits are reproducible per device type."""
    device = torch.device(device)
    gen = torch.Generator(device="cpu")
    gen.manual_seed(cfg.seed)
    context_lens = draw_context_lens(cfg, gen)
    block_tables = build_block_tables(cfg, context_lens, gen)
    slot_mapping = slot_of_last_token(block_tables, context_lens, cfg.block_size)
    if not cfg.write_new_token:
        slot_mapping = torch.full_like(slot_mapping, -1)

    vgen = torch.Generator(device=device)
    vgen.manual_seed(cfg.seed + 7919)
    dt = cfg.torch_dtype
    cache_shape = (cfg.num_blocks, cfg.block_size, cfg.num_kv_heads, cfg.head_dim)
    key_cache = _fill_normal(torch.empty(cache_shape, dtype=dt, device=device), vgen)
    value_cache = _fill_normal(torch.empty(cache_shape, dtype=dt, device=device), vgen)
    query = _fill_normal(torch.empty((cfg.num_seqs, cfg.num_heads, cfg.head_dim),
                                     dtype=dt, device=device), vgen)
    key = _fill_normal(torch.empty((cfg.num_seqs, cfg.num_kv_heads, cfg.head_dim),
                                   dtype=dt, device=device), vgen)
    value = _fill_normal(torch.empty((cfg.num_seqs, cfg.num_kv_heads, cfg.head_dim),
                                     dtype=dt, device=device), vgen)
    group_starts = prefix_blocks = None
    if cfg.shared_prefix_blocks > 0:
        starts = list(range(0, cfg.num_seqs, cfg.share_group)) + [cfg.num_seqs]
        group_starts = torch.tensor(starts, dtype=torch.int32, device=device)
        prefix_blocks = torch.full((len(starts) - 1,), cfg.shared_prefix_blocks,
                                   dtype=torch.int32, device=device)
    return DecodeBatch(cfg, context_lens.to(device), block_tables.to(device),
                       slot_mapping.to(device), key_cache, value_cache, query, key, value,
                       group_starts, prefix_blocks)


@dataclass
class PrefillBatch:
    """A chunked-prefill step: each sequence's `chunk` newest tokens are the
    queries (packed [T, H, D], offsets query_starts), their K/V already in the
    paged cache of `cache`."""
    cache: DecodeBatch
    query: torch.Tensor
    query_starts: torch.Tensor
    chunk: int


PREFILL_CONFIG = CONFIGS["gqa_llama3_8b"].scaled(
    name="chunked_prefill_gqa", num_seqs=8, num_blocks=4096, ctx=("uniform", 512, 4096),
    seed=444_006)


def make_prefill_batch(cfg: DecodeConfig = PREFILL_CONFIG, chunk: int = 512,
                       device: str | torch.device = "cpu") -> PrefillBatch:
    """The chunked-prefill workload: cfg's caches and contexts (every context
    >= chunk), queries N(0,1) in the cache dtype from a generator seeded
    seed + 1, chunk query tokens per sequence."""
    b = make_batch(cfg, device)
    T = cfg.num_seqs * chunk
    g = torch.Generator(device=device).manual_seed(cfg.seed + 1)
    query = torch.randn((T, cfg.num_heads, cfg.head_dim), generator=g, device=device).to(
        cfg.torch_dtype)
    starts = torch.arange(0, T + 1, chunk, dtype=torch.int32, device=device)
    return PrefillBatch(b, query, starts, chunk)


def algorithmic_bytes(cfg: DecodeConfig, context_lens) -> dict:
    """Bytes the decode step must move at least once, by part:
    K+V of every context token of every KV head, the block-table entries
    read, q, out and context_lens; plus the cache write (read new K/V and
    slots, write the K/V rows)."""
    e = 2
    ctx = [int(c) for c in context_lens]
    kv = sum(ctx) * cfg.num_kv_heads * cfg.head_dim * e * 2
    bt = sum((c + cfg.block_size - 1) // cfg.block_size for c in ctx) * 4
    q = cfg.num_seqs * cfg.num_heads * cfg.head_dim * e
    out = q
    cl = cfg.num_seqs * 4
    writes = sum(1 for c in ctx if c > 0) if cfg.write_new_token else 0
    write = writes * cfg.num_kv_heads * cfg.head_dim * e * 2 * 2 + cfg.num_seqs * 8
    return {"kv": kv, "block_table": bt, "query": q, "out": out, "context_lens": cl,
            "attention": kv + bt + q + out + cl, "write": write,
            "step": kv + bt + q + out + cl + write}


def unique_kv_bytes(cfg: DecodeConfig, block_tables, context_lens) -> int:
    """K+V bytes of the distinct (physical block, token row) pairs read: a
    shared prefix counts once per group."""
    seen = set()
    for s in range(len(context_lens)):
        c = int(context_lens[s])
        for j in range(c):
            seen.add((int(block_tables[s][j // cfg.block_size]), j % cfg.block_size))
    return len(seen) * cfg.num_kv_heads * cfg.head_dim * 2 * 2
