"""Plant plausible mistakes in a copy of the oracle and check that the pins
catch every one of them (CPU only; the planted copies live in a temp dir).

Each planted copy runs the pin suite in a child process, because some
mistakes (a write one row too far) corrupt memory; a child that crashes has
been caught as surely as one whose pins fail."""
import subprocess
import sys
from pathlib import Path

import pytest

import oracle as oracle_mod

TESTS_DIR = Path(__file__).resolve().parent
ROOT = TESTS_DIR.parent

_RUNNER = """
import sys
sys.path[:0] = [{tests!r}, {root!r}]
import oracle
from oracle_pins import ALL_PINS
orc = oracle.Oracle({lib!r})
caught = []
for pin in ALL_PINS:
    try:
        pin(orc)
    except (AssertionError, ValueError):
        caught.append(pin.__name__)
print("CAUGHT", ",".join(caught))
"""

# (what the mistake is, original text, replacement) -- each applied alone.
MUTATIONS = [
    ("slot: wrong logical block", "int64_t logical_block = pos / block_size;",
     "int64_t logical_block = pos / (block_size + 1);"),
    ("slot: offset off by one", "int64_t offset = pos % block_size;",
     "int64_t offset = (pos + 1) % block_size;"),
    ("f16 decode: exponent bias", "mag = ldexp((double)(1024 + frac), expo - 25);",
     "mag = ldexp((double)(1024 + frac), expo - 24);"),
    ("f16 decode: subnormal scale", "mag = ldexp((double)frac, -24);",
     "mag = ldexp((double)frac, -25);"),
    ("bf16 decode: shift", "uint32_t w = (uint32_t)bits << 16;", "uint32_t w = (uint32_t)bits << 15;"),
    ("rounding: truncation", "return nearbyint(x / quantum) * quantum;",
     "return trunc(x / quantum) * quantum;"),
    ("rounding: ties away", "return nearbyint(x / quantum) * quantum;",
     "return round(x / quantum) * quantum;"),
    ("kv bytes: K and V counted once", "return 2 * num_layers * num_kv_heads * head_dim * elem_bytes;",
     "return num_layers * num_kv_heads * head_dim * elem_bytes;"),
    ("page size: K and V counted once", "return num_kv_heads * head_dim * elem_bytes * block_size * 2;",
     "return num_kv_heads * head_dim * elem_bytes * block_size;"),
    ("write: slot off by one row", "memcpy(key_cache + slot * row,", "memcpy(key_cache + (slot + 1) * row,"),
    ("write: slot 0 treated as padding", "if (slot < 0) continue;", "if (slot <= 0) continue;"),
    ("write: value written from key", "memcpy(value_cache + slot * row, value + t * value_stride",
     "memcpy(value_cache + slot * row, key + t * key_stride"),
    ("write: stride ignored", "key + t * key_stride", "key + t * row"),
    ("gather: cache layout transposed",
     "int64_t base = ((block * block_size + r) * num_kv_heads + kv_head) * head_dim;",
     "int64_t base = ((block * num_kv_heads + kv_head) * block_size + r) * head_dim;"),
    ("gather: logical block ignored", "int64_t block = block_table[j / block_size];",
     "int64_t block = block_table[0];"),
    ("gather: row offset ignored", "int64_t r = j % block_size;", "int64_t r = 0;"),
    ("GQA: interleaved head grouping", "int64_t kvh = h / group;", "int64_t kvh = h % num_kv_heads;"),
    ("scale dropped", "z[j - t0] = scale * dot;", "z[j - t0] = dot;"),
    ("softmax: max not subtracted per range", "double p = exp(z[j - t0] - m);", "double p = exp(z[j - t0]);"),
    ("softmax: no normalisation", "for (int64_t d = 0; d < head_dim; ++d) acc[d] /= l;",
     "for (int64_t d = 0; d < head_dim; ++d) acc[d] /= 1.0;"),
    ("decode: last token dropped", "attend_range(q, kc, vc, head_dim, 0, ctx, scale, z, &m, &l, acc);",
     "attend_range(q, kc, vc, head_dim, 0, ctx > 1 ? ctx - 1 : ctx, scale, z, &m, &l, acc);"),
    ("merge: partition weight dropped", "double w = exp(part_max[base + p] - big_m);", "double w = 1.0;"),
    ("merge: sum not weighted", "big_l += w * part_sum[base + p];", "big_l += part_sum[base + p];"),
    ("copy: destination and source swapped",
     "memmove(key_cache + dst * block_bytes, key_cache + src * block_bytes, block_bytes);",
     "memmove(key_cache + src * block_bytes, key_cache + dst * block_bytes, block_bytes);"),
    ("copy: half a block", "size_t block_bytes = (size_t)(block_size * num_kv_heads * head_dim * elem_bytes);",
     "size_t block_bytes = (size_t)(block_size * num_kv_heads * head_dim * elem_bytes / 2);"),
    ("e4m3 decode: exponent bias", "mag = ldexp((double)(8 + frac), expo - 10);",
     "mag = ldexp((double)(8 + frac), expo - 11);"),
    ("e4m3 encode: no saturation", "if (a > 448.0 || isinf(a)) a = 448.0;", "if (isinf(a)) a = 448.0;"),
    ("e4m3 encode: scale not applied", "key_cache[slot * row + e] = oracle_f64_to_e4m3((double)(kx * inv_k));",
     "key_cache[slot * row + e] = oracle_f64_to_e4m3((double)kx);"),
    ("fp8 decode: v scale dropped", "vc[j * head_dim + d] = oracle_e4m3_to_f64(value_cache[base + d]) * v_scale;",
     "vc[j * head_dim + d] = oracle_e4m3_to_f64(value_cache[base + d]);"),
    ("prefill: query position off by one", "int64_t pos = ctx - q_len + i;",
     "int64_t pos = ctx - q_len + i - 1;"),
    ("prefill: not causal", "attend_range(q, kc, vc, head_dim, 0, pos + 1, scale, z, &m, &l, acc);",
     "attend_range(q, kc, vc, head_dim, 0, ctx, scale, z, &m, &l, acc);"),
    ("partition: end not clipped to ctx",
     "int64_t t1 = t0 + partition_size < ctx ? t0 + partition_size : ctx;",
     "int64_t t1 = t0 + partition_size < ctx ? t0 + partition_size : ctx - 1;"),
]


def _plant_and_run(what, old, new, workdir: Path):
    """Compile the oracle with one planted mistake and run the pin suite on it
    in a child process; returns (returncode, stdout)."""
    src = oracle_mod.SOURCE.read_text(encoding="utf-8")
    if old not in src:
        return None, f"mutation anchor no longer in the oracle source: {old!r}"
    workdir.mkdir(parents=True, exist_ok=True)
    mutant_src = workdir / "pa_oracle_mutant.c"
    mutant_src.write_text(src.replace(old, new), encoding="utf-8")
    lib = oracle_mod.compile_oracle(mutant_src, workdir / "libmutant.so")
    code = _RUNNER.format(tests=str(TESTS_DIR), root=str(ROOT), lib=str(lib))
    proc = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True,
                          timeout=600)
    return proc.returncode, proc.stdout


@pytest.fixture(scope="module")
def mutant_results(tmp_path_factory):
    """Every planted copy built and run at once, one worker per CPU (each is
    a gcc build and a child process, independent of the others)."""
    import os
    from concurrent.futures import ThreadPoolExecutor
    base = tmp_path_factory.mktemp("mutants")
    with ThreadPoolExecutor(max_workers=max(1, os.cpu_count() or 1)) as pool:
        futures = {what: pool.submit(_plant_and_run, what, old, new, base / f"m{i}")
                   for i, (what, old, new) in enumerate(MUTATIONS)}
        return {what: f.result() for what, f in futures.items()}


@pytest.mark.parametrize("what", [m[0] for m in MUTATIONS])
def test_pins_catch_planted_mistake(what, mutant_results):
    returncode, out = mutant_results[what]
    assert returncode is not None, out
    if returncode != 0:
        return  # the planted mistake crashed the pin suite: caught
    line = [ln for ln in out.splitlines() if ln.startswith("CAUGHT")][-1]
    caught = [c for c in line[len("CAUGHT"):].strip().split(",") if c]
    assert caught, f"no pin caught the planted mistake: {what}"
