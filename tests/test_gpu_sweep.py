"""A seeded sweep of small random layouts through the CUDA path against the
fp64 oracle (GPU): group sizes 1 to 8 (every width of the transposed page
steps' query columns, odd ones included), head_dim 64 and 128, both 16-bit
dtypes, empty and ragged contexts, single pass and split at several partition
sizes; then the same for E4M3 caches (head_dim 128)."""
import random

import numpy as np
import pytest
import torch

from paged_kv_cache_444_b200 import (SplitWorkspace, pa_check_error, pa_decode_fp8,
                                     pa_decode_split_fp8, pa_reduce, pa_reshape_and_cache_fp8,
                                     workloads)
from parity_helpers import (K_SCALE, V_SCALE, TOL, HostCopy, fp8_batch, fp8_oracle, gpu_step,
                            oracle_step, to_f64)

pytestmark = pytest.mark.gpu


def _layout(i: int, head_dims=(64, 128)):
    r = random.Random(4440 + i)
    G = r.randint(1, 8)
    Hk = r.choice([1, 2, 4])
    D = r.choice(head_dims)
    dtype = r.choice(["f16", "bf16"])
    S = r.randint(1, 6)
    hi = r.choice([16, 100, 700])
    ps = r.choice([0, 16, 48, 256])
    cfg = workloads.CONFIGS["gqa_llama3_8b"].scaled(
        name=f"sweep{i}", num_seqs=S, num_heads=G * Hk, num_kv_heads=Hk, head_dim=D,
        dtype=dtype, num_blocks=S * ((hi + 15) // 16) + 16, ctx=("uniform", 0, hi),
        seed=4440 + i)
    return cfg, ps


def _what(cfg, ps):
    return (f"{cfg.name}: G={cfg.num_heads // cfg.num_kv_heads} Hk={cfg.num_kv_heads} "
            f"D={cfg.head_dim} {cfg.dtype} S={cfg.num_seqs} partition={ps}")


@pytest.mark.parametrize("i", range(16))
def test_sweep_16bit_matches_oracle(i, cuda_device, oracle_lib):
    cfg, ps = _layout(i)
    batch = workloads.make_batch(cfg, cuda_device)
    host = HostCopy(batch)
    ref, _, _ = oracle_step(oracle_lib, host)
    out, _ = gpu_step(batch, partition_size=ps)
    pa_check_error()
    g = to_f64(out)
    assert np.isfinite(g).all(), _what(cfg, ps)
    err = np.max(np.abs(g - ref))
    assert err <= TOL[cfg.dtype], f"{_what(cfg, ps)}: {err:.3e}"


@pytest.mark.parametrize("i", range(10))
def test_sweep_fp8_matches_oracle(i, cuda_device, oracle_lib):
    cfg, ps = _layout(100 + i, head_dims=(128,))
    b, kc, vc = fp8_batch(cfg, cuda_device)
    ref, _, _ = fp8_oracle(oracle_lib, b, kc, vc)
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
    assert np.isfinite(g).all(), _what(cfg, ps)
    err = np.max(np.abs(g - ref))
    assert err <= TOL[cfg.dtype], f"{_what(cfg, ps)}: {err:.3e}"
