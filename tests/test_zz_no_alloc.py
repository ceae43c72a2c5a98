"""pa_decode_noalloc: the long-context decode whose partition scratch is a
fixed device array inside libpa, for callers that cannot allocate device
memory when they call (runtimes that own all device memory through their own
pool, plugin hosts without an allocator, latency-critical paths that cannot
take an allocation's synchronisation).

The GPU test calls it through the C ABI twice in a row, on two different
batches.  Each result must equal the caller-scratch entry points
pa_decode_split + pa_reduce bit for bit (same kernels, same partition count,
only the scratch differs), and must match the fp64 oracle within the parity
tolerance, so that a second call cannot pass on the first call's leftovers.
The size limit is pinned at its edge: the largest accepted call runs on the
GPU, the smallest rejected one is refused on the host.  This file is named
to be collected last."""
import numpy as np
import pytest
import torch

from paged_kv_cache_444_b200 import _lib, workloads
from parity_helpers import TOL, HostCopy, gpu_step, max_err, oracle_step, to_f64

OK, SHAPE = 0, 2
FAKE = 0x10000
LIMIT = _lib.NOALLOC_SCRATCH_BYTES
# One sequence, one head, head_dim 128, 16-token partitions: the scratch need
# is P * (128 + 2) * 4 bytes with P = max_blocks_per_seq partitions.
ROW_BYTES = (128 + 2) * 4
P_FITS = LIMIT // ROW_BYTES          # largest partition count that fits
assert P_FITS * ROW_BYTES <= LIMIT < (P_FITS + 1) * ROW_BYTES


def _call_fake(lib, max_blocks, num_seqs=1):
    return lib.pa_decode_noalloc(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 0.1, num_seqs, 1, 1, 128,
                                 64, 16, max_blocks, 16, 1, None)


def test_noalloc_rejects_scratch_beyond_its_limit():
    lib = _lib.load()
    # the smallest call past the limit, refused on the host before any CUDA call
    assert _call_fake(lib, P_FITS + 1) == SHAPE
    # far past it: 64 seqs x 32 heads x 2048 partitions x 130 floats (~2 GiB)
    assert lib.pa_decode_noalloc(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 0.1, 64, 32, 8, 128, 1 << 20,
                                 16, 1 << 16, 512, 1, None) == SHAPE
    assert lib.pa_decode_noalloc(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 0.1, 0, 32, 8, 128, 64, 16,
                                 8, 512, 1, None) == OK   # empty batch
    # the binding computes the same need and refuses the same call (host
    # tensors: it raises before reaching the library)
    q = torch.empty((1, 1, 128), dtype=torch.bfloat16)
    kc = torch.empty((64, 16, 1, 128), dtype=torch.bfloat16)
    with pytest.raises(_lib.PagedAttentionError):
        _lib.pa_decode_noalloc(q, q, kc, kc, torch.zeros((1, P_FITS + 1), dtype=torch.int32),
                               torch.ones(1, dtype=torch.int32), 0.1, 16)


@pytest.mark.skipif(torch.cuda.is_available(), reason="the accepted call would launch kernels")
def test_noalloc_accepts_the_largest_call_that_fits_on_the_host():
    # passes the size check; without a device the next step (looking up the
    # array's address) fails with PA_ERR_CUDA, not PA_ERR_SHAPE
    assert _call_fake(_lib.load(), P_FITS) not in (OK, SHAPE)


@pytest.mark.gpu
def test_noalloc_matches_split_entry_points_twice(cuda_device, oracle_lib):
    from paged_kv_cache_444_b200 import pa_check_error, pa_decode_noalloc
    base = workloads.CONFIGS["long_context_split"]
    cases = [
        base.scaled(name="noalloc_a", num_seqs=3, num_heads=16, num_kv_heads=4, num_blocks=1024,
                    ctx=("uniform", 2000, 5000), seed=31),
        # second call: different lengths, heads and dtype, so that stale
        # partitions of the first call would show
        base.scaled(name="noalloc_b", num_seqs=5, num_heads=8, num_kv_heads=8, dtype="f16",
                    num_blocks=512, ctx=("uniform", 1, 1500), seed=32),
    ]
    for cfg in cases:
        batch = workloads.make_batch(cfg, cuda_device)
        ref, _, _ = oracle_step(oracle_lib, HostCopy(batch), write=False)
        want, _ = gpu_step(batch, write=False, partition_size=cfg.partition_size)
        got = torch.full_like(batch.query, float("nan"))
        pa_decode_noalloc(got, batch.query, batch.key_cache, batch.value_cache,
                          batch.block_tables, batch.context_lens, cfg.scale, cfg.partition_size)
        torch.cuda.synchronize()
        pa_check_error()
        assert np.isfinite(to_f64(got)).all(), cfg.name
        assert torch.equal(got, want), f"{cfg.name}: differs from pa_decode_split + pa_reduce"
        err = max_err(got, ref)
        assert err <= TOL[cfg.dtype], f"{cfg.name}: max-abs {err:.3e} vs the oracle"


@pytest.mark.gpu
def test_noalloc_largest_call_that_fits(cuda_device, oracle_lib):
    """The largest call the fixed array holds (one sequence, one head, d = 128,
    16-token partitions, P_FITS partitions) runs and matches the oracle."""
    from paged_kv_cache_444_b200 import pa_check_error, pa_decode_noalloc
    cfg = workloads.CONFIGS["long_context_split"].scaled(
        name="noalloc_edge", num_seqs=1, num_heads=1, num_kv_heads=1, num_blocks=64,
        ctx=("fixed", (777,)), seed=33)
    batch = workloads.make_batch(cfg, cuda_device)
    wide = torch.full((1, P_FITS), -1, dtype=torch.int32, device=cuda_device)
    wide[:, :batch.block_tables.shape[1]] = batch.block_tables
    batch.block_tables = wide
    ref, _, _ = oracle_step(oracle_lib, HostCopy(batch), write=False)
    got = torch.full_like(batch.query, float("nan"))
    pa_decode_noalloc(got, batch.query, batch.key_cache, batch.value_cache, batch.block_tables,
                      batch.context_lens, cfg.scale, 16)
    torch.cuda.synchronize()
    pa_check_error()
    err = max_err(got, ref)
    assert np.isfinite(to_f64(got)).all() and err <= TOL[cfg.dtype], f"max-abs {err:.3e}"
