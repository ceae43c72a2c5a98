"""pa_decode_noalloc: the long-context decode whose partition scratch is a
fixed device array inside libpa, for callers that cannot allocate device
memory when they call (runtimes that own all device memory through their own
pool, plugin hosts without an allocator, latency-critical paths that cannot
take an allocation's synchronisation).

The GPU test calls it through the C ABI twice in a row, on two different
batches, and checks each result against the caller-scratch entry points
pa_decode_split + pa_reduce within the parity tolerance, so that a second
call cannot pass on the first call's leftovers.  This file is named to be
collected last."""
import numpy as np
import pytest
import torch

from paged_kv_cache_444_b200 import _lib, workloads
from parity_helpers import TOL, gpu_step, to_f64

OK, SHAPE = 0, 2
FAKE = 0x10000


def test_noalloc_rejects_scratch_beyond_its_limit():
    lib = _lib.load()
    # 64 seqs x 32 heads x 2048 partitions x 130 floats needs ~2 GiB > 64 MiB:
    # rejected on the host, before any CUDA call
    st = lib.pa_decode_noalloc(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 0.1, 64, 32, 8, 128, 1 << 20,
                               16, 1 << 16, 512, 1, None)
    assert st == SHAPE
    assert lib.pa_decode_noalloc(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 0.1, 0, 32, 8, 128, 64, 16,
                                 8, 512, 1, None) == OK   # empty batch


@pytest.mark.gpu
def test_noalloc_matches_split_entry_points_twice(cuda_device):
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
        want, _ = gpu_step(batch, write=False, partition_size=cfg.partition_size)
        got = torch.full_like(batch.query, float("nan"))
        pa_decode_noalloc(got, batch.query, batch.key_cache, batch.value_cache,
                          batch.block_tables, batch.context_lens, cfg.scale, cfg.partition_size)
        torch.cuda.synchronize()
        pa_check_error()
        g, w = to_f64(got), to_f64(want)
        assert np.isfinite(g).all()
        assert np.max(np.abs(g - w)) <= TOL[cfg.dtype], cfg.name
