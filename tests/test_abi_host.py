"""The C-ABI library on the host: it builds, loads, exports every symbol the
header declares, and rejects bad arguments before touching the GPU (CPU only)."""
import ctypes

import pytest
import torch

from paged_kv_cache_444_b200 import _lib
from paged_kv_cache_444_b200 import build as pa_build

OK, NULL, SHAPE, DTYPE, ALIGN, UNSUP, CUDA, BOUNDS = range(8)
FAKE = 0x10000          # 16-byte aligned stand-in pointer; never dereferenced on these paths

# Calls with stand-in pointers must be rejected before any launch.  They run
# only where no GPU is visible, so that a validation gap can never turn into
# a launch on stand-in pointers.
host_only = pytest.mark.skipif(torch.cuda.is_available(),
                               reason="stand-in pointers: host-only validation test")


@pytest.fixture(scope="module")
def lib():
    pa_build.build()
    return _lib.load()


def test_library_built_for_sm100a(lib):
    assert _lib.LIBRARY.exists()
    assert "arch=compute_100a,code=sm_100a" in " ".join(pa_build.NVCC_FLAGS)


def test_exports_every_header_symbol(lib):
    names = _lib.header_functions()
    assert set(names) == set(_lib.SIGNATURES), names
    for n in names:
        assert hasattr(lib, n), n


def test_binding_signatures_match_header():
    """Every ctypes signature has the header's parameter count and kinds."""
    import ctypes
    kind = {"ptr": ctypes.c_void_p, "int64_t": ctypes.c_int64, "float": ctypes.c_float,
            "pa_status": ctypes.c_int, "pa_dtype": ctypes.c_int, "int32_t": ctypes.c_int32}
    decl = _lib.header_signatures()
    assert set(decl) == set(_lib.SIGNATURES)
    for name, params in decl.items():
        args = _lib.SIGNATURES[name][1]
        assert len(args) == len(params), (name, len(args), len(params))
        for a, p in zip(args, params):
            want = kind[p]
            ok = (a is want or (p == "ptr" and a in (ctypes.c_void_p, ctypes.c_char_p) or
                                (p == "ptr" and hasattr(a, "_type_"))) or
                  (p in ("pa_status", "pa_dtype") and a is ctypes.c_int))
            assert ok, (name, p, a)


def test_status_strings_and_version(lib):
    assert lib.pa_abi_version() >> 16 == 1
    for code in range(8):
        assert lib.pa_status_string(code).decode()
    assert lib.pa_status_string(99).decode() == "unknown status"


def _decode(lib, **kw):
    args = dict(out=FAKE, query=FAKE, kc=FAKE, vc=FAKE, bt=FAKE, cl=FAKE, scale=0.125, S=4, H=8,
                Hk=2, D=128, NB=64, bs=16, MB=8, dt=0)
    args.update(kw)
    return lib.pa_decode(args["out"], args["query"], args["kc"], args["vc"], args["bt"],
                         args["cl"], args["scale"], args["S"], args["H"], args["Hk"], args["D"],
                         args["NB"], args["bs"], args["MB"], args["dt"], None)


@host_only
def test_decode_validation(lib):
    assert _decode(lib, dt=5) == DTYPE
    assert _decode(lib, query=None) == NULL
    assert _decode(lib, out=None) == NULL
    assert _decode(lib, bt=None) == NULL
    assert _decode(lib, H=6, Hk=4) == SHAPE
    assert _decode(lib, Hk=0) == SHAPE
    assert _decode(lib, S=-1) == SHAPE
    assert _decode(lib, scale=float("nan")) == SHAPE
    assert _decode(lib, D=96) == UNSUP
    assert _decode(lib, D=100) == ALIGN
    assert _decode(lib, bs=8) == UNSUP
    assert _decode(lib, H=64, Hk=2) == UNSUP          # group of 32 query heads
    assert _decode(lib, query=FAKE + 8) == ALIGN
    assert _decode(lib, kc=FAKE + 2) == ALIGN
    assert _decode(lib, bt=FAKE + 2) == ALIGN
    assert _decode(lib, NB=1 << 28) == SHAPE          # rows beyond 32-bit TMA coordinates
    assert _decode(lib, S=0, out=None, query=None) == OK  # empty batch: nothing to do


@host_only
def test_split_and_reduce_validation(lib):
    f = lib.pa_decode_split
    base = [FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 0.1, 4, 8, 2, 128, 64, 16, 8]
    assert f(*base, 0, 1, 1, None) == SHAPE
    assert f(*base, 24, 1, 1, None) == UNSUP            # not a multiple of block_size
    assert f(*base, 512, 0, 1, None) == SHAPE
    assert f(None, *base[1:], 512, 1, 1, None) == NULL
    assert f(*base, 512, 1, 9, None) == DTYPE
    r = lib.pa_reduce
    assert r(FAKE, FAKE, FAKE, FAKE, FAKE, 4, 8, 128, 0, 1, 0, None) == SHAPE
    assert r(None, FAKE, FAKE, FAKE, FAKE, 4, 8, 128, 512, 1, 0, None) == NULL
    assert r(FAKE, FAKE, FAKE, FAKE, FAKE, 4, 8, 130, 512, 1, 0, None) == UNSUP
    assert r(FAKE, FAKE, FAKE, FAKE, FAKE, 4, 8, 1028, 512, 1, 0, None) == UNSUP
    assert r(FAKE, FAKE, FAKE, FAKE, FAKE, 0, 8, 128, 512, 1, 0, None) == OK


@host_only
def test_reshape_validation(lib):
    f = lib.pa_reshape_and_cache
    good = [FAKE, FAKE, 256, 256, FAKE, FAKE, FAKE, 4, 2, 128, 64, 16, 0, None]

    def call(i, v):
        a = list(good)
        a[i] = v
        return f(*a)

    assert call(7, 0) == OK                 # no tokens: no-op
    assert call(12, 3) == DTYPE
    assert call(0, None) == NULL
    assert call(2, 100) == SHAPE            # stride shorter than a row
    assert call(2, 260) == ALIGN            # stride not a multiple of 8 elements
    assert call(6, FAKE + 4) == ALIGN       # slot_mapping not 8-byte aligned
    assert call(4, FAKE + 8) == ALIGN
    assert call(11, 0) == SHAPE


@pytest.mark.skipif(torch.cuda.is_available(), reason="only meaningful without a GPU")
def test_valid_call_without_gpu_reports_cuda_error(lib):
    # every argument is valid, so the library reaches the CUDA runtime, which
    # has no device here: the call must fail with PA_ERR_CUDA, not crash
    assert _decode(lib) == CUDA
    detail = ctypes.c_int64(0)
    assert lib.pa_check_error(None, ctypes.byref(detail)) == CUDA
    assert lib.pa_selftest_wait_timeout(None) == CUDA


def test_binding_raises_without_library(tmp_path):
    with pytest.raises(_lib.PagedAttentionError):
        _lib.load(tmp_path / "missing.so")


@host_only
def test_shared_prefix_validation(lib):
    f = lib.pa_decode_shared_prefix
    base = [FAKE] * 8 + [0.1, 8]            # out .. prefix_blocks, scale, num_seqs
    sizes = [2, 4, 8, 2, 128, 64, 16, 8, 0, None]  # groups, max size, H, Hk, D, NB, bs, MB, dt
    assert f(*base, *sizes[:1], 0, *sizes[2:]) == SHAPE          # max_group_size 0
    assert f(*base, -1, *sizes[1:]) == SHAPE                      # negative group count
    assert f(*base, 0, *sizes[1:]) == OK                          # no groups: nothing to do
    b = list(base)
    b[6] = None
    assert f(*b, *sizes) == NULL                                  # group_starts
    b = list(base)
    b[7] = FAKE + 2
    assert f(*b, *sizes) == ALIGN                                 # prefix_blocks
    assert f(*base, 2, 4, 64, 2, 128, 64, 16, 8, 0, None) == UNSUP  # 32 query heads per KV head


@host_only
def test_copy_blocks_validation(lib):
    f = lib.pa_copy_blocks
    assert f(FAKE, FAKE, FAKE, 0, 64, 16, 2, 128, 2, None) == OK        # no pairs
    assert f(FAKE, FAKE, FAKE, 3, 64, 16, 2, 128, 4, None) == SHAPE     # element size
    assert f(None, FAKE, FAKE, 3, 64, 16, 2, 128, 2, None) == NULL
    assert f(FAKE + 8, FAKE, FAKE, 3, 64, 16, 2, 128, 2, None) == ALIGN
    assert f(FAKE, FAKE, FAKE + 4, 3, 64, 16, 2, 128, 2, None) == ALIGN
    assert f(FAKE, FAKE, FAKE, 3, 64, 1, 1, 4, 2, None) == ALIGN        # 8-byte blocks


@host_only
def test_fp8_validation(lib):
    f = lib.pa_decode_fp8
    base = [FAKE] * 6 + [0.1]
    ok_sizes = [4, 8, 2, 128, 64, 16, 8, 0, None]
    assert f(*base, 0.0, 1.0, *ok_sizes) == SHAPE                     # k_scale must be > 0
    assert f(*base, 1.0, float("inf"), *ok_sizes) == SHAPE
    assert f(*base, 1.0, 1.0, 4, 8, 2, 64, 64, 16, 8, 0, None) == UNSUP   # head_dim 64
    assert f(*base, 1.0, 1.0, 0, 8, 2, 128, 64, 16, 8, 0, None) == OK     # empty batch
    w = lib.pa_reshape_and_cache_fp8
    good = [FAKE, FAKE, 256, 256, FAKE, FAKE, FAKE, 4, 2, 128, 64, 16, 0.5, 0.5, 0, None]
    bad = list(good)
    bad[12] = -1.0
    assert w(*bad) == SHAPE
    bad = list(good)
    bad[9] = 72                                                        # not a multiple of 16
    bad[2] = bad[3] = 144
    assert w(*bad) == ALIGN
    bad = list(good)
    bad[7] = 0
    assert w(*bad) == OK


@host_only
def test_step_host_packed_pairs_validation(lib):
    """pa_decode_step_host: value/slot_mapping (and block_tables/context_lens)
    are both given or both NULL (packed after key/query); one NULL alone is
    PA_ERR_NULL, found before any CUDA call.  An empty batch is a no-op."""
    f = lib.pa_decode_step_host
    W = FAKE

    def call(value, slots, tables, lens, S=4):
        return f(W, W, W, value, slots, tables, lens, W, W, W, 1 << 30, 0.125, S, 8, 2, 128, 64,
                 16, 8, 0, 0, None)
    assert call(None, W, W, W) == NULL
    assert call(W, None, W, W) == NULL
    assert call(W, W, None, W) == NULL
    assert call(W, W, W, None) == NULL
    assert call(None, W, None, W, S=0) == OK
