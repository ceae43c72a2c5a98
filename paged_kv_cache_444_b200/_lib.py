"""ctypes binding of libpa (include/pa.h): argument marshalling only.

Every function here takes torch CUDA tensors, checks that their dtype,
device and layout match what the C entry point expects, and passes raw
pointers, sizes and the current CUDA stream.  All arithmetic runs in the
library's kernels; there is no fallback.  If libpa.so is missing the first
call raises ``PagedAttentionError``.
"""
from __future__ import annotations

import ctypes
import re
from pathlib import Path

import torch

from . import build as _build

LIBRARY = _build.LIBRARY
HEADER = _build.INCLUDE / "pa.h"

PA_OK = 0
STATUS_NAMES = {0: "PA_OK", 1: "PA_ERR_NULL", 2: "PA_ERR_SHAPE", 3: "PA_ERR_DTYPE",
                4: "PA_ERR_ALIGN", 5: "PA_ERR_UNSUPPORTED", 6: "PA_ERR_CUDA",
                7: "PA_ERR_BOUNDS"}
CHECK_CODES = {1: "slot", 2: "block_id", 3: "context_len", 4: "partitions", 5: "wait_timeout",
               6: "group", 7: "query", 8: "value"}
DTYPE_CODES = {torch.float16: 0, torch.bfloat16: 1}


class PagedAttentionError(RuntimeError):
    def __init__(self, status: int, what: str, detail: int | None = None):
        self.status = status
        self.detail = detail
        msg = f"{what}: {STATUS_NAMES.get(status, status)}"
        if detail:
            msg += (f" (device check {CHECK_CODES.get(detail >> 56, detail >> 56)}, "
                    f"index {detail & ((1 << 56) - 1)})")
        super().__init__(msg)


_i64 = ctypes.c_int64
_p = ctypes.c_void_p
_f = ctypes.c_float
_i = ctypes.c_int

# name -> (restype, argtypes); the order is the header's.
SIGNATURES = {
    "pa_status_string": (ctypes.c_char_p, [_i]),
    "pa_abi_version": (ctypes.c_int32, []),
    "pa_reshape_and_cache": (_i, [_p, _p, _i64, _i64, _p, _p, _p, _i64, _i64, _i64, _i64, _i64,
                                  _i, _p]),
    "pa_decode": (_i, [_p, _p, _p, _p, _p, _p, _f, _i64, _i64, _i64, _i64, _i64, _i64, _i64,
                       _i, _p]),
    "pa_decode_split": (_i, [_p, _p, _p, _p, _p, _p, _p, _p, _f, _i64, _i64, _i64, _i64, _i64,
                             _i64, _i64, _i64, _i64, _i, _p]),
    "pa_reduce": (_i, [_p, _p, _p, _p, _p, _i64, _i64, _i64, _i64, _i64, _i, _p]),
    "pa_check_error": (_i, [_p, ctypes.POINTER(_i64)]),
    "pa_selftest_wait_timeout": (_i, [_p]),
    "pa_decode_noalloc": (_i, [_p, _p, _p, _p, _p, _p, _f, _i64, _i64, _i64, _i64, _i64, _i64,
                               _i64, _i64, _i, _p]),
    "pa_decode_shared_prefix": (_i, [_p, _p, _p, _p, _p, _p, _p, _p, _f, _i64, _i64, _i64, _i64,
                                     _i64, _i64, _i64, _i64, _i64, _i, _p]),
    "pa_copy_blocks": (_i, [_p, _p, _p, _i64, _i64, _i64, _i64, _i64, _i64, _p]),
    "pa_reshape_and_cache_fp8": (_i, [_p, _p, _i64, _i64, _p, _p, _p, _i64, _i64, _i64, _i64,
                                      _i64, _f, _f, _i, _p]),
    "pa_decode_fp8": (_i, [_p, _p, _p, _p, _p, _p, _f, _f, _f, _i64, _i64, _i64, _i64, _i64,
                           _i64, _i64, _i, _p]),
    "pa_decode_split_fp8": (_i, [_p, _p, _p, _p, _p, _p, _p, _p, _f, _f, _f, _i64, _i64, _i64,
                                 _i64, _i64, _i64, _i64, _i64, _i64, _i, _p]),
    "pa_decode_step_host_workspace_bytes": (_i64, [_i64] * 7),
    "pa_decode_step_host": (_i, [_p] * 10 + [_i64, _f] + [_i64] * 8 + [_i, _p]),
    "pa_prefill": (_i, [_p] * 7 + [_f] + [_i64] * 9 + [_i, _p]),
}

_lib: ctypes.CDLL | None = None


def load(path: Path | str | None = None) -> ctypes.CDLL:
    """Load libpa.so (built in-tree by ``build.build()``) and bind signatures."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    p = Path(path) if path else LIBRARY
    if not p.exists():
        raise PagedAttentionError(6, f"libpa.so not found at {p}; run "
                                     "`python -m paged_kv_cache_444_b200.build`")
    lib = ctypes.CDLL(str(p))
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    if path is None:
        _lib = lib
    return lib


def header_functions() -> list[str]:
    """Names of the functions include/pa.h declares."""
    text = HEADER.read_text(encoding="utf-8")
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(pa_[a-z0-9_]+)\s*\(", text)))


def header_signatures() -> dict[str, list[str]]:
    """Parameter type of every function include/pa.h declares, as C text
    (pointers collapse to 'ptr')."""
    text = HEADER.read_text(encoding="utf-8")
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    out = {}
    for m in re.finditer(r"\b(?:pa_status|int64_t|int32_t|const char\s*\*)\s*(pa_[a-z0-9_]+)"
                         r"\s*\(([^)]*)\)\s*;", text):
        params = [p.strip() for p in m.group(2).split(",") if p.strip() and p.strip() != "void"]
        kinds = []
        for p_ in params:
            if "*" in p_:
                kinds.append("ptr")
            else:
                kinds.append(p_.rsplit(None, 1)[0].replace("const ", ""))
        out[m.group(1)] = kinds
    return out


def status_string(status: int) -> str:
    return load().pa_status_string(status).decode()


def _check(status: int, what: str) -> None:
    if status != PA_OK:
        raise PagedAttentionError(status, what)


def _stream(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return int(stream.cuda_stream) if hasattr(stream, "cuda_stream") else int(stream)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype not in DTYPE_CODES:
        raise TypeError(f"expected float16 or bfloat16, got {t.dtype}")
    return DTYPE_CODES[t.dtype]


def _need(cond: bool, msg: str) -> None:
    if not cond:
        raise ValueError(msg)


# ---------------------------------------------------------------------------
# One wrapper per C entry point, same names
# ---------------------------------------------------------------------------
def pa_reshape_and_cache(key: torch.Tensor, value: torch.Tensor, key_cache: torch.Tensor,
                         value_cache: torch.Tensor, slot_mapping: torch.Tensor,
                         stream=None) -> None:
    """key/value [T, Hk, D] (token rows may be strided), caches
    [NB, bs, Hk, D] contiguous, slot_mapping [T] int64 on the device."""
    T, Hk, D = key.shape
    NB, bs = key_cache.shape[0], key_cache.shape[1]
    _need(value.shape == key.shape, "key/value shapes differ")
    _need(key_cache.shape == (NB, bs, Hk, D) and value_cache.shape == key_cache.shape,
          "cache shape must be [num_blocks, block_size, num_kv_heads, head_dim]")
    _need(key_cache.is_contiguous() and value_cache.is_contiguous(), "caches must be contiguous")
    _need(key.stride()[1:] == (D, 1) and value.stride()[1:] == (D, 1),
          "key/value token rows must be dense")
    _need(slot_mapping.dtype == torch.int64 and slot_mapping.shape == (T,), "slot_mapping [T] int64")
    dt = _dtype_code(key)
    _need(value.dtype == key.dtype == key_cache.dtype == value_cache.dtype, "dtype mismatch")
    st = load().pa_reshape_and_cache(
        key.data_ptr(), value.data_ptr(), key.stride(0) if T else Hk * D,
        value.stride(0) if T else Hk * D, key_cache.data_ptr(), value_cache.data_ptr(),
        slot_mapping.data_ptr(), T, Hk, D, NB, bs, dt, _stream(stream))
    _check(st, "pa_reshape_and_cache")


def _attention_common(query, key_cache, value_cache, block_tables, context_lens):
    S, H, D = query.shape
    NB, bs, Hk, D2 = key_cache.shape
    _need(D2 == D, "head_dim of query and cache differ")
    _need(value_cache.shape == key_cache.shape, "key/value cache shapes differ")
    _need(query.is_contiguous() and key_cache.is_contiguous() and value_cache.is_contiguous(),
          "query and caches must be contiguous")
    _need(block_tables.dtype == torch.int32 and block_tables.dim() == 2 and
          block_tables.shape[0] == S and block_tables.is_contiguous(),
          "block_tables must be [num_seqs, max_blocks] int32 contiguous")
    _need(context_lens.dtype == torch.int32 and context_lens.shape == (S,),
          "context_lens must be [num_seqs] int32")
    _need(query.dtype == key_cache.dtype == value_cache.dtype, "dtype mismatch")
    return S, H, D, NB, bs, Hk, block_tables.shape[1], _dtype_code(query)


def pa_decode(out: torch.Tensor, query: torch.Tensor, key_cache: torch.Tensor,
              value_cache: torch.Tensor, block_tables: torch.Tensor,
              context_lens: torch.Tensor, scale: float, stream=None) -> None:
    S, H, D, NB, bs, Hk, MB, dt = _attention_common(query, key_cache, value_cache,
                                                    block_tables, context_lens)
    _need(out.shape == query.shape and out.dtype == query.dtype and out.is_contiguous(),
          "out must match query")
    st = load().pa_decode(out.data_ptr(), query.data_ptr(), key_cache.data_ptr(),
                          value_cache.data_ptr(), block_tables.data_ptr(),
                          context_lens.data_ptr(), float(scale), S, H, Hk, D, NB, bs, MB, dt,
                          _stream(stream))
    _check(st, "pa_decode")


def pa_decode_split(tmp_out: torch.Tensor, max_logits: torch.Tensor, exp_sums: torch.Tensor,
                    query: torch.Tensor, key_cache: torch.Tensor, value_cache: torch.Tensor,
                    block_tables: torch.Tensor, context_lens: torch.Tensor, scale: float,
                    partition_size: int, stream=None) -> None:
    S, H, D, NB, bs, Hk, MB, dt = _attention_common(query, key_cache, value_cache,
                                                    block_tables, context_lens)
    P = max_logits.shape[-1]
    _need(tmp_out.shape == (S, H, P, D) and tmp_out.dtype == torch.float32
          and tmp_out.is_contiguous(), "tmp_out must be [S, H, P, D] float32")
    _need(max_logits.shape == (S, H, P) and exp_sums.shape == (S, H, P) and
          max_logits.dtype == exp_sums.dtype == torch.float32, "max_logits/exp_sums [S, H, P] f32")
    st = load().pa_decode_split(tmp_out.data_ptr(), max_logits.data_ptr(), exp_sums.data_ptr(),
                                query.data_ptr(), key_cache.data_ptr(), value_cache.data_ptr(),
                                block_tables.data_ptr(), context_lens.data_ptr(), float(scale),
                                S, H, Hk, D, NB, bs, MB, int(partition_size), P, dt,
                                _stream(stream))
    _check(st, "pa_decode_split")


def pa_reduce(out: torch.Tensor, tmp_out: torch.Tensor, max_logits: torch.Tensor,
              exp_sums: torch.Tensor, context_lens: torch.Tensor, partition_size: int,
              stream=None) -> None:
    S, H, P, D = tmp_out.shape
    _need(out.shape == (S, H, D) and out.is_contiguous(), "out must be [S, H, D]")
    _need(max_logits.shape == (S, H, P) and exp_sums.shape == (S, H, P), "partials shape")
    _need(context_lens.dtype == torch.int32 and context_lens.shape == (S,), "context_lens")
    st = load().pa_reduce(out.data_ptr(), tmp_out.data_ptr(), max_logits.data_ptr(),
                          exp_sums.data_ptr(), context_lens.data_ptr(), S, H, D,
                          int(partition_size), P, _dtype_code(out), _stream(stream))
    _check(st, "pa_reduce")


def pa_decode_shared_prefix(out: torch.Tensor, query: torch.Tensor, key_cache: torch.Tensor,
                            value_cache: torch.Tensor, block_tables: torch.Tensor,
                            context_lens: torch.Tensor, group_starts: torch.Tensor,
                            prefix_blocks: torch.Tensor, scale: float, max_group_size: int,
                            stream=None) -> None:
    """pa_decode for sequences grouped by a shared table prefix: group g is
    sequences group_starts[g] .. group_starts[g+1]-1, whose first
    prefix_blocks[g] table entries are the same ids (read once per group)."""
    S, H, D, NB, bs, Hk, MB, dt = _attention_common(query, key_cache, value_cache,
                                                    block_tables, context_lens)
    _need(out.shape == query.shape and out.dtype == query.dtype and out.is_contiguous(),
          "out must match query")
    n_groups = prefix_blocks.shape[0]
    _need(group_starts.dtype == torch.int32 and group_starts.shape == (n_groups + 1,),
          "group_starts must be [num_groups + 1] int32")
    _need(prefix_blocks.dtype == torch.int32, "prefix_blocks must be int32")
    st = load().pa_decode_shared_prefix(
        out.data_ptr(), query.data_ptr(), key_cache.data_ptr(), value_cache.data_ptr(),
        block_tables.data_ptr(), context_lens.data_ptr(), group_starts.data_ptr(),
        prefix_blocks.data_ptr(), float(scale), S, n_groups, int(max_group_size), H, Hk, D, NB,
        bs, MB, dt, _stream(stream))
    _check(st, "pa_decode_shared_prefix")


def pa_copy_blocks(key_cache: torch.Tensor, value_cache: torch.Tensor,
                   block_mapping: torch.Tensor, stream=None) -> None:
    """Copy whole blocks (copy-on-write): block_mapping [n, 2] int64 holds
    (source, destination) pairs; caches [NB, bs, Hk, D] contiguous."""
    NB, bs, Hk, D = key_cache.shape
    _need(value_cache.shape == key_cache.shape and key_cache.dtype == value_cache.dtype,
          "key/value caches differ")
    _need(key_cache.is_contiguous() and value_cache.is_contiguous(), "caches must be contiguous")
    _need(block_mapping.dtype == torch.int64 and block_mapping.dim() == 2 and
          block_mapping.shape[1] == 2 and block_mapping.is_contiguous(),
          "block_mapping must be [n, 2] int64")
    st = load().pa_copy_blocks(key_cache.data_ptr(), value_cache.data_ptr(),
                               block_mapping.data_ptr(), block_mapping.shape[0], NB, bs, Hk, D,
                               key_cache.element_size(), _stream(stream))
    _check(st, "pa_copy_blocks")


def _fp8_caches(key_cache, value_cache):
    _need(key_cache.dtype == torch.uint8 and value_cache.dtype == torch.uint8,
          "fp8 caches are uint8 tensors of E4M3 codes")
    _need(key_cache.shape == value_cache.shape and key_cache.dim() == 4, "cache shapes")
    _need(key_cache.is_contiguous() and value_cache.is_contiguous(), "caches must be contiguous")
    return key_cache.shape


def pa_reshape_and_cache_fp8(key: torch.Tensor, value: torch.Tensor, key_cache: torch.Tensor,
                             value_cache: torch.Tensor, slot_mapping: torch.Tensor,
                             k_scale: float, v_scale: float, stream=None) -> None:
    """Quantising write of 16-bit key/value [T, Hk, D] into uint8 E4M3 caches."""
    T, Hk, D = key.shape
    NB, bs, _, _ = _fp8_caches(key_cache, value_cache)
    _need(value.shape == key.shape and key.dtype == value.dtype, "key/value differ")
    _need(key.stride()[1:] == (D, 1) and value.stride()[1:] == (D, 1), "rows must be dense")
    _need(slot_mapping.dtype == torch.int64 and slot_mapping.shape == (T,), "slot_mapping")
    st = load().pa_reshape_and_cache_fp8(
        key.data_ptr(), value.data_ptr(), key.stride(0) if T else Hk * D,
        value.stride(0) if T else Hk * D, key_cache.data_ptr(), value_cache.data_ptr(),
        slot_mapping.data_ptr(), T, Hk, D, NB, bs, float(k_scale), float(v_scale),
        _dtype_code(key), _stream(stream))
    _check(st, "pa_reshape_and_cache_fp8")


def _fp8_attention_common(query, key_cache, value_cache, block_tables, context_lens):
    S, H, D = query.shape
    NB, bs, Hk, D2 = _fp8_caches(key_cache, value_cache)
    _need(D2 == D, "head_dim of query and cache differ")
    _need(query.is_contiguous(), "query must be contiguous")
    _need(block_tables.dtype == torch.int32 and block_tables.dim() == 2 and
          block_tables.shape[0] == S and block_tables.is_contiguous(), "block_tables")
    _need(context_lens.dtype == torch.int32 and context_lens.shape == (S,), "context_lens")
    return S, H, D, NB, bs, Hk, block_tables.shape[1], _dtype_code(query)


def pa_decode_fp8(out: torch.Tensor, query: torch.Tensor, key_cache: torch.Tensor,
                  value_cache: torch.Tensor, block_tables: torch.Tensor,
                  context_lens: torch.Tensor, scale: float, k_scale: float, v_scale: float,
                  stream=None) -> None:
    S, H, D, NB, bs, Hk, MB, dt = _fp8_attention_common(query, key_cache, value_cache,
                                                        block_tables, context_lens)
    _need(out.shape == query.shape and out.dtype == query.dtype and out.is_contiguous(), "out")
    st = load().pa_decode_fp8(out.data_ptr(), query.data_ptr(), key_cache.data_ptr(),
                              value_cache.data_ptr(), block_tables.data_ptr(),
                              context_lens.data_ptr(), float(scale), float(k_scale),
                              float(v_scale), S, H, Hk, D, NB, bs, MB, dt, _stream(stream))
    _check(st, "pa_decode_fp8")


def pa_decode_split_fp8(tmp_out, max_logits, exp_sums, query, key_cache, value_cache,
                        block_tables, context_lens, scale: float, k_scale: float,
                        v_scale: float, partition_size: int, stream=None) -> None:
    S, H, D, NB, bs, Hk, MB, dt = _fp8_attention_common(query, key_cache, value_cache,
                                                        block_tables, context_lens)
    P = max_logits.shape[-1]
    _need(tmp_out.shape == (S, H, P, D) and tmp_out.dtype == torch.float32, "tmp_out")
    _need(max_logits.shape == (S, H, P) and exp_sums.shape == (S, H, P), "partials")
    st = load().pa_decode_split_fp8(tmp_out.data_ptr(), max_logits.data_ptr(),
                                    exp_sums.data_ptr(), query.data_ptr(), key_cache.data_ptr(),
                                    value_cache.data_ptr(), block_tables.data_ptr(),
                                    context_lens.data_ptr(), float(scale), float(k_scale),
                                    float(v_scale), S, H, Hk, D, NB, bs, MB, int(partition_size),
                                    P, dt, _stream(stream))
    _check(st, "pa_decode_split_fp8")


def pa_prefill(out: torch.Tensor, query: torch.Tensor, key_cache: torch.Tensor,
               value_cache: torch.Tensor, block_tables: torch.Tensor,
               context_lens: torch.Tensor, query_starts: torch.Tensor, scale: float,
               max_query_len: int, stream=None) -> None:
    """Chunked prefill: query [T, H, D] rows grouped by sequence
    (query_starts [S + 1] int32); each sequence's rows are the last q_len
    positions of its context and attend causally over the paged cache."""
    T, H, D = query.shape
    NB, bs, Hk, D2 = key_cache.shape
    S = context_lens.shape[0]
    _need(D2 == D and value_cache.shape == key_cache.shape, "cache shapes")
    _need(query.is_contiguous() and key_cache.is_contiguous() and value_cache.is_contiguous(),
          "query and caches must be contiguous")
    _need(block_tables.dtype == torch.int32 and block_tables.shape[0] == S and
          block_tables.is_contiguous(), "block_tables must be [S, MB] int32")
    _need(context_lens.dtype == torch.int32, "context_lens must be int32")
    _need(query_starts.dtype == torch.int32 and query_starts.shape == (S + 1,),
          "query_starts must be [S + 1] int32")
    _need(out.shape == query.shape and out.dtype == query.dtype and out.is_contiguous(), "out")
    _need(query.dtype == key_cache.dtype == value_cache.dtype, "dtype mismatch")
    st = load().pa_prefill(out.data_ptr(), query.data_ptr(), key_cache.data_ptr(),
                           value_cache.data_ptr(), block_tables.data_ptr(),
                           context_lens.data_ptr(), query_starts.data_ptr(), float(scale), S, T,
                           int(max_query_len), H, Hk, D, NB, bs, block_tables.shape[1],
                           _dtype_code(query), _stream(stream))
    _check(st, "pa_prefill")


class DecodePlan:
    """One decode step (cache write, then attention) over fixed tensors,
    validated once: the argument lists of its C calls are built here, and
    run() only adds the stream.  Tensors are held by reference, so their
    contents may change between runs but not their storage.  The calls can
    be captured in a CUDA graph (run() inside torch.cuda.graph)."""

    def __init__(self, query, key, value, key_cache, value_cache, slot_mapping, block_tables,
                 context_lens, scale: float, out=None, partition_size: int = 0, workspace=None):
        S, H, D, NB, bs, Hk, MB, dt = _attention_common(query, key_cache, value_cache,
                                                        block_tables, context_lens)
        self.out = torch.empty_like(query) if out is None else out
        _need(self.out.shape == query.shape and self.out.dtype == query.dtype and
              self.out.is_contiguous(), "out must match query")
        self._keep = [query, key, value, key_cache, value_cache, slot_mapping, block_tables,
                      context_lens, self.out]
        self.calls = []
        if key is not None and key.shape[0] > 0:
            T = key.shape[0]
            _need(key.shape == (T, Hk, D) and value.shape == key.shape, "key/value shape")
            _need(key.stride()[1:] == (D, 1) and value.stride()[1:] == (D, 1), "rows dense")
            _need(slot_mapping.dtype == torch.int64 and slot_mapping.shape == (T,), "slots")
            self.calls.append(("pa_reshape_and_cache", (
                key.data_ptr(), value.data_ptr(), key.stride(0), value.stride(0),
                key_cache.data_ptr(), value_cache.data_ptr(), slot_mapping.data_ptr(), T, Hk, D,
                NB, bs, dt)))
        if partition_size > 0:
            if workspace is None:
                P = (MB * bs + partition_size - 1) // partition_size
                from . import SplitWorkspace
                workspace = SplitWorkspace(S, H, D, P, query.device)
            self._keep.append(workspace)
            P = workspace.max_partitions
            self.calls.append(("pa_decode_split", (
                workspace.tmp_out.data_ptr(), workspace.max_logits.data_ptr(),
                workspace.exp_sums.data_ptr(), query.data_ptr(), key_cache.data_ptr(),
                value_cache.data_ptr(), block_tables.data_ptr(), context_lens.data_ptr(),
                float(scale), S, H, Hk, D, NB, bs, MB, int(partition_size), P, dt)))
            self.calls.append(("pa_reduce", (
                self.out.data_ptr(), workspace.tmp_out.data_ptr(),
                workspace.max_logits.data_ptr(), workspace.exp_sums.data_ptr(),
                context_lens.data_ptr(), S, H, D, int(partition_size), P, dt)))
        else:
            self.calls.append(("pa_decode", (
                self.out.data_ptr(), query.data_ptr(), key_cache.data_ptr(),
                value_cache.data_ptr(), block_tables.data_ptr(), context_lens.data_ptr(),
                float(scale), S, H, Hk, D, NB, bs, MB, dt)))
        lib = load()
        self._bound = [(getattr(lib, name), args, name) for name, args in self.calls]

    def run(self, stream=None) -> torch.Tensor:
        s = _stream(stream)
        for fn, args, name in self._bound:
            st = fn(*args, s)
            if st != PA_OK:
                raise PagedAttentionError(st, name)
        return self.out


class HostStep:
    """pa_decode_step_host for one layer: per-step inputs live in (pinned)
    host tensors, the caches and a device workspace stay resident.  `run()`
    enqueues copies in, the cache write, attention and the copy out."""

    def __init__(self, key_cache, value_cache, num_seqs, num_heads, max_blocks_per_seq,
                 scale: float, partition_size: int = 0, dtype=torch.float16):
        NB, bs, Hk, D = key_cache.shape
        self.key_cache, self.value_cache = key_cache, value_cache
        self.dims = (num_seqs, num_heads, Hk, D, NB, bs, max_blocks_per_seq)
        self.scale, self.partition_size, self.dtype = float(scale), int(partition_size), dtype
        n = load().pa_decode_step_host_workspace_bytes(num_seqs, num_heads, Hk, D,
                                                       max_blocks_per_seq, bs, partition_size)
        _need(n >= 0, "bad step sizes")
        self.workspace = torch.empty(n, dtype=torch.uint8, device=key_cache.device)
        # one pinned host buffer laid out like the workspace (key, value,
        # slot_mapping, then query, block_tables, context_lens), so each of the
        # step's two input stages travels in a single copy
        S, H, D_ = num_seqs, num_heads, D
        parts = [((S, Hk, D_), dtype), ((S, Hk, D_), dtype), ((S,), torch.int64),
                 ((S, H, D_), dtype), ((S, max_blocks_per_seq), torch.int32), ((S,), torch.int32)]
        offs, at = [], 0
        for shape, dt in parts:
            offs.append(at)
            nbytes = int(torch.Size(shape).numel()) * torch.tensor([], dtype=dt).element_size()
            at = (at + nbytes + 255) // 256 * 256
        self.staging = torch.empty(at, dtype=torch.uint8).pin_memory()
        views = []
        for (shape, dt), o in zip(parts, offs):
            nbytes = int(torch.Size(shape).numel()) * torch.tensor([], dtype=dt).element_size()
            views.append(self.staging[o:o + nbytes].view(dt).view(shape))
        (self.key, self.value, self.slot_mapping, self.query, self.block_tables,
         self.context_lens) = views
        # pinned, so the attention writes its output straight into it
        self.out = torch.empty((S, H, D_), dtype=dtype).pin_memory()

    @property
    def h2d_bytes(self) -> int:
        return sum(t.numel() * t.element_size() for t in
                   (self.query, self.key, self.value, self.slot_mapping, self.block_tables,
                    self.context_lens))

    @property
    def d2h_bytes(self) -> int:
        return self.out.numel() * self.out.element_size()

    def run(self, stream=None) -> None:
        S, H, Hk, D, NB, bs, MB = self.dims
        # parts still in the staging buffer go as packed (NULL): one copy per stage
        packed = self.staging.data_ptr()
        inside = lambda t: packed <= t.data_ptr() < packed + self.staging.numel()
        kv_packed = all(inside(t) for t in (self.key, self.value, self.slot_mapping))
        q_packed = all(inside(t) for t in (self.query, self.block_tables, self.context_lens))
        st = load().pa_decode_step_host(
            self.out.data_ptr(), self.query.data_ptr(), self.key.data_ptr(),
            None if kv_packed else self.value.data_ptr(),
            None if kv_packed else self.slot_mapping.data_ptr(),
            None if q_packed else self.block_tables.data_ptr(),
            None if q_packed else self.context_lens.data_ptr(),
            self.key_cache.data_ptr(), self.value_cache.data_ptr(),
            self.workspace.data_ptr(), self.workspace.numel(), self.scale, S, H, Hk, D, NB, bs,
            MB, self.partition_size, DTYPE_CODES[self.dtype], _stream(stream))
        _check(st, "pa_decode_step_host")


def pa_check_error(stream=None) -> int:
    """Synchronise the stream; raise PagedAttentionError if a kernel met an
    out-of-range index since the last check; return 0 otherwise."""
    detail = _i64(0)
    st = load().pa_check_error(_stream(stream), ctypes.byref(detail))
    if st != PA_OK:
        raise PagedAttentionError(st, "pa_check_error", int(detail.value))
    return 0


def pa_selftest_wait_timeout(stream=None) -> None:
    """Run the bounded-wait failure path on purpose: a kernel waits (2 s) on a
    barrier nothing completes and records PA_CHECK_WAIT_TIMEOUT, which the
    next pa_check_error reports."""
    _check(load().pa_selftest_wait_timeout(_stream(stream)), "pa_selftest_wait_timeout")


NOALLOC_SCRATCH_BYTES = 64 * 1024 * 1024


def pa_decode_noalloc(out: torch.Tensor, query: torch.Tensor, key_cache: torch.Tensor,
                      value_cache: torch.Tensor, block_tables: torch.Tensor,
                      context_lens: torch.Tensor, scale: float, partition_size: int,
                      stream=None) -> None:
    """Long-context decode (split + merge) whose partition scratch is a fixed
    64 MiB device array inside libpa instead of caller-owned buffers, for
    callers that cannot allocate device memory when they call.  Calls that
    overlap on the GPU share that array and race; make the first call on a
    device before any stream capture."""
    S, H, D, NB, bs, Hk, MB, dt = _attention_common(query, key_cache, value_cache,
                                                    block_tables, context_lens)
    _need(out.shape == query.shape and out.dtype == query.dtype and out.is_contiguous(),
          "out must match query")
    parts = (MB * bs + partition_size - 1) // partition_size
    need = S * H * parts * (D + 2) * 4
    if need > NOALLOC_SCRATCH_BYTES:
        raise PagedAttentionError(2, f"pa_decode_noalloc needs {need} bytes of scratch, "
                                     f"more than its fixed {NOALLOC_SCRATCH_BYTES}")
    st = load().pa_decode_noalloc(out.data_ptr(), query.data_ptr(), key_cache.data_ptr(),
                                  value_cache.data_ptr(), block_tables.data_ptr(),
                                  context_lens.data_ptr(), float(scale), S, H, Hk, D, NB, bs, MB,
                                  int(partition_size), dt, _stream(stream))
    _check(st, "pa_decode_noalloc")
