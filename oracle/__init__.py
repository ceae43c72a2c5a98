"""fp64 CPU oracle for paged decode attention and the paged cache write.

TEST INFRASTRUCTURE ONLY.  The tests, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` use it; the
product package never imports it, and it shares no code with the CUDA path.

The arithmetic lives in ``pa_oracle.c`` (plain C, single thread, ``-O2``
without fast-math).  This module only compiles it with gcc, loads it with
ctypes and marshals numpy arrays.  16-bit floats cross the boundary as raw
``uint16`` bit patterns; results come back as ``float64``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import sys
from pathlib import Path

import numpy as np

_HERE = Path(__file__).resolve().parent
SOURCE = _HERE / "pa_oracle.c"
LIBRARY = _HERE / "libpa_oracle.so"

F16 = 0
BF16 = 1

OK = 0
BAD_ARG = 1
BAD_BLOCK = 2
BAD_SLOT = 3
NO_MEMORY = 4

_CFLAGS = ["-O2", "-std=c11", "-fPIC", "-shared", "-fno-fast-math", "-ffp-contract=off"]


def compile_oracle(source: Path = SOURCE, output: Path = LIBRARY) -> Path:
    """Compile the C oracle into a shared library with gcc (no fast-math)."""
    output = Path(output)
    tmp = output.with_suffix(f".{os.getpid()}.tmp.so")
    cmd = ["gcc", *_CFLAGS, "-o", str(tmp), str(source), "-lm"]
    subprocess.run(cmd, check=True, capture_output=True, text=True)
    os.replace(tmp, output)
    return output


def _needs_build(source: Path, output: Path) -> bool:
    return (not output.exists()) or output.stat().st_mtime < source.stat().st_mtime


_i64 = ctypes.c_int64
_p = ctypes.c_void_p


class Oracle:
    """ctypes view of one compiled oracle library (the default one, or a
    deliberately broken copy built by the mutation tests)."""

    def __init__(self, lib_path: Path | str):
        self.path = Path(lib_path)
        self._tables: dict[int, np.ndarray] = {}
        lib = ctypes.CDLL(str(self.path))
        self._lib = lib
        lib.oracle_f16_to_f64.argtypes = [ctypes.c_uint16]
        lib.oracle_f16_to_f64.restype = ctypes.c_double
        lib.oracle_bf16_to_f64.argtypes = [ctypes.c_uint16]
        lib.oracle_bf16_to_f64.restype = ctypes.c_double
        lib.oracle_f64_to_f16.argtypes = [ctypes.c_double]
        lib.oracle_f64_to_f16.restype = ctypes.c_uint16
        lib.oracle_f64_to_bf16.argtypes = [ctypes.c_double]
        lib.oracle_f64_to_bf16.restype = ctypes.c_uint16
        lib.oracle_kv_bytes_per_token.argtypes = [_i64] * 4
        lib.oracle_kv_bytes_per_token.restype = _i64
        lib.oracle_page_size_bytes.argtypes = [_i64] * 4
        lib.oracle_page_size_bytes.restype = _i64
        lib.oracle_num_blocks.argtypes = [_i64] * 3
        lib.oracle_num_blocks.restype = _i64
        lib.oracle_slot.argtypes = [_p, _i64, _i64]
        lib.oracle_slot.restype = _i64
        lib.oracle_reshape_and_cache.argtypes = [_p] * 5 + [_i64] * 7
        lib.oracle_reshape_and_cache.restype = ctypes.c_int
        lib.oracle_decode.argtypes = [_p] * 6 + [_i64] * 7 + [ctypes.c_double, ctypes.c_int]
        lib.oracle_decode.restype = ctypes.c_int
        lib.oracle_decode_partitioned.argtypes = (
            [_p] * 8 + [_i64] * 7 + [ctypes.c_double, ctypes.c_int, _i64, _i64])
        lib.oracle_decode_partitioned.restype = ctypes.c_int
        lib.oracle_lse_merge.argtypes = [_p] * 5 + [_i64] * 5
        lib.oracle_lse_merge.restype = ctypes.c_int
        lib.oracle_copy_blocks.argtypes = [_p] * 3 + [_i64] * 6
        lib.oracle_copy_blocks.restype = ctypes.c_int
        lib.oracle_e4m3_to_f64.argtypes = [ctypes.c_uint8]
        lib.oracle_e4m3_to_f64.restype = ctypes.c_double
        lib.oracle_f64_to_e4m3.argtypes = [ctypes.c_double]
        lib.oracle_f64_to_e4m3.restype = ctypes.c_uint8
        lib.oracle_reshape_and_cache_fp8.argtypes = ([_p] * 5 + [_i64] * 7 +
                                                     [ctypes.c_float, ctypes.c_float, ctypes.c_int])
        lib.oracle_reshape_and_cache_fp8.restype = ctypes.c_int
        lib.oracle_decode_fp8.argtypes = ([_p] * 6 + [_i64] * 7 +
                                          [ctypes.c_double] * 3 + [ctypes.c_int])
        lib.oracle_decode_fp8.restype = ctypes.c_int
        lib.oracle_prefill.argtypes = [_p] * 7 + [_i64] * 7 + [ctypes.c_double, ctypes.c_int]
        lib.oracle_prefill.restype = ctypes.c_int

    # ---- scalar helpers -------------------------------------------------
    def f16_to_f64(self, bits: int) -> float:
        return self._lib.oracle_f16_to_f64(int(bits))

    def bf16_to_f64(self, bits: int) -> float:
        return self._lib.oracle_bf16_to_f64(int(bits))

    def f64_to_f16(self, x: float) -> int:
        return int(self._lib.oracle_f64_to_f16(float(x)))

    def f64_to_bf16(self, x: float) -> int:
        return int(self._lib.oracle_f64_to_bf16(float(x)))

    def decode_bits(self, bits: np.ndarray, dtype: int) -> np.ndarray:
        """Element-wise exact decode of 16-bit patterns to float64."""
        table = self._tables.get(dtype)
        if table is None:
            f = self.bf16_to_f64 if dtype == BF16 else self.f16_to_f64
            table = np.array([f(b) for b in range(65536)], dtype=np.float64)
            self._tables[dtype] = table
        return table[np.asarray(bits, dtype=np.uint16)]

    def round_to_dtype(self, x: np.ndarray, dtype: int) -> np.ndarray:
        """Round float64 values to 16-bit patterns, nearest-even."""
        f = self.f64_to_bf16 if dtype == BF16 else self.f64_to_f16
        flat = np.asarray(x, dtype=np.float64).ravel()
        return np.array([f(v) for v in flat], dtype=np.uint16).reshape(np.shape(x))

    def kv_bytes_per_token(self, num_layers, num_kv_heads, head_dim, elem_bytes) -> int:
        return int(self._lib.oracle_kv_bytes_per_token(num_layers, num_kv_heads, head_dim, elem_bytes))

    def page_size_bytes(self, num_kv_heads, head_dim, elem_bytes, block_size) -> int:
        return int(self._lib.oracle_page_size_bytes(num_kv_heads, head_dim, elem_bytes, block_size))

    def num_blocks(self, available_bytes, page_size_bytes, num_layers) -> int:
        return int(self._lib.oracle_num_blocks(available_bytes, page_size_bytes, num_layers))

    def slot(self, block_table: np.ndarray, pos: int, block_size: int) -> int:
        bt = np.ascontiguousarray(block_table, dtype=np.int32)
        return int(self._lib.oracle_slot(bt.ctypes.data, pos, block_size))

    # ---- array routines -------------------------------------------------
    def reshape_and_cache(self, key, value, key_cache, value_cache, slot_mapping,
                          num_blocks: int, block_size: int) -> int:
        """In-place byte-copy write of key/value [T, Hk, D] (uint16 bits,
        rows may be strided views of a larger buffer) into the caches
        [NB, bs, Hk, D] (uint16 bits, contiguous).  Returns the oracle code."""
        assert key_cache.dtype == np.uint16 and key_cache.flags.c_contiguous
        assert value_cache.dtype == np.uint16 and value_cache.flags.c_contiguous
        T, Hk, D = key.shape
        key_stride = key.strides[0] // 2 if T > 0 else Hk * D
        value_stride = value.strides[0] // 2 if T > 0 else Hk * D
        assert key.strides[1:] == (D * 2, 2) and value.strides[1:] == (D * 2, 2)
        slots = np.ascontiguousarray(slot_mapping, dtype=np.int64)
        return int(self._lib.oracle_reshape_and_cache(
            key.ctypes.data, value.ctypes.data, key_cache.ctypes.data,
            value_cache.ctypes.data, slots.ctypes.data, T, Hk, D, num_blocks,
            block_size, key_stride, value_stride))

    def e4m3_to_f64(self, bits: int) -> float:
        return self._lib.oracle_e4m3_to_f64(int(bits))

    def f64_to_e4m3(self, x: float) -> int:
        return int(self._lib.oracle_f64_to_e4m3(float(x)))

    def reshape_and_cache_fp8(self, key, value, key_cache, value_cache, slot_mapping,
                              num_blocks: int, block_size: int, k_scale: float, v_scale: float,
                              dtype: int) -> int:
        """Quantising write of 16-bit key/value [T, Hk, D] into uint8 E4M3
        caches [NB, bs, Hk, D] (in place)."""
        assert key_cache.dtype == np.uint8 and key_cache.flags.c_contiguous
        assert value_cache.dtype == np.uint8 and value_cache.flags.c_contiguous
        T, Hk, D = key.shape
        key_stride = key.strides[0] // 2 if T > 0 else Hk * D
        value_stride = value.strides[0] // 2 if T > 0 else Hk * D
        slots = np.ascontiguousarray(slot_mapping, dtype=np.int64)
        return int(self._lib.oracle_reshape_and_cache_fp8(
            key.ctypes.data, value.ctypes.data, key_cache.ctypes.data, value_cache.ctypes.data,
            slots.ctypes.data, T, Hk, D, num_blocks, block_size, key_stride, value_stride,
            float(k_scale), float(v_scale), dtype))

    def decode_fp8(self, query, key_cache, value_cache, block_tables, context_lens,
                   scale: float, k_scale: float, v_scale: float, dtype: int) -> np.ndarray:
        """softmax(scale q K^T) V with K = code * k_scale, V = code * v_scale."""
        q = np.ascontiguousarray(query, dtype=np.uint16)
        kc = np.ascontiguousarray(key_cache, dtype=np.uint8)
        vc = np.ascontiguousarray(value_cache, dtype=np.uint8)
        bt = np.ascontiguousarray(block_tables, dtype=np.int32)
        cl = np.ascontiguousarray(context_lens, dtype=np.int32)
        S, H, D = q.shape
        NB, bs, Hk, _ = kc.shape
        out = np.zeros((S, H, D), dtype=np.float64)
        rc = self._lib.oracle_decode_fp8(out.ctypes.data, q.ctypes.data, kc.ctypes.data,
                                         vc.ctypes.data, bt.ctypes.data, cl.ctypes.data,
                                         S, H, Hk, D, NB, bs, bt.shape[1], float(scale),
                                         float(k_scale), float(v_scale), dtype)
        if rc != OK:
            raise ValueError(f"oracle_decode_fp8 failed with code {rc}")
        return out

    def prefill(self, query, key_cache, value_cache, block_tables, context_lens, query_starts,
                scale: float, dtype: int) -> np.ndarray:
        """Causal attention of each sequence's last q_len positions (query
        [T, H, D], T = query_starts[-1]) over its paged context; float64 [T, H, D]."""
        q = np.ascontiguousarray(query, dtype=np.uint16)
        kc = np.ascontiguousarray(key_cache, dtype=np.uint16)
        vc = np.ascontiguousarray(value_cache, dtype=np.uint16)
        bt = np.ascontiguousarray(block_tables, dtype=np.int32)
        cl = np.ascontiguousarray(context_lens, dtype=np.int32)
        qs = np.ascontiguousarray(query_starts, dtype=np.int32)
        T, H, D = q.shape
        NB, bs, Hk, _ = kc.shape
        S = cl.shape[0]
        assert qs.shape == (S + 1,) and qs[-1] == T
        out = np.zeros((T, H, D), dtype=np.float64)
        rc = self._lib.oracle_prefill(out.ctypes.data, q.ctypes.data, kc.ctypes.data,
                                      vc.ctypes.data, bt.ctypes.data, cl.ctypes.data,
                                      qs.ctypes.data, S, H, Hk, D, NB, bs, bt.shape[1],
                                      float(scale), dtype)
        if rc != OK:
            raise ValueError(f"oracle_prefill failed with code {rc}")
        return out

    def copy_blocks(self, key_cache, value_cache, block_mapping) -> int:
        """In-place copy of whole blocks src -> dst (pairs [n, 2] int64) in
        both caches [NB, bs, Hk, D] (any fixed-size element, contiguous)."""
        assert key_cache.flags.c_contiguous and value_cache.flags.c_contiguous
        NB, bs, Hk, D = key_cache.shape
        pairs = np.ascontiguousarray(block_mapping, dtype=np.int64).reshape(-1, 2)
        return int(self._lib.oracle_copy_blocks(key_cache.ctypes.data, value_cache.ctypes.data,
                                                pairs.ctypes.data, pairs.shape[0], NB, bs, Hk,
                                                D, key_cache.itemsize))

    def decode(self, query, key_cache, value_cache, block_tables, context_lens,
               scale: float, dtype: int) -> np.ndarray:
        """softmax(scale * q k^T) v per (sequence, head), float64 [S, H, D]."""
        q = np.ascontiguousarray(query, dtype=np.uint16)
        kc = np.ascontiguousarray(key_cache, dtype=np.uint16)
        vc = np.ascontiguousarray(value_cache, dtype=np.uint16)
        bt = np.ascontiguousarray(block_tables, dtype=np.int32)
        cl = np.ascontiguousarray(context_lens, dtype=np.int32)
        S, H, D = q.shape
        NB, bs, Hk, D2 = kc.shape
        assert D2 == D and vc.shape == kc.shape and bt.shape[0] == S and cl.shape == (S,)
        out = np.zeros((S, H, D), dtype=np.float64)
        rc = self._lib.oracle_decode(out.ctypes.data, q.ctypes.data, kc.ctypes.data,
                                     vc.ctypes.data, bt.ctypes.data, cl.ctypes.data,
                                     S, H, Hk, D, NB, bs, bt.shape[1], float(scale), dtype)
        if rc != OK:
            raise ValueError(f"oracle_decode failed with code {rc}")
        return out

    def decode_partitioned(self, query, key_cache, value_cache, block_tables,
                           context_lens, scale: float, dtype: int,
                           partition_size: int, max_partitions: int):
        """Per-partition (acc, max, sum), each float64 [S, H, P(, D)];
        untouched partitions hold NaN."""
        q = np.ascontiguousarray(query, dtype=np.uint16)
        kc = np.ascontiguousarray(key_cache, dtype=np.uint16)
        vc = np.ascontiguousarray(value_cache, dtype=np.uint16)
        bt = np.ascontiguousarray(block_tables, dtype=np.int32)
        cl = np.ascontiguousarray(context_lens, dtype=np.int32)
        S, H, D = q.shape
        NB, bs, Hk, _ = kc.shape
        acc = np.full((S, H, max_partitions, D), np.nan)
        pmax = np.full((S, H, max_partitions), np.nan)
        psum = np.full((S, H, max_partitions), np.nan)
        rc = self._lib.oracle_decode_partitioned(
            acc.ctypes.data, pmax.ctypes.data, psum.ctypes.data, q.ctypes.data,
            kc.ctypes.data, vc.ctypes.data, bt.ctypes.data, cl.ctypes.data,
            S, H, Hk, D, NB, bs, bt.shape[1], float(scale), dtype,
            partition_size, max_partitions)
        if rc != OK:
            raise ValueError(f"oracle_decode_partitioned failed with code {rc}")
        return acc, pmax, psum

    def lse_merge(self, acc, pmax, psum, context_lens, partition_size: int) -> np.ndarray:
        acc = np.ascontiguousarray(acc, dtype=np.float64)
        pmax = np.ascontiguousarray(pmax, dtype=np.float64)
        psum = np.ascontiguousarray(psum, dtype=np.float64)
        cl = np.ascontiguousarray(context_lens, dtype=np.int32)
        S, H, P, D = acc.shape
        out = np.zeros((S, H, D), dtype=np.float64)
        rc = self._lib.oracle_lse_merge(out.ctypes.data, acc.ctypes.data, pmax.ctypes.data,
                                        psum.ctypes.data, cl.ctypes.data, S, H, D,
                                        partition_size, P)
        if rc != OK:
            raise ValueError(f"oracle_lse_merge failed with code {rc}")
        return out


_default: Oracle | None = None


def load() -> Oracle:
    """The oracle built from ``pa_oracle.c`` (compiled on first use)."""
    global _default
    if _default is None:
        if _needs_build(SOURCE, LIBRARY):
            compile_oracle()
        _default = Oracle(LIBRARY)
    return _default


if __name__ == "__main__":  # pragma: no cover
    print(compile_oracle())
    sys.exit(0)
