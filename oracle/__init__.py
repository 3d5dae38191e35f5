"""fp64 CPU oracle for paged-KV-cache attention -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py``
may import this package.  It shares no code with the CUDA library: the attention,
cache-write and block-copy definitions live in ``pa_oracle.c`` (plain C, double
precision), the block allocator model in ``block_model.py`` (plain Python).

Every function takes numpy arrays.  bf16 data is carried as ``np.uint16`` bit
patterns, fp32 as ``np.float32``.  Attention results come back as ``np.float64``.
Parity of every function here is pinned by the ``-m "not gpu"`` tests in
``tests/test_oracle_pins.py`` and ``tests/test_block_model.py``.
"""
from __future__ import annotations

import ctypes as C
import os

import numpy as np

from . import build as _build
from .block_model import BlockManagerModel, OutOfBlocks  # noqa: F401

F32, BF16 = 0, 1

_lib = None


def _load():
    global _lib
    if _lib is None:
        path = _build.build()
        lib = C.CDLL(path)
        vp, i32, i64, dbl = C.c_void_p, C.c_int32, C.c_int64, C.c_double
        lib.oracle_decode.argtypes = [vp, vp, vp, C.c_int, i32, i32, i32, i32, vp, i32, vp, i32,
                                      i32, dbl, vp]
        lib.oracle_prefill.argtypes = [vp, vp, vp, C.c_int, i32, i32, i32, i32, vp, i32, vp, vp,
                                       i32, i32, i32, dbl, vp, vp]
        lib.oracle_cache_write.argtypes = [vp, vp, vp, i32, vp, vp, i32, i32, i32, i32, i32]
        lib.oracle_copy_blocks.argtypes = [vp, vp, vp, i32, i32, i64]
        for f in ("oracle_decode", "oracle_prefill", "oracle_cache_write", "oracle_copy_blocks"):
            getattr(lib, f).restype = C.c_int
        lib.oracle_e4m3_encode.argtypes = [vp, i64, C.c_float, vp]
        lib.oracle_e4m3_decode.argtypes = [vp, i64, vp]
        lib.oracle_cache_write_fp8.argtypes = [vp, vp, vp, i32, vp, vp, i32, i32, i32, i32, C.c_float, C.c_float]
        lib.oracle_cache_write_fp8.restype = C.c_int
        lib.oracle_decode_fp8.argtypes = [vp, vp, vp, i32, i32, i32, i32, vp, i32, vp, i32, i32, dbl, dbl,
                                          dbl, vp]
        lib.oracle_decode_fp8.restype = C.c_int
        lib.oracle_num_threads.restype = C.c_int
        lib.oracle_set_num_threads.argtypes = [C.c_int]
        _lib = lib
    return _lib


def _ptr(a: np.ndarray):
    assert a.flags.c_contiguous, "oracle inputs must be C-contiguous"
    return a.ctypes.data_as(C.c_void_p)


def _dtype_code(a: np.ndarray) -> int:
    if a.dtype == np.float32:
        return F32
    if a.dtype == np.uint16:
        return BF16
    raise TypeError(f"oracle takes float32 or bf16-as-uint16, got {a.dtype}")


def num_threads() -> int:
    return _load().oracle_num_threads()


def set_num_threads(n: int) -> None:
    _load().oracle_set_num_threads(int(n))


def decode(q, k_cache, v_cache, block_tables, context_lens, scale):
    """Decode attention, one query token per sequence.

    q [S, Hq, d]; k_cache/v_cache [NB, Hkv, B, d]; block_tables int32 [S, max_blocks];
    context_lens int32 [S].  Returns float64 [S, Hq, d].
    """
    S, Hq, d = q.shape
    NB, Hkv, B, d2 = k_cache.shape
    assert d == d2 and v_cache.shape == k_cache.shape and Hq % Hkv == 0
    assert q.dtype == k_cache.dtype == v_cache.dtype
    bt = np.ascontiguousarray(block_tables, dtype=np.int32)
    cl = np.ascontiguousarray(context_lens, dtype=np.int32)
    out = np.zeros((S, Hq, d), dtype=np.float64)
    rc = _load().oracle_decode(_ptr(q), _ptr(k_cache), _ptr(v_cache), _dtype_code(q), NB, Hkv, B,
                               d, _ptr(bt), bt.shape[1], _ptr(cl), S, Hq, float(scale), _ptr(out))
    if rc != 0:
        raise ValueError(f"oracle_decode failed with code {rc}")
    return out


def prefill(q, k_cache, v_cache, block_tables, context_lens, chunk_lens, scale, row_mask=None):
    """Causal chunked prefill against the paged cache.

    q [S, max_chunk, Hq, d]: row i of sequence s is at position
    context_lens[s] - chunk_lens[s] + i and attends to keys 0..that position.
    row_mask (bool [S, max_chunk]) selects the rows to compute (others stay NaN).
    Returns float64 [S, max_chunk, Hq, d].
    """
    S, MC, Hq, d = q.shape
    NB, Hkv, B, d2 = k_cache.shape
    assert d == d2 and v_cache.shape == k_cache.shape and Hq % Hkv == 0
    bt = np.ascontiguousarray(block_tables, dtype=np.int32)
    cl = np.ascontiguousarray(context_lens, dtype=np.int32)
    ch = np.ascontiguousarray(chunk_lens, dtype=np.int32)
    out = np.full((S, MC, Hq, d), np.nan, dtype=np.float64)
    mask = None if row_mask is None else np.ascontiguousarray(row_mask, dtype=np.uint8)
    rc = _load().oracle_prefill(_ptr(q), _ptr(k_cache), _ptr(v_cache), _dtype_code(q), NB, Hkv, B,
                                d, _ptr(bt), bt.shape[1], _ptr(cl), _ptr(ch), S, MC, Hq,
                                float(scale), None if mask is None else _ptr(mask), _ptr(out))
    if rc != 0:
        raise ValueError(f"oracle_prefill failed with code {rc}")
    return out


def cache_write(k, v, slot_mapping, k_cache, v_cache):
    """Scatter k, v [T, Hkv, d] into the pools (in place) at slot_mapping int64 [T]."""
    T, Hkv, d = k.shape
    NB, Hkv2, B, d2 = k_cache.shape
    assert (Hkv, d) == (Hkv2, d2) and k.dtype == k_cache.dtype and v.shape == k.shape
    sm = np.ascontiguousarray(slot_mapping, dtype=np.int64)
    rc = _load().oracle_cache_write(_ptr(k), _ptr(v), _ptr(sm), T, _ptr(k_cache), _ptr(v_cache),
                                    NB, Hkv, B, d, k.dtype.itemsize)
    if rc != 0:
        raise ValueError("oracle_cache_write: slot outside the pool")


def copy_blocks(k_cache, v_cache, pairs):
    """Copy whole blocks src -> dst (in place) for each row (src, dst) of pairs int32 [P, 2]."""
    NB = k_cache.shape[0]
    pr = np.ascontiguousarray(pairs, dtype=np.int32).reshape(-1, 2)
    block_bytes = k_cache[0].nbytes
    rc = _load().oracle_copy_blocks(_ptr(k_cache), _ptr(v_cache), _ptr(pr), pr.shape[0], NB,
                                    block_bytes)
    if rc != 0:
        raise ValueError("oracle_copy_blocks: block id outside the pool")


def lib_path() -> str:
    return os.path.abspath(_build.LIB)


# ---- FP8 (e4m3) KV cache -----------------------------------------------------
def e4m3_encode(x, scale=1.0):
    """uint8 e4m3 codes of float32(x) / float32(scale): nearest, ties to even,
    saturated to +-448, NaN -> 0x7F."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty(x.shape, np.uint8)
    _load().oracle_e4m3_encode(_ptr(x), x.size, float(np.float32(scale)), _ptr(out))
    return out


def e4m3_decode(codes):
    """Exact float64 values of uint8 e4m3 codes."""
    c = np.ascontiguousarray(codes, dtype=np.uint8)
    out = np.empty(c.shape, np.float64)
    _load().oracle_e4m3_decode(_ptr(c), c.size, _ptr(out))
    return out


def cache_write_fp8(k, v, slot_mapping, k_cache, v_cache, k_scale, v_scale):
    """Append bf16 K/V [T, Hkv, d] into uint8 e4m3 pools [NB, Hkv, 16, d]."""
    assert k.dtype == v.dtype == np.uint16 and k_cache.dtype == v_cache.dtype == np.uint8
    nb, nkv, bs, d = k_cache.shape
    sl = np.ascontiguousarray(slot_mapping, dtype=np.int64)
    st = _load().oracle_cache_write_fp8(_ptr(np.ascontiguousarray(k)), _ptr(np.ascontiguousarray(v)), _ptr(sl),
                                        len(sl), _ptr(k_cache), _ptr(v_cache), nb, nkv, bs, d,
                                        float(np.float32(k_scale)), float(np.float32(v_scale)))
    if st != 0:
        raise IndexError("slot beyond the pool")


def decode_fp8(q, k_cache, v_cache, block_tables, context_lens, scale, k_scale, v_scale):
    """Decode attention over e4m3 pools: bf16 q [S, Hq, d] -> float64 [S, Hq, d]."""
    assert q.dtype == np.uint16 and k_cache.dtype == np.uint8
    nb, nkv, bs, d = k_cache.shape
    S, hq, _ = q.shape
    t = np.ascontiguousarray(block_tables, dtype=np.int32)
    l = np.ascontiguousarray(context_lens, dtype=np.int32)
    out = np.zeros((S, hq, d), np.float64)
    st = _load().oracle_decode_fp8(_ptr(np.ascontiguousarray(q)), _ptr(k_cache), _ptr(v_cache), nb, nkv, bs, d,
                                   _ptr(t), t.shape[1], _ptr(l), S, hq, float(scale),
                                   float(np.float32(k_scale)), float(np.float32(v_scale)), _ptr(out))
    if st != 0:
        raise ValueError(f"oracle_decode_fp8 failed ({st})")
    return out

