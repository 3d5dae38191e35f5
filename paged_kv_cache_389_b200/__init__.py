"""Thin Python binding of the sm_100a paged-KV-cache attention library.

Argument marshalling only: every function here checks shapes/dtypes of torch
tensors, fills the C structs and calls the same-named entry point of
``libpa_b200.so`` (declared in ``include/pa.h`` and ``include/pa_block_manager.h``).
All computation runs in the library's CUDA kernels; there is no fallback path.
If the shared library is missing the import fails loudly.
"""
from __future__ import annotations

import ctypes as C
import os

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libpa_b200.so")

PA_OK, PA_ERR_INVALID_ARG, PA_ERR_UNSUPPORTED, PA_ERR_OOM = 0, 1, 2, 3
PA_ERR_DEVICE_INDEX, PA_ERR_CUDA, PA_ERR_TIMEOUT, PA_ERR_NOT_FOUND = 4, 5, 6, 7
PA_F32, PA_BF16, PA_FP8_E4M3 = 0, 1, 2
PA_DEVERR_BLOCK_ID, PA_DEVERR_SLOT, PA_DEVERR_CONTEXT_LEN = 1, 2, 4
PA_DEVERR_PAIR, PA_DEVERR_TIMEOUT, PA_DEVERR_CHUNK = 8, 16, 32
BLOCK_SIZE = 16


class PAError(RuntimeError):
    def __init__(self, status: int, what: str = ""):
        self.status = int(status)
        super().__init__(f"{what}: {status_string(status)} ({status})" if what else status_string(status))


class CacheDesc(C.Structure):
    _fields_ = [("num_blocks", C.c_int32), ("num_kv_heads", C.c_int32), ("block_size", C.c_int32),
                ("head_dim", C.c_int32), ("dtype", C.c_int32), ("k_scale", C.c_float),
                ("v_scale", C.c_float)]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with `python paged_kv_cache_389_b200/build.py`")
    lib = C.CDLL(LIB_PATH)
    vp, i32, i64, f32, sz = C.c_void_p, C.c_int32, C.c_int64, C.c_float, C.c_size_t
    desc = C.POINTER(CacheDesc)
    sig = {
        "pa_abi_version": (i32, []),
        "pa_status_string": (C.c_char_p, [C.c_int]),
        "pa_cache_write": (C.c_int, [vp, vp, vp, i32, vp, vp, desc, vp, vp]),
        "pa_copy_blocks": (C.c_int, [vp, vp, vp, i32, desc, vp, vp]),
        "pa_check_copy_pairs": (C.c_int, [vp, i32, i32]),
        "pa_decode_workspace_size": (sz, [i32, i32, i32, i32, i32]),
        "pa_decode_launches": (i32, [i32, i32, i32, i32, i32, i32]),
        "pa_decode": (C.c_int, [vp, vp, vp, vp, i32, vp, i32, i32, i32, f32, i32, vp, sz, vp, desc,
                                vp, vp]),
        "pa_append_decode": (C.c_int, [vp, vp, vp, i32, vp, vp, vp, vp, i32, vp, i32, i32, i32, f32, i32,
                                       vp, sz, vp, desc, vp, vp]),
        "pa_prefill_chunk": (C.c_int, [vp, vp, vp, vp, i32, vp, vp, i32, i32, i32, f32, vp, desc,
                                       vp, vp]),
        "pa_wait": (C.c_int, [vp, vp, i32, C.POINTER(i32)]),
        "pa_set_wait_timeout_ns": (C.c_uint64, [C.c_uint64]),
        "pa_bm_create": (C.c_int, [i32, i32, vp, C.POINTER(vp)]),
        "pa_bm_destroy": (None, [vp]),
        "pa_bm_add_seq": (C.c_int, [vp, i64]),
        "pa_bm_append_slots": (C.c_int, [vp, i64, i32, vp, vp, i32, C.POINTER(i32)]),
        "pa_bm_append_step": (C.c_int, [vp, vp, vp, i32, vp, vp, i32, C.POINTER(i32)]),
        "pa_bm_fork": (C.c_int, [vp, i64, i64]),
        "pa_bm_free_seq": (C.c_int, [vp, i64]),
        "pa_bm_num_tokens": (i64, [vp, i64]),
        "pa_bm_num_seq_blocks": (i32, [vp, i64]),
        "pa_bm_max_seq_blocks": (i32, [vp, vp, i32]),
        "pa_bm_block_table": (C.c_int, [vp, i64, vp, i32, C.POINTER(i32)]),
        "pa_bm_build_tables": (C.c_int, [vp, vp, i32, i32, vp, vp]),
        "pa_bm_refcount": (i32, [vp, i32]),
        "pa_bm_num_free": (i32, [vp]),
        "pa_bm_num_blocks": (i32, [vp]),
        "pa_bm_block_size": (i32, [vp]),
        "pa_bm_free_stack": (i32, [vp, vp, i32]),
        "pa_bm_tokens_stored": (i64, [vp]),
        "pa_bm_add_seq_tokens": (C.c_int, [vp, i64, vp, i32, vp, C.POINTER(i32)]),
        "pa_bm_num_evictable": (i32, [vp]),
        "pa_bm_num_cached": (i32, [vp]),
        "pa_bm_evictable": (i32, [vp, vp, i32]),
        "pa_bm_snapshot_size": (sz, [vp]),
        "pa_bm_snapshot": (C.c_int, [vp, vp, sz, C.POINTER(sz)]),
        "pa_bm_restore": (C.c_int, [vp, sz, C.POINTER(vp)]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


_lib = _load()

EXPORTED = (
    "pa_abi_version", "pa_status_string", "pa_cache_write", "pa_copy_blocks", "pa_check_copy_pairs",
    "pa_decode_workspace_size", "pa_decode_launches", "pa_decode", "pa_append_decode", "pa_prefill_chunk",
    "pa_wait", "pa_set_wait_timeout_ns",
)


def status_string(status: int) -> str:
    return _lib.pa_status_string(int(status)).decode()


def abi_version() -> int:
    return _lib.pa_abi_version()


def _check(status: int, what: str):
    if status != PA_OK:
        raise PAError(status, what)


# ----------------------------------------------------------------- device calls
def _torch():
    import torch
    return torch


def _dtype_code(t) -> int:
    torch = _torch()
    if t.dtype == torch.bfloat16:
        return PA_BF16
    if t.dtype == torch.float32:
        return PA_F32
    if t.dtype == torch.float8_e4m3fn:
        return PA_FP8_E4M3
    raise TypeError(f"unsupported dtype {t.dtype}")


def io_dtype(key_cache):
    """dtype of queries, outputs and appended K/V for a pool: bf16 for an fp8 pool."""
    torch = _torch()
    return torch.bfloat16 if key_cache.dtype == torch.float8_e4m3fn else key_cache.dtype


def cache_desc(key_cache, k_scale=1.0, v_scale=1.0) -> CacheDesc:
    """Descriptor of a pool tensor [num_blocks, num_kv_heads, block_size, head_dim]; the
    scales matter for torch.float8_e4m3fn pools only."""
    nb, hkv, bs, d = key_cache.shape
    return CacheDesc(nb, hkv, bs, d, _dtype_code(key_cache), float(k_scale), float(v_scale))


def _ptr(t):
    if t is None:
        return None
    assert t.is_contiguous(), "tensors passed to the library must be contiguous"
    return C.c_void_p(t.data_ptr())


def _stream(stream):
    torch = _torch()
    s = stream if stream is not None else torch.cuda.current_stream()
    return C.c_void_p(s.cuda_stream)


def _same_pool(key_cache, value_cache):
    assert key_cache.shape == value_cache.shape and key_cache.dtype == value_cache.dtype
    assert key_cache.is_cuda and value_cache.is_cuda


def pa_cache_write(key, value, slot_mapping, key_cache, value_cache, err_flag=None, stream=None,
                   k_scale=1.0, v_scale=1.0):
    """Scatter key/value [T, Hkv, d] into the pools at slot_mapping (int64 [T]); fp8 pools
    store e4m3(x / k_scale) and e4m3(x / v_scale)."""
    torch = _torch()
    _same_pool(key_cache, value_cache)
    assert key.shape == value.shape and key.dim() == 3 and key.shape[1:] == (key_cache.shape[1], key_cache.shape[3])
    assert key.dtype == io_dtype(key_cache) == value.dtype and slot_mapping.dtype == torch.int64
    assert slot_mapping.shape == (key.shape[0],)
    d = cache_desc(key_cache, k_scale, v_scale)
    _check(_lib.pa_cache_write(_ptr(key), _ptr(value), _ptr(slot_mapping), key.shape[0],
                               _ptr(key_cache), _ptr(value_cache), C.byref(d), _ptr(err_flag),
                               _stream(stream)), "pa_cache_write")


def pa_copy_blocks(key_cache, value_cache, src_dst_pairs, err_flag=None, stream=None):
    """Copy whole blocks src -> dst for each row of int32 [P, 2]."""
    torch = _torch()
    _same_pool(key_cache, value_cache)
    assert src_dst_pairs.dtype == torch.int32 and src_dst_pairs.dim() == 2 and src_dst_pairs.shape[1] == 2
    d = cache_desc(key_cache)
    if d.dtype == PA_FP8_E4M3:
        d.k_scale = d.v_scale = 1.0       # a byte copy: the scales are not used
    _check(_lib.pa_copy_blocks(_ptr(key_cache), _ptr(value_cache), _ptr(src_dst_pairs),
                               src_dst_pairs.shape[0], C.byref(d), _ptr(err_flag), _stream(stream)),
           "pa_copy_blocks")


def pa_check_copy_pairs(pairs, num_blocks) -> int:
    """Host-side check of copy pairs (int32 [P, 2], host memory): PA_OK or PA_ERR_INVALID_ARG."""
    arr = np.ascontiguousarray(np.asarray(pairs, dtype=np.int32).reshape(-1, 2))
    return int(_lib.pa_check_copy_pairs(arr.ctypes.data_as(C.c_void_p) if len(arr) else None, len(arr),
                                        int(num_blocks)))


def pa_decode_workspace_size(num_seqs, num_q_heads, head_dim, max_context_len, partition_size) -> int:
    return int(_lib.pa_decode_workspace_size(num_seqs, num_q_heads, head_dim, max_context_len,
                                             partition_size))


def pa_decode_launches(num_seqs, num_q_heads, num_kv_heads, head_dim, dtype, partition_size) -> int:
    """Kernels one pa_decode call launches; dtype PA_F32 / PA_BF16 / PA_FP8_E4M3."""
    return int(_lib.pa_decode_launches(num_seqs, num_q_heads, num_kv_heads, head_dim, dtype, partition_size))


def pa_decode(query, key_cache, value_cache, block_tables, context_lens, max_context_len, scale,
              out, partition_size=0, workspace=None, err_flag=None, stream=None, k_scale=1.0, v_scale=1.0):
    """Decode attention; query/out [S, Hq, d]; tables int32 [S, max_blocks]; lens int32 [S]."""
    torch = _torch()
    _same_pool(key_cache, value_cache)
    S, hq, dd = query.shape
    assert out.shape == query.shape and out.dtype == query.dtype == io_dtype(key_cache)
    assert block_tables.dtype == torch.int32 and block_tables.dim() == 2 and block_tables.shape[0] == S
    assert context_lens.dtype == torch.int32 and context_lens.shape == (S,)
    d = cache_desc(key_cache, k_scale, v_scale)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(_lib.pa_decode(_ptr(query), _ptr(key_cache), _ptr(value_cache), _ptr(block_tables),
                          block_tables.shape[1], _ptr(context_lens), int(max_context_len), S, hq,
                          float(scale), int(partition_size), _ptr(workspace), ws_bytes, _ptr(out),
                          C.byref(d), _ptr(err_flag), _stream(stream)), "pa_decode")


def pa_append_decode(key, value, slot_mapping, query, key_cache, value_cache, block_tables, context_lens,
                     max_context_len, scale, out, partition_size=0, workspace=None, err_flag=None,
                     stream=None, k_scale=1.0, v_scale=1.0):
    """pa_cache_write(key, value, slot_mapping, ...) then pa_decode(...) in one call."""
    torch = _torch()
    _same_pool(key_cache, value_cache)
    assert key.shape == value.shape and key.dim() == 3 and key.shape[1:] == (key_cache.shape[1], key_cache.shape[3])
    assert key.dtype == io_dtype(key_cache) == value.dtype and slot_mapping.dtype == torch.int64
    assert slot_mapping.shape == (key.shape[0],)
    S, hq, dd = query.shape
    assert out.shape == query.shape and out.dtype == query.dtype == io_dtype(key_cache)
    assert block_tables.dtype == torch.int32 and block_tables.dim() == 2 and block_tables.shape[0] == S
    assert context_lens.dtype == torch.int32 and context_lens.shape == (S,)
    d = cache_desc(key_cache, k_scale, v_scale)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(_lib.pa_append_decode(_ptr(key), _ptr(value), _ptr(slot_mapping), key.shape[0], _ptr(query),
                                 _ptr(key_cache), _ptr(value_cache), _ptr(block_tables), block_tables.shape[1],
                                 _ptr(context_lens), int(max_context_len), S, hq, float(scale),
                                 int(partition_size), _ptr(workspace), ws_bytes, _ptr(out), C.byref(d),
                                 _ptr(err_flag), _stream(stream)), "pa_append_decode")


def pa_prefill_chunk(query, key_cache, value_cache, block_tables, context_lens, chunk_lens, scale,
                     out, err_flag=None, stream=None):
    """Causal chunked prefill; query/out [S, max_chunk, Hq, d]."""
    torch = _torch()
    _same_pool(key_cache, value_cache)
    S, mc, hq, dd = query.shape
    assert out.shape == query.shape and out.dtype == query.dtype == key_cache.dtype
    assert block_tables.dtype == torch.int32 and block_tables.shape[0] == S
    assert context_lens.dtype == torch.int32 and chunk_lens.dtype == torch.int32
    d = cache_desc(key_cache)
    _check(_lib.pa_prefill_chunk(_ptr(query), _ptr(key_cache), _ptr(value_cache), _ptr(block_tables),
                                 block_tables.shape[1], _ptr(context_lens), _ptr(chunk_lens), S, mc,
                                 hq, float(scale), _ptr(out), C.byref(d), _ptr(err_flag),
                                 _stream(stream)), "pa_prefill_chunk")


def pa_wait(err_flag=None, stream=None, timeout_ms: int = 10000) -> int:
    """Wait for the stream (bounded) and return the device error flag (raises on CUDA errors)."""
    flag = C.c_int32(0)
    st = _lib.pa_wait(_stream(stream), _ptr(err_flag), int(timeout_ms), C.byref(flag))
    if st not in (PA_OK, PA_ERR_DEVICE_INDEX, PA_ERR_TIMEOUT) or (st == PA_ERR_TIMEOUT and flag.value == 0):
        raise PAError(st, "pa_wait")
    return int(flag.value)


def pa_set_wait_timeout_ns(ns: int) -> int:
    """Bound of every in-kernel wait of later launches (0: the 1 s default); returns the
    previous bound."""
    return int(_lib.pa_set_wait_timeout_ns(int(ns)))


# ------------------------------------------------------------------ host manager
class OutOfBlocks(PAError):
    pass


class BlockManager:
    """Host C++ block allocator (pa_bm_*): LIFO free list, reference counts, fork, CoW."""

    def __init__(self, num_blocks: int, block_size: int = BLOCK_SIZE, free_order=None):
        h = C.c_void_p()
        fo = None
        if free_order is not None:
            self._fo = np.ascontiguousarray(free_order, dtype=np.int32)
            assert self._fo.shape == (num_blocks,)
            fo = self._fo.ctypes.data_as(C.c_void_p)
        _check(_lib.pa_bm_create(int(num_blocks), int(block_size), fo, C.byref(h)), "pa_bm_create")
        self._h = h
        self.num_blocks = int(num_blocks)
        self.block_size = int(block_size)

    def snapshot(self) -> bytes:
        """The manager's whole state as bytes (pa_bm_snapshot)."""
        n = int(_lib.pa_bm_snapshot_size(self._h))
        buf = (C.c_ubyte * max(n, 1))()
        got = C.c_size_t(0)
        _check(_lib.pa_bm_snapshot(self._h, buf, n, C.byref(got)), "pa_bm_snapshot")
        return bytes(buf[:got.value])

    @classmethod
    def restore(cls, data: bytes) -> "BlockManager":
        """A new manager from snapshot() bytes (pa_bm_restore)."""
        raw = bytes(data)
        h = C.c_void_p()
        _check(_lib.pa_bm_restore(raw, len(raw), C.byref(h)), "pa_bm_restore")
        self = cls.__new__(cls)
        self._h = h
        self.num_blocks = int(_lib.pa_bm_num_blocks(h))
        self.block_size = int(_lib.pa_bm_block_size(h))
        return self

    def __del__(self):
        h = getattr(self, "_h", None)
        if h and _lib is not None:  # at interpreter exit the module globals may be gone
            _lib.pa_bm_destroy(h)
            self._h = None

    def _st(self, st, what):
        if st == PA_ERR_OOM:
            raise OutOfBlocks(st, what)
        if st == PA_ERR_NOT_FOUND:
            raise KeyError(what)
        _check(st, what)

    def add_seq(self, seq: int):
        self._st(_lib.pa_bm_add_seq(self._h, int(seq)), f"add_seq({seq})")

    def append_step(self, seqs, counts=None):
        """One step for distinct sequences in one call (all or nothing): append counts[i]
        tokens (default 1) to seqs[i] in order.  Returns (int64 slots [sum counts],
        int32 copy pairs [P, 2])."""
        ids = np.ascontiguousarray(seqs, dtype=np.int64)
        cnt = None if counts is None else np.ascontiguousarray(counts, dtype=np.int32)
        total = len(ids) if cnt is None else int(cnt.sum())
        slots = np.empty(max(total, 1), dtype=np.int64)
        pairs = np.empty((max(len(ids), 1), 2), dtype=np.int32)   # at most one copy per sequence
        ncow = C.c_int32(0)
        self._st(_lib.pa_bm_append_step(self._h, ids.ctypes.data_as(C.c_void_p),
                                        None if cnt is None else cnt.ctypes.data_as(C.c_void_p), len(ids),
                                        slots.ctypes.data_as(C.c_void_p), pairs.ctypes.data_as(C.c_void_p),
                                        len(pairs), C.byref(ncow)),
                 f"append_step({len(ids)} sequences)")
        return slots[:total].copy(), pairs[:ncow.value].copy()

    def append_slots(self, seq: int, n: int):
        """Append n tokens; return (int64 slots [n], list of (src, dst) copy pairs)."""
        slots = np.empty(int(n), dtype=np.int64)
        pairs = np.empty(2, dtype=np.int32)   # at most one copy per call
        ncow = C.c_int32(0)
        self._st(_lib.pa_bm_append_slots(self._h, int(seq), int(n), slots.ctypes.data_as(C.c_void_p),
                                         pairs.ctypes.data_as(C.c_void_p), 1, C.byref(ncow)),
                 f"append_slots({seq}, {n})")
        return slots, [(int(pairs[0]), int(pairs[1]))] if ncow.value else []

    def append_slot(self, seq: int):
        slots, pairs = self.append_slots(seq, 1)
        return int(slots[0]), (pairs[0] if pairs else None)

    def fork(self, parent: int, child: int):
        self._st(_lib.pa_bm_fork(self._h, int(parent), int(child)), f"fork({parent}, {child})")

    def free(self, seq: int):
        self._st(_lib.pa_bm_free_seq(self._h, int(seq)), f"free({seq})")

    def num_tokens(self, seq: int) -> int:
        return int(_lib.pa_bm_num_tokens(self._h, int(seq)))

    def num_seq_blocks(self, seq: int) -> int:
        n = int(_lib.pa_bm_num_seq_blocks(self._h, int(seq)))
        if n < 0:
            raise KeyError(seq)
        return n

    def max_seq_blocks(self, seqs) -> int:
        """Longest block table among seqs (one call)."""
        ids = np.ascontiguousarray(seqs, dtype=np.int64)
        n = int(_lib.pa_bm_max_seq_blocks(self._h, ids.ctypes.data_as(C.c_void_p) if len(ids) else None, len(ids)))
        if n < 0:
            raise KeyError("unknown sequence id")
        return n

    def block_table(self, seq: int) -> list:
        n = _lib.pa_bm_num_seq_blocks(self._h, int(seq))
        if n < 0:
            raise KeyError(seq)
        out = np.empty(max(n, 1), dtype=np.int32)
        self._st(_lib.pa_bm_block_table(self._h, int(seq), out.ctypes.data_as(C.c_void_p), n, None),
                 "block_table")
        return out[:n].tolist()

    def build_tables(self, seqs, max_blocks: int):
        ids = np.ascontiguousarray(seqs, dtype=np.int64)
        tables = np.empty((len(ids), int(max_blocks)), dtype=np.int32)
        lens = np.empty(len(ids), dtype=np.int32)
        self._st(_lib.pa_bm_build_tables(self._h, ids.ctypes.data_as(C.c_void_p), len(ids),
                                         int(max_blocks), tables.ctypes.data_as(C.c_void_p),
                                         lens.ctypes.data_as(C.c_void_p)), "build_tables")
        return tables, lens

    def refcount(self, block: int) -> int:
        return int(_lib.pa_bm_refcount(self._h, int(block)))

    def num_free(self) -> int:
        return int(_lib.pa_bm_num_free(self._h))

    def free_stack(self) -> list:
        n = _lib.pa_bm_free_stack(self._h, None, 0)
        out = np.empty(max(n, 1), dtype=np.int32)
        _lib.pa_bm_free_stack(self._h, out.ctypes.data_as(C.c_void_p), n)
        return out[:n].tolist()

    def tokens_stored(self) -> int:
        return int(_lib.pa_bm_tokens_stored(self._h))

    def add_seq_tokens(self, seq: int, tokens):
        """Create a sequence from its prompt token ids with automatic prefix caching.
        Returns (number of leading tokens whose K/V are already cached, int64 slots
        of the remaining tokens)."""
        toks = np.ascontiguousarray(tokens, dtype=np.int32)
        slots = np.empty(max(len(toks), 1), dtype=np.int64)
        ncached = C.c_int32(0)
        self._st(_lib.pa_bm_add_seq_tokens(self._h, int(seq), toks.ctypes.data_as(C.c_void_p), len(toks),
                                           slots.ctypes.data_as(C.c_void_p), C.byref(ncached)),
                 f"add_seq_tokens({seq}, {len(toks)})")
        return int(ncached.value), slots[:len(toks) - ncached.value].copy()

    def num_evictable(self) -> int:
        return int(_lib.pa_bm_num_evictable(self._h))

    def num_cached(self) -> int:
        return int(_lib.pa_bm_num_cached(self._h))

    def evictable(self) -> list:
        n = _lib.pa_bm_evictable(self._h, None, 0)
        out = np.empty(max(n, 1), dtype=np.int32)
        _lib.pa_bm_evictable(self._h, out.ctypes.data_as(C.c_void_p), n)
        return out[:n].tolist()
