"""PagedKVCache: one layer's K/V pool on the GPU plus the host block manager.

Orchestration only: the host C++ BlockManager decides slots, tables and copy
pairs; pa_copy_blocks / pa_cache_write / pa_decode / pa_prefill_chunk do all the
device work.  Order within a step follows the pages' data flow (a new token is
written back into the cache, then attended to): copy-on-write copies, then the
cache write, then attention, all on one stream.
"""
from __future__ import annotations

import math

import numpy as np

from . import (BlockManager, pa_cache_write, pa_copy_blocks, pa_decode, pa_decode_workspace_size,
               pa_prefill_chunk, BLOCK_SIZE)


def _torch():
    import torch
    return torch


class PagedKVCache:
    def __init__(self, num_blocks: int, num_kv_heads: int, head_dim: int, dtype, device="cuda",
                 free_order=None, fill_nan: bool = True, k_scale: float = 1.0, v_scale: float = 1.0):
        """dtype torch.float32, torch.bfloat16 or torch.float8_e4m3fn; an fp8 pool stores
        e4m3(x / k_scale) and e4m3(x / v_scale) and takes bf16 queries and K/V."""
        torch = _torch()
        self.num_blocks, self.num_kv_heads, self.head_dim = num_blocks, num_kv_heads, head_dim
        self.dtype, self.device = dtype, torch.device(device)
        self.k_scale, self.v_scale = float(k_scale), float(v_scale)
        shape = (num_blocks, num_kv_heads, BLOCK_SIZE, head_dim)
        # NaN in every slot nothing has written: a stray read poisons the output
        if dtype == torch.float8_e4m3fn:
            code = 0x7F if fill_nan else 0x00          # e4m3 NaN / +0
            self.key_cache = torch.full(shape, code, dtype=torch.uint8, device=self.device).view(dtype)
            self.value_cache = torch.full(shape, code, dtype=torch.uint8, device=self.device).view(dtype)
        else:
            fill = float("nan") if fill_nan else 0.0
            self.key_cache = torch.full(shape, fill, dtype=dtype, device=self.device)
            self.value_cache = torch.full(shape, fill, dtype=dtype, device=self.device)
        self.manager = BlockManager(num_blocks, BLOCK_SIZE, free_order)
        self.err_flag = torch.zeros(1, dtype=torch.int32, device=self.device)

    # -- allocator passthroughs ------------------------------------------------
    def add_seq(self, seq):
        self.manager.add_seq(seq)

    def fork(self, parent, child):
        self.manager.fork(parent, child)

    def free(self, seq):
        self.manager.free(seq)

    # -- step pieces -----------------------------------------------------------
    def plan_append(self, seqs, counts=None):
        """Allocate slots for ``counts[i]`` new tokens of each seq (default 1), all or
        nothing, in one call to the host manager.  Returns (int64 slots [sum counts],
        int32 copy pairs [P, 2]) as numpy arrays."""
        return self.manager.append_step(seqs, counts)

    def write(self, k, v, slots, pairs=None, stream=None):
        """Copy-on-write copies (if any), then scatter k/v [T, Hkv, d] into ``slots``."""
        torch = _torch()
        if pairs is not None and len(pairs):
            pa_copy_blocks(self.key_cache, self.value_cache, torch.as_tensor(pairs, device=self.device),
                           self.err_flag, stream)
        if len(slots):
            pa_cache_write(k, v, torch.as_tensor(slots, device=self.device), self.key_cache,
                           self.value_cache, self.err_flag, stream, self.k_scale, self.v_scale)

    def append(self, seqs, k, v, counts=None, stream=None):
        slots, pairs = self.plan_append(seqs, counts)
        self.write(k, v, slots, pairs, stream)
        return slots, pairs

    def tables(self, seqs, max_blocks=None):
        """int32 block tables [S, max_blocks] (padded with -1) and lengths, on the device."""
        torch = _torch()
        if max_blocks is None:
            max_blocks = max(1, self.manager.max_seq_blocks(seqs))
        t, lens = self.manager.build_tables(seqs, max_blocks)
        return torch.from_numpy(t).to(self.device), torch.from_numpy(lens).to(self.device), int(lens.max(initial=0))

    def decode(self, q, seqs, scale, out=None, partition_size=0, max_blocks=None, stream=None,
               workspace=None):
        torch = _torch()
        tables, lens, max_len = self.tables(seqs, max_blocks)
        max_len = max(max_len, 1)
        out = torch.empty_like(q) if out is None else out
        if partition_size and workspace is None:
            ws = pa_decode_workspace_size(len(seqs), q.shape[1], q.shape[2], max_len, partition_size)
            workspace = torch.empty(max(ws, 16), dtype=torch.uint8, device=self.device)
        pa_decode(q, self.key_cache, self.value_cache, tables, lens, max_len, scale, out,
                  partition_size, workspace, self.err_flag, stream, self.k_scale, self.v_scale)
        return out

    def prefill(self, q, seqs, chunk_lens, scale, out=None, max_blocks=None, stream=None):
        torch = _torch()
        tables, lens, _ = self.tables(seqs, max_blocks)
        out = torch.empty_like(q) if out is None else out
        ch = torch.as_tensor(np.asarray(chunk_lens, np.int32), device=self.device)
        pa_prefill_chunk(q, self.key_cache, self.value_cache, tables, lens, ch, scale, out,
                         self.err_flag, stream)
        return out


def default_scale(head_dim: int) -> float:
    return 1.0 / math.sqrt(head_dim)
