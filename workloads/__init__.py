"""Seeded synthetic workloads for paged-KV-cache attention.

This module is shared by the tests, the benchmark and the smoke check.  It holds
no attention, allocation or copy arithmetic: it only draws lengths, free-list
orders and N(0,1) data, and describes each workload as a list of allocator
operations ("add", "append", "fork", "free") plus decode / prefill steps.  The
CUDA path and the CPU oracle each replay that description with their own block
manager and their own cache-write; tests check that both replays agree.

Workloads (shapes of the pages' serving scenarios; every draw comes from
``numpy.random.Generator(PCG64(1000 + config_id))`` in a fixed order):

1. tiny fp32: 4 sequences of 17/33/64/100 tokens, pool of 64 blocks in a seeded
   random free order, 4 query = 4 kv heads, head_dim 64, scale 1/8; one step
   appends one token to each sequence and decodes.
2. Llama-7B-shaped MHA, bf16: 64 sequences, lengths uniform in [128, 2048],
   32/32 heads, head_dim 128, pool = ceil(1.25 x blocks needed), shuffled.
3. Llama-3-8B-shaped GQA with prefix sharing, bf16: 16 groups of 16 sequences;
   each group forks one 512-token prefix (32 shared blocks, 16 references) and
   then appends a private suffix of round(600 * exp(N(0,1))) tokens clamped to
   [1, 8192]; 32 query / 8 kv heads.
4. parallel sampling: 128 parents of lengths uniform in [200, 3000] (redrawn
   until not a multiple of 16, so the last block is partly filled), each forked
   into 4 children, parent freed; 16 steps in which every child appends a token
   (step 1 copies the shared last block for 3 of the 4 children).
5. long context: 8 sequences of 32768 tokens, 64 query / 8 kv heads, pool of
   exactly 16384 blocks in shuffled order; one decode step over the whole
   context and one 512-row causal prefill chunk (the last 512 positions).

``mini=True`` keeps each workload's structure at a size the oracle finishes in
seconds (still several blocks, partitions and ragged tails).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

BLOCK_SIZE = 16


def rng_for(config_id: int, seed_offset: int = 0) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(1000 + int(config_id) + int(seed_offset)))


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bf16 (ties to even); return the uint16 bit patterns."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    rounded = u + (np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1)))
    return (rounded >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32)


def normal(rng: np.random.Generator, shape, dtype: str) -> np.ndarray:
    """N(0,1) data: float32, or bf16 bit patterns (uint16) for dtype 'bf16'."""
    x = rng.standard_normal(size=shape, dtype=np.float32)
    return x if dtype == "f32" else to_bf16_bits(x)


@dataclass
class Step:
    """One decode step: every sequence in ``seqs`` appends one token, then decodes."""
    seqs: list
    k_new: np.ndarray   # [S, Hkv, d]
    v_new: np.ndarray   # [S, Hkv, d]
    q: np.ndarray       # [S, Hq, d]


@dataclass
class PrefillChunk:
    """Causal query chunk: the last ``chunk`` positions of each sequence in ``seqs``."""
    seqs: list
    chunk: int
    q: np.ndarray       # [S, chunk, Hq, d]


@dataclass
class Workload:
    config_id: int
    name: str
    dtype: str                      # "f32" or "bf16"
    num_blocks: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    scale: float
    free_order: np.ndarray          # permutation of range(num_blocks); pop() takes the last
    ops: list = field(default_factory=list)
    steps: list = field(default_factory=list)
    prefill: PrefillChunk | None = None
    block_size: int = BLOCK_SIZE

    @property
    def elem_bytes(self) -> int:
        return 4 if self.dtype == "f32" else 2

    @property
    def np_dtype(self):
        return np.float32 if self.dtype == "f32" else np.uint16

    def cache_shape(self):
        return (self.num_blocks, self.num_kv_heads, self.block_size, self.head_dim)

    def max_context(self) -> int:
        """Longest context reached by any sequence over the whole workload."""
        n, best = {}, 0
        for op in self.ops:
            if op[0] == "add":
                n[op[1]] = 0
            elif op[0] == "append":
                n[op[1]] += op[2].shape[0]
            elif op[0] == "fork":
                n[op[2]] = n[op[1]]
            elif op[0] == "free":
                del n[op[1]]
        best = max(n.values(), default=0)
        return best + sum(1 for st in self.steps if st.k_new is not None)


def replay(wl: Workload, manager, write):
    """Run the workload's allocator operations.

    ``manager`` needs add_seq / append_slots / fork / free (the C++ manager or the
    Python model); ``write(k, v, slots)`` stores appended K/V at the returned
    slots.  Allocation never needs a block copy during set-up.
    """
    for op in wl.ops:
        kind = op[0]
        if kind == "add":
            manager.add_seq(op[1])
        elif kind == "append":
            _, seq, k, v = op
            slots, pairs = manager.append_slots(seq, k.shape[0])
            assert not pairs, "set-up appends never share a partly filled block"
            write(k, v, np.asarray(slots, dtype=np.int64))
        elif kind == "fork":
            manager.fork(op[1], op[2])
        elif kind == "free":
            manager.free(op[1])
        else:
            raise ValueError(kind)


def _pool_free_order(rng, num_blocks):
    return rng.permutation(num_blocks).astype(np.int32)


def _blocks(n):
    return -(-n // BLOCK_SIZE)


def make(config_id: int, mini: bool = False) -> Workload:
    """Build workload ``config_id`` (1..5); ``mini`` shrinks it for fast oracle runs."""
    rng = rng_for(config_id, 100 if mini else 0)
    if config_id == 1:
        return _config1(rng)
    if config_id == 2:
        return _config2(rng, mini)
    if config_id == 3:
        return _config3(rng, mini)
    if config_id == 4:
        return _config4(rng, mini)
    if config_id == 5:
        return _config5(rng, mini)
    raise ValueError(f"unknown workload {config_id}")


def _decode_step(rng, seqs, hkv, hq, d, dtype):
    S = len(seqs)
    k = normal(rng, (S, hkv, d), dtype)
    v = normal(rng, (S, hkv, d), dtype)
    q = normal(rng, (S, hq, d), dtype)
    return Step(list(seqs), k, v, q)


def _config1(rng):
    lens = [17, 33, 64, 100]
    hq = hkv = 4
    d = 64
    nb = 64
    wl = Workload(1, "tiny-fp32", "f32", nb, hq, hkv, d, 1.0 / 8.0, _pool_free_order(rng, nb))
    for s, L in enumerate(lens):
        wl.ops.append(("add", s))
        wl.ops.append(("append", s, normal(rng, (L, hkv, d), "f32"), normal(rng, (L, hkv, d), "f32")))
    wl.steps.append(_decode_step(rng, range(len(lens)), hkv, hq, d, "f32"))
    return wl


def _config2(rng, mini):
    S, hq, hkv, d = (64, 32, 32, 128) if not mini else (12, 4, 4, 128)
    lo, hi = (128, 2048) if not mini else (20, 300)
    lens = rng.integers(lo, hi, size=S, endpoint=True)
    nb = math.ceil(1.25 * sum(_blocks(int(L) + 1) for L in lens))
    wl = Workload(2, "mha-7b" + ("-mini" if mini else ""), "bf16", nb, hq, hkv, d,
                  1.0 / math.sqrt(d), _pool_free_order(rng, nb))
    for s, L in enumerate(lens):
        L = int(L)
        wl.ops.append(("add", s))
        wl.ops.append(("append", s, normal(rng, (L, hkv, d), "bf16"), normal(rng, (L, hkv, d), "bf16")))
    wl.steps.append(_decode_step(rng, range(S), hkv, hq, d, "bf16"))
    return wl


def _config3(rng, mini):
    groups, per, prefix = (16, 16, 512) if not mini else (3, 4, 64)
    hq, hkv, d = 32, 8, 128
    median, cap = (600, 8192) if not mini else (60, 400)
    S = groups * per
    suffix = np.clip(np.rint(median * np.exp(rng.standard_normal(S))), 1, cap).astype(np.int64)
    need = groups * _blocks(prefix) + sum(_blocks(prefix + int(x) + 1) - _blocks(prefix) for x in suffix)
    nb = math.ceil(1.25 * need)
    wl = Workload(3, "gqa-8b-prefix" + ("-mini" if mini else ""), "bf16", nb, hq, hkv, d,
                  1.0 / math.sqrt(d), _pool_free_order(rng, nb))
    for g in range(groups):
        parent = S + g  # parent ids follow the children's
        wl.ops.append(("add", parent))
        wl.ops.append(("append", parent, normal(rng, (prefix, hkv, d), "bf16"),
                       normal(rng, (prefix, hkv, d), "bf16")))
        for c in range(per):
            wl.ops.append(("fork", parent, g * per + c))
        wl.ops.append(("free", parent))
        for c in range(per):
            s = g * per + c
            n = int(suffix[s])
            wl.ops.append(("append", s, normal(rng, (n, hkv, d), "bf16"), normal(rng, (n, hkv, d), "bf16")))
    wl.steps.append(_decode_step(rng, range(S), hkv, hq, d, "bf16"))
    return wl


def _config4(rng, mini):
    P, n_child, nsteps = (128, 4, 16) if not mini else (6, 4, 4)
    lo, hi = (200, 3000) if not mini else (20, 200)
    hq, hkv, d = 32, 8, 128
    lens = []
    while len(lens) < P:
        L = int(rng.integers(lo, hi, endpoint=True))
        if L % BLOCK_SIZE != 0:
            lens.append(L)
    need = sum(_blocks(L) for L in lens) + P * n_child * (1 + _blocks(nsteps))
    nb = math.ceil(1.25 * need)
    wl = Workload(4, "fork-cow" + ("-mini" if mini else ""), "bf16", nb, hq, hkv, d,
                  1.0 / math.sqrt(d), _pool_free_order(rng, nb))
    S = P * n_child
    for p, L in enumerate(lens):
        parent = S + p
        wl.ops.append(("add", parent))
        wl.ops.append(("append", parent, normal(rng, (L, hkv, d), "bf16"), normal(rng, (L, hkv, d), "bf16")))
        for c in range(n_child):
            wl.ops.append(("fork", parent, p * n_child + c))
        wl.ops.append(("free", parent))
    for _ in range(nsteps):
        wl.steps.append(_decode_step(rng, range(S), hkv, hq, d, "bf16"))
    return wl


def _config5(rng, mini):
    S, L, chunk = (8, 32768, 512) if not mini else (2, 1500, 200)
    hq, hkv, d = 64, 8, 128
    nb = S * _blocks(L) if not mini else S * _blocks(L) + 7
    wl = Workload(5, "long-context" + ("-mini" if mini else ""), "bf16", nb, hq, hkv, d,
                  1.0 / math.sqrt(d), _pool_free_order(rng, nb))
    for s in range(S):
        wl.ops.append(("add", s))
        wl.ops.append(("append", s, normal(rng, (L, hkv, d), "bf16"), normal(rng, (L, hkv, d), "bf16")))
    # decode over the whole context: the query token's own K/V is already cached
    q = normal(rng, (S, hq, d), "bf16")
    wl.steps.append(Step(list(range(S)), None, None, q))
    wl.prefill = PrefillChunk(list(range(S)), chunk, normal(rng, (S, chunk, hq, d), "bf16"))
    return wl
