"""Plain-Python model of the paged-KV block allocator -- TEST INFRASTRUCTURE ONLY.

This is the oracle for the host C++ ``BlockAllocator``/``BlockManager``: written
independently from the same specification, it must produce bit-identical block
tables, slot mappings and copy pairs on any trace.

Specification (page titles and sections; the readings chosen where the pages are
silent or buggy are marked READING):

* Pool and free list -- devpress.csdn.net/amd vLLM v0.6.x teardown, section
  "关键设计一：分页管理": ``free_blocks = list(range(num_blocks))``; ``allocate``
  pops from the END and fails with out-of-memory when the list is empty; ``free``
  appends.  So the free list is a LIFO stack.  READING: the initial order may be
  any permutation (configs use a seeded shuffle); ``pop()`` takes its last entry.
* Block table -- same section, and chenxutan "vLLM 深度拆解" 2.1: a sequence's
  logical block j is the physical block ``table[j]``; 16 tokens per block.
  Token position t of a sequence is at slot ``table[t // B] * B + t % B``.
* append_slot -- chenxutan 3.3 (write into the current block if it is not full,
  else take a new block from the pool).  READING: the page's code allocates on
  every call and returns the block id; here a block is allocated iff the token
  count is a multiple of B (empty table or last block full), and the returned
  value is the token's slot.
* fork -- devpress "关键设计二" (the child shares the parent's physical blocks).
  READING: the page's code does not raise reference counts; here every shared
  block's count is incremented, so a shared block is freed only by its last user.
* Copy-on-Write -- devpress "关键设计二": if the block about to be written is
  shared (count > 1), take a new block, copy the old one into it, drop one
  reference to the old one and put the new one in the table.  READING: this
  applies only when the token goes into an existing, partially filled block; a
  full last block is never copied (the token opens a fresh block instead).
  Siblings are appended one after another, so with n sharers the first n-1 copy
  and the last one writes in place.
* free -- chenxutan 3.3 (a finished request returns all its blocks).  READING:
  references are dropped in logical-block order and each block whose count
  reaches zero is pushed on the free stack at that moment.
* Out of memory leaves every structure unchanged (devpress "关键设计一" raises
  before touching the table).
* Automatic prefix caching -- chenxutan 5.2 (prompts sharing a prefix reuse its
  KV; automatic).  READING (the pages give no mechanism): a sequence created from
  its prompt's token ids (``add_seq_tokens``) reuses the longest run of leading
  full blocks whose exact key is known, key = (parent block, the parent's
  generation, the block's token ids), parent = the prompt's previous block (-1
  for the first), generation = how often the block has been allocated.  Its own
  full blocks are entered under their keys.  A keyed block reaching count zero
  becomes evictable instead of free (a freed sequence's such blocks from the last
  to the first); allocation uses the free stack first, then reclaims the
  earliest evictable block and forgets its key.  Appended blocks get no key.
"""
from __future__ import annotations

import numpy as np


class OutOfBlocks(RuntimeError):
    """The pool has fewer free blocks than the operation needs."""


class BlockManagerModel:
    def __init__(self, num_blocks: int, block_size: int = 16, free_order=None):
        self.num_blocks = int(num_blocks)
        self.block_size = int(block_size)
        if free_order is None:
            free_order = list(range(self.num_blocks))
        free_order = [int(b) for b in free_order]
        if sorted(free_order) != list(range(self.num_blocks)):
            raise ValueError("free_order must be a permutation of range(num_blocks)")
        self.free_stack = free_order            # allocate() = pop() from the end
        self.ref = [0] * self.num_blocks
        self.tables: dict[int, list[int]] = {}
        self.ntok: dict[int, int] = {}
        self.gen = [0] * self.num_blocks          # times each block was allocated
        self.key: dict[int, tuple] = {}            # keyed block -> its key
        self.index: dict[tuple, int] = {}          # key -> block
        self.evictable_list: list[int] = []        # front = next reclaimed

    # -- allocator -----------------------------------------------------------
    def _allocate(self) -> int:
        if self.free_stack:
            b = self.free_stack.pop()
        elif self.evictable_list:
            b = self.evictable_list.pop(0)
            del self.index[self.key.pop(b)]
        else:
            raise OutOfBlocks("no free blocks")
        self.ref[b] = 1
        self.gen[b] += 1
        return b

    def _drop(self, b: int) -> bool:
        """Drop a reference; True when a keyed block reached zero (the caller
        makes it evictable)."""
        self.ref[b] -= 1
        if self.ref[b] == 0:
            if b in self.key:
                return True
            self.free_stack.append(b)
        return False

    def _available(self) -> int:
        return len(self.free_stack) + len(self.evictable_list)

    def num_free(self) -> int:
        return len(self.free_stack)

    def refcount(self, b: int) -> int:
        return self.ref[b]

    # -- sequences -----------------------------------------------------------
    def add_seq(self, seq: int) -> None:
        if seq in self.tables:
            raise KeyError(f"sequence {seq} exists")
        self.tables[seq] = []
        self.ntok[seq] = 0

    def _blocks_needed(self, seq: int, n: int) -> int:
        B = self.block_size
        n0 = self.ntok[seq]
        fresh = -(-(n0 + n) // B) - (-(-n0 // B))
        cow = 1 if (n > 0 and n0 % B != 0 and self.ref[self.tables[seq][-1]] > 1) else 0
        return fresh + cow

    def append_slot(self, seq: int):
        """Append one token; return (slot, (src, dst) copy pair or None)."""
        slots, pairs = self.append_slots(seq, 1)
        return slots[0], (pairs[0] if pairs else None)

    def append_slots(self, seq: int, n: int):
        """Append n tokens; return (slots list, list of (src, dst) copy pairs)."""
        if seq not in self.tables:
            raise KeyError(f"no sequence {seq}")
        if self._blocks_needed(seq, n) > self._available():
            raise OutOfBlocks(f"sequence {seq} needs more blocks than are free")
        B = self.block_size
        table = self.tables[seq]
        slots, pairs = [], []
        for _ in range(n):
            k = self.ntok[seq]
            if k % B == 0:
                table.append(self._allocate())
            elif self.ref[table[-1]] > 1:
                old = table[-1]
                new = self._allocate()
                pairs.append((old, new))
                if self._drop(old):
                    self.evictable_list.append(old)
                table[-1] = new
            slots.append(table[-1] * B + k % B)
            self.ntok[seq] = k + 1
        return slots, pairs

    def fork(self, parent: int, child: int) -> None:
        if parent not in self.tables:
            raise KeyError(f"no sequence {parent}")
        if child in self.tables:
            raise KeyError(f"sequence {child} exists")
        self.tables[child] = list(self.tables[parent])
        self.ntok[child] = self.ntok[parent]
        for b in self.tables[child]:
            self.ref[b] += 1

    def free(self, seq: int) -> None:
        if seq not in self.tables:
            raise KeyError(f"no sequence {seq}")
        reached_zero = [b for b in self.tables.pop(seq) if self._drop(b)]
        self.evictable_list.extend(reversed(reached_zero))
        del self.ntok[seq]

    def add_seq_tokens(self, seq: int, tokens):
        """Create a sequence from its prompt token ids; return (tokens whose K/V are
        cached already, slots of the remaining tokens)."""
        if seq in self.tables:
            raise KeyError(f"sequence {seq} exists")
        B = self.block_size
        tokens = [int(t) for t in tokens]
        n = len(tokens)
        hits, parent, pgen = [], -1, 0
        for j in range(n // B):
            b = self.index.get((parent, pgen, tuple(tokens[j * B:(j + 1) * B])))
            if b is None:
                break
            hits.append(b)
            parent, pgen = b, self.gen[b]
        need = -(-n // B) - len(hits)
        if need > self._available() - sum(1 for b in hits if b in self.evictable_list):
            raise OutOfBlocks(f"sequence {seq} needs more blocks than are free")
        for b in hits:
            if b in self.evictable_list:
                self.evictable_list.remove(b)
            self.ref[b] += 1
        table = list(hits)
        slots = []
        for i in range(len(hits) * B, n):
            off = i % B
            if off == 0:
                table.append(self._allocate())
            slots.append(table[-1] * B + off)
            if off == B - 1:
                j = i // B
                par = table[j - 1] if j > 0 else -1
                k = (par, self.gen[par] if par >= 0 else 0, tuple(tokens[j * B:(j + 1) * B]))
                self.index[k] = table[j]
                self.key[table[j]] = k
        self.tables[seq] = table
        self.ntok[seq] = n
        return len(hits) * B, slots

    def num_evictable(self) -> int:
        return len(self.evictable_list)

    def num_cached(self) -> int:
        return len(self.index)

    def evictable(self) -> list[int]:
        return list(self.evictable_list)

    def block_table(self, seq: int) -> list[int]:
        return list(self.tables[seq])

    def num_tokens(self, seq: int) -> int:
        return self.ntok[seq]

    def build_tables(self, seqs, max_blocks: int):
        """int32 [len(seqs), max_blocks] tables padded with -1, and int32 lengths."""
        out = np.full((len(seqs), max_blocks), -1, dtype=np.int32)
        lens = np.zeros(len(seqs), dtype=np.int32)
        for i, s in enumerate(seqs):
            t = self.tables[s]
            if len(t) > max_blocks:
                raise ValueError(f"sequence {s} has {len(t)} blocks > max_blocks {max_blocks}")
            out[i, :len(t)] = t
            lens[i] = self.ntok[s]
        return out, lens

    # -- statistics (devpress "先理解问题" and "关键设计一") -------------------
    def tokens_stored(self) -> int:
        return sum(self.ntok.values())

    def blocks_in_use(self) -> int:
        return self.num_blocks - len(self.free_stack)
