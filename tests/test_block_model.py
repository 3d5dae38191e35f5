"""Pins of the Python block-allocator model (the oracle for the host C++ manager).

Pinned to the pages' worked examples (tests/golden/, each with its citation) and to
invariants any correct allocator keeps: LIFO free list, OOM leaves state untouched,
sum of reference counts = sum of table lengths, free + used = pool size, internal
fragmentation below one block, Copy-on-Write only on a shared partly filled block.
"""
import json
import os

import numpy as np
import pytest
from hypothesis import given, settings, strategies as st

from oracle.block_model import BlockManagerModel, OutOfBlocks

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def check_invariants(m: BlockManagerModel):
    refs = sum(m.ref)
    assert refs == sum(len(t) for t in m.tables.values())
    used = sum(1 for r in m.ref if r > 0)
    assert used + m.num_free() == m.num_blocks
    assert len(set(m.free_stack)) == m.num_free()
    assert all(m.ref[b] == 0 for b in m.free_stack)
    for s, t in m.tables.items():
        n = m.num_tokens(s)
        assert len(t) == -(-n // m.block_size)           # exactly the blocks the tokens need
        assert len(t) * m.block_size - n <= m.block_size - 1


def test_page_pool_picture():
    """Alternating appends of whole blocks reproduce the page's pool picture
    A=[0,2,5,8], B=[1,4,9] when pop() yields 0,1,2,... (free list reversed)."""
    g = json.load(open(os.path.join(GOLDEN, "p3_block_table_picture.json")))
    pool = g["pool"]
    m = BlockManagerModel(len(pool), g["block_size"], list(range(len(pool)))[::-1])
    ids = {"A": 0, "B": 1, "-": 2}
    for s in ids.values():
        m.add_seq(s)
    for owner in pool:
        m.append_slots(ids[owner[0]], g["block_size"])
    m.free(ids["-"])
    assert m.block_table(0) == g["tables"]["A"]
    assert m.block_table(1) == g["tables"]["B"]
    assert sorted(m.free_stack) == g["free_after"]
    check_invariants(m)


def test_page_utilisation_example():
    """The page's contiguous pre-allocation example uses ~64% of what it reserves;
    paging the same three requests wastes at most 15 tokens each."""
    g = json.load(open(os.path.join(GOLDEN, "p3_contiguous_utilisation.json")))
    ctx, res = g["context_tokens"], g["reserved_tokens"]
    assert abs(sum(ctx) / sum(res) - g["contiguous_utilisation_printed"]) < g["printed_precision"]
    m = BlockManagerModel(2000, g["block_size"])
    for s, L in enumerate(ctx):
        m.add_seq(s)
        m.append_slots(s, L)
    assert m.tokens_stored() == sum(ctx)
    assert m.blocks_in_use() == sum(-(-L // 16) for L in ctx) == 657
    for s, L in enumerate(ctx):
        assert len(m.block_table(s)) * 16 - L <= 15
    assert m.tokens_stored() / (m.blocks_in_use() * 16) > 0.99


def test_lifo_free_list_and_slots():
    m = BlockManagerModel(8, 16, [5, 3, 7, 1, 0, 2, 6, 4])
    m.add_seq(0)
    slots, pairs = m.append_slots(0, 40)
    assert pairs == []
    assert m.block_table(0) == [4, 6, 2]                  # popped from the end
    assert slots[:3] == [64, 65, 66] and slots[16] == 96 and slots[39] == 2 * 16 + 7
    m.free(0)
    assert m.free_stack[-3:] == [4, 6, 2]                  # pushed in logical order
    m.add_seq(1)
    m.append_slots(1, 1)
    assert m.block_table(1) == [2]                        # last freed, first reused


def test_out_of_blocks_leaves_state_unchanged():
    m = BlockManagerModel(3, 16)
    m.add_seq(0)
    m.append_slots(0, 20)
    before = (list(m.free_stack), list(m.ref), m.block_table(0), m.num_tokens(0))
    with pytest.raises(OutOfBlocks):
        m.append_slots(0, 40)                             # needs 2 more, 1 free
    assert (list(m.free_stack), list(m.ref), m.block_table(0), m.num_tokens(0)) == before
    m.fork(0, 1)
    m.append_slots(0, 1)                                   # CoW takes the last free block
    with pytest.raises(OutOfBlocks):
        m.append_slots(1, 13)                              # crosses into a third block; none free
    check_invariants(m)


def test_copy_on_write_siblings():
    """n children share a partly filled last block: the first n-1 copy, the last writes in place."""
    m = BlockManagerModel(20, 16)
    m.add_seq(9)
    m.append_slots(9, 21)                                  # blocks [19, 18], last has 5 tokens
    for c in range(4):
        m.fork(9, c)
    m.free(9)
    assert m.refcount(18) == 4 and m.refcount(19) == 4
    got = [m.append_slot(c) for c in range(4)]
    assert [p is not None for _, p in got] == [True, True, True, False]
    assert [p[0] for _, p in got[:3]] == [18, 18, 18]
    assert got[3][0] == 18 * 16 + 5                        # last child writes into the old block
    for c in range(3):
        new = got[c][1][1]
        assert got[c][0] == new * 16 + 5 and m.block_table(c) == [19, new]
    assert m.refcount(18) == 1 and m.refcount(19) == 4
    check_invariants(m)


def test_full_shared_block_is_not_copied():
    m = BlockManagerModel(10, 16)
    m.add_seq(0)
    m.append_slots(0, 32)
    m.fork(0, 1)
    slot, pair = m.append_slot(1)
    assert pair is None and len(m.block_table(1)) == 3 and m.block_table(1)[:2] == m.block_table(0)
    assert slot == m.block_table(1)[2] * 16


def test_build_tables_pads_with_minus_one():
    m = BlockManagerModel(10, 16)
    m.add_seq(3)
    m.add_seq(4)
    m.append_slots(3, 17)
    t, lens = m.build_tables([4, 3], 4)
    assert t.dtype == np.int32 and t.tolist()[0] == [-1] * 4 and t.tolist()[1][2:] == [-1, -1]
    assert lens.tolist() == [0, 17]


ops = st.lists(st.tuples(st.sampled_from(["add", "append", "fork", "free"]),
                         st.integers(0, 5), st.integers(0, 5), st.integers(1, 40)), max_size=60)


@settings(max_examples=150, deadline=None)
@given(ops)
def test_random_traces_keep_invariants(trace):
    m = BlockManagerModel(24, 16)
    for kind, a, b, n in trace:
        try:
            if kind == "add":
                m.add_seq(a)
            elif kind == "append":
                m.append_slots(a, n)
            elif kind == "fork":
                m.fork(a, b)
            else:
                m.free(a)
        except (KeyError, OutOfBlocks):
            pass
        check_invariants(m)
