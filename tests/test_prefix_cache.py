"""Automatic prefix caching in the host block manager (C++) against the Python
model, and worked scenarios: a shared system prompt, reuse after free, eviction
under memory pressure (tail of a prefix first), out of memory changing nothing.

Page: chenxutan "vLLM 深度拆解" 5.2 (requests with the same system prompt reuse the
prefix's KV automatically).  The mechanism is the reading stated in
include/pa_block_manager.h and oracle/block_model.py.
"""
import numpy as np
import pytest

from oracle.block_model import BlockManagerModel, OutOfBlocks


@pytest.fixture
def both(pa):
    def make(num_blocks, free_order=None):
        return pa.BlockManager(num_blocks, 16, free_order), BlockManagerModel(num_blocks, 16, free_order)
    return make


def same_state(c, m, seqs):
    assert c.free_stack() == m.free_stack
    assert c.evictable() == m.evictable()
    assert c.num_cached() == m.num_cached()
    for b in range(m.num_blocks):
        assert c.refcount(b) == m.refcount(b)
    for s in seqs:
        assert c.block_table(s) == m.block_table(s)
        assert c.num_tokens(s) == m.num_tokens(s)


def test_shared_system_prompt_reuses_full_blocks(both):
    c, m = both(32)
    system = list(range(1000, 1032))                       # a 32-token system prompt
    a = system + [1, 2, 3, 4, 5, 6, 7, 8]                  # 40 tokens
    b = system + list(range(50, 70))                       # 52 tokens
    for mgr in (c, m):
        na, sa = mgr.add_seq_tokens(0, a)
        nb, sb = mgr.add_seq_tokens(1, b)
        assert (na, len(sa)) == (0, 40)
        assert (nb, len(sb)) == (32, 20)                   # both system-prompt blocks hit
    ta, tb = m.block_table(0), m.block_table(1)
    assert ta[:2] == tb[:2] and ta[2] != tb[2]
    assert m.refcount(ta[0]) == m.refcount(ta[1]) == 2
    assert m.num_cached() == 3                             # a's two full blocks, b's third
    same_state(c, m, [0, 1])
    # a fresh manager has nothing cached: every token needs a slot
    _, sb = BlockManagerModel(32, 16).add_seq_tokens(9, b)
    assert len(sb) == 52


def test_freed_prefix_stays_cached_until_reclaimed(both):
    c, m = both(8)
    p = list(range(48))                                    # three full blocks
    for mgr in (c, m):
        mgr.add_seq_tokens(0, p + [7])                     # plus one token in a fourth block
        mgr.free(0)
    assert m.num_evictable() == 3 and m.num_free() == 5   # the partial block is simply free
    tab = m.evictable()
    for mgr in (c, m):
        n, slots = mgr.add_seq_tokens(1, p[:40])           # same first 40 tokens
        assert (n, len(slots)) == (32, 8)                  # blocks 0 and 1 revived, block 2 not
    assert m.block_table(1)[:2] == list(reversed(tab))[:2]
    same_state(c, m, [1])


def test_eviction_takes_the_tail_of_a_prefix_first(both):
    c, m = both(4)
    p = list(range(64))                                    # four full blocks
    for mgr in (c, m):
        mgr.add_seq_tokens(0, p)
        mgr.free(0)
    blocks = m.evictable()
    assert len(blocks) == 4
    for mgr in (c, m):
        mgr.add_seq_tokens(1, [9] * 16)                    # one fresh block: reclaims the tail
    assert m.num_cached() == 4                             # 3 of p's blocks + the new one
    for mgr in (c, m):
        n, _ = mgr.add_seq_tokens(2, p[:48])
        assert n == 48                                     # the head of p is still there
    same_state(c, m, [1, 2])


def test_out_of_blocks_changes_nothing(both):
    c, m = both(3)
    for mgr in (c, m):
        mgr.add_seq_tokens(0, list(range(32)))
    before = (m.free_stack[:], m.evictable(), m.num_cached())
    with pytest.raises(OutOfBlocks):
        m.add_seq_tokens(1, list(range(100, 140)))         # needs 3 blocks, 1 left
    with pytest.raises(Exception):
        c.add_seq_tokens(1, list(range(100, 140)))
    assert (m.free_stack, m.evictable(), m.num_cached()) == before
    same_state(c, m, [0])
    # a hit on evictable blocks is not counted as allocatable
    for mgr in (c, m):
        mgr.free(0)
    for mgr in (c, m):
        n, _ = mgr.add_seq_tokens(2, list(range(32)) + list(range(500, 516)))
        assert n == 32
    same_state(c, m, [2])


def test_plain_sequences_are_never_cached(both):
    c, m = both(8)
    for mgr in (c, m):
        mgr.add_seq(0)
        mgr.append_slots(0, 40)
        mgr.free(0)
    assert m.num_cached() == 0 and m.num_evictable() == 0 and m.num_free() == 8
    same_state(c, m, [])


@pytest.mark.parametrize("seed", range(6))
def test_random_traces_match_the_model(both, seed):
    rng = np.random.default_rng(seed)
    free_order = rng.permutation(48).tolist()
    c, m = both(48, free_order)
    prefixes = [rng.integers(0, 50, size=int(n)).tolist() for n in (16, 32, 40, 64)]
    live, next_id = [], 0
    for _ in range(300):
        op = rng.integers(0, 5)
        if op <= 1 or not live:                            # new prompt sharing some prefix
            base = prefixes[rng.integers(0, len(prefixes))]
            cut = int(rng.integers(0, len(base) + 1))
            toks = base[:cut] + rng.integers(0, 50, size=int(rng.integers(0, 40))).tolist()
            res = []
            for mgr in (c, m):
                try:
                    res.append(mgr.add_seq_tokens(next_id, toks))
                except Exception as e:                     # both must run out together
                    res.append(type(e).__name__)
            if isinstance(res[1], str):
                assert isinstance(res[0], str)
            else:
                assert res[0][0] == res[1][0] and res[0][1].tolist() == list(res[1][1])
                live.append(next_id)
            next_id += 1
        elif op == 2:                                      # append a few tokens
            s = live[rng.integers(0, len(live))]
            n = int(rng.integers(1, 20))
            res = []
            for mgr in (c, m):
                try:
                    sl, pr = mgr.append_slots(s, n)
                    res.append((list(sl), [tuple(p) for p in pr]))
                except Exception as e:
                    res.append(type(e).__name__)
            assert isinstance(res[0], str) == isinstance(res[1], str)
            if not isinstance(res[1], str):
                assert res[0] == res[1]
        elif op == 3:                                      # fork
            s = live[rng.integers(0, len(live))]
            for mgr in (c, m):
                mgr.fork(s, next_id)
            live.append(next_id)
            next_id += 1
        else:                                              # free
            s = live.pop(int(rng.integers(0, len(live))))
            for mgr in (c, m):
                mgr.free(s)
        same_state(c, m, live)
