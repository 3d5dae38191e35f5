"""pa_bm_append_step (one C call per step) against the Python model's sequential
appends: the same slots, copy pairs and state when the step fits, nothing changed
when it does not (out of blocks, unknown or repeated id, too little pair room).

Page: devpress vLLM v0.6.x teardown, 关键设计二 (forked siblings share blocks; the
block to be written is copied when shared) -- the copy-on-write order within a
step is the reading stated in include/pa_block_manager.h.
"""
import copy

import numpy as np
import pytest

from oracle.block_model import BlockManagerModel, OutOfBlocks


def state(mgr, seqs, num_blocks):
    return (list(mgr.free_stack() if callable(getattr(mgr, "free_stack", None)) else mgr.free_stack),
            [mgr.refcount(b) for b in range(num_blocks)],
            [list(mgr.block_table(s)) for s in seqs], [mgr.num_tokens(s) for s in seqs])


def test_forked_siblings_copy_in_order(pa):
    """A parent with a partly filled last block forks 4 children and is freed: in one
    step the first three children copy the shared block and the last writes in place."""
    c, m = pa.BlockManager(64, 16), BlockManagerModel(64, 16)
    for mgr in (c, m):
        mgr.add_seq(0)
        mgr.append_slots(0, 37)
        for ch in (1, 2, 3, 4):
            mgr.fork(0, ch)
        mgr.free(0)
    slots, pairs = c.append_step([1, 2, 3, 4])
    want_slots, want_pairs = [], []
    for ch in (1, 2, 3, 4):
        sl, pr = m.append_slots(ch, 1)
        want_slots.extend(int(x) for x in sl)
        want_pairs.extend(pr)
    assert slots.tolist() == want_slots
    assert [tuple(p) for p in pairs.tolist()] == want_pairs
    assert len(want_pairs) == 3
    assert state(c, [1, 2, 3, 4], 64) == state(m, [1, 2, 3, 4], 64)


def test_counts_and_empty_step(pa):
    c, m = pa.BlockManager(64, 16), BlockManagerModel(64, 16)
    for mgr in (c, m):
        for s in (5, 6, 7):
            mgr.add_seq(s)
        mgr.append_slots(6, 15)
    slots, pairs = c.append_step([5, 6, 7], [0, 3, 17])
    want = []
    for s, n in ((5, 0), (6, 3), (7, 17)):
        want.extend(int(x) for x in m.append_slots(s, n)[0])
    assert slots.tolist() == want and len(pairs) == 0
    s0, p0 = c.append_step([])
    assert len(s0) == 0 and len(p0) == 0
    assert state(c, [5, 6, 7], 64) == state(m, [5, 6, 7], 64)


def test_invalid_steps_change_nothing(pa):
    c = pa.BlockManager(8, 16)
    for s in (1, 2):
        c.add_seq(s)
        c.append_slots(s, 20)                     # 2 blocks each: 4 left
    before = state(c, [1, 2], 8)
    with pytest.raises(pa.PAError) as e:
        c.append_step([1, 1])                     # repeated id
    assert e.value.status == pa.PA_ERR_INVALID_ARG
    with pytest.raises(KeyError):
        c.append_step([1, 99])                    # unknown id (PA_ERR_NOT_FOUND)
    with pytest.raises(pa.OutOfBlocks):
        c.append_step([1, 2], [60, 60])           # needs 3 + 3 blocks, 4 free: all or nothing
    with pytest.raises(pa.PAError) as e:
        c.append_step([1, 2], [1, -1])
    assert e.value.status == pa.PA_ERR_INVALID_ARG
    assert state(c, [1, 2], 8) == before
    # pair room: a raw call with no room for the one copy this step needs
    import ctypes as C
    c.fork(1, 3)
    ids = np.array([3], np.int64)
    pairs = np.zeros(2, np.int32)
    st = pa._lib.pa_bm_append_step(c._h, ids.ctypes.data_as(C.c_void_p), None, 1, None,
                                   pairs.ctypes.data_as(C.c_void_p), 0, None)
    assert st == pa.PA_ERR_INVALID_ARG
    assert c.num_tokens(3) == 20


@pytest.mark.parametrize("seed", range(6))
def test_random_steps_match_sequential_model(pa, seed):
    rng = np.random.default_rng(100 + seed)
    nb = 48
    order = rng.permutation(nb).tolist()
    c, m = pa.BlockManager(nb, 16, order), BlockManagerModel(nb, 16, order)
    live, nxt = [], 0
    for _ in range(250):
        op = rng.integers(0, 6)
        if op == 0 or not live:
            for mgr in (c, m):
                mgr.add_seq(nxt)
            live.append(nxt)
            nxt += 1
        elif op == 1:
            p = live[rng.integers(0, len(live))]
            for mgr in (c, m):
                mgr.fork(p, nxt)
            live.append(nxt)
            nxt += 1
        elif op == 2 and len(live) > 1:
            s = live.pop(int(rng.integers(0, len(live))))
            for mgr in (c, m):
                mgr.free(s)
        else:                                     # a step over a random subset
            k = int(rng.integers(1, len(live) + 1))
            seqs = [int(x) for x in rng.choice(live, size=k, replace=False)]
            counts = rng.integers(0, 4, size=k).tolist()
            trial = copy.deepcopy(m)
            want_slots, want_pairs, failed = [], [], False
            try:
                for s, n in zip(seqs, counts):
                    sl, pr = trial.append_slots(s, n)
                    want_slots.extend(int(x) for x in sl)
                    want_pairs.extend(pr)
            except OutOfBlocks:
                failed = True
            if failed:
                with pytest.raises(pa.OutOfBlocks):
                    c.append_step(seqs, counts)
            else:
                slots, pairs = c.append_step(seqs, counts)
                assert slots.tolist() == want_slots
                assert [tuple(p) for p in pairs.tolist()] == want_pairs
                m = trial
        assert state(c, live, nb) == state(m, live, nb)


def test_max_seq_blocks(pa):
    c = pa.BlockManager(64, 16)
    for s, n in ((1, 0), (2, 17), (3, 40)):
        c.add_seq(s)
        c.append_slots(s, n)
    assert c.max_seq_blocks([1, 2, 3]) == 3 and c.max_seq_blocks([1]) == 0 and c.max_seq_blocks([]) == 0
    assert c.max_seq_blocks([2, 1]) == max(c.num_seq_blocks(2), c.num_seq_blocks(1))
    with pytest.raises(KeyError):
        c.max_seq_blocks([1, 42])
