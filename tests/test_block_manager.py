"""Host C++ block manager (product, via its C ABI) against the Python model (oracle):
bit-identical slots, copy pairs, block tables, reference counts and free stacks on
random traces and on every workload's allocator script."""
import numpy as np
import pytest
from hypothesis import given, settings, strategies as st

import workloads
from oracle.block_model import BlockManagerModel, OutOfBlocks as ModelOOM


def same_state(cpp, model, seqs):
    assert cpp.free_stack() == model.free_stack
    assert [cpp.refcount(b) for b in range(model.num_blocks)] == model.ref
    for s in seqs:
        assert cpp.block_table(s) == model.block_table(s)
        assert cpp.num_tokens(s) == model.num_tokens(s)


ops = st.lists(st.tuples(st.sampled_from(["add", "append", "append", "fork", "free"]),
                         st.integers(0, 6), st.integers(0, 6), st.integers(0, 50)), max_size=80)


@settings(max_examples=200, deadline=None)
@given(trace=ops, nb=st.integers(1, 40), seed=st.integers(0, 2**31 - 1))
def test_random_traces_match_model(pa, trace, nb, seed):
    order = np.random.default_rng(seed).permutation(nb).astype(np.int32)
    cpp = pa.BlockManager(nb, 16, order)
    model = BlockManagerModel(nb, 16, order.tolist())
    for kind, a, b, n in trace:
        got = want = None
        try:
            if kind == "add":
                model.add_seq(a)
            elif kind == "append":
                want = model.append_slots(a, n)
            elif kind == "fork":
                model.fork(a, b)
            else:
                model.free(a)
            model_err = None
        except (KeyError, ModelOOM) as e:
            model_err = type(e)
        try:
            if kind == "add":
                cpp.add_seq(a)
            elif kind == "append":
                got = cpp.append_slots(a, n)
            elif kind == "fork":
                cpp.fork(a, b)
            else:
                cpp.free(a)
            cpp_err = None
        except pa.OutOfBlocks:
            cpp_err = ModelOOM
        except (KeyError, pa.PAError):
            cpp_err = KeyError
        assert cpp_err == model_err, (kind, a, b, n)
        if want is not None and model_err is None:
            assert got[0].tolist() == want[0] and got[1] == want[1]
        same_state(cpp, model, list(model.tables))


def test_build_tables_match(pa):
    cpp = pa.BlockManager(50, 16)
    model = BlockManagerModel(50, 16)
    for s, n in [(3, 40), (1, 0), (7, 17)]:
        cpp.add_seq(s); model.add_seq(s)
        cpp.append_slots(s, n); model.append_slots(s, n)
    t1, l1 = cpp.build_tables([7, 1, 3], 5)
    t2, l2 = model.build_tables([7, 1, 3], 5)
    assert np.array_equal(t1, t2) and np.array_equal(l1, l2)
    with pytest.raises(pa.PAError):
        cpp.build_tables([3], 2)   # table longer than max_blocks


@pytest.mark.parametrize("cid", [1, 2, 3, 4, 5])
def test_workload_scripts_match_model(pa, cid):
    wl = workloads.make(cid, mini=cid != 1)
    cpp = pa.BlockManager(wl.num_blocks, wl.block_size, wl.free_order)
    model = BlockManagerModel(wl.num_blocks, wl.block_size, wl.free_order.tolist())
    got, want = [], []
    workloads.replay(wl, cpp, lambda k, v, s: got.append(s.copy()))
    workloads.replay(wl, model, lambda k, v, s: want.append(s.copy()))
    assert all(np.array_equal(a, b) for a, b in zip(got, want)) and len(got) == len(want)
    for st_ in wl.steps:
        if st_.k_new is None:
            continue
        for s in st_.seqs:
            a, b = cpp.append_slot(s), model.append_slot(s)
            assert a == b
    same_state(cpp, model, list(model.tables))


def test_fork_cow_counts_in_parallel_sampling_workload(pa):
    """Parallel-sampling workload: step 1 copies the shared last block for 3 of 4 children."""
    wl = workloads.make(4, mini=True)
    cpp = pa.BlockManager(wl.num_blocks, wl.block_size, wl.free_order)
    workloads.replay(wl, cpp, lambda k, v, s: None)
    pairs = [cpp.append_slot(s)[1] for s in wl.steps[0].seqs]
    n_parents = len(wl.steps[0].seqs) // 4
    assert sum(p is not None for p in pairs) == 3 * n_parents
    assert [p is None for p in pairs[:4]] == [False, False, False, True]
    pairs2 = [cpp.append_slot(s)[1] for s in wl.steps[0].seqs]
    assert all(p is None for p in pairs2)
