"""Multi-rank host path on CPU (gloo, world size 2 and 3): sequence sharding, timing
reduction, reassembly of per-rank outputs, the tensor-parallel kv-head split with its
output all-gather, and a rank that dies.

The decode path shards by sequence with no data-path exchange; here each rank
runs the CPU oracle on its shard and the shards must reassemble bit-exactly into
the unsharded result.  No GPU is touched.
"""
import os
import socket
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

from paged_kv_cache_389_b200.dist import shard_ranges  # noqa: E402  (pure Python; no library load)


def free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_shard_ranges_cover_balance_and_keep_groups():
    rng = np.random.default_rng(1)
    costs = rng.integers(100, 3000, size=256).tolist()
    groups = [i // 16 for i in range(256)]           # 16 sibling groups of 16
    for world in (1, 2, 3, 4, 8):
        r = shard_ranges(costs, world, groups)
        assert len(r) == world and r[0][0] == 0 and r[-1][1] == 256
        assert all(a[1] == b[0] for a, b in zip(r, r[1:]))
        assert all(s % 16 == 0 and e % 16 == 0 for s, e in r)   # never split a group
        loads = [sum(costs[s:e]) for s, e in r]
        biggest_group = max(sum(costs[g * 16:(g + 1) * 16]) for g in range(16))
        assert max(loads) - sum(costs) / world <= biggest_group
    r = shard_ranges([5, 5], 4)              # more ranks than sequences: some get nothing
    assert len(r) == 4 and sum(e - s for s, e in r) == 2 and max(e - s for s, e in r) == 1
    with pytest.raises(ValueError):
        shard_ranges([1, 1, 1], 2, groups=[0, 1, 0])


def _worker(rank, world, port, q):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=30))
    try:
        import oracle
        import workloads
        from oracle.block_model import BlockManagerModel
        from paged_kv_cache_389_b200.dist import max_over_ranks
        res = {"max": max_over_ranks(1.5 + rank)}
        wl = workloads.make(3, mini=True)
        model = BlockManagerModel(wl.num_blocks, wl.block_size, wl.free_order.tolist())
        kc = np.zeros(wl.cache_shape(), wl.np_dtype)
        vc = np.zeros_like(kc)
        workloads.replay(wl, model, lambda k, v, s: oracle.cache_write(k, v, s, kc, vc))
        step = wl.steps[0]
        seqs = step.seqs
        lens = [model.num_tokens(s) for s in seqs]
        groups = [s // 4 for s in seqs]             # mini workload: groups of 4 siblings
        lo, hi = shard_ranges(lens, world, groups)[rank]
        mb = max(len(model.block_table(s)) for s in seqs)
        t, l = model.build_tables(seqs[lo:hi], mb)
        mine = oracle.decode(np.ascontiguousarray(step.q[lo:hi]), kc, vc, t, l, wl.scale)
        parts = [None] * world
        dist.all_gather_object(parts, (lo, hi, mine))
        res["parts"] = parts
        q.put((rank, res))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_shard_without_exchange():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = dict(q.get(timeout=120) for _ in range(2))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert out[0]["max"] == out[1]["max"] == 2.5
    # reassemble and compare with one process doing everything
    import oracle
    import workloads
    from oracle.block_model import BlockManagerModel
    wl = workloads.make(3, mini=True)
    model = BlockManagerModel(wl.num_blocks, wl.block_size, wl.free_order.tolist())
    kc = np.zeros(wl.cache_shape(), wl.np_dtype)
    vc = np.zeros_like(kc)
    workloads.replay(wl, model, lambda k, v, s: oracle.cache_write(k, v, s, kc, vc))
    step = wl.steps[0]
    mb = max(len(model.block_table(s)) for s in step.seqs)
    t, l = model.build_tables(step.seqs, mb)
    full = oracle.decode(step.q, kc, vc, t, l, wl.scale)
    parts = sorted(out[0]["parts"], key=lambda x: x[0])
    assert parts[0][0] == 0 and parts[-1][1] == len(step.seqs)
    assert np.array_equal(np.concatenate([p[2] for p in parts]), full)


def _dying_worker(rank, world, port, q):
    import datetime
    import torch
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=5))
    if rank == 1:
        os._exit(3)                     # leaves between steps, nothing in flight
    try:
        dist.all_reduce(torch.ones(1))
        q.put("no error")
    except Exception as e:              # the survivor learns of it on the host
        q.put(type(e).__name__)


def test_rank_that_dies_is_detected_on_the_host():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = free_port()
    procs = [ctx.Process(target=_dying_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    msg = q.get(timeout=120)
    for p in procs:
        p.join(timeout=60)
        if p.is_alive():
            p.kill()
    assert msg != "no error"
    assert procs[1].exitcode == 3


def test_kv_head_shards_are_contiguous_and_even():
    from paged_kv_cache_389_b200.dist import shard_kv_heads
    for hkv in (1, 2, 8, 32):
        for world in range(1, hkv + 1):
            r = shard_kv_heads(hkv, world)
            assert r[0][0] == 0 and r[-1][1] == hkv and all(a[1] == b[0] for a, b in zip(r, r[1:]))
            w = [hi - lo for lo, hi in r]
            assert max(w) - min(w) <= 1 and min(w) >= 1
    with pytest.raises(ValueError):
        shard_kv_heads(4, 5)


def _tp_worker(rank, world, port, q):
    """Tensor-parallel split: this rank stores only its kv heads (same tables as every
    other rank), decodes them with the oracle, and all-gathers the output heads."""
    import datetime
    import torch
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=30))
    try:
        import oracle
        import workloads
        from oracle.block_model import BlockManagerModel
        from paged_kv_cache_389_b200.dist import gather_heads, shard_kv_heads
        wl = workloads.make(3, mini=True)
        g = wl.num_q_heads // wl.num_kv_heads
        lo, hi = shard_kv_heads(wl.num_kv_heads, world)[rank]
        model = BlockManagerModel(wl.num_blocks, wl.block_size, wl.free_order.tolist())
        shape = list(wl.cache_shape())
        shape[1] = hi - lo
        kc = np.zeros(shape, wl.np_dtype)
        vc = np.zeros_like(kc)
        workloads.replay(wl, model, lambda k, v, s: oracle.cache_write(
            np.ascontiguousarray(k[:, lo:hi]), np.ascontiguousarray(v[:, lo:hi]), s, kc, vc))
        step = wl.steps[0]
        mb = max(len(model.block_table(s)) for s in step.seqs)
        t, l = model.build_tables(step.seqs, mb)
        mine = oracle.decode(np.ascontiguousarray(step.q[:, lo * g:hi * g]), kc, vc, t, l, wl.scale)
        full = gather_heads(torch.from_numpy(mine), shard_kv_heads(wl.num_kv_heads, world), g)
        q.put((rank, full.numpy()))
    finally:
        dist.destroy_process_group()


def test_three_gloo_ranks_split_kv_heads_and_gather():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = free_port()
    world = 3                                        # 8 kv heads: 3 + 3 + 2 (uneven shards)
    procs = [ctx.Process(target=_tp_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = dict(q.get(timeout=180) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    import oracle
    import workloads
    from oracle.block_model import BlockManagerModel
    wl = workloads.make(3, mini=True)
    model = BlockManagerModel(wl.num_blocks, wl.block_size, wl.free_order.tolist())
    kc = np.zeros(wl.cache_shape(), wl.np_dtype)
    vc = np.zeros_like(kc)
    workloads.replay(wl, model, lambda k, v, s: oracle.cache_write(k, v, s, kc, vc))
    step = wl.steps[0]
    mb = max(len(model.block_table(s)) for s in step.seqs)
    t, l = model.build_tables(step.seqs, mb)
    want = oracle.decode(step.q, kc, vc, t, l, wl.scale)
    for r in range(world):                          # every rank holds the whole, bit for bit
        assert np.array_equal(out[r], want)


def _shard_ops(wl, keep):
    """The workload's allocator operations for the sequences in ``keep`` and every
    parent they were forked from (a group stays on one rank with its parent)."""
    parent = {}
    for op in wl.ops:
        if op[0] == "fork":
            parent[op[2]] = op[1]
    mine = set(keep)
    for s in list(keep):
        while s in parent:
            s = parent[s]
            mine.add(s)
    return [op for op in wl.ops if op[1] in mine]


def _manager_worker(rank, world, port, q):
    """Each rank owns a pool and the library's C++ block manager for its shard only,
    and a Python model of the same shard: tables, lengths, slots and copy-on-write
    pairs of every step must agree bit for bit (the host side of the sharded path)."""
    import datetime
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=30))
    try:
        import workloads
        from oracle.block_model import BlockManagerModel
        import paged_kv_cache_389_b200 as pa
        wl = workloads.make(4, mini=True)             # parents forked into 4 children each
        seqs = wl.steps[0].seqs
        groups = [s // 4 for s in seqs]
        n = {}
        for op in wl.ops:
            if op[0] == "add":
                n[op[1]] = 0
            elif op[0] == "append":
                n[op[1]] += op[2].shape[0]
            elif op[0] == "fork":
                n[op[2]] = n[op[1]]
        lo, hi = shard_ranges([n[s] for s in seqs], world, groups)[rank]
        mine = seqs[lo:hi]
        ops = _shard_ops(wl, mine)
        cpp = pa.BlockManager(wl.num_blocks, wl.block_size, wl.free_order)
        model = BlockManagerModel(wl.num_blocks, wl.block_size, wl.free_order.tolist())
        shard = workloads.Workload(wl.config_id, wl.name, wl.dtype, wl.num_blocks, wl.num_q_heads,
                                   wl.num_kv_heads, wl.head_dim, wl.scale, wl.free_order)
        shard.ops = ops
        workloads.replay(shard, cpp, lambda k, v, s: None)
        workloads.replay(shard, model, lambda k, v, s: None)
        steps = []
        for st in wl.steps:
            part = [s for s in st.seqs if s in set(mine)]
            if not part:
                continue
            slots_c, pairs_c = cpp.append_step(part, [1] * len(part))
            slots_m, pairs_m = [], []
            for s in part:
                sl, pr = model.append_slot(s)
                slots_m.append(sl)
                if pr is not None:
                    pairs_m.append(pr)
            mb = max(len(model.block_table(s)) for s in part)
            tc, lc = cpp.build_tables(part, mb)
            tm, lm = model.build_tables(part, mb)
            steps.append((slots_c.tolist() == slots_m,
                          [tuple(p) for p in pairs_c.tolist()] == pairs_m,
                          np.array_equal(tc, tm) and np.array_equal(lc, lm), len(part), len(pairs_m)))
        got = [None] * world
        dist.all_gather_object(got, (lo, hi, steps))
        q.put((rank, got))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_run_the_block_manager_on_their_shards():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = free_port()
    procs = [ctx.Process(target=_manager_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = dict(q.get(timeout=180) for _ in range(2))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    ranges = sorted((lo, hi) for lo, hi, _ in out[0])
    assert ranges[0][0] == 0 and ranges[0][1] == ranges[1][0] and ranges[1][0] > 0
    for lo, hi, steps in out[0]:
        assert steps, "every rank ran steps"
        for slots_ok, pairs_ok, tables_ok, n, _ in steps:
            assert slots_ok and pairs_ok and tables_ok and n == hi - lo
        assert sum(st[4] for st in steps) > 0, "the shard's first step copies shared last blocks"
