"""GPU parity: cache write, copy-on-write block copy and decode attention (unsplit
and split-K) against the CPU oracle, on every workload, through the C ABI.

Bit-exact: pools after every cache write / block copy, block tables, slot mappings.
Attention: fp32 max |err| <= 1e-5; bf16 |err| <= 1.5e-2 + 1e-2 |ref| per element.
"""
import copy

import numpy as np
import pytest

import workloads
from gpu_harness import TwoSided, check_close, to_dev, to_host, torch_mod

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _lib(pa):
    torch = torch_mod()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return pa


def partitions_for(wl):
    return (0, 16, 32) if wl.config_id == 1 else (0, 512, 256)


def run_workload(cid, mini, full_every=1, sample=64):
    wl = workloads.make(cid, mini=mini)
    ts = TwoSided(wl)
    assert ts.pools_equal(), "cache write of the set-up tokens is not bit-exact"
    assert ts.err_flag() == 0
    rng = np.random.default_rng(cid)
    for i, step in enumerate(wl.steps):
        ts.append_step(step)
        if i in (0, 1, len(wl.steps) - 1):
            assert ts.pools_equal(), f"step {i}: pools differ after copy-on-write + cache write"
        S = len(step.seqs)
        full = (i % full_every == 0) or i == len(wl.steps) - 1
        rows = None if full or S <= sample else np.sort(rng.choice(S, sample, replace=False))
        ref = ts.oracle_decode(step, rows)
        for part in partitions_for(wl):
            got = ts.gpu_decode(step, part)
            if rows is not None:
                got = got[rows]
            check_close(got, ref, wl.dtype, f"config {cid} step {i} partition {part}")
    assert ts.err_flag() == 0
    return ts


def test_tiny_fp32():
    run_workload(1, False)


@pytest.mark.parametrize("cid", [2, 3, 4, 5])
def test_mini_workloads(cid):
    run_workload(cid, True)


def test_mha_7b():
    run_workload(2, False)


def test_gqa_prefix_sharing():
    run_workload(3, False)


def test_parallel_sampling_fork_cow():
    ts = run_workload(4, False, full_every=5, sample=64)
    assert ts.model.num_free() == ts.gpu.manager.num_free()


def test_long_context_decode():
    run_workload(5, False)


def test_copy_on_write_pairs_in_first_step_only():
    wl = workloads.make(4, mini=True)
    ts = TwoSided(wl)
    ts.append_step(wl.steps[0])
    assert len(ts.last_pairs) == 3 * (len(wl.steps[0].seqs) // 4)
    ts.append_step(wl.steps[1])
    assert len(ts.last_pairs) == 0
    assert ts.pools_equal()


def _permuted(wl, seed):
    wl2 = copy.copy(wl)
    wl2.free_order = np.random.default_rng(seed).permutation(wl.num_blocks).astype(np.int32)
    return wl2


@pytest.mark.parametrize("part", [0, 256])
def test_physical_placement_is_bitwise_invisible(part):
    """Same logical data in two differently shuffled pools: identical GPU outputs,
    since every reduction runs in logical-block order."""
    wl = workloads.make(3, mini=True)
    outs = []
    for seed in (1, 2):
        w = _permuted(wl, seed)
        ts = TwoSided(w)
        ts.append_step(w.steps[0])
        outs.append(ts.gpu_decode(w.steps[0], part))
    assert outs[0].tobytes() == outs[1].tobytes()


def _custom(lens, hq, hkv, d, dtype, seed=5, extra_blocks=4):
    rng = np.random.default_rng(seed)
    need = sum(-(-L // 16) for L in lens) + extra_blocks
    wl = workloads.Workload(0, "custom", dtype, need, hq, hkv, d, 1.0 / np.sqrt(d),
                            rng.permutation(need).astype(np.int32))
    for s, L in enumerate(lens):
        wl.ops.append(("add", s))
        if L:
            wl.ops.append(("append", s, workloads.normal(rng, (L, hkv, d), dtype),
                           workloads.normal(rng, (L, hkv, d), dtype)))
    q = workloads.normal(rng, (len(lens), hq, d), dtype)
    wl.steps.append(workloads.Step(list(range(len(lens))), None, None, q))
    return wl


@pytest.mark.parametrize("dtype,d", [("bf16", 128), ("bf16", 64), ("f32", 128), ("f32", 64)])
@pytest.mark.parametrize("g", [1, 2, 4, 8])
def test_edge_lengths_all_variants(dtype, d, g):
    """Empty context, a single token, block and partition boundaries +-1, ragged tails,
    and lengths around the per-sequence unit sizes (1024, 2048 tokens)."""
    lens = [0, 1, 15, 16, 17, 31, 33, 255, 256, 257, 511, 512, 513, 700, 1023, 1024, 1025, 2047, 2049, 3001]
    wl = _custom(lens, 2 * g, 2, d, dtype)
    ts = TwoSided(wl)
    step = wl.steps[0]
    ref = ts.oracle_decode(step)
    assert np.array_equal(ref[0], np.zeros_like(ref[0]))
    for part in (0, 16, 256):
        got = ts.gpu_decode(step, part)
        assert np.array_equal(got[0], np.zeros_like(got[0])), "empty context must give 0"
        check_close(got, ref, dtype, f"{dtype} d{d} g{g} part {part}")
    assert ts.err_flag() == 0


def test_gqa_equals_repeated_mha():
    wl = _custom([40, 300, 129], 8, 2, 128, "bf16")
    ts = TwoSided(wl)
    out_gqa = ts.gpu_decode(wl.steps[0], 0)
    # same data with kv heads repeated 4x: an MHA pool
    kc = np.repeat(ts.kc, 4, axis=1)
    vc = np.repeat(ts.vc, 4, axis=1)
    torch = torch_mod()
    import paged_kv_cache_389_b200 as pa
    t, l = ts.tables(wl.steps[0].seqs)
    kd, vd = to_dev(kc), to_dev(vc)
    q = to_dev(wl.steps[0].q)
    out = torch.empty_like(q)
    pa.pa_decode(q, kd, vd, torch.from_numpy(t).cuda(), torch.from_numpy(l).cuda(), int(l.max()),
                 wl.scale, out)
    check_close(to_host(out), np.asarray(workloads.bf16_bits_to_f32(out_gqa), np.float64), "bf16", "gqa vs mha")


def test_many_sequences_split_limit():
    """4096 short sequences with split-K (the largest batch the split path takes)."""
    rng = np.random.default_rng(9)
    lens = rng.integers(1, 80, size=4096).tolist()
    wl = _custom(lens, 4, 1, 64, "bf16")
    ts = TwoSided(wl)
    ref = ts.oracle_decode(wl.steps[0])
    check_close(ts.gpu_decode(wl.steps[0], 32), ref, "bf16", "4096 seqs split")
    check_close(ts.gpu_decode(wl.steps[0], 0), ref, "bf16", "4096 seqs")


def test_device_index_errors_are_flagged_not_fatal():
    torch = torch_mod()
    import paged_kv_cache_389_b200 as pa
    wl = _custom([40, 20], 4, 4, 128, "bf16")
    ts = TwoSided(wl)
    g = ts.gpu
    step = wl.steps[0]
    t, l = ts.tables(step.seqs)
    # table entry outside the pool
    bad = t.copy()
    bad[0, 1] = wl.num_blocks + 3
    g.err_flag.zero_()
    ts.gpu_decode(step, 0, tables=bad, lens=l)
    assert pa.pa_wait(g.err_flag) & pa.PA_DEVERR_BLOCK_ID
    # context longer than max_context_len
    g.err_flag.zero_()
    ts.gpu_decode(step, 0, tables=t, lens=l, max_context=30)
    assert pa.pa_wait(g.err_flag) & pa.PA_DEVERR_CONTEXT_LEN
    # slot outside the pool; negative slot is padding (no flag, nothing written)
    g.err_flag.zero_()
    k = torch.zeros((2, 4, 128), dtype=torch.bfloat16, device="cuda")
    before = to_host(g.key_cache).tobytes()
    pa.pa_cache_write(k, k, torch.tensor([-1, wl.num_blocks * 16], dtype=torch.int64, device="cuda"),
                      g.key_cache, g.value_cache, g.err_flag)
    assert pa.pa_wait(g.err_flag) == pa.PA_DEVERR_SLOT
    assert to_host(g.key_cache).tobytes() == before
    # copy pair outside the pool
    g.err_flag.zero_()
    pa.pa_copy_blocks(g.key_cache, g.value_cache,
                      torch.tensor([[0, wl.num_blocks]], dtype=torch.int32, device="cuda"), g.err_flag)
    assert pa.pa_wait(g.err_flag) == pa.PA_DEVERR_PAIR
    assert to_host(g.key_cache).tobytes() == before
    # the context is still healthy: a clean decode matches the oracle
    g.err_flag.zero_()
    check_close(ts.gpu_decode(step, 0), ts.oracle_decode(step), "bf16", "after flagged errors")
    assert pa.pa_wait(g.err_flag) == 0


def _grouped_workload(g=4):
    """Sibling structures the shared-prefix grouping must get right (g query heads
    per kv head): large families become tile groups of at most 128 / g members,
    families with members x g <= 16 rows become row groups."""
    rng = np.random.default_rng(21)
    hkv, d = 4, 128
    hq = g * hkv
    # (parent tokens, [suffix lengths]) per family; forked parents end on a block
    # boundary so that no sibling's first append needs a copy.  A tile group needs
    # at least 4 members and takes at most 128 / g; a row group 2 to 16 / g.
    spec = []
    spec.append((1104, [int(x) for x in rng.integers(0, 300, size=20)]))   # 20 siblings
    spec.append((608, [5, 77, 130, 3, 9, 27, 81, 1, 40]))   # 9 siblings sharing 38 full blocks
    spec.append((208, [40, 41, 0, 7, 13, 90, 5, 60]))        # shares 13 blocks: < one 256-token partition
    spec.append((512, [0] * 8))                  # members entirely inside the shared prefix
    spec.append((333, []))                       # singleton (parent kept, partly filled last block)
    spec.append((400, [3, 9, 27]))               # 3 siblings: a row group for g <= 4, none for g = 8
    nb = 20 + sum(-(-(pt + max(sx, default=0) + 2) // 16) * (len(sx) + 1) for pt, sx in spec)
    wl = workloads.Workload(0, "groups", "bf16", nb, hq, hkv, d, 1.0 / np.sqrt(d),
                            rng.permutation(nb).astype(np.int32))
    seq = 0
    seqs = []
    for fi, (pt, sx) in enumerate(spec):
        parent = 1000 + fi
        wl.ops.append(("add", parent))
        wl.ops.append(("append", parent, workloads.normal(rng, (pt, hkv, d), "bf16"),
                       workloads.normal(rng, (pt, hkv, d), "bf16")))
        if not sx:
            seqs.append(parent)
            continue
        kids = []
        for _ in sx:
            wl.ops.append(("fork", parent, seq))
            kids.append(seq)
            seq += 1
        wl.ops.append(("free", parent))
        for kid, n in zip(kids, sx):
            if n:
                wl.ops.append(("append", kid, workloads.normal(rng, (n, hkv, d), "bf16"),
                               workloads.normal(rng, (n, hkv, d), "bf16")))
        seqs.extend(kids)
    # a sequence that reuses family 0's prefix but is not next to it: not grouped, still correct
    wl.ops.append(("fork", 0, 5000))
    seqs.append(5000)
    S = len(seqs)
    wl.steps.append(workloads.Step(seqs, workloads.normal(rng, (S, hkv, d), "bf16"),
                                   workloads.normal(rng, (S, hkv, d), "bf16"),
                                   workloads.normal(rng, (S, hq, d), "bf16")))
    return wl


@pytest.mark.parametrize("g", [1, 2, 4, 8])
def test_shared_prefix_groups_match_oracle(g):
    wl = _grouped_workload(g)
    ts = TwoSided(wl)
    step = wl.steps[0]
    ts.append_step(step)
    assert ts.pools_equal()
    ref = ts.oracle_decode(step)
    for part in (0, 48, 256, 512, 1024):
        check_close(ts.gpu_decode(step, part), ref, "bf16", f"g{g} grouped decode partition {part}")
    # members whose whole context lies inside the shared blocks: every partition
    # comes from the group units (contexts cut back to 1024 and 512 tokens)
    t, l = ts.tables(step.seqs)
    l2 = l.copy()
    l2[:4] = 1024
    fam = [i for i, L in enumerate(l) if L == 513]
    assert len(fam) == 8
    l2[fam] = 512
    ref2 = ts.oracle_decode(step, tables=t, lens=l2)
    for part in (48, 256, 512, 1024):
        got = ts.gpu_decode(step, part, tables=t, lens=l2, max_context=int(l.max()))
        check_close(got, ref2, "bf16", f"g{g} fully shared members, partition {part}")
    assert ts.err_flag() == 0


def _families_workload(spec, g, n_loners, seed=31):
    """Sibling families (parent tokens, [suffix lengths]) followed by n_loners unrelated
    sequences of 40 tokens, g query heads per kv head, 2 kv heads, head_dim 128."""
    rng = np.random.default_rng(seed)
    hkv, d = 2, 128
    hq = g * hkv
    nb = 16 + sum(-(-(pt + max(sx, default=0) + 2) // 16) * (len(sx) + 1) for pt, sx in spec) + 4 * n_loners
    wl = workloads.Workload(0, "families", "bf16", nb, hq, hkv, d, 1.0 / np.sqrt(d),
                            rng.permutation(nb).astype(np.int32))
    seq, seqs = 0, []
    for fi, (pt, sx) in enumerate(spec):
        parent = 10000 + fi
        wl.ops.append(("add", parent))
        wl.ops.append(("append", parent, workloads.normal(rng, (pt, hkv, d), "bf16"),
                       workloads.normal(rng, (pt, hkv, d), "bf16")))
        kids = []
        for _ in sx:
            wl.ops.append(("fork", parent, seq))
            kids.append(seq)
            seq += 1
        wl.ops.append(("free", parent))
        for kid, n in zip(kids, sx):
            if n:
                wl.ops.append(("append", kid, workloads.normal(rng, (n, hkv, d), "bf16"),
                               workloads.normal(rng, (n, hkv, d), "bf16")))
        seqs.extend(kids)
    for _ in range(n_loners):
        wl.ops.append(("add", seq))
        wl.ops.append(("append", seq, workloads.normal(rng, (40, hkv, d), "bf16"),
                       workloads.normal(rng, (40, hkv, d), "bf16")))
        seqs.append(seq)
        seq += 1
    S = len(seqs)
    wl.steps.append(workloads.Step(seqs, workloads.normal(rng, (S, hkv, d), "bf16"),
                                   workloads.normal(rng, (S, hkv, d), "bf16"),
                                   workloads.normal(rng, (S, hq, d), "bf16")))
    return wl


@pytest.mark.parametrize("g", [1, 2, 4])
def test_long_shared_runs_and_tail_boundaries(g):
    """More than 64 sequences (the table comparison runs in the detection grid's extra
    blocks), siblings sharing 4800 tokens (300 blocks: more than one 256-entry round),
    and 4-sibling families whose private tails are exactly 4 blocks (taken by the
    group-rows unit) or 5 blocks (left to the per-sequence kernel), against the oracle;
    the detection output against the rule."""
    spec = [(4800, [1, 17, 40, 3]),          # 300 shared blocks
            (512, [63, 48, 10, 1]),          # tails of at most 4 blocks
            (512, [64, 80, 5, 0]),           # a 5-block tail: no tails
            (1040, [15, 16, 47, 63])]        # 65 shared blocks, tails 1..4 blocks
    wl = _families_workload(spec, g, n_loners=60)
    ts = TwoSided(wl)
    step = wl.steps[0]
    ts.append_step(step)
    assert ts.pools_equal()
    ref = ts.oracle_decode(step)
    for part in (256, 512):
        check_close(ts.gpu_decode(step, part), ref, "bf16", f"g{g} families partition {part}")
    assert ts.err_flag() == 0
    # the detection's output in a fresh workspace against the rule
    torch = torch_mod()
    t, l = ts.tables(step.seqs)
    S, part = len(step.seqs), 512
    maxc = int(l.max())
    ws = torch.zeros(ts.pa.pa_decode_workspace_size(S, wl.num_q_heads, wl.head_dim, maxc, part),
                     dtype=torch.uint8, device="cuda")
    out = torch.empty((S, wl.num_q_heads, wl.head_dim), dtype=torch.bfloat16, device="cuda")
    ts.pa.pa_decode(to_dev(step.q), ts.gpu.key_cache, ts.gpu.value_cache, torch.from_numpy(t).cuda(),
                    torch.from_numpy(l).cuda(), maxc, wl.scale, out, part, ws, ts.gpu.err_flag)
    assert ts.err_flag() == 0
    rows = S * wl.num_q_heads * -(-maxc // part)
    at = -(-(rows * wl.head_dim * 4 + rows * 8) // 16) * 16
    raw = ws.cpu().numpy()
    want_ft, want_tiles, want_rows = _expected_groups(t, l, part, g, wl.num_kv_heads)
    assert raw[at:at + 4 * S].view(np.int32).tolist() == want_ft
    assert sum(1 for r in want_rows if r[3] == 1) == 3      # three families take their tails
    assert any(r[3] == 0 for r in want_rows)                # the 5-block tail does not


@pytest.mark.parametrize("cid,part", [(1, 0), (1, 16), (2, 256), (3, 0), (3, 256), (4, 256)])
def test_append_decode_one_call(cid, part):
    """pa_append_decode (cache write + decode in one call, chained launches) gives the
    oracle's result for every step and leaves the pools bit-identical to the oracle's."""
    wl = workloads.make(cid, mini=cid != 1)
    ts = TwoSided(wl)
    for i, step in enumerate(wl.steps[:3]):
        got = ts.append_decode_step(step, part)
        assert ts.pools_equal(), f"config {cid} step {i}: pools differ"
        check_close(got, ts.oracle_decode(step), wl.dtype, f"append+decode config {cid} step {i} partition {part}")
    assert ts.err_flag() == 0


def test_append_decode_full_size_in_the_timed_configuration():
    """The benchmark's timed step itself: the GQA-8B prefix-sharing workload at full size,
    one pa_append_decode call at 512-token partitions; pools bit-exact, rows sampled."""
    wl = workloads.make(3)
    ts = TwoSided(wl)
    step = wl.steps[0]
    got = ts.append_decode_step(step, 512)
    assert ts.pools_equal(), "pools differ after the one-call write"
    rows = np.sort(np.random.default_rng(7).choice(len(step.seqs), 48, replace=False))
    check_close(got[rows], ts.oracle_decode(step, rows), "bf16", "append+decode full size, partition 512")
    assert ts.err_flag() == 0


def test_append_decode_matches_two_calls_bitwise():
    """Same kernels, same order of arithmetic: one call and two calls agree bit for bit."""
    wl = workloads.make(3, mini=True)
    a, b = TwoSided(wl), TwoSided(wl)
    step = wl.steps[0]
    got = a.append_decode_step(step, 256)
    b.append_step(step)
    ref = b.gpu_decode(step, 256)
    assert got.tobytes() == ref.tobytes()


def test_prefix_cached_prompts_decode_as_if_written_in_full():
    """Automatic prefix caching on the hot path: prompts sharing a system prompt are
    created from their token ids, only the tokens not found in the cache get their K/V
    written, and decode through the shared blocks matches (a) the oracle over the same
    pool and (b) a dense reference over each prompt's own K/V.  A token's K/V depend only
    on the prompt up to it, as a model's would."""
    import zlib
    import oracle
    from oracle.block_model import BlockManagerModel
    from paged_kv_cache_389_b200.cache import PagedKVCache
    torch = torch_mod()
    import paged_kv_cache_389_b200 as pa
    rng = np.random.default_rng(31)
    hq, hkv, d, nb = 32, 8, 128, 96
    scale = 1.0 / np.sqrt(d)

    def kv_of(prompt, p):
        g = np.random.default_rng(zlib.crc32(np.asarray(prompt[:p + 1], np.int32).tobytes()))
        return workloads.normal(g, (2, hkv, d), "bf16")

    system = rng.integers(0, 1000, size=80).tolist()            # five full blocks
    prompts = [system + rng.integers(0, 1000, size=int(n)).tolist() for n in (3, 17, 40, 0, 25)]
    prompts += [system[:48] + rng.integers(0, 1000, size=9).tolist()]   # shares three blocks
    free_order = rng.permutation(nb).astype(np.int32)
    gpu = PagedKVCache(nb, hkv, d, torch.bfloat16, "cuda", free_order)
    model = BlockManagerModel(nb, 16, free_order.tolist())
    kc = np.full((nb, hkv, 16, d), 0x7FC0, np.uint16)           # NaN-filled like the GPU pools
    vc = kc.copy()
    cached = []
    order = list(range(len(prompts)))
    for i in order:
        n_g, slots_g = gpu.manager.add_seq_tokens(i, prompts[i])
        n_m, slots_m = model.add_seq_tokens(i, prompts[i])
        assert n_g == n_m and slots_g.tolist() == list(slots_m)
        cached.append(n_m)
        new = [kv_of(prompts[i], p) for p in range(n_m, len(prompts[i]))]
        if new:
            k = np.stack([x[0] for x in new])
            v = np.stack([x[1] for x in new])
            sl = np.asarray(slots_m, np.int64)
            oracle.cache_write(k, v, sl, kc, vc)
            pa.pa_cache_write(to_dev(k), to_dev(v), torch.from_numpy(sl).cuda(), gpu.key_cache,
                              gpu.value_cache, gpu.err_flag)
        if i == 2:                                               # free one prompt midway
            gpu.manager.free(1)
            model.free(1)
    assert cached[1:] == [80, 80, 80, 80, 48] and cached[0] == 0
    live = [i for i in order if i != 1]
    assert to_host(gpu.key_cache).tobytes() == kc.tobytes()
    t, l = model.build_tables(live, max(len(model.block_table(i)) for i in live))
    q = workloads.normal(rng, (len(live), hq, d), "bf16")
    ref = oracle.decode(q, kc, vc, t, l, scale)
    # dense reference over each prompt's own K/V
    g = hq // hkv
    for row, i in enumerate(live):
        kv = np.stack([kv_of(prompts[i], p) for p in range(len(prompts[i]))])   # [L, 2, hkv, d]
        K = workloads.bf16_bits_to_f32(kv[:, 0]).astype(np.float64)
        V = workloads.bf16_bits_to_f32(kv[:, 1]).astype(np.float64)
        Q = workloads.bf16_bits_to_f32(q[row]).astype(np.float64)
        for h in range(hq):
            sc = K[:, h // g] @ Q[h] * scale
            w = np.exp(sc - sc.max())
            dense = (w[:, None] * V[:, h // g]).sum(0) / w.sum()
            assert np.allclose(ref[row, h], dense, rtol=1e-9, atol=1e-9)
    for part in (0, 32):
        got = ts_free_decode(pa, torch, q, gpu, t, l, scale, part)
        check_close(got, ref, "bf16", f"prefix-cached decode partition {part}")
    assert pa.pa_wait(gpu.err_flag) == 0


def ts_free_decode(pa, torch, q_np, gpu, t, l, scale, part):
    q = to_dev(q_np)
    out = torch.empty_like(q)
    maxc = int(l.max())
    ws = None
    if part:
        n = pa.pa_decode_workspace_size(q.shape[0], q.shape[1], q.shape[2], maxc, part)
        ws = torch.empty(max(n, 16), dtype=torch.uint8, device="cuda")
    pa.pa_decode(q, gpu.key_cache, gpu.value_cache, torch.from_numpy(t).cuda(), torch.from_numpy(l).cuda(),
                 maxc, scale, out, part, ws, gpu.err_flag)
    return to_host(out)


def _expected_groups(tables, lens, part, g, hkv, min_members=4):
    """The shared-prefix grouping rule, written out on the host: lcp[s] = leading
    full blocks of s's table equal to those of s - 1; a run is a stretch of
    sequences each sharing >= part tokens of full blocks with its predecessor.
    With row groups (g <= 4) a run of n sequences with n * g <= 16 stays whole;
    other runs are cut into chunks of 128 / g counted from their start.  A chunk
    shares nb = min(lcp over its members after the first) blocks and is a row
    group when row groups are on, 2 <= n and n * g <= 16, else a tile group when
    n >= 4.  A row group whose members' tails (blocks past the nb shared ones) are
    at most 4 blocks long covers its members entirely.  Returns first_t (tokens
    per sequence covered by its group), the tile groups' records, then the row
    groups' records (their last field: 1 when they take the tails)."""
    S = len(lens)
    bpp = part // 16
    M = 128 // g
    row_groups = g <= 4
    lcp = [0] * S
    for s in range(1, S):
        n = min(int(lens[s]), int(lens[s - 1])) // 16
        k = 0
        while k < n and tables[s, k] == tables[s - 1, k]:
            k += 1
        lcp[s] = k
    runs, rs = {}, 0
    for s in range(S):
        if s == 0 or lcp[s] < bpp:
            rs = s
        runs.setdefault(rs, []).append(s)
    chunks = []
    for r0, mem in sorted(runs.items()):
        if row_groups and len(mem) * g <= 16:
            chunks.append(mem)
        else:
            chunks += [mem[i:i + M] for i in range(0, len(mem), M)]
    first_t, tiles, rows = [0] * S, [], []
    for mem in chunks:
        n = len(mem)
        row = row_groups and n >= 2 and n * g <= 16
        tile = not row and n >= min_members
        mn = min(lcp[m] for m in mem[1:]) if n > 1 else 0
        nb = min(mn, (1 << 21) - 1) if (row or tile) and mn >= bpp else 0
        if nb == 0:
            continue
        # a row group takes its members' private tails when none is longer than 4 blocks
        tails = row and max(-(-int(lens[m]) // 16) - nb for m in mem) <= 4
        for m in mem:
            # members of a row group with tails carry bit 30 (their output is written
            # by the group's unit; the combine skips them)
            first_t[m] = (max(int(lens[m]), nb * 16) | (1 << 30)) if tails else nb * 16
        if row:
            rows.append((mem[0], n, nb * 16, 1 if tails else 0))
        else:
            tiles.append((mem[0], n, nb * 16, len(tiles) * hkv))
    return first_t, tiles, rows


@pytest.mark.parametrize("cid,part", [(3, 512), (4, 512), (3, 64)])
def test_group_detection_matches_the_rule(cid, part):
    """The detection kernel's output in the workspace (first shared partitions per
    sequence, the group list, the counts) equals the grouping rule computed on the
    host from the same tables."""
    torch = torch_mod()
    wl = workloads.make(cid, mini=(part == 64))
    ts = TwoSided(wl)
    step = wl.steps[0]
    ts.append_step(step)
    t, l = ts.tables(step.seqs)
    S = len(step.seqs)
    maxc = int(l.max())
    n = ts.pa.pa_decode_workspace_size(S, wl.num_q_heads, wl.head_dim, maxc, part)
    ws = torch.zeros(n, dtype=torch.uint8, device="cuda")
    out = torch.empty((S, wl.num_q_heads, wl.head_dim), dtype=torch.bfloat16, device="cuda")
    ts.pa.pa_decode(to_dev(step.q), ts.gpu.key_cache, ts.gpu.value_cache, torch.from_numpy(t).cuda(),
                    torch.from_numpy(l).cuda(), maxc, wl.scale, out, part, ws, ts.gpu.err_flag)
    assert ts.err_flag() == 0
    parts = -(-maxc // part)
    rows = S * wl.num_q_heads * parts
    at = -(-(rows * wl.head_dim * 4 + rows * 8) // 16) * 16
    raw = ws.cpu().numpy()
    first_t = raw[at:at + 4 * S].view(np.int32)
    gat = at + -(-4 * S // 16) * 16
    meta = raw[gat + 16 * S:gat + 16 * S + 32].view(np.int32)
    want_ft, want_tiles, want_rows = _expected_groups(t, l, part, wl.num_q_heads // wl.num_kv_heads,
                                                      wl.num_kv_heads)
    assert first_t.tolist() == want_ft
    assert meta[0] == len(want_tiles) and meta[1] == len(want_tiles) * wl.num_kv_heads
    assert meta[5] == len(want_rows)
    n_g = len(want_tiles) + len(want_rows)
    got = [tuple(int(x) for x in r) for r in raw[gat:gat + 16 * n_g].view(np.int32).reshape(-1, 4)]
    assert got[:len(want_tiles)] == want_tiles            # tile groups in sequence order
    got_rows = got[len(want_tiles):]
    assert sorted(got_rows) == sorted(want_rows)          # row groups: longest first by buckets
    keys = [31 - min(31, (r[2] // 16) >> 3) for r in got_rows]
    assert keys == sorted(keys)
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    if want_tiles:   # SMs the detection kernel gave the group tiles
        assert 1 <= meta[4] <= sms
    else:
        assert meta[4] == 0
    if want_rows:    # and the group rows
        assert 1 <= meta[7] <= sms
    else:
        assert meta[7] == 0
    want_groups = want_tiles + want_rows
    if cid == 3:
        assert len(want_groups) > 0
    if cid == 4:   # four forked siblings of g = 4: 16 query rows, one row group each
        assert len(want_rows) > 0
