"""Host block manager snapshot / restore (pa_bm_snapshot, pa_bm_restore): a restored
manager continues exactly like the original, snapshots are deterministic, and
malformed buffers are refused without a crash."""
import struct

import numpy as np
import pytest


def full_state(mgr, seqs):
    return (mgr.free_stack(), mgr.evictable(), mgr.num_cached(),
            [mgr.refcount(b) for b in range(mgr.num_blocks)],
            [mgr.block_table(s) for s in seqs], [mgr.num_tokens(s) for s in seqs])


def random_ops(rng, n, start_id=0):
    """A reproducible list of operations over prompts that share prefixes."""
    prefixes = [rng.integers(0, 40, size=int(k)).tolist() for k in (16, 32, 48)]
    ops, live, nxt = [], [], start_id
    for _ in range(n):
        op = int(rng.integers(0, 6))
        if op <= 1 or not live:
            base = prefixes[int(rng.integers(0, len(prefixes)))]
            toks = base[:int(rng.integers(0, len(base) + 1))] + rng.integers(0, 40, size=int(rng.integers(0, 30))).tolist()
            ops.append(("tokens", nxt, toks))
            live.append(nxt)
            nxt += 1
        elif op == 2:
            ops.append(("fork", live[int(rng.integers(0, len(live)))], nxt))
            live.append(nxt)
            nxt += 1
        elif op == 3 and len(live) > 1:
            ops.append(("free", live.pop(int(rng.integers(0, len(live))))))
        else:
            k = int(rng.integers(1, len(live) + 1))
            seqs = [int(x) for x in rng.choice(live, size=k, replace=False)]
            ops.append(("step", seqs, rng.integers(0, 3, size=k).tolist()))
    return ops


def apply(pa, mgr, op):
    """Run one op; returns its result (or the exception type) for comparison."""
    try:
        if op[0] == "tokens":
            n, slots = mgr.add_seq_tokens(op[1], op[2])
            return ("tokens", n, slots.tolist())
        if op[0] == "fork":
            mgr.fork(op[1], op[2])
            return ("fork",)
        if op[0] == "free":
            mgr.free(op[1])
            return ("free",)
        slots, pairs = mgr.append_step(op[1], op[2])
        return ("step", slots.tolist(), pairs.tolist())
    except (pa.PAError, KeyError) as e:
        return type(e).__name__


@pytest.mark.parametrize("seed", range(4))
def test_restored_manager_continues_like_the_original(pa, seed):
    rng = np.random.default_rng(300 + seed)
    nb = 40
    order = rng.permutation(nb).tolist()
    ops = random_ops(rng, 240)
    a = pa.BlockManager(nb, 16, order)
    cut = int(rng.integers(40, 200))
    for op in ops[:cut]:
        apply(pa, a, op)                             # failed ops (out of blocks) change nothing
    snap = a.snapshot()
    b = pa.BlockManager.restore(snap)
    assert b.snapshot() == snap                      # byte for byte
    assert b.num_blocks == nb and b.block_size == 16
    for op in ops[cut:]:
        ra, rb = apply(pa, a, op), apply(pa, b, op)
        assert ra == rb, op
    seqs = sorted({o[1] for o in ops if o[0] == "tokens"} | {o[2] for o in ops if o[0] == "fork"})
    alive = [s for s in seqs if a.num_tokens(s) >= 0]
    assert full_state(a, alive) == full_state(b, alive)
    assert a.snapshot() == b.snapshot()


def test_snapshot_is_deterministic_and_small(pa):
    def build():
        m = pa.BlockManager(64, 16)
        for i in range(10):
            m.add_seq_tokens(i, list(range(100)) + [i] * 7)
        m.free(3)
        return m
    s1, s2 = build().snapshot(), build().snapshot()
    assert s1 == s2
    assert s1[:4] == b"PABM" and struct.unpack("<I", s1[4:8])[0] == 1
    assert len(s1) < 16 * 1024


def test_malformed_snapshots_are_refused(pa):
    m = pa.BlockManager(32, 16)
    m.add_seq_tokens(0, list(range(40)))
    m.add_seq(1)
    m.append_slots(1, 5)
    good = m.snapshot()
    bad = [b"", good[:3], b"XXXX" + good[4:], good[:4] + struct.pack("<I", 99) + good[8:],
           good[:-1], good + b"\0"]
    # a sequence block id pushed out of the pool: find the first table entry of seq 0
    nfree = struct.unpack("<I", good[16:20])[0]
    seq_at = 20 + 4 * nfree + 4 * 32 * 2 + 4     # after free stack, counts, generations, count
    blk_at = seq_at + 8 + 8 + 4                    # after id, tokens, table length
    corrupt = bytearray(good)
    corrupt[blk_at:blk_at + 4] = struct.pack("<i", 32)
    bad.append(bytes(corrupt))
    for data in bad:
        with pytest.raises(pa.PAError) as e:
            pa.BlockManager.restore(data)
        assert e.value.status == pa.PA_ERR_INVALID_ARG
    assert pa.BlockManager.restore(good).snapshot() == good


# ---- cross-checked restore: one malformed snapshot per consistency rule --------
def _parse(data):
    """Split a version-1 snapshot into its fields (layout of pa_bm_snapshot)."""
    at = 0

    def take(fmt):
        nonlocal at
        v = struct.unpack_from("<" + fmt, data, at)
        at += struct.calcsize("<" + fmt)
        return v

    magic, ver, nb, bs = take("4sIii")
    (nfree,) = take("I")
    free = list(take(f"{nfree}i")) if nfree else []
    refs = list(take(f"{nb}i"))
    gen = list(take(f"{nb}I"))
    (nseq,) = take("I")
    seqs = []
    for _ in range(nseq):
        sid, tokens, n = take("qqI")
        seqs.append([sid, tokens, list(take(f"{n}i")) if n else []])
    (ncached,) = take("I")
    cached = []
    for _ in range(ncached):
        b, parent, pgen, n = take("iiII")
        cached.append([b, parent, pgen, list(take(f"{n}i"))])
    (nev,) = take("I")
    ev = list(take(f"{nev}i")) if nev else []
    assert at == len(data)
    return dict(head=(magic, ver, nb, bs), free=free, refs=refs, gen=gen, seqs=seqs, cached=cached, ev=ev)


def _pack(f):
    out = struct.pack("<4sIii", *f["head"])
    out += struct.pack("<I", len(f["free"])) + struct.pack(f"<{len(f['free'])}i", *f["free"])
    nb = f["head"][2]
    out += struct.pack(f"<{nb}i", *f["refs"]) + struct.pack(f"<{nb}I", *f["gen"])
    out += struct.pack("<I", len(f["seqs"]))
    for sid, tokens, blocks in f["seqs"]:
        out += struct.pack("<qqI", sid, tokens, len(blocks)) + struct.pack(f"<{len(blocks)}i", *blocks)
    out += struct.pack("<I", len(f["cached"]))
    for b, parent, pgen, toks in f["cached"]:
        out += struct.pack("<iiII", b, parent, pgen, len(toks)) + struct.pack(f"<{len(toks)}i", *toks)
    out += struct.pack("<I", len(f["ev"])) + struct.pack(f"<{len(f['ev'])}i", *f["ev"])
    return out


def test_inconsistent_snapshots_are_refused(pa):
    """pa_bm_restore rebuilds every block's count from the tables and requires each
    block to be exactly one of free, evictable or held; a snapshot that breaks this
    would let take() hand a live block to a second sequence."""
    import copy
    m = pa.BlockManager(32, 16)
    m.add_seq_tokens(0, list(range(40)))      # 3 blocks, 2 of them indexed
    m.fork(0, 1)                              # counts 2
    m.add_seq_tokens(2, [7] * 33)             # 3 blocks, 2 indexed
    m.free(2)                                 # 2 evictable, 1 free
    m.add_seq(3)
    m.append_slots(3, 5)
    good = m.snapshot()
    f = _parse(good)
    assert _pack(f) == good                   # the test's own parser round-trips
    assert len(f["ev"]) == 2 and len(f["free"]) >= 3
    held = f["seqs"][0][2][0]
    cases = {}
    g = copy.deepcopy(f); g["free"][-1] = g["free"][-2]; cases["free stack lists a block twice"] = g
    g = copy.deepcopy(f); g["free"][-1] = held; cases["a held block on the free stack"] = g
    g = copy.deepcopy(f); g["refs"][held] += 1; cases["count above the tables holding it"] = g
    g = copy.deepcopy(f); g["refs"][held] -= 1; cases["count below the tables holding it"] = g
    g = copy.deepcopy(f); g["free"].pop(0); cases["a count-0 block neither free nor evictable"] = g
    g = copy.deepcopy(f); g["ev"].pop(0); cases["an indexed count-0 block off the evictable list"] = g
    g = copy.deepcopy(f); g["free"].append(g["ev"][0]); cases["an evictable block also free"] = g
    g = copy.deepcopy(f)
    ev0 = g["ev"].pop(0)
    g["free"].append(ev0)
    cases["an indexed block on the free stack"] = g
    for what, bad in cases.items():
        with pytest.raises(pa.PAError) as e:
            pa.BlockManager.restore(_pack(bad))
        assert e.value.status == pa.PA_ERR_INVALID_ARG, what
    assert pa.BlockManager.restore(good).snapshot() == good
