"""GPU parity of the tcgen05 chunked-prefill kernel against the CPU oracle.

Row i of a chunk of C_s rows sits at position L_s - C_s + i and attends causally to
keys 0..that position through the block table.  bf16 tolerance per element:
|gpu - oracle| <= 1.5e-2 + 1e-2 |oracle|.
"""
import numpy as np
import pytest

import oracle
import workloads
from gpu_harness import TwoSided, check_close, to_dev, to_host, torch_mod

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _lib(pa):
    return pa


def gpu_prefill(ts, q_np, chunk_lens, tables, lens):
    torch = torch_mod()
    q = to_dev(q_np)
    out = torch.full_like(q, float("nan"))
    ts.pa.pa_prefill_chunk(q, ts.gpu.key_cache, ts.gpu.value_cache, torch.from_numpy(tables).cuda(),
                           torch.from_numpy(lens).cuda(), torch.from_numpy(np.asarray(chunk_lens, np.int32)).cuda(),
                           ts.wl.scale, out, ts.gpu.err_flag)
    return to_host(out)


def rows_mask(chunk_lens, mc):
    m = np.zeros((len(chunk_lens), mc), bool)
    for s, c in enumerate(chunk_lens):
        m[s, :c] = True
    return m


def test_long_context_chunk_mini():
    wl = workloads.make(5, mini=True)
    ts = TwoSided(wl)
    pf = wl.prefill
    t, l = ts.tables(pf.seqs)
    ch = [pf.chunk] * len(pf.seqs)
    got = gpu_prefill(ts, pf.q, ch, t, l)
    ref = oracle.prefill(pf.q, ts.kc, ts.vc, t, l, np.array(ch, np.int32), wl.scale)
    check_close(got, ref, "bf16", "prefill mini")
    assert ts.err_flag() == 0


def _custom(lens, hq, hkv, seed=3, extra=5):
    rng = np.random.default_rng(seed)
    need = sum(-(-L // 16) for L in lens) + extra
    wl = workloads.Workload(0, "custom", "bf16", need, hq, hkv, 128, 1.0 / np.sqrt(128),
                            rng.permutation(need).astype(np.int32))
    for s, L in enumerate(lens):
        wl.ops.append(("add", s))
        wl.ops.append(("append", s, workloads.normal(rng, (L, hkv, 128), "bf16"),
                       workloads.normal(rng, (L, hkv, 128), "bf16")))
    return wl, rng


@pytest.mark.parametrize("g", [1, 2, 4, 8])
def test_ragged_chunks_all_group_sizes(g):
    """Chunks of 1 row, a whole prompt, lengths off tile and block boundaries, an empty chunk."""
    lens = [1, 37, 300, 129, 16, 600]
    chunks = [1, 37, 130, 0, 16, 257]
    wl, rng = _custom(lens, 2 * g, 2)
    ts = TwoSided(wl)
    t, l = ts.tables(list(range(len(lens))))
    mc = max(chunks)
    q = workloads.normal(rng, (len(lens), mc, 2 * g, 128), "bf16")
    got = gpu_prefill(ts, q, chunks, t, l)
    ref = oracle.prefill(q, ts.kc, ts.vc, t, l, np.array(chunks, np.int32), wl.scale)
    mask = rows_mask(chunks, mc)
    check_close(got[mask], ref[mask], "bf16", f"prefill g={g}")
    assert np.isnan(workloads.bf16_bits_to_f32(got[~mask])).all(), "rows past the chunk must not be written"
    assert ts.err_flag() == 0


def test_single_row_chunk_equals_decode():
    wl, rng = _custom([777, 65, 2049], 32, 8, seed=9)
    ts = TwoSided(wl)
    t, l = ts.tables([0, 1, 2])
    q1 = workloads.normal(rng, (3, 1, 32, 128), "bf16")
    pre = gpu_prefill(ts, q1, [1, 1, 1], t, l)
    step = workloads.Step([0, 1, 2], None, None, np.ascontiguousarray(q1[:, 0]))
    dec = ts.gpu_decode(step, 0)
    check_close(pre[:, 0], workloads.bf16_bits_to_f32(dec).astype(np.float64), "bf16", "1-row chunk vs decode")


def test_long_context_chunk_full_sampled_rows():
    """8 x 32768 tokens, 512-row chunk, 64/8 heads, the launch the benchmark times:
    every output finite; every row and head of sequence 0 and 64 random rows (all
    heads) of each other sequence against the oracle, element by element."""
    wl = workloads.make(5)
    ts = TwoSided(wl)
    pf = wl.prefill
    t, l = ts.tables(pf.seqs)
    ch = [pf.chunk] * len(pf.seqs)
    got = gpu_prefill(ts, pf.q, ch, t, l)
    assert np.isfinite(workloads.bf16_bits_to_f32(got)).all()
    rng = np.random.default_rng(5)
    mask = np.zeros((len(pf.seqs), pf.chunk), bool)
    mask[0, :] = True
    for s in range(1, len(pf.seqs)):
        mask[s, rng.choice(pf.chunk, 64, replace=False)] = True
    ref = oracle.prefill(pf.q, ts.kc, ts.vc, t, l, np.array(ch, np.int32), wl.scale, row_mask=mask)
    check_close(got[mask], ref[mask], "bf16", "prefill full (sequence 0 whole, sampled rows)")
    assert ts.err_flag() == 0


@pytest.mark.parametrize("hq,hkv", [(32, 8), (16, 16), (64, 8)])
def test_speculative_verify_chunks(hq, hkv):
    """Speculative-decoding verify: every sequence appends k_s in [1, 8] draft tokens and
    the k_s new positions attend causally to the paged cache -- a k_s-row chunk.  Shapes of
    the prefix-sharing workload (siblings sharing prefix blocks), ragged k_s."""
    rng = np.random.default_rng(17)
    d, S, prefix = 128, 12, 96
    ks = rng.integers(1, 9, size=S).tolist()
    suffix = rng.integers(1, 200, size=S).tolist()
    need = 3 * (prefix // 16) + sum(-(-(prefix + x + k) // 16) for x, k in zip(suffix, ks)) + 8
    wl = workloads.Workload(0, "verify", "bf16", need, hq, hkv, d, 1.0 / np.sqrt(d),
                            rng.permutation(need).astype(np.int32))
    for grp in range(3):                       # 3 parents x 4 forked siblings
        parent = 100 + grp
        wl.ops.append(("add", parent))
        wl.ops.append(("append", parent, workloads.normal(rng, (prefix, hkv, d), "bf16"),
                       workloads.normal(rng, (prefix, hkv, d), "bf16")))
        for c in range(4):
            wl.ops.append(("fork", parent, grp * 4 + c))
        wl.ops.append(("free", parent))
    for s in range(S):                         # private suffix, then the k_s draft tokens
        n = suffix[s] + ks[s]
        wl.ops.append(("append", s, workloads.normal(rng, (n, hkv, d), "bf16"),
                       workloads.normal(rng, (n, hkv, d), "bf16")))
    ts = TwoSided(wl)
    assert ts.pools_equal()
    t, l = ts.tables(list(range(S)))
    q = workloads.normal(rng, (S, 8, hq, d), "bf16")
    got = gpu_prefill(ts, q, ks, t, l)
    ref = oracle.prefill(q, ts.kc, ts.vc, t, l, np.array(ks, np.int32), wl.scale)
    mask = rows_mask(ks, 8)
    check_close(got[mask], ref[mask], "bf16", f"verify {hq}/{hkv}")
    assert ts.err_flag() == 0


def test_many_short_chunks_static_jobs():
    """256 sequences x 8 kv heads = 2048 one-tile jobs, more than 8 per CTA: the launch
    takes the static round robin of jobs (fewer per CTA are drawn from a counter, as
    in every other case here).  Ragged draft counts in [0, 8] (0: an empty job) over
    contexts of 20..400 tokens."""
    rng = np.random.default_rng(29)
    S, hq, hkv = 256, 32, 8
    lens = rng.integers(20, 401, size=S).tolist()
    ks = [int(min(k, L)) for k, L in zip(rng.integers(0, 9, size=S), lens)]
    wl, rng2 = _custom(lens, hq, hkv, seed=31)
    ts = TwoSided(wl)
    t, l = ts.tables(list(range(S)))
    q = workloads.normal(rng2, (S, 8, hq, 128), "bf16")
    got = gpu_prefill(ts, q, ks, t, l)
    ref = oracle.prefill(q, ts.kc, ts.vc, t, l, np.array(ks, np.int32), wl.scale)
    mask = rows_mask(ks, 8)
    check_close(got[mask], ref[mask], "bf16", "2048 static jobs")
    assert np.isnan(workloads.bf16_bits_to_f32(got[~mask])).all(), "rows past the chunk must not be written"
    assert ts.err_flag() == 0
