"""Pins of the fp64 CPU oracle against things other than itself.

Each check would fail on a plausible slip in the oracle: a wrong kv-head mapping,
a swapped block/slot index, a transposed pool layout, a dropped scale, a wrong
sign in the max shift, a missing causal bound.  Nothing here touches the CUDA
library.

* brute force: a pure-Python, non-paged softmax attention over the dense K/V that
  the test drew before scattering it into blocks (tiny sizes);
* the pool layout [num_blocks, kv_heads, block_size, head_dim] written with numpy
  multi-dimensional indexing, independently of the oracle's offset arithmetic;
* closed forms: identical keys / zero query / zero scale give the mean of V;
  one key gives that V row exactly; one key 40 above the rest gives its V row
  within e^-40 (L-1) max|V|;
* invariants: permuting physical blocks, sharing prefix blocks, GQA vs
  repeat-interleaved MHA, last prefill row vs decode, thread count.
"""
import math

import numpy as np
import pytest

import oracle
from oracle.block_model import BlockManagerModel
from workloads import to_bf16_bits, bf16_bits_to_f32

pytestmark = pytest.mark.usefixtures("oracle_lib")


# ---------------------------------------------------------------- helpers
def brute_attention(q, K, V, scale):
    """Pure-Python softmax attention of one query over dense keys/values (lists)."""
    if len(K) == 0:
        return [0.0] * len(q)
    xs = [scale * math.fsum(a * b for a, b in zip(q, k)) for k in K]
    m = max(xs)
    ws = [math.exp(x - m) for x in xs]
    z = math.fsum(ws)
    return [math.fsum(w * v[i] for w, v in zip(ws, V)) / z for i in range(len(q))]


def as_float(a):
    return bf16_bits_to_f32(a).astype(np.float64) if a.dtype == np.uint16 else a.astype(np.float64)


def paged_pool(dense_k, dense_v, tables, num_blocks, block_size, fill=np.nan, dtype=np.float32):
    """Scatter per-sequence dense K/V [L, Hkv, d] into a pool [NB, Hkv, B, d] with numpy
    indexing: token t of sequence s goes to pool[tables[s][t // B], :, t % B, :]."""
    Hkv, d = dense_k[0].shape[1:]
    if dtype == np.uint16:
        kc = np.full((num_blocks, Hkv, block_size, d), 0x7FC0, dtype=np.uint16)  # bf16 NaN
    else:
        kc = np.full((num_blocks, Hkv, block_size, d), fill, dtype=dtype)
    vc = kc.copy()
    for s, (K, V) in enumerate(zip(dense_k, dense_v)):
        for t in range(K.shape[0]):
            kc[tables[s][t // block_size], :, t % block_size, :] = K[t]
            vc[tables[s][t // block_size], :, t % block_size, :] = V[t]
    return kc, vc


def random_tables(rng, lens, block_size, num_blocks):
    perm = rng.permutation(num_blocks)
    tables, i = [], 0
    for L in lens:
        nb = -(-L // block_size)
        tables.append([int(b) for b in perm[i:i + nb]])
        i += nb
    mb = max(1, max(len(t) for t in tables))
    arr = np.full((len(lens), mb), -1, dtype=np.int32)
    for s, t in enumerate(tables):
        arr[s, :len(t)] = t
    return tables, arr


def tiny_case(rng, lens, hq, hkv, d, block_size, dtype):
    nb = sum(-(-L // block_size) for L in lens) + 3
    dense_k = [rng.standard_normal((L, hkv, d)).astype(np.float32) for L in lens]
    dense_v = [rng.standard_normal((L, hkv, d)).astype(np.float32) for L in lens]
    if dtype == np.uint16:
        dense_k = [to_bf16_bits(x) for x in dense_k]
        dense_v = [to_bf16_bits(x) for x in dense_v]
    tables, tarr = random_tables(rng, lens, block_size, nb)
    kc, vc = paged_pool(dense_k, dense_v, tables, nb, block_size, dtype=dtype)
    q = rng.standard_normal((len(lens), hq, d)).astype(np.float32)
    if dtype == np.uint16:
        q = to_bf16_bits(q)
    return dense_k, dense_v, tables, tarr, kc, vc, q


# ---------------------------------------------------------------- brute force
@pytest.mark.parametrize("dtype", [np.float32, np.uint16])
@pytest.mark.parametrize("block_size", [4, 16])
@pytest.mark.parametrize("hq,hkv", [(1, 1), (4, 2), (6, 3), (4, 1)])
def test_decode_matches_brute_force(dtype, block_size, hq, hkv):
    rng = np.random.default_rng(7 + hq * 10 + hkv + block_size)
    lens = [1, 13, 40] if block_size == 4 else [0, 17, 33]
    d = 8
    dk, dv, tables, tarr, kc, vc, q = tiny_case(rng, lens, hq, hkv, d, block_size, dtype)
    scale = 0.37
    got = oracle.decode(q, kc, vc, tarr, np.array(lens, np.int32), scale)
    g = hq // hkv
    for s, L in enumerate(lens):
        for h in range(hq):
            K = as_float(dk[s][:, h // g, :]).tolist()
            V = as_float(dv[s][:, h // g, :]).tolist()
            want = brute_attention(as_float(q[s, h]).tolist(), K, V, scale)
            np.testing.assert_allclose(got[s, h], want, rtol=0, atol=1e-12)


@pytest.mark.parametrize("dtype", [np.float32, np.uint16])
def test_prefill_matches_brute_force(dtype):
    rng = np.random.default_rng(11)
    lens, chunks, block_size, hq, hkv, d = [9, 30, 21], [3, 7, 21], 4, 4, 2, 8
    dk, dv, tables, tarr, kc, vc, _ = tiny_case(rng, lens, hq, hkv, d, block_size, dtype)
    mc = max(chunks)
    q = rng.standard_normal((len(lens), mc, hq, d)).astype(np.float32)
    if dtype == np.uint16:
        q = to_bf16_bits(q)
    scale = 0.5
    got = oracle.prefill(q, kc, vc, tarr, np.array(lens, np.int32), np.array(chunks, np.int32), scale)
    g = hq // hkv
    for s, (L, C) in enumerate(zip(lens, chunks)):
        for i in range(mc):
            if i >= C:
                assert np.isnan(got[s, i]).all()   # rows past the chunk are left alone
                continue
            pos = L - C + i
            for h in range(hq):
                K = as_float(dk[s][:pos + 1, h // g, :]).tolist()
                V = as_float(dv[s][:pos + 1, h // g, :]).tolist()
                want = brute_attention(as_float(q[s, i, h]).tolist(), K, V, scale)
                np.testing.assert_allclose(got[s, i, h], want, rtol=0, atol=1e-12)


def test_prefill_row_mask_computes_only_selected_rows():
    rng = np.random.default_rng(3)
    lens, chunks = [20, 12], [6, 4]
    dk, dv, tables, tarr, kc, vc, _ = tiny_case(rng, lens, 2, 1, 8, 4, np.float32)
    q = rng.standard_normal((2, 6, 2, 8)).astype(np.float32)
    mask = np.zeros((2, 6), bool)
    mask[0, 2] = mask[1, 3] = True
    full = oracle.prefill(q, kc, vc, tarr, np.array(lens, np.int32), np.array(chunks, np.int32), 0.3)
    part = oracle.prefill(q, kc, vc, tarr, np.array(lens, np.int32), np.array(chunks, np.int32), 0.3,
                          row_mask=mask)
    assert np.array_equal(part[mask], full[mask])
    assert np.isnan(part[~mask]).all()


# ---------------------------------------------------------------- pool layout
@pytest.mark.parametrize("dtype", [np.float32, np.uint16])
def test_cache_write_matches_page_layout(dtype):
    """oracle.cache_write puts token t of a sequence at pool[table[t//B], h, t%B, :]
    (numpy indexing on the [num_blocks, heads, block_size, head_size] shape), touches
    nothing else, and skips negative slots."""
    rng = np.random.default_rng(5)
    lens, hkv, d, B = [5, 19, 33], 3, 8, 16
    dk, dv, tables, tarr, want_k, want_v, _ = tiny_case(rng, lens, hkv, hkv, d, B, dtype)
    nb = want_k.shape[0]
    kc = np.full_like(want_k, 0x7FC0 if dtype == np.uint16 else np.nan)
    vc = kc.copy()
    for s, L in enumerate(lens):
        slots = np.array([tables[s][t // B] * B + t % B for t in range(L)], np.int64)
        slots_pad = np.concatenate([slots, [-1, -7]])
        kk = np.concatenate([dk[s], np.zeros((2, hkv, d), dk[s].dtype)])
        vv = np.concatenate([dv[s], np.zeros((2, hkv, d), dv[s].dtype)])
        oracle.cache_write(kk, vv, slots_pad, kc, vc)
    assert kc.tobytes() == want_k.tobytes() and vc.tobytes() == want_v.tobytes()
    with pytest.raises(ValueError):
        oracle.cache_write(dk[0][:1], dv[0][:1], np.array([nb * B], np.int64), kc, vc)


def test_copy_blocks_copies_whole_blocks_only():
    rng = np.random.default_rng(9)
    kc = rng.standard_normal((10, 2, 16, 8)).astype(np.float32)
    vc = rng.standard_normal((10, 2, 16, 8)).astype(np.float32)
    k0, v0 = kc.copy(), vc.copy()
    pairs = np.array([[1, 7], [4, 2], [9, 0]], np.int32)
    oracle.copy_blocks(kc, vc, pairs)
    for b in range(10):
        src = {7: 1, 2: 4, 0: 9}.get(b, b)
        assert kc[b].tobytes() == k0[src].tobytes()
        assert vc[b].tobytes() == v0[src].tobytes()
    with pytest.raises(ValueError):
        oracle.copy_blocks(kc, vc, np.array([[0, 10]], np.int32))


# ---------------------------------------------------------------- closed forms
def _single_seq(K, V, block_size=16, dtype=np.float32):
    L, hkv, d = K.shape
    nb = -(-L // block_size) + 2
    tables, tarr = random_tables(np.random.default_rng(L), [L], block_size, nb)
    kc, vc = paged_pool([K], [V], tables, nb, block_size, dtype=dtype)
    return kc, vc, tarr


def test_identical_keys_give_mean_of_values():
    rng = np.random.default_rng(1)
    L, d = 37, 16
    K = np.repeat(rng.standard_normal((1, 1, d)).astype(np.float32), L, axis=0)
    V = rng.standard_normal((L, 1, d)).astype(np.float32)
    kc, vc, tarr = _single_seq(K, V)
    q = rng.standard_normal((1, 1, d)).astype(np.float32)
    out = oracle.decode(q, kc, vc, tarr, np.array([L], np.int32), 0.9)
    np.testing.assert_allclose(out[0, 0], V[:, 0].astype(np.float64).mean(0), rtol=1e-13, atol=1e-14)


@pytest.mark.parametrize("zero", ["q", "scale"])
def test_zero_query_or_scale_gives_mean_of_values(zero):
    rng = np.random.default_rng(2)
    L, d = 50, 16
    K = rng.standard_normal((L, 1, d)).astype(np.float32)
    V = rng.standard_normal((L, 1, d)).astype(np.float32)
    kc, vc, tarr = _single_seq(K, V)
    q = rng.standard_normal((1, 1, d)).astype(np.float32)
    if zero == "q":
        q[:] = 0
    out = oracle.decode(q, kc, vc, tarr, np.array([L], np.int32), 0.0 if zero == "scale" else 1.3)
    np.testing.assert_allclose(out[0, 0], V[:, 0].astype(np.float64).mean(0), rtol=1e-13, atol=1e-14)


def test_single_key_returns_its_value_exactly():
    rng = np.random.default_rng(4)
    K = rng.standard_normal((1, 2, 8)).astype(np.float32)
    V = rng.standard_normal((1, 2, 8)).astype(np.float32)
    kc, vc, tarr = _single_seq(K, V)
    q = rng.standard_normal((1, 4, 8)).astype(np.float32)
    out = oracle.decode(q, kc, vc, tarr, np.array([1], np.int32), 0.7)
    for h in range(4):
        assert np.array_equal(out[0, h], V[0, h // 2].astype(np.float64))


def test_dominant_key_returns_its_value():
    rng = np.random.default_rng(6)
    L, d, j = 45, 8, 29
    K = np.zeros((L, 1, d), np.float32)
    K[:, 0, 1:] = rng.standard_normal((L, d - 1))   # orthogonal to q
    K[j, 0, 0] = 40.0 / (0.5 * 2.0)                  # scale * <q, K_j> = 40
    V = rng.standard_normal((L, 1, d)).astype(np.float32)
    kc, vc, tarr = _single_seq(K, V)
    q = np.zeros((1, 1, d), np.float32)
    q[0, 0, 0] = 2.0
    out = oracle.decode(q, kc, vc, tarr, np.array([L], np.int32), 0.5)
    bound = math.exp(-40) * (L - 1) * np.abs(V).max() * 2
    assert np.abs(out[0, 0] - V[j, 0]).max() <= bound
    assert not np.array_equal(out[0, 0], V[j, 0].astype(np.float64))  # the others still count


def test_huge_scores_two_keys_follow_the_logistic_closed_form():
    """Two keys with scores near 1000 (exp would overflow without the max shift):
    softmax over two scores is the logistic function of their difference."""
    rng = np.random.default_rng(10)
    d, scale, c = 4, 0.5, 2.0
    K = np.zeros((2, 1, d), np.float32)
    K[0, 0, 0] = 1000.0 / (scale * c)
    K[1, 0, 0] = (1000.0 - math.log(3.0)) / (scale * c)
    V = rng.standard_normal((2, 1, d)).astype(np.float32)
    kc, vc, tarr = _single_seq(K, V)
    q = np.zeros((1, 1, d), np.float32)
    q[0, 0, 0] = c
    out = oracle.decode(q, kc, vc, tarr, np.array([2], np.int32), scale)
    delta = scale * c * (float(K[0, 0, 0]) - float(K[1, 0, 0]))
    w0 = 1.0 / (1.0 + math.exp(-delta))
    want = w0 * V[0, 0].astype(np.float64) + (1 - w0) * V[1, 0].astype(np.float64)
    assert abs(w0 - 0.75) < 1e-4
    np.testing.assert_allclose(out[0, 0], want, rtol=0, atol=1e-12)


def test_empty_context_gives_zero():
    rng = np.random.default_rng(8)
    dk, dv, tables, tarr, kc, vc, q = tiny_case(rng, [0, 5], 2, 2, 8, 16, np.float32)
    out = oracle.decode(q, kc, vc, tarr, np.array([0, 5], np.int32), 1.0)
    assert np.array_equal(out[0], np.zeros((2, 8)))


# ---------------------------------------------------------------- invariants
@pytest.mark.parametrize("dtype", [np.float32, np.uint16])
def test_physical_block_permutation_is_invisible(dtype):
    rng = np.random.default_rng(12)
    lens = [3, 40, 77, 16]
    dk, dv, tables, tarr, kc, vc, q = tiny_case(rng, lens, 4, 2, 16, 16, dtype)
    lens_a = np.array(lens, np.int32)
    out1 = oracle.decode(q, kc, vc, tarr, lens_a, 0.25)
    perm = rng.permutation(kc.shape[0])            # new position of block b is perm[b]
    kc2, vc2 = np.empty_like(kc), np.empty_like(vc)
    kc2[perm], vc2[perm] = kc, vc
    tarr2 = np.where(tarr >= 0, perm[np.maximum(tarr, 0)], -1).astype(np.int32)
    out2 = oracle.decode(q, kc2, vc2, tarr2, lens_a, 0.25)
    assert np.array_equal(out1, out2)


def test_shared_prefix_equals_private_copies():
    rng = np.random.default_rng(13)
    B, hkv, d, prefix = 16, 2, 8, 48
    pk = rng.standard_normal((prefix, hkv, d)).astype(np.float32)
    pv = rng.standard_normal((prefix, hkv, d)).astype(np.float32)
    suf = [rng.standard_normal((n, hkv, d)).astype(np.float32) for n in (5, 21)]
    sufv = [rng.standard_normal((n, hkv, d)).astype(np.float32) for n in (5, 21)]
    dk = [np.concatenate([pk, s]) for s in suf]
    dv = [np.concatenate([pv, s]) for s in sufv]
    lens = np.array([x.shape[0] for x in dk], np.int32)
    q = rng.standard_normal((2, 4, d)).astype(np.float32)
    # private: every block distinct
    _, tp = random_tables(rng, list(lens), B, 20)
    tables_p = [[int(b) for b in row if b >= 0] for row in tp]
    kcp, vcp = paged_pool(dk, dv, tables_p, 20, B)
    # shared: both sequences point at blocks 0..2 for the prefix
    tables_s = [[0, 1, 2, 3], [0, 1, 2, 4, 5]]
    kcs, vcs = paged_pool(dk, dv, tables_s, 20, B)
    ts = np.full((2, 5), -1, np.int32)
    ts[0, :4], ts[1, :5] = tables_s[0], tables_s[1]
    assert np.array_equal(oracle.decode(q, kcp, vcp, tp, lens, 0.3), oracle.decode(q, kcs, vcs, ts, lens, 0.3))


def test_gqa_equals_repeat_interleaved_mha():
    rng = np.random.default_rng(14)
    lens, hq, hkv, d = [10, 37], 6, 2, 8
    dk, dv, tables, tarr, kc, vc, q = tiny_case(rng, lens, hq, hkv, d, 16, np.float32)
    g = hq // hkv
    kc_m = np.repeat(kc, g, axis=1)   # kv head j becomes heads j*g .. j*g+g-1
    vc_m = np.repeat(vc, g, axis=1)
    la = np.array(lens, np.int32)
    assert np.array_equal(oracle.decode(q, kc, vc, tarr, la, 0.4), oracle.decode(q, kc_m, vc_m, tarr, la, 0.4))


def test_prefill_rows_equal_decode_at_the_same_length():
    rng = np.random.default_rng(15)
    lens, hq, hkv, d = [25, 40], 4, 2, 8
    dk, dv, tables, tarr, kc, vc, _ = tiny_case(rng, lens, hq, hkv, d, 16, np.float32)
    C = 5
    q = rng.standard_normal((2, C, hq, d)).astype(np.float32)
    la = np.array(lens, np.int32)
    pre = oracle.prefill(q, kc, vc, tarr, la, np.array([C, C], np.int32), 0.6)
    for i in range(C):   # row i sees the context truncated to L - C + i + 1
        dec = oracle.decode(np.ascontiguousarray(q[:, i]), kc, vc, tarr, la - C + i + 1, 0.6)
        assert np.array_equal(pre[:, i], dec)
    one = oracle.prefill(np.ascontiguousarray(q[:, :1]), kc, vc, tarr, la, np.array([1, 1], np.int32), 0.6)
    assert np.array_equal(one[:, 0], oracle.decode(np.ascontiguousarray(q[:, 0]), kc, vc, tarr, la, 0.6))


def test_thread_count_does_not_change_results():
    rng = np.random.default_rng(16)
    dk, dv, tables, tarr, kc, vc, q = tiny_case(rng, [30, 60, 90], 4, 4, 16, 16, np.float32)
    la = np.array([30, 60, 90], np.int32)
    n0 = oracle.num_threads()
    try:
        oracle.set_num_threads(1)
        a = oracle.decode(q, kc, vc, tarr, la, 0.2)
        oracle.set_num_threads(max(2, n0))
        b = oracle.decode(q, kc, vc, tarr, la, 0.2)
    finally:
        oracle.set_num_threads(n0)
    assert np.array_equal(a, b)


def test_bad_table_entry_is_reported():
    rng = np.random.default_rng(17)
    dk, dv, tables, tarr, kc, vc, q = tiny_case(rng, [20], 1, 1, 8, 16, np.float32)
    tarr = tarr.copy()
    tarr[0, 1] = kc.shape[0]
    with pytest.raises(ValueError):
        oracle.decode(q, kc, vc, tarr, np.array([20], np.int32), 1.0)


def test_block_model_replay_feeds_the_oracle_like_the_page_layout():
    """Replaying a workload through the Python block model and oracle.cache_write
    yields the same pool as scattering with numpy indexing through the model's tables."""
    import workloads
    wl = workloads.make(3, mini=True)
    mgr = BlockManagerModel(wl.num_blocks, wl.block_size, wl.free_order.tolist())
    kc = np.full(wl.cache_shape(), 0x7FC0, wl.np_dtype)   # bf16 NaN where nothing is written
    vc = kc.copy()
    workloads.replay(wl, mgr, lambda k, v, s: oracle.cache_write(k, v, s, kc, vc))
    # rebuild each live sequence's dense K from the op list (children share the prefix)
    dense = {}
    for op in wl.ops:
        if op[0] == "add":
            dense[op[1]] = ([], [])
        elif op[0] == "append":
            dense[op[1]][0].append(op[2]); dense[op[1]][1].append(op[3])
        elif op[0] == "fork":
            dense[op[2]] = (list(dense[op[1]][0]), list(dense[op[1]][1]))
        elif op[0] == "free":
            del dense[op[1]]
    seqs = sorted(dense)
    dk = [np.concatenate(dense[s][0]) for s in seqs]
    dv = [np.concatenate(dense[s][1]) for s in seqs]
    tables = [mgr.block_table(s) for s in seqs]
    want_k, want_v = paged_pool(dk, dv, tables, wl.num_blocks, wl.block_size, dtype=np.uint16)
    used = sorted({b for t in tables for b in t})
    assert kc[used].tobytes() == want_k[used].tobytes()
    assert vc[used].tobytes() == want_v[used].tobytes()
