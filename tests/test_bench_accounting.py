"""The benchmark's algorithmic byte counts (the roofline numerators) against hand
counts on a tiny shared-prefix case: unique bytes count each (physical block, slot)
once, logical bytes count per sequence, fp8 pools count one byte per cached element
while queries and outputs stay bf16."""
import types

import numpy as np

import bench


def tiny_wl(elem=2):
    return types.SimpleNamespace(num_kv_heads=2, num_q_heads=4, head_dim=8, elem_bytes=elem)


def test_unique_and_logical_bytes_by_hand():
    wl = tiny_wl()
    # two sequences share physical blocks 7 and 3 (32 tokens); seq 0 then uses block 5
    # for 4 more tokens, seq 1 uses block 9 for 20 tokens (block 9 full + block 2 with 4)
    tables = np.array([[7, 3, 5, -1], [7, 3, 9, 2]], np.int32)
    lens = np.array([36, 52], np.int32)
    row = 2 * 8 * 2 * 2                  # K + V of one token over both kv heads, bf16
    qo = 2 * 4 * 8 * 2 * 2               # q in and out, 2 sequences, 4 heads, bf16
    unique, logical = bench.step_bytes(wl, tables, lens)
    # block 7: 16, block 3: 16, block 5: 4, block 9: 16, block 2: 4 tokens
    assert unique == (16 + 16 + 4 + 16 + 4) * row + qo
    assert logical == (36 + 52) * row + qo


def test_shared_partial_block_counts_its_longest_use():
    wl = tiny_wl()
    tables = np.array([[4], [4]], np.int32)
    lens = np.array([5, 11], np.int32)   # both read block 4: 11 slots are touched
    unique, logical = bench.step_bytes(wl, tables, lens)
    row, qo = 2 * 8 * 2 * 2, 2 * 4 * 8 * 2 * 2
    assert unique == 11 * row + qo and logical == 16 * row + qo


def test_fp8_pools_count_one_byte_per_cached_element():
    wl = tiny_wl()
    tables = np.array([[1, 2]], np.int32)
    lens = np.array([20], np.int32)
    u16, _ = bench.step_bytes(wl, tables, lens)
    u8, _ = bench.step_bytes(wl, tables, lens, kv_elem=1)
    qo = 1 * 4 * 8 * 2 * 2
    assert u16 - qo == 2 * (u8 - qo)     # K/V halve, q/out do not
    # cache write: bf16 read, e4m3 written
    assert bench.cache_write_bytes(wl, 3) == 3 * 2 * 8 * 2 * (2 + 2)
    assert bench.cache_write_bytes(wl, 3, kv_elem=1) == 3 * 2 * 8 * 2 * (2 + 1)


def _record():
    import json
    return json.load(open(bench.TRAFFIC_RECORD))


def test_traffic_record_is_self_consistent():
    """The committed DRAM-traffic record: one entry per kernel of the call, summing to
    the call's total, and hashes for every kernel source the bench checks."""
    rec = _record()
    assert sum(rec["per_kernel_bytes"].values()) == rec["dram_bytes_per_call"]
    assert len(rec["per_kernel_bytes"]) == 5
    assert set(rec["sources_sha256"]) == set(bench.kernel_sources_sha256())


def test_traffic_is_dropped_once_a_kernel_source_changes(monkeypatch):
    """A record taken for other kernel sources is not reported (traffic null)."""
    cur = bench.kernel_sources_sha256()
    changed = dict(cur, **{"decode.cu": "0" * 64})
    monkeypatch.setattr(bench, "kernel_sources_sha256", lambda: changed)
    assert bench.recorded_traffic() is None


def test_traffic_is_reported_for_the_sources_it_was_taken_on():
    rec = _record()
    if rec["sources_sha256"] != bench.kernel_sources_sha256():
        import pytest
        pytest.skip("kernel sources changed since the capture: the bench reports traffic null")
    assert bench.recorded_traffic() == rec["dram_bytes_per_call"]
