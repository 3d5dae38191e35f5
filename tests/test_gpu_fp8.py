"""GPU parity of the FP8 (e4m3) KV cache against the oracle, through the C ABI.

Pages: chenxutan "vLLM 深度拆解" 5.3 (FP8 KV cache) and the devpress teardown's
architecture figure (FP8/INT8 quantisation in the kernel layer); the e4m3 reading
with one scale per pool is stated in include/pa.h.

Bit-exact: the e4m3 pools after every cache write and copy-on-write copy (the
quantisation is a deterministic rounding the oracle fixes).  Attention: bf16
output within 1.5e-2 + 1e-2 |ref| of the oracle's fp64 attention over the same codes.
"""
import numpy as np
import pytest

import oracle
import workloads
from gpu_harness import TwoSided, check_close, to_dev, to_host, torch_mod

pytestmark = pytest.mark.gpu

K_SCALE, V_SCALE = 6.0 / 448, 5.0 / 448     # |x| above 6 (K) / 5 (V) saturates


@pytest.fixture(autouse=True)
def _lib(pa):
    torch = torch_mod()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return pa


def test_cache_write_quantises_like_the_oracle(pa):
    """Random values, saturating ones, subnormal and zero results, exact ties of the
    e4m3 grid, padding slots; scales that are and are not powers of two."""
    torch = torch_mod()
    rng = np.random.default_rng(21)
    nb, hkv, d, T = 40, 4, 128, 300
    grid = oracle.e4m3_decode(np.arange(0x7F, dtype=np.uint8))
    ties = (grid[:-1] + grid[1:]) / 2                        # 5 significant bits: exact in bf16
    for ks, vs in ((0.25, 0.0625), (K_SCALE, V_SCALE)):
        x = rng.standard_normal((T, hkv, d)).astype(np.float32) * 3
        x.reshape(-1)[:4000:7] = rng.choice([1e4, -1e4, 1e-7, -1e-7, 0.0, 449 * ks], size=572)
        x.reshape(-1)[1:2 * len(ties):2] = (ties * ks).astype(np.float32)
        k = workloads.to_bf16_bits(x)
        v = workloads.to_bf16_bits(rng.standard_normal((T, hkv, d)).astype(np.float32) * 2)
        slots = rng.permutation(nb * 16)[:T].astype(np.int64)
        slots[::37] = -1
        kc = np.full((nb, hkv, 16, d), 0x7F, np.uint8)
        vc = kc.copy()
        oracle.cache_write_fp8(k, v, slots, kc, vc, ks, vs)
        gk = torch.full(kc.shape, 0x7F, dtype=torch.uint8, device="cuda").view(torch.float8_e4m3fn)
        gv = torch.full(kc.shape, 0x7F, dtype=torch.uint8, device="cuda").view(torch.float8_e4m3fn)
        err = torch.zeros(1, dtype=torch.int32, device="cuda")
        pa.pa_cache_write(to_dev(k), to_dev(v), torch.from_numpy(slots).cuda(), gk, gv, err,
                          k_scale=ks, v_scale=vs)
        assert to_host(gk).tobytes() == kc.tobytes()
        assert to_host(gv).tobytes() == vc.tobytes()
        assert pa.pa_wait(err) == 0


def run_fp8(cid, mini, parts, sample=None):
    wl = workloads.make(cid, mini=mini)
    ts = TwoSided(wl, (K_SCALE, V_SCALE))
    assert ts.pools_equal(), "fp8 cache write of the set-up tokens is not bit-exact"
    rng = np.random.default_rng(cid + 100)
    for i, step in enumerate(wl.steps):
        ts.append_step(step)
        if i in (0, 1, len(wl.steps) - 1):
            assert ts.pools_equal(), f"step {i}: fp8 pools differ after copy-on-write + cache write"
        S = len(step.seqs)
        rows = None if sample is None or S <= sample else np.sort(rng.choice(S, sample, replace=False))
        ref = ts.oracle_decode(step, rows)
        for part in parts:
            got = ts.gpu_decode(step, part)
            if rows is not None:
                got = got[rows]
            check_close(got, ref, "bf16", f"fp8 config {cid} step {i} partition {part}")
    assert ts.err_flag() == 0
    return ts


@pytest.mark.parametrize("cid", [2, 3, 4, 5])
def test_fp8_mini_workloads(cid):
    run_fp8(cid, True, (0, 256, 512))


def test_fp8_gqa_prefix_sharing_full_size():
    """The GQA-8B prefix-sharing decode at full size, in the launch configuration the
    benchmark times (512-token partitions), rows sampled."""
    run_fp8(3, False, (512,), sample=48)


def test_fp8_fork_copy_on_write():
    ts = run_fp8(4, True, (0, 256))
    assert ts.model.num_free() == ts.gpu.manager.num_free()


@pytest.mark.parametrize("g", [1, 2, 4, 8])
def test_fp8_sibling_families_match_oracle(g):
    """The sibling families of the bf16 grouping test on fp8 pools (no grouping:
    every sequence reads its shared blocks itself), at several partitions, against
    the oracle over the same codes."""
    from test_gpu_decode import _grouped_workload
    wl = _grouped_workload(g)
    ts = TwoSided(wl, (K_SCALE, V_SCALE))
    step = wl.steps[0]
    ts.append_step(step)
    assert ts.pools_equal()
    ref = ts.oracle_decode(step)
    for part in (0, 48, 256, 512, 1024):
        check_close(ts.gpu_decode(step, part), ref, "bf16", f"fp8 g{g} grouped decode partition {part}")
    assert ts.err_flag() == 0


def _custom(lens, hq, hkv, seed=5):
    rng = np.random.default_rng(seed)
    need = sum(-(-L // 16) for L in lens) + 4
    wl = workloads.Workload(0, "custom", "bf16", need, hq, hkv, 128, 1.0 / np.sqrt(128),
                            rng.permutation(need).astype(np.int32))
    for s, L in enumerate(lens):
        wl.ops.append(("add", s))
        if L:
            wl.ops.append(("append", s, workloads.normal(rng, (L, hkv, 128), "bf16"),
                           workloads.normal(rng, (L, hkv, 128), "bf16")))
    q = workloads.normal(rng, (len(lens), hq, 128), "bf16")
    wl.steps.append(workloads.Step(list(range(len(lens))), None, None, q))
    return wl


@pytest.mark.parametrize("g", [1, 2, 4, 8])
def test_fp8_edge_lengths(g):
    lens = [0, 1, 15, 16, 17, 31, 33, 255, 256, 257, 511, 512, 513, 1023, 1024, 1025, 2049, 3001]
    wl = _custom(lens, 2 * g, 2)
    ts = TwoSided(wl, (K_SCALE, V_SCALE))
    assert ts.pools_equal()
    step = wl.steps[0]
    ref = ts.oracle_decode(step)
    for part in (0, 16, 256, 512):
        got = ts.gpu_decode(step, part)
        assert np.array_equal(got[0], np.zeros_like(got[0])), "empty context must give 0"
        check_close(got, ref, "bf16", f"fp8 g{g} part {part}")
    assert ts.err_flag() == 0


def test_fp8_scales_are_applied():
    """Doubling k_scale doubles every score and doubling v_scale the output: the same
    codes give what the oracle gives with the new scales."""
    wl = _custom([40, 300, 129, 2000], 8, 2, seed=8)
    ts = TwoSided(wl, (K_SCALE, V_SCALE))
    step = wl.steps[0]
    for ks, vs in ((2 * K_SCALE, V_SCALE), (K_SCALE, 2 * V_SCALE), (0.5 * K_SCALE, 3 * V_SCALE)):
        ts.ks, ts.vs = ks, vs                     # same codes, other dequantisation scales
        ref = ts.oracle_decode(step)
        for part in (0, 256):
            check_close(ts.gpu_decode(step, part), ref, "bf16", f"scales {ks:.4g} {vs:.4g} part {part}")


@pytest.mark.parametrize("cid,part", [(3, 0), (3, 512), (4, 256)])
def test_fp8_append_decode_one_call(cid, part):
    wl = workloads.make(cid, mini=True)
    ts = TwoSided(wl, (K_SCALE, V_SCALE))
    for i, step in enumerate(wl.steps):
        got = ts.append_decode_step(step, part)
        assert ts.pools_equal(), f"step {i}: pools differ after the one-call write"
        check_close(got, ts.oracle_decode(step), "bf16", f"fp8 append+decode config {cid} step {i}")
    assert ts.err_flag() == 0


def test_fp8_matches_bf16_pool_within_quantisation_error():
    """Sanity of the whole reading: decode over the fp8 pool stays close to decode over
    the bf16 pool it was quantised from (the error of 3-bit mantissas, not a bug-sized
    one)."""
    wl = _custom([700, 1500, 64], 8, 2, seed=12)
    t8 = TwoSided(wl, (K_SCALE, V_SCALE))
    t16 = TwoSided(wl)
    step = wl.steps[0]
    a = np.asarray(workloads.bf16_bits_to_f32(t8.gpu_decode(step, 256)), np.float64)
    b = np.asarray(workloads.bf16_bits_to_f32(t16.gpu_decode(step, 256)), np.float64)
    assert np.abs(a - b).max() < 0.1 and np.abs(a - b).mean() < 0.02
