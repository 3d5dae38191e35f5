"""Pins of the oracle's FP8 (e4m3) KV-cache functions against things other than itself.

Pages: chenxutan "vLLM 深度拆解" 5.3 (FP8 KV cache: nearly lossless, half the bytes of
bf16) and the devpress teardown's architecture figure (FP8/INT8 quantisation in the
kernel layer).  The pages name no format; the reading is e4m3 (OCP 8-bit floating
point) with one float scale per pool: code = e4m3(fp32(x) / scale), value = e4m3 * scale.

* the codec against PyTorch's own float8_e4m3fn conversion (a library routine written
  from the same specification), code by code and on round-to-nearest-even ties;
* the values the format fixes: 448 the largest finite, 2^-6 the smallest normal, 2^-9
  the smallest subnormal, S.1111.111 NaN; saturation and underflow at the edges;
* the fp8 cache write against the page layout written with numpy indexing;
* the fp8 decode against pure-Python brute-force attention over the dequantised keys
  and values.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from workloads import to_bf16_bits, bf16_bits_to_f32

pytestmark = pytest.mark.usefixtures("oracle_lib")


def torch_e4m3_values(codes):
    return torch.from_numpy(np.asarray(codes, np.uint8)).view(torch.float8_e4m3fn).double().numpy()


def torch_e4m3_codes(x32):
    return torch.from_numpy(np.asarray(x32, np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def test_decode_table_matches_the_library_for_all_codes():
    codes = np.arange(256, dtype=np.uint8)
    got, want = oracle.e4m3_decode(codes), torch_e4m3_values(codes)
    assert np.array_equal(np.isnan(got), np.isnan(want))
    ok = ~np.isnan(want)
    assert np.array_equal(got[ok], want[ok])
    assert np.isnan(got).sum() == 2                     # only 0x7F and 0xFF


def test_values_the_format_fixes():
    v = oracle.e4m3_decode(np.array([0x7E, 0xFE, 0x08, 0x01, 0x07, 0x38, 0x3F, 0x40, 0x00, 0x80, 0x7F], np.uint8))
    assert v[0] == 448.0 and v[1] == -448.0
    assert v[2] == 2.0 ** -6                            # smallest normal
    assert v[3] == 2.0 ** -9                            # smallest subnormal
    assert v[4] == 7 * 2.0 ** -9                        # largest subnormal
    assert v[5] == 1.0 and v[6] == 1.875 and v[7] == 2.0
    assert v[8] == 0.0 and math.copysign(1.0, v[9]) == -1.0
    assert math.isnan(v[10])


def test_encode_matches_the_library_in_range_and_on_ties():
    rng = np.random.default_rng(3)
    x = np.concatenate([rng.standard_normal(20000) * s for s in (1e-3, 0.1, 1.0, 30.0, 200.0)])
    x = x[np.abs(x) <= 448].astype(np.float32)
    finite = oracle.e4m3_decode(np.arange(256, dtype=np.uint8))
    grid = np.unique(finite[~np.isnan(finite)])
    ties = ((grid[:-1] + grid[1:]) / 2).astype(np.float32)     # exact midpoints: ties to even
    assert np.array_equal(ties.astype(np.float64), (grid[:-1] + grid[1:]) / 2)
    for arr in (x, ties, -ties, grid.astype(np.float32)):
        assert np.array_equal(oracle.e4m3_encode(arr), torch_e4m3_codes(arr))


def test_encode_divides_by_the_scale_in_float32():
    rng = np.random.default_rng(4)
    x = (rng.standard_normal(5000) * 3).astype(np.float32)
    for scale in (0.0137, 0.5, 1.7):
        s32 = np.float32(scale)
        q = (x / s32).astype(np.float32)
        keep = np.abs(q) <= 448
        assert np.array_equal(oracle.e4m3_encode(x, scale)[keep], torch_e4m3_codes(q[keep]))


def test_saturation_underflow_and_nan():
    x = np.array([448, 460, 463.99, 464, 1e6, np.inf, -500, -np.inf, np.nan,
                  2.0 ** -10, 2.0 ** -11, -2.0 ** -10, 1.5 * 2.0 ** -9, 2.5 * 2.0 ** -9], np.float32)
    got = oracle.e4m3_encode(x).tolist()
    assert got[:8] == [0x7E, 0x7E, 0x7E, 0x7E, 0x7E, 0x7E, 0xFE, 0xFE]   # saturate to +-448
    assert got[8] in (0x7F, 0xFF)
    assert got[9] == 0x00 and got[10] == 0x00 and got[11] == 0x80      # half the smallest: to even 0
    assert got[12] == 0x02 and got[13] == 0x02                         # 1.5, 2.5 x 2^-9 -> 2 x 2^-9


def test_round_trip_of_every_finite_code():
    codes = np.arange(256, dtype=np.uint8)
    v = oracle.e4m3_decode(codes)
    ok = ~np.isnan(v)
    assert np.array_equal(oracle.e4m3_encode(v[ok].astype(np.float32)), codes[ok])


def test_cache_write_fp8_matches_page_layout():
    rng = np.random.default_rng(11)
    nb, hkv, B, d = 9, 2, 16, 8
    T = 40
    k = to_bf16_bits(rng.standard_normal((T, hkv, d)).astype(np.float32) * 4)
    v = to_bf16_bits(rng.standard_normal((T, hkv, d)).astype(np.float32))
    slots = rng.permutation(nb * B)[:T].astype(np.int64)
    slots[[3, 17]] = -1
    kc = np.full((nb, hkv, B, d), 0xAB, np.uint8)
    vc = kc.copy()
    ks, vs = 0.05, 0.013
    oracle.cache_write_fp8(k, v, slots, kc, vc, ks, vs)
    want_k = np.full_like(kc, 0xAB)
    want_v = want_k.copy()
    kq = torch_e4m3_codes(bf16_bits_to_f32(k) / np.float32(ks))
    vq = torch_e4m3_codes(bf16_bits_to_f32(v) / np.float32(vs))
    for t, s in enumerate(slots):
        if s >= 0:
            want_k[s // B, :, s % B, :] = kq[t]
            want_v[s // B, :, s % B, :] = vq[t]
    assert kc.tobytes() == want_k.tobytes() and vc.tobytes() == want_v.tobytes()
    with pytest.raises(IndexError):
        oracle.cache_write_fp8(k[:1], v[:1], np.array([nb * B], np.int64), kc, vc, ks, vs)


def brute_attention(q, K, V, scale):
    if len(K) == 0:
        return [0.0] * len(q)
    xs = [scale * math.fsum(a * b for a, b in zip(q, kk)) for kk in K]
    m = max(xs)
    ws = [math.exp(x - m) for x in xs]
    z = math.fsum(ws)
    return [math.fsum(w * vv[i] for w, vv in zip(ws, V)) / z for i in range(len(q))]


@pytest.mark.parametrize("ks,vs", [(0.02, 0.011), (0.25, 1.0)])
def test_decode_fp8_matches_brute_force(ks, vs):
    rng = np.random.default_rng(12)
    lens, hq, hkv, d, B = [0, 1, 17, 40], 4, 2, 8, 16
    nb = sum(-(-L // B) for L in lens) + 2
    perm = rng.permutation(nb)
    kc = rng.integers(0, 256, (nb, hkv, B, d), dtype=np.uint8)
    kc[(kc & 0x7F) == 0x7F] = 0x3C                      # no NaN codes
    vc = rng.integers(0, 256, (nb, hkv, B, d), dtype=np.uint8)
    vc[(vc & 0x7F) == 0x7F] = 0x44
    tables = np.full((len(lens), 3), -1, np.int32)
    i = 0
    for s, L in enumerate(lens):
        n = -(-L // B)
        tables[s, :n] = perm[i:i + n]
        i += n
    q = to_bf16_bits(rng.standard_normal((len(lens), hq, d)).astype(np.float32) * 0.1)
    scale = d ** -0.5
    got = oracle.decode_fp8(q, kc, vc, tables, np.array(lens, np.int32), scale, ks, vs)
    kval = torch_e4m3_values(kc) * float(np.float32(ks))
    vval = torch_e4m3_values(vc) * float(np.float32(vs))
    qf = bf16_bits_to_f32(q).astype(np.float64)
    g = hq // hkv
    for s, L in enumerate(lens):
        for h in range(hq):
            K = [kval[tables[s, t // B], h // g, t % B].tolist() for t in range(L)]
            V = [vval[tables[s, t // B], h // g, t % B].tolist() for t in range(L)]
            want = brute_attention(qf[s, h].tolist(), K, V, scale)
            assert np.allclose(got[s, h], want, rtol=1e-12, atol=1e-12 * max(1.0, np.abs(vval).max()))
