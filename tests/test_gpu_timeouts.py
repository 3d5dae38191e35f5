"""Failure handling on the GPU without a fault: waits that run out.

Host side: pa_wait on a stream that is still busy returns PA_ERR_TIMEOUT, and
returns PA_OK once the stream drains.  Device side: with the in-kernel wait bound
set to a few nanoseconds (pa_set_wait_timeout_ns), ordinary hand-over waits
between warps run out; the kernels set PA_DEVERR_TIMEOUT, drain what they have in
flight, free their tensor memory and return.  The context stays usable: with the
default bound restored, the same calls match the oracle again.  Every wait stays
bounded throughout and nothing traps.
"""
import ctypes as C

import numpy as np
import pytest

import oracle
import workloads
from gpu_harness import TwoSided, check_close, to_dev, to_host, torch_mod

pytestmark = pytest.mark.gpu


@pytest.fixture
def short_waits(pa):
    """Yields a function that shortens the bound; the default is restored afterwards."""
    prev = []

    def set_bound(ns):
        prev.append(pa.pa_set_wait_timeout_ns(ns))

    yield set_bound
    pa.pa_set_wait_timeout_ns(0)


def test_pa_wait_times_out_on_a_busy_stream(pa):
    torch = torch_mod()
    stream = torch.cuda.current_stream()
    flag = C.c_int32(-1)
    torch.cuda._sleep(int(4e8))                  # a bounded spin of a few hundred ms
    st = pa._lib.pa_wait(C.c_void_p(stream.cuda_stream), None, 1, C.byref(flag))
    assert st == pa.PA_ERR_TIMEOUT
    st = pa._lib.pa_wait(C.c_void_p(stream.cuda_stream), None, -1, C.byref(flag))
    assert st == pa.PA_OK and flag.value == 0


def test_set_wait_timeout_returns_the_previous_bound(pa):
    assert pa.pa_set_wait_timeout_ns(5000) == 1_000_000_000
    assert pa.pa_set_wait_timeout_ns(0) == 5000
    assert pa.pa_set_wait_timeout_ns(0) == 1_000_000_000


def test_decode_waits_run_out_then_recover(pa, short_waits):
    """Split decode with shared-prefix groups (3 groups of 4 siblings sharing a 64-token
    prefix, 64-token partitions): the tile kernel's stage hand-overs and the
    per-sequence kernel's merge hand-over."""
    wl = workloads.make(3, mini=True)
    ts = TwoSided(wl)
    step = wl.steps[0]
    ts.append_step(step)
    assert ts.err_flag() == 0
    short_waits(1)
    seen = 0
    for _ in range(8):
        ts.gpu_decode(step, 64)
        f = ts.err_flag()          # pa_wait returned: every kernel of the call ended
        assert f & ~pa.PA_DEVERR_TIMEOUT == 0, f
        seen |= f
        ts.clear_err()
        if seen:
            break
    assert seen & pa.PA_DEVERR_TIMEOUT, "no wait ran out with a 1 ns bound"
    pa.pa_set_wait_timeout_ns(0)
    ref = ts.oracle_decode(step, None)
    for part in (0, 64):
        check_close(ts.gpu_decode(step, part), ref, wl.dtype, f"after recovery, partition {part}")
    assert ts.err_flag() == 0


def test_prefill_waits_run_out_then_recover(pa, short_waits):
    wl = workloads.make(5, mini=True)
    ts = TwoSided(wl)
    pf = wl.prefill
    t, l = ts.tables(pf.seqs)
    torch = torch_mod()
    ch = np.array([pf.chunk] * len(pf.seqs), np.int32)

    def run():
        q = to_dev(pf.q)
        out = torch.zeros_like(q)
        pa.pa_prefill_chunk(q, ts.gpu.key_cache, ts.gpu.value_cache, torch.from_numpy(t).cuda(),
                            torch.from_numpy(l).cuda(), torch.from_numpy(ch).cuda(), wl.scale, out,
                            ts.gpu.err_flag)
        return to_host(out)

    short_waits(1)
    seen = 0
    for _ in range(8):
        run()
        f = ts.err_flag()
        assert f & ~pa.PA_DEVERR_TIMEOUT == 0, f
        seen |= f
        ts.clear_err()
        if seen:
            break
    assert seen & pa.PA_DEVERR_TIMEOUT, "no wait ran out with a 1 ns bound"
    pa.pa_set_wait_timeout_ns(0)
    ref = oracle.prefill(pf.q, ts.kc, ts.vc, t, l, ch, wl.scale)
    check_close(run(), ref, "bf16", "prefill after recovery")
    assert ts.err_flag() == 0
