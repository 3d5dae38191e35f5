"""pa_decode_static_scratch: split-K decode that takes no workspace from the caller.

It serves callers that cannot allocate device memory (an allocator's own
callbacks, a framework that owns and caps the device memory, a plugin handed only
a step's tensors).  Its output must match pa_decode with a caller-owned workspace,
call after call, even though every call reuses the same in-library array.
Collected last on purpose: it must also pass after everything else has run.
"""
import ctypes as C

import numpy as np
import pytest

import workloads
from gpu_harness import TwoSided, as_f64, check_close, to_dev, to_host, torch_mod

pytestmark = pytest.mark.gpu


def _entry(pa):
    fn = pa._lib.pa_decode_static_scratch
    vp, i32 = C.c_void_p, C.c_int32
    fn.argtypes = [vp, vp, vp, vp, i32, vp, i32, i32, i32, C.c_float, i32, vp,
                   C.POINTER(pa.CacheDesc), vp, vp]
    fn.restype = C.c_int
    return fn


def _ptr(t):
    return C.c_void_p(t.data_ptr())


@pytest.mark.parametrize("cid,part", [(5, 256), (3, 64)])
def test_static_scratch_matches_caller_workspace(pa, cid, part):
    torch = torch_mod()
    fn = _entry(pa)
    wl = workloads.make(cid, mini=True)
    ts = TwoSided(wl)
    step = wl.steps[0]
    ts.append_step(step)
    t, l = ts.tables(step.seqs)
    td, ld = torch.from_numpy(t).cuda(), torch.from_numpy(l).cuda()
    maxc = int(l.max())
    g = ts.gpu
    desc = pa.cache_desc(g.key_cache)
    stream = torch.cuda.current_stream()
    rng = np.random.default_rng(77)
    n_ws = pa.pa_decode_workspace_size(len(step.seqs), wl.num_q_heads, wl.head_dim, maxc, part)
    assert 0 < n_ws <= (32 << 20)
    for call in range(2):   # two calls in a row: the array keeps the previous call's partials
        q_np = step.q if call == 0 else workloads.normal(rng, step.q.shape, "bf16")
        q = to_dev(q_np)
        want = torch.empty_like(q)
        ws = torch.empty(n_ws, dtype=torch.uint8, device="cuda")
        pa.pa_decode(q, g.key_cache, g.value_cache, td, ld, maxc, wl.scale, want, part, ws, g.err_flag)
        got = torch.full_like(q, float("nan"))
        st = fn(_ptr(q), _ptr(g.key_cache), _ptr(g.value_cache), _ptr(td), t.shape[1], _ptr(ld), maxc,
                len(step.seqs), wl.num_q_heads, wl.scale, part, _ptr(got), C.byref(desc),
                _ptr(g.err_flag), C.c_void_p(stream.cuda_stream))
        assert st == pa.PA_OK, pa.status_string(st)
        assert pa.pa_wait(g.err_flag) == 0
        check_close(to_host(got), as_f64(to_host(want)), "bf16", f"call {call}")


def test_static_scratch_rejects_requests_beyond_its_array(pa):
    """A request whose partials would not fit in the array is refused before any
    launch.  Every buffer is a real device allocation of the size the arguments
    declare, and every context is empty, so even if the size check ever regressed
    the launched kernels would stay inside these buffers (an fp32 pool takes no
    shared-prefix path and an empty context writes no partial)."""
    torch = torch_mod()
    fn = _entry(pa)
    S, hkv, d, maxc, part, mb = 4096, 8, 64, 2048, 16, 128
    need = pa.pa_decode_workspace_size(S, hkv, d, maxc, part)
    assert need > (32 << 20)                      # 4096 x 8 x 128 partitions x 264 B
    kc = torch.zeros((16, hkv, 16, d), dtype=torch.float32, device="cuda")
    vc = torch.zeros_like(kc)
    q = torch.zeros((S, hkv, d), dtype=torch.float32, device="cuda")
    out = torch.zeros_like(q)
    tables = torch.zeros((S, mb), dtype=torch.int32, device="cuda")
    lens = torch.zeros(S, dtype=torch.int32, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    desc = pa.cache_desc(kc)
    st = fn(_ptr(q), _ptr(kc), _ptr(vc), _ptr(tables), mb, _ptr(lens), maxc, S, hkv, 0.125, part,
            _ptr(out), C.byref(desc), _ptr(err), C.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == pa.PA_ERR_UNSUPPORTED
    torch.cuda.synchronize()
    assert int(err.item()) == 0
