"""Runs one workload on both sides -- the CUDA library (through its C ABI) and the
CPU oracle -- from the same seeded inputs, and exposes what tests compare.

Oracle side: Python block model + oracle.cache_write / copy_blocks / decode.
CUDA side: host C++ BlockManager + pa_cache_write / pa_copy_blocks / pa_decode.
No oracle input or expected value ever comes from the CUDA side.
"""
from __future__ import annotations

import numpy as np

import oracle
import workloads
from oracle.block_model import BlockManagerModel

# Tolerances: the pages fix no precision; these are the stated targets.
F32_ABS = 1e-5                     # fp32 inputs: max |gpu - oracle|
BF16_ABS, BF16_REL = 1.5e-2, 1e-2  # bf16 inputs: |gpu - oracle| <= ABS + REL * |oracle|
BF16_NAN = 0x7FC0


def torch_mod():
    import torch
    return torch


def to_dev(a):
    torch = torch_mod()
    if a.dtype == np.uint16:
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda().view(torch.bfloat16)
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def to_host(t):
    torch = torch_mod()
    if t.dtype == torch.float8_e4m3fn:
        return t.contiguous().view(torch.uint8).cpu().numpy()
    if t.dtype == torch.bfloat16:
        return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)
    return t.contiguous().cpu().numpy()


def as_f64(a):
    if a.dtype == np.uint16:
        return workloads.bf16_bits_to_f32(a).astype(np.float64)
    return a.astype(np.float64)


def check_close(got, ref, dtype: str, what: str = ""):
    """Element-wise tolerance check; returns (max_abs, max_rel over |ref| > 1e-3)."""
    g = as_f64(got)
    assert g.shape == ref.shape, (g.shape, ref.shape)
    assert np.isfinite(g).all(), f"{what}: non-finite output"
    err = np.abs(g - ref)
    big = np.abs(ref) > 1e-3
    max_rel = float((err[big] / np.abs(ref[big])).max()) if big.any() else 0.0
    if dtype == "f32":
        assert err.max() <= F32_ABS, f"{what}: max abs {err.max():.3g} > {F32_ABS}"
    else:
        bound = BF16_ABS + BF16_REL * np.abs(ref)
        bad = err > bound
        assert not bad.any(), (f"{what}: {bad.sum()} elements out of tolerance, "
                               f"worst {err.max():.3g} (max_rel {max_rel:.3g})")
    return float(err.max()), max_rel


class TwoSided:
    """A workload set up on the oracle and on the GPU, stepped in lockstep."""

    def __init__(self, wl: workloads.Workload, fp8_scales=None):
        """fp8_scales = (k_scale, v_scale): a bf16 workload stored in e4m3 pools."""
        torch = torch_mod()
        import paged_kv_cache_389_b200 as pa
        from paged_kv_cache_389_b200.cache import PagedKVCache
        self.pa, self.wl = pa, wl
        self.fp8 = fp8_scales is not None
        ks, vs = fp8_scales if self.fp8 else (1.0, 1.0)
        self.ks, self.vs = ks, vs
        # oracle side
        self.model = BlockManagerModel(wl.num_blocks, wl.block_size, wl.free_order.tolist())
        if self.fp8:
            assert wl.dtype == "bf16"
            self.kc = np.full(wl.cache_shape(), 0x7F, np.uint8)     # e4m3 NaN
            self.vc = self.kc.copy()
        else:
            fill = BF16_NAN if wl.dtype == "bf16" else np.nan
            self.kc = np.full(wl.cache_shape(), fill, wl.np_dtype)
            self.vc = np.full(wl.cache_shape(), fill, wl.np_dtype)
        workloads.replay(wl, self.model, self._oracle_write)
        # GPU side
        tdt = torch.float8_e4m3fn if self.fp8 else torch.bfloat16 if wl.dtype == "bf16" else torch.float32
        self.gpu = PagedKVCache(wl.num_blocks, wl.num_kv_heads, wl.head_dim, tdt, "cuda", wl.free_order,
                                k_scale=ks, v_scale=vs)
        g = self.gpu

        def write(k, v, slots):
            pa.pa_cache_write(to_dev(k), to_dev(v), torch.from_numpy(slots).cuda(), g.key_cache,
                              g.value_cache, g.err_flag, k_scale=ks, v_scale=vs)
        workloads.replay(wl, g.manager, write)
        self.step_index = 0
        self.last_pairs = np.zeros((0, 2), np.int32)

    def _oracle_write(self, k, v, slots):
        if self.fp8:
            oracle.cache_write_fp8(k, v, slots, self.kc, self.vc, self.ks, self.vs)
        else:
            oracle.cache_write(k, v, slots, self.kc, self.vc)

    # -- comparisons -------------------------------------------------------
    def pools_equal(self):
        return (to_host(self.gpu.key_cache).tobytes() == self.kc.tobytes()
                and to_host(self.gpu.value_cache).tobytes() == self.vc.tobytes())

    def err_flag(self):
        return self.pa.pa_wait(self.gpu.err_flag)

    def clear_err(self):
        self.gpu.err_flag.zero_()

    def tables(self, seqs):
        mb = max(1, max(len(self.model.block_table(s)) for s in seqs))
        t_o, l_o = self.model.build_tables(seqs, mb)
        t_g, l_g = self.gpu.manager.build_tables(seqs, mb)
        assert np.array_equal(t_o, t_g) and np.array_equal(l_o, l_g), "block tables differ"
        return t_o, l_o

    # -- one decode step on both sides -------------------------------------
    def append_step(self, step):
        """Copy-on-write + cache write of the step's new tokens on both sides."""
        torch = torch_mod()
        pa = self.pa
        if step.k_new is None:
            return
        slots_o, pairs_o = [], []
        for s in step.seqs:
            sl, pr = self.model.append_slot(s)
            slots_o.append(sl)
            if pr is not None:
                pairs_o.append(pr)
        slots_g, pairs_g = self.gpu.plan_append(step.seqs)
        assert slots_g.tolist() == slots_o and [tuple(p) for p in pairs_g.tolist()] == pairs_o
        if pairs_o:
            oracle.copy_blocks(self.kc, self.vc, np.array(pairs_o, np.int32))
            pa.pa_copy_blocks(self.gpu.key_cache, self.gpu.value_cache,
                              torch.from_numpy(pairs_g).cuda(), self.gpu.err_flag)
        sl = np.array(slots_o, np.int64)
        self._oracle_write(step.k_new, step.v_new, sl)
        pa.pa_cache_write(to_dev(step.k_new), to_dev(step.v_new), torch.from_numpy(sl).cuda(),
                          self.gpu.key_cache, self.gpu.value_cache, self.gpu.err_flag,
                          k_scale=self.ks, v_scale=self.vs)
        self.last_pairs = np.array(pairs_o, np.int32).reshape(-1, 2)

    def append_decode_step(self, step, partition_size=0):
        """The step's copy-on-write and cache write on both sides, then the GPU side's
        write + decode as one pa_append_decode call.  Returns the GPU output."""
        torch = torch_mod()
        pa = self.pa
        slots_o, pairs_o = [], []
        for s in step.seqs:
            sl, pr = self.model.append_slot(s)
            slots_o.append(sl)
            if pr is not None:
                pairs_o.append(pr)
        slots_g, pairs_g = self.gpu.plan_append(step.seqs)
        assert slots_g.tolist() == slots_o and [tuple(p) for p in pairs_g.tolist()] == pairs_o
        if pairs_o:
            oracle.copy_blocks(self.kc, self.vc, np.array(pairs_o, np.int32))
            pa.pa_copy_blocks(self.gpu.key_cache, self.gpu.value_cache,
                              torch.from_numpy(pairs_g).cuda(), self.gpu.err_flag)
        sl = np.array(slots_o, np.int64)
        self._oracle_write(step.k_new, step.v_new, sl)
        t, l = self.tables(step.seqs)
        q = to_dev(step.q)
        out = torch.empty_like(q)
        maxc = max(int(l.max(initial=1)), 1)
        ws = None
        if partition_size:
            n = pa.pa_decode_workspace_size(len(step.seqs), q.shape[1], q.shape[2], maxc, partition_size)
            ws = torch.empty(max(n, 16), dtype=torch.uint8, device="cuda")
        pa.pa_append_decode(to_dev(step.k_new), to_dev(step.v_new), torch.from_numpy(sl).cuda(), q,
                            self.gpu.key_cache, self.gpu.value_cache, torch.from_numpy(t).cuda(),
                            torch.from_numpy(l).cuda(), maxc, self.wl.scale, out, partition_size, ws,
                            self.gpu.err_flag, k_scale=self.ks, v_scale=self.vs)
        self.last_pairs = np.array(pairs_o, np.int32).reshape(-1, 2)
        return to_host(out)

    def gpu_decode(self, step, partition_size=0, tables=None, lens=None, max_context=None):
        torch = torch_mod()
        t, l = self.tables(step.seqs) if tables is None else (tables, lens)
        q = to_dev(step.q)
        out = torch.empty_like(q)
        maxc = int(l.max(initial=1)) if max_context is None else max_context
        maxc = max(maxc, 1)
        ws = None
        if partition_size:
            n = self.pa.pa_decode_workspace_size(len(step.seqs), q.shape[1], q.shape[2], maxc, partition_size)
            ws = torch.empty(max(n, 16), dtype=torch.uint8, device="cuda")
        self.pa.pa_decode(q, self.gpu.key_cache, self.gpu.value_cache, torch.from_numpy(t).cuda(),
                          torch.from_numpy(l).cuda(), maxc, self.wl.scale, out, partition_size, ws,
                          self.gpu.err_flag, k_scale=self.ks, v_scale=self.vs)
        return to_host(out)

    def oracle_decode(self, step, rows=None, tables=None, lens=None):
        t, l = self.tables(step.seqs) if tables is None else (tables, lens)
        if rows is not None:
            rows = np.asarray(rows)
            q, t, l = (np.ascontiguousarray(step.q[rows]), np.ascontiguousarray(t[rows]),
                       np.ascontiguousarray(l[rows]))
        else:
            q = step.q
        if self.fp8:
            return oracle.decode_fp8(q, self.kc, self.vc, t, l, self.wl.scale, self.ks, self.vs)
        return oracle.decode(q, self.kc, self.vc, t, l, self.wl.scale)
