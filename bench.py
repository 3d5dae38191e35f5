"""Paged-decode benchmark: KV GB/s and sequence-steps/s on B200, % of HBM roofline.

Workload (default): Llama-3-8B-shaped GQA decode with prefix sharing, bf16 -- 256
sequences in 16 groups of 16 sharing a 512-token prefix (32 shared blocks), private
lognormal suffixes (median 600, cap 8192), 32 query / 8 kv heads, head_dim 128,
block_size 16.  One step = the whole decode hot path for one batch: the 256 new
tokens' K/V written through their slot mapping, then decode attention over every
sequence (split-K partitions of 512 tokens; sibling runs that share whole
partitions read them once as a group; LSE reduce) -- one pa_append_decode call.
The same step as two calls (pa_cache_write, pa_decode) is timed as well.

Timed region: K steps after W warm-up steps, CUDA events on the launching stream,
barrier + synchronize on both sides, max over ranks.  The step's inputs (1.1 GB of
KV) are larger than L2 (126 MB), so no flush is needed between steps.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

N > 1 runs under torchrun: every rank holds its own copy of the workload on its GPU
(the path shards by sequence with no exchange) -> weak scaling; `value` is the
total over ranks.  `--impl reference` times the CPU oracle on the host cores on a
bounded sample of the same workload (rank 0 only).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads  # noqa: E402

PARTITION = 512
CONFIG_ID = 3
# FP8 pools: one scale per pool, amax / 448 with amax = 6 (K) and 5 (V) for the
# synthetic N(0, 1) keys and values
FP8_SCALES = (6.0 / 448, 5.0 / 448)
WORKLOAD_NAME = "llama3-8b-gqa-prefix-sharing-decode"


def log(*a):
    print(*a, file=sys.stderr, flush=True)


# ----------------------------------------------------------------- accounting
def step_bytes(wl, tables, lens, kv_elem=None):
    """Algorithmic bytes of one decode launch: K+V of every token attended, q in,
    out written.  'unique' counts each (physical block, token slot) once -- the
    HBM floor when siblings share prefix blocks; 'logical' counts per sequence.
    kv_elem: bytes per cached element (1 for an fp8 pool; default the workload's)."""
    e = wl.elem_bytes
    row = wl.num_kv_heads * wl.head_dim * (kv_elem or e) * 2   # K + V of one token, all kv heads
    qo = len(lens) * wl.num_q_heads * wl.head_dim * e * 2
    used = {}
    for s, L in enumerate(lens):
        for j in range(-(-int(L) // 16)):
            b = int(tables[s, j])
            used[b] = max(used.get(b, 0), min(16, int(L) - 16 * j))
    unique = sum(used.values()) * row + qo
    logical = int(np.sum(lens)) * row + qo
    return unique, logical


def cache_write_bytes(wl, ntok, kv_elem=None):
    # K,V read (workload dtype) + written (pool dtype)
    return ntok * wl.num_kv_heads * wl.head_dim * 2 * (wl.elem_bytes + (kv_elem or wl.elem_bytes))


# ----------------------------------------------------------------- clocks
class ClockSampler:
    """NVML polling of SM clock and clock-event reasons in a background thread."""
    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x2: "applications_clocks_setting", 0x1: "gpu_idle", 0x10: "sync_boost"}

    def __init__(self, torch, device, period_s=0.005):
        self.samples, self.period, self.ok = [], period_s, False
        try:
            import pynvml as nv
            nv.nvmlInit()
            self.nv = nv
            try:
                props = torch.cuda.get_device_properties(device)
                bus = "%08x:%02x:%02x.0" % (getattr(props, "pci_domain_id", 0), props.pci_bus_id,
                                            props.pci_device_id)
                self.h = nv.nvmlDeviceGetHandleByPciBusId(bus.encode())
            except Exception:
                self.h = nv.nvmlDeviceGetHandleByIndex(device)
            self.max_mhz = nv.nvmlDeviceGetMaxClockInfo(self.h, nv.NVML_CLOCK_SM)
            self.ok = True
        except Exception as ex:  # NVML missing: report no clocks rather than guess
            log("clock sampling unavailable:", ex)
        self._stop = threading.Event()
        self._t = None

    def _reasons(self):
        nv = self.nv
        f = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            nv.nvmlDeviceGetCurrentClocksThrottleReasons
        return int(f(self.h))

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append((time.perf_counter(),
                                     self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM),
                                     self._reasons()))
            except Exception:
                pass
            time.sleep(self.period)

    def start(self):
        if self.ok:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()

    def stop(self):
        self._stop.set()
        if self._t:
            self._t.join()

    def summary(self, t0, t1):
        if not self.ok:
            return None
        inside = [s for s in self.samples if t0 <= s[0] <= t1]
        window = "timed_region"
        if not inside:   # region shorter than the poll period: nearest samples around it
            inside = sorted(self.samples, key=lambda s: min(abs(s[0] - t0), abs(s[0] - t1)))[:2]
            window = "nearest_to_timed_region"
        bits = 0
        for s in inside:
            bits |= s[2]
        reasons = [n for b, n in self.REASONS.items() if bits & b and n != "gpu_idle"]
        return {"sm_mhz": float(np.median([s[1] for s in inside])) if inside else None,
                "sm_max_mhz": float(self.max_mhz), "reasons": reasons,
                "samples": len(inside), "window": window}


# ----------------------------------------------------------------- distributed
def dist_setup(n_gpus):
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    if n_gpus != world:
        log(f"note: --gpus {n_gpus} but WORLD_SIZE {world}; using WORLD_SIZE")
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x, world):
    if world == 1:
        return x
    from paged_kv_cache_389_b200.dist import max_over_ranks as _max
    return _max(x, device="cuda")


# ----------------------------------------------------------------- profiles
TRAFFIC_RECORD = os.path.join(ROOT, "profiles", "decode_gqa8b_prefix_traffic.json")


def kernel_sources_sha256():
    """sha256 of every kernel source that one pa_append_decode call runs."""
    out = {}
    for name in ("cache_ops.cu", "cache_write.cuh", "decode.cu", "prefill.cu", "pa_common.cuh"):
        src = os.path.join(ROOT, "paged_kv_cache_389_b200", "csrc", name)
        out[name] = hashlib.sha256(open(src, "rb").read()).hexdigest()
    return out


def recorded_traffic():
    """DRAM bytes (read + write) of one pa_append_decode call, all its kernels, from
    the committed ncu record -- or None if a kernel source changed since the counters
    were taken (the record stores the sources' sha256)."""
    if not os.path.exists(TRAFFIC_RECORD):
        return None
    rec = json.load(open(TRAFFIC_RECORD))
    if rec.get("sources_sha256") != kernel_sources_sha256():
        return None
    return int(rec["dram_bytes_per_call"])


def headline_config(wl, S, max_ctx, mean_ctx, part, world):
    """The `config` of the headline line, the same for both arms."""
    return {"workload": WORKLOAD_NAME, "num_seqs": S, "num_q_heads": wl.num_q_heads,
            "num_kv_heads": wl.num_kv_heads, "head_dim": wl.head_dim, "block_size": 16,
            "prefix_tokens": 512, "group_size": 16, "max_context": int(max_ctx),
            "mean_context": float(mean_ctx), "partition_size": int(part),
            "parallelism": f"dp{world} (sequences sharded, no exchange)",
            "l2": "inputs larger than L2 (126 MB); no flush"}


# ----------------------------------------------------------------- our arm
def run_ours(args):
    import torch
    world, rank, local = dist_setup(args.gpus)
    import paged_kv_cache_389_b200 as pa
    from paged_kv_cache_389_b200.cache import PagedKVCache

    t_setup = time.time()
    wl = workloads.make(CONFIG_ID)
    step = wl.steps[0]
    S = len(step.seqs)
    cache = PagedKVCache(wl.num_blocks, wl.num_kv_heads, wl.head_dim, torch.bfloat16, "cuda",
                         wl.free_order)
    dev = lambda a: torch.from_numpy(a.view(np.int16)).cuda().view(torch.bfloat16)
    workloads.replay(wl, cache.manager, lambda k, v, s: pa.pa_cache_write(
        dev(k), dev(v), torch.from_numpy(s).cuda(), cache.key_cache, cache.value_cache, cache.err_flag))
    slots, pairs = cache.plan_append(step.seqs)
    assert len(pairs) == 0
    max_blocks = cache.manager.max_seq_blocks(step.seqs)
    tables_h, lens_h = cache.manager.build_tables(step.seqs, max_blocks)
    max_ctx = int(lens_h.max())
    # device-resident step inputs
    q = dev(step.q)
    k_new, v_new = dev(step.k_new), dev(step.v_new)
    slots_d = torch.from_numpy(slots).cuda()
    tables_d = torch.from_numpy(tables_h).cuda()
    lens_d = torch.from_numpy(lens_h).cuda()
    out = torch.empty_like(q)
    part = args.partition
    ws_n = pa.pa_decode_workspace_size(S, wl.num_q_heads, wl.head_dim, max_ctx, part)
    ws = torch.empty(max(ws_n, 16), dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream()
    unique_b, logical_b = step_bytes(wl, tables_h, lens_h)
    cw_b = cache_write_bytes(wl, S)
    log(f"rank {rank}: setup {time.time() - t_setup:.1f}s; {S} seqs, max ctx {max_ctx}, "
        f"unique {unique_b / 1e9:.3f} GB, logical {logical_b / 1e9:.3f} GB")

    # one step = write the new tokens' K/V, then decode every sequence: one
    # pa_append_decode call (the write and the decode kernels chained)
    def step_fn(ev_a=None, ev_b=None):
        if ev_a is not None:
            ev_a.record(stream)
        pa.pa_append_decode(k_new, v_new, slots_d, q, cache.key_cache, cache.value_cache, tables_d, lens_d,
                            max_ctx, wl.scale, out, part, ws, cache.err_flag, stream)
        if ev_b is not None:
            ev_b.record(stream)

    # the same step as two calls, pa_cache_write then pa_decode (the decode bracketed)
    def two_calls_fn(ev_a=None, ev_b=None):
        pa.pa_cache_write(k_new, v_new, slots_d, cache.key_cache, cache.value_cache, cache.err_flag, stream)
        if ev_a is not None:
            ev_a.record(stream)
        pa.pa_decode(q, cache.key_cache, cache.value_cache, tables_d, lens_d, max_ctx, wl.scale, out,
                     part, ws, cache.err_flag, stream)
        if ev_b is not None:
            ev_b.record(stream)

    for _ in range(args.warmup):
        step_fn()
    torch.cuda.synchronize()
    flag = pa.pa_wait(cache.err_flag)
    assert flag == 0, f"device error flag {flag} during warm-up"

    K = args.steps
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(torch, local)
    sampler.start()
    barrier(world)
    torch.cuda.synchronize()
    h0 = time.perf_counter()
    e0.record(stream)
    for i in range(K):
        step_fn()
    e1.record(stream)
    torch.cuda.synchronize()
    h1 = time.perf_counter()
    barrier(world)
    sampler.stop()
    ms = e0.elapsed_time(e1)
    # one call per step, back to back: its average duration over the timed region
    call_ms = ms / K
    ms_max = max_over_ranks(ms, world)
    clocks = sampler.summary(h0, h1)

    # the same step as two calls, for comparison: whole step and the decode call alone
    for _ in range(3):
        two_calls_fn()
    nf = min(K, 500)
    ev2 = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(nf)]
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    f0.record(stream)
    for i in range(nf):
        two_calls_fn(*ev2[i])
    f1.record(stream)
    torch.cuda.synchronize()
    two_ms = max_over_ranks(f0.elapsed_time(f1) / nf, world)
    dec_ms = float(np.mean([a.elapsed_time(b) for a, b in ev2]))
    assert pa.pa_wait(cache.err_flag) == 0

    # end to end: every step's inputs from pinned host memory (query, new K/V, slots,
    # lengths; the block tables only when they change -- here once), the step, and the
    # output read back to pinned host memory.  Host-to-device and device-to-host copies
    # run on two streams of their own into two device buffer sets, so step i+1's inputs
    # and step i's output cross PCIe while a step computes; events order each buffer's
    # reuse.
    e2e = None
    if not args.no_e2e:
        pin = lambda t: torch.empty(t.shape, dtype=t.dtype, pin_memory=True).copy_(t.cpu())
        hq, hk, hv, hs, hl = pin(q), pin(k_new), pin(v_new), pin(slots_d), pin(lens_d)
        ht = pin(tables_d)
        hout = [torch.empty(out.shape, dtype=out.dtype, pin_memory=True) for _ in range(2)]
        sets = [dict(q=torch.empty_like(q), k=torch.empty_like(k_new), v=torch.empty_like(v_new),
                     s=torch.empty_like(slots_d), l=torch.empty_like(lens_d), o=torch.empty_like(out))
                for _ in range(2)]
        tab = torch.empty_like(tables_d)
        h2d_stream, d2h_stream = torch.cuda.Stream(), torch.cuda.Stream()
        ev_in = [torch.cuda.Event() for _ in range(2)]     # inputs of a set landed
        ev_used = [torch.cuda.Event() for _ in range(2)]   # the step reading a set is done
        ev_out = [torch.cuda.Event() for _ in range(2)]    # a set's output read back
        h2d_step = sum(t.numel() * t.element_size() for t in (hq, hk, hv, hs, hl))
        d2h = hout[0].numel() * hout[0].element_size()
        tables_bytes = ht.numel() * ht.element_size()
        state = {"i": 0}

        def e2e_step():
            i = state["i"]
            b = i & 1
            st = sets[b]
            with torch.cuda.stream(h2d_stream):
                if i == 0:
                    tab.copy_(ht, non_blocking=True)           # tables: only when they change
                if i >= 2:
                    h2d_stream.wait_event(ev_used[b])          # step i-2 has read this set
                for dst, src in ((st["q"], hq), (st["k"], hk), (st["v"], hv), (st["s"], hs), (st["l"], hl)):
                    dst.copy_(src, non_blocking=True)
                ev_in[b].record(h2d_stream)
            stream.wait_event(ev_in[b])
            if i >= 2:
                stream.wait_event(ev_out[b])                   # step i-2's output was read back
            pa.pa_append_decode(st["k"], st["v"], st["s"], st["q"], cache.key_cache, cache.value_cache, tab,
                                st["l"], max_ctx, wl.scale, st["o"], part, ws, cache.err_flag, stream)
            ev_used[b].record(stream)
            with torch.cuda.stream(d2h_stream):
                d2h_stream.wait_event(ev_used[b])
                hout[b].copy_(st["o"], non_blocking=True)
                ev_out[b].record(d2h_stream)
            state["i"] = i + 1

        for _ in range(args.warmup):
            e2e_step()
        torch.cuda.synchronize()
        state["i"] = 0
        barrier(world)
        torch.cuda.synchronize()
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        f0.record(stream)
        for _ in range(K):
            e2e_step()
        stream.wait_event(ev_out[(K - 1) & 1])              # the last output is on the host
        f1.record(stream)
        torch.cuda.synchronize()
        barrier(world)
        e2e_ms = max_over_ranks(f0.elapsed_time(f1), world)
        ref = out.cpu()
        assert torch.equal(hout[(K - 1) & 1], ref), "end-to-end output differs from the device-resident step"
        e2e = {"value": round(world * (unique_b + cw_b) * K / (e2e_ms * 1e-3) / 1e9, 2), "unit": "GB/s",
               "ms_per_step": round(e2e_ms / K, 5),
               "seq_steps_per_s": round(world * S * K / (e2e_ms * 1e-3), 1),
               "h2d_bytes_per_step": int(h2d_step + tables_bytes / K), "d2h_bytes_per_step": int(d2h),
               "h2d_tables_bytes_once": int(tables_bytes),
               "overlap": "h2d and d2h streams, two device buffer sets; tables uploaded once (unchanged "
                          "across the repeated step)"}

    # the same step with L2 flushed before each call (a 2 x L2 write outside the
    # timed events): shared prefix blocks can no longer be found in L2 from the
    # previous step, only within the call
    flushed = None
    if not args.no_e2e:
        l2 = torch.cuda.get_device_properties(local).L2_cache_size
        scrub = torch.empty(max(2 * l2, 256 << 20), dtype=torch.uint8, device="cuda")
        nfl = min(K, 100)
        evf = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(nfl)]
        for i in range(nfl):
            scrub.fill_(i & 0xFF)
            step_fn(*evf[i])
        torch.cuda.synchronize()
        fl_ms = float(np.mean([a.elapsed_time(b) for a, b in evf]))
        flushed = {"ms_per_call": round(fl_ms, 5), "value": round((unique_b + cw_b) / (fl_ms * 1e-3) / 1e9, 2),
                   "unit": "GB/s", "calls": nfl, "flush_bytes": int(scrub.numel())}
        del scrub
    flag = pa.pa_wait(cache.err_flag)
    assert flag == 0, f"device error flag {flag}"

    rows = None
    if rank == 0 and world == 1 and not args.no_rows:
        peaks0 = load_peaks()
        del cache, ws, out, q, k_new, v_new, tables_d, lens_d, slots_d
        torch.cuda.empty_cache()
        rows = run_rows(args.row_reps, peaks0, args.partition)
        if not args.no_cpu_baseline:
            for name, cb in cpu_rows(set(ROW_GROUPS)).items():
                rows.setdefault(name, {})["cpu_baseline"] = cb

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(wl, None, step, tables_h, lens_h, budget_s=args.cpu_seconds)

    if rank == 0:
        # kernels of one pa_append_decode call: the decode chain, plus the write's own
        # launch unless the shared-prefix chain (5 kernels) takes the write into its first
        n_dec = pa.pa_decode_launches(S, wl.num_q_heads, wl.num_kv_heads, wl.head_dim, pa.PA_BF16, part)
        step_launches = n_dec if n_dec == 5 else n_dec + 1
        peaks = load_peaks()
        peak = float(peaks["hbm_gbs"]) if peaks else 6650.0
        achieved = (unique_b + cw_b) / (call_ms * 1e-3) / 1e9
        value = world * (unique_b + cw_b) * K / (ms_max * 1e-3) / 1e9
        line = {
            "metric": "paged-decode KV GB/s (unique algorithmic bytes) on B200",
            "value": round(value, 2), "unit": "GB/s", "n_gpus": world, "steps": K,
            "warmup": args.warmup, "ms_per_step": round(ms_max / K, 5), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": headline_config(wl, S, max_ctx, np.mean(lens_h), part, world),
            "seq_steps_per_s": round(world * S * K / (ms_max * 1e-3), 1),
            "pct_of_8tbs": round(100 * value / world / 8000, 2),
            "pct_of_measured_hbm": round(100 * value / world / peak, 2),
            "logical_gbs": round(world * (logical_b + cw_b) * K / (ms_max * 1e-3) / 1e9, 2),
            "bytes_per_step": {"decode_unique": unique_b, "decode_logical": logical_b, "cache_write": cw_b},
            "roofline": {"bound": "hbm", "kernel": "pa_append_decode call (cache write fused with group detection, tcgen05 group tiles, 16-row group units, decode_kernel, lse reduce)",
                         "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                         "frac": round(achieved / peak, 4),
                         "peak_source": "MEASURED_PEAKS.json hbm_gbs (of measured)" if peaks else "fallback",
                         "traffic": recorded_traffic(),
                         "call_ms": round(call_ms, 5)},
            "l2_flushed": flushed,
            "two_calls": {"ms_per_step": round(two_ms, 5),
                          "value": round(world * (unique_b + cw_b) / (two_ms * 1e-3) / 1e9, 2), "unit": "GB/s",
                          "pa_decode_ms": round(dec_ms, 5),
                          "pa_decode_gbs": round(unique_b / (dec_ms * 1e-3) / 1e9, 1), "steps": nf},
            "e2e": e2e,
            "gpu_launches": K * step_launches,
            "clocks": clocks,
            "cpu_baseline": cpu,
            "rows": rows,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


# ----------------------------------------------------------------- per-row figures
def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    return json.load(open(path)) if os.path.exists(path) else None


def _setup(wl, fp8=None):
    """The workload's pool (bf16, or e4m3 with fp8 = (k_scale, v_scale)) filled by
    replaying its set-up writes through pa_cache_write."""
    import torch
    import paged_kv_cache_389_b200 as pa
    from paged_kv_cache_389_b200.cache import PagedKVCache
    ks, vs = fp8 if fp8 else (1.0, 1.0)
    dt = torch.float8_e4m3fn if fp8 else torch.bfloat16
    cache = PagedKVCache(wl.num_blocks, wl.num_kv_heads, wl.head_dim, dt, "cuda", wl.free_order,
                         k_scale=ks, v_scale=vs)
    dev = lambda a: torch.from_numpy(a.view(np.int16)).cuda().view(torch.bfloat16)
    workloads.replay(wl, cache.manager, lambda k, v, s: pa.pa_cache_write(
        dev(k), dev(v), torch.from_numpy(s).cuda(), cache.key_cache, cache.value_cache, cache.err_flag,
        k_scale=ks, v_scale=vs))
    return cache, dev


def _time(fn, reps, warm=3, graph=False):
    """Mean device ms of fn() over reps (CUDA events on the current stream).  With
    graph=True the reps are captured into one CUDA graph first, so microsecond
    kernels are timed on the device rather than at Python's launch rate."""
    import torch
    for _ in range(warm):
        fn()
    torch.cuda.synchronize()
    g = None
    if graph:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for _ in range(reps):
                fn()
        g.replay()
        torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    if g is not None:
        g.replay()
    else:
        for _ in range(reps):
            fn()
    b.record()
    torch.cuda.synchronize()
    return a.elapsed_time(b) / reps


ROW_GROUPS = ("mha7b", "fork", "spec", "fp8", "prefix", "long")


def _warm_kernels():
    """One small call of each kernel family before any row is timed, so no row pays
    for loading the library's kernels (the fork row times single launches)."""
    import torch
    import paged_kv_cache_389_b200 as pa
    wl = workloads.make(3, mini=True)
    cache, dev = _setup(wl)
    st = wl.steps[0]
    slots, _ = cache.plan_append(st.seqs)
    mb = cache.manager.max_seq_blocks(st.seqs)
    t, l = cache.manager.build_tables(st.seqs, mb)
    td, ld, q = torch.from_numpy(t).cuda(), torch.from_numpy(l).cuda(), dev(st.q)
    out = torch.empty_like(q)
    for part in (0, 64, 512):
        n = pa.pa_decode_workspace_size(len(st.seqs), wl.num_q_heads, wl.head_dim, int(l.max()), part) if part else 0
        ws = torch.empty(max(n, 16), dtype=torch.uint8, device="cuda")
        pa.pa_append_decode(dev(st.k_new), dev(st.v_new), torch.from_numpy(slots).cuda(), q, cache.key_cache,
                            cache.value_cache, td, ld, int(l.max()), wl.scale, out, part, ws, cache.err_flag)
    qp = dev(np.zeros((len(st.seqs), 4, wl.num_q_heads, wl.head_dim), np.uint16))
    pa.pa_prefill_chunk(qp, cache.key_cache, cache.value_cache, td, ld,
                        torch.full((len(st.seqs),), 4, dtype=torch.int32, device="cuda"), wl.scale,
                        torch.empty_like(qp), cache.err_flag)
    # a block copy into the pool's last block (the pool is dropped right after)
    pa.pa_copy_blocks(cache.key_cache, cache.value_cache,
                      torch.tensor([[0, wl.num_blocks - 1]], dtype=torch.int32, device="cuda"), cache.err_flag)
    torch.cuda.synchronize()
    del cache
    torch.cuda.empty_cache()


def run_rows(reps, peaks, partition=PARTITION, groups=None):
    """Each hot-path row on its own workload; device time, inputs resident in HBM.
    groups: the row groups to run (default all of ROW_GROUPS)."""
    groups = set(ROW_GROUPS) if not groups else groups
    unknown = groups - set(ROW_GROUPS)
    if unknown:
        raise ValueError(f"unknown row groups {sorted(unknown)}; known: {ROW_GROUPS}")
    import torch
    import paged_kv_cache_389_b200 as pa
    hbm = float(peaks["hbm_gbs"]) if peaks else 6650.0
    tf_burst = float(peaks["bf16_tflops"]) if peaks else 1590.0
    rows = {}
    _warm_kernels()

    def dec_entry(name, cache, q, td, ld, maxc, scale, part, bytes_u, bytes_l, nseq):
        out = torch.empty_like(q)
        n = pa.pa_decode_workspace_size(q.shape[0], q.shape[1], q.shape[2], maxc, part) if part else 0
        ws = torch.empty(max(n, 16), dtype=torch.uint8, device="cuda")
        ms = _time(lambda: pa.pa_decode(q, cache.key_cache, cache.value_cache, td, ld, maxc, scale, out,
                                        part, ws, cache.err_flag, None, cache.k_scale, cache.v_scale), reps)
        rows[name] = {"ms": round(ms, 5), "unique_gbs": round(bytes_u / ms / 1e6, 1),
                      "logical_gbs": round(bytes_l / ms / 1e6, 1), "frac_of_measured_hbm": round(bytes_u / ms / 1e6 / hbm, 4),
                      "seq_steps_per_s": round(nseq / ms * 1e3, 1), "partition_size": part}

    if "mha7b" in groups:
        # -- MHA-7B decode (64 seqs, 32/32 heads): unsplit and split-K
        wl = workloads.make(2)
        cache, dev = _setup(wl)
        st = wl.steps[0]
        cache.append(st.seqs, dev(st.k_new), dev(st.v_new))
        mb = cache.manager.max_seq_blocks(st.seqs)
        t, l = cache.manager.build_tables(st.seqs, mb)
        ub, lb = step_bytes(wl, t, l)
        td, ld, q = torch.from_numpy(t).cuda(), torch.from_numpy(l).cuda(), dev(st.q)
        for part in (0, 1024):
            dec_entry(f"a3_decode_mha7b_p{part}", cache, q, td, ld, int(l.max()), wl.scale, part, ub, lb, len(st.seqs))
        del cache
        torch.cuda.empty_cache()

    if "fork" in groups:
        # -- parallel sampling: 128 parents x 4 children, 16 steps of copy-on-write + cache write + decode
        wl = workloads.make(4)
        cache, dev = _setup(wl)
        S = len(wl.steps[0].seqs)
        part = partition
        host_s = 0.0
        total_pairs = 0
        ub_sum = 0
        pairs1 = None
        # host side first: each step's slots, copy-on-write pairs and tables (the
        # manager's plans do not depend on the GPU), uploaded before any timing, so
        # that the 16 steps' GPU work is issued back to back
        plan = []
        for st in wl.steps:
            h0 = time.perf_counter()
            slots, pairs = cache.plan_append(st.seqs)
            mb = cache.manager.max_seq_blocks(st.seqs)
            t, l = cache.manager.build_tables(st.seqs, mb)
            host_s += time.perf_counter() - h0
            ub, _ = step_bytes(wl, t, l)
            ub_sum += ub
            total_pairs += len(pairs)
            pr = torch.from_numpy(pairs).cuda() if len(pairs) else None
            if pairs1 is None and pr is not None:
                pairs1 = pr
            maxc = int(l.max())
            n = pa.pa_decode_workspace_size(S, wl.num_q_heads, wl.head_dim, maxc, part)
            plan.append(dict(td=torch.from_numpy(t).cuda(), ld=torch.from_numpy(l).cuda(), q=dev(st.q),
                             kn=dev(st.k_new), vn=dev(st.v_new), sl=torch.from_numpy(slots).cuda(), pr=pr,
                             np=len(pairs), maxc=maxc, out=torch.empty_like(dev(st.q)),
                             ws=torch.empty(max(n, 16), dtype=torch.uint8, device="cuda")))
        torch.cuda.synchronize()
        ev = []
        for st in plan:
            e = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
            e[0].record()
            if st["pr"] is not None:
                pa.pa_copy_blocks(cache.key_cache, cache.value_cache, st["pr"], cache.err_flag)
            e[1].record()
            pa.pa_cache_write(st["kn"], st["vn"], st["sl"], cache.key_cache, cache.value_cache, cache.err_flag)
            e[2].record()
            pa.pa_decode(st["q"], cache.key_cache, cache.value_cache, st["td"], st["ld"], st["maxc"], wl.scale,
                         st["out"], part, st["ws"], cache.err_flag)
            e[3].record()
            ev.append((e, st["np"]))
        torch.cuda.synchronize()
        assert pa.pa_wait(cache.err_flag) == 0
        copy_ms = sum(e[0].elapsed_time(e[1]) for e, _ in ev)
        cw_ms = sum(e[1].elapsed_time(e[2]) for e, _ in ev)
        dec_ms = sum(e[2].elapsed_time(e[3]) for e, _ in ev)
        # the 16 decodes again (same inputs: the pool holds every step's tokens now,
        # and each call reads only its step's lengths), L2 flushed before each
        scrub = torch.empty(max(2 * torch.cuda.get_device_properties(0).L2_cache_size, 256 << 20),
                            dtype=torch.uint8, device="cuda")
        fl_ms = 0.0
        for st in plan:
            scrub.fill_(1)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            pa.pa_decode(st["q"], cache.key_cache, cache.value_cache, st["td"], st["ld"], st["maxc"], wl.scale,
                         st["out"], part, st["ws"], cache.err_flag)
            e1.record()
            torch.cuda.synchronize()
            fl_ms += e0.elapsed_time(e1)
        del scrub
        blk_bytes = wl.num_kv_heads * 16 * wl.head_dim * 2 * 2          # K + V of one block
        e1, np1 = ev[0]
        c1 = e1[0].elapsed_time(e1[1])
        rows["fork_cow_16_steps"] = {"seq_steps_per_s_device": round(S * len(wl.steps) / ((copy_ms + cw_ms + dec_ms) * 1e-3), 1),
                                     "device_ms_total": round(copy_ms + cw_ms + dec_ms, 4), "host_plan_ms_total": round(1e3 * host_s, 3),
                                     "decode_ms_total": round(dec_ms, 4), "decode_unique_gbs": round(ub_sum / dec_ms / 1e6, 1),
                                     "decode_ms_total_l2_flushed": round(fl_ms, 4),
                                     "decode_unique_gbs_l2_flushed": round(ub_sum / fl_ms / 1e6, 1),
                                     "cache_write_ms_total": round(cw_ms, 4), "copy_blocks_ms_total": round(copy_ms, 4),
                                     "copy_pairs_total": total_pairs}
        rows["a2_copy_blocks_step1"] = {"pairs": np1, "ms_first_launch": round(c1, 5),
                                        "gbs_first_launch": round(np1 * blk_bytes * 2 / c1 / 1e6, 1)}   # read + write
        if pairs1 is not None:   # same pairs again (the pool is not used afterwards)
            ms = _time(lambda: pa.pa_copy_blocks(cache.key_cache, cache.value_cache, pairs1, cache.err_flag), reps, graph=True)
            rows["a2_copy_blocks_step1"].update({"ms": round(ms, 5), "gbs": round(np1 * blk_bytes * 2 / ms / 1e6, 1)})
        # steady-state copy of the same 384 pairs (idempotent), and the 512-token cache write
        st = wl.steps[-1]
        kn, vn = dev(st.k_new), dev(st.v_new)
        slots = torch.from_numpy(np.array([cache.manager.block_table(s)[-1] * 16 for s in st.seqs], np.int64)).cuda()
        ms = _time(lambda: pa.pa_cache_write(kn, vn, slots, cache.key_cache, cache.value_cache, cache.err_flag), reps,
                   graph=True)
        rows["a1_cache_write_512tok"] = {"ms": round(ms, 5), "gbs": round(cache_write_bytes(wl, S) / ms / 1e6, 1)}
        del cache
        torch.cuda.empty_cache()

    if "spec" in groups:
        # -- speculative verify on the prefix-sharing workload: every sequence appends 4
        #    draft tokens; the 4 new positions attend causally (a 4-row chunk)
        wl = workloads.make(CONFIG_ID)
        cache, dev = _setup(wl)
        seqs = wl.steps[0].seqs
        S, kdraft = len(seqs), 4
        rng = np.random.default_rng(7)
        kd = dev(workloads.normal(rng, (S * kdraft, wl.num_kv_heads, wl.head_dim), "bf16"))
        vd = dev(workloads.normal(rng, (S * kdraft, wl.num_kv_heads, wl.head_dim), "bf16"))
        cache.append(seqs, kd, vd, counts=[kdraft] * S)
        mb = cache.manager.max_seq_blocks(seqs)
        t, l = cache.manager.build_tables(seqs, mb)
        td, ld = torch.from_numpy(t).cuda(), torch.from_numpy(l).cuda()
        qv = dev(workloads.normal(rng, (S, kdraft, wl.num_q_heads, wl.head_dim), "bf16"))
        outv = torch.empty_like(qv)
        chv = torch.full((S,), kdraft, dtype=torch.int32, device="cuda")
        ms = _time(lambda: pa.pa_prefill_chunk(qv, cache.key_cache, cache.value_cache, td, ld, chv, wl.scale, outv,
                                               cache.err_flag), reps)
        ub, lb = step_bytes(wl, t, l)
        rows["a6_spec_verify_k4"] = {"ms": round(ms, 5), "verified_tokens_per_s": round(S * kdraft / ms * 1e3, 1),
                                     "kv_logical_gbs": round(lb / ms / 1e6, 1), "kv_unique_gbs": round(ub / ms / 1e6, 1),
                                     "draft_tokens": kdraft, "num_seqs": S}
        assert pa.pa_wait(cache.err_flag) == 0
        del cache
        torch.cuda.empty_cache()

    if "fp8" in groups:
        # -- FP8 (e4m3) pools on the same workload: the headline step (cache write +
        #    decode in one pa_append_decode call) and the decode alone; half the K/V bytes
        wl = workloads.make(CONFIG_ID)
        cache, dev = _setup(wl, fp8=FP8_SCALES)
        st = wl.steps[0]
        slots, pairs = cache.plan_append(st.seqs)
        assert len(pairs) == 0
        mb = cache.manager.max_seq_blocks(st.seqs)
        t, l = cache.manager.build_tables(st.seqs, mb)
        ub, lb = step_bytes(wl, t, l, kv_elem=1)
        cwb = cache_write_bytes(wl, len(st.seqs), kv_elem=1)
        td, ld, q = torch.from_numpy(t).cuda(), torch.from_numpy(l).cuda(), dev(st.q)
        kn, vn, sl = dev(st.k_new), dev(st.v_new), torch.from_numpy(slots).cuda()
        maxc = int(l.max())
        n = pa.pa_decode_workspace_size(len(st.seqs), wl.num_q_heads, wl.head_dim, maxc, partition)
        ws8 = torch.empty(max(n, 16), dtype=torch.uint8, device="cuda")
        out8 = torch.empty_like(q)
        ms = _time(lambda: pa.pa_append_decode(kn, vn, sl, q, cache.key_cache, cache.value_cache, td, ld, maxc,
                                               wl.scale, out8, partition, ws8, cache.err_flag, None,
                                               cache.k_scale, cache.v_scale), reps)
        rows["a8_fp8_append_decode"] = {"ms": round(ms, 5), "unique_gbs": round((ub + cwb) / ms / 1e6, 1),
                                        "frac_of_measured_hbm": round((ub + cwb) / ms / 1e6 / hbm, 4),
                                        "seq_steps_per_s": round(len(st.seqs) / ms * 1e3, 1),
                                        "kv_bytes_per_element": 1, "partition_size": partition,
                                        "k_scale": cache.k_scale, "v_scale": cache.v_scale}
        dec_entry("a8_fp8_decode", cache, q, td, ld, maxc, wl.scale, partition, ub, lb, len(st.seqs))
        assert pa.pa_wait(cache.err_flag) == 0
        del cache
        torch.cuda.empty_cache()

    if "prefix" in groups:
        # -- automatic prefix caching (host): 256 prompts = a shared 512-token system
        #    prompt + a private lognormal tail, created from their token ids
        bm = pa.BlockManager(32768, 16)
        prng = np.random.default_rng(11)
        system = prng.integers(0, 32000, size=512).tolist()
        tails = np.clip(np.rint(600 * np.exp(prng.standard_normal(256))), 1, 8192).astype(int)
        prompts = [system + prng.integers(0, 32000, size=int(n)).tolist() for n in tails]
        arrays = [np.asarray(pr, dtype=np.int32) for pr in prompts]   # token ids as a server holds them
        h0 = time.perf_counter()
        hit = sum(bm.add_seq_tokens(i, a)[0] for i, a in enumerate(arrays))
        host_s = time.perf_counter() - h0
        bm_lists = pa.BlockManager(32768, 16)                           # the same from Python lists
        h0 = time.perf_counter()
        for i, pr in enumerate(prompts):
            bm_lists.add_seq_tokens(i, pr)
        host_lists_s = time.perf_counter() - h0
        del bm_lists
        total = sum(len(pr) for pr in prompts)
        rows["a7_prefix_cache_host"] = {"prompts": len(prompts), "prompt_tokens": total, "cached_tokens": int(hit),
                                        "hit_fraction": round(hit / total, 4), "kv_writes_saved_bytes":
                                        int(hit) * 8 * 128 * 2 * 2,
                                        "host_us_per_prompt": round(1e6 * host_s / len(prompts), 2),
                                        "host_us_per_prompt_from_python_lists":
                                        round(1e6 * host_lists_s / len(prompts), 2)}
        del bm

    if "long" in groups:
        # -- long context: split-K decode + tcgen05 prefill chunk
        wl = workloads.make(5)
        cache, dev = _setup(wl)
        st = wl.steps[0]
        mb = cache.manager.max_seq_blocks(st.seqs)
        t, l = cache.manager.build_tables(st.seqs, mb)
        ub, lb = step_bytes(wl, t, l)
        td, ld, q = torch.from_numpy(t).cuda(), torch.from_numpy(l).cuda(), dev(st.q)
        for part in (512, 2048):
            dec_entry(f"a4_decode_long_p{part}", cache, q, td, ld, int(l.max()), wl.scale, part, ub, lb, len(st.seqs))
        pf = wl.prefill
        qp = dev(pf.q)
        outp = torch.empty_like(qp)
        ch = torch.full((len(pf.seqs),), pf.chunk, dtype=torch.int32, device="cuda")
        ms = _time(lambda: pa.pa_prefill_chunk(qp, cache.key_cache, cache.value_cache, td, ld, ch, wl.scale, outp,
                                               cache.err_flag), max(3, reps // 10))
        keys = sum(int(L) - pf.chunk + i + 1 for L in l for i in range(pf.chunk))
        flops = 4.0 * wl.num_q_heads * wl.head_dim * keys
        rows["a5_prefill_chunk_long"] = {"ms": round(ms, 4), "tflops": round(flops / ms / 1e9, 1),
                                         "frac_of_measured_bf16": round(flops / ms / 1e9 / tf_burst, 4),
                                         "flops": flops, "rows": len(pf.seqs) * pf.chunk}
        assert pa.pa_wait(cache.err_flag) == 0
        del cache
        torch.cuda.empty_cache()

    return rows


# ----------------------------------------------------------------- CPU oracle
def _oracle_pools(wl):
    import oracle
    from oracle.block_model import BlockManagerModel
    model = BlockManagerModel(wl.num_blocks, wl.block_size, wl.free_order.tolist())
    kc = np.full(wl.cache_shape(), 0x7FC0, wl.np_dtype)
    vc = np.full(wl.cache_shape(), 0x7FC0, wl.np_dtype)
    workloads.replay(wl, model, lambda k, v, s: oracle.cache_write(k, v, s, kc, vc))
    step = wl.steps[0]
    slots = np.array([model.append_slot(s)[0] for s in step.seqs], np.int64)
    return model, kc, vc, slots


def _time_oracle_steps(wl, model, kc, vc, slots, n_seqs, reps):
    """Time `reps` oracle steps (cache write of the new tokens + decode) over the first
    n_seqs sequences; returns (seconds per step, unique bytes per step)."""
    import oracle
    step = wl.steps[0]
    seqs = step.seqs[:n_seqs]
    mb = max(len(model.block_table(s)) for s in seqs)
    t, l = model.build_tables(seqs, mb)
    ub, _ = step_bytes(wl, t, l)
    cw = cache_write_bytes(wl, n_seqs)
    q = np.ascontiguousarray(step.q[:n_seqs])
    k, v = np.ascontiguousarray(step.k_new[:n_seqs]), np.ascontiguousarray(step.v_new[:n_seqs])
    sl = slots[:n_seqs]
    t0 = time.perf_counter()
    for _ in range(reps):
        oracle.cache_write(k, v, sl, kc, vc)
        oracle.decode(q, kc, vc, t, l, wl.scale)
    return (time.perf_counter() - t0) / reps, ub + cw


def cpu_baseline(wl, cache, step, tables_h, lens_h, budget_s=15.0):
    import oracle
    model, kc, vc, slots = _oracle_pools(wl)
    S = len(step.seqs)
    per, b = _time_oracle_steps(wl, model, kc, vc, slots, S, 1)
    reps = max(1, min(int(budget_s / max(per, 1e-3)), 20))
    per, b = _time_oracle_steps(wl, model, kc, vc, slots, S, reps)
    out = {"value": round(b / per / 1e9, 4), "unit": "GB/s", "cores": oracle.num_threads(),
           "kind": "oracle", "seconds_per_step": round(per, 4),
           "sample": f"full step ({S} sequences: cache write + decode), {reps} rep(s), fp64 C + OpenMP",
           "cpu": _cpu_model()}
    # the same oracle on one thread, over the first eighth of the sequences
    threads = oracle.num_threads()
    n1 = max(1, S // 8)
    oracle.set_num_threads(1)
    try:
        per1, b1 = _time_oracle_steps(wl, model, kc, vc, slots, n1, 1)
    finally:
        oracle.set_num_threads(threads)
    out["single_thread"] = {"value": round(b1 / per1 / 1e9, 4), "unit": "GB/s", "cores": 1,
                            "seconds_per_step": round(per1, 4),
                            "sample": f"first {n1} of {S} sequences (cache write + decode), 1 rep"}
    return out


def _oracle_setup(wl):
    """The oracle's pools and block model after the workload's set-up operations."""
    import oracle
    from oracle.block_model import BlockManagerModel
    model = BlockManagerModel(wl.num_blocks, wl.block_size, wl.free_order.tolist())
    fill = np.nan if wl.dtype == "f32" else 0x7FC0
    kc = np.full(wl.cache_shape(), fill, wl.np_dtype)
    vc = np.full(wl.cache_shape(), fill, wl.np_dtype)
    workloads.replay(wl, model, lambda k, v, sl: oracle.cache_write(k, v, sl, kc, vc))
    return model, kc, vc


def _oracle_step(wl, model, kc, vc, step):
    """One step of the hot path on the oracle: copy-on-write pairs, the new tokens'
    cache write, decode of every sequence.  Returns (tables, lens) of the decode."""
    import oracle
    slots, pairs = [], []
    for sq in step.seqs:
        sl, pr = model.append_slot(sq)
        slots.append(sl)
        if pr is not None:
            pairs.append(pr)
    if pairs:
        oracle.copy_blocks(kc, vc, np.array(pairs, np.int32))
    oracle.cache_write(step.k_new, step.v_new, np.array(slots, np.int64), kc, vc)
    mb = max(len(model.block_table(sq)) for sq in step.seqs)
    t, l = model.build_tables(step.seqs, mb)
    oracle.decode(step.q, kc, vc, t, l, wl.scale)
    return t, l


def cpu_rows(groups, budget_s=12.0):
    """The oracle, as it stands, timed on the host cores for the rows' workloads
    (a baseline, not a target): config 1 and 2 steps, config 4's fork / copy-on-write
    steps (all 16 when they fit the budget, else the first ones), config 5's decode in
    full and its prefill chunk on one sequence scaled x8.  Returns {row: cpu_baseline}."""
    import oracle
    cores, cpu = oracle.num_threads(), _cpu_model()
    out = {}

    def entry(value, unit, secs, sample):
        return {"value": round(value, 4), "unit": unit, "cores": cores, "kind": "oracle",
                "seconds": round(secs, 3), "sample": sample, "cpu": cpu}

    wl = workloads.make(1)
    model, kc, vc = _oracle_setup(wl)
    t0 = time.perf_counter()
    t, l = _oracle_step(wl, model, kc, vc, wl.steps[0])
    el = time.perf_counter() - t0
    ub, _ = step_bytes(wl, t, l)
    out["c1_tiny_fp32"] = entry((ub + cache_write_bytes(wl, len(l))) / el / 1e9, "GB/s", el,
                                "config 1: the whole step (4 sequences, cache write + decode)")
    if "mha7b" in groups:
        wl = workloads.make(2)
        model, kc, vc = _oracle_setup(wl)
        t0 = time.perf_counter()
        t, l = _oracle_step(wl, model, kc, vc, wl.steps[0])
        el = time.perf_counter() - t0
        ub, _ = step_bytes(wl, t, l)
        e = entry((ub + cache_write_bytes(wl, len(l))) / el / 1e9, "GB/s", el,
                  "config 2: the whole step (64 sequences, cache write + decode, unsplit)")
        out["a3_decode_mha7b_p0"] = out["a3_decode_mha7b_p1024"] = e
    if "fork" in groups:
        wl = workloads.make(4)
        model, kc, vc = _oracle_setup(wl)
        n = done = 0
        ub_sum = 0
        t0 = time.perf_counter()
        for st in wl.steps:
            t, l = _oracle_step(wl, model, kc, vc, st)
            ub_sum += step_bytes(wl, t, l)[0]
            n += len(st.seqs)
            done += 1
            if time.perf_counter() - t0 > budget_s:
                break
        el = time.perf_counter() - t0
        out["fork_cow_16_steps"] = entry(n / el, "seq_steps/s", el,
                                         f"config 4: the first {done} of {len(wl.steps)} steps (copy-on-write, "
                                         f"cache write, decode of 512 sequences)")
        out["fork_cow_16_steps"]["decode_unique_gbs"] = round(ub_sum / el / 1e9, 4)
    if "long" in groups:
        wl = workloads.make(5)
        model, kc, vc = _oracle_setup(wl)
        st = wl.steps[0]
        mb = max(len(model.block_table(sq)) for sq in st.seqs)
        t, l = model.build_tables(st.seqs, mb)
        t0 = time.perf_counter()
        oracle.decode(st.q, kc, vc, t, l, wl.scale)
        el = time.perf_counter() - t0
        ub, _ = step_bytes(wl, t, l)
        e = entry(ub / el / 1e9, "GB/s", el, "config 5: decode of all 8 x 32768-token sequences")
        out["a4_decode_long_p512"] = out["a4_decode_long_p2048"] = e
        pf = wl.prefill
        rows = np.arange(0, pf.chunk, pf.chunk // 64)          # 64 rows of sequence 0, evenly spread
        mask = np.zeros((len(pf.seqs), pf.chunk), bool)
        mask[0, rows] = True
        ch = np.full(len(pf.seqs), pf.chunk, np.int32)
        t0 = time.perf_counter()
        oracle.prefill(pf.q, kc, vc, t, l, ch, wl.scale, row_mask=mask)
        el = time.perf_counter() - t0
        keys = sum(int(l[0]) - pf.chunk + int(i) + 1 for i in rows)
        flops = 4.0 * wl.num_q_heads * wl.head_dim * keys
        scale_up = len(pf.seqs) * pf.chunk / len(rows)
        out["a5_prefill_chunk_long"] = entry(flops / el / 1e12, "TFLOP/s", el * scale_up,
                                             f"config 5: {len(rows)} of the 512 chunk rows of sequence 0 (all "
                                             f"heads) timed; seconds = the timed ones x {scale_up:.0f} for all 8 "
                                             "sequences' rows")
    return out


def _cpu_model():
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return None


def run_reference(args):
    """The oracle as it stands, timed on the host cores, on this workload."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    wl = workloads.make(CONFIG_ID)
    model, kc, vc, slots = _oracle_pools(wl)
    S = len(wl.steps[0].seqs)
    _, lens_all = model.build_tables(wl.steps[0].seqs, max(len(model.block_table(s)) for s in wl.steps[0].seqs))
    one, _ = _time_oracle_steps(wl, model, kc, vc, slots, 1, 1)
    budget = 150.0 / max(1, args.steps + args.warmup)          # seconds of oracle work per step
    n = int(max(1, min(S, budget / max(one, 1e-4))))
    for _ in range(args.warmup):
        _time_oracle_steps(wl, model, kc, vc, slots, n, 1)
    t0 = time.perf_counter()
    total_b = 0
    for _ in range(args.steps):
        _, b = _time_oracle_steps(wl, model, kc, vc, slots, n, 1)
        total_b += b
    el = time.perf_counter() - t0
    value = total_b / el / 1e9
    line = {
        "impl": "reference", "metric": "paged-decode KV GB/s (unique algorithmic bytes) on B200",
        "value": round(value, 4), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(1e3 * el / args.steps, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": headline_config(wl, S, int(lens_all.max()), np.mean(lens_all), args.partition, world),
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": oracle.num_threads(),
                         "kind": "oracle", "sample": f"first {n} of {S} sequences per step "
                                                     "(cache write + decode), fp64 C + OpenMP",
                         "cpu": _cpu_model()},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-rows", action="store_true", help="skip the per-row figures of the other workloads")
    ap.add_argument("--row-reps", type=int, default=50)
    ap.add_argument("--rows-only", default="",
                    help="comma list of row groups (mha7b, fork, spec, fp8, prefix, long): time only "
                         "those rows, print them as one JSON line and skip the headline step")
    ap.add_argument("--partition", type=int, default=PARTITION,
                    help="split-K partition size in tokens (multiple of 16) of the timed decode")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        run_reference(args)
    elif args.rows_only:
        groups = set(args.rows_only.split(","))
        rows = run_rows(args.row_reps, load_peaks(), args.partition, groups)
        if not args.no_cpu_baseline:
            for name, cb in cpu_rows(groups).items():
                rows.setdefault(name, {})["cpu_baseline"] = cb
        print(json.dumps({"rows": rows}), flush=True)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
