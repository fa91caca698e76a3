"""Benchmark: paged FP8-KV decode attention tokens/s and HBM GB/s vs concurrency.

One "step" is one pass of the whole decode hot path for one layer over one
batch: the batched page-tag check, the FP8 quantise-and-append of every
request's new K/V token, and paged decode attention (split-K partial + LSE
merge), all through the C ABI on one stream.  The headline workload is the
concurrency sweep's largest batch: 64 requests x 8,192 tokens of context,
page size 64, 64 query heads / 8 KV heads, head_dim 128, FP8 E4M3 KV with
per-tensor scales (synthetic, seeded).  tokens/s = requests / step time.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

Prints one JSON line (rank 0).  N > 1 runs N independent replicas (one per
GPU, each with its own batch; no data-path collective) and reports the
aggregate over ranks with the slowest rank's time.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "paged FP8-KV decode attention tokens/s & HBM GB/s (% peak) vs concurrency"
UNIT = "tokens/s"
HEADLINE_BATCH = 64
CONTEXT = 8192
SWEEP = (1, 8, 16, 32, 64)
NOMINAL_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0
L2_BYTES = 126 * 2**20


# --------------------------------------------------------------------------
# small host-side helpers (also exercised by the CPU tests)
# --------------------------------------------------------------------------

def kv_bytes_per_step(seq_lens, num_kv_heads, head_dim, elem_bytes):
    """Algorithmic K+V bytes attention reads in one step."""
    return int(sum(int(L) for L in seq_lens)) * num_kv_heads * head_dim * 2 * elem_bytes


def attn_algorithmic_bytes(seq_lens, page_size, num_q_heads, num_kv_heads, head_dim,
                           elem_bytes):
    """KV + q/out/lse + page-table bytes of one attention call."""
    B = len(seq_lens)
    kv = kv_bytes_per_step(seq_lens, num_kv_heads, head_dim, elem_bytes)
    qo = B * num_q_heads * (2 * head_dim * 2 + 4)
    pt = sum((int(L) + page_size - 1) // page_size for L in seq_lens) * 4
    return kv + qo + pt


def unique_kv_tokens(seq_lens, page_table, page_size):
    """Distinct (physical page, slot) positions attention reads in one step:
    a page shared by several requests counts once, with the most slots any of
    them reads from it."""
    import numpy as np
    per_page = {}
    for b, L in enumerate(seq_lens):
        L = int(L)
        n = (L + page_size - 1) // page_size
        for j in range(n):
            pg = int(page_table[b][j])
            used = min(page_size, L - j * page_size)
            if used > per_page.get(pg, 0):
                per_page[pg] = used
    return int(sum(per_page.values()))


def reduce_max_time(local_ms: float, world: int) -> float:
    """Max of a per-rank time over the process group (identity if world == 1)."""
    if world <= 1:
        return local_ms
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([local_ms], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_seed(base: int, rank: int) -> int:
    """Each replica draws its own batch."""
    return base + 1000 * rank


def headline_config(world):
    """The `config` object of both arms' lines: the headline workload."""
    kv_gb = HEADLINE_BATCH * CONTEXT * 8 * 128 * 2 / 1e9
    return {"workload": f"concurrency sweep, batch {HEADLINE_BATCH} x context {CONTEXT}, "
                        "page 64, 64 q heads / 8 kv heads, head_dim 128, FP8 E4M3 KV",
            "step": "tag check + FP8 append (one fused kernel) + paged attention, one layer",
            "global_batch": world * HEADLINE_BATCH, "seq_len": CONTEXT,
            "kv_dtype": "fp8_e4m3", "parallelism": f"replicas x{world}",
            "l2": f"inputs larger than L2 ({kv_gb:.2f} GB of KV per step)"}


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def source_hash(paths):
    h = hashlib.sha256()
    for p in paths:
        with open(p, "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


ATTN_SOURCES = [os.path.join(ROOT, "paged_fp8_kv_attn_b200", "csrc", n)
                for n in ("attention.cu", "device.cuh", "internal.h")]
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "attn_fp8_traffic.json")


def ncu_traffic_per_launch(num_kv_tokens):
    """DRAM bytes per attention launch from the committed ncu capture, scaled to
    this launch by KV tokens; None if no capture exists or the kernel source
    changed since it was taken."""
    try:
        with open(TRAFFIC_FILE) as f:
            rec = json.load(f)
    except Exception:
        return None
    if rec.get("source_hash") != source_hash(ATTN_SOURCES):
        return None
    per_token = float(rec["dram_bytes_per_launch"]) / float(rec["kv_tokens"])
    return per_token * num_kv_tokens


class ClockSampler:
    """nvidia-smi clock / throttle samples while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self._t = threading.Thread(target=self._read, daemon=True)
            self._t.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.15)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for name, val in zip(names, parts[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


# --------------------------------------------------------------------------
# GPU arm
# --------------------------------------------------------------------------

class Step:
    """Device buffers and the C-ABI calls of one decode step."""

    def __init__(self, wl, kv="fp8"):
        import numpy as np
        import torch
        import paged_fp8_kv_attn_b200 as pkv
        self.pkv = pkv
        self.wl = wl
        self.kv = kv
        dev = torch.device("cuda")
        B, Hq, D = wl.q.shape
        # The per-step inputs and outputs live in one packed device buffer each,
        # so that an end-to-end step moves them with one copy in and one out.
        ins = [("q", wl.q.contiguous()), ("k_new", wl.k_new.contiguous()),
               ("v_new", wl.v_new.contiguous()),
               ("seq_lens", torch.from_numpy(wl.seq_lens)),
               ("page_table", torch.from_numpy(wl.page_table)),
               ("expected", torch.from_numpy(wl.expected_tags.view(np.int32)))]
        outs = [("out", torch.empty((B, Hq, D), dtype=torch.bfloat16)),
                ("lse", torch.empty((B, Hq), dtype=torch.float32)),
                ("abort", torch.zeros(B, dtype=torch.uint8))]
        self._ins_meta = [(n, t.dtype, tuple(t.shape)) for n, t in ins]
        self._outs_meta = [(n, t.dtype, tuple(t.shape)) for n, t in outs]
        self.dev_in, self.in_views = self._pack(ins, dev)
        self.dev_out, self.out_views = self._pack(outs, dev)
        for name, t in {**self.in_views, **self.out_views}.items():
            setattr(self, name, t)
        for name, src in ins:
            getattr(self, name).copy_(src.to(dev))
        self.page_tags = torch.from_numpy(wl.page_tags.view(np.int32)).to(dev)
        if kv == "fp8":
            self.k_cache = torch.empty(wl.k_pool.shape, dtype=torch.uint8, device=dev)
            self.v_cache = torch.empty(wl.v_pool.shape, dtype=torch.uint8, device=dev)
            ids = torch.arange(wl.num_pages, dtype=torch.int32, device=dev)
            pkv.kv_requant_pages_fp8(wl.k_pool, ids, self.k_cache, ids, wl.k_scale)
            pkv.kv_requant_pages_fp8(wl.v_pool, ids, self.v_cache, ids, wl.v_scale)
            code = pkv.PKV_KV_FP8
        else:
            self.k_cache = wl.k_pool
            self.v_cache = wl.v_pool
            code = pkv.PKV_KV_BF16
        self.ws = pkv.alloc_workspace(code, B, Hq, wl.num_kv_heads, D, device=dev)
        torch.cuda.synchronize()

    def twin(self):
        """The same step over a second set of packed input/output buffers
        (shared caches, tags and workspace), for double-buffered end-to-end
        steps: one set is copied while the other computes."""
        import copy
        import torch
        t = copy.copy(self)
        ins = [(n, torch.empty(shape, dtype=dt)) for n, dt, shape in self._ins_meta]
        outs = [(n, torch.empty(shape, dtype=dt)) for n, dt, shape in self._outs_meta]
        t.dev_in, t.in_views = self._pack(ins, self.dev_in.device)
        t.dev_out, t.out_views = self._pack(outs, self.dev_out.device)
        for name, v in {**t.in_views, **t.out_views}.items():
            setattr(t, name, v)
        t.dev_in.copy_(self.dev_in)
        return t

    @staticmethod
    def _pack(named, dev):
        """One uint8 device buffer holding every tensor (256-byte aligned
        slots) and typed views into it."""
        import torch
        offs, total = [], 0
        for _, t in named:
            offs.append(total)
            total += (t.numel() * t.element_size() + 255) // 256 * 256
        buf = torch.zeros(total, dtype=torch.uint8, device=dev)
        views = {}
        for (name, t), off in zip(named, offs):
            n = t.numel() * t.element_size()
            views[name] = buf[off: off + n].view(t.dtype).view(t.shape)
        return buf, views

    def check(self):
        wl = self.wl
        self.pkv.kv_tag_check(self.page_tags, self.page_table, self.expected, self.seq_lens,
                              wl.page_size, self.abort)

    def append(self, checked=True):
        wl = self.wl
        ab = self.abort if checked else None
        if self.kv == "fp8":
            self.pkv.kv_append_fp8(self.k_new, self.v_new, self.page_table, self.seq_lens,
                                   wl.page_size, wl.k_scale, wl.v_scale, self.k_cache,
                                   self.v_cache, ab)
        else:
            self.pkv.kv_append_bf16(self.k_new, self.v_new, self.page_table, self.seq_lens,
                                    wl.page_size, self.k_cache, self.v_cache, ab)

    def attend(self, checked=True):
        wl = self.wl
        ab = self.abort if checked else None
        if self.kv == "fp8":
            self.pkv.paged_decode_attn_fp8(self.q, self.k_cache, self.v_cache, wl.k_scale,
                                           wl.v_scale, self.page_table, self.seq_lens,
                                           wl.sm_scale, self.out, self.lse, self.ws, abort=ab)
        else:
            self.pkv.paged_decode_attn_bf16(self.q, self.k_cache, self.v_cache, self.page_table,
                                            self.seq_lens, wl.sm_scale, self.out, self.lse,
                                            self.ws, abort=ab)

    def check_append(self):
        wl = self.wl
        if self.kv == "fp8":
            self.pkv.kv_check_append_fp8(self.page_tags, self.page_table, self.expected,
                                         self.seq_lens, wl.page_size, self.k_new, self.v_new,
                                         wl.k_scale, wl.v_scale, self.k_cache, self.v_cache,
                                         self.abort)
        else:
            self.pkv.kv_check_append_bf16(self.page_tags, self.page_table, self.expected,
                                          self.seq_lens, wl.page_size, self.k_new, self.v_new,
                                          self.k_cache, self.v_cache, self.abort)

    def full(self):
        """The checked step: tag check and append (one fused kernel), then
        attention with the abort mask."""
        self.check_append()
        self.attend(True)

    def unchecked(self):
        self.append(False)
        self.attend(False)


def _graph(fn):
    import torch
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        fn()                         # warm the library's per-device set-up outside capture
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    torch.cuda.synchronize()
    return g


class L2Flush:
    """Evicts L2 between timed calls: writes one buffer of twice the L2 size,
    then reads another of the same size, so that neither the previous call's
    inputs nor dirty lines (which the timed call would otherwise have to
    write back) remain in L2."""

    def __init__(self):
        import torch
        n = 2 * L2_BYTES // 4
        self.w = torch.zeros(n, dtype=torch.float32, device="cuda")
        self.r = torch.zeros(n, dtype=torch.float32, device="cuda")
        self.sink = torch.zeros((), dtype=torch.float32, device="cuda")

    def __call__(self):
        import torch
        self.w.add_(1)
        torch.sum(self.r, dim=0, out=self.sink)

    describe = f"flushed between calls (write {2 * L2_BYTES >> 20} MiB, then read another {2 * L2_BYTES >> 20} MiB)"


def time_per_call(fn, steps, warmup, flush=None):
    """Median/mean device time (us) of fn, one CUDA-event pair per call on the
    current stream; an optional L2 flush between calls is outside the events."""
    import torch
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    for i in range(steps):
        if flush is not None:
            flush()
        starts[i].record()
        fn()
        ends[i].record()
    torch.cuda.synchronize()
    ts = [s.elapsed_time(e) * 1e3 for s, e in zip(starts, ends)]
    return statistics.median(ts), sum(ts) / len(ts)


def time_pair(fn_a, fn_b, steps, warmup, flush=None):
    """Device times (us) of two calls measured alternately so that clock and
    thermal drift affect both alike, the order within a pair swapped every
    other pair (a b, b a, a b, ...) so that neither call always follows the
    other: (median a, median b, samples a, samples b), sample i of a and of
    b forming one pair."""
    import torch
    for _ in range(warmup):
        fn_a()
        fn_b()
    torch.cuda.synchronize()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(steps)]
    for i in range(steps):
        order = ((0, fn_a), (1, fn_b)) if i % 2 == 0 else ((1, fn_b), (0, fn_a))
        for j, fn in order:
            if flush is not None:
                flush()
            ev[i][2 * j].record()
            fn()
            ev[i][2 * j + 1].record()
    torch.cuda.synchronize()
    ta = [e[0].elapsed_time(e[1]) * 1e3 for e in ev]
    tb = [e[2].elapsed_time(e[3]) * 1e3 for e in ev]
    return statistics.median(ta), statistics.median(tb), ta, tb


def paired_overhead(ta, tb, n_boot=4000, seed=0):
    """Overhead of a over b in percent from alternately measured pairs
    (a_i, b_i): the median of the paired differences 100 (a_i - b_i) / b_i,
    and a percentile-bootstrap 95% interval of that median (pairs resampled
    with replacement, n_boot resamples, seeded)."""
    import numpy as np
    a = np.asarray(ta, dtype=np.float64)
    b = np.asarray(tb, dtype=np.float64)
    d = 100.0 * (a - b) / b
    rng = np.random.Generator(np.random.PCG64(seed))
    meds = np.median(d[rng.integers(0, d.size, (n_boot, d.size))], axis=1)
    lo, hi = np.percentile(meds, [2.5, 97.5])
    return float(np.median(d)), float(lo), float(hi)


def measure_overhead(fn_a, fn_b, warmup, flush=None, pairs=200, max_pairs=1600, bound=1.0):
    """Paired overhead of fn_a over fn_b with its 95% interval.  While the
    interval straddles `bound` percent, more pairs are measured (doubling, up
    to max_pairs), so the figure says on which side of the bound it lies
    whenever the noise allows."""
    ta, tb = [], []
    n = pairs
    while True:
        _, _, a, b = time_pair(fn_a, fn_b, n - len(ta), warmup, flush)
        ta += a
        tb += b
        med, lo, hi = paired_overhead(ta, tb)
        if not (lo < bound < hi) or len(ta) >= max_pairs:
            break
        n = min(2 * n, max_pairs)
    return {"median_pct": round(med, 3), "ci95_pct": [round(lo, 3), round(hi, 3)],
            "pairs": len(ta), "t_a_us": round(statistics.median(ta), 2),
            "t_b_us": round(statistics.median(tb), 2)}


def gpu_arm(args, rank, world):
    import numpy as np
    import torch
    import torch.distributed as dist
    import workloads

    torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", 0)))
    props = torch.cuda.get_device_properties(torch.cuda.current_device())
    try:
        gpu_index = f"{props.pci_domain_id:08X}:{props.pci_bus_id:02X}:{props.pci_device_id:02X}.0"
    except AttributeError:
        gpu_index = str(torch.cuda.current_device())
    peak, peak_kind = load_peaks()
    flush = L2Flush()

    # ---- headline: full step on the B=64 batch, CUDA-graph replays ------
    wl = workloads.concurrency_sweep(HEADLINE_BATCH, seed=replica_seed(2, rank), device="cuda")
    st = Step(wl, "fp8")
    g_full = _graph(st.full)
    g_unchecked = _graph(st.unchecked)
    for _ in range(args.warmup):
        g_full.replay()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clocks = ClockSampler(gpu_index)
    clocks.start()
    # keep the GPU busy for ~1 s before the timed steps so that the clock
    # samples describe the same load the timed region runs under
    soak_until = time.perf_counter() + 1.0
    while time.perf_counter() < soak_until:
        for _ in range(200):
            g_full.replay()
        torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        g_full.replay()
    e1.record()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    local_ms = e0.elapsed_time(e1)
    clk = clocks.stop()
    total_ms = reduce_max_time(local_ms, world)
    ms_per_step = total_ms / args.steps
    value = world * HEADLINE_BATCH / (ms_per_step / 1e3)
    kv_bytes = kv_bytes_per_step(wl.seq_lens, wl.num_kv_heads, wl.head_dim, 1)

    # ---- roofline of the dominant kernel: the FP8 attention call ------------
    attn_bytes = attn_algorithmic_bytes(wl.seq_lens, wl.page_size, wl.num_q_heads,
                                        wl.num_kv_heads, wl.head_dim, 1)
    import paged_fp8_kv_attn_b200 as pkv
    clu, ctas, attn_launches = pkv.paged_decode_attn_plan(
        pkv.PKV_KV_FP8, HEADLINE_BATCH, wl.num_q_heads, wl.num_kv_heads, wl.head_dim,
        wl.page_table.shape[1], wl.page_size)
    split = (f"cluster mode, {ctas} CTAs in clusters of {clu}, one launch" if clu
             else f"split-K over {ctas} CTAs + LSE merge")
    # the call's device duration: CUDA-graph replays (no host launch gaps inside
    # the events), one event pair per replay, mean over the timed replays
    g_attn = _graph(lambda: st.attend(True))
    attn_med, attn_mean = time_per_call(g_attn.replay, max(args.steps, 20), args.warmup)
    del g_attn
    achieved = attn_bytes / (attn_mean * 1e-6) / 1e9
    traffic = ncu_traffic_per_launch(wl.logical_tokens() * wl.num_kv_heads)

    # ---- tag-check overhead: full step vs step without the check ---------
    overhead = measure_overhead(g_full.replay, g_unchecked.replay, args.warmup)

    # ---- end to end through the public API with host buffers -------------
    B = HEADLINE_BATCH
    # pinned host staging with the device buffers' packed layout: the step's
    # inputs (q, new K/V, lengths, page table, expected tags) go in with one
    # copy; its results (out, lse, abort mask) come back with one copy.  Two
    # device buffer sets alternate (double buffering, as a serving loop
    # would): the inputs of step i+1 are copied in on one stream and the
    # results of step i-1 copied out on another while step i computes.
    h_in = st.dev_in.cpu().pin_memory()
    h_outs = [torch.empty_like(st.dev_out, device="cpu").pin_memory() for _ in range(2)]
    h2d = h_in.numel()       # bytes copied in per step (packed, 256-byte aligned slots)
    d2h = h_outs[0].numel()  # bytes copied out per step
    sts = [st, st.twin()]
    comp = torch.cuda.current_stream()
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_done = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]

    def e2e_run(n):
        """n double-buffered steps; returns after enqueueing, with every copy
        ordered before the compute stream's next work."""
        with torch.cuda.stream(s_in):
            s_in.wait_stream(comp)
            sts[0].dev_in.copy_(h_in, non_blocking=True)
            ev_in[0].record(s_in)
        for i in range(n):
            cur, nxt = i % 2, (i + 1) % 2
            comp.wait_event(ev_in[cur])
            if i >= 2:
                comp.wait_event(ev_out[cur])      # step i-2's results have left this set
            sts[cur].full()
            ev_done[cur].record(comp)
            if i + 1 < n:
                with torch.cuda.stream(s_in):
                    if i >= 1:
                        s_in.wait_event(ev_done[nxt])   # step i-1 no longer reads this set
                    sts[nxt].dev_in.copy_(h_in, non_blocking=True)
                    ev_in[nxt].record(s_in)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_done[cur])
                h_outs[cur].copy_(sts[cur].dev_out, non_blocking=True)
                ev_out[cur].record(s_out)
        comp.wait_stream(s_out)
        comp.wait_stream(s_in)

    e2e_run(max(args.warmup, 2))
    torch.cuda.synchronize()
    # the same ~1 s of sustained load as before the device-timed steps, so
    # that both figures are taken at the clocks that load settles at
    soak_until = time.perf_counter() + 1.0
    while time.perf_counter() < soak_until:
        e2e_run(50)
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    e0.record()
    e2e_run(args.steps)
    e1.record()
    torch.cuda.synchronize()
    e2e_ms = reduce_max_time(e0.elapsed_time(e1), world) / args.steps
    e2e_value = world * B / (e2e_ms / 1e3)
    assert all(pkv_status_ok(x) for x in sts)
    del sts
    assert pkv_status_ok(st)
    del g_full, g_unchecked, st
    torch.cuda.empty_cache()

    # ---- concurrency sweep, FP8 and BF16 side by side ---------------------
    rows = []
    if not args.no_sweep:
        for b in SWEEP:
            wlb = workloads.concurrency_sweep(b, seed=replica_seed(2, rank), device="cuda")
            row = [b]
            for kv in ("fp8", "bf16"):
                sb = Step(wlb, kv)
                eb = 1 if kv == "fp8" else 2
                byts = attn_algorithmic_bytes(wlb.seq_lens, wlb.page_size, wlb.num_q_heads,
                                              wlb.num_kv_heads, wlb.head_dim, eb)
                fl = flush if byts < 2 * L2_BYTES else None
                gf = _graph(sb.full)
                gu = _graph(sb.unchecked)
                ga = _graph(lambda: sb.attend(True))
                ov = measure_overhead(gf.replay, gu.replay, args.warmup, fl)
                t_a, _ = time_per_call(ga.replay, max(args.steps, 50), args.warmup, fl)
                gbs = byts / (t_a * 1e-6) / 1e9
                row += [round(t_a, 2), round(gbs / peak, 4), round(gbs / NOMINAL_HBM_GBS, 4),
                        round(b / (ov["t_a_us"] * 1e-6), 1), ov["median_pct"], *ov["ci95_pct"]]
                assert pkv_status_ok(sb)
                del gf, gu, ga, sb
                torch.cuda.empty_cache()
            rows.append(row)
            del wlb
            torch.cuda.empty_cache()
    sweep = {
        "cols": ["B"] + [f"{kv}_{c}" for kv in ("fp8", "bf16")
                         for c in ("attn_us", "frac_meas", "frac_8tbs", "step_tok_s",
                                   "chk_pct", "chk_ci_lo", "chk_ci_hi")],
        "rows": rows,
        "how": "attn: CUDA-graph replays of the attention call; step: check+append then "
               "attention; chk: paired median overhead of the checked step over the unchecked "
               "one, bootstrap 95% CI; L2 flushed between calls when KV < 2x L2 (B=1, 8 FP8; "
               "B=1 BF16)"}
    by_b = {r[0]: r for r in rows}
    target = {"goal_frac_of_8tbs": 0.70,
              "fp8_attn_frac_of_8tbs": {str(b): by_b[b][3] for b in (32, 64) if b in by_b}}
    target["met_at_32_and_64"] = (len(target["fp8_attn_frac_of_8tbs"]) == 2 and
                                  all(v >= 0.70 for v in target["fp8_attn_frac_of_8tbs"].values()))

    # ---- INT4 weight dequantisation GEMV (decode), against concurrency ----
    int4 = [] if args.no_int4 else int4_gemv_lines(args, rank, peak)

    # ---- capacity, integrity stress, ragged + prefix workloads -----------
    configs = {} if args.no_configs else config_lines(args, rank, peak)

    line = {
        "metric": METRIC,
        "value": round(value, 1),
        "unit": UNIT,
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_per_step, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "e4m3 cache; f16 tensor-core products, f32 accumulate",
        "data": "synthetic (seeded; Q~N(0,1), K/V~N(0,1) with 1% x20 outliers, bf16 -> e4m3 at amax/448)",
        "config": headline_config(world),
        "launch": "CUDA graph of the step (programmatic dependent launch)",
        "step_kv_gbs": round(kv_bytes / (ms_per_step * 1e-3) / 1e9, 1),
        "step_kv_frac_of_8tbs": round(kv_bytes / (ms_per_step * 1e-3) / 1e9 / NOMINAL_HBM_GBS, 4),
        "check_overhead_pct": overhead["median_pct"],
        "check_overhead_ci95_pct": overhead["ci95_pct"],
        "roofline": {"kernel": f"paged_decode_attn_fp8 ({split})",
                     "bound": "hbm", "achieved": round(achieved, 1), "peak": peak,
                     "unit": "GB/s", "frac": round(achieved / peak, 4),
                     "peak_kind": f"{peak_kind} (copy bandwidth)",
                     "traffic": None if traffic is None else round(traffic),
                     "algorithmic_bytes_per_launch": attn_bytes,
                     "launch_us_mean": round(attn_mean, 2),
                     "timing": "CUDA-graph replays of the call, one event pair each, mean"},
        "e2e": {"value": round(e2e_value, 1), "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h,
                "api": "python binding -> C ABI, eager calls; one pinned H2D copy of the "
                       "packed inputs and one D2H copy of the packed results per step, "
                       "double-buffered on two copy streams (step i+1 in and step i-1 out "
                       "while step i computes); timed after ~1 s of the same load, as the "
                       "device-timed steps are"},
        "gpu_launches": (1 + attn_launches) * args.steps,   # check+append, then attention
        "clocks": clk,
        "int4_gemv": int4,
        "configs": configs,
        # kept last so that a reader of the line's tail sees them
        "sweep": sweep,
        "target": target,
    }
    return line


def _kv_row(byts, t_us, peak):
    gbs = byts / (t_us * 1e-6) / 1e9
    return {"gbs": round(gbs, 1), "frac_of_measured": round(gbs / peak, 4),
            "frac_of_8tbs": round(gbs / NOMINAL_HBM_GBS, 4)}


def config_lines(args, rank, peak):
    """The capacity, integrity-stress and ragged + prefix workloads, each
    larger than L2 (no flush), CUDA-graph replays of the checked step
    (fused check + append, then attention) and of the attention call."""
    import numpy as np
    import torch
    import workloads
    steps = max(args.steps, 20)
    out = {}

    # capacity: the same byte budget as 64 FP8 or 32 BF16 requests of 21,440
    # tokens; both read ~2.81 GB of KV per step
    cap = {}
    for kv in ("fp8", "bf16"):
        wl = workloads.capacity(kv, seed=replica_seed(3, rank), device="cuda")
        st = Step(wl, kv)
        eb = 1 if kv == "fp8" else 2
        byts = attn_algorithmic_bytes(wl.seq_lens, wl.page_size, wl.num_q_heads,
                                      wl.num_kv_heads, wl.head_dim, eb)
        gf = _graph(st.full)
        ga = _graph(lambda: st.attend(True))
        t_step, _ = time_per_call(gf.replay, steps, args.warmup)
        t_a, _ = time_per_call(ga.replay, steps, args.warmup)
        torch.cuda.synchronize()
        assert pkv_status_ok(st) and not bool(st.abort.any())
        cap[kv] = {"batch": wl.batch, "tokens_per_request": int(wl.seq_lens[0]),
                   "cached_tokens": wl.logical_tokens(),
                   "kv_bytes": kv_bytes_per_step(wl.seq_lens, wl.num_kv_heads, wl.head_dim, eb),
                   "step_us": round(t_step, 2),
                   "tokens_per_s": round(wl.batch / (t_step * 1e-6), 1),
                   "attn_us": round(t_a, 2), **_kv_row(byts, t_a, peak)}
        del gf, ga, st, wl
        torch.cuda.empty_cache()
    cap["fp8_over_bf16_tokens_per_s"] = round(cap["fp8"]["tokens_per_s"] /
                                              cap["bf16"]["tokens_per_s"], 3)
    out["capacity"] = cap

    # integrity stress: 256 requests, L ~ U[1024, 16384], pages reallocated
    # three times; the overhead is measured with every expected tag current
    # (equal work), then 0.1% of the entries are made stale
    wl = workloads.integrity_stress(seed=replica_seed(4, rank), device="cuda")
    st = Step(wl, "fp8")
    stale_tags = wl.expected_tags.copy()
    clean = wl.expected_tags.copy()
    for b, j in wl.stale_entries:
        clean[b, j] = wl.page_tags[wl.page_table[b, j]]
    st.expected.copy_(torch.from_numpy(clean.view(np.int32)))
    byts = attn_algorithmic_bytes(wl.seq_lens, wl.page_size, wl.num_q_heads,
                                  wl.num_kv_heads, wl.head_dim, 1)
    gf = _graph(st.full)
    gu = _graph(st.unchecked)
    gc = _graph(lambda: (st.check(), st.attend(True)))
    ga = _graph(lambda: st.attend(False))
    ov_fused = measure_overhead(gf.replay, gu.replay, args.warmup)
    ov_sep = measure_overhead(gc.replay, ga.replay, args.warmup)
    t_full, t_unch = ov_fused["t_a_us"], ov_fused["t_b_us"]
    t_ca, t_a = ov_sep["t_a_us"], ov_sep["t_b_us"]
    torch.cuda.synchronize()
    assert not bool(st.abort.any())
    st.expected.copy_(torch.from_numpy(stale_tags.view(np.int32)))
    t_stale, _ = time_per_call(gf.replay, steps, args.warmup)
    torch.cuda.synchronize()
    aborted = np.nonzero(st.abort.cpu().numpy())[0].tolist()
    want = sorted({b for b, _ in wl.stale_entries})
    live = [b for b in range(wl.batch) if b not in set(want)]
    live_bytes = attn_algorithmic_bytes(wl.seq_lens[live], wl.page_size, wl.num_q_heads,
                                        wl.num_kv_heads, wl.head_dim, 1)
    assert pkv_status_ok(st)
    out["integrity_stress"] = {
        "batch": wl.batch, "kv_tokens": wl.logical_tokens(),
        "page_table_entries": int(sum(wl.used_pages(b) for b in range(wl.batch))),
        "step_us": t_full, "step_unchecked_us": t_unch,
        "check_overhead_pct": ov_fused["median_pct"],
        "check_overhead_ci95_pct": ov_fused["ci95_pct"],
        "tag_check_then_attn_us": t_ca, "attn_alone_us": t_a,
        "separate_check_overhead_pct": ov_sep["median_pct"],
        "separate_check_overhead_ci95_pct": ov_sep["ci95_pct"],
        "attn": _kv_row(byts, t_a, peak),
        "stale": {"entries": len(wl.stale_entries), "requests": len(want),
                  "aborted_match": aborted == want, "step_us": round(t_stale, 2),
                  "bytes_of_live_requests": live_bytes,
                  **_kv_row(live_bytes, t_stale, peak)},
        "overhead": "graph replays alternated: (fused check + append, attention with the "
                    "mask) vs (append, attention without it); and (kv_tag_check, attention) "
                    "vs attention alone; median of paired differences, bootstrap 95% CI"}
    assert aborted == want, "abort mask differs from the stale requests"
    del gf, gu, gc, ga, st, wl
    torch.cuda.empty_cache()

    # ragged + prefix: 512 requests, lognormal lengths, groups of 8 sharing a
    # 4,096-token prefix; GB/s against unique bytes (L2 serves the repeats)
    wl = workloads.ragged_prefix(seed=replica_seed(5, rank), device="cuda")
    st = Step(wl, "fp8")
    logical = attn_algorithmic_bytes(wl.seq_lens, wl.page_size, wl.num_q_heads,
                                     wl.num_kv_heads, wl.head_dim, 1)
    kv_logical = kv_bytes_per_step(wl.seq_lens, wl.num_kv_heads, wl.head_dim, 1)
    u_tok = unique_kv_tokens(wl.seq_lens, wl.page_table, wl.page_size)
    unique = logical - kv_logical + u_tok * wl.num_kv_heads * wl.head_dim * 2
    gf = _graph(st.full)
    ga = _graph(lambda: st.attend(True))
    t_step, _ = time_per_call(gf.replay, steps, args.warmup)
    t_a, _ = time_per_call(ga.replay, steps, args.warmup)
    torch.cuda.synchronize()
    assert pkv_status_ok(st) and not bool(st.abort.any())
    # the shared-prefix call on the same batch (groups found on the device)
    import paged_fp8_kv_attn_b200 as pkv
    B, Hq, D = wl.q.shape
    wsp = pkv.alloc_prefix_workspace(B, Hq, wl.num_kv_heads, D)
    begin = torch.zeros(B, dtype=torch.int32, device="cuda")

    def attend_prefix():
        pkv.paged_decode_attn_fp8_prefix(st.q, st.k_cache, st.v_cache, wl.k_scale, wl.v_scale,
                                         st.page_table, st.seq_lens, wl.sm_scale, st.out, st.lse,
                                         wsp, abort=st.abort, chunk_begin_out=begin)

    gp = _graph(attend_prefix)
    t_p, _ = time_per_call(gp.replay, steps, args.warmup)
    torch.cuda.synchronize()
    assert pkv.workspace_status(wsp) == 0
    n_chunks = np.asarray([(int(L) + 63) // 64 for L in wl.seq_lens])
    cb = begin.cpu().numpy()
    lens = wl.seq_lens.astype(np.int64)
    out["ragged_prefix"] = {
        "batch": wl.batch, "logical_tokens": int(lens.sum()), "unique_tokens": u_tok,
        "min_len": int(lens.min()), "median_len": int(np.median(lens)), "max_len": int(lens.max()),
        "requests_over_8192": int((lens > 8192).sum()),
        "logical_bytes": logical, "unique_bytes": unique,
        "step_us": round(t_step, 2), "tokens_per_s": round(wl.batch / (t_step * 1e-6), 1),
        "attn_us": round(t_a, 2),
        "attn_logical_gbs": round(logical / (t_a * 1e-6) / 1e9, 1),
        "attn_unique": _kv_row(unique, t_a, peak),
        "shared_prefix_call": {
            "attn_us": round(t_p, 2), "attn_unique": _kv_row(unique, t_p, peak),
            "requests_in_tiles": int((cb > 0).sum()),
            "requests_finished_in_tiles": int(((cb > 0) & (cb == n_chunks)).sum()),
            "chunks_in_tiles": int(cb.sum())}}
    del gf, ga, gp, st, wl, wsp
    torch.cuda.empty_cache()
    return out


def int4_algorithmic_bytes(batch, n, k, group):
    """Codes + scales + x + y of one GEMV call."""
    return n * k // 2 + n * (k // group) * 2 + batch * k * 2 + batch * n * 2


def int4_gemv_lines(args, rank, peak):
    """One entry per concurrency level: device time of int4_dequant_gemv on
    one synthetic [32768 x 8192] INT4 weight matrix (134 MB of codes and
    scales, larger than L2, so no flush is needed)."""
    import torch
    import paged_fp8_kv_attn_b200 as pkv
    import workloads
    rows = []
    base = workloads.int4_gemv_case(1, seed=replica_seed(6, rank), device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    for b in workloads.INT4_BATCHES:
        case = workloads.int4_gemv_case(b, seed=replica_seed(6, rank), device="cuda",
                                        w_tiles=base.w_tiles, scales=base.scales)
        y = torch.empty((b, case.n), dtype=torch.bfloat16, device="cuda")
        g = _graph(lambda: pkv.int4_dequant_gemv(case.x, case.w_tiles, case.scales, y,
                                                 case.group, status=status))
        t_med, t_mean = time_per_call(g.replay, max(args.steps, 20), args.warmup)
        byts = int4_algorithmic_bytes(b, case.n, case.k, case.group)
        gbs = byts / (t_med * 1e-6) / 1e9
        rows.append({"batch": b, "us": round(t_med, 2), "us_mean": round(t_mean, 2),
                     "gbs": round(gbs, 1), "frac_of_measured": round(gbs / peak, 4),
                     "frac_of_8tbs": round(gbs / NOMINAL_HBM_GBS, 4),
                     "tflops": round(2.0 * b * case.n * case.k / (t_med * 1e-6) / 1e12, 1),
                     "tokens_per_s": round(b / (t_med * 1e-6), 1)})
        del g, y, case
    torch.cuda.synchronize()
    assert int(status.item()) == 0, "int4_dequant_gemv reported an expired wait"
    shape = {"n": base.n, "k": base.k, "group": base.group,
             "algorithmic_bytes": "n k/2 + 2 n k/group + 2 B k + 2 B n",
             "l2": "weights larger than L2 (no flush)",
             "dtype": "int4 codes, bf16 scales and x, bf16 tensor-core products, f32 accumulate"}
    del base
    torch.cuda.empty_cache()
    return {"shape": shape, "rows": rows}


def pkv_status_ok(st) -> bool:
    return st.pkv.workspace_status(st.ws) == 0


# --------------------------------------------------------------------------
# CPU oracle (baseline leg and reference arm)
# --------------------------------------------------------------------------

class OracleSampler:
    """The CPU oracle, as it stands, on a bounded sample of the headline
    workload: R requests with the headline's per-request shape (8,192 tokens,
    64 q heads / 8 KV heads, D=128, P=64, FP8).  One oracle step is the tag
    check and the append of those requests plus attention over all their
    (request, KV head) items, spread over the host cores."""

    def __init__(self, requests: int, seed: int = 2):
        import numpy as np
        import oracle
        import workloads
        from workloads import bf16_bits
        self.oracle = oracle
        self.np = np
        self.threads = os.cpu_count() or 1
        self.requests = requests
        wl = workloads.concurrency_sweep(requests, seed=seed, device="cpu", context=CONTEXT)
        self.wl = wl
        self.kbits, self.vbits = bf16_bits(wl.k_pool), bf16_bits(wl.v_pool)
        self.kc = self._quantize(self.kbits, wl.k_scale)
        self.vc = self._quantize(self.vbits, wl.v_scale)
        self.q = bf16_bits(wl.q)
        self.kn, self.vn = bf16_bits(wl.k_new), bf16_bits(wl.v_new)

    def _quantize(self, bits, scale):
        from concurrent.futures import ThreadPoolExecutor
        flat = bits.reshape(-1)
        parts = self.np.array_split(self.np.arange(flat.size), self.threads)
        out = self.np.empty(flat.size, dtype=self.np.uint8)

        def job(ix):
            out[ix[0]: ix[-1] + 1] = self.oracle.quantize_bf16(flat[ix[0]: ix[-1] + 1], scale)

        with ThreadPoolExecutor(self.threads) as ex:
            list(ex.map(job, [p for p in parts if p.size]))
        return out.reshape(bits.shape)

    def step(self, n_items=None, threads=None):
        """Seconds of one oracle step over the first n_items items (all by
        default) on `threads` threads (all host cores by default)."""
        wl, o = self.wl, self.oracle
        total = wl.batch * wl.num_kv_heads
        items = self.np.arange(total if n_items is None else min(n_items, total),
                               dtype=self.np.int32)
        t0 = time.perf_counter()
        abort, _ = o.kv_tag_check(wl.page_tags, wl.page_table, wl.expected_tags, wl.seq_lens,
                                  wl.page_size)
        o.kv_append_fp8(self.kn, self.vn, wl.page_table, wl.seq_lens, wl.page_size, wl.k_scale,
                        wl.v_scale, self.kc, self.vc, abort)
        o.paged_decode_attn(self.q, self.kc, self.vc, wl.page_table, wl.seq_lens,
                            wl.num_kv_heads, wl.page_size, wl.sm_scale, wl.k_scale, wl.v_scale,
                            abort=abort, items=items, threads=threads or self.threads)
        return time.perf_counter() - t0, int(items.size)


def oracle_requests_per_step(threads=None):
    """Requests per oracle step: enough (request, KV head) items, 8 per
    request, to give every host core one."""
    threads = threads or os.cpu_count() or 1
    return max(1, -(-threads // 8))


def oracle_run(steps, warmup, seed=2):
    """The oracle timed over whole steps of R requests (R from
    oracle_requests_per_step) on all host cores, plus one item on a single
    thread.  tokens/s = R requests per step / measured step time (each request
    yields one token per decode step)."""
    requests = oracle_requests_per_step()
    sampler = OracleSampler(requests=requests, seed=seed)
    for _ in range(warmup):
        sampler.step()
    times = [sampler.step()[0] for _ in range(steps)]
    step_s = sum(times) / len(times)
    t1, _ = sampler.step(n_items=1, threads=1)
    items_per_request = sampler.wl.num_kv_heads
    return {"requests": requests, "items": requests * items_per_request,
            "threads": sampler.threads, "steps": steps, "step_s": step_s,
            "tokens_per_s": requests / step_s,
            "single_thread_item_s": t1,
            "single_thread_tokens_per_s": 1.0 / (t1 * items_per_request)}


def _cpu_baseline_entry(r):
    return {"value": round(r["tokens_per_s"], 4), "unit": UNIT, "cores": r["threads"],
            "kind": "oracle",
            "sample": f"{r['steps']} oracle steps, each the tag check, append and attention of "
                      f"{r['requests']} request(s) ({r['items']} (request, KV head) items) of "
                      f"the batch-64 step's shape (8,192 tokens, P=64, 64/8 heads, D=128, FP8) "
                      f"on {r['threads']} threads; {r['step_s'] * 1e3:.1f} ms per step",
            "single_thread": {"value": round(r["single_thread_tokens_per_s"], 4), "unit": UNIT,
                              "cores": 1,
                              "sample": f"one item on one thread ({r['single_thread_item_s']:.3f} "
                                        f"s), times the 8 items of a request"}}


def oracle_sample(target_s: float = 10.0, seed: int = 2):
    """cpu_baseline entry of the GPU arm's line: the same measurement as the
    reference arm, with as many steps as fit in about target_s seconds."""
    probe = OracleSampler(requests=oracle_requests_per_step(), seed=seed)
    t, _ = probe.step()
    del probe
    steps = int(min(50, max(3, target_s / max(t, 1e-6))))
    return _cpu_baseline_entry(oracle_run(steps, 1, seed))


def reference_arm(args, rank, world, gpu_config=None):
    """The oracle as the reference arm: each step is one oracle step over R
    requests of the headline shape (enough items for every host core);
    ms_per_step is that step's measured wall time and tokens/s = R / step
    time.  Rank 0 only."""
    if rank != 0:
        return None
    r = oracle_run(args.steps, args.warmup)
    value = r["tokens_per_s"]
    return {"impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": UNIT,
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(r["step_s"] * 1e3, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64 (oracle)",
            "data": "synthetic (seeded)",
            "config": gpu_config if gpu_config is not None else headline_config(world),
            "cpu_baseline": _cpu_baseline_entry(r),
            "e2e": {"value": round(value, 4), "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


# --------------------------------------------------------------------------

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-sweep", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-int4", action="store_true")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the capacity, integrity-stress and ragged + prefix workloads")
    ap.add_argument("--kernel-only", choices=["fp8", "bf16", "int4", "prefix"], default=None,
                    help="profiling target: run only the decode step (fp8/bf16) on a --batch "
                         "request concurrency-sweep batch, only the INT4 GEMV at --batch, or "
                         "only the shared-prefix attention call on a --batch request ragged "
                         "prefix-reuse batch; warmup + steps times; prints nothing")
    ap.add_argument("--batch", type=int, default=16)
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if args.impl == "reference":
        line = reference_arm(args, rank, world)
        if line is not None:
            print(json.dumps(line), flush=True)
        return

    import torch
    if args.kernel_only == "int4":
        import paged_fp8_kv_attn_b200 as pkv
        import workloads
        case = workloads.int4_gemv_case(args.batch, device="cuda")
        y = torch.empty((case.batch, case.n), dtype=torch.bfloat16, device="cuda")
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        for _ in range(args.warmup + args.steps):
            pkv.int4_dequant_gemv(case.x, case.w_tiles, case.scales, y, case.group, status=status)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        return
    if args.kernel_only == "prefix":
        import paged_fp8_kv_attn_b200 as pkv
        import workloads
        wl = workloads.ragged_prefix(device="cuda", batch=args.batch)
        st = Step(wl, "fp8")
        del wl.k_pool, wl.v_pool     # (the FP8 caches are built)
        torch.cuda.empty_cache()
        B, Hq, D = wl.q.shape
        wsp = pkv.alloc_prefix_workspace(B, Hq, wl.num_kv_heads, D)
        for _ in range(args.warmup + args.steps):
            pkv.paged_decode_attn_fp8_prefix(st.q, st.k_cache, st.v_cache, wl.k_scale, wl.v_scale,
                                             st.page_table, st.seq_lens, wl.sm_scale, st.out,
                                             st.lse, wsp, abort=st.abort)
        torch.cuda.synchronize()
        assert pkv.workspace_status(wsp) == 0
        return
    if args.kernel_only:
        import workloads
        wl = workloads.concurrency_sweep(args.batch, device="cuda")
        st = Step(wl, args.kernel_only)
        for _ in range(args.warmup + args.steps):
            st.full()
        torch.cuda.synchronize()
        assert pkv_status_ok(st)
        return
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", 0)))
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    try:
        line = gpu_arm(args, rank, world)
        if rank == 0 and not args.no_cpu_baseline:
            line["cpu_baseline"] = oracle_sample()
        if rank == 0:
            for k in ("sweep", "target"):      # keep the sweep at the end of the line
                line[k] = line.pop(k)
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.barrier()
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
