"""Helpers shared by the GPU parity tests: run the CUDA path through the C ABI
and the CPU oracle on the same seeded inputs, and compare.

The oracle never receives anything the CUDA path computed: both sides start
from the workload's bf16 pools, queries and new tokens and each quantises,
appends and attends on its own.
"""
from __future__ import annotations

import math

import numpy as np
import torch

import oracle
import paged_fp8_kv_attn_b200 as pkv
from workloads import DecodeBatch, bf16_bits

# Tolerances: bf16 output within atol 1e-2 / rtol 1e-2 of the fp64 oracle;
# LSE within 1e-4 relative, measured against max(|lse|, 1) (an absolute error
# in LSE is a relative error of the softmax normaliser).
OUT_ATOL = 1e-2
OUT_RTOL = 1e-2
LSE_RTOL = 1e-4


class DeviceBatch:
    """A workload's inputs on the GPU plus the outputs of one decode step."""

    def __init__(self, wl: DecodeBatch, device="cuda", kv_dtype="fp8"):
        self.wl = wl
        self.kv_dtype = kv_dtype
        dev = torch.device(device)
        self.q = wl.q.to(dev).contiguous()
        self.k_new = wl.k_new.to(dev).contiguous()
        self.v_new = wl.v_new.to(dev).contiguous()
        self.page_table = torch.from_numpy(wl.page_table).to(dev)
        self.seq_lens = torch.from_numpy(wl.seq_lens).to(dev)
        self.page_tags = torch.from_numpy(wl.page_tags.view(np.int32)).to(dev)
        self.expected = torch.from_numpy(wl.expected_tags.view(np.int32)).to(dev)
        B, Hq, D = wl.q.shape
        self.out = torch.empty((B, Hq, D), dtype=torch.bfloat16, device=dev)
        self.lse = torch.empty((B, Hq), dtype=torch.float32, device=dev)
        self.abort = torch.zeros(B, dtype=torch.uint8, device=dev)
        self.num_aborted = torch.zeros(1, dtype=torch.int32, device=dev)
        if kv_dtype == "fp8":
            kp = wl.k_pool.to(dev)
            vp = wl.v_pool.to(dev)
            self.k_cache = torch.empty(kp.shape, dtype=torch.uint8, device=dev)
            self.v_cache = torch.empty(vp.shape, dtype=torch.uint8, device=dev)
            ids = torch.arange(wl.num_pages, dtype=torch.int32, device=dev)
            pkv.kv_requant_pages_fp8(kp, ids, self.k_cache, ids, wl.k_scale)
            pkv.kv_requant_pages_fp8(vp, ids, self.v_cache, ids, wl.v_scale)
            del kp, vp
        else:
            self.k_cache = wl.k_pool.to(dev).contiguous().clone()
            self.v_cache = wl.v_pool.to(dev).contiguous().clone()
        self.kv_code = pkv.PKV_KV_FP8 if kv_dtype == "fp8" else pkv.PKV_KV_BF16
        self.ws = None

    def workspace(self, num_ctas=0):
        wl = self.wl
        n = pkv.paged_decode_attn_workspace_size(self.kv_code, wl.batch, wl.num_q_heads,
                                                 wl.num_kv_heads, wl.head_dim, num_ctas)
        if self.ws is None or self.ws.numel() < n:
            self.ws = torch.zeros(n, dtype=torch.uint8, device=self.q.device)
        return self.ws

    def tag_check(self):
        wl = self.wl
        pkv.kv_tag_check(self.page_tags, self.page_table, self.expected, self.seq_lens,
                         wl.page_size, self.abort, self.num_aborted)

    def append(self, use_abort=True):
        wl = self.wl
        ab = self.abort if use_abort else None
        if self.kv_dtype == "fp8":
            pkv.kv_append_fp8(self.k_new, self.v_new, self.page_table, self.seq_lens, wl.page_size,
                              wl.k_scale, wl.v_scale, self.k_cache, self.v_cache, ab)
        else:
            pkv.kv_append_bf16(self.k_new, self.v_new, self.page_table, self.seq_lens,
                               wl.page_size, self.k_cache, self.v_cache, ab)

    def attend(self, use_abort=True, num_ctas=0):
        wl = self.wl
        ab = self.abort if use_abort else None
        ws = self.workspace(num_ctas)
        if self.kv_dtype == "fp8":
            pkv.paged_decode_attn_fp8(self.q, self.k_cache, self.v_cache, wl.k_scale, wl.v_scale,
                                      self.page_table, self.seq_lens, wl.sm_scale, self.out,
                                      self.lse, ws, abort=ab, num_ctas=num_ctas)
        else:
            pkv.paged_decode_attn_bf16(self.q, self.k_cache, self.v_cache, self.page_table,
                                       self.seq_lens, wl.sm_scale, self.out, self.lse, ws,
                                       abort=ab, num_ctas=num_ctas)

    def check_append(self):
        wl = self.wl
        if self.kv_dtype == "fp8":
            pkv.kv_check_append_fp8(self.page_tags, self.page_table, self.expected, self.seq_lens,
                                    wl.page_size, self.k_new, self.v_new, wl.k_scale, wl.v_scale,
                                    self.k_cache, self.v_cache, self.abort, self.num_aborted)
        else:
            pkv.kv_check_append_bf16(self.page_tags, self.page_table, self.expected,
                                     self.seq_lens, wl.page_size, self.k_new, self.v_new,
                                     self.k_cache, self.v_cache, self.abort, self.num_aborted)

    def step(self, check=True, append=True, num_ctas=0, fused=True):
        """One decode step.  With check and append, fused=True uses the fused
        check+append call (the benchmark's configuration); fused=False the two
        separate calls."""
        if check and append and fused:
            self.check_append()
        else:
            if check:
                self.tag_check()
            if append:
                self.append(use_abort=check)
        self.attend(use_abort=check, num_ctas=num_ctas)
        torch.cuda.synchronize()

    def outputs(self):
        out = self.out.float().cpu().numpy().astype(np.float64)
        lse = self.lse.cpu().numpy().astype(np.float64)
        return out, lse


def oracle_step(wl: DecodeBatch, items, kv_dtype="fp8", check=True, append=True,
                threads=8, table_override=None, lens_override=None):
    """The oracle's own decode step on the pages the listed items read.

    items: list of b * Hkv + kv_head.  Returns (out, lse, abort) where out/lse
    are filled for the listed items only.  The pages those requests use are
    gathered into a compact pool (host-side indexing only), quantised by the
    oracle (FP8), given the new token by the oracle's append, then attended.
    """
    table = wl.page_table if table_override is None else table_override
    lens = wl.seq_lens if lens_override is None else lens_override
    B = wl.batch
    P = wl.page_size
    abort = np.zeros(B, dtype=np.uint8)
    if check:
        abort, _ = oracle.kv_tag_check(wl.page_tags, table, wl.expected_tags, lens, P)
    reqs = sorted({int(i) // wl.num_kv_heads for i in items})
    used = set()
    for b in reqs:
        L = int(lens[b])
        if 1 <= L <= table.shape[1] * P:
            n = (L + P - 1) // P
            used.update(int(x) for x in table[b, :n] if 0 <= int(x) < wl.num_pages)
    pages = sorted(used) if used else [0]
    remap = {p: i for i, p in enumerate(pages)}
    # entries that name a page the sampled requests read are remapped into the
    # compact pool; every other entry (including ids outside [0, NP)) becomes -1,
    # which is just as invalid for the compact pool
    ctable = np.full_like(table, -1)
    for b in reqs:
        for j in range(table.shape[1]):
            p = int(table[b, j])
            if p in remap:
                ctable[b, j] = remap[p]
    idx = torch.tensor(pages, dtype=torch.long)
    k_bits = bf16_bits(wl.k_pool.index_select(0, idx.to(wl.k_pool.device)))
    v_bits = bf16_bits(wl.v_pool.index_select(0, idx.to(wl.v_pool.device)))
    if kv_dtype == "fp8":
        kc = oracle.quantize_bf16(k_bits, wl.k_scale)
        vc = oracle.quantize_bf16(v_bits, wl.v_scale)
    else:
        kc, vc = k_bits.copy(), v_bits.copy()
    if append:
        kn, vn = bf16_bits(wl.k_new), bf16_bits(wl.v_new)
        ab = abort if check else None
        if kv_dtype == "fp8":
            oracle.kv_append_fp8(kn, vn, ctable, lens, P, wl.k_scale, wl.v_scale, kc, vc, ab)
        else:
            oracle.kv_append_bf16(kn, vn, ctable, lens, P, kc, vc, ab)
    ks, vs = (wl.k_scale, wl.v_scale) if kv_dtype == "fp8" else (1.0, 1.0)
    out, lse = oracle.paged_decode_attn(bf16_bits(wl.q), kc, vc, ctable, lens,
                                        wl.num_kv_heads, P, wl.sm_scale, ks, vs,
                                        abort=abort if check else None,
                                        items=np.asarray(items, dtype=np.int32), threads=threads)
    return out, lse, abort


def heads_of(wl, items):
    G = wl.num_q_heads // wl.num_kv_heads
    return [(int(i) // wl.num_kv_heads, (int(i) % wl.num_kv_heads) * G + g)
            for i in items for g in range(G)]


# Worst tolerance margin seen by compare() per label in this process:
# max over elements of |out - ref| / (OUT_ATOL + OUT_RTOL |ref|) (1.0 = at the
# tolerance) and of the LSE error over its bound.  Printed in the pytest
# terminal summary.
MARGINS = {}


def compare(wl, items, gpu_out, gpu_lse, ref_out, ref_lse, label=""):
    """Element-wise comparison of the listed items; returns (max |out error|,
    max relative LSE error, worst margin), the margin being the largest
    |out - ref| / (OUT_ATOL + OUT_RTOL |ref|) over the compared outputs."""
    worst_o = worst_l = worst_m = worst_lm = 0.0
    for b, h in heads_of(wl, items):
        go, ro = gpu_out[b, h], ref_out[b, h]
        gl, rl = gpu_lse[b, h], ref_lse[b, h]
        if np.isneginf(rl):
            assert np.isneginf(gl), f"{label} b={b} h={h}: lse {gl} but request is dead"
            assert not go.any(), f"{label} b={b} h={h}: dead request has nonzero output"
            continue
        if np.isnan(rl):
            assert np.isnan(gl), f"{label} b={b} h={h}: expected NaN lse, got {gl}"
            continue
        err = np.abs(go - ro)
        bad = err > OUT_ATOL + OUT_RTOL * np.abs(ro)
        assert not bad.any(), (f"{label} b={b} h={h}: out mismatch at dims "
                               f"{np.nonzero(bad)[0][:8]}: gpu {go[bad][:4]} ref {ro[bad][:4]}")
        lerr = abs(gl - rl) / max(1.0, abs(rl))
        assert lerr <= LSE_RTOL, f"{label} b={b} h={h}: lse {gl} vs {rl} (rel {lerr:.3g})"
        worst_o = max(worst_o, float(err.max()))
        worst_l = max(worst_l, lerr)
        worst_m = max(worst_m, float((err / (OUT_ATOL + OUT_RTOL * np.abs(ro))).max()))
        worst_lm = max(worst_lm, lerr / LSE_RTOL)
    key = label.split(" ")[0] if label else "unlabelled"
    prev = MARGINS.get(key, (0.0, 0.0))
    MARGINS[key] = (max(prev[0], worst_m), max(prev[1], worst_lm))
    return worst_o, worst_l, worst_m


def sample_items(wl, n, seed=0, must=()):
    """n distinct items (b * Hkv + kv_head), always including `must` and the
    longest request."""
    rng = np.random.Generator(np.random.PCG64(seed))
    total = wl.batch * wl.num_kv_heads
    longest = int(np.argmax(wl.seq_lens)) * wl.num_kv_heads + int(rng.integers(wl.num_kv_heads))
    chosen = {longest, *[int(m) for m in must]}
    while len(chosen) < min(n, total):
        chosen.add(int(rng.integers(total)))
    return sorted(chosen)
