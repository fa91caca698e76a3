"""paged_decode_attn_fp8_noalloc: the FP8 attention call for callers that
cannot allocate device memory (a plugin whose host framework owns every
allocation, or a path where cudaMalloc would synchronise the device).

It must give the same results as paged_decode_attn_fp8 with a caller
workspace, call after call, even though its built-in scratch keeps the
previous call's contents.  This file is collected last on purpose.
"""
import numpy as np
import pytest
import torch

import paged_fp8_kv_attn_b200 as pkv
import workloads

from _pkv_helpers import LSE_RTOL, OUT_ATOL, OUT_RTOL, DeviceBatch, compare, oracle_step

pytestmark = pytest.mark.gpu


def _close(a_out, a_lse, b_out, b_lse):
    ao, bo = a_out.float().cpu().numpy(), b_out.float().cpu().numpy()
    al, bl = a_lse.cpu().numpy().astype(np.float64), b_lse.cpu().numpy().astype(np.float64)
    assert np.array_equal(np.isneginf(al), np.isneginf(bl))
    fin = np.isfinite(bl)
    assert np.all(np.abs(ao - bo) <= OUT_ATOL + OUT_RTOL * np.abs(bo))
    assert np.all(np.abs(al[fin] - bl[fin]) <= LSE_RTOL * np.maximum(1.0, np.abs(bl[fin])))


def _run_pair(db, abort=None):
    wl = db.wl
    out_ref = torch.empty_like(db.out)
    lse_ref = torch.empty_like(db.lse)
    pkv.paged_decode_attn_fp8(db.q, db.k_cache, db.v_cache, wl.k_scale, wl.v_scale,
                              db.page_table, db.seq_lens, wl.sm_scale, out_ref, lse_ref,
                              db.workspace(), abort=abort)
    out_na = torch.full_like(db.out, float("nan"))
    lse_na = torch.full_like(db.lse, float("nan"))
    pkv.paged_decode_attn_fp8_noalloc(db.q, db.k_cache, db.v_cache, wl.k_scale, wl.v_scale,
                                      db.page_table, db.seq_lens, wl.sm_scale, out_na, lse_na,
                                      abort=abort)
    torch.cuda.synchronize()
    return out_ref, lse_ref, out_na, lse_na


def test_noalloc_matches_workspace_call_twice(cuda_device):
    # two different batches back to back: the second call runs over scratch
    # that still holds the first call's partial results
    wl1 = workloads.concurrency_sweep(8, device="cuda", context=3000)
    wl2 = workloads.custom([5000, 17, 64, 2500, 1], page_size=64, num_q_heads=64,
                           num_kv_heads=8, head_dim=128, seed=99, device="cuda")
    for wl in (wl1, wl2):
        db = DeviceBatch(wl, kv_dtype="fp8")
        out_ref, lse_ref, out_na, lse_na = _run_pair(db)
        _close(out_na, lse_na, out_ref, lse_ref)
        assert pkv.noalloc_status() == 0


def test_noalloc_matches_the_oracle(cuda_device):
    """The no-allocation call against the CPU oracle directly, on every item
    of a ragged batch that splits requests over several CTAs."""
    wl = workloads.custom([3000, 70, 9000, 1, 640, 64, 65], page_size=64, num_q_heads=64,
                          num_kv_heads=8, head_dim=128, seed=31, device="cuda")
    db = DeviceBatch(wl, kv_dtype="fp8")
    items = list(range(wl.batch * wl.num_kv_heads))
    ref_o, ref_l, _ = oracle_step(wl, items, kv_dtype="fp8", check=False, append=False)
    for ctas in (0, 37):
        out = torch.full_like(db.out, float("nan"))
        lse = torch.full_like(db.lse, float("nan"))
        pkv.paged_decode_attn_fp8_noalloc(db.q, db.k_cache, db.v_cache, wl.k_scale, wl.v_scale,
                                          db.page_table, db.seq_lens, wl.sm_scale, out, lse,
                                          num_ctas=ctas)
        torch.cuda.synchronize()
        compare(wl, items, out.float().cpu().numpy().astype(np.float64),
                lse.cpu().numpy().astype(np.float64), ref_o, ref_l, label=f"noalloc ctas={ctas}")
        assert pkv.noalloc_status() == 0


def test_noalloc_with_aborted_requests(cuda_device):
    wl = workloads.tiny_decode(device="cuda")
    db = DeviceBatch(wl, kv_dtype="fp8")
    db.tag_check()
    for _ in range(2):
        out_ref, lse_ref, out_na, lse_na = _run_pair(db, abort=db.abort)
        _close(out_na, lse_na, out_ref, lse_ref)
        assert torch.isneginf(lse_na[1]).all()


def test_noalloc_rejects_sizes_beyond_its_scratch(cuda_device):
    assert pkv.noalloc_scratch_bytes() == 8 << 20
    wl = workloads.custom([64] * 300, page_size=64, num_q_heads=64, num_kv_heads=8,
                          head_dim=128, seed=5, device="cuda")
    db = DeviceBatch(wl, kv_dtype="fp8")
    with pytest.raises(pkv.PagedKVError, match="built-in scratch"):
        pkv.paged_decode_attn_fp8_noalloc(db.q, db.k_cache, db.v_cache, wl.k_scale, wl.v_scale,
                                          db.page_table, db.seq_lens, wl.sm_scale, db.out,
                                          db.lse)
