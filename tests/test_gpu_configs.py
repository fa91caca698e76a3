"""GPU parity at the workloads' full sizes, in the launch configuration the
benchmark times (default grid, check -> append -> attention on one stream),
on sampled items the oracle computes one by one.
"""
import numpy as np
import pytest
import torch

import paged_fp8_kv_attn_b200 as pkv
import workloads

from _pkv_helpers import DeviceBatch, compare, oracle_step, sample_items

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("batch", [1, 8, 32, 64])
@pytest.mark.parametrize("kv", ["fp8", "bf16"])
def test_concurrency_sweep_sampled(cuda_device, batch, kv):
    wl = workloads.concurrency_sweep(batch, device="cuda")
    db = DeviceBatch(wl, kv_dtype=kv)
    db.step(check=True, append=True)
    out, lse = db.outputs()
    items = sample_items(wl, 6, seed=batch, must=[0, wl.batch * wl.num_kv_heads - 1])
    ref_o, ref_l, ref_abort = oracle_step(wl, items, kv_dtype=kv)
    assert not ref_abort.any() and not db.abort.any()
    compare(wl, items, out, lse, ref_o, ref_l, label=f"{kv} B={batch}")
    assert pkv.workspace_status(db.ws) == 0


@pytest.mark.parametrize("kv", ["fp8", "bf16"])
def test_capacity_sampled(cuda_device, kv):
    wl = workloads.capacity(kv, device="cuda")
    db = DeviceBatch(wl, kv_dtype=kv)
    db.step(check=True, append=True)
    out, lse = db.outputs()
    items = sample_items(wl, 4, seed=3)
    ref_o, ref_l, _ = oracle_step(wl, items, kv_dtype=kv)
    compare(wl, items, out, lse, ref_o, ref_l, label=f"capacity {kv}")


def test_integrity_stress_sampled(cuda_device):
    wl = workloads.integrity_stress(device="cuda")
    db = DeviceBatch(wl, kv_dtype="fp8")
    db.step(check=True, append=True)
    out, lse = db.outputs()
    ref_abort = oracle_step(wl, [0], kv_dtype="fp8")[2]
    assert np.array_equal(db.abort.cpu().numpy(), ref_abort)
    stale_req = sorted({b for b, _ in wl.stale_entries})
    assert ref_abort.sum() == len(stale_req) > 0
    dead = [b * wl.num_kv_heads + h for b in stale_req[:2] for h in (0, 7)]
    items = sample_items(wl, 6, seed=4, must=dead)
    ref_o, ref_l, _ = oracle_step(wl, items, kv_dtype="fp8")
    compare(wl, items, out, lse, ref_o, ref_l, label="integrity stress")
    for b in stale_req:
        assert np.all(np.isneginf(lse[b])) and not out[b].any()


def test_ragged_prefix_sampled(cuda_device):
    wl = workloads.ragged_prefix(device="cuda")
    assert wl.unique_pages() < sum(wl.used_pages(b) for b in range(wl.batch))
    db = DeviceBatch(wl, kv_dtype="fp8")
    db.step(check=True, append=True)
    out, lse = db.outputs()
    shortest = int(np.argmin(wl.seq_lens)) * wl.num_kv_heads
    items = sample_items(wl, 8, seed=5, must=[shortest, 8 * wl.num_kv_heads + 3])
    ref_o, ref_l, _ = oracle_step(wl, items, kv_dtype="fp8")
    compare(wl, items, out, lse, ref_o, ref_l, label="ragged prefix")
    assert pkv.workspace_status(db.ws) == 0
