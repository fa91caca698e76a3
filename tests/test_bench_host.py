"""Host-side logic of bench.py on the CPU: byte accounting, replica seeds and
the max-over-ranks timing reduction with two gloo ranks."""
import os
import socket
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def test_algorithmic_bytes_headline():
    lens = [8192] * 64
    kv = bench.kv_bytes_per_step(lens, 8, 128, 1)
    assert kv == 64 * 8192 * 8 * 128 * 2 == 1_073_741_824
    total = bench.attn_algorithmic_bytes(lens, 64, 64, 8, 128, 1)
    assert total == kv + 64 * 64 * (2 * 128 * 2 + 4) + 64 * 128 * 4
    assert bench.attn_algorithmic_bytes(lens, 64, 64, 8, 128, 2) - total == kv


def test_replica_seeds_are_distinct():
    seeds = {bench.replica_seed(2, r) for r in range(8)}
    assert len(seeds) == 8


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import datetime
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        out[rank] = bench.reduce_max_time(1.5 + rank, world)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo():
    world = 2
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    ctx = mp.get_context("spawn")
    procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    assert dict(out) == {0: 2.5, 1: 2.5}


def test_reference_arm_line_shape(monkeypatch):
    class FakeSampler:
        threads = 3

        def __init__(self, requests, seed=2):
            self.requests = requests
            self.wl = type("W", (), {"num_kv_heads": 8})()

        def step(self, n_items=None, threads=None):
            return (0.05, 1) if n_items == 1 else (0.5, 8 * self.requests)

    monkeypatch.setattr(bench, "OracleSampler", FakeSampler)
    monkeypatch.setattr(bench.os, "cpu_count", lambda: 16)
    args = type("A", (), {"warmup": 3, "steps": 2})()
    line = bench.reference_arm(args, 0, 1)
    assert line["impl"] == "reference"
    # 16 cores -> 2 requests (16 items) per step; a step of 0.5 s -> 4 tokens/s
    assert line["value"] == 4.0 and line["ms_per_step"] == 500.0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] == 3
    assert line["cpu_baseline"]["value"] == line["value"]
    # one item on one thread in 0.05 s -> a request (8 items) in 0.4 s
    assert line["cpu_baseline"]["single_thread"]["value"] == 2.5
    assert line["e2e"]["h2d_bytes_per_step"] == 0
    # the same workload description as the GPU arm
    assert line["config"] == bench.headline_config(1)
    assert bench.reference_arm(args, 1, 2) is None


def test_oracle_requests_cover_every_core():
    assert bench.oracle_requests_per_step(1) == 1
    assert bench.oracle_requests_per_step(8) == 1
    assert bench.oracle_requests_per_step(9) == 2
    assert bench.oracle_requests_per_step(16) == 2
    assert bench.oracle_requests_per_step(96) == 12


def test_paired_overhead_median_and_interval():
    import numpy as np
    rng = np.random.Generator(np.random.PCG64(1))
    b = 100.0 + rng.normal(0, 1.0, 400)
    a = b * 1.02 + rng.normal(0, 0.2, 400)          # +2% with paired noise
    med, lo, hi = bench.paired_overhead(a, b)
    assert lo <= med <= hi
    assert 1.9 < med < 2.1 and lo > 1.8 and hi < 2.2
    # identical timings: zero with a zero-width interval
    med, lo, hi = bench.paired_overhead(b, b)
    assert med == lo == hi == 0.0
    # seeded: repeatable
    assert bench.paired_overhead(a, b) == bench.paired_overhead(a, b)


def test_measure_overhead_adds_pairs_while_the_interval_straddles_the_bound(monkeypatch):
    import numpy as np
    rng = np.random.Generator(np.random.PCG64(2))
    calls = []

    def fake_time_pair(fa, fb, steps, warmup, flush=None):
        calls.append(steps)
        b = list(100.0 + rng.normal(0, 3.0, steps))
        a = [x * 1.01 for x in b]                      # exactly +1%: always straddles
        a = [x + rng.normal(0, 3.0) for x in a]
        return 0.0, 0.0, a, b

    monkeypatch.setattr(bench, "time_pair", fake_time_pair)
    r = bench.measure_overhead(None, None, 3, pairs=100, max_pairs=400)
    assert r["pairs"] == 400 and sum(calls) == 400
    assert r["ci95_pct"][0] <= r["median_pct"] <= r["ci95_pct"][1]


def test_unique_kv_tokens_counts_shared_pages_once():
    # P = 4.  Request 0 (10 tokens) reads pages 5, 6, 7 with 4, 4, 2 slots;
    # request 1 (6 tokens) reads pages 5, 8 with 4, 2; request 2 (3 tokens)
    # reads 3 slots of page 6.  Distinct positions: page 5 -> 4, page 6 -> 4,
    # page 7 -> 2, page 8 -> 2 = 12 of 19 logical tokens.
    table = [[5, 6, 7], [5, 8, -1], [6, -1, -1]]
    assert bench.unique_kv_tokens([10, 6, 3], table, 4) == 12
    assert bench.unique_kv_tokens([10], table[:1], 4) == 10
    # a shorter reader of a shared page never raises its count
    assert bench.unique_kv_tokens([3, 10], [[6, -1, -1], [5, 6, 7]], 4) == 10
