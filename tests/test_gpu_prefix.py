"""GPU tests of the shared-prefix attention call (paged_decode_attn_fp8_prefix).

Two things are checked on batches whose consecutive requests name the same
leading pages:
  * which chunks the call finds shared, bit-exact against `expected_begin`,
    a host re-statement of the rule the header documents;
  * the outputs, element by element against the oracle (plain attention over
    each request's whole page table: the oracle knows nothing of sharing).
"""
import math

import numpy as np
import pytest
import torch

import paged_fp8_kv_attn_b200 as pkv
import workloads

from _pkv_helpers import DeviceBatch, compare, oracle_step, sample_items

pytestmark = pytest.mark.gpu

CHUNK = 64
MIN_CHUNKS = 4
TAIL_CHUNKS = 2


def expected_begin(lens, table, page_size, num_pages, max_pages, group):
    """Per request, the leading chunks the shared pass covers, by the rule in
    pagedkv.h: b joins b - 1's group when they share >= 4 leading chunks that
    lie before both newest tokens (equal, valid page ids); a group's reference
    is its member with the most chunks before its newest token (the first on
    a tie) and each member's chunks are those it shares with the reference;
    runs of 64 / group consecutive members (from the group's first request)
    form a tile if they have at least 2 members and a non-reference member
    with >= 4 chunks, and the reference, if in the run, takes the run's
    largest count;
    a tile member with at most 2 chunks after those is finished by the tile
    (all of its chunks count)."""
    B = len(lens)
    max_tok = max_pages * page_size

    def full(b):
        L = int(lens[b])
        return (L - 1) // CHUNK if 1 <= L <= max_tok else None

    def common(b0, b1):
        f0, f1 = full(b0), full(b1)
        if f0 is None or f1 is None:
            return 0
        f = min(f0, f1)
        pages = -(-f * CHUNK // page_size)
        same = pages
        for j in range(pages):
            p1, p0 = int(table[b1][j]), int(table[b0][j])
            if not (p1 == p0 and 0 <= p1 < num_pages):
                same = j
                break
        return min(f, same * page_size // CHUNK)

    link = [0] + [common(b - 1, b) for b in range(1, B)]
    leader = list(range(B))
    for b in range(1, B):
        if link[b] >= MIN_CHUNKS:
            leader[b] = leader[b - 1]
    ref = {}
    for b in range(B):
        f = full(b)
        key = (-1 if f is None else f, -b)
        if leader[b] not in ref or key > ref[leader[b]][0]:
            ref[leader[b]] = (key, b)
    refrow = [ref[leader[b]][1] for b in range(B)]
    share = [0 if refrow[b] == b else common(refrow[b], b) for b in range(B)]
    T = 64 // group
    begin = [0] * B
    for b in range(B):
        if (b - leader[b]) % T:
            continue
        members = []
        for m in range(b, min(b + T, B)):
            if leader[m] != leader[b]:
                break
            members.append(m)
        mx = max([share[m] for m in members if m != refrow[b]], default=0)
        if len(members) >= 2 and mx >= MIN_CHUNKS:
            for m in members:
                ps = mx if m == refrow[b] else share[m]
                n = full(m) + 1
                begin[m] = n if n - ps <= TAIL_CHUNKS else ps
    return begin


def make_batch(specs, page_size=64, num_q_heads=32, num_kv_heads=4, seed=0):
    """specs: (group or None, shared pages, length) per request.  Each group
    owns a list of prefix pages; a request names the first `shared` of them,
    then private pages up to its length."""
    rng = np.random.Generator(np.random.PCG64(seed))
    need = [-(-int(L) // page_size) for _, _, L in specs]
    prefix_len = {}
    for (g, s, _), n in zip(specs, need):
        if g is not None:
            assert s < n, "the newest token's page must stay private"
            prefix_len[g] = max(prefix_len.get(g, 0), s)
    total = sum(prefix_len.values()) + sum(n - (s if g is not None else 0)
                                           for (g, s, _), n in zip(specs, need))
    perm = rng.permutation(total).astype(np.int32)
    off = 0
    pages = {}
    for g in sorted(prefix_len):
        pages[g] = perm[off:off + prefix_len[g]]
        off += prefix_len[g]
    table = np.full((len(specs), max(need)), -1, dtype=np.int32)
    for b, ((g, s, _), n) in enumerate(zip(specs, need)):
        s = s if g is not None else 0
        if s:
            table[b, :s] = pages[g][:s]
        table[b, s:n] = perm[off:off + n - s]
        off += n - s
    lens = [int(L) for _, _, L in specs]
    return workloads.from_table(lens, table, total, page_size, num_q_heads, num_kv_heads, 128,
                                seed=seed, device="cuda", name="shared prefix")


BASIC = [(0, 6, 600), (0, 6, 900), (0, 6, 390), (0, 4, 700), (0, 6, 1000),
         (None, 0, 300),
         (1, 10, 1500), (1, 10, 641), (1, 8, 2000), (1, 3, 800),
         (2, 5, 321), (2, 5, 500)]


def run_prefix(db, num_ctas=0):
    wl = db.wl
    B, Hq, D = wl.q.shape
    ws = pkv.alloc_prefix_workspace(B, Hq, wl.num_kv_heads, D, num_ctas)
    ws.fill_(0xFF)   # the call must not depend on the workspace's contents
    begin = torch.full((B,), -7, dtype=torch.int32, device="cuda")
    pkv.paged_decode_attn_fp8_prefix(db.q, db.k_cache, db.v_cache, wl.k_scale, wl.v_scale,
                                     db.page_table, db.seq_lens, wl.sm_scale, db.out, db.lse, ws,
                                     abort=db.abort, num_ctas=num_ctas, chunk_begin_out=begin)
    torch.cuda.synchronize()
    return begin.cpu().numpy(), ws


def check_case(wl, num_ctas, label, items=None):
    db = DeviceBatch(wl, kv_dtype="fp8")
    db.check_append()
    begin, ws = run_prefix(db, num_ctas)
    G = wl.num_q_heads // wl.num_kv_heads
    exp = expected_begin(wl.seq_lens, wl.page_table, wl.page_size, wl.num_pages,
                         wl.page_table.shape[1], G)
    supported = wl.head_dim == 128 and wl.num_kv_heads % 2 == 0 and G <= 8
    if not supported:
        exp = [0] * wl.batch
    assert list(begin) == exp, f"{label}: chunk begins {list(begin)} != {exp}"
    out, lse = db.outputs()
    if items is None:
        items = list(range(wl.batch * wl.num_kv_heads))
    ref_o, ref_l, ref_abort = oracle_step(wl, items, kv_dtype="fp8")
    assert np.array_equal(db.abort.cpu().numpy(), ref_abort)
    compare(wl, items, out, lse, ref_o, ref_l, label=f"prefix {label}")
    assert pkv.workspace_status(ws) == 0
    return begin


@pytest.mark.parametrize("num_ctas", [0, 7, 64])
@pytest.mark.parametrize("page_size", [16, 32, 64, 128])
def test_prefix_groups(cuda_device, page_size, num_ctas):
    scale = 64 // page_size if page_size <= 64 else None
    specs = []
    for g, s, L in BASIC:
        if page_size <= 64:
            specs.append((g, s * scale, L))
        else:   # 128-token pages: half as many shared pages
            specs.append((g, s // 2, L))
    wl = make_batch(specs, page_size=page_size, seed=page_size + num_ctas)
    begin = check_case(wl, num_ctas, f"P={page_size} ctas={num_ctas}")
    assert begin.sum() > 0


def test_prefix_nan_code_in_a_shared_page_reaches_every_member(cuda_device):
    """A NaN code in a shared page's K reaches, through the shared pass, every
    member's query heads of that KV head (as in the oracle and the plain
    call), and no other head."""
    specs = [(0, 6, 600), (0, 6, 700), (0, 6, 650), (0, 6, 800)]
    wl = make_batch(specs, seed=9)
    G = wl.num_q_heads // wl.num_kv_heads
    db = DeviceBatch(wl, kv_dtype="fp8")
    db.check_append()
    pid = int(wl.page_table[0, 2])
    assert all(int(wl.page_table[b, 2]) == pid for b in range(len(specs)))
    db.k_cache[pid, 1, 5, 9] = 0x7F               # KV head 1, token 5 of chunk 2, dim 9
    begin, ws = run_prefix(db)
    assert int(begin.min()) > 2                    # chunk 2 went through the shared pass
    out, lse = db.outputs()
    for b in range(len(specs)):
        assert np.isnan(lse[b, G:2 * G]).all() and np.isnan(out[b, G:2 * G]).all()
        assert np.isfinite(lse[b, :G]).all() and np.isfinite(out[b, :G]).all()
        assert np.isfinite(lse[b, 2 * G:]).all() and np.isfinite(out[b, 2 * G:]).all()
    assert pkv.workspace_status(ws) == 0


def test_prefix_large_groups_and_lone_member(cuda_device):
    # 11 members (tiles of 8 + 3) and 9 members (8 + a lone last member, which
    # the shared pass leaves alone)
    specs = [(0, 8, 700 + 37 * i) for i in range(11)] + [(1, 6, 520 + 11 * i) for i in range(9)]
    wl = make_batch(specs, seed=3)
    begin = check_case(wl, 0, "large groups")
    assert begin[19] == 0 and begin[18] > 0 and begin[11] > 0


def test_prefix_group_of_four(cuda_device):
    # G = 4: tiles of 16 members
    specs = [(0, 7, 600 + 50 * i) for i in range(18)] + [(None, 0, 200)]
    wl = make_batch(specs, num_q_heads=16, num_kv_heads=4, seed=4)
    check_case(wl, 0, "G=4")


def test_prefix_aborted_and_invalid(cuda_device):
    specs = [(0, 6, 600), (0, 6, 650), (0, 6, 700), (0, 6, 750), (0, 6, 800), (0, 6, 850)]
    wl = make_batch(specs, seed=5)
    # request 1: a stale expected tag (aborted by the check); request 3: an
    # invalid page id inside the shared pages (breaks its links and makes the
    # request dead); request 5: length 0 (invalid)
    wl.expected_tags[1, 0] ^= 1
    wl.page_table[3, 2] = -1
    wl.seq_lens[5] = 0
    begin = check_case(wl, 0, "aborted/invalid")
    assert begin[3] == 0 and begin[5] == 0


def test_prefix_unsupported_shape_runs_plain(cuda_device):
    # G = 16: no shared tile; the call runs the plain kernels
    specs = [(0, 6, 600), (0, 6, 700), (0, 6, 800)]
    wl = make_batch(specs, num_q_heads=64, num_kv_heads=4, seed=6)
    begin = check_case(wl, 0, "unsupported")
    assert not begin.any()


def test_prefix_back_to_back_reuse(cuda_device):
    """Two calls on one stream share a workspace with no synchronisation."""
    wa = make_batch(BASIC, seed=7)
    wb = make_batch(list(reversed(BASIC)), seed=8)
    da, dbb = DeviceBatch(wa, kv_dtype="fp8"), DeviceBatch(wb, kv_dtype="fp8")
    B, Hq, D = wa.q.shape
    ws = pkv.alloc_prefix_workspace(B, Hq, wa.num_kv_heads, D)
    ws.fill_(0xFF)
    for d in (da, dbb):
        w = d.wl
        pkv.paged_decode_attn_fp8_prefix(d.q, d.k_cache, d.v_cache, w.k_scale, w.v_scale,
                                         d.page_table, d.seq_lens, w.sm_scale, d.out, d.lse, ws)
    torch.cuda.synchronize()
    for d, name in ((da, "a"), (dbb, "b")):
        items = list(range(d.wl.batch * d.wl.num_kv_heads))
        out, lse = d.outputs()
        ref_o, ref_l, _ = oracle_step(d.wl, items, kv_dtype="fp8", check=False, append=False)
        compare(d.wl, items, out, lse, ref_o, ref_l, label=f"prefix reuse {name}")


def test_ragged_prefix_shared_pass_sampled(cuda_device):
    """The ragged prefix-reuse workload at full size, in the configuration the
    benchmark times (fused check + append, then the shared-prefix call)."""
    wl = workloads.ragged_prefix(device="cuda")
    db = DeviceBatch(wl, kv_dtype="fp8")
    db.check_append()
    begin, ws = run_prefix(db)
    exp = expected_begin(wl.seq_lens, wl.page_table, wl.page_size, wl.num_pages,
                         wl.page_table.shape[1], wl.num_q_heads // wl.num_kv_heads)
    assert list(begin) == exp
    assert sum(begin) > 0
    out, lse = db.outputs()
    shortest = int(np.argmin(wl.seq_lens)) * wl.num_kv_heads
    longest = int(np.argmax(wl.seq_lens)) * wl.num_kv_heads + 5
    shared = [int(b) * wl.num_kv_heads + 2 for b in np.nonzero(begin)[0][:3]]
    items = sample_items(wl, 10, seed=55, must=[shortest, longest, *shared])
    ref_o, ref_l, _ = oracle_step(wl, items, kv_dtype="fp8")
    compare(wl, items, out, lse, ref_o, ref_l, label="ragged prefix shared")
    assert pkv.workspace_status(ws) == 0
