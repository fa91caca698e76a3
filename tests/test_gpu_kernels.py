"""GPU parity tests: the CUDA path (through the C ABI) against the CPU oracle.

Bit-exact for the tag check's abort mask and for every byte the FP8 append
and the page handoff write; attention output within atol/rtol 1e-2 and LSE
within 1e-4 (relative to max(|lse|, 1)).
"""
import numpy as np
import pytest
import torch

import oracle
import paged_fp8_kv_attn_b200 as pkv
import workloads
from workloads import bf16_bits

from _pkv_helpers import DeviceBatch, compare, oracle_step, sample_items

pytestmark = pytest.mark.gpu


def _cuda_u32(a):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int32)).cuda()


# --------------------------------------------------------------------------
# tag check
# --------------------------------------------------------------------------

def test_tag_check_tiny_decode(cuda_device):
    wl = workloads.tiny_decode()
    db = DeviceBatch(wl, kv_dtype="fp8")
    db.tag_check()
    torch.cuda.synchronize()
    assert db.abort.cpu().tolist() == [0, 1]
    assert int(db.num_aborted.item()) == 1


@pytest.mark.parametrize("seed", range(12))
def test_tag_check_random_vs_oracle(cuda_device, seed):
    rng = np.random.Generator(np.random.PCG64(500 + seed))
    B = int(rng.integers(1, 300))
    P = int(rng.choice([16, 32, 64, 128]))
    MP = int(rng.integers(1, 40))
    NP = int(rng.integers(1, 500))
    tags = rng.integers(0, 2**32, NP, dtype=np.uint64).astype(np.uint32)
    table = rng.integers(-3, NP + 3, (B, MP)).astype(np.int32)
    expected = tags[np.clip(table, 0, NP - 1)].copy()
    flip = rng.random((B, MP)) < 0.02
    expected[flip] += np.uint32(1)
    lens = rng.integers(-2, MP * P + 5, B).astype(np.int32)
    want, n_want = oracle.kv_tag_check(tags, table, expected, lens, P)
    abort = torch.full((B,), 7, dtype=torch.uint8, device="cuda")
    n = torch.full((1,), 99, dtype=torch.int32, device="cuda")
    pkv.kv_tag_check(_cuda_u32(tags), torch.from_numpy(table).cuda(), _cuda_u32(expected),
                     torch.from_numpy(lens).cuda(), P, abort, n)
    torch.cuda.synchronize()
    assert np.array_equal(abort.cpu().numpy(), want)
    assert int(n.item()) == n_want


def test_tag_check_integrity_stress_full_size(cuda_device):
    wl = workloads.integrity_stress(device="cpu")
    want, n_want = oracle.kv_tag_check(wl.page_tags, wl.page_table, wl.expected_tags,
                                       wl.seq_lens, wl.page_size)
    assert n_want > 0
    abort = torch.zeros(wl.batch, dtype=torch.uint8, device="cuda")
    n = torch.zeros(1, dtype=torch.int32, device="cuda")
    pkv.kv_tag_check(_cuda_u32(wl.page_tags), torch.from_numpy(wl.page_table).cuda(),
                     _cuda_u32(wl.expected_tags), torch.from_numpy(wl.seq_lens).cuda(),
                     wl.page_size, abort, n)
    torch.cuda.synchronize()
    assert np.array_equal(abort.cpu().numpy(), want)
    assert int(n.item()) == n_want


# --------------------------------------------------------------------------
# quantise-and-append and page handoff: bit-exact
# --------------------------------------------------------------------------

ALL_BF16 = np.arange(65536, dtype=np.uint32).astype(np.uint16)


@pytest.mark.parametrize("scale", [1.0, 0.0137, 2.0 ** -7, 7 * 2.0 ** -8, 1.75, 3.3e-3, 0.25])
def test_requant_every_bf16_value_bit_exact(cuda_device, scale):
    """All 65,536 bf16 bit patterns (NaN, Inf, subnormals, ties) through the
    page handoff, against the oracle's quantiser."""
    src = torch.from_numpy(ALL_BF16.view(np.int16).copy()).view(torch.bfloat16)
    src = src.reshape(4, 2, 64, 128).cuda()          # 4 pages x 2 heads x 64 slots x 128
    dst = torch.zeros((4, 2, 64, 128), dtype=torch.uint8, device="cuda")
    ids = torch.arange(4, dtype=torch.int32, device="cuda")
    pkv.kv_requant_pages_fp8(src, ids, dst, ids, scale)
    torch.cuda.synchronize()
    want = oracle.quantize_bf16(ALL_BF16, scale).reshape(4, 2, 64, 128)
    got = dst.cpu().numpy()
    bad = np.nonzero(got != want)
    assert got.shape == want.shape
    assert bad[0].size == 0, (f"{bad[0].size} mismatches; first bf16 "
                              f"{ALL_BF16.reshape(4, 2, 64, 128)[tuple(b[0] for b in bad)]:#06x}")


def test_requant_page_mapping_and_invalid_pairs(cuda_device):
    wl = workloads.custom([100, 50], page_size=16, num_q_heads=4, num_kv_heads=2, head_dim=64,
                          seed=3, spare_pages=4)
    src = wl.k_pool.cuda()
    NP = wl.num_pages
    rng = np.random.Generator(np.random.PCG64(9))
    src_ids = rng.permutation(NP).astype(np.int32)
    dst_ids = rng.permutation(NP).astype(np.int32)
    src_ids[3] = NP + 1          # invalid pair: skipped
    dst_ids[5] = -1              # invalid pair: skipped
    dst = torch.full((NP, 2, 16, 64), 0xAB, dtype=torch.uint8, device="cuda")
    pkv.kv_requant_pages_fp8(src, torch.from_numpy(src_ids).cuda(), dst,
                             torch.from_numpy(dst_ids).cuda(), wl.k_scale)
    torch.cuda.synchronize()
    want = np.full((NP, 2, 16, 64), 0xAB, dtype=np.uint8)
    oracle.kv_requant_pages_fp8(bf16_bits(wl.k_pool), src_ids, want, dst_ids, wl.k_scale)
    assert np.array_equal(dst.cpu().numpy(), want)


@pytest.mark.parametrize("kv", ["fp8", "bf16"])
@pytest.mark.parametrize("P,D,Hkv", [(16, 64, 1), (64, 128, 8), (32, 128, 2), (128, 64, 4)])
def test_append_bit_exact(cuda_device, kv, P, D, Hkv):
    rng = np.random.Generator(np.random.PCG64(P + D + Hkv))
    lens = rng.integers(1, 6 * P, 37).astype(np.int32)
    wl = workloads.custom(lens, page_size=P, num_q_heads=Hkv, num_kv_heads=Hkv, head_dim=D,
                          seed=int(P * D), spare_pages=3)
    db = DeviceBatch(wl, kv_dtype=kv)
    abort = np.zeros(wl.batch, dtype=np.uint8)
    abort[::5] = 1
    db.abort.copy_(torch.from_numpy(abort))
    before_k = db.k_cache.cpu().numpy().copy() if kv == "fp8" else None
    db.append(use_abort=True)
    torch.cuda.synchronize()
    if kv == "fp8":
        want_k = oracle.quantize_bf16(bf16_bits(wl.k_pool), wl.k_scale)
        want_v = oracle.quantize_bf16(bf16_bits(wl.v_pool), wl.v_scale)
        # the GPU pool was built by the handoff kernel; it must already agree
        assert np.array_equal(before_k, want_k)
        oracle.kv_append_fp8(bf16_bits(wl.k_new), bf16_bits(wl.v_new), wl.page_table,
                             wl.seq_lens, P, wl.k_scale, wl.v_scale, want_k, want_v, abort)
        got_k, got_v = db.k_cache.cpu().numpy(), db.v_cache.cpu().numpy()
    else:
        want_k, want_v = bf16_bits(wl.k_pool).copy(), bf16_bits(wl.v_pool).copy()
        oracle.kv_append_bf16(bf16_bits(wl.k_new), bf16_bits(wl.v_new), wl.page_table,
                              wl.seq_lens, P, want_k, want_v, abort)
        got_k, got_v = bf16_bits(db.k_cache), bf16_bits(db.v_cache)
    assert np.array_equal(got_k, want_k)
    assert np.array_equal(got_v, want_v)


def test_append_special_values_bit_exact(cuda_device):
    """NaN (both signs), +-Inf, values beyond 448 * scale, signed zeros and
    subnormals go through the append exactly as the oracle writes them."""
    B, Hkv, D, P = 8, 8, 128, 64
    wl = workloads.custom([5] * B, page_size=P, num_q_heads=8, num_kv_heads=Hkv, head_dim=D,
                          seed=77)
    specials = np.array([0x7FC0, 0xFFC0, 0x7F80, 0xFF80, 0x0000, 0x8000, 0x0001, 0x8001,
                         0x4480, 0xC480, 0x43E0, 0x3C00], dtype=np.uint16)
    kn = bf16_bits(wl.k_new).copy()
    kn.reshape(-1)[: specials.size * 40] = np.tile(specials, 40)
    wl.k_new = torch.from_numpy(kn.view(np.int16)).view(torch.bfloat16)
    db = DeviceBatch(wl, kv_dtype="fp8")
    db.append(use_abort=False)
    torch.cuda.synchronize()
    want_k = oracle.quantize_bf16(bf16_bits(wl.k_pool), wl.k_scale)
    want_v = oracle.quantize_bf16(bf16_bits(wl.v_pool), wl.v_scale)
    oracle.kv_append_fp8(kn, bf16_bits(wl.v_new), wl.page_table, wl.seq_lens, P, wl.k_scale,
                         wl.v_scale, want_k, want_v)
    assert np.array_equal(db.k_cache.cpu().numpy(), want_k)
    assert np.array_equal(db.v_cache.cpu().numpy(), want_v)


@pytest.mark.parametrize("kv", ["fp8", "bf16"])
@pytest.mark.parametrize("seed", range(4))
def test_check_append_fused_bit_exact(cuda_device, kv, seed):
    """The fused call equals the oracle's tag check followed by its append with
    that mask: abort bytes, count and every cache byte."""
    rng = np.random.Generator(np.random.PCG64(900 + seed))
    P = int(rng.choice([16, 64]))
    lens = rng.integers(1, 9 * P, 45).astype(np.int32)
    wl = workloads.custom(lens, page_size=P, num_q_heads=16, num_kv_heads=int(rng.choice([1, 8])),
                          head_dim=int(rng.choice([64, 128])), seed=77 + seed, spare_pages=5)
    table, expected, lens2 = wl.page_table.copy(), wl.expected_tags.copy(), wl.seq_lens.copy()
    expected[3, 0] += np.uint32(1)                       # stale first page
    expected[7, wl.used_pages(7) - 1] += np.uint32(1)    # stale page holding the new token
    table[11, 0] = wl.num_pages + 3                      # page id out of range
    lens2[13] = 0                                        # invalid length
    wl.page_table, wl.expected_tags, wl.seq_lens = table, expected, lens2
    db = DeviceBatch(wl, kv_dtype=kv)
    before_k = (db.k_cache.cpu().numpy() if kv == "fp8" else bf16_bits(db.k_cache)).copy()
    before_v = (db.v_cache.cpu().numpy() if kv == "fp8" else bf16_bits(db.v_cache)).copy()
    if kv == "fp8":
        pkv.kv_check_append_fp8(db.page_tags, db.page_table, db.expected, db.seq_lens, P,
                                db.k_new, db.v_new, wl.k_scale, wl.v_scale, db.k_cache,
                                db.v_cache, db.abort, db.num_aborted)
    else:
        pkv.kv_check_append_bf16(db.page_tags, db.page_table, db.expected, db.seq_lens, P,
                                 db.k_new, db.v_new, db.k_cache, db.v_cache, db.abort,
                                 db.num_aborted)
    torch.cuda.synchronize()
    want_abort, n_want = oracle.kv_tag_check(wl.page_tags, table, expected, lens2, P)
    assert want_abort[[3, 7, 11, 13]].all()
    assert np.array_equal(db.abort.cpu().numpy(), want_abort)
    assert int(db.num_aborted.item()) == n_want
    if kv == "fp8":
        oracle.kv_append_fp8(bf16_bits(wl.k_new), bf16_bits(wl.v_new), table, lens2, P,
                             wl.k_scale, wl.v_scale, before_k, before_v, want_abort)
        got_k, got_v = db.k_cache.cpu().numpy(), db.v_cache.cpu().numpy()
    else:
        oracle.kv_append_bf16(bf16_bits(wl.k_new), bf16_bits(wl.v_new), table, lens2, P,
                              before_k, before_v, want_abort)
        got_k, got_v = bf16_bits(db.k_cache), bf16_bits(db.v_cache)
    assert np.array_equal(got_k, before_k)
    assert np.array_equal(got_v, before_v)


# --------------------------------------------------------------------------
# attention: small cases, every item compared
# --------------------------------------------------------------------------

SMALL = [
    # lens, P, Hq, Hkv, D
    ([37, 100], 16, 4, 1, 64),                       # the tiny decode step's shapes
    ([1, 2, 63, 64, 65, 130, 257], 64, 64, 8, 128),  # chunk boundaries, ragged tail
    ([1000, 3, 511], 64, 64, 8, 128),
    ([70, 200, 33], 32, 16, 2, 128),
    ([90, 5, 300], 128, 8, 4, 64),
    ([129, 17], 16, 32, 2, 128),                     # GQA group 16
    ([40, 41], 64, 6, 2, 64),                        # GQA group 3
    ([77], 64, 2, 2, 128),                           # group 1 (MHA)
]


@pytest.mark.parametrize("kv", ["fp8", "bf16"])
@pytest.mark.parametrize("case", SMALL, ids=[f"c{i}" for i in range(len(SMALL))])
def test_attention_small_all_items(cuda_device, case, kv):
    lens, P, Hq, Hkv, D = case
    wl = workloads.custom(lens, page_size=P, num_q_heads=Hq, num_kv_heads=Hkv, head_dim=D,
                          seed=sum(lens) * 7 + P, spare_pages=3)
    db = DeviceBatch(wl, kv_dtype=kv)
    items = list(range(wl.batch * Hkv))
    ref_o, ref_l, _ = oracle_step(wl, items, kv_dtype=kv, check=True, append=True)
    for ctas in (0, 1, 3, 37):
        db2 = DeviceBatch(wl, kv_dtype=kv)
        db2.step(check=True, append=True, num_ctas=ctas, fused=ctas in (0, 3))
        out, lse = db2.outputs()
        compare(wl, items, out, lse, ref_o, ref_l, label=f"{kv} ctas={ctas}")
        assert pkv.workspace_status(db2.ws) == 0


def _cluster_sizes_that_fit(db):
    """Cluster sizes 1..16 the device can run for this batch's variant: every
    size up to 8 must fit; above 8 (non-portable sizes) the device may refuse."""
    sizes = []
    for c in range(1, 17):
        try:
            db.attend(use_abort=False, num_ctas=-c)
        except pkv.PagedKVError as err:
            assert c > 8 and "do not fit" in str(err), err
            continue
        sizes.append(c)
    torch.cuda.synchronize()
    return sizes


@pytest.mark.parametrize("kv", ["fp8", "bf16"])
@pytest.mark.parametrize("case", SMALL, ids=[f"c{i}" for i in range(len(SMALL))])
def test_attention_cluster_mode_every_size(cuda_device, case, kv):
    """The single-launch cluster mode (each request's CTAs form a thread-block
    cluster and combine their split-K partials in distributed shared memory,
    no merge kernel), forced at every cluster size: every item against the
    oracle."""
    lens, P, Hq, Hkv, D = case
    wl = workloads.custom(lens, page_size=P, num_q_heads=Hq, num_kv_heads=Hkv, head_dim=D,
                          seed=sum(lens) * 7 + P, spare_pages=3)
    items = list(range(wl.batch * Hkv))
    ref_o, ref_l, _ = oracle_step(wl, items, kv_dtype=kv, check=True, append=True)
    db = DeviceBatch(wl, kv_dtype=kv)
    db.step(check=True, append=True)
    sizes = _cluster_sizes_that_fit(db)
    assert sizes[:8] == list(range(1, 9))
    for c in sizes:
        db.out.fill_(float("nan"))
        db.lse.fill_(float("nan"))
        db.attend(use_abort=True, num_ctas=-c)
        torch.cuda.synchronize()
        out, lse = db.outputs()
        compare(wl, items, out, lse, ref_o, ref_l, label=f"{kv} cluster={c}")
        assert pkv.workspace_status(db.ws) == 0


@pytest.mark.parametrize("kv", ["fp8", "bf16"])
def test_attention_cluster_mode_long_requests(cuda_device, kv):
    """Cluster mode where each cluster owns several long requests, cut into
    many CTA ranges (items split over up to 16 CTAs, records in both the
    dedicated buffer and a pipeline stage), plus an aborted request."""
    wl = workloads.custom([9000, 64, 4097, 1, 12000, 640, 3000], page_size=64, num_q_heads=64,
                          num_kv_heads=8, head_dim=128, seed=57, spare_pages=2)
    items = list(range(wl.batch * 8))
    wl.expected_tags[3, 0] ^= np.uint32(1)      # request 3 fails its check
    ref_o, ref_l, ref_abort = oracle_step(wl, items, kv_dtype=kv, check=True, append=True)
    assert ref_abort.tolist() == [0, 0, 0, 1, 0, 0, 0]
    db = DeviceBatch(wl, kv_dtype=kv)
    db.step(check=True, append=True)
    for c in _cluster_sizes_that_fit(db):
        db.out.fill_(float("nan"))
        db.attend(use_abort=True, num_ctas=-c)
        torch.cuda.synchronize()
        out, lse = db.outputs()
        compare(wl, items, out, lse, ref_o, ref_l, label=f"{kv} cluster={c}")
        assert np.all(np.isneginf(lse[3])) and not out[3].any()


def test_attention_plan_matches_the_documented_choice(cuda_device):
    """The library's default work split: cluster mode (one launch) while the
    batch's items fit in one wave of CTAs, split-K plus merge beyond; an
    explicit cluster size or grid is honoured."""
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    for kv, ipr in ((pkv.PKV_KV_FP8, 4), (pkv.PKV_KV_BF16, 8)):
        for b in (1, 8, 16, 32, 64, 256):
            clu, ctas, launches = pkv.paged_decode_attn_plan(kv, b, 64, 8, 128, 128, 64)
            assert launches == (1 if clu else 2)
            if b * ipr <= sms:
                assert clu > 0, (kv, b)
            if b == 256:
                assert clu == 0 and ctas >= sms
            if clu:
                assert ctas % clu == 0 and clu <= 16
        assert pkv.paged_decode_attn_plan(kv, 8, 64, 8, 128, 128, 64, -3)[0] == 3
        assert pkv.paged_decode_attn_plan(kv, 8, 64, 8, 128, 128, 64, 37) == (0, 37, 2)


@pytest.mark.parametrize("kv", ["fp8", "bf16"])
def test_attention_workspace_reused_across_calls(cuda_device, kv):
    """One workspace serves consecutive calls with different grids and a
    different batch.  The workspace holds the status word and the partial
    (m, l, lr) and O slots; every call rewrites what it reads, so no clearing
    is needed."""
    wl1 = workloads.custom([3000, 70, 9000, 1, 640], page_size=64, num_q_heads=64, num_kv_heads=8,
                           head_dim=128, seed=41, spare_pages=2)
    wl2 = workloads.custom([129] * 9 + [2000], page_size=64, num_q_heads=64, num_kv_heads=8,
                           head_dim=128, seed=42, spare_pages=2)
    db1 = DeviceBatch(wl1, kv_dtype=kv)
    db2 = DeviceBatch(wl2, kv_dtype=kv)
    n1 = pkv.paged_decode_attn_workspace_size(db1.kv_code, wl1.batch, 64, 8, 128, 0)
    n2 = pkv.paged_decode_attn_workspace_size(db2.kv_code, wl2.batch, 64, 8, 128, 0)
    ws = torch.zeros(max(n1, n2), dtype=torch.uint8, device=db1.q.device)
    db1.ws = ws
    db2.ws = ws
    items1 = list(range(wl1.batch * 8))
    items2 = list(range(wl2.batch * 8))
    ref1 = oracle_step(wl1, items1, kv_dtype=kv, check=False, append=True)
    ref2 = oracle_step(wl2, items2, kv_dtype=kv, check=False, append=True)
    for db, wl, items, ref, ctas in ((db1, wl1, items1, ref1, 37), (db2, wl2, items2, ref2, 5),
                                     (db1, wl1, items1, ref1, 0), (db2, wl2, items2, ref2, 0),
                                     (db1, wl1, items1, ref1, -6), (db2, wl2, items2, ref2, -2),
                                     (db1, wl1, items1, ref1, 3)):
        db.out.fill_(float("nan"))
        db.step(check=False, append=True, num_ctas=ctas)
        out, lse = db.outputs()
        compare(wl, items, out, lse, ref[0], ref[1], label=f"{kv} B={wl.batch} ctas={ctas}")
        assert pkv.workspace_status(ws) == 0


@pytest.mark.parametrize("kv", ["fp8", "bf16"])
def test_attention_workspace_back_to_back_without_sync(cuda_device, kv):
    """Calls on one stream that share a workspace, with different lengths and
    batches and no synchronisation between them (each call's kernels may be
    scheduled while the previous call's merge still runs): every output must
    match the oracle.  The workspace starts filled with 0xFF, which the calls
    must not need cleared, and the status word must read 0 afterwards."""
    shapes = ([3000, 70, 9000, 1, 640], [129] * 9 + [2000], [64, 65, 8192, 300, 4097, 1, 2, 33],
              [5000, 17])
    wls = [workloads.custom(lens, page_size=64, num_q_heads=64, num_kv_heads=8, head_dim=128,
                            seed=70 + i, spare_pages=2) for i, lens in enumerate(shapes)]
    dbs = [DeviceBatch(wl, kv_dtype=kv) for wl in wls]
    n = max(pkv.paged_decode_attn_workspace_size(db.kv_code, wl.batch, 64, 8, 128, 0)
            for db, wl in zip(dbs, wls))
    ws = torch.full((n,), 0xFF, dtype=torch.uint8, device=dbs[0].q.device)
    for db in dbs:
        db.ws = ws
        db.append(use_abort=False)
    torch.cuda.synchronize()
    outs = []
    for rnd in range(2):
        for db in dbs:
            out = torch.full_like(db.out, float("nan"))
            lse = torch.full_like(db.lse, float("nan"))
            db.out, db.lse = out, lse
            db.attend(use_abort=False)       # no synchronisation between calls
            outs.append((db, out, lse))
    torch.cuda.synchronize()
    assert pkv.workspace_status(ws) == 0
    refs = {}
    for db, out, lse in outs:
        wl = db.wl
        items = list(range(wl.batch * 8))
        if id(db) not in refs:
            refs[id(db)] = oracle_step(wl, items, kv_dtype=kv, check=False, append=True)
        ref = refs[id(db)]
        o = out.float().cpu().numpy().astype(np.float64)
        l = lse.cpu().numpy().astype(np.float64)
        compare(wl, items, o, l, ref[0], ref[1], label=f"{kv} B={wl.batch} back-to-back")


@pytest.mark.parametrize("kv", ["fp8", "bf16"])
def test_attention_tiny_decode_with_check(cuda_device, kv):
    wl = workloads.tiny_decode()
    ref_o, ref_l, ref_abort = oracle_step(wl, [0, 1], kv_dtype=kv)
    assert ref_abort.tolist() == [0, 1]
    for fused in (True, False):
        db = DeviceBatch(wl, kv_dtype=kv)
        db.step(check=True, append=True, fused=fused)
        out, lse = db.outputs()
        assert db.abort.cpu().tolist() == [0, 1]
        compare(wl, [0, 1], out, lse, ref_o, ref_l, label=f"{kv} fused={fused}")
    assert np.all(np.isneginf(lse[1])) and not out[1].any()
    # with the check switched off (abort = NULL) both requests are computed
    db = DeviceBatch(wl, kv_dtype=kv)
    db.step(check=False, append=True)
    out, lse = db.outputs()
    ref_o, ref_l, _ = oracle_step(wl, [0, 1], kv_dtype=kv, check=False)
    compare(wl, [0, 1], out, lse, ref_o, ref_l, label=kv + " unchecked")


@pytest.mark.parametrize("kv", ["fp8", "bf16"])
@pytest.mark.parametrize("num_ctas", [0, 5, -4])
def test_attention_full_page_table_rows(cuda_device, kv, num_ctas):
    """Requests at the longest length their page-table rows allow (every entry
    used, the new token in the last slot of the last page) beside a one-token
    request, in the library's split, split-K over 5 CTAs and clusters of 4."""
    lens = [2048, 1, 2048, 1000]
    wl = workloads.custom(lens, page_size=64, num_q_heads=64, num_kv_heads=8, head_dim=128,
                          seed=91)
    assert wl.page_table.shape[1] * wl.page_size == max(lens)
    db = DeviceBatch(wl, kv_dtype=kv)
    db.step(check=False, append=True, num_ctas=num_ctas)
    out, lse = db.outputs()
    items = list(range(wl.batch * wl.num_kv_heads))
    ref_o, ref_l, _ = oracle_step(wl, items, kv_dtype=kv, check=False, append=True)
    compare(wl, items, out, lse, ref_o, ref_l, label=f"{kv} full rows ctas={num_ctas}")
    assert pkv.workspace_status(db.ws) == 0


@pytest.mark.parametrize("kv", ["fp8", "bf16"])
def test_attention_dead_requests(cuda_device, kv):
    lens = [100, 100, 100, 100, 300, 5]
    wl = workloads.custom(lens, page_size=16, num_q_heads=16, num_kv_heads=2, head_dim=128,
                          seed=31, spare_pages=2)
    table = wl.page_table.copy()
    table[1, 3] = wl.num_pages + 4       # page id out of range
    table[4, 17] = -9                    # page id out of range, deep in a long request
    lens_bad = wl.seq_lens.copy()
    lens_bad[2] = 0                      # length outside [1, MP * P]
    lens_bad[3] = table.shape[1] * 16 + 1
    wl.page_table = table
    wl.seq_lens = lens_bad
    db = DeviceBatch(wl, kv_dtype=kv)
    items = list(range(wl.batch * 2))
    for ctas in (0, 2, 5, -1, -3, -8):
        db.step(check=False, append=True, num_ctas=ctas)
        out, lse = db.outputs()
        ref_o, ref_l, _ = oracle_step(wl, items, kv_dtype=kv, check=False)
        compare(wl, items, out, lse, ref_o, ref_l, label=f"{kv} ctas={ctas}")
        for b in (1, 2, 3, 4):
            assert np.all(np.isneginf(lse[b])) and not out[b].any()
        db = DeviceBatch(wl, kv_dtype=kv)


def test_attention_constant_v_exact(cuda_device):
    wl = workloads.custom([333, 64, 1], page_size=64, num_q_heads=64, num_kv_heads=8,
                          head_dim=128, seed=41)
    # V pool: every element 1.375 (E4M3 0x3B) with scale 0.25 -> 0.34375 exactly
    db = DeviceBatch(wl, kv_dtype="fp8")
    db.v_cache.fill_(0x3B)
    pkv.paged_decode_attn_fp8(db.q, db.k_cache, db.v_cache, wl.k_scale, 0.25, db.page_table,
                              db.seq_lens, wl.sm_scale, db.out, db.lse, db.workspace())
    torch.cuda.synchronize()
    assert torch.all(db.out.float() == 0.34375)


def test_attention_nan_code_propagates(cuda_device):
    wl = workloads.custom([200, 200], page_size=64, num_q_heads=16, num_kv_heads=2,
                          head_dim=128, seed=43)
    db = DeviceBatch(wl, kv_dtype="fp8")
    pid = int(wl.page_table[0, 1])
    db.k_cache[pid, 1, 5, 9] = 0x7F                  # token 69 of request 0, KV head 1
    pid_tail = int(wl.page_table[1, 3])
    db.k_cache[pid_tail, 0, 63, 0] = 0x7F            # slot past the end of request 1: unread
    db.v_cache[pid_tail, 0, 63, :] = 0xFF
    db.attend(use_abort=False)
    torch.cuda.synchronize()
    out, lse = db.outputs()
    assert np.isnan(lse[0, 8:16]).all() and np.isnan(out[0, 8:16]).all()
    assert np.isfinite(lse[0, :8]).all() and np.isfinite(out[0, :8]).all()
    assert np.isfinite(lse[1]).all() and np.isfinite(out[1]).all()


def test_attention_rejects_bad_arguments(cuda_device):
    wl = workloads.custom([10], page_size=16, num_q_heads=4, num_kv_heads=1, head_dim=64, seed=1)
    db = DeviceBatch(wl, kv_dtype="fp8")
    ws = db.workspace()
    with pytest.raises(pkv.PagedKVError):
        pkv.paged_decode_attn_fp8(db.q, db.k_cache, db.v_cache, wl.k_scale, 0.0, db.page_table,
                                  db.seq_lens, wl.sm_scale, db.out, db.lse, ws)
    with pytest.raises(pkv.PagedKVError):
        pkv.paged_decode_attn_fp8(db.q, db.k_cache, db.v_cache, wl.k_scale, wl.v_scale,
                                  db.page_table, db.seq_lens, wl.sm_scale, db.out, db.lse,
                                  ws[:64])


# --------------------------------------------------------------------------
# page reallocation bookkeeping: bit-exact
# --------------------------------------------------------------------------

def test_retag_and_expected_tags_bit_exact(cuda_device):
    wl = workloads.integrity_stress(batch=64, lo=64, hi=4000, stale_fraction=0.01)
    rng = np.random.Generator(np.random.PCG64(3))
    moved = rng.choice(wl.num_pages, size=500, replace=True).astype(np.int32)   # duplicates
    moved[:5] = [-1, wl.num_pages, wl.num_pages + 100, -50, 0]
    tags = wl.page_tags.copy()
    tags[0] = np.uint32(0xFFFFFFFF)
    d_tags = _cuda_u32(tags)
    pkv.kv_retag_pages(d_tags, torch.from_numpy(moved).cuda())
    want_tags = tags.copy()
    oracle.kv_retag_pages(want_tags, moved)
    torch.cuda.synchronize()
    assert np.array_equal(d_tags.cpu().numpy().view(np.uint32), want_tags)
    exp = np.full_like(wl.expected_tags, 0x5A5A5A5A)
    d_exp = _cuda_u32(exp)
    lens = wl.seq_lens.copy()
    lens[3] = 0
    pkv.kv_expected_tags(d_tags, torch.from_numpy(wl.page_table).cuda(),
                         torch.from_numpy(lens).cuda(), 64, d_exp)
    oracle.kv_expected_tags(want_tags, wl.page_table, lens, 64, exp)
    torch.cuda.synchronize()
    assert np.array_equal(d_exp.cpu().numpy().view(np.uint32), exp)
