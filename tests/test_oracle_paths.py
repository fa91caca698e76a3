"""Pins for the oracle's tag check, append, page handoff and attention (CPU).

Each oracle function is checked against something other than itself:
brute-force enumeration written independently in Python, torch's fp64
scaled_dot_product_attention on the gathered (dense) cache, invariances that
any correct implementation satisfies bit for bit, and closed forms.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import workloads
from workloads import bf16_bits


def _rng(seed):
    return np.random.Generator(np.random.PCG64(seed))


# --------------------------------------------------------------------------
# tag check
# --------------------------------------------------------------------------

def _brute_tag_check(page_tags, page_table, expected, seq_lens, P):
    B, MP = page_table.shape
    NP = len(page_tags)
    out = []
    for b in range(B):
        L = int(seq_lens[b])
        if L < 1 or L > MP * P:
            out.append(1)
            continue
        entries = range(0, L, P)                 # one entry per started page
        bad = 0
        for t in entries:
            j = t // P
            pid = int(page_table[b, j])
            if not (0 <= pid < NP) or int(page_tags[pid]) != int(expected[b, j]):
                bad = 1
        out.append(bad)
    return np.array(out, dtype=np.uint8)


def test_tag_check_tiny_decode_expected_mask():
    wl = workloads.tiny_decode()
    abort, n = oracle.kv_tag_check(wl.page_tags, wl.page_table, wl.expected_tags,
                                   wl.seq_lens, wl.page_size)
    assert abort.tolist() == [0, 1]
    assert n == 1


@pytest.mark.parametrize("seed", range(40))
def test_tag_check_brute_force(seed):
    rng = _rng(100 + seed)
    B = int(rng.integers(1, 9))
    P = int(rng.choice([16, 64]))
    MP = int(rng.integers(1, 6))
    NP = int(rng.integers(1, 20))
    tags = rng.integers(0, 2**32, NP, dtype=np.uint64).astype(np.uint32)
    table = rng.integers(-2, NP + 2, (B, MP)).astype(np.int32)
    expected = tags[np.clip(table, 0, NP - 1)].copy()
    flip = rng.random((B, MP)) < 0.15
    expected[flip] ^= np.uint32(1 << int(rng.integers(0, 32)))
    lens = rng.integers(-1, MP * P + 3, B).astype(np.int32)
    abort, n = oracle.kv_tag_check(tags, table, expected, lens, P)
    want = _brute_tag_check(tags, table, expected, lens, P)
    assert np.array_equal(abort, want)
    assert n == int(want.sum())


def test_tag_check_ignores_entries_past_length():
    tags = np.array([5, 6, 7], dtype=np.uint32)
    table = np.array([[0, 1, 99]], dtype=np.int32)     # entry 2 is garbage
    expected = np.array([[5, 6, 0]], dtype=np.uint32)
    abort, _ = oracle.kv_tag_check(tags, table, expected, np.array([32], np.int32), 16)
    assert abort.tolist() == [0]
    abort, _ = oracle.kv_tag_check(tags, table, expected, np.array([33], np.int32), 16)
    assert abort.tolist() == [1]


def test_integrity_stress_stale_entries_abort_exactly_their_requests():
    wl = workloads.integrity_stress(batch=40, lo=64, hi=2000, stale_fraction=0.01)
    abort, _ = oracle.kv_tag_check(wl.page_tags, wl.page_table, wl.expected_tags,
                                   wl.seq_lens, wl.page_size)
    stale_reqs = {b for b, _ in wl.stale_entries}
    assert len(wl.stale_entries) > 0
    assert set(np.nonzero(abort)[0].tolist()) == stale_reqs


# --------------------------------------------------------------------------
# append and page handoff
# --------------------------------------------------------------------------

def _small_batch(seed, lens, P=16, Hq=4, Hkv=2, D=64, spare=3):
    return workloads.custom(lens, page_size=P, num_q_heads=Hq, num_kv_heads=Hkv, head_dim=D,
                            seed=seed, spare_pages=spare)


def test_append_writes_exactly_the_new_slot():
    wl = _small_batch(7, [1, 16, 17, 40])
    k_cache = np.zeros((wl.num_pages, 2, 16, 64), dtype=np.uint8)
    v_cache = np.full_like(k_cache, 0x55)
    k0, v0 = k_cache.copy(), v_cache.copy()
    abort = np.array([0, 0, 1, 0], dtype=np.uint8)
    kn, vn = bf16_bits(wl.k_new), bf16_bits(wl.v_new)
    oracle.kv_append_fp8(kn, vn, wl.page_table, wl.seq_lens, 16, wl.k_scale, wl.v_scale,
                         k_cache, v_cache, abort)
    touched = np.zeros(k_cache.shape, dtype=bool)
    for b, L in enumerate(wl.seq_lens):
        if abort[b]:
            continue
        pos = int(L) - 1
        pid = wl.page_table[b, pos // 16]
        touched[pid, :, pos % 16, :] = True
        # value check against torch's E4M3 cast of the binary32 quotient
        xk = oracle.bf16_to_double(kn[b]).astype(np.float32) / np.float32(wl.k_scale)
        ref = torch.from_numpy(xk).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
        ok = np.abs(xk) < 448
        assert np.array_equal(k_cache[pid, :, pos % 16, :][ok], ref[ok])
    assert np.array_equal(k_cache[~touched], k0[~touched])
    assert np.array_equal(v_cache[~touched], v0[~touched])
    assert touched.sum() == 3 * 2 * 64


def test_append_skips_invalid_requests():
    wl = _small_batch(8, [5, 20])
    table = wl.page_table.copy()
    table[1, 1] = 10_000                         # page id outside the pool
    lens = np.array([0, 20], dtype=np.int32)     # length 0 is invalid
    k_cache = np.zeros((wl.num_pages, 2, 16, 64), dtype=np.uint8)
    v_cache = np.zeros_like(k_cache)
    oracle.kv_append_fp8(bf16_bits(wl.k_new), bf16_bits(wl.v_new), table, lens, 16, 1.0, 1.0,
                         k_cache, v_cache)
    assert not k_cache.any() and not v_cache.any()


def test_requant_pages_equals_elementwise_quantise():
    wl = _small_batch(9, [30, 50])
    src = bf16_bits(wl.k_pool)
    dst = np.zeros(src.shape, dtype=np.uint8)
    ids = np.arange(wl.num_pages, dtype=np.int32)
    oracle.kv_requant_pages_fp8(src, ids, dst, ids[::-1].copy(), wl.k_scale)
    want = oracle.quantize_bf16(src, wl.k_scale)
    assert np.array_equal(dst[::-1], want)


# --------------------------------------------------------------------------
# attention
# --------------------------------------------------------------------------

def _fp8_pools(wl):
    kc = oracle.quantize_bf16(bf16_bits(wl.k_pool), wl.k_scale)
    vc = oracle.quantize_bf16(bf16_bits(wl.v_pool), wl.v_scale)
    return kc, vc


def _dense_reference(wl, kc, vc, fp8):
    """torch SDPA in fp64 on the gathered, dequantised cache of each request."""
    B, Hq, D = wl.q.shape
    Hkv, P = wl.num_kv_heads, wl.page_size
    G = Hq // Hkv
    q = torch.from_numpy(oracle.bf16_to_double(bf16_bits(wl.q)))
    if fp8:
        kd = torch.from_numpy(oracle.e4m3_decode(kc.ravel()).reshape(kc.shape) * wl.k_scale)
        vd = torch.from_numpy(oracle.e4m3_decode(vc.ravel()).reshape(vc.shape) * wl.v_scale)
    else:
        kd = torch.from_numpy(oracle.bf16_to_double(kc))
        vd = torch.from_numpy(oracle.bf16_to_double(vc))
    outs, lses = [], []
    for b in range(B):
        L = int(wl.seq_lens[b])
        n = (L + P - 1) // P
        pages = wl.page_table[b, :n]
        K = kd[pages].permute(1, 0, 2, 3).reshape(Hkv, n * P, D)[:, :L]   # [Hkv][L][D]
        V = vd[pages].permute(1, 0, 2, 3).reshape(Hkv, n * P, D)[:, :L]
        K = K.repeat_interleave(G, dim=0)
        V = V.repeat_interleave(G, dim=0)
        o = torch.nn.functional.scaled_dot_product_attention(
            q[b][:, None, :], K, V, scale=wl.sm_scale)[:, 0, :]
        s = (q[b][:, None, :] @ K.transpose(1, 2))[:, 0, :] * wl.sm_scale
        outs.append(o.numpy())
        lses.append(torch.logsumexp(s, dim=-1).numpy())
    return np.stack(outs), np.stack(lses)


CASES = [
    # lens, P, Hq, Hkv, D
    ([37, 100], 16, 4, 1, 64),
    ([1, 2, 15, 16, 17], 16, 8, 2, 64),
    ([64, 65, 130], 64, 8, 1, 128),
    ([200, 3], 32, 16, 1, 128),
    ([5, 77], 128, 2, 2, 64),
]


@pytest.mark.parametrize("fp8", [True, False])
@pytest.mark.parametrize("case", CASES)
def test_attention_matches_dense_sdpa(case, fp8):
    lens, P, Hq, Hkv, D = case
    wl = workloads.custom(lens, page_size=P, num_q_heads=Hq, num_kv_heads=Hkv, head_dim=D,
                          seed=sum(lens) + P, spare_pages=2)
    if fp8:
        kc, vc = _fp8_pools(wl)
        ks, vs = wl.k_scale, wl.v_scale
    else:
        kc, vc = bf16_bits(wl.k_pool), bf16_bits(wl.v_pool)
        ks = vs = 1.0
    out, lse = oracle.paged_decode_attn(bf16_bits(wl.q), kc, vc, wl.page_table, wl.seq_lens,
                                        Hkv, P, wl.sm_scale, ks, vs)
    ref_o, ref_l = _dense_reference(wl, kc, vc, fp8)
    np.testing.assert_allclose(out, ref_o, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(lse, ref_l, rtol=1e-12, atol=1e-12)


def test_attention_invariant_under_page_permutation():
    wl = _small_batch(21, [45, 3, 64])
    kc, vc = _fp8_pools(wl)
    out, lse = oracle.paged_decode_attn(bf16_bits(wl.q), kc, vc, wl.page_table, wl.seq_lens,
                                        2, 16, wl.sm_scale, wl.k_scale, wl.v_scale)
    perm = _rng(5).permutation(wl.num_pages)
    inv = np.argsort(perm)
    kc2, vc2 = kc[perm].copy(), vc[perm].copy()         # new page i holds old page perm[i]
    table2 = np.where(wl.page_table >= 0, inv[np.maximum(wl.page_table, 0)], -1).astype(np.int32)
    out2, lse2 = oracle.paged_decode_attn(bf16_bits(wl.q), kc2, vc2, table2, wl.seq_lens,
                                          2, 16, wl.sm_scale, wl.k_scale, wl.v_scale)
    assert np.array_equal(out, out2) and np.array_equal(lse, lse2)


def test_attention_constant_v_returns_v_exactly():
    wl = _small_batch(22, [33, 70, 1])
    kc, _ = _fp8_pools(wl)
    vc = np.full_like(kc, 0x3B)                  # E4M3 0x3B = 1.375
    out, _ = oracle.paged_decode_attn(bf16_bits(wl.q), kc, vc, wl.page_table, wl.seq_lens,
                                      2, 16, wl.sm_scale, wl.k_scale, 0.25)
    # sum_t w_t * c with sum w_t = 1 in fp64: c up to a few ulps
    np.testing.assert_allclose(out, 1.375 * 0.25, rtol=4e-16 * 70, atol=0)


def test_attention_single_token_closed_form():
    wl = _small_batch(23, [1, 1])
    kc, vc = _fp8_pools(wl)
    out, lse = oracle.paged_decode_attn(bf16_bits(wl.q), kc, vc, wl.page_table, wl.seq_lens,
                                        2, 16, wl.sm_scale, wl.k_scale, wl.v_scale)
    q = oracle.bf16_to_double(bf16_bits(wl.q))
    for b in range(2):
        pid = wl.page_table[b, 0]
        for h in range(4):
            k0 = oracle.e4m3_decode(kc[pid, h // 2, 0]) * wl.k_scale
            v0 = oracle.e4m3_decode(vc[pid, h // 2, 0]) * wl.v_scale
            assert np.array_equal(out[b, h], v0)
            assert lse[b, h] == pytest.approx(float(np.dot(q[b, h], k0)) * wl.sm_scale, rel=1e-13)


def test_attention_zero_keys_gives_mean_and_log_length():
    wl = _small_batch(24, [1, 9, 48])
    _, vc = _fp8_pools(wl)
    kc = np.zeros_like(vc)
    out, lse = oracle.paged_decode_attn(bf16_bits(wl.q), kc, vc, wl.page_table, wl.seq_lens,
                                        2, 16, wl.sm_scale, 1.0, wl.v_scale)
    for b, L in enumerate(wl.seq_lens):
        n = (int(L) + 15) // 16
        vals = oracle.e4m3_decode(vc[wl.page_table[b, :n]].ravel()).reshape(n, 2, 16, 64) * wl.v_scale
        seqv = vals.transpose(1, 0, 2, 3).reshape(2, n * 16, 64)[:, : int(L)]
        for h in range(4):
            np.testing.assert_allclose(out[b, h], seqv[h // 2].mean(axis=0), rtol=1e-13, atol=1e-15)
            assert lse[b, h] == pytest.approx(math.log(int(L)), rel=1e-14)


def test_attention_dead_requests():
    wl = _small_batch(25, [20, 20, 20, 20])
    kc, vc = _fp8_pools(wl)
    table = wl.page_table.copy()
    table[2, 1] = -5
    lens = wl.seq_lens.copy()
    lens[3] = 0
    abort = np.array([1, 0, 0, 0], dtype=np.uint8)
    out, lse = oracle.paged_decode_attn(bf16_bits(wl.q), kc, vc, table, lens, 2, 16,
                                        wl.sm_scale, wl.k_scale, wl.v_scale, abort=abort)
    for b in (0, 2, 3):
        assert not out[b].any() and np.all(np.isneginf(lse[b]))
    assert np.all(np.isfinite(lse[1])) and out[1].any()


def test_attention_items_subset_and_threads_agree():
    wl = _small_batch(26, [40, 41, 42])
    kc, vc = _fp8_pools(wl)
    full, fl = oracle.paged_decode_attn(bf16_bits(wl.q), kc, vc, wl.page_table, wl.seq_lens, 2,
                                        16, wl.sm_scale, wl.k_scale, wl.v_scale, threads=3)
    sub, sl = oracle.paged_decode_attn(bf16_bits(wl.q), kc, vc, wl.page_table, wl.seq_lens, 2,
                                       16, wl.sm_scale, wl.k_scale, wl.v_scale, items=[3])
    assert np.array_equal(sub[1, 2:4], full[1, 2:4]) and np.array_equal(sl[1, 2:4], fl[1, 2:4])
    assert np.isnan(sub[0]).all()


def test_attention_nan_code_propagates():
    wl = _small_batch(27, [10, 10])
    kc, vc = _fp8_pools(wl)
    kc[wl.page_table[0, 0], 1, 3, 5] = 0x7F
    out, lse = oracle.paged_decode_attn(bf16_bits(wl.q), kc, vc, wl.page_table, wl.seq_lens, 2,
                                        16, wl.sm_scale, wl.k_scale, wl.v_scale)
    assert np.isnan(out[0, 2:4]).all() and np.isnan(lse[0, 2:4]).all()
    assert np.isfinite(out[0, 0:2]).all() and np.isfinite(out[1]).all()


# --------------------------------------------------------------------------
# page reallocation bookkeeping
# --------------------------------------------------------------------------

def test_retag_pages_brute_force():
    rng = _rng(41)
    tags = rng.integers(0, 2**32, 50, dtype=np.uint64).astype(np.uint32)
    tags[7] = np.uint32(0xFFFFFFFF)                   # wraps to 0
    pages = np.array([7, 3, 3, -1, 50, 12, 7, 0], dtype=np.int32)
    want = [int(t) for t in tags]
    for p in pages:                                   # written out independently
        if 0 <= p < 50:
            want[p] = (want[p] + 1) % 2**32
    got = tags.copy()
    oracle.kv_retag_pages(got, pages)
    assert [int(t) for t in got] == want
    assert got[7] == 1 and got[3] == tags[3] + 2


def test_expected_tags_rebuild_then_check_passes():
    wl = workloads.integrity_stress(batch=30, lo=64, hi=3000, stale_fraction=0.02)
    a, _ = oracle.kv_tag_check(wl.page_tags, wl.page_table, wl.expected_tags, wl.seq_lens, 64)
    assert a.any()
    exp = np.full_like(wl.expected_tags, 0xDEADBEEF)
    oracle.kv_expected_tags(wl.page_tags, wl.page_table, wl.seq_lens, 64, exp)
    a2, n2 = oracle.kv_tag_check(wl.page_tags, wl.page_table, exp, wl.seq_lens, 64)
    assert n2 == 0 and not a2.any()
    for b in range(wl.batch):                         # untouched past the used entries
        assert (exp[b, wl.used_pages(b):] == 0xDEADBEEF).all()


def test_reallocation_round_trip():
    """Reassigning pages bumps their tags: requests still holding them fail the
    check until their expected tags are rebuilt."""
    wl = workloads.custom([100, 200, 50], page_size=16, num_q_heads=4, num_kv_heads=1,
                          head_dim=64, seed=8)
    tags = wl.page_tags.copy()
    moved = wl.page_table[1, :3].copy()
    oracle.kv_retag_pages(tags, moved)
    a, _ = oracle.kv_tag_check(tags, wl.page_table, wl.expected_tags, wl.seq_lens, 16)
    assert a.tolist() == [0, 1, 0]
    exp = wl.expected_tags.copy()
    oracle.kv_expected_tags(tags, wl.page_table, wl.seq_lens, 16, exp)
    a, _ = oracle.kv_tag_check(tags, wl.page_table, exp, wl.seq_lens, 16)
    assert a.tolist() == [0, 0, 0]
