"""Pins of the oracle's split-K pieces and their log-sum-exp merge: the step
that combines the partial results of one query head computed over disjoint
token ranges (the decomposition the CUDA path uses; the pages give no kernel
design).

- Split invariance: for random cut points (empty ranges included), merging
  the pieces' partials reproduces the whole-sequence oracle attention to
  1e-12, and that attention is pinned on its own (tests/test_oracle_paths.py:
  torch's scaled_dot_product_attention in fp64 on the gathered cache, closed
  forms).
- Closed forms: a single piece merges to o / l and m + ln l; only empty
  pieces give out = 0 and LSE = -inf; an empty piece among others changes
  nothing.
- Order: permuting the pieces leaves the merge unchanged up to rounding.
"""
import numpy as np
import pytest

import oracle
import workloads
from workloads import bf16_bits


def _fp8_inputs(wl):
    kc = oracle.quantize_bf16(bf16_bits(wl.k_pool), wl.k_scale)
    vc = oracle.quantize_bf16(bf16_bits(wl.v_pool), wl.v_scale)
    return bf16_bits(wl.q), kc, vc


@pytest.mark.parametrize("seed", [3, 4])
def test_merge_of_random_splits_equals_whole_sequence(seed):
    wl = workloads.custom([37, 130, 5, 64], page_size=16, num_q_heads=4, num_kv_heads=2,
                          head_dim=64, seed=seed)
    q, kc, vc = _fp8_inputs(wl)
    out, lse = oracle.paged_decode_attn(q, kc, vc, wl.page_table, wl.seq_lens, wl.num_kv_heads,
                                        wl.page_size, wl.sm_scale, wl.k_scale, wl.v_scale)
    rng = np.random.default_rng(seed)
    for b in range(wl.batch):
        L = int(wl.seq_lens[b])
        for h in range(wl.num_q_heads):
            n_cuts = int(rng.integers(0, 5))
            cuts = np.sort(np.concatenate([[0, L], rng.integers(0, L + 1, n_cuts)]))
            parts = [oracle.attn_partial(q, kc, vc, wl.page_table, wl.num_kv_heads, wl.page_size,
                                         wl.sm_scale, b, h, int(t0), int(t1), wl.k_scale,
                                         wl.v_scale)
                     for t0, t1 in zip(cuts[:-1], cuts[1:])]
            ms, ls, os_ = zip(*parts)
            got, got_lse = oracle.lse_merge(ms, ls, np.stack(os_))
            np.testing.assert_allclose(got, out[b, h], rtol=1e-12, atol=1e-12)
            assert abs(got_lse - lse[b, h]) <= 1e-12 * max(1.0, abs(lse[b, h]))


def test_single_piece_and_empty_pieces():
    o = np.array([[1.5, -2.0, 0.25]])
    out, lse = oracle.lse_merge([0.75], [2.0], o)
    np.testing.assert_array_equal(out, o[0] / 2.0)
    assert lse == 0.75 + np.log(2.0)
    # empty pieces alone: a dead result
    out, lse = oracle.lse_merge([-np.inf, -np.inf], [0.0, 0.0], np.zeros((2, 3)))
    assert np.all(out == 0.0) and lse == -np.inf
    # an empty piece among others changes nothing
    a = oracle.lse_merge([0.75, -np.inf], [2.0, 0.0], np.vstack([o, np.zeros((1, 3))]))
    np.testing.assert_array_equal(a[0], o[0] / 2.0)
    assert a[1] == 0.75 + np.log(2.0)


def test_order_does_not_matter():
    rng = np.random.default_rng(9)
    ms = rng.normal(0.0, 3.0, 6)
    ls = rng.uniform(0.5, 20.0, 6)
    os_ = rng.normal(0.0, 1.0, (6, 16))
    ref, ref_lse = oracle.lse_merge(ms, ls, os_)
    for _ in range(5):
        p = rng.permutation(6)
        got, got_lse = oracle.lse_merge(ms[p], ls[p], os_[p])
        np.testing.assert_allclose(got, ref, rtol=1e-14, atol=1e-15)
        assert abs(got_lse - ref_lse) <= 1e-14 * abs(ref_lse) + 1e-15
