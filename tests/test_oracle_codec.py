"""Pins for the oracle's E4M3 and bf16 codecs (CPU only).

The oracle's codec is checked against things other than itself: the values
the OCP FP8 specification prints, torch's float8_e4m3fn dtype (a library
implementation of the same format), exhaustive structural properties of the
256 codes, and IEEE binary32 division done by numpy.
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "e4m3_ocp_table.txt")
ALL = np.arange(256, dtype=np.uint8)


def _torch_decode(codes):
    t = torch.from_numpy(np.asarray(codes, dtype=np.uint8)).view(torch.float8_e4m3fn)
    return t.to(torch.float64).numpy()


def test_published_values():
    rows = [ln.split() for ln in open(GOLDEN) if ln.strip() and not ln.startswith("#")]
    assert len(rows) >= 8
    for row in rows:
        code = int(row[0], 16)
        want = float(row[1])
        got = float(oracle.e4m3_decode([code])[0])
        if math.isnan(want):
            assert math.isnan(got), hex(code)
        else:
            assert got == want, hex(code)
            assert math.copysign(1.0, got) == math.copysign(1.0, want), hex(code)


def test_decode_matches_torch_all_codes():
    ours = oracle.e4m3_decode(ALL)
    ref = _torch_decode(ALL)
    assert np.array_equal(np.isnan(ours), np.isnan(ref))
    ok = ~np.isnan(ref)
    assert np.array_equal(ours[ok], ref[ok])
    assert np.array_equal(np.signbit(ours[ok]), np.signbit(ref[ok]))
    assert int(np.isnan(ours).sum()) == 2  # only S.1111.111


def test_roundtrip_every_code():
    vals = oracle.e4m3_decode(ALL)
    ok = ~np.isnan(vals)
    back = oracle.e4m3_encode(vals[ok].astype(np.float32))
    assert np.array_equal(back, ALL[ok])  # -0 (0x80) included


def test_monotone_and_count():
    pos = oracle.e4m3_decode(np.arange(0x7F, dtype=np.uint8))
    assert np.all(np.diff(pos) > 0)
    assert pos[-1] == 448.0
    neg = oracle.e4m3_decode(np.arange(0x80, 0xFF, dtype=np.uint8))
    assert np.array_equal(neg, -pos)


def test_midpoints_round_to_even_code():
    pos = oracle.e4m3_decode(np.arange(0x7F, dtype=np.uint8))
    mids = ((pos[:-1] + pos[1:]) / 2).astype(np.float32)
    # every midpoint of two adjacent E4M3 values is exact in binary32
    assert np.array_equal(mids.astype(np.float64), (pos[:-1] + pos[1:]) / 2)
    got = oracle.e4m3_encode(mids)
    lower = np.arange(0x7E, dtype=np.uint8)
    want = np.where(lower % 2 == 0, lower, lower + 1).astype(np.uint8)
    assert np.array_equal(got, want)
    above = np.nextafter(mids, np.float32(np.inf))
    below = np.nextafter(mids, np.float32(0))
    assert np.array_equal(oracle.e4m3_encode(above), lower + 1)
    assert np.array_equal(oracle.e4m3_encode(below), lower)
    assert np.array_equal(oracle.e4m3_encode(-mids), want | 0x80)


def test_saturation_nan_and_zero():
    f = np.float32
    cases = [
        (f(448.0), 0x7E), (f(449.0), 0x7E), (f(463.99), 0x7E), (f(464.0), 0x7E),
        (f(465.0), 0x7E), (f(1e30), 0x7E), (f(np.inf), 0x7E), (f(-np.inf), 0xFE),
        (f(-500.0), 0xFE), (f(0.0), 0x00), (f(-0.0), 0x80), (f(1e-30), 0x00),
        (f(-1e-30), 0x80),
        (f(2.0 ** -10), 0x00),                    # tie between 0 and 2^-9 -> even (0)
        (f(2.0 ** -10 * 1.0001), 0x01), (f(3 * 2.0 ** -10), 0x02),  # tie 1<->2 -> 2
    ]
    ys = np.array([c[0] for c in cases], dtype=np.float32)
    got = oracle.e4m3_encode(ys)
    assert [int(x) for x in got] == [c[1] for c in cases]
    nan = np.array([np.nan, -np.nan], dtype=np.float32)
    nan[1] = -np.abs(nan[1])
    got = oracle.e4m3_encode(nan)
    assert int(got[0]) == 0x7F and int(got[1]) == 0xFF


def test_encode_matches_torch_in_range():
    rng = np.random.Generator(np.random.PCG64(11))
    # dense sweep: every binary32 value between 2^-12 and 2^9 with a step of
    # 2^13 ulps, plus random magnitudes and signs
    lo = np.float32(2.0 ** -12).view(np.uint32)
    hi = np.float32(463.9).view(np.uint32)
    sweep = np.arange(lo, hi, 1 << 13, dtype=np.uint32).view(np.float32)
    rand = (rng.standard_normal(200_000) * rng.choice([1e-3, 0.1, 1, 30, 200], 200_000)).astype(np.float32)
    rand = rand[np.abs(rand) < 463.9]
    ys = np.concatenate([sweep, -sweep, rand])
    ours = oracle.e4m3_encode(ys)
    ref = torch.from_numpy(ys).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(ours, ref)


def test_quantize_is_fp32_division_then_rne():
    rng = np.random.Generator(np.random.PCG64(12))
    x = rng.standard_normal(100_000).astype(np.float32) * 7
    bits = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    xb = oracle.bf16_to_double(bits).astype(np.float32)
    for scale in (np.float32(0.0137), np.float32(1.0), np.float32(3.3e-3)):
        y = xb / scale                      # numpy binary32 division (IEEE)
        want = oracle.e4m3_encode(y)
        got = oracle.quantize_bf16(bits, float(scale))
        assert np.array_equal(got, want)
        inrange = np.abs(y) < 448
        ref = torch.from_numpy(y[inrange]).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
        assert np.array_equal(got[inrange], ref)


def test_bf16_rounding_matches_torch_on_binary32_values():
    rng = np.random.Generator(np.random.PCG64(13))
    x = (rng.standard_normal(100_000) * rng.choice([1e-30, 1e-3, 1, 1e5, 1e35], 100_000))
    x = x.astype(np.float32).astype(np.float64)   # representable in binary32: no double rounding
    ours = oracle.bf16_from_double(x)
    ref = torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)


def test_bf16_rounding_ties_and_specials():
    one = 1.0
    ulp = 2.0 ** -7
    xs = np.array([one + ulp / 2, one + 3 * ulp / 2, -(one + ulp / 2), 3.4e38, 3.5e38, -0.0,
                   np.inf, 2.0 ** -133, 2.0 ** -134, 1.5 * 2.0 ** -133], dtype=np.float64)
    got = oracle.bf16_from_double(xs)
    want = [0x3F80, 0x3F82, 0xBF80, 0x7F80, 0x7F80, 0x8000, 0x7F80, 0x0001, 0x0000, 0x0002]
    # 3.4e38 rounds up past the largest finite bf16 (3.3895e38) -> inf
    assert [int(v) for v in got] == want
    back = oracle.bf16_to_double(np.array([0x3F80, 0xC000, 0x0001], dtype=np.uint16))
    assert list(back) == [1.0, -2.0, 2.0 ** -133]


@pytest.mark.parametrize("scale", [7 * 2.0 ** -8, 1.75, 3 * 2.0 ** -5, 5 * 2.0 ** -7])
def test_quantize_exact_quotients_on_midpoints(scale):
    """x = mu * scale with mu a midpoint of two adjacent E4M3 values: when x
    is a bf16 value the binary32 quotient x / scale is exactly mu, so round
    to nearest even must pick the even code of the pair.  A quantiser that
    multiplies by a rounded reciprocal instead misses some of these."""
    pos = oracle.e4m3_decode(np.arange(0x7F, dtype=np.uint8))
    mids = (pos[:-1] + pos[1:]) / 2
    x = torch.from_numpy(mids * scale).to(torch.bfloat16)
    exact = x.to(torch.float64).numpy() == mids * scale
    assert exact.sum() >= 60
    bits = x.view(torch.int16).numpy().view(np.uint16)[exact]
    lower = np.arange(0x7E, dtype=np.uint8)[exact]
    want = np.where(lower % 2 == 0, lower, lower + 1).astype(np.uint8)
    assert np.array_equal(oracle.quantize_bf16(bits, scale), want)


def test_quantize_nan_takes_the_input_sign():
    """IEEE 754 does not fix the sign of a NaN quotient, so the quantiser's
    NaN rule is stated on its input: every NaN bf16 pattern becomes
    S.1111.111 with the sign bit of the input, for any scale."""
    nans = np.array([b for b in range(65536) if (b & 0x7F80) == 0x7F80 and (b & 0x7F)],
                    dtype=np.uint16)
    assert nans.size == 254
    for scale in (1.0, 0.0137, 3.0):
        got = oracle.quantize_bf16(nans, scale)
        assert np.array_equal(got, np.where(nans & 0x8000, 0xFF, 0x7F).astype(np.uint8))
