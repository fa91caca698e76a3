"""Pins of the oracle's INT4 weight dequantisation GEMV against facts that do
not come from the oracle itself.

Format reading (the pages say only that weights are 4-bit integers expanded
to floating point before the multiply: "压缩模型权重" on the first-party
post, "模型權重壓縮" on the siami.tw editorial): signed two's complement codes
in tiles of 128 rows x 256 columns (row-major inside a tile, tiles ordered by
row block then column block); each little-endian 32-bit word holds 8
consecutive columns, the even ones in nibbles 0-3 of the low half-word and
the odd ones in nibbles 0-3 of the high half-word; one bf16 scale per group
of 128 columns of a row, stored as [row block][group][row in block].

- Two's complement by hand: the nibble 0x8 is -8, 0xF is -1, 0x7 is 7.
- Layout round trip: codes and scales laid out by numpy reshapes written
  here unpack to the same values.
- y equals numpy's fp64 matrix product of x and the expanded weights (a
  library routine), and its bf16 output is the RNE rounding of that.
- Closed forms: all-ones codes with unit scales sum x; a one-hot x reads one
  weight exactly; doubling one group's scales adds exactly that group's
  contribution again.
"""
import numpy as np
import pytest

import oracle
import workloads

GROUP = 128


def tile_codes(codes: np.ndarray) -> np.ndarray:
    """Independent packer: 32-bit words of 8 columns (even columns in the low
    half-word, odd in the high), then 128 x 128-byte tiles."""
    n, k = codes.shape
    c = (codes.astype(np.int64) & 0xF).reshape(n, k // 8, 8)
    words = np.zeros((n, k // 8), dtype=np.uint64)
    for i in range(4):
        words |= (c[:, :, 2 * i] << (4 * i)).astype(np.uint64)
        words |= (c[:, :, 2 * i + 1] << (16 + 4 * i)).astype(np.uint64)
    rowmajor = words.astype("<u4").view(np.uint8).reshape(n, k // 2)     # [n][k/2]
    return rowmajor.reshape(n // 128, 128, k // 256, 128).transpose(0, 2, 1, 3).copy()


def tile_scales(scales: np.ndarray) -> np.ndarray:
    """[n][k/group] -> [n/128][k/group][128]."""
    n, groups = scales.shape
    return scales.reshape(n // 128, 128, groups).transpose(0, 2, 1).copy()


def bf16_bits_of(values: np.ndarray) -> np.ndarray:
    """bf16 bits of values that are exactly representable in bf16."""
    f = np.asarray(values, dtype=np.float32)
    bits = f.view(np.uint32)
    assert np.all((bits & 0xFFFF) == 0), "value not exactly representable in bf16"
    return (bits >> 16).astype(np.uint16)


def expand(codes: np.ndarray, scales: np.ndarray, group: int) -> np.ndarray:
    """w [n][k] from codes [n][k] and logical scales [n][k/group] (fp64)."""
    return codes.astype(np.float64) * np.repeat(scales, group, axis=1)


def test_twos_complement_nibbles():
    # tile row 0 starts with the word 0xE921708F (bytes 8F 70 21 E9): low
    # half-word 0x708F holds columns 0, 2, 4, 6 = F, 8, 0, 7 -> -1, -8, 0, 7;
    # high half-word 0xE921 holds columns 1, 3, 5, 7 = 1, 2, 9, E -> 1, 2, -7, -2
    w = np.zeros((1, 1, 128, 128), dtype=np.uint8)
    w[0, 0, 0, :4] = [0x8F, 0x70, 0x21, 0xE9]
    assert oracle.int4_unpack(w, 128, 256)[0, :8].tolist() == [-1, 1, -8, 2, 0, -7, 7, -2]


def test_layout_round_trip():
    rng = np.random.default_rng(0)
    n, k = 256, 768
    codes = rng.integers(-8, 8, size=(n, k), dtype=np.int8)
    codes[0, :16] = np.arange(-8, 8)
    assert np.array_equal(oracle.int4_unpack(tile_codes(codes), n, k), codes)
    s = np.exp2(rng.integers(-12, 0, size=(n, k // GROUP))).astype(np.float32)
    got = oracle.int4_scales(bf16_bits_of(tile_scales(s)), n, k, GROUP)
    assert np.array_equal(got, s.astype(np.float64))


@pytest.mark.parametrize("batch,n,k", [(1, 128, 256), (5, 256, 512), (8, 128, 1024)])
def test_matches_numpy_fp64_product(batch, n, k):
    rng = np.random.default_rng(batch * 1000 + n)
    codes = rng.integers(-8, 8, size=(n, k), dtype=np.int8)
    x = rng.standard_normal((batch, k)).astype(np.float32)
    x_bits = (x.view(np.uint32) >> 16).astype(np.uint16)   # truncated to bf16
    s = np.exp2(rng.integers(-12, -2, size=(n, k // GROUP))).astype(np.float32) * \
        (1 + rng.integers(0, 128, size=(n, k // GROUP)) / 128.0).astype(np.float32)
    y_exact, y = oracle.int4_gemv(x_bits, tile_codes(codes), bf16_bits_of(tile_scales(s)), n, GROUP)
    ref = oracle.bf16_to_double(x_bits) @ expand(codes, s.astype(np.float64), GROUP).T
    np.testing.assert_allclose(y_exact, ref, rtol=1e-12, atol=1e-12)
    assert np.array_equal(y, oracle.bf16_from_double(y_exact))


def test_all_ones_sum_x():
    rng = np.random.default_rng(3)
    n, k = 128, 512
    x_bits = bf16_bits_of(rng.integers(-64, 64, size=(2, k)).astype(np.float32))
    w = np.full(n * k // 2, 0x11, dtype=np.uint8)
    s_bits = bf16_bits_of(np.ones(n * k // GROUP, dtype=np.float32))
    y_exact, _ = oracle.int4_gemv(x_bits, w, s_bits, n, GROUP)
    expect = oracle.bf16_to_double(x_bits).sum(axis=1)
    assert np.array_equal(y_exact, np.repeat(expect[:, None], n, axis=1))


def test_one_hot_reads_one_weight():
    rng = np.random.default_rng(4)
    n, k = 256, 512
    codes = rng.integers(-8, 8, size=(n, k), dtype=np.int8)
    s = np.exp2(rng.integers(-8, 0, size=(n, k // GROUP))).astype(np.float32)
    cols = [0, 1, 127, 128, 255, 256, 383, 511]
    x = np.zeros((len(cols), k), dtype=np.float32)
    x[np.arange(len(cols)), cols] = 1.0
    y_exact, _ = oracle.int4_gemv(bf16_bits_of(x), tile_codes(codes), bf16_bits_of(tile_scales(s)),
                                  n, GROUP)
    for b, i in enumerate(cols):
        assert np.array_equal(y_exact[b], codes[:, i] * s[:, i // GROUP].astype(np.float64))


def test_group_scale_linearity():
    rng = np.random.default_rng(5)
    n, k = 128, 512
    codes = rng.integers(-8, 8, size=(n, k), dtype=np.int8)
    x_bits = bf16_bits_of(rng.integers(-16, 16, size=(1, k)).astype(np.float32))
    s = np.ones((n, k // GROUP), dtype=np.float32)
    y1, _ = oracle.int4_gemv(x_bits, tile_codes(codes), bf16_bits_of(tile_scales(s)), n, GROUP)
    s[:, 2] = 2.0
    y2, _ = oracle.int4_gemv(x_bits, tile_codes(codes), bf16_bits_of(tile_scales(s)), n, GROUP)
    xs = oracle.bf16_to_double(x_bits)[0, 2 * GROUP:3 * GROUP]
    part = codes[:, 2 * GROUP:3 * GROUP].astype(np.float64) @ xs
    assert np.array_equal(y2[0] - y1[0], part)


def test_row_subset_matches_full():
    case = workloads.int4_gemv_case(3, n=256, k=512)
    xb = workloads.bf16_bits(case.x)
    sb = workloads.bf16_bits(case.scales)
    w = case.w_tiles.numpy()
    full_e, full = oracle.int4_gemv(xb, w, sb, case.n, case.group)
    rows = np.array([255, 0, 17, 128], dtype=np.int32)
    sub_e, sub = oracle.int4_gemv(xb, w, sb, case.n, case.group, rows=rows, threads=2)
    assert np.array_equal(sub_e, full_e[:, rows]) and np.array_equal(sub, full[:, rows])
