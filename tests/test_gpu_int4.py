"""INT4 weight dequantisation GEMV on the GPU against the fp64 oracle.

Tolerance, from the arithmetic: the kernel's products x * code are exact in
fp32; each 128-column group is summed in fp32 (at most 128 roundings), scaled
once and added to the running sum (k / 128 more), so the fp32 result is
within E = (k/128 + 130) * 2^-24 * sum_i |x_i w_i| of the exact sum; the
bf16 output adds at most 2^-9 of its magnitude.  The test allows
2^-8 |y| + 4 E (a factor 4 for the tensor cores' accumulation order).
"""
import numpy as np
import pytest
import torch

import oracle
import paged_fp8_kv_attn_b200 as pkv
import workloads

pytestmark = pytest.mark.gpu


def _abs_weights(case, rows=None):
    """|w| [rows][k] for the tolerance bound, read straight from the tiled
    bytes with numpy (only the listed rows, so the full shape stays small)."""
    rows = np.arange(case.n) if rows is None else np.asarray(rows)
    tiles = case.w_tiles.cpu().numpy()                      # [n/128][k/256][128][128]
    sc = oracle.bf16_to_double(workloads.bf16_bits(case.scales))   # [n/128][k/g][128]
    by = tiles[rows // 128, :, rows % 128, :].reshape(rows.size, -1, 4).astype(np.int64)
    words = by[..., 0] | (by[..., 1] << 8) | (by[..., 2] << 16) | (by[..., 3] << 24)   # 8 columns each
    codes = np.empty((rows.size, case.k // 8, 8), dtype=np.int64)
    for i in range(4):
        codes[:, :, 2 * i] = (words >> (4 * i)) & 0xF
        codes[:, :, 2 * i + 1] = (words >> (16 + 4 * i)) & 0xF
    codes = codes.reshape(rows.size, case.k)
    codes = np.where(codes >= 8, codes - 16, codes)
    s = sc[rows // 128, :, rows % 128]                      # [rows][k/g]
    return np.abs(codes) * np.repeat(s, case.group, axis=1)


def run_gpu(case, y=None):
    y = torch.full((case.batch, case.n), float("nan"), dtype=torch.bfloat16, device="cuda") \
        if y is None else y
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    pkv.int4_dequant_gemv(case.x, case.w_tiles, case.scales, y, case.group, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    return y


def compare(case, y_gpu, rows=None):
    xb = workloads.bf16_bits(case.x)
    sb = workloads.bf16_bits(case.scales)
    w = case.w_tiles.cpu().numpy()
    y_exact, _ = oracle.int4_gemv(xb, w, sb, case.n, case.group, rows=rows, threads=8)
    absw = _abs_weights(case, rows)
    mag = np.abs(oracle.bf16_to_double(xb)) @ absw.T                    # sum |x w|
    got = oracle.bf16_to_double(workloads.bf16_bits(y_gpu.cpu()))
    if rows is not None:
        got = got[:, rows]
    E = (case.k / 128 + 130) * 2.0 ** -24 * mag
    tol = 2.0 ** -8 * np.abs(y_exact) + 4 * E
    err = np.abs(got - y_exact)
    bad = ~(err <= tol)
    assert not bad.any(), (f"{bad.sum()} of {bad.size} outside tolerance; worst "
                           f"err {err.max():.3e} at {np.unravel_index(np.argmax(err - tol), err.shape)}")


@pytest.mark.parametrize("batch,n,k", [(1, 128, 256), (3, 256, 512), (8, 128, 1024),
                                       (9, 384, 256), (16, 256, 768), (17, 128, 512),
                                       (32, 256, 1024), (33, 128, 256), (64, 256, 512)])
def test_small_cases_every_output(batch, n, k):
    case = workloads.int4_gemv_case(batch, n=n, k=k, seed=7, device="cuda")
    compare(case, run_gpu(case))


def test_extreme_codes_and_scales():
    # every byte 0x88 (codes -8) and 0x77 (7) in alternate rows, scales at
    # the ends of the bf16 exponent range a model would use
    n, k = 256, 512
    case = workloads.int4_gemv_case(5, n=n, k=k, seed=8, device="cuda")
    case.w_tiles[:, :, 0::2] = 0x88
    case.w_tiles[:, :, 1::2] = 0x77
    case.scales[:, :, 0::2] = 2.0 ** -14
    case.scales[:, :, 1::2] = 2.0 ** 6
    compare(case, run_gpu(case))


def test_one_hot_x_reads_weights_exactly():
    n, k = 128, 256
    case = workloads.int4_gemv_case(8, n=n, k=k, seed=9, device="cuda")
    cols = [0, 1, 15, 16, 127, 128, 200, 255]
    case.x.zero_()
    for b, i in enumerate(cols):
        case.x[b, i] = 1.0
    y = run_gpu(case)
    codes = oracle.int4_unpack(case.w_tiles.cpu().numpy(), n, k)
    s = oracle.int4_scales(workloads.bf16_bits(case.scales), n, k, case.group)   # [n][k/g]
    want = np.stack([codes[:, i] * s[:, i // 128] for i in cols])
    assert np.array_equal(oracle.bf16_to_double(workloads.bf16_bits(y.cpu())),
                          oracle.bf16_to_double(oracle.bf16_from_double(want)))


@pytest.mark.parametrize("batch", workloads.INT4_BATCHES)
def test_full_size_sampled_rows(batch):
    """The benchmark's shape (n = 32768, k = 8192): 48 sampled rows against
    the oracle, and every output finite."""
    case = workloads.int4_gemv_case(batch, device="cuda")
    y = run_gpu(case)
    assert torch.isfinite(y.float()).all()
    rng = np.random.default_rng(batch)
    rows = np.unique(np.concatenate([[0, 127, 128, case.n - 1],
                                     rng.integers(0, case.n, 44)])).astype(np.int32)
    compare(case, y, rows=rows)


def test_batch_rows_are_independent():
    # each row of a batch-64 call (tcgen05 kernel) equals the same row
    # computed alone (warp-level kernel): the group sums of these inputs are
    # exact in fp32 and both kernels scale and add the groups in the same
    # order
    case = workloads.int4_gemv_case(64, n=256, k=512, seed=10, device="cuda")
    y = run_gpu(case)
    for b in (0, 31, 32, 63):
        one = workloads.Int4Gemv("one", 0, case.group, case.x[b:b + 1].contiguous(),
                                 case.w_tiles, case.scales)
        y1 = run_gpu(one)
        assert torch.equal(y1[0], y[b])


def test_stream_ordering_and_reuse():
    s = torch.cuda.Stream()
    case = workloads.int4_gemv_case(4, n=128, k=256, seed=11, device="cuda")
    y = torch.empty((4, 128), dtype=torch.bfloat16, device="cuda")
    with torch.cuda.stream(s):
        for _ in range(3):
            pkv.int4_dequant_gemv(case.x, case.w_tiles, case.scales, y)
    s.synchronize()
    compare(case, y)


def test_tile_layout_helper_matches_the_format():
    """int4_tile_layout re-lays row-major codes and row-wise scales into the
    layout whose definition the oracle reads."""
    rng = np.random.default_rng(12)
    n, k = 256, 512
    codes = rng.integers(-8, 8, size=(n, k), dtype=np.int8)
    c = codes.astype(np.int16) & 0xF
    rowmajor = torch.from_numpy((c[:, 0::2] | (c[:, 1::2] << 4)).astype(np.uint8)).cuda()
    s = torch.exp2(torch.from_numpy(rng.integers(-9, -3, size=(n, k // 128)).astype(np.float32)))
    tiles, sc = pkv.int4_tile_layout(rowmajor, s.to(torch.bfloat16).cuda())
    assert np.array_equal(oracle.int4_unpack(tiles.cpu().numpy(), n, k), codes)
    assert np.array_equal(oracle.int4_scales(workloads.bf16_bits(sc), n, k, 128), s.double().numpy())


@pytest.mark.parametrize("batch", [3, 16, 17, 40])
def test_odd_numbers_of_row_blocks_and_k_tiles(batch):
    """37 row blocks x 9 k-tiles: CTA counts and k-tile loops that are not
    powers of two, on both kernels."""
    case = workloads.int4_gemv_case(batch, n=128 * 37, k=256 * 9, seed=13, device="cuda")
    compare(case, run_gpu(case))


def test_repeated_calls_are_bit_identical():
    case = workloads.int4_gemv_case(8, n=128 * 37, k=256 * 9, seed=14, device="cuda")
    y1 = run_gpu(case)
    for _ in range(3):
        assert torch.equal(y1, run_gpu(case))
