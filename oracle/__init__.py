"""CPU oracle for paged FP8-KV decode attention (test infrastructure).

This package wraps ``oracle.c``, a plain fp64 C implementation of the
operations of the decode hot path: the page-tag integrity check, the FP8
quantise-and-append of a new token, the BF16 -> FP8 page handoff, paged
decode attention over an FP8 or BF16 cache, the page re-tagging helpers and
the INT4 weight dequantisation GEMV.

Only the test suite, the smoke check in ``__graft_entry__`` and the CPU
baseline / reference arm of ``bench.py`` may import this package.  The CUDA
library never imports it, links it or shares code with it.

Arrays cross the boundary as numpy arrays; bf16 values travel as their raw
``uint16`` bit patterns so that no conversion happens on the Python side.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from concurrent.futures import ThreadPoolExecutor

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

# Flags: no fused multiply-add contraction and no fast math, so every C
# expression is evaluated exactly as written in IEEE binary64/binary32.
CFLAGS = ["-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off",
          "-fno-fast-math", "-Wall", "-Wextra"]


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so next to it (gcc)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".{os.getpid()}.tmp"
        subprocess.run(["gcc", *CFLAGS, _SRC, "-o", tmp, "-lm"], check=True)
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            path = os.environ.get("PAGEDKV_ORACLE_LIB")   # a test may point at a planted-mistake build
            if not path:
                path = build()
            lib = ctypes.CDLL(path)
            P = ctypes.c_void_p
            i32, i64, f32 = ctypes.c_int32, ctypes.c_int64, ctypes.c_float
            lib.orc_e4m3_decode.argtypes = [ctypes.c_uint8]
            lib.orc_e4m3_decode.restype = ctypes.c_double
            lib.orc_e4m3_encode.argtypes = [f32]
            lib.orc_e4m3_encode.restype = ctypes.c_uint8
            lib.orc_e4m3_encode_array.argtypes = [P, P, i64]
            lib.orc_quantize_bf16_array.argtypes = [P, f32, P, i64]
            lib.orc_bf16_from_double_array.argtypes = [P, P, i64]
            lib.orc_kv_tag_check.argtypes = [P, i32, P, P, i32, P, i32, i32, P]
            lib.orc_kv_tag_check.restype = i32
            lib.orc_kv_append_fp8.argtypes = [P, P, P, i32, P, i32, i32, i32, i32,
                                              f32, f32, P, P, i32, P]
            lib.orc_kv_append_bf16.argtypes = [P, P, P, i32, P, i32, i32, i32, i32,
                                               P, P, i32, P]
            lib.orc_kv_requant_pages_fp8.argtypes = [P, i32, P, P, i32, P, i32, i32,
                                                     i32, i32, f32]
            lib.orc_kv_retag_pages.argtypes = [P, i32, P, i32]
            lib.orc_kv_expected_tags.argtypes = [P, i32, P, i32, P, i32, i32, P]
            lib.orc_paged_decode_attn.argtypes = [i32, P, P, P, f32, f32, P, i32, P, i32,
                                                  i32, i32, i32, i32, i32, f32, P, P, i32,
                                                  P, P]
            lib.orc_attn_partial.argtypes = [i32, P, P, P, f32, f32, P, i32, i32, i32, i32,
                                             i32, f32, i32, i32, i32, i32, P, P, P]
            lib.orc_lse_merge.argtypes = [i32, i32, P, P, P, P, P]
            lib.orc_int4_code.argtypes = [P, i32, i32, i32]
            lib.orc_int4_code.restype = i32
            lib.orc_int4_scale.argtypes = [P, i32, i32, i32, i32]
            lib.orc_int4_scale.restype = ctypes.c_double
            lib.orc_int4_unpack.argtypes = [P, i32, i32, P]
            lib.orc_int4_gemv.argtypes = [P, P, P, i32, i32, i32, i32, P, i32, P, P]
            _lib = lib
    return _lib


def _ptr(a):
    return None if a is None else ctypes.c_void_p(a.ctypes.data)


def _c(a, dtype):
    """Contiguous array of the given dtype (no value conversion for bit arrays)."""
    a = np.asarray(a)
    if a.dtype != np.dtype(dtype):
        raise TypeError(f"expected {np.dtype(dtype)}, got {a.dtype}")
    return np.ascontiguousarray(a)


# --------------------------------------------------------------------------
# codecs
# --------------------------------------------------------------------------

def e4m3_decode(codes) -> np.ndarray:
    """fp64 values of E4M3 codes (OCP E4M3 definition)."""
    lib = _load()
    codes = np.asarray(codes, dtype=np.uint8)
    return np.array([lib.orc_e4m3_decode(int(c)) for c in codes.ravel()],
                    dtype=np.float64).reshape(codes.shape)


def e4m3_encode(y) -> np.ndarray:
    """E4M3 codes of binary32 values: RNE, saturating at +-448, NaN kept."""
    lib = _load()
    y = _c(y, np.float32)
    out = np.empty(y.shape, dtype=np.uint8)
    lib.orc_e4m3_encode_array(_ptr(y), _ptr(out), y.size)
    return out


def quantize_bf16(x_bits, scale: float) -> np.ndarray:
    """E4M3 codes of fp32(bf16 x) / fp32(scale)."""
    lib = _load()
    x_bits = _c(x_bits, np.uint16)
    out = np.empty(x_bits.shape, dtype=np.uint8)
    lib.orc_quantize_bf16_array(_ptr(x_bits), ctypes.c_float(scale), _ptr(out), x_bits.size)
    return out


def bf16_from_double(x) -> np.ndarray:
    """bf16 bit patterns of fp64 values, round to nearest even."""
    lib = _load()
    x = _c(x, np.float64)
    out = np.empty(x.shape, dtype=np.uint16)
    lib.orc_bf16_from_double_array(_ptr(x), _ptr(out), x.size)
    return out


def bf16_to_double(bits) -> np.ndarray:
    """fp64 values of bf16 bit patterns (exact)."""
    bits = np.asarray(bits, dtype=np.uint16)
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


# --------------------------------------------------------------------------
# the four operations
# --------------------------------------------------------------------------

def kv_tag_check(page_tags, page_table, expected_tags, seq_lens, page_size):
    """Returns (abort mask uint8[B], number aborted)."""
    lib = _load()
    page_tags = _c(page_tags, np.uint32)
    page_table = _c(page_table, np.int32)
    expected_tags = _c(expected_tags, np.uint32)
    seq_lens = _c(seq_lens, np.int32)
    B, MP = page_table.shape
    abort = np.empty(B, dtype=np.uint8)
    n = lib.orc_kv_tag_check(_ptr(page_tags), page_tags.size, _ptr(page_table),
                             _ptr(expected_tags), MP, _ptr(seq_lens), B, page_size,
                             _ptr(abort))
    return abort, int(n)


def kv_retag_pages(page_tags, pages):
    """Bump (mod 2^32) the tag of every listed page id inside the pool, in place."""
    lib = _load()
    if page_tags.dtype != np.uint32 or not page_tags.flags.c_contiguous:
        raise TypeError("page_tags must be a C-contiguous uint32 array")
    pages = _c(pages, np.int32)
    lib.orc_kv_retag_pages(_ptr(page_tags), page_tags.size, _ptr(pages), pages.size)


def kv_expected_tags(page_tags, page_table, seq_lens, page_size, expected_tags):
    """Rebuild each request's expected tags from the current page tags, in place."""
    lib = _load()
    page_tags = _c(page_tags, np.uint32)
    page_table = _c(page_table, np.int32)
    seq_lens = _c(seq_lens, np.int32)
    if expected_tags.dtype != np.uint32 or not expected_tags.flags.c_contiguous:
        raise TypeError("expected_tags must be a C-contiguous uint32 array")
    B, MP = page_table.shape
    lib.orc_kv_expected_tags(_ptr(page_tags), page_tags.size, _ptr(page_table), MP,
                             _ptr(seq_lens), B, page_size, _ptr(expected_tags))


def kv_append_fp8(k_new_bits, v_new_bits, page_table, seq_lens, page_size,
                  k_scale, v_scale, k_cache, v_cache, abort=None):
    """Quantise and write each request's new token into its page (in place)."""
    lib = _load()
    k_new_bits = _c(k_new_bits, np.uint16)
    v_new_bits = _c(v_new_bits, np.uint16)
    page_table = _c(page_table, np.int32)
    seq_lens = _c(seq_lens, np.int32)
    if not (k_cache.flags.c_contiguous and v_cache.flags.c_contiguous):
        raise ValueError("caches must be C-contiguous")
    if k_cache.dtype != np.uint8 or v_cache.dtype != np.uint8:
        raise TypeError("FP8 caches are uint8 code arrays")
    B, Hkv, D = k_new_bits.shape
    NP = k_cache.shape[0]
    ab = None if abort is None else _c(abort, np.uint8)
    lib.orc_kv_append_fp8(_ptr(k_new_bits), _ptr(v_new_bits), _ptr(page_table),
                          page_table.shape[1], _ptr(seq_lens), B, Hkv, D, page_size,
                          ctypes.c_float(k_scale), ctypes.c_float(v_scale),
                          _ptr(k_cache), _ptr(v_cache), NP, _ptr(ab))


def kv_append_bf16(k_new_bits, v_new_bits, page_table, seq_lens, page_size,
                   k_cache, v_cache, abort=None):
    """Write each request's new BF16 token into its page (in place)."""
    lib = _load()
    k_new_bits = _c(k_new_bits, np.uint16)
    v_new_bits = _c(v_new_bits, np.uint16)
    page_table = _c(page_table, np.int32)
    seq_lens = _c(seq_lens, np.int32)
    if k_cache.dtype != np.uint16 or v_cache.dtype != np.uint16:
        raise TypeError("BF16 caches are uint16 bit arrays")
    B, Hkv, D = k_new_bits.shape
    NP = k_cache.shape[0]
    ab = None if abort is None else _c(abort, np.uint8)
    lib.orc_kv_append_bf16(_ptr(k_new_bits), _ptr(v_new_bits), _ptr(page_table),
                           page_table.shape[1], _ptr(seq_lens), B, Hkv, D, page_size,
                           _ptr(k_cache), _ptr(v_cache), NP, _ptr(ab))


def kv_requant_pages_fp8(src_pool_bits, src_pages, dst_pool, dst_pages, scale):
    """Re-quantise BF16 pages into FP8 pages (in place in dst_pool)."""
    lib = _load()
    src_pool_bits = _c(src_pool_bits, np.uint16)
    src_pages = _c(src_pages, np.int32)
    dst_pages = _c(dst_pages, np.int32)
    if dst_pool.dtype != np.uint8 or not dst_pool.flags.c_contiguous:
        raise TypeError("dst_pool must be a C-contiguous uint8 array")
    NPs, Hkv, P, D = src_pool_bits.shape
    lib.orc_kv_requant_pages_fp8(_ptr(src_pool_bits), NPs, _ptr(src_pages), _ptr(dst_pool),
                                 dst_pool.shape[0], _ptr(dst_pages), src_pages.size,
                                 Hkv, P, D, ctypes.c_float(scale))


def paged_decode_attn(q_bits, k_cache, v_cache, page_table, seq_lens, num_kv_heads,
                      page_size, sm_scale, k_scale=1.0, v_scale=1.0, abort=None,
                      items=None, threads: int = 1):
    """fp64 paged decode attention.

    ``k_cache``/``v_cache`` are uint8 E4M3 code pools (FP8) or uint16 bf16 bit
    pools, shaped [NP][Hkv][P][D].  Returns (out fp64 [B][Hq][D], lse fp64
    [B][Hq]); entries of items not computed are NaN.  ``items`` lists
    b * Hkv + kv_head pairs (default: all); ``threads`` > 1 splits the items
    over host threads (the C call releases the GIL).
    """
    lib = _load()
    q_bits = _c(q_bits, np.uint16)
    page_table = _c(page_table, np.int32)
    seq_lens = _c(seq_lens, np.int32)
    if k_cache.dtype == np.uint8:
        kv_dtype = 0
    elif k_cache.dtype == np.uint16:
        kv_dtype = 1
    else:
        raise TypeError("cache must be uint8 (E4M3 codes) or uint16 (bf16 bits)")
    k_cache = np.ascontiguousarray(k_cache)
    v_cache = np.ascontiguousarray(v_cache)
    B, Hq, D = q_bits.shape
    NP = k_cache.shape[0]
    out = np.full((B, Hq, D), np.nan, dtype=np.float64)
    lse = np.full((B, Hq), np.nan, dtype=np.float64)
    ab = None if abort is None else _c(abort, np.uint8)
    if items is None:
        items = np.arange(B * num_kv_heads, dtype=np.int32)
    items = _c(np.asarray(items, dtype=np.int32), np.int32)

    def run(chunk):
        lib.orc_paged_decode_attn(kv_dtype, _ptr(q_bits), _ptr(k_cache), _ptr(v_cache),
                                  ctypes.c_float(k_scale), ctypes.c_float(v_scale),
                                  _ptr(page_table), page_table.shape[1], _ptr(seq_lens), B,
                                  Hq, num_kv_heads, D, page_size, NP,
                                  ctypes.c_float(sm_scale), _ptr(ab), _ptr(chunk),
                                  chunk.size, _ptr(out), _ptr(lse))

    if threads <= 1 or items.size <= 1:
        run(items)
    else:
        chunks = [np.ascontiguousarray(c) for c in np.array_split(items, min(threads, items.size))]
        with ThreadPoolExecutor(max_workers=len(chunks)) as ex:
            list(ex.map(run, chunks))
    return out, lse


def attn_partial(q_bits, k_cache, v_cache, page_table, num_kv_heads, page_size, sm_scale,
                 b, h, t0, t1, k_scale=1.0, v_scale=1.0):
    """Split-K piece of query head h of request b over tokens [t0, t1):
    (m, l, o) with m = max s_t, l = sum exp(s_t - m), o = sum exp(s_t - m) v_t
    (unnormalised, fp64 [D])."""
    lib = _load()
    q_bits = _c(q_bits, np.uint16)
    page_table = _c(page_table, np.int32)
    kv_dtype = 0 if k_cache.dtype == np.uint8 else 1
    k_cache = np.ascontiguousarray(k_cache)
    v_cache = np.ascontiguousarray(v_cache)
    B, Hq, D = q_bits.shape
    m = np.zeros(1, dtype=np.float64)
    l = np.zeros(1, dtype=np.float64)
    o = np.zeros(D, dtype=np.float64)
    lib.orc_attn_partial(kv_dtype, _ptr(q_bits), _ptr(k_cache), _ptr(v_cache),
                         ctypes.c_float(k_scale), ctypes.c_float(v_scale), _ptr(page_table),
                         page_table.shape[1], Hq, num_kv_heads, D, page_size,
                         ctypes.c_float(sm_scale), b, h, t0, t1, _ptr(m), _ptr(l), _ptr(o))
    return float(m[0]), float(l[0]), o


def lse_merge(ms, ls, os_):
    """Merge of split-K partials (m_s, l_s, o_s [D]): (out fp64 [D], lse)."""
    lib = _load()
    ms = _c(np.asarray(ms, dtype=np.float64), np.float64)
    ls = _c(np.asarray(ls, dtype=np.float64), np.float64)
    os_ = _c(np.asarray(os_, dtype=np.float64).reshape(ms.size, -1), np.float64)
    D = os_.shape[1]
    out = np.zeros(D, dtype=np.float64)
    lse = np.zeros(1, dtype=np.float64)
    lib.orc_lse_merge(ms.size, D, _ptr(ms), _ptr(ls), _ptr(os_), _ptr(out), _ptr(lse))
    return out, float(lse[0])


# --------------------------------------------------------------------------
# INT4 weight dequantisation GEMV
# --------------------------------------------------------------------------

def int4_unpack(w_tiles, n: int, k: int) -> np.ndarray:
    """Signed codes [n][k] (int8) of a tiled INT4 matrix (n * k / 2 bytes)."""
    lib = _load()
    w_tiles = _c(w_tiles, np.uint8)
    if w_tiles.size * 2 != n * k:
        raise ValueError("w_tiles must hold n * k / 2 bytes")
    codes = np.empty((n, k), dtype=np.int8)
    lib.orc_int4_unpack(_ptr(w_tiles), n, k, _ptr(codes))
    return codes


def int4_scales(scale_bits, n: int, k: int, group: int) -> np.ndarray:
    """fp64 scale of every (row, group): [n][k/group]."""
    lib = _load()
    scale_bits = _c(scale_bits, np.uint16)
    if scale_bits.size != n * (k // group):
        raise ValueError("scales must hold n * k / group values")
    return np.array([[lib.orc_int4_scale(_ptr(scale_bits), k, group, j, g * group)
                      for g in range(k // group)] for j in range(n)], dtype=np.float64)


def int4_gemv(x_bits, w_tiles, scale_bits, n: int, group: int, rows=None, threads: int = 1):
    """y = x W^T with W expanded from tiled INT4 codes and group scales.

    ``x_bits`` [B][k] bf16 bits, ``w_tiles`` the n * k / 2 code bytes in the
    tiled layout, ``scale_bits`` the n * k / group bf16 scale bits.  Returns
    (y_exact fp64 [B][r], y bf16 bits [B][r]) for the listed ``rows``
    (default: all n, in order); ``threads`` > 1 splits the rows over host
    threads (the C call releases the GIL).
    """
    lib = _load()
    x_bits = _c(x_bits, np.uint16)
    w_tiles = _c(w_tiles, np.uint8)
    scale_bits = _c(scale_bits, np.uint16)
    B, k = x_bits.shape
    if w_tiles.size * 2 != n * k or scale_bits.size * group != n * k or k % group:
        raise ValueError("inconsistent INT4 GEMV shapes")
    rows = np.arange(n, dtype=np.int32) if rows is None else _c(np.asarray(rows, dtype=np.int32), np.int32)
    y_exact = np.empty((B, rows.size), dtype=np.float64)
    y = np.empty((B, rows.size), dtype=np.uint16)

    def run(lo, hi):
        sub = np.ascontiguousarray(rows[lo:hi])
        ye = np.empty((B, sub.size), dtype=np.float64)
        yb = np.empty((B, sub.size), dtype=np.uint16)
        lib.orc_int4_gemv(_ptr(x_bits), _ptr(w_tiles), _ptr(scale_bits), B, n, k, group,
                          _ptr(sub), sub.size, _ptr(ye), _ptr(yb))
        y_exact[:, lo:hi] = ye
        y[:, lo:hi] = yb

    if threads <= 1 or rows.size <= 1:
        run(0, rows.size)
    else:
        bounds = np.linspace(0, rows.size, min(threads, rows.size) + 1).astype(int)
        with ThreadPoolExecutor(max_workers=len(bounds) - 1) as ex:
            list(ex.map(lambda i: run(bounds[i], bounds[i + 1]), range(len(bounds) - 1)))
    return y_exact, y
