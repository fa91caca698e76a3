"""CPU checks of the C-ABI library: it builds for sm_100a, loads without a
GPU, exports every symbol the header declares, and rejects bad arguments on
the host before touching a device."""
import ctypes
import os
import re

import pytest

import paged_fp8_kv_attn_b200 as pkv
from paged_fp8_kv_attn_b200 import build as pkv_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "pagedkv.h")


def _declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^\s*PKV_API\s+(?:const\s+)?[a-z_0-9]+\s*\*?\s*([a-z_][a-z_0-9]*)\s*\(", text, re.M)
    return sorted(set(names))


@pytest.fixture(scope="module")
def lib():
    pkv_build.build()
    return pkv.library()


def test_header_declares_the_hot_path(lib):
    names = _declared_functions()
    for want in ("kv_tag_check", "kv_append_fp8", "paged_decode_attn_fp8",
                 "paged_decode_attn_bf16", "paged_decode_attn_workspace_size", "pkv_last_error",
                 "int4_dequant_gemv"):
        assert want in names


def test_every_declared_symbol_is_exported(lib):
    for name in _declared_functions():
        assert hasattr(lib, name), name


def test_library_is_built_for_sm100a():
    flags = " ".join(pkv_build.NVCC_FLAGS)
    assert "arch=compute_100a,code=sm_100a" in flags
    assert "compute_90" not in flags and "sm_90" not in flags


def test_version_and_error_string(lib):
    assert pkv.version() >= 100
    assert isinstance(lib.pkv_last_error(), bytes)


def test_host_validation_without_a_gpu(lib):
    P = ctypes.c_void_p
    # unsupported head_dim is rejected before any device work
    st = lib.kv_append_fp8(P(16), P(16), P(16), 4, P(16), 1, 1, 96, 16, 1.0, 1.0, P(16), P(16),
                           4, None, None)
    assert st == 3
    assert b"head_dim" in lib.pkv_last_error()
    # non-positive scale
    st = lib.kv_append_fp8(P(16), P(16), P(16), 4, P(16), 1, 1, 64, 16, 0.0, 1.0, P(16), P(16),
                           4, None, None)
    assert st == 1
    # GQA group not a divisor
    st = lib.paged_decode_attn_bf16(P(16), P(16), P(16), P(16), 4, P(16), 1, 6, 4, 64, 16, 8,
                                    0.1, None, P(16), P(16), P(256), 1 << 20, 1, None)
    assert st == 1
    # empty batch is a no-op
    assert lib.kv_tag_check(None, 1, None, None, 1, None, 0, 16, None, None, None) == 0
    # workspace query with invalid sizes returns 0
    assert lib.paged_decode_attn_workspace_size(0, 4, 6, 4, 64, 10) == 0
    # explicit grid: size is computable without a device
    assert lib.paged_decode_attn_workspace_size(0, 4, 64, 8, 128, 296) > 0
    # the work-split query validates like the attention call, before any device query
    out = [ctypes.c_int32(0) for _ in range(3)]
    refs = [ctypes.byref(o) for o in out]
    assert lib.paged_decode_attn_plan(7, 4, 64, 8, 128, 128, 64, 0, *refs) == 1
    assert lib.paged_decode_attn_plan(0, 4, 64, 8, 128, 128, 64, 0, None, None, None) == 1
    assert lib.paged_decode_attn_plan(0, 4, 64, 8, 96, 128, 64, 0, *refs) == 3
    assert lib.paged_decode_attn_plan(0, 4, 64, 8, 128, 128, 64, -17, *refs) == 1
    # the no-allocation status copy needs a destination
    assert lib.paged_decode_attn_fp8_noalloc_status(None, None) == 1
    assert b"status_out" in lib.pkv_last_error()



def test_int4_gemv_host_validation_without_a_gpu(lib):
    P = ctypes.c_void_p
    # batch above 64, n not a multiple of 128, k not a multiple of 256,
    # unsupported group size, misaligned x: all rejected before any device work
    assert lib.int4_dequant_gemv(P(256), P(256), P(256), 65, 128, 256, 128, P(256), None, None) == 1
    assert b"batch" in lib.pkv_last_error()
    assert lib.int4_dequant_gemv(P(256), P(256), P(256), 4, 96, 256, 128, P(256), None, None) == 1
    assert lib.int4_dequant_gemv(P(256), P(256), P(256), 4, 128, 320, 128, P(256), None, None) == 1
    assert lib.int4_dequant_gemv(P(256), P(256), P(256), 4, 128, 256, 64, P(256), None, None) == 3
    assert lib.int4_dequant_gemv(P(258), P(256), P(256), 4, 128, 256, 128, P(256), None, None) == 1
    assert lib.int4_dequant_gemv(None, P(256), P(256), 4, 128, 256, 128, P(256), None, None) == 1
