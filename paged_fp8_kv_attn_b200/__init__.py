"""Paged FP8-KV decode attention for NVIDIA B200 (sm_100a).

A thin Python binding over the C-ABI library ``libpagedkv.so`` (declared in
``include/pagedkv.h``).  Each function here only checks and marshals its torch
tensors into pointers and sizes and calls the C entry point of the same name
on the current CUDA stream; every step of the computation runs in the
library's CUDA kernels.  Nothing here falls back to PyTorch or to the CPU: if
the library is missing or fails, the call raises.

Tensors (all on one CUDA device, contiguous):
  q            [B][Hq][D]      torch.bfloat16
  k/v caches   [NP][Hkv][P][D] torch.uint8 (E4M3 codes) or torch.bfloat16
  k_new/v_new  [B][Hkv][D]     torch.bfloat16
  page_table   [B][MP]         torch.int32
  seq_lens     [B]             torch.int32   (counts the new token)
  page_tags    [NP]            torch.int32 / uint32 view (raw 32-bit tags)
  expected     [B][MP]         same dtype as page_tags
  abort        [B]             torch.uint8

INT4 weight dequantisation GEMV (int4_dequant_gemv):
  x            [B][k]                      torch.bfloat16
  w_tiles      [n/128][k/256][128][128]    torch.uint8 (two signed 4-bit codes per byte)
  scales       [n/128][k/group][128]       torch.bfloat16
  y            [B][n]                      torch.bfloat16
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libpagedkv.so")

PKV_OK = 0
PKV_KV_FP8 = 0
PKV_KV_BF16 = 1
_STATUS = {1: "invalid argument", 2: "workspace", 3: "unsupported", 4: "CUDA error"}


class PagedKVError(RuntimeError):
    """A library call returned a non-OK status."""

    def __init__(self, func: str, status: int, message: str):
        super().__init__(f"{func}: {_STATUS.get(status, status)}: {message}")
        self.status = status


_lib = None


def _load():
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing; build it with "
                              "`python -m paged_fp8_kv_attn_b200.build`")
        lib = ctypes.CDLL(LIB_PATH)
        P, i32, f32, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_float, ctypes.c_size_t
        sig = {
            "kv_tag_check": [P, i32, P, P, i32, P, i32, i32, P, P, P],
            "kv_append_fp8": [P, P, P, i32, P, i32, i32, i32, i32, f32, f32, P, P, i32, P, P],
            "kv_append_bf16": [P, P, P, i32, P, i32, i32, i32, i32, P, P, i32, P, P],
            "kv_requant_pages_fp8": [P, i32, P, P, i32, P, i32, i32, i32, i32, f32, P],
            "kv_retag_pages": [P, i32, P, i32, P],
            "kv_expected_tags": [P, i32, P, i32, P, i32, i32, P, P],
            "kv_check_append_fp8": [P, i32, P, P, i32, P, i32, i32, P, P, i32, i32, f32, f32, P, P,
                                    P, P, P],
            "kv_check_append_bf16": [P, i32, P, P, i32, P, i32, i32, P, P, i32, i32, P, P, P, P,
                                     P],
            "paged_decode_attn_fp8": [P, P, P, f32, f32, P, i32, P, i32, i32, i32, i32, i32, i32,
                                      f32, P, P, P, P, sz, i32, P],
            "paged_decode_attn_bf16": [P, P, P, P, i32, P, i32, i32, i32, i32, i32, i32, f32, P,
                                       P, P, P, sz, i32, P],
            "paged_decode_attn_fp8_prefix": [P, P, P, f32, f32, P, i32, P, i32, i32, i32, i32, i32,
                                             i32, f32, P, P, P, P, sz, i32, P, P],
            "int4_dequant_gemv": [P, P, P, i32, i32, i32, i32, P, P, P],
        }
        for name, args in sig.items():
            fn = getattr(lib, name)
            fn.argtypes = args
            fn.restype = i32
        lib.paged_decode_attn_fp8_noalloc.argtypes = [P, P, P, f32, f32, P, i32, P, i32, i32,
                                                      i32, i32, i32, i32, f32, P, P, P, i32, P]
        lib.paged_decode_attn_fp8_noalloc.restype = i32
        lib.paged_decode_attn_fp8_noalloc_scratch_bytes.argtypes = []
        lib.paged_decode_attn_fp8_noalloc_scratch_bytes.restype = sz
        lib.paged_decode_attn_fp8_noalloc_status.argtypes = [P, P]
        lib.paged_decode_attn_fp8_noalloc_status.restype = i32
        pi32 = ctypes.POINTER(i32)
        lib.paged_decode_attn_plan.argtypes = [i32, i32, i32, i32, i32, i32, i32, i32, pi32,
                                               pi32, pi32]
        lib.paged_decode_attn_plan.restype = i32
        lib.paged_decode_attn_workspace_size.argtypes = [i32, i32, i32, i32, i32, i32]
        lib.paged_decode_attn_workspace_size.restype = sz
        lib.paged_decode_attn_fp8_prefix_workspace_size.argtypes = [i32, i32, i32, i32, i32]
        lib.paged_decode_attn_fp8_prefix_workspace_size.restype = sz
        lib.pkv_last_error.argtypes = []
        lib.pkv_last_error.restype = ctypes.c_char_p
        lib.pkv_version.argtypes = []
        lib.pkv_version.restype = i32
        _lib = lib
    return _lib


def library() -> ctypes.CDLL:
    """The loaded C library (raises if it has not been built)."""
    return _load()


def _check(name: str, status: int):
    if status != PKV_OK:
        raise PagedKVError(name, status, _load().pkv_last_error().decode())


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _need(t, dtype, ndim, name):
    if t is None:
        raise ValueError(f"{name} is required")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype not in (dtype if isinstance(dtype, tuple) else (dtype,)):
        raise TypeError(f"{name} has dtype {t.dtype}, expected {dtype}")
    if t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t


_TAG_DTYPES = (torch.int32, torch.uint32) if hasattr(torch, "uint32") else (torch.int32,)


def kv_tag_check(page_tags, page_table, expected_tags, seq_lens, page_size, abort_out,
                 num_aborted=None, stream=None):
    """Batched page-tag integrity check; writes abort_out [B] (uint8)."""
    _need(page_tags, _TAG_DTYPES, 1, "page_tags")
    _need(page_table, torch.int32, 2, "page_table")
    _need(expected_tags, _TAG_DTYPES, 2, "expected_tags")
    _need(seq_lens, torch.int32, 1, "seq_lens")
    _need(abort_out, torch.uint8, 1, "abort_out")
    B, MP = page_table.shape
    if num_aborted is not None:
        _need(num_aborted, torch.int32, 1, "num_aborted")
    _check("kv_tag_check", _load().kv_tag_check(
        _ptr(page_tags), page_tags.shape[0], _ptr(page_table), _ptr(expected_tags), MP,
        _ptr(seq_lens), B, page_size, _ptr(abort_out), _ptr(num_aborted), _stream(stream)))


def kv_retag_pages(page_tags, pages, stream=None):
    """Bump (mod 2^32) the tag of every listed page id inside the pool, in place."""
    _need(page_tags, _TAG_DTYPES, 1, "page_tags")
    _need(pages, torch.int32, 1, "pages")
    _check("kv_retag_pages", _load().kv_retag_pages(
        _ptr(page_tags), page_tags.shape[0], _ptr(pages), pages.shape[0], _stream(stream)))


def kv_expected_tags(page_tags, page_table, seq_lens, page_size, expected_tags, stream=None):
    """Rebuild each request's expected tags from the current page tags, in place."""
    _need(page_tags, _TAG_DTYPES, 1, "page_tags")
    _need(page_table, torch.int32, 2, "page_table")
    _need(seq_lens, torch.int32, 1, "seq_lens")
    _need(expected_tags, _TAG_DTYPES, 2, "expected_tags")
    B, MP = page_table.shape
    _check("kv_expected_tags", _load().kv_expected_tags(
        _ptr(page_tags), page_tags.shape[0], _ptr(page_table), MP, _ptr(seq_lens), B, page_size,
        _ptr(expected_tags), _stream(stream)))


def kv_append_fp8(k_new, v_new, page_table, seq_lens, page_size, k_scale, v_scale,
                  k_cache, v_cache, abort=None, stream=None):
    """Quantise each request's new K/V token to E4M3 and write it into its page."""
    _need(k_new, torch.bfloat16, 3, "k_new")
    _need(v_new, torch.bfloat16, 3, "v_new")
    _need(page_table, torch.int32, 2, "page_table")
    _need(seq_lens, torch.int32, 1, "seq_lens")
    _need(k_cache, torch.uint8, 4, "k_cache")
    _need(v_cache, torch.uint8, 4, "v_cache")
    if abort is not None:
        _need(abort, torch.uint8, 1, "abort")
    B, Hkv, D = k_new.shape
    _check("kv_append_fp8", _load().kv_append_fp8(
        _ptr(k_new), _ptr(v_new), _ptr(page_table), page_table.shape[1], _ptr(seq_lens), B, Hkv,
        D, page_size, float(k_scale), float(v_scale), _ptr(k_cache), _ptr(v_cache),
        k_cache.shape[0], _ptr(abort), _stream(stream)))


def kv_append_bf16(k_new, v_new, page_table, seq_lens, page_size, k_cache, v_cache,
                   abort=None, stream=None):
    """Write each request's new BF16 K/V token into its page."""
    _need(k_new, torch.bfloat16, 3, "k_new")
    _need(v_new, torch.bfloat16, 3, "v_new")
    _need(page_table, torch.int32, 2, "page_table")
    _need(seq_lens, torch.int32, 1, "seq_lens")
    _need(k_cache, torch.bfloat16, 4, "k_cache")
    _need(v_cache, torch.bfloat16, 4, "v_cache")
    if abort is not None:
        _need(abort, torch.uint8, 1, "abort")
    B, Hkv, D = k_new.shape
    _check("kv_append_bf16", _load().kv_append_bf16(
        _ptr(k_new), _ptr(v_new), _ptr(page_table), page_table.shape[1], _ptr(seq_lens), B, Hkv,
        D, page_size, _ptr(k_cache), _ptr(v_cache), k_cache.shape[0], _ptr(abort),
        _stream(stream)))


def kv_check_append_fp8(page_tags, page_table, expected_tags, seq_lens, page_size, k_new, v_new,
                        k_scale, v_scale, k_cache, v_cache, abort_out, num_aborted=None,
                        stream=None):
    """kv_tag_check then kv_append_fp8 (with that abort mask) in one kernel."""
    _need(page_tags, _TAG_DTYPES, 1, "page_tags")
    _need(page_table, torch.int32, 2, "page_table")
    _need(expected_tags, _TAG_DTYPES, 2, "expected_tags")
    _need(seq_lens, torch.int32, 1, "seq_lens")
    _need(k_new, torch.bfloat16, 3, "k_new")
    _need(v_new, torch.bfloat16, 3, "v_new")
    _need(k_cache, torch.uint8, 4, "k_cache")
    _need(v_cache, torch.uint8, 4, "v_cache")
    _need(abort_out, torch.uint8, 1, "abort_out")
    if num_aborted is not None:
        _need(num_aborted, torch.int32, 1, "num_aborted")
    B, MP = page_table.shape
    _, Hkv, D = k_new.shape
    _check("kv_check_append_fp8", _load().kv_check_append_fp8(
        _ptr(page_tags), k_cache.shape[0], _ptr(page_table), _ptr(expected_tags), MP,
        _ptr(seq_lens), B, page_size, _ptr(k_new), _ptr(v_new), Hkv, D, float(k_scale),
        float(v_scale), _ptr(k_cache), _ptr(v_cache), _ptr(abort_out), _ptr(num_aborted),
        _stream(stream)))


def kv_check_append_bf16(page_tags, page_table, expected_tags, seq_lens, page_size, k_new, v_new,
                         k_cache, v_cache, abort_out, num_aborted=None, stream=None):
    """kv_tag_check then kv_append_bf16 (with that abort mask) in one kernel."""
    _need(page_tags, _TAG_DTYPES, 1, "page_tags")
    _need(page_table, torch.int32, 2, "page_table")
    _need(expected_tags, _TAG_DTYPES, 2, "expected_tags")
    _need(seq_lens, torch.int32, 1, "seq_lens")
    _need(k_new, torch.bfloat16, 3, "k_new")
    _need(v_new, torch.bfloat16, 3, "v_new")
    _need(k_cache, torch.bfloat16, 4, "k_cache")
    _need(v_cache, torch.bfloat16, 4, "v_cache")
    _need(abort_out, torch.uint8, 1, "abort_out")
    if num_aborted is not None:
        _need(num_aborted, torch.int32, 1, "num_aborted")
    B, MP = page_table.shape
    _, Hkv, D = k_new.shape
    _check("kv_check_append_bf16", _load().kv_check_append_bf16(
        _ptr(page_tags), k_cache.shape[0], _ptr(page_table), _ptr(expected_tags), MP,
        _ptr(seq_lens), B, page_size, _ptr(k_new), _ptr(v_new), Hkv, D, _ptr(k_cache),
        _ptr(v_cache), _ptr(abort_out), _ptr(num_aborted), _stream(stream)))


def kv_requant_pages_fp8(src_pool, src_pages, dst_pool, dst_pages, scale, stream=None):
    """BF16 -> FP8 page handoff: page src_pages[i] -> dst_pages[i]."""
    _need(src_pool, torch.bfloat16, 4, "src_pool")
    _need(dst_pool, torch.uint8, 4, "dst_pool")
    _need(src_pages, torch.int32, 1, "src_pages")
    _need(dst_pages, torch.int32, 1, "dst_pages")
    if src_pages.shape != dst_pages.shape:
        raise ValueError("src_pages and dst_pages must have the same length")
    NPs, Hkv, P, D = src_pool.shape
    if tuple(dst_pool.shape[1:]) != (Hkv, P, D):
        raise ValueError("pools must share [Hkv][P][D]")
    _check("kv_requant_pages_fp8", _load().kv_requant_pages_fp8(
        _ptr(src_pool), NPs, _ptr(src_pages), _ptr(dst_pool), dst_pool.shape[0], _ptr(dst_pages),
        src_pages.shape[0], Hkv, P, D, float(scale), _stream(stream)))


def paged_decode_attn_workspace_size(kv_dtype, batch, num_q_heads, num_kv_heads, head_dim,
                                     num_ctas=0) -> int:
    n = _load().paged_decode_attn_workspace_size(kv_dtype, batch, num_q_heads, num_kv_heads,
                                                 head_dim, num_ctas)
    if n == 0:
        raise PagedKVError("paged_decode_attn_workspace_size", 1,
                           _load().pkv_last_error().decode())
    return int(n)


def alloc_workspace(kv_dtype, batch, num_q_heads, num_kv_heads, head_dim, num_ctas=0,
                    device=None):
    """A uint8 CUDA tensor large enough for the attention call."""
    n = paged_decode_attn_workspace_size(kv_dtype, batch, num_q_heads, num_kv_heads, head_dim,
                                         num_ctas)
    return torch.zeros(n, dtype=torch.uint8, device=device or "cuda")


def paged_decode_attn_fp8_prefix_workspace_size(batch, num_q_heads, num_kv_heads, head_dim,
                                                num_ctas=0):
    n = _load().paged_decode_attn_fp8_prefix_workspace_size(int(batch), int(num_q_heads),
                                                            int(num_kv_heads), int(head_dim),
                                                            int(num_ctas))
    if n == 0:
        raise PagedKVError("paged_decode_attn_fp8_prefix_workspace_size", 1,
                           _load().pkv_last_error().decode())
    return int(n)


def alloc_prefix_workspace(batch, num_q_heads, num_kv_heads, head_dim, num_ctas=0, device=None):
    """A uint8 CUDA tensor large enough for paged_decode_attn_fp8_prefix."""
    n = paged_decode_attn_fp8_prefix_workspace_size(batch, num_q_heads, num_kv_heads, head_dim,
                                                    num_ctas)
    return torch.zeros(n, dtype=torch.uint8, device=device or "cuda")


def paged_decode_attn_plan(kv_dtype, batch, num_q_heads, num_kv_heads, head_dim, max_pages,
                           page_size, num_ctas=0):
    """The attention call's work split on the current device:
    (cluster_size, ctas, launches); cluster_size 0 means split-K + merge."""
    out = [ctypes.c_int32(0) for _ in range(3)]
    _check("paged_decode_attn_plan", _load().paged_decode_attn_plan(
        int(kv_dtype), int(batch), int(num_q_heads), int(num_kv_heads), int(head_dim),
        int(max_pages), int(page_size), int(num_ctas), *[ctypes.byref(o) for o in out]))
    return tuple(int(o.value) for o in out)


def workspace_status(workspace) -> int:
    """The workspace status word (0 = no internal wait ever expired)."""
    return int(workspace[:4].view(torch.int32).item())


def _attn_common(q, k_cache, page_table, seq_lens, out, lse, workspace, abort):
    _need(q, torch.bfloat16, 3, "q")
    _need(page_table, torch.int32, 2, "page_table")
    _need(seq_lens, torch.int32, 1, "seq_lens")
    _need(out, torch.bfloat16, 3, "out")
    _need(lse, torch.float32, 2, "lse")
    _need(workspace, torch.uint8, 1, "workspace")
    if abort is not None:
        _need(abort, torch.uint8, 1, "abort")
    B, Hq, D = q.shape
    NP, Hkv, P, D2 = k_cache.shape
    if D2 != D:
        raise ValueError("head_dim of q and cache differ")
    return B, Hq, D, NP, Hkv, P


def paged_decode_attn_fp8(q, k_cache, v_cache, k_scale, v_scale, page_table, seq_lens,
                          sm_scale, out, lse, workspace, abort=None, num_ctas=0, stream=None):
    """Decode attention over a paged E4M3 cache; writes out (bf16) and lse (fp32)."""
    _need(k_cache, torch.uint8, 4, "k_cache")
    _need(v_cache, torch.uint8, 4, "v_cache")
    B, Hq, D, NP, Hkv, P = _attn_common(q, k_cache, page_table, seq_lens, out, lse, workspace,
                                        abort)
    _check("paged_decode_attn_fp8", _load().paged_decode_attn_fp8(
        _ptr(q), _ptr(k_cache), _ptr(v_cache), float(k_scale), float(v_scale), _ptr(page_table),
        page_table.shape[1], _ptr(seq_lens), B, Hq, Hkv, D, P, NP, float(sm_scale), _ptr(abort),
        _ptr(out), _ptr(lse), _ptr(workspace), workspace.numel(), num_ctas, _stream(stream)))


def paged_decode_attn_fp8_prefix(q, k_cache, v_cache, k_scale, v_scale, page_table, seq_lens,
                                 sm_scale, out, lse, workspace, abort=None, num_ctas=0,
                                 chunk_begin_out=None, stream=None):
    """paged_decode_attn_fp8 for batches whose consecutive requests share leading
    pages: the shared chunks are attended once per group.  chunk_begin_out
    (optional int32 [batch] CUDA tensor) receives, per request, the leading
    chunks attended in its tile (all of them when the tile finished it)."""
    _need(k_cache, torch.uint8, 4, "k_cache")
    _need(v_cache, torch.uint8, 4, "v_cache")
    B, Hq, D, NP, Hkv, P = _attn_common(q, k_cache, page_table, seq_lens, out, lse, workspace,
                                        abort)
    if chunk_begin_out is not None:
        _need(chunk_begin_out, torch.int32, 1, "chunk_begin_out")
        if chunk_begin_out.numel() < B:
            raise ValueError("chunk_begin_out needs batch entries")
    _check("paged_decode_attn_fp8_prefix", _load().paged_decode_attn_fp8_prefix(
        _ptr(q), _ptr(k_cache), _ptr(v_cache), float(k_scale), float(v_scale), _ptr(page_table),
        page_table.shape[1], _ptr(seq_lens), B, Hq, Hkv, D, P, NP, float(sm_scale), _ptr(abort),
        _ptr(out), _ptr(lse), _ptr(workspace), workspace.numel(), num_ctas,
        _ptr(chunk_begin_out), _stream(stream)))


def paged_decode_attn_bf16(q, k_cache, v_cache, page_table, seq_lens, sm_scale, out, lse,
                           workspace, abort=None, num_ctas=0, stream=None):
    """Decode attention over a paged BF16 cache; writes out (bf16) and lse (fp32)."""
    _need(k_cache, torch.bfloat16, 4, "k_cache")
    _need(v_cache, torch.bfloat16, 4, "v_cache")
    B, Hq, D, NP, Hkv, P = _attn_common(q, k_cache, page_table, seq_lens, out, lse, workspace,
                                        abort)
    _check("paged_decode_attn_bf16", _load().paged_decode_attn_bf16(
        _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(page_table), page_table.shape[1],
        _ptr(seq_lens), B, Hq, Hkv, D, P, NP, float(sm_scale), _ptr(abort), _ptr(out), _ptr(lse),
        _ptr(workspace), workspace.numel(), num_ctas, _stream(stream)))


def paged_decode_attn_fp8_noalloc(q, k_cache, v_cache, k_scale, v_scale, page_table, seq_lens,
                                  sm_scale, out, lse, abort=None, num_ctas=0, stream=None):
    """paged_decode_attn_fp8 without a workspace argument, for callers that
    cannot allocate device memory: the library uses its built-in scratch array
    (see paged_decode_attn_fp8_noalloc_scratch_bytes()).  Calls that overlap
    on the GPU share that array and must not run concurrently."""
    _need(k_cache, torch.uint8, 4, "k_cache")
    _need(v_cache, torch.uint8, 4, "v_cache")
    _need(q, torch.bfloat16, 3, "q")
    _need(page_table, torch.int32, 2, "page_table")
    _need(seq_lens, torch.int32, 1, "seq_lens")
    _need(out, torch.bfloat16, 3, "out")
    _need(lse, torch.float32, 2, "lse")
    if abort is not None:
        _need(abort, torch.uint8, 1, "abort")
    B, Hq, D = q.shape
    NP, Hkv, P, _ = k_cache.shape
    _check("paged_decode_attn_fp8_noalloc", _load().paged_decode_attn_fp8_noalloc(
        _ptr(q), _ptr(k_cache), _ptr(v_cache), float(k_scale), float(v_scale), _ptr(page_table),
        page_table.shape[1], _ptr(seq_lens), B, Hq, Hkv, D, P, NP, float(sm_scale), _ptr(abort),
        _ptr(out), _ptr(lse), num_ctas, _stream(stream)))


def noalloc_scratch_bytes() -> int:
    return int(_load().paged_decode_attn_fp8_noalloc_scratch_bytes())


def noalloc_status(stream=None) -> int:
    """The built-in scratch's status word after the last no-allocation call
    on the current device (0 = no internal wait expired).  Copies 4 bytes to
    host memory on `stream` and waits for that copy."""
    import numpy as np
    word = np.zeros(1, dtype=np.uint32)
    _check("paged_decode_attn_fp8_noalloc_status", _load().paged_decode_attn_fp8_noalloc_status(
        ctypes.c_void_p(word.ctypes.data), _stream(stream)))
    (torch.cuda.current_stream() if stream is None else stream).synchronize()
    return int(word[0])


def version() -> int:
    return int(_load().pkv_version())


def int4_dequant_gemv(x, w_tiles, scales, y, group_size=128, status=None, stream=None):
    """y = x W^T with W expanded from tiled INT4 codes and per-group bf16
    scales (layouts in include/pagedkv.h; int4_tile_layout builds them)."""
    _need(x, torch.bfloat16, 2, "x")
    _need(w_tiles, torch.uint8, 4, "w_tiles")
    _need(scales, torch.bfloat16, 3, "scales")
    _need(y, torch.bfloat16, 2, "y")
    if status is not None:
        _need(status, _TAG_DTYPES, 1, "status")
    B, k = x.shape
    n = w_tiles.shape[0] * 128
    if tuple(w_tiles.shape) != (n // 128, k // 256, 128, 128) or y.shape != (B, n) or \
            k % group_size or tuple(scales.shape) != (n // 128, k // group_size, 128):
        raise ValueError("inconsistent INT4 GEMV shapes")
    _check("int4_dequant_gemv", _load().int4_dequant_gemv(
        _ptr(x), _ptr(w_tiles), _ptr(scales), B, n, k, group_size, _ptr(y), _ptr(status),
        _stream(stream)))


def int4_tile_layout(w_rowmajor, scales_rows, group_size=128):
    """Re-lay a row-major code matrix [n][k/2] (uint8, two codes per byte,
    even column in the low nibble) and row-wise scales [n][k/group_size]
    into the layouts int4_dequant_gemv reads: each 32-bit word of 8 columns
    holds the even columns in its low half-word and the odd ones in its high
    half-word, and rows are cut into 128 x 256 tiles.  Pure data movement,
    done once per weight matrix."""
    n, half = w_rowmajor.shape
    k = 2 * half
    if n % 128 or k % 256 or tuple(scales_rows.shape) != (n, k // group_size):
        raise ValueError("n must be a multiple of 128, k of 256, scales [n][k/group]")
    c = torch.stack([w_rowmajor & 0xF, w_rowmajor >> 4], dim=-1).reshape(n, k // 8, 8)
    words = torch.stack([c[..., 0] | (c[..., 2] << 4), c[..., 4] | (c[..., 6] << 4),
                         c[..., 1] | (c[..., 3] << 4), c[..., 5] | (c[..., 7] << 4)], dim=-1)
    packed = words.reshape(n, half)
    tiles = packed.reshape(n // 128, 128, k // 256, 128).permute(0, 2, 1, 3).contiguous()
    sc = scales_rows.reshape(n // 128, 128, k // group_size).permute(0, 2, 1).contiguous()
    return tiles, sc
