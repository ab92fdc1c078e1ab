"""Exact grouped-query attention forward on B200 (sm_100a): Python binding.

Argument marshalling only: every step of the computation runs in the CUDA kernels of
``libgqa_attn.so`` (built in-tree from ``csrc/``).  PyTorch supplies device memory and
the current stream.  There is no fallback: if the library cannot be loaded, the calls
raise.

The C contract is ``include/gqa_attn.h``; the names here are the same.
"""
from __future__ import annotations

import ctypes
import math
import os

__all__ = [
    "gqa_attn_fwd", "gqa_attn_choose", "gqa_attn_workspace_bytes", "gqa_attn_status_string",
    "gqa_attn_device_status", "gqa_attn_fwd_noalloc", "gqa_attn_fwd_kvcache",
    "gqa_attn_fwd_paged", "gqa_attn_fwd_fp8", "GqaError", "lib_path", "load",
    "GQA_NOALLOC_SCRATCH_BYTES",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
lib_path = os.path.join(_HERE, "libgqa_attn.so")

GQA_OK = 0
STATUS_NAMES = {
    0: "GQA_OK", 1: "GQA_ERR_NULL", 2: "GQA_ERR_SHAPE", 3: "GQA_ERR_HEADS",
    4: "GQA_ERR_HEADDIM", 5: "GQA_ERR_ALIGN", 6: "GQA_ERR_ARCH", 7: "GQA_ERR_ALLOC",
    8: "GQA_ERR_CUDA", 9: "GQA_ERR_TIMEOUT", 10: "GQA_ERR_SCRATCH",
}

# size of the library's fixed split-KV scratch used by gqa_attn_fwd_noalloc (the header's
# GQA_NOALLOC_SCRATCH_BYTES)
GQA_NOALLOC_SCRATCH_BYTES = 32 * 1024 * 1024


def _nvtx_enabled() -> bool:
    return os.environ.get("GQA_NVTX", "") not in ("", "0")


class _range:
    """An NVTX range named after the entry point around each library call, when GQA_NVTX is
    set (for timeline profilers); otherwise nothing.  It marks the host-side call, inside
    which the kernels are launched."""

    def __init__(self, name: str):
        self.name = name
        self.on = _nvtx_enabled()

    def __enter__(self):
        if self.on:
            import torch
            torch.cuda.nvtx.range_push(self.name)
        return self

    def __exit__(self, *exc):
        if self.on:
            import torch
            torch.cuda.nvtx.range_pop()
        return False


class GqaError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {msg}")
        self.status = status


_lib = None


def load():
    """Load ``libgqa_attn.so`` (building it in-tree first if it is absent or stale and
    nvcc is available).  Raises if it cannot be loaded."""
    global _lib
    if _lib is not None:
        return _lib
    try:
        from . import _build
        if _build._stale() and _have_nvcc():
            _build.build()
    except Exception as e:  # a failed build must not hide behind an old library
        if not os.path.exists(lib_path):
            raise RuntimeError(f"libgqa_attn.so is missing and could not be built: {e}") from e
    if not os.path.exists(lib_path):
        raise RuntimeError(f"libgqa_attn.so not found at {lib_path}; run the package build")
    L = ctypes.CDLL(lib_path)
    i, f, p, sz = ctypes.c_int, ctypes.c_float, ctypes.c_void_p, ctypes.c_size_t
    L.gqa_attn_fwd.argtypes = [p, p, p, p, p, i, i, i, i, i, i, f, i, i, i, p]
    L.gqa_attn_fwd.restype = i
    L.gqa_attn_choose.argtypes = [i, i, i, i, i, i, i, i, ctypes.POINTER(i), ctypes.POINTER(i)]
    L.gqa_attn_choose.restype = i
    L.gqa_attn_workspace_bytes.argtypes = [i, i, i, i, i, i, i, i, i]
    L.gqa_attn_workspace_bytes.restype = sz
    L.gqa_attn_status_string.argtypes = [i]
    L.gqa_attn_status_string.restype = ctypes.c_char_p
    L.gqa_attn_device_status.argtypes = [i]
    L.gqa_attn_device_status.restype = i
    L.gqa_attn_fwd_noalloc.argtypes = [p, p, p, p, p, i, i, i, i, i, i, f, i, i, i, p]
    L.gqa_attn_fwd_noalloc.restype = i
    L.gqa_attn_fwd_kvcache.argtypes = [p, p, p, p, p, i, p, i, i, i, i, i, i, f, i, i, i, p]
    L.gqa_attn_fwd_kvcache.restype = i
    L.gqa_attn_fwd_paged.argtypes = [p, p, p, p, i, p, i, i, p, i, p, i, i, i, i, i, f, i, i, i, p]
    L.gqa_attn_fwd_paged.restype = i
    L.gqa_attn_fwd_fp8.argtypes = [p, p, p, f, f, f, p, p, i, p, i, i, i, i, i, i, f, i, i, i, p]
    L.gqa_attn_fwd_fp8.restype = i
    _lib = L
    return L


def _have_nvcc() -> bool:
    from shutil import which
    return which("nvcc") is not None


def gqa_attn_status_string(status: int) -> str:
    return load().gqa_attn_status_string(int(status)).decode()


def _check(status: int):
    if status != GQA_OK:
        raise GqaError(status, gqa_attn_status_string(status))


def gqa_attn_choose(B, Sq, Sk, Hq, Hk, d, causal, num_sms=0):
    """The heuristic's (pack_gqa, num_splits) for this shape, planned for ``num_sms`` SMs
    (0: the current device's count, as gqa_attn_fwd plans; 148 without a device)."""
    pk, ns = ctypes.c_int(), ctypes.c_int()
    _check(load().gqa_attn_choose(B, Sq, Sk, Hq, Hk, d, int(bool(causal)), num_sms,
                                  ctypes.byref(pk), ctypes.byref(ns)))
    return pk.value, ns.value


def gqa_attn_workspace_bytes(B, Sq, Sk, Hq, Hk, d, causal, pack_gqa=-1, num_splits=0):
    return int(load().gqa_attn_workspace_bytes(B, Sq, Sk, Hq, Hk, d, int(bool(causal)),
                                               pack_gqa, num_splits))


def gqa_attn_device_status(reset: bool = False) -> int:
    """The device status word (0 = ok, 9 = a bounded wait timed out); synchronous."""
    return int(load().gqa_attn_device_status(int(bool(reset))))


def gqa_attn_fwd(q, k, v, out=None, lse=None, scale=None, causal=False, pack_gqa=-1,
                 num_splits=0, stream=None, _entry="gqa_attn_fwd"):
    """out, lse = gqa_attn_fwd(q, k, v, ...) on the current CUDA stream.

    q: bf16 [B, Sq, Hq, d]; k, v: bf16 [B, Sk, Hk, d]; all contiguous CUDA tensors.
    out: fp32 [B, Sq, Hq, d] and lse: fp32 [B, Hq, Sq] are allocated when not given.
    scale defaults to 1/sqrt(d).
    """
    import torch

    B, Sq, Hq, d = q.shape
    Sk, Hk = k.shape[1], k.shape[2]
    for name, t in (("q", q), ("k", k), ("v", v)):
        if t.dtype != torch.bfloat16 or not t.is_cuda or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous bf16 CUDA tensor")
    if k.shape != v.shape or k.shape[0] != B or k.shape[3] != d:
        raise ValueError("k and v must be [B, Sk, Hk, d] matching q")
    if out is None:
        out = torch.empty((B, Sq, Hq, d), dtype=torch.float32, device=q.device)
    if lse is None:
        lse = torch.empty((B, Hq, Sq), dtype=torch.float32, device=q.device)
    for name, t in (("out", out), ("lse", lse)):
        if t.dtype != torch.float32 or not t.is_contiguous() or t.device != q.device:
            raise ValueError(f"{name} must be a contiguous fp32 tensor on q's device")
    if tuple(out.shape) != (B, Sq, Hq, d) or tuple(lse.shape) != (B, Hq, Sq):
        raise ValueError("out must be [B, Sq, Hq, d] and lse [B, Hq, Sq]")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if stream is None:
        stream = torch.cuda.current_stream(q.device)
    with torch.cuda.device(q.device), _range(_entry):
        _check(getattr(load(), _entry)(q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                       out.data_ptr(), lse.data_ptr(), B, Sq, Sk, Hq, Hk, d,
                                       float(scale), int(bool(causal)), int(pack_gqa),
                                       int(num_splits), stream.cuda_stream))
    return out, lse


def gqa_attn_fwd_noalloc(q, k, v, out, lse, scale=None, causal=False, pack_gqa=-1,
                         num_splits=0, stream=None):
    """gqa_attn_fwd for callers that must not allocate device memory (a serving process
    that reserved its device memory up front, code that must not block on the device,
    a host under another runtime's allocator).  ``out`` and ``lse`` are required; the
    split-KV partials use the library's fixed scratch of GQA_NOALLOC_SCRATCH_BYTES per
    device, and calls that overlap on the GPU race on it."""
    if out is None or lse is None:
        raise ValueError("gqa_attn_fwd_noalloc writes into caller-provided out and lse")
    return gqa_attn_fwd(q, k, v, out=out, lse=lse, scale=scale, causal=causal,
                        pack_gqa=pack_gqa, num_splits=num_splits, stream=stream,
                        _entry="gqa_attn_fwd_noalloc")


GQA_OUT_F32 = 0
GQA_OUT_BF16 = 1


def gqa_attn_fwd_kvcache(q, k_cache, v_cache, cache_seqlens=None, out=None, lse=None,
                         out_dtype=None, scale=None, causal=False, pack_gqa=-1, num_splits=0,
                         stream=None):
    """out, lse = gqa_attn_fwd_kvcache(q, k_cache, v_cache, cache_seqlens, ...).

    k_cache, v_cache: bf16 [B, Sk, Hk, d] (Sk = the cache's capacity per sequence);
    cache_seqlens: int32 CUDA tensor [B] (sequence b uses keys [0, cache_seqlens[b]),
    clamped to [0, Sk]) or None for full length.  out is fp32 or bf16 [B, Sq, Hq, d]
    (``out_dtype`` torch.float32 / torch.bfloat16 when out is not given; default fp32).
    Causal masks are bottom-right aligned to each sequence's own length.
    """
    import torch

    B, Sq, Hq, d = q.shape
    Sk, Hk = k_cache.shape[1], k_cache.shape[2]
    for name, t in (("q", q), ("k_cache", k_cache), ("v_cache", v_cache)):
        if t.dtype != torch.bfloat16 or not t.is_cuda or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous bf16 CUDA tensor")
    if k_cache.shape != v_cache.shape or k_cache.shape[0] != B or k_cache.shape[3] != d:
        raise ValueError("k_cache and v_cache must be [B, Sk, Hk, d] matching q")
    if cache_seqlens is not None:
        if (cache_seqlens.dtype != torch.int32 or not cache_seqlens.is_contiguous()
                or cache_seqlens.device != q.device or tuple(cache_seqlens.shape) != (B,)):
            raise ValueError("cache_seqlens must be a contiguous int32 tensor [B] on q's device")
    if out is None:
        dt = torch.float32 if out_dtype is None else out_dtype
        out = torch.empty((B, Sq, Hq, d), dtype=dt, device=q.device)
    if out.dtype not in (torch.float32, torch.bfloat16) or not out.is_contiguous() \
            or out.device != q.device or tuple(out.shape) != (B, Sq, Hq, d):
        raise ValueError("out must be a contiguous fp32 or bf16 tensor [B, Sq, Hq, d] on q's device")
    if lse is None:
        lse = torch.empty((B, Hq, Sq), dtype=torch.float32, device=q.device)
    if lse.dtype != torch.float32 or not lse.is_contiguous() or tuple(lse.shape) != (B, Hq, Sq):
        raise ValueError("lse must be a contiguous fp32 tensor [B, Hq, Sq]")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if stream is None:
        stream = torch.cuda.current_stream(q.device)
    code = GQA_OUT_BF16 if out.dtype == torch.bfloat16 else GQA_OUT_F32
    with torch.cuda.device(q.device), _range("gqa_attn_fwd_kvcache"):
        _check(load().gqa_attn_fwd_kvcache(
            q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(),
            None if cache_seqlens is None else cache_seqlens.data_ptr(), out.data_ptr(), code,
            lse.data_ptr(), B, Sq, Sk, Hq, Hk, d, float(scale), int(bool(causal)),
            int(pack_gqa), int(num_splits), stream.cuda_stream))
    return out, lse


def gqa_attn_fwd_paged(q, k_pages, v_pages, block_table, cache_seqlens, out=None, lse=None,
                       out_dtype=None, scale=None, causal=False, pack_gqa=-1, num_splits=0,
                       stream=None):
    """out, lse = gqa_attn_fwd_paged(q, k_pages, v_pages, block_table, cache_seqlens, ...).

    k_pages, v_pages: bf16 [num_pages, page_size, Hk, d] page pools; block_table: int32
    CUDA tensor [B, max_pages_per_seq] (key j of sequence b is row j % page_size of page
    block_table[b, j // page_size]); cache_seqlens: int32 CUDA tensor [B].  out is fp32 or
    bf16 [B, Sq, Hq, d]; lse fp32 [B, Hq, Sq].  Causal masks are bottom-right aligned to
    each sequence's own length.
    """
    import torch

    B, Sq, Hq, d = q.shape
    num_pages, page_size, Hk = k_pages.shape[0], k_pages.shape[1], k_pages.shape[2]
    for name, t in (("q", q), ("k_pages", k_pages), ("v_pages", v_pages)):
        if t.dtype != torch.bfloat16 or not t.is_cuda or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous bf16 CUDA tensor")
    if k_pages.shape != v_pages.shape or k_pages.shape[3] != d:
        raise ValueError("k_pages and v_pages must be [num_pages, page_size, Hk, d] matching q")
    for name, t in (("block_table", block_table), ("cache_seqlens", cache_seqlens)):
        if t.dtype != torch.int32 or not t.is_contiguous() or t.device != q.device:
            raise ValueError(f"{name} must be a contiguous int32 tensor on q's device")
    if block_table.dim() != 2 or block_table.shape[0] != B or tuple(cache_seqlens.shape) != (B,):
        raise ValueError("block_table must be [B, max_pages_per_seq] and cache_seqlens [B]")
    if out is None:
        dt = torch.float32 if out_dtype is None else out_dtype
        out = torch.empty((B, Sq, Hq, d), dtype=dt, device=q.device)
    if out.dtype not in (torch.float32, torch.bfloat16) or not out.is_contiguous() \
            or out.device != q.device or tuple(out.shape) != (B, Sq, Hq, d):
        raise ValueError("out must be a contiguous fp32 or bf16 tensor [B, Sq, Hq, d] on q's device")
    if lse is None:
        lse = torch.empty((B, Hq, Sq), dtype=torch.float32, device=q.device)
    if lse.dtype != torch.float32 or not lse.is_contiguous() or tuple(lse.shape) != (B, Hq, Sq):
        raise ValueError("lse must be a contiguous fp32 tensor [B, Hq, Sq]")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if stream is None:
        stream = torch.cuda.current_stream(q.device)
    code = GQA_OUT_BF16 if out.dtype == torch.bfloat16 else GQA_OUT_F32
    with torch.cuda.device(q.device), _range("gqa_attn_fwd_paged"):
        _check(load().gqa_attn_fwd_paged(
            q.data_ptr(), k_pages.data_ptr(), v_pages.data_ptr(), block_table.data_ptr(),
            int(block_table.shape[1]), cache_seqlens.data_ptr(), num_pages, page_size,
            out.data_ptr(), code, lse.data_ptr(), B, Sq, Hq, Hk, d, float(scale),
            int(bool(causal)), int(pack_gqa), int(num_splits), stream.cuda_stream))
    return out, lse


def gqa_attn_fwd_fp8(q, k, v, q_scale, k_scale, v_scale, cache_seqlens=None, out=None,
                     lse=None, out_dtype=None, scale=None, causal=False, pack_gqa=-1,
                     num_splits=0, stream=None):
    """out, lse = gqa_attn_fwd_fp8(q, k, v, q_scale, k_scale, v_scale, ...).

    q [B, Sq, Hq, d], k and v [B, Sk, Hk, d]: e4m3 tensors (torch.float8_e4m3fn or the raw
    bytes as torch.uint8); the values they stand for are q * q_scale, k * k_scale and
    v * v_scale (per-tensor fp32 scales).  cache_seqlens as in gqa_attn_fwd_kvcache.  out is
    fp32 or bf16 [B, Sq, Hq, d]; lse fp32 [B, Hq, Sq].  scale defaults to 1/sqrt(d).
    """
    import torch

    B, Sq, Hq, d = q.shape
    Sk, Hk = k.shape[1], k.shape[2]
    for name, t in (("q", q), ("k", k), ("v", v)):
        if t.element_size() != 1 or not t.is_cuda or not t.is_contiguous() or \
                t.dtype not in (torch.uint8, getattr(torch, "float8_e4m3fn", torch.uint8)):
            raise ValueError(f"{name} must be a contiguous e4m3 (or uint8) CUDA tensor")
    if k.shape != v.shape or k.shape[0] != B or k.shape[3] != d:
        raise ValueError("k and v must be [B, Sk, Hk, d] matching q")
    if cache_seqlens is not None:
        if (cache_seqlens.dtype != torch.int32 or not cache_seqlens.is_contiguous()
                or cache_seqlens.device != q.device or tuple(cache_seqlens.shape) != (B,)):
            raise ValueError("cache_seqlens must be a contiguous int32 tensor [B] on q's device")
    if out is None:
        dt = torch.float32 if out_dtype is None else out_dtype
        out = torch.empty((B, Sq, Hq, d), dtype=dt, device=q.device)
    if out.dtype not in (torch.float32, torch.bfloat16) or not out.is_contiguous() \
            or out.device != q.device or tuple(out.shape) != (B, Sq, Hq, d):
        raise ValueError("out must be a contiguous fp32 or bf16 tensor [B, Sq, Hq, d] on q's device")
    if lse is None:
        lse = torch.empty((B, Hq, Sq), dtype=torch.float32, device=q.device)
    if lse.dtype != torch.float32 or not lse.is_contiguous() or tuple(lse.shape) != (B, Hq, Sq):
        raise ValueError("lse must be a contiguous fp32 tensor [B, Hq, Sq]")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if stream is None:
        stream = torch.cuda.current_stream(q.device)
    code = GQA_OUT_BF16 if out.dtype == torch.bfloat16 else GQA_OUT_F32
    with torch.cuda.device(q.device), _range("gqa_attn_fwd_fp8"):
        _check(load().gqa_attn_fwd_fp8(
            q.data_ptr(), k.data_ptr(), v.data_ptr(), float(q_scale), float(k_scale),
            float(v_scale), None if cache_seqlens is None else cache_seqlens.data_ptr(),
            out.data_ptr(), code, lse.data_ptr(), B, Sq, Sk, Hq, Hk, d, float(scale),
            int(bool(causal)), int(pack_gqa), int(num_splits), stream.cuda_stream))
    return out, lse
