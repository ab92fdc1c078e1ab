"""Seeded synthetic inputs for the GQA attention tests and benchmark.

Shared input infrastructure: the oracle side and the GPU side both take Q, K and V
from here, element for element the same.  It holds none of the attention
arithmetic; the generator's definition is in ``inputs/gen.h``.

Host generation goes through ``libgqa_inputs_host.so`` (gcc, OpenMP); device
generation, for inputs too large to copy from the host, through
``libgqa_inputs_dev.so`` (nvcc, sm_100a).  Both are built in-tree by :func:`build`.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
HOST_LIB = os.path.join(HERE, "libgqa_inputs_host.so")
DEV_LIB = os.path.join(HERE, "libgqa_inputs_dev.so")

# tensor ids of the generator's counter space
TID_Q, TID_K, TID_V = 1, 2, 3


def _stale(target, sources):
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(s) > t for s in sources)


def build(device: bool = True) -> None:
    """Compile the host generator (and, with ``device``, the CUDA generator)."""
    srcs = [os.path.join(HERE, "gen.c"), os.path.join(HERE, "gen.h")]
    if _stale(HOST_LIB, srcs):
        subprocess.run(["gcc", "-O2", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
                        "-o", HOST_LIB, srcs[0], "-lm"], check=True)
    dsrcs = [os.path.join(HERE, "gen_device.cu")]
    if device and _stale(DEV_LIB, dsrcs):
        subprocess.run(["nvcc", "-O3", "-shared", "-Xcompiler", "-fPIC",
                        "-gencode", "arch=compute_100a,code=sm_100a",
                        "-o", DEV_LIB, dsrcs[0]], check=True)


_host = None
_dev = None


def _host_lib():
    global _host
    if _host is None:
        build(device=False)
        lib = ctypes.CDLL(HOST_LIB)
        u64, p = ctypes.c_uint64, ctypes.c_void_p
        lib.gqa_gen_bf16_one.argtypes = [u64, u64, u64]
        lib.gqa_gen_bf16_one.restype = ctypes.c_uint16
        lib.gqa_gen_bf16_range.argtypes = [u64, u64, u64, u64, p]
        lib.gqa_gen_bf16_range.restype = None
        lib.gqa_gen_bf16_strided.argtypes = [u64, u64, u64, u64, u64, u64, p]
        lib.gqa_gen_bf16_strided.restype = None
        lib.gqa_e4m3_rne_from_double.argtypes = [ctypes.c_double]
        lib.gqa_e4m3_rne_from_double.restype = ctypes.c_uint8
        lib.gqa_gen_e4m3_range.argtypes = [u64, u64, u64, u64, ctypes.c_double, p]
        lib.gqa_gen_e4m3_range.restype = None
        _host = lib
    return _host


def _dev_lib():
    global _dev
    if _dev is None:
        build(device=True)
        lib = ctypes.CDLL(DEV_LIB)
        u64, p = ctypes.c_uint64, ctypes.c_void_p
        lib.gqa_gen_bf16_device.argtypes = [u64, u64, u64, u64, p, p]
        lib.gqa_gen_bf16_device.restype = ctypes.c_int
        lib.gqa_gen_e4m3_device.argtypes = [u64, u64, u64, u64, ctypes.c_double, p, p]
        lib.gqa_gen_e4m3_device.restype = ctypes.c_int
        _dev = lib
    return _dev


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns (uint16) to float64."""
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def bits_range(seed: int, tid: int, start: int, count: int) -> np.ndarray:
    out = np.empty(count, dtype=np.uint16)
    if count:
        _host_lib().gqa_gen_bf16_range(seed, tid, start, count, out.ctypes.data)
    return out


def bits_tensor(seed: int, tid: int, shape) -> np.ndarray:
    """The whole tensor (row-major ``shape``) as bf16 bit patterns."""
    n = int(np.prod(shape))
    return bits_range(seed, tid, 0, n).reshape(shape)


def bits_strided(seed: int, tid: int, offset: int, inner: int, outer: int,
                 outer_stride: int) -> np.ndarray:
    out = np.empty(inner * outer, dtype=np.uint16)
    if inner * outer:
        _host_lib().gqa_gen_bf16_strided(seed, tid, offset, inner, outer, outer_stride,
                                         out.ctypes.data)
    return out.reshape(outer, inner)


def head_rows_f64(seed: int, tid: int, shape, b: int, h: int, s_lo: int = 0,
                  s_hi: int | None = None) -> np.ndarray:
    """Rows ``[b, s_lo:s_hi, h, :]`` of a BSHD tensor of ``shape`` (B, S, H, d), in fp64."""
    B, S, H, d = shape
    if s_hi is None:
        s_hi = S
    off = ((b * S + s_lo) * H + h) * d
    return bf16_bits_to_f64(bits_strided(seed, tid, off, d, s_hi - s_lo, H * d))


def host_tensor(seed: int, tid: int, shape):
    """The tensor as a CPU ``torch.bfloat16`` tensor."""
    import torch
    bits = bits_tensor(seed, tid, shape)
    return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16)


def device_tensor(seed: int, tid: int, shape, device="cuda", stream=None):
    """The tensor generated directly in device memory (same values as the host)."""
    import torch
    t = torch.empty(tuple(shape), dtype=torch.bfloat16, device=device)
    n = t.numel()
    if n:
        s = stream if stream is not None else torch.cuda.current_stream(t.device)
        rc = _dev_lib().gqa_gen_bf16_device(seed, tid, 0, n, t.data_ptr(), s.cuda_stream)
        if rc != 0:
            raise RuntimeError(f"device input generator failed (code {rc})")
    return t


# ------------------------------------------------------------------ e4m3 (8-bit) inputs

def e4m3_bits_to_f64(bits: np.ndarray, scale: float = 1.0) -> np.ndarray:
    """Exact value of e4m3 bit patterns (uint8) times scale, in float64 (0x7F/0xFF, the
    format's NaN, never come out of the generator)."""
    b = np.asarray(bits, dtype=np.uint8).astype(np.int64)
    sign = np.where(b & 0x80, -1.0, 1.0)
    e = (b >> 3) & 15
    m = (b & 7).astype(np.float64)
    mag = np.where(e == 0, m * 2.0 ** -9, (1.0 + m / 8.0) * np.exp2((e - 7).astype(np.float64)))
    return sign * mag * scale


def e4m3_encode(t) -> np.ndarray:
    """e4m3 bit patterns of the values t (round to nearest even, saturating), with the
    generator's own encoder."""
    lib = _host_lib()
    flat = np.asarray(t, dtype=np.float64).ravel()
    return np.array([lib.gqa_e4m3_rne_from_double(float(x)) for x in flat],
                    dtype=np.uint8).reshape(np.shape(t))


def e4m3_bits_tensor(seed: int, tid: int, shape, scale: float) -> np.ndarray:
    """e4m3(z / scale) for the whole tensor, as uint8 bit patterns."""
    n = int(np.prod(shape))
    out = np.empty(n, dtype=np.uint8)
    if n:
        _host_lib().gqa_gen_e4m3_range(seed, tid, 0, n, float(scale), out.ctypes.data)
    return out.reshape(shape)


def e4m3_device_tensor(seed: int, tid: int, shape, scale: float, device="cuda", stream=None):
    """The e4m3 tensor generated in device memory, as torch.uint8 (same bits as the host)."""
    import torch
    t = torch.empty(tuple(shape), dtype=torch.uint8, device=device)
    n = t.numel()
    if n:
        s = stream if stream is not None else torch.cuda.current_stream(t.device)
        rc = _dev_lib().gqa_gen_e4m3_device(seed, tid, 0, n, float(scale), t.data_ptr(), s.cuda_stream)
        if rc != 0:
            raise RuntimeError(f"device input generator failed (code {rc})")
    return t
