"""fp64 CPU oracle for exact grouped-query attention forward (ctypes binding).

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference legs of ``bench.py``; never by the product package.  The
computation lives in ``oracle/ref_attn.c`` (plain C, fp64), which cites the passages
of the pages it follows.  It shares no code with the CUDA path.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
LIB = os.path.join(HERE, "liboracle.so")
SRC = os.path.join(HERE, "ref_attn.c")
HDR = os.path.join(HERE, "ref_attn.h")


def compile_oracle(src: str, out: str, include_dir: str = HERE) -> None:
    """gcc a (possibly modified) copy of the oracle source into a shared library."""
    subprocess.run(["gcc", "-O2", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
                    "-I", include_dir, "-o", out, src, "-lm"], check=True)


def build() -> None:
    """Compile ``liboracle.so`` (no CUDA involved)."""
    if os.path.exists(LIB) and all(os.path.getmtime(s) <= os.path.getmtime(LIB)
                                   for s in (SRC, HDR)):
        return
    compile_oracle(SRC, LIB)


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.float64)


class Oracle:
    """The oracle's entry points, bound from one compiled library."""

    def __init__(self, path: str = LIB):
        lib = ctypes.CDLL(path)
        p, i, d, l = ctypes.c_void_p, ctypes.c_int, ctypes.c_double, ctypes.c_long
        lib.gqa_oracle_row.argtypes = [p, p, p, l, i, i, i, i, d, i, i, i, p, p]
        lib.gqa_oracle_row.restype = None
        lib.gqa_oracle_fwd_range.argtypes = [p, p, p, i, i, i, i, i, i, d, i, i, i, p, p]
        lib.gqa_oracle_fwd_range.restype = ctypes.c_int
        lib.gqa_oracle_combine.argtypes = [i, l, i, p, p, p, p]
        lib.gqa_oracle_combine.restype = None
        self.lib = lib

    def attn_fwd(self, q, k, v, scale: float, causal: bool, key_lo: int = 0,
                 key_hi: int | None = None, return_threads: bool = False):
        """Exact GQA forward.  q [B,Sq,Hq,d], k/v [B,Sk,Hk,d].

        Returns ``(out [B,Sq,Hq,d], lse [B,Hq,Sq])`` in fp64, restricted to keys
        ``[key_lo, key_hi)`` when given (the partial one split of the key axis computes).
        """
        q, k, v = _f64(q), _f64(k), _f64(v)
        B, Sq, Hq, d = q.shape
        Bk, Sk, Hk, dk = k.shape
        if Bk != B or dk != d or v.shape != k.shape:
            raise ValueError("shape mismatch")
        if Hk <= 0 or Hq % Hk != 0:
            raise ValueError("Hq must be a multiple of Hk")
        if key_hi is None:
            key_hi = Sk
        out = np.empty((B, Sq, Hq, d), dtype=np.float64)
        lse = np.empty((B, Hq, Sq), dtype=np.float64)
        threads = self.lib.gqa_oracle_fwd_range(
            q.ctypes.data, k.ctypes.data, v.ctypes.data, B, Sq, Sk, Hq, Hk, d, float(scale),
            int(bool(causal)), key_lo, key_hi, out.ctypes.data, lse.ctypes.data)
        if return_threads:
            return out, lse, threads
        return out, lse

    def attn_row(self, q_row, k_rows, v_rows, Sq: int, i: int, scale: float, causal: bool,
                 key_lo: int = 0, key_hi: int | None = None):
        """Query row ``q_row`` [d] at position ``i`` (of ``Sq``) against one kv-head's
        keys ``k_rows``/``v_rows`` [Sk, d].  Returns ``(o [d], lse)``."""
        q_row, k_rows, v_rows = _f64(q_row), _f64(k_rows), _f64(v_rows)
        Sk, d = k_rows.shape
        if key_hi is None:
            key_hi = Sk
        o = np.empty(d, dtype=np.float64)
        lse = np.empty(1, dtype=np.float64)
        self.lib.gqa_oracle_row(q_row.ctypes.data, k_rows.ctypes.data, v_rows.ctypes.data, d, d,
                                Sq, Sk, i, float(scale), int(bool(causal)), key_lo, key_hi,
                                o.ctypes.data, lse.ctypes.data)
        return o, float(lse[0])

    def combine(self, o_parts, lse_parts):
        """Merge split partials: o_parts [S, rows, d], lse_parts [S, rows]."""
        o_parts, lse_parts = _f64(o_parts), _f64(lse_parts)
        S, rows, d = o_parts.shape
        out = np.empty((rows, d), dtype=np.float64)
        lse = np.empty(rows, dtype=np.float64)
        self.lib.gqa_oracle_combine(S, rows, d, o_parts.ctypes.data, lse_parts.ctypes.data,
                                    out.ctypes.data, lse.ctypes.data)
        return out, lse


_default: Oracle | None = None


def default() -> Oracle:
    global _default
    if _default is None:
        build()
        _default = Oracle(LIB)
    return _default


def attn_fwd(*a, **kw):
    return default().attn_fwd(*a, **kw)


def attn_row(*a, **kw):
    return default().attn_row(*a, **kw)


def combine(*a, **kw):
    return default().combine(*a, **kw)
