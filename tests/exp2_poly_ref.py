"""Host-side pieces for the exp2 polynomial tests: the coefficients as the header states
them, and a float32 restatement of the header's steps (numpy), used to check the method's
error bound on the CPU and the device code's bits on the GPU."""
import os
import re

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
HEADER = os.path.join(os.path.dirname(HERE), "gqa_exact_attention_b200", "csrc", "exp2_poly.cuh")


def header_constants() -> dict:
    src = open(HEADER).read()
    out = {}
    for name in ("kRound", "kLow", "c1", "c2", "c3"):
        m = re.search(rf"static constexpr float {name} = ([-0-9.e+]+)f;", src)
        assert m, name
        out[name] = np.float32(float(m.group(1)))
    return out


def _fma32(a, b, c):
    # a*b is exact in fp64 (24-bit significands); one fp64 add, then rounding to fp32
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


def exp2_poly_f32(x) -> np.ndarray:
    k = header_constants()
    x = np.maximum(np.asarray(x, dtype=np.float32), k["kLow"])
    t = (x + k["kRound"]).astype(np.float32)
    r = (t - k["kRound"]).astype(np.float32)
    f = (x - r).astype(np.float32)
    one = np.float32(1.0)
    q = _fma32(f, np.full_like(f, k["c3"]), np.full_like(f, k["c2"]))
    q = _fma32(q, f, np.full_like(f, k["c1"]))
    q = _fma32(q, f, np.full_like(f, one))
    bits = q.view(np.int32).astype(np.int64) + (t.view(np.int32).astype(np.int64) << 23)
    return (bits & 0xFFFFFFFF).astype(np.uint32).view(np.float32)
