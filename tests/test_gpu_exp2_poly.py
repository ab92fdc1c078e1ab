"""The device code of the softmax's polynomial 2^x (compiled from its header into a small
probe library) against exact 2^x and against the host restatement of its steps."""
import ctypes
import os
import subprocess
import tempfile

import numpy as np
import pytest

from tests.exp2_poly_ref import HEADER, exp2_poly_f32

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")

HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.fixture(scope="module")
def probe():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    out = os.path.join(tempfile.mkdtemp(), "libexp2probe.so")
    csrc = os.path.dirname(HEADER)
    subprocess.run(["nvcc", "-O3", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a",
                    "-shared", "-Xcompiler", "-fPIC", "-I", csrc, "-o", out,
                    os.path.join(HERE, "exp2_poly_probe.cu")], check=True)
    lib = ctypes.CDLL(out)
    lib.exp2_poly_eval.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int]
    lib.exp2_poly_eval.restype = ctypes.c_int
    return lib


def _eval(lib, x):
    xd = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).cuda()
    yd = torch.empty_like(xd)
    assert lib.exp2_poly_eval(xd.data_ptr(), yd.data_ptr(), xd.numel()) == 0
    return yd.cpu().numpy()


def test_device_polynomial(probe):
    x = np.concatenate([np.linspace(-125.0, 8.0, 1_000_001), np.linspace(-1, 1, 100_001),
                        np.arange(-126, 9), [-127.5, -1000.0, -np.inf]]).astype(np.float32)
    y = _eval(probe, x)
    ok = x >= -125.0
    rel = np.abs(y[ok].astype(np.float64) / np.exp2(x[ok].astype(np.float64)) - 1.0)
    assert rel.max() <= 1.05e-4, rel.max()
    assert np.all(y[-3:] == np.float32(2.0 ** -126))
    ints = np.arange(-126, 9, dtype=np.float32)
    assert np.array_equal(_eval(probe, ints), np.exp2(ints.astype(np.float64)).astype(np.float32))
    # same steps as the host restatement: equal up to one ulp (the host emulates fma in fp64)
    h = exp2_poly_f32(x)
    ulps = np.abs(y.view(np.int32).astype(np.int64) - h.view(np.int32).astype(np.int64))
    assert ulps.max() <= 1
