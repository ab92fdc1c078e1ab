"""The seeded input generator (shared by both sides of every parity check)."""
import math
from fractions import Fraction

import numpy as np
from scipy import stats

import inputs

G = 0x9E3779B97F4A7C15
M64 = (1 << 64) - 1


def _mix(z):
    z ^= z >> 30
    z = (z * 0xbf58476d1ce4e5b9) & M64
    z ^= z >> 27
    z = (z * 0x94d049bb133111eb) & M64
    z ^= z >> 31
    return z


def _bf16_rne_exact(z: float) -> int:
    """Round-to-nearest-even of z to 8 significant bits, done in exact rationals."""
    if z == 0.0:
        return 0x8000 if math.copysign(1.0, z) < 0 else 0
    fz = Fraction(z)
    e = math.floor(math.log2(abs(z)))
    while Fraction(2) ** e > abs(fz):
        e -= 1
    while Fraction(2) ** (e + 1) <= abs(fz):
        e += 1
    scaled = fz / Fraction(2) ** (e - 7)
    r = round(scaled)  # Python rounds half to even
    y = float(r * Fraction(2) ** (e - 7))
    return int(np.array([y], dtype=np.float32).view(np.uint32)[0] >> 16)


def test_definition_matches_python_restatement():
    seed, tid = 1234, 2
    bits = inputs.bits_range(seed, tid, 0, 2000)
    base = _mix((seed * G + tid) & M64)
    for i in range(2000):
        r = _mix((base + (i + 1) * G) & M64)
        u1 = ((r >> 40) + 1) * 2.0 ** -24
        u2 = ((r >> 16) & 0xFFFFFF) * 2.0 ** -24
        z = math.sqrt(-2.0 * math.log(u1)) * math.cos(6.283185307179586 * u2)
        assert bits[i] == _bf16_rne_exact(z), i


def test_counter_based_slices_agree():
    full = inputs.bits_range(7, 3, 0, 10000)
    assert np.array_equal(inputs.bits_range(7, 3, 1234, 500), full[1234:1734])
    st = inputs.bits_strided(7, 3, 100, 8, 20, 64)
    for o in range(20):
        assert np.array_equal(st[o], full[100 + 64 * o: 108 + 64 * o])
    assert not np.array_equal(inputs.bits_range(8, 3, 0, 100), full[:100])
    assert not np.array_equal(inputs.bits_range(7, 2, 0, 100), full[:100])


def test_standard_normal():
    x = inputs.bf16_bits_to_f64(inputs.bits_range(1001, 1, 0, 1 << 20))
    assert abs(x.mean()) < 5e-3 and abs(x.std() - 1.0) < 5e-3
    assert stats.kstest(x, "norm").pvalue > 1e-4


def test_head_rows_slice():
    shape = (2, 5, 3, 4)
    full = inputs.bf16_bits_to_f64(inputs.bits_tensor(11, 2, shape))
    rows = inputs.head_rows_f64(11, 2, shape, 1, 2, 1, 4)
    assert np.array_equal(rows, full[1, 1:4, 2, :])
