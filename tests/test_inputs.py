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


# ------------------------------------------------------------------ e4m3 encoder

def _e4m3_rne_exact(t: float) -> int:
    """OCP FP8 E4M3 rounding of t, to nearest even, saturating at +-448, restated with
    exact rationals: every finite code's value is enumerated and the nearest taken."""
    vals = sorted({_e4m3_value(c) for c in range(0x7F)})  # non-negative codes 0..0x7E
    a = Fraction(abs(t))
    if a >= 448:
        code = 0x7E
    else:
        best = min(vals, key=lambda v: (abs(Fraction(v) - a), _e4m3_code(v) & 1))
        code = _e4m3_code(best)
    return code | (0x80 if math.copysign(1.0, t) < 0 else 0)


def _e4m3_value(code: int) -> float:
    code = int(code)
    e, m = (code >> 3) & 15, code & 7
    return m * 2.0 ** -9 if e == 0 else (1 + m / 8) * 2.0 ** (e - 7)


def _e4m3_code(v: float) -> int:
    for c in range(0x7F):
        if _e4m3_value(c) == v:
            return c
    raise ValueError(v)


def test_e4m3_codes_round_trip_and_decode():
    # every finite code decodes to its format value and encodes back to itself
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], dtype=np.uint8)
    vals = inputs.e4m3_bits_to_f64(codes)
    expect = np.array([(-1.0 if c & 0x80 else 1.0) * _e4m3_value(c & 0x7F) for c in codes])
    assert np.array_equal(vals, expect)
    back = inputs.e4m3_encode(vals)
    zero_neg = codes == 0x80  # -0.0 encodes to 0x80, decodes to -0.0
    assert np.array_equal(back[~zero_neg], codes[~zero_neg])
    assert vals.max() == 448.0 and vals.min() == -448.0


def test_e4m3_encoder_matches_exact_rounding():
    rng = np.random.default_rng(5)
    pts = list(rng.standard_normal(400) * 40) + list(rng.standard_normal(200) * 2.0 ** -7)
    # midpoints between neighbouring codes (ties go to the even code), and the saturation edge
    vals = sorted({_e4m3_value(c) for c in range(0x7F)})
    pts += [(a + b) / 2 for a, b in zip(vals[:-1], vals[1:])]
    pts += [447.9, 448.0, 463.9, 464.0, 1e6, -1e6, 2.0 ** -10, 3 * 2.0 ** -11, 0.0]
    got = inputs.e4m3_encode(pts)
    want = np.array([_e4m3_rne_exact(float(t)) for t in pts], dtype=np.uint8)
    assert np.array_equal(got, want)


def test_e4m3_generator_definition():
    seed, tid, scale = 321, 2, 1.0 / 64
    bits = inputs.e4m3_bits_tensor(seed, tid, (50,), scale)
    z = inputs.bf16_bits_to_f64(inputs.bits_range(seed, tid, 0, 50))  # same z, rounded to bf16
    # the e4m3 element is z / scale rounded: within e4m3's relative step of z
    vals = inputs.e4m3_bits_to_f64(bits, scale)
    assert np.all(np.abs(vals - z) <= np.abs(z) * 2.0 ** -3 + 2.0 ** -9 * scale + 2.0 ** -8 * np.abs(z))
