"""Pins for the fp64 oracle: checks against what the pages and the mathematics fix.

Each ``pin_*`` takes an :class:`oracle.Oracle` and raises ``AssertionError`` when the
oracle disagrees with something that does not come from the oracle itself: the
pages' worked head-mapping example, closed forms, invariants, a library softmax,
and brute force at high precision on tiny inputs.  ``tests/test_oracle_pins.py``
runs them on the real oracle and on deliberately broken copies of it.
"""
from __future__ import annotations

import decimal
import json
import math
import os

import numpy as np
from scipy.special import logsumexp, softmax

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _rng(seed):
    return np.random.default_rng(seed)


def _bf16ish(rng, shape):
    """Random values on the bf16 grid (what the oracle sees from the generator)."""
    x = rng.standard_normal(shape).astype(np.float32)
    bits = (x.view(np.uint32) + 0x8000) & 0xFFFF0000
    return bits.view(np.float32).astype(np.float64)


def _library_attn(q, k, v, scale, causal):
    """Textbook attention from numpy matmul + scipy softmax/logsumexp, one head pair
    at a time, with the kv head for q-head h given by ``h // (Hq // Hk)``."""
    B, Sq, Hq, d = q.shape
    _, Sk, Hk, _ = k.shape
    g = Hq // Hk
    out = np.zeros((B, Sq, Hq, d))
    lse = np.full((B, Hq, Sq), -np.inf)
    i = np.arange(Sq)[:, None]
    j = np.arange(Sk)[None, :]
    allowed = (j <= i + (Sk - Sq)) if causal else np.ones((Sq, Sk), bool)
    for b in range(B):
        for h in range(Hq):
            s = scale * (q[b, :, h, :] @ k[b, :, h // g, :].T)
            s = np.where(allowed, s, -np.inf)
            rows = allowed.any(axis=1)
            p = np.zeros_like(s)
            p[rows] = softmax(s[rows], axis=1)
            out[b, :, h, :] = p @ v[b, :, h // g, :]
            lse[b, h, rows] = logsumexp(s[rows], axis=1)
    return out, lse


# --------------------------------------------------------------------------- pins

def pin_head_mapping_page_example(O):
    """The pages' own example: Hq=6, Hk=2, q-heads 0,1,2 -> kv 0 and 3,4,5 -> kv 1.
    With V constant per kv-head (powers of two, so the average is exact) each
    q-head's output equals its kv-head's constant."""
    with open(os.path.join(GOLDEN, "head_mapping_hq6_hk2.json")) as f:
        gold = json.load(f)
    Hq, Hk, m = gold["Hq"], gold["Hk"], gold["kv_head_of_q_head"]
    rng = _rng(1)
    B, S, d = 2, 9, 8
    q = _bf16ish(rng, (B, S, Hq, d))
    k = _bf16ish(rng, (B, S, Hk, d))
    consts = [1.0, -2.0]
    v = np.zeros((B, S, Hk, d))
    for kvh in range(Hk):
        v[:, :, kvh, :] = consts[kvh]
    for causal in (False, True):
        out, _ = O.attn_fwd(q, k, v, 0.35, causal)
        for h in range(Hq):
            assert np.all(out[:, :, h, :] == consts[m[h]]), f"q-head {h} must read kv-head {m[h]}"


def pin_mha_and_gqa_match_library_softmax(O):
    """Against numpy matmul + scipy softmax/logsumexp, for the MHA, GQA and MQA cases
    of the pages' comparison tables, causal and not, Sq != Sk."""
    with open(os.path.join(GOLDEN, "attention_variants.json")) as f:
        cases = json.load(f)["cases"]
    rng = _rng(2)
    for c in cases:
        Hq, Hk = c["Hq"], c["Hk"]
        for (Sq, Sk, causal) in ((7, 7, True), (5, 11, True), (6, 6, False), (3, 13, False)):
            d = 16
            q = _bf16ish(rng, (1, Sq, Hq, d))
            k = _bf16ish(rng, (1, Sk, Hk, d))
            v = _bf16ish(rng, (1, Sk, Hk, d))
            scale = 1.0 / math.sqrt(d)
            o1, l1 = O.attn_fwd(q, k, v, scale, causal)
            o2, l2 = _library_attn(q, k, v, scale, causal)
            np.testing.assert_allclose(o1, o2, rtol=0, atol=1e-12)
            np.testing.assert_allclose(l1, l2, rtol=0, atol=1e-12)


def pin_gqa_equals_replicated_mha(O):
    """GQA = MHA with each kv head replicated Hq/Hk times (adjacent q-heads share it)."""
    rng = _rng(3)
    B, Sq, Sk, Hq, Hk, d = 2, 6, 10, 6, 2, 8
    q = _bf16ish(rng, (B, Sq, Hq, d))
    k = _bf16ish(rng, (B, Sk, Hk, d))
    v = _bf16ish(rng, (B, Sk, Hk, d))
    g = Hq // Hk
    kr, vr = np.repeat(k, g, axis=2), np.repeat(v, g, axis=2)
    for causal in (False, True):
        o1, l1 = O.attn_fwd(q, k, v, 0.3, causal)
        o2, l2 = O.attn_fwd(q, kr, vr, 0.3, causal)
        assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


def pin_rows_are_probability_vectors(O):
    """With V = identity rows (value j = unit vector e_j) the output row is the
    softmax row itself: non-negative, summing to 1, masked keys exactly 0."""
    rng = _rng(4)
    Sq, Sk, d = 5, 8, 8
    q = _bf16ish(rng, (1, Sq, 1, d))
    k = _bf16ish(rng, (1, Sk, 1, d))
    v = np.eye(Sk).reshape(1, Sk, 1, d)
    for causal in (False, True):
        out, _ = O.attn_fwd(q, k, v, 0.7, causal)
        P = out[0, :, 0, :]
        assert np.all(P >= 0)
        np.testing.assert_allclose(P.sum(axis=1), 1.0, rtol=0, atol=1e-14)
        if causal:
            for i in range(Sq):
                assert np.all(P[i, i + (Sk - Sq) + 1:] == 0)


def pin_constant_v(O):
    """V = c everywhere gives O = c."""
    rng = _rng(5)
    q = _bf16ish(rng, (1, 7, 4, 16))
    k = _bf16ish(rng, (1, 9, 2, 16))
    v = np.full((1, 9, 2, 16), 0.3)
    for causal in (False, True):
        out, _ = O.attn_fwd(q, k, v, 0.25, causal)
        np.testing.assert_allclose(out, 0.3, rtol=1e-15, atol=0)


def pin_single_key_row(O):
    """Causal, Sq = Sk: row 0 sees only key 0, so O = v_0 and LSE = scale q_0.k_0."""
    rng = _rng(6)
    S, d = 6, 16
    q = _bf16ish(rng, (1, S, 2, d))
    k = _bf16ish(rng, (1, S, 1, d))
    v = _bf16ish(rng, (1, S, 1, d))
    out, lse = O.attn_fwd(q, k, v, 0.2, True)
    for h in range(2):
        assert np.array_equal(out[0, 0, h, :], v[0, 0, 0, :])
        assert math.isclose(lse[0, h, 0], 0.2 * float(np.dot(q[0, 0, h], k[0, 0, 0])),
                            rel_tol=0, abs_tol=1e-14)


def pin_zero_scale_counts_keys(O):
    """scale = 0 makes every allowed key weigh the same: O = mean of V over the allowed
    set and LSE = ln |allowed|.  |allowed| for row i, causal, is i + 1 + (Sk - Sq)
    clamped to [0, Sk] (bottom-right alignment); an empty row gives O = 0, LSE = -inf."""
    rng = _rng(7)
    d = 4
    for (Sq, Sk) in ((6, 6), (4, 9), (9, 4)):
        q = _bf16ish(rng, (1, Sq, 1, d))
        k = _bf16ish(rng, (1, Sk, 1, d))
        v = _bf16ish(rng, (1, Sk, 1, d))
        for causal in (False, True):
            out, lse = O.attn_fwd(q, k, v, 0.0, causal)
            for i in range(Sq):
                n = min(Sk, max(0, i + 1 + Sk - Sq)) if causal else Sk
                if n == 0:
                    assert lse[0, 0, i] == -np.inf and np.all(out[0, i, 0] == 0)
                    continue
                assert math.isclose(lse[0, 0, i], math.log(n), rel_tol=0, abs_tol=1e-14)
                np.testing.assert_allclose(out[0, i, 0], v[0, :n, 0].mean(axis=0),
                                           rtol=0, atol=1e-14)


def pin_identical_keys(O):
    """All keys equal to one vector kk: weights are uniform, O = mean V and
    LSE = scale q.kk + ln Sk."""
    rng = _rng(8)
    Sq, Sk, d = 3, 7, 8
    q = _bf16ish(rng, (1, Sq, 1, d))
    kk = _bf16ish(rng, (d,))
    k = np.broadcast_to(kk, (1, Sk, 1, d)).copy()
    v = _bf16ish(rng, (1, Sk, 1, d))
    out, lse = O.attn_fwd(q, k, v, 0.9, False)
    for i in range(Sq):
        np.testing.assert_allclose(out[0, i, 0], v[0, :, 0].mean(axis=0), rtol=0, atol=1e-14)
        assert math.isclose(lse[0, 0, i], 0.9 * float(q[0, i, 0] @ kk) + math.log(Sk),
                            rel_tol=0, abs_tol=1e-13)


def pin_bruteforce_decimal(O):
    """Tiny shapes against a 40-digit decimal evaluation of the unshifted definition
    w_j = exp(s_j) / sum_k exp(s_k) (no max subtraction), LSE = ln sum exp(s_j)."""
    decimal.getcontext().prec = 40
    D = decimal.Decimal
    rng = _rng(9)
    B, Sq, Sk, Hq, Hk, d = 1, 3, 5, 4, 2, 4
    q = _bf16ish(rng, (B, Sq, Hq, d))
    k = _bf16ish(rng, (B, Sk, Hk, d))
    v = _bf16ish(rng, (B, Sk, Hk, d))
    scale = 0.6
    for causal in (False, True):
        out, lse = O.attn_fwd(q, k, v, scale, causal)
        for h in range(Hq):
            kvh = h // (Hq // Hk)
            for i in range(Sq):
                keys = [j for j in range(Sk) if not causal or j <= i + Sk - Sq]
                e = {}
                for j in keys:
                    s = D(scale) * sum(D(float(q[0, i, h, c])) * D(float(k[0, j, kvh, c]))
                                       for c in range(d))
                    e[j] = s.exp()
                z = sum(e.values())
                for c in range(d):
                    ref = sum(e[j] * D(float(v[0, j, kvh, c])) for j in keys) / z
                    assert abs(out[0, i, h, c] - float(ref)) <= 1e-13
                assert abs(lse[0, h, i] - float(z.ln())) <= 1e-13


def pin_split_combine_identity(O):
    """Partials over disjoint key ranges, merged by the combine, give the full result;
    a range with no allowed key has LSE = -inf and weight 0."""
    rng = _rng(10)
    B, Sq, Sk, Hq, Hk, d = 1, 6, 13, 4, 2, 8
    q = _bf16ish(rng, (B, Sq, Hq, d))
    k = _bf16ish(rng, (B, Sk, Hk, d))
    v = _bf16ish(rng, (B, Sk, Hk, d))
    for causal in (False, True):
        full_o, full_l = O.attn_fwd(q, k, v, 0.4, causal)
        bounds = [0, 3, 8, 13]
        parts = [O.attn_fwd(q, k, v, 0.4, causal, lo, hi) for lo, hi in zip(bounds, bounds[1:])]
        # rows ordered (b, h, i) as in the LSE layout
        o_parts = np.stack([p[0].transpose(0, 2, 1, 3).reshape(-1, d) for p in parts])
        l_parts = np.stack([p[1].reshape(-1) for p in parts])
        if causal:
            assert np.any(np.isneginf(l_parts)), "a late range must be empty for early rows"
        o, l = O.combine(o_parts, l_parts)
        np.testing.assert_allclose(o, full_o.transpose(0, 2, 1, 3).reshape(-1, d), rtol=0,
                                   atol=1e-13)
        np.testing.assert_allclose(l, full_l.reshape(-1), rtol=0, atol=1e-13)


def pin_combine_closed_forms(O):
    """Two partials with equal LSE average their outputs and add ln 2; partials that
    are all empty give O = 0 and LSE = -inf; one empty partial drops out."""
    a = np.array([[1.0, 2.0]])
    b = np.array([[3.0, -2.0]])
    o, l = O.combine(np.stack([a, b]), np.array([[0.5], [0.5]]))
    np.testing.assert_allclose(o, [[2.0, 0.0]], atol=1e-15)
    assert math.isclose(l[0], 0.5 + math.log(2.0), abs_tol=1e-15)
    o, l = O.combine(np.stack([a, b]), np.array([[-np.inf], [-np.inf]]))
    assert np.all(o == 0) and l[0] == -np.inf
    o, l = O.combine(np.stack([a, b]), np.array([[-np.inf], [1.25]]))
    np.testing.assert_allclose(o, b, atol=0)
    assert l[0] == 1.25
    # unequal weights: w = (e^0, e^ln3) -> (1/4, 3/4)
    o, l = O.combine(np.stack([a, b]), np.array([[0.0], [math.log(3.0)]]))
    np.testing.assert_allclose(o, 0.25 * a + 0.75 * b, atol=1e-15)
    assert math.isclose(l[0], math.log(4.0), abs_tol=1e-15)


def pin_negative_scale(O):
    """The scale may be any real; a negative one reverses the ranking of keys."""
    rng = _rng(11)
    q = _bf16ish(rng, (1, 4, 2, 8))
    k = _bf16ish(rng, (1, 6, 1, 8))
    v = _bf16ish(rng, (1, 6, 1, 8))
    o1, l1 = O.attn_fwd(q, k, v, -0.8, True)
    o2, l2 = _library_attn(q, k, v, -0.8, True)
    np.testing.assert_allclose(o1, o2, atol=1e-12)
    np.testing.assert_allclose(l1, l2, atol=1e-12)


def pin_row_entry_matches_full(O):
    """The per-row entry point (used for sampled rows at full sizes) agrees exactly with
    the whole-tensor entry point, for a kv-head picked by the mapping h // g."""
    rng = _rng(12)
    B, Sq, Sk, Hq, Hk, d = 2, 5, 9, 6, 3, 8
    q = _bf16ish(rng, (B, Sq, Hq, d))
    k = _bf16ish(rng, (B, Sk, Hk, d))
    v = _bf16ish(rng, (B, Sk, Hk, d))
    out, lse = O.attn_fwd(q, k, v, 0.5, True)
    for b in range(B):
        for h in range(Hq):
            for i in range(Sq):
                o, l = O.attn_row(q[b, i, h], k[b, :, h // 2], v[b, :, h // 2], Sq, i, 0.5, True)
                assert np.array_equal(o, out[b, i, h]) and l == lse[b, h, i]


PINS = [
    pin_head_mapping_page_example,
    pin_mha_and_gqa_match_library_softmax,
    pin_gqa_equals_replicated_mha,
    pin_rows_are_probability_vectors,
    pin_constant_v,
    pin_single_key_row,
    pin_zero_scale_counts_keys,
    pin_identical_keys,
    pin_bruteforce_decimal,
    pin_split_combine_identity,
    pin_combine_closed_forms,
    pin_negative_scale,
    pin_row_entry_matches_full,
]
