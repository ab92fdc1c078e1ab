"""Shared helpers of the GPU parity tests: seeded inputs for both sides, the oracle on
the same inputs, and the tolerance check.

Tolerances (bf16 inputs, fp32 accumulation): output max |err| <= 2e-2 and mean
|err| <= 2e-3, LSE max |err| <= 1e-3 against the fp64 oracle; scheduling variants
(pack_gqa, num_splits) within 1e-3 of the unpacked, unsplit GPU result.
"""
from __future__ import annotations

import math

import numpy as np

import inputs
import oracle

OUT_MAX, OUT_MEAN, LSE_MAX, VARIANT_MAX = 2e-2, 2e-3, 1e-3, 1e-3


def shapes(B, Sq, Sk, Hq, Hk, d):
    return (B, Sq, Hq, d), (B, Sk, Hk, d)


def device_inputs(seed, B, Sq, Sk, Hq, Hk, d, on_device_gen=False):
    """q, k, v as CUDA bf16 tensors, element for element the generator's values."""
    qs, ks = shapes(B, Sq, Sk, Hq, Hk, d)
    if on_device_gen:
        return (inputs.device_tensor(seed, inputs.TID_Q, qs),
                inputs.device_tensor(seed, inputs.TID_K, ks),
                inputs.device_tensor(seed, inputs.TID_V, ks))
    return (inputs.host_tensor(seed, inputs.TID_Q, qs).cuda(),
            inputs.host_tensor(seed, inputs.TID_K, ks).cuda(),
            inputs.host_tensor(seed, inputs.TID_V, ks).cuda())


def host_inputs_f64(seed, B, Sq, Sk, Hq, Hk, d):
    qs, ks = shapes(B, Sq, Sk, Hq, Hk, d)
    f = inputs.bf16_bits_to_f64
    return (f(inputs.bits_tensor(seed, inputs.TID_Q, qs)),
            f(inputs.bits_tensor(seed, inputs.TID_K, ks)),
            f(inputs.bits_tensor(seed, inputs.TID_V, ks)))


def oracle_full(seed, B, Sq, Sk, Hq, Hk, d, scale, causal):
    q, k, v = host_inputs_f64(seed, B, Sq, Sk, Hq, Hk, d)
    return oracle.attn_fwd(q, k, v, scale, causal)


def oracle_rows(seed, B, Sq, Sk, Hq, Hk, d, scale, causal, rows):
    """Oracle output for sampled rows [(b, h, i)], regenerating only the inputs they read."""
    qs, ks = shapes(B, Sq, Sk, Hq, Hk, d)
    g = Hq // Hk
    cache = {}
    outs, lses = [], []
    for (b, h, i) in rows:
        kvh = h // g
        if (b, kvh) not in cache:
            cache.clear()
            cache[(b, kvh)] = (inputs.head_rows_f64(seed, inputs.TID_K, ks, b, kvh),
                               inputs.head_rows_f64(seed, inputs.TID_V, ks, b, kvh))
        kr, vr = cache[(b, kvh)]
        qr = inputs.head_rows_f64(seed, inputs.TID_Q, qs, b, h, i, i + 1)[0]
        o, l = oracle.attn_row(qr, kr, vr, Sq, i, scale, causal)
        outs.append(o)
        lses.append(l)
    return np.array(outs), np.array(lses)


def check(out_gpu, lse_gpu, out_ref, lse_ref, what=""):
    """Element-wise comparison within the stated tolerances; -inf LSE must match exactly
    (and then the output row must be exactly 0)."""
    out_gpu = np.asarray(out_gpu, dtype=np.float64)
    lse_gpu = np.asarray(lse_gpu, dtype=np.float64)
    assert np.all(np.isfinite(out_gpu)), f"{what}: non-finite output"
    inf_ref = np.isneginf(lse_ref)
    assert np.array_equal(inf_ref, np.isneginf(lse_gpu)), f"{what}: -inf LSE rows differ"
    err = np.abs(out_gpu - out_ref)
    lerr = np.abs(np.where(inf_ref, 0.0, lse_gpu - np.where(inf_ref, 0.0, lse_ref)))
    stats = dict(out_max=float(err.max()) if err.size else 0.0,
                 out_mean=float(err.mean()) if err.size else 0.0,
                 lse_max=float(lerr.max()) if lerr.size else 0.0)
    assert stats["out_max"] <= OUT_MAX, f"{what}: {stats}"
    assert stats["out_mean"] <= OUT_MEAN, f"{what}: {stats}"
    assert stats["lse_max"] <= LSE_MAX, f"{what}: {stats}"
    return stats


def sample_rows(rng, B, Sq, Hq, Hk, n, tile=128):
    """Seeded row sample: every head of one kv group, first/last/tile-edge positions,
    plus random rows."""
    g = Hq // Hk
    rows = set()
    b0 = int(rng.integers(B))
    grp = int(rng.integers(Hk))
    special = sorted({0, 1, tile - 1, tile, Sq // 2, Sq - 2, Sq - 1} & set(range(Sq)))
    for h in range(grp * g, grp * g + g):
        for i in special:
            rows.add((b0, h, i))
    rows.add((B - 1, Hq - 1, Sq - 1))
    while len(rows) < n:
        rows.add((int(rng.integers(B)), int(rng.integers(Hq)), int(rng.integers(Sq))))
    return sorted(rows)


def default_scale(d):
    return 1.0 / math.sqrt(d)
