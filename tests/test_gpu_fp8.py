"""GPU parity of gqa_attn_fwd_fp8: Q, K and V in e4m3 with one fp32 scale per tensor.

The oracle is the exact (fp64) attention of the values the inputs stand for, code value x
scale.  The kernel multiplies e4m3 operands exactly and accumulates in fp32, as the bf16
path does; the one new rounding is P, which goes to e4m3 (to nearest even) before P V,
while the row sum keeps the unrounded P.  The tolerance is derived from that rounding
rather than fitted:

* e4m3 keeps 3 fraction bits, so rounding a normal p moves it by at most 2^-4 p, and a
  subnormal one (below 2^-6, steps of 2^-9) by at most 2^-10.  With w_j the exact softmax
  weights and l the kernel's row sum, O - O* = sum_j (p^_j - p_j) v_j / l, so per element

      |O - O*| <= 2^-4 sum_j w_j |v_j|  +  2^-10 sum_j |v_j| / l.

  The kernel keeps its reference max m at most one octave above the row's largest score
  x_max (log2 units).  With l = 2^(X - m), X = log2 sum_j 2^(x_j), and w_max = 2^(x_max - X),
  that gives 1 / l <= 2 w_max, so the second term is at most 2^-9 w_max sum_j |v_j| (split
  partials bound the same way, each with its own m).  The first term is the oracle itself
  run on |V|.

* A mean-size check: the relative roundings are spread over [-2^-4, 2^-4], so the error of
  an element has standard deviation at most sigma = 2^-4 / sqrt(3) * sqrt(sum_j w_j^2 v_j^2).
  sum_j w_j^2 v_j^2 is the oracle on V^2 at twice the scale, times exp(L(2 scale) - 2 L).
  The root mean square of (O - O*) / sigma over all elements must stay below 1.25.

* fp32 arithmetic (score sums, the exp2 polynomial's 1.05e-4 relative error, the P V sums)
  adds at most 3e-4 of sum_j w_j |v_j| plus 1e-6; LSE is unaffected by P's rounding and
  keeps the bf16 path's bound (1e-3).  Scheduling variants stay within 1e-3 of the
  unpacked, unsplit result.
"""
import math

import numpy as np
import pytest

from tests import parity as P

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")

import inputs as _inputs

TID_Q, TID_K, TID_V = _inputs.TID_Q, _inputs.TID_K, _inputs.TID_V


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import gqa_exact_attention_b200 as G
    G.load()
    yield
    assert G.gqa_attn_device_status(reset=True) == 0, "an in-kernel wait timed out"


def fp8_case(seed, B, Sq, Sk, Hq, Hk, d, scales, shift=(0.0, 0.0)):
    """e4m3 codes for q, k, v (host), their fp64 values, and the CUDA uint8 tensors.

    Without a shift the codes are the generator's e4m3(z / scale).  With shift=(a, b) every
    q element is z + a and every k element z + b before encoding (a common offset that makes
    all logits large and of one sign: the reference max has to move)."""
    import inputs
    qs, ks, vs = scales
    shp_q, shp_k = (B, Sq, Hq, d), (B, Sk, Hk, d)
    if shift == (0.0, 0.0):
        qb = inputs.e4m3_bits_tensor(seed, TID_Q, shp_q, qs)
        kb = inputs.e4m3_bits_tensor(seed, TID_K, shp_k, ks)
    else:
        zq = inputs.bf16_bits_to_f64(inputs.bits_tensor(seed, TID_Q, shp_q)) + shift[0]
        zk = inputs.bf16_bits_to_f64(inputs.bits_tensor(seed, TID_K, shp_k)) + shift[1]
        qb = inputs.e4m3_encode(zq / qs)
        kb = inputs.e4m3_encode(zk / ks)
    vb = inputs.e4m3_bits_tensor(seed, TID_V, shp_k, vs)
    f = inputs.e4m3_bits_to_f64
    vals = (f(qb, qs), f(kb, ks), f(vb, vs))
    dev = tuple(torch.from_numpy(np.ascontiguousarray(x)).cuda() for x in (qb, kb, vb))
    return vals, dev


def oracle_terms(vals, lens, scale, causal):
    """Per sequence: the exact output and LSE, the first-term bound sum w|v|, the second
    term's w_max * sum|v|, and sigma^2's sum w^2 v^2."""
    import oracle
    q, k, v = vals
    B, Sq, Hq, d = q.shape
    Hk = k.shape[2]
    g = Hq // Hk
    outs, lses, absw, tail, w2v2 = [], [], [], [], []
    for b, L in enumerate(lens):
        qb, kb, vb = q[b:b + 1], k[b:b + 1, :L], v[b:b + 1, :L]
        o, lse = oracle.attn_fwd(qb, kb, vb, scale, causal)
        a, _ = oracle.attn_fwd(qb, kb, np.abs(vb), scale, causal)
        o2, lse2 = oracle.attn_fwd(qb, kb, vb * vb, 2 * scale, causal)
        outs.append(o)
        lses.append(lse)
        absw.append(a)
        fin = np.isfinite(lse)
        expo = np.where(fin, lse2, 0.0) - 2 * np.where(fin, lse, 0.0)
        factor = np.where(fin, np.exp(expo), 0.0)  # [1, Hq, Sq]
        w2v2.append(o2 * factor.transpose(0, 2, 1)[..., None])
        # w_max and sum |v| over each row's allowed keys (bounds only; the mask is the
        # bottom-right-aligned causal one the entry point defines)
        t = np.zeros((1, Sq, Hq, d))
        for h in range(Hq):
            kh, vh = kb[0, :, h // g], vb[0, :, h // g]
            sc = (qb[0, :, h] @ kh.T) * scale  # [Sq, L]
            for i in range(Sq):
                hi = L if not causal else min(L, i + 1 + L - Sq)
                if hi <= 0:
                    continue
                wmax = math.exp(sc[i, :hi].max() - lse[0, h, i])
                t[0, i, h] = wmax * np.abs(vh[:hi]).sum(axis=0)
        tail.append(t)
    cat = np.concatenate
    return cat(outs), cat(lses), cat(absw), cat(tail), cat(w2v2)


def check_fp8(out, lse, terms, what, rms_max=1.25):
    o_ref, l_ref, absw, tail, w2v2 = terms
    out = out.double().cpu().numpy()
    lse = lse.double().cpu().numpy()
    assert np.all(np.isfinite(out)), f"{what}: non-finite output"
    inf_ref = np.isneginf(l_ref)
    assert np.array_equal(inf_ref, np.isneginf(lse)), f"{what}: -inf LSE rows differ"
    assert not out[np.broadcast_to(inf_ref.transpose(0, 2, 1)[..., None], out.shape)].any()
    lerr = np.abs(np.where(inf_ref, 0.0, lse - np.where(inf_ref, 0.0, l_ref)))
    assert lerr.max() <= P.LSE_MAX, f"{what}: LSE err {lerr.max()}"
    err = np.abs(out - o_ref)
    bound = 2.0 ** -4 * absw + 2.0 ** -9 * tail + 3e-4 * absw + 1e-6
    worst = float((err / bound).max())
    assert worst <= 1.0, f"{what}: element error {err.max()} over its bound ({worst:.3f} of it)"
    sigma = np.sqrt((2.0 ** -4 / math.sqrt(3)) ** 2 * w2v2 + (1e-5 * absw + 1e-6) ** 2)
    rms = float(np.sqrt(np.mean((err / sigma) ** 2)))
    assert rms <= rms_max, f"{what}: rms(err / sigma) = {rms:.3f}"
    print(f"fp8 {what}: max_err {err.max():.3e} worst/bound {worst:.3f} rms_z {rms:.3f} "
          f"lse_err {lerr.max():.2e}")
    return dict(max_err=float(err.max()), worst_frac=worst, rms_z=rms)


def run_fp8(dev, scales, lens, causal, pack=-1, splits=0, bf16=False):
    import gqa_exact_attention_b200 as G
    q, k, v = dev
    sl = None if lens is None else torch.tensor(lens, dtype=torch.int32, device="cuda")
    out, lse = G.gqa_attn_fwd_fp8(q, k, v, *scales, cache_seqlens=sl, causal=causal,
                                  pack_gqa=pack, num_splits=splits,
                                  out_dtype=torch.bfloat16 if bf16 else torch.float32)
    torch.cuda.synchronize()
    return out, lse


SCALES = (0.0371, 0.0813, 0.83)  # not powers of two


@pytest.mark.parametrize("causal", [0, 1])
def test_tiny_shape_all_variants(causal):
    """B=1, Hq=6, Hk=2, Sq=Sk=128, d=64: pack_gqa on/off x num_splits 1 and 2."""
    B, Sq, Sk, Hq, Hk, d = 1, 128, 128, 6, 2, 64
    vals, dev = fp8_case(8100 + causal, B, Sq, Sk, Hq, Hk, d, SCALES)
    scale = P.default_scale(d)
    terms = oracle_terms(vals, [Sk] * B, scale, causal)
    base, base_lse = run_fp8(dev, SCALES, None, causal, pack=0, splits=1)
    check_fp8(base, base_lse, terms, f"tiny c{causal}")
    for pack in (0, 1):
        for splits in (1, 2):
            o, l = run_fp8(dev, SCALES, None, causal, pack, splits)
            check_fp8(o, l, terms, f"tiny c{causal} p{pack} s{splits}")
            assert (o - base).abs().max().item() <= P.VARIANT_MAX
            assert (l - base_lse).abs().max().item() <= P.VARIANT_MAX
            if splits == 1 and not causal:
                # every block max sits in the window around m = 0, so P is the same in both
                # head mappings: the same bits.  (Causal rows whose first visited block holds
                # a few low scores move m, at a block that depends on the mapping; the x - m
                # rounding then differs in the last bit, within the 1e-3 above.)
                assert torch.equal(o, base) and torch.equal(l, base_lse)


CASES = [
    # (B, Sq, Sk, Hq, Hk, d), lengths (None: all Sk), causal
    ((4, 1, 2048, 32, 8, 128), None, 0),                         # decode
    ((8, 1, 1000, 32, 8, 128), [1000, 1, 0, 517, 128, 129, 999, 256], 0),  # ragged, empty
    ((4, 1, 3000, 32, 4, 64), [3000, 2048, 77, 1500], 0),        # d=64, g=8
    ((2, 300, 300, 8, 2, 128), None, 1),                         # prefill, tail tile
    ((1, 77, 1000, 32, 32, 128), None, 0),                       # Sq=77, MHA
    ((2, 130, 400, 6, 3, 64), [400, 131], 1),                    # g=3, L < Sq
    ((1, 200, 200, 4, 1, 128), None, 0),                         # MQA
]


@pytest.mark.parametrize("case", CASES, ids=[f"{c[0]}-c{c[2]}" for c in CASES])
@pytest.mark.parametrize("pack,splits", [(-1, 0), (0, 1), (1, 3)])
def test_against_oracle(case, pack, splits):
    shp, lens, causal = case
    B, Sq, Sk, Hq, Hk, d = shp
    vals, dev = fp8_case(8200 + sum(shp), *shp, SCALES)
    lens_o = [Sk] * B if lens is None else lens
    terms = oracle_terms(vals, lens_o, P.default_scale(d), causal)
    out, lse = run_fp8(dev, SCALES, lens, causal, pack, splits)
    check_fp8(out, lse, terms, f"{shp} c{causal} p{pack} s{splits}")
    ob, lb = run_fp8(dev, SCALES, lens, causal, pack, splits, bf16=True)
    assert torch.equal(ob, out.to(torch.bfloat16)) and torch.equal(lb, lse)


@pytest.mark.parametrize("shift", [(2.0, -2.0), (2.0, 2.0)], ids=["logits-low", "logits-high"])
@pytest.mark.parametrize("d", [64, 128])
def test_reference_max_moves(shift, d):
    """Every logit far below zero (about -46 in log2 units), or far above (+46): the
    reference max must move off 0, down or up, without P underflowing or overflowing
    e4m3."""
    B, Sq, Sk, Hq, Hk = 1, 130, 300, 4, 2
    scales = (1 / 32, 1 / 32, 0.5)
    vals, dev = fp8_case(8300 + d, B, Sq, Sk, Hq, Hk, d, scales, shift=shift)
    scale = 1.0 / 8.0 * (8.0 / math.sqrt(d))  # 1/sqrt(d)
    for causal in (0, 1):
        terms = oracle_terms(vals, [Sk], scale, causal)
        assert np.abs(terms[1]).min() > 15, "the logits are not shifted as intended"
        for pack, splits in ((0, 1), (1, 2)):
            out, lse = run_fp8(dev, scales, None, causal, pack, splits)
            check_fp8(out, lse, terms, f"shift {shift} d{d} c{causal} p{pack} s{splits}")


def test_single_key_rows():
    """Causal, Sq = Sk: row 0 sees one key, so O = v_0 x (its p rounded / p) — within
    2^-4 of v_0 relative — and LSE = scale q.k_0."""
    B, S, Hq, Hk, d = 1, 64, 8, 2, 128
    vals, dev = fp8_case(8400, B, S, S, Hq, Hk, d, SCALES)
    out, lse = run_fp8(dev, SCALES, None, 1)
    q, k, v = vals
    scale = P.default_scale(d)
    for h in range(Hq):
        v0 = v[0, 0, h // (Hq // Hk)]
        assert np.all(np.abs(out[0, 0, h].double().cpu().numpy() - v0) <= 2.0 ** -4 * np.abs(v0) + 1e-6)
        l0 = scale * float(q[0, 0, h] @ k[0, 0, h // (Hq // Hk)])
        assert abs(lse[0, h, 0].item() - l0) <= 1e-4 * (1 + abs(l0))


def test_scales_enter_linearly():
    """Doubling v_scale doubles O bit for bit (the factor is a power of two); swapping a
    factor of two between q_scale and k_scale changes nothing."""
    B, Sq, Sk, Hq, Hk, d = 2, 64, 500, 8, 2, 128
    vals, dev = fp8_case(8500, B, Sq, Sk, Hq, Hk, d, SCALES)
    qs, ks, vs = SCALES
    o1, l1 = run_fp8(dev, (qs, ks, vs), None, 0)
    o2, l2 = run_fp8(dev, (qs, ks, 2 * vs), None, 0)
    assert torch.equal(o2, 2 * o1) and torch.equal(l1, l2)
    o3, l3 = run_fp8(dev, (2 * qs, ks / 2, vs), None, 0)
    assert torch.equal(o3, o1) and torch.equal(l3, l1)


@pytest.mark.parametrize("shape", [(3, 1, 4097, 8, 128), (2, 5, 70, 3, 64)])
def test_device_generator_matches_host(shape):
    import inputs
    for tid, sc in ((TID_Q, 0.0371), (TID_K, 1.0), (TID_V, 0.83)):
        host = inputs.e4m3_bits_tensor(8600, tid, shape, sc)
        dev = inputs.e4m3_device_tensor(8600, tid, shape, sc)
        torch.cuda.synchronize()
        assert np.array_equal(dev.cpu().numpy(), host)


@pytest.mark.parametrize("Sk", [8192, 32768])
def test_decode_full_size_sampled(Sk):
    """Decode at the benchmark's head shape (B=32, Hq=32, Hk=8, d=128), inputs generated on
    the device; sampled rows against the oracle under the automatic schedule and every
    forced split count, which must agree within 1e-3."""
    import inputs
    import oracle
    B, Hq, Hk, d = 32, 32, 8, 128
    q = inputs.e4m3_device_tensor(8700, TID_Q, (B, 1, Hq, d), SCALES[0])
    k = inputs.e4m3_device_tensor(8700, TID_K, (B, Sk, Hk, d), SCALES[1])
    v = inputs.e4m3_device_tensor(8700, TID_V, (B, Sk, Hk, d), SCALES[2])
    dev = (q, k, v)
    out, lse = run_fp8(dev, SCALES, None, 0)
    for splits in (1, 2, 4, 8):
        o, l = run_fp8(dev, SCALES, None, 0, splits=splits)
        assert (o - out).abs().max().item() <= P.VARIANT_MAX
        assert (l - lse).abs().max().item() <= P.VARIANT_MAX
    f = inputs.e4m3_bits_to_f64
    for b in (0, 17, B - 1):
        vals = (f(q[b:b + 1].cpu().numpy(), SCALES[0]), f(k[b:b + 1].cpu().numpy(), SCALES[1]),
                f(v[b:b + 1].cpu().numpy(), SCALES[2]))
        terms = oracle_terms(vals, [Sk], P.default_scale(d), 0)
        check_fp8(out[b:b + 1], lse[b:b + 1], terms, f"decode Sk={Sk} b={b}")
    del q, k, v, dev
    torch.cuda.empty_cache()
