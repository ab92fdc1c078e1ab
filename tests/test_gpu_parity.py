"""GPU parity: the CUDA path through the C ABI against the fp64 oracle on the same
seeded inputs, element by element, within the stated tolerances."""
import numpy as np
import pytest

from tests import parity as P

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import gqa_exact_attention_b200 as G
    G.load()
    yield
    assert G.gqa_attn_device_status(reset=True) == 0, "an in-kernel wait timed out"


def run(q, k, v, causal, pack=-1, splits=0, scale=None):
    import gqa_exact_attention_b200 as G
    out, lse = G.gqa_attn_fwd(q, k, v, scale=scale, causal=causal, pack_gqa=pack,
                              num_splits=splits)
    torch.cuda.synchronize()
    return out, lse


# --- the tiny configuration: B=1, Hq=6, Hk=2, Sq=Sk=128, d=64, all 8 variants
@pytest.mark.parametrize("causal", [0, 1])
@pytest.mark.parametrize("pack", [0, 1])
@pytest.mark.parametrize("splits", [1, 2])
def test_tiny_all_variants(causal, pack, splits):
    seed, shp = 1000, (1, 128, 128, 6, 2, 64)
    q, k, v = P.device_inputs(seed, *shp)
    o_ref, l_ref = P.oracle_full(seed, *shp, P.default_scale(64), causal)
    out, lse = run(q, k, v, causal, pack, splits)
    P.check(out.cpu().numpy(), lse.cpu().numpy(), o_ref, l_ref, f"tiny c{causal} p{pack} s{splits}")
    base, lbase = run(q, k, v, causal, 0, 1)
    assert (out - base).abs().max().item() <= P.VARIANT_MAX
    assert (lse - lbase).abs().max().item() <= P.VARIANT_MAX


# --- ragged shapes: tails in Sq and Sk, several tiles, head ratios from MHA to MQA
RAGGED = [
    # B, Sq, Sk, Hq, Hk, d
    (2, 77, 300, 8, 2, 128),
    (1, 300, 300, 4, 4, 128),
    (2, 130, 257, 8, 1, 64),
    (1, 1, 700, 32, 8, 128),
    (3, 5, 129, 6, 3, 64),
    (1, 384, 200, 4, 2, 128),
    (1, 200, 384, 8, 4, 64),
]


@pytest.mark.parametrize("shp", RAGGED, ids=[str(s) for s in RAGGED])
@pytest.mark.parametrize("causal", [0, 1])
@pytest.mark.parametrize("pack,splits", [(0, 1), (1, 1), (0, 3), (1, 2), (-1, 0)])
def test_ragged(shp, causal, pack, splits):
    seed = 2000 + sum(shp)
    q, k, v = P.device_inputs(seed, *shp)
    o_ref, l_ref = P.oracle_full(seed, *shp, P.default_scale(shp[-1]), causal)
    out, lse = run(q, k, v, causal, pack, splits)
    P.check(out.cpu().numpy(), lse.cpu().numpy(), o_ref, l_ref, f"{shp} c{causal} p{pack} s{splits}")


# --- causal with Sq > Sk: leading rows see no key (O = 0, LSE = -inf)
@pytest.mark.parametrize("pack,splits", [(0, 1), (1, 1), (0, 2), (1, 3)])
def test_empty_rows(pack, splits):
    shp = (2, 260, 70, 4, 2, 64)
    seed = 3000
    q, k, v = P.device_inputs(seed, *shp)
    o_ref, l_ref = P.oracle_full(seed, *shp, P.default_scale(64), 1)
    assert np.isneginf(l_ref).any()
    out, lse = run(q, k, v, 1, pack, splits)
    P.check(out.cpu().numpy(), lse.cpu().numpy(), o_ref, l_ref, "empty rows")
    empty = torch.from_numpy(np.isneginf(l_ref)).cuda()
    assert torch.all(out.permute(0, 2, 1, 3)[empty] == 0)


# --- closed forms on the GPU: scale 0 gives the mean of V over the allowed keys;
#     causal row 0 with Sq == Sk sees one key: O = v_0 and LSE = scale q_0 . k_0.  The
#     kernel keeps its reference max integral (so that every schedule rounds P alike), so
#     the single weight is p = 2^(x - ceil(x)) in (1/2, 1]; the MMA takes p rounded to bf16
#     while l keeps p, so O = v_0 * bf16(p) / p: within a relative 2^-8 of v_0 (the
#     round-to-nearest bound of bf16's 8-bit significand), plus fp32 rounding.
def test_scale_zero_and_single_key():
    shp = (1, 200, 200, 4, 2, 128)
    seed = 3100
    q, k, v = P.device_inputs(seed, *shp)
    out, lse = run(q, k, v, 1, 0, 1, scale=0.0)
    vf = v.float()
    csum = torch.cumsum(vf, dim=1) / torch.arange(1, 201, device="cuda").view(1, -1, 1, 1)
    ref = csum.repeat_interleave(2, dim=2)
    assert (out - ref).abs().max().item() <= 1e-4
    ln = torch.log(torch.arange(1, 201, device="cuda", dtype=torch.float32))
    assert (lse - ln.view(1, 1, -1)).abs().max().item() <= 1e-5
    out, lse = run(q, k, v, 1, 0, 1)
    for h, kvh in ((0, 0), (3, 1)):
        v0 = vf[0, 0, kvh]
        assert ((out[0, 0, h] - v0).abs() <= 2.0 ** -8 * 1.0001 * v0.abs() + 1e-30).all()
        s0 = (q[0, 0, h].double() * k[0, 0, kvh].double()).sum().item() / 128 ** 0.5
        assert abs(lse[0, h, 0].item() - s0) <= 1e-5 * max(1.0, abs(s0))


# --- odd shapes / head ratios: Sq=77 vs Sk=4096 non-causal, d in {64,128},
#     (Hq,Hk) in {(32,32),(32,8),(32,4),(32,1)}, full oracle
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("hk", [32, 8, 4, 1])
def test_odd_sq77_sk4096(d, hk):
    shp = (4, 77, 4096, 32, hk, d)
    seed = 1004
    q, k, v = P.device_inputs(seed, *shp)
    o_ref, l_ref = P.oracle_full(seed, *shp, P.default_scale(d), 0)
    out, lse = run(q, k, v, 0)
    P.check(out.cpu().numpy(), lse.cpu().numpy(), o_ref, l_ref, f"Sq77 d{d} hk{hk}")


# --- many units per persistent CTA with causal split-KV: units whose tiles have zero or
#     one key block let a softmax warpgroup run ahead of the epilogue; full oracle
@pytest.mark.parametrize("shp,splits", [((8, 2048, 2048, 4, 2, 128), 3),
                                         ((16, 1024, 1024, 4, 2, 128), 3),
                                         ((8, 2048, 2048, 4, 2, 64), 4)])
def test_many_units_causal_splits(shp, splits):
    seed = 3300 + splits
    q, k, v = P.device_inputs(seed, *shp)
    o_ref, l_ref = P.oracle_full(seed, *shp, P.default_scale(shp[-1]), 1)
    out, lse = run(q, k, v, 1, 0, splits)
    P.check(out.cpu().numpy(), lse.cpu().numpy(), o_ref, l_ref, f"{shp} s{splits}")


# --- scales other than 1/sqrt(d): a negative scale (the extremum becomes a row minimum) and
#     a large one (exponents far below -126, the polynomial's clamp), causal and not
@pytest.mark.parametrize("scale", [-0.09, 1.5])
@pytest.mark.parametrize("causal", [0, 1])
@pytest.mark.parametrize("pack,splits", [(0, 1), (1, 2), (-1, 0)])
def test_other_scales(scale, causal, pack, splits):
    shp = (2, 300, 300, 8, 2, 128)
    seed = 3400
    q, k, v = P.device_inputs(seed, *shp)
    o_ref, l_ref = P.oracle_full(seed, *shp, scale, causal)
    out, lse = run(q, k, v, causal, pack, splits, scale=scale)
    P.check(out.cpu().numpy(), lse.cpu().numpy(), o_ref, l_ref, f"scale {scale} c{causal} p{pack} s{splits}")


# --- short query axes (decode, a few positions): tiles with at most 32 real rows, every
# pack/split schedule against the oracle and against nine splits.
SHORT_Q = [
    # B, Sq, Sk, Hq, Hk, d           real rows per tile (packed)
    (4, 1, 3000, 32, 8, 128),        # g=4: 4
    (2, 8, 1200, 32, 8, 128),        # 4 x 8 = 32, causal rows end at different keys
    (2, 3, 1200, 30, 3, 64),         # g=10: 30, a quarter box of 3 positions
    (1, 20, 1300, 4, 4, 64),         # MHA: 20 positions
    (3, 1, 1153, 32, 1, 128),        # MQA g=32: 32; one key past the last full block
]


@pytest.mark.parametrize("shp", SHORT_Q, ids=[str(s) for s in SHORT_Q])
@pytest.mark.parametrize("causal", [0, 1])
def test_short_query_axis_schedules(shp, causal):
    seed = 3500 + sum(shp)
    q, k, v = P.device_inputs(seed, *shp)
    d = shp[5]
    o_ref, l_ref = P.oracle_full(seed, *shp, P.default_scale(d), causal)
    whole, lwhole = run(q, k, v, causal, 1, 9)
    P.check(whole.cpu().numpy(), lwhole.cpu().numpy(), o_ref, l_ref, f"{shp} c{causal} p1 s9")
    for pack, splits in ((-1, 0), (1, 1), (0, 1), (1, 3), (0, 8)):
        out, lse = run(q, k, v, causal, pack, splits)
        P.check(out.cpu().numpy(), lse.cpu().numpy(), o_ref, l_ref, f"{shp} c{causal} p{pack} s{splits}")
        assert (out - whole).abs().max().item() <= P.VARIANT_MAX
        assert (lse - lwhole).abs().max().item() <= P.VARIANT_MAX


# --- tiles whose later warps hold only padding rows (the query axis ends inside warp 0 of
# the unit's last tile) while other tiles run full: those warps skip the softmax but keep
# every hand-off with the MMA warp.  Many units and repeated calls give a hand-off that
# arrives a phase early many chances to corrupt P; the kernel is deterministic, so every
# repetition must match the first bit for bit.
PADDING_WARPS = [
    # B, Sq, Sk, Hq, Hk, d, pack: last tile holds 12 rows (g = 3), 2 rows (one head),
    # 8 rows (g = 8, the unit's second tile empty)
    ((8, 130, 700, 6, 2, 64), 1),
    ((8, 130, 700, 6, 2, 64), 0),
    ((8, 33, 520, 16, 2, 64), 1),
    ((8, 130, 700, 6, 2, 128), 1),
]


@pytest.mark.parametrize("case", PADDING_WARPS, ids=[f"{c[0]}-p{c[1]}" for c in PADDING_WARPS])
@pytest.mark.parametrize("causal", [0, 1])
def test_padding_only_warps(case, causal):
    shp, pack = case
    seed = 7100 + sum(shp)
    q, k, v = P.device_inputs(seed, *shp)
    o_ref, l_ref = P.oracle_full(seed, *shp, P.default_scale(shp[-1]), causal)
    out, lse = run(q, k, v, causal, pack, 1)
    P.check(out.cpu().numpy(), lse.cpu().numpy(), o_ref, l_ref, f"{shp} c{causal} p{pack}")
    for _ in range(8):
        o2, l2 = run(q, k, v, causal, pack, 1)
        assert torch.equal(o2, out) and torch.equal(l2, lse)
