"""GPU parity at the benchmark configurations' full sizes, on sampled rows.

Inputs are generated on the device (the same counter-based definition as the host);
the oracle regenerates on the host only the rows a sampled output reads and computes
that row exactly.  Shapes: prefill B=64 (Hq=32, Hk=8, S=2048, d=128, causal, the
scheduler's own choice of pack/splits, as the benchmark runs it); the batch-size sweep
B in {16..256}, causal and not, with pack/split variants; decode Sq=1 against
Sk in {2048, 8192, 32768} for B in {32, 128, 256} and splits in {1, 2, 4, 8}; and the
long causal case Sq=Sk=16384, B=4, for d in {64, 128} and MHA/GQA/MQA head ratios.

Scheduling variants (pack_gqa, num_splits) are also compared as whole tensors with the
unsplit GPU run of the same inputs: out and lse within 1e-3 everywhere, in every cell of
the batch sweep (B 16..256 x causal x 6 variants) and of the decode grid (splits 2/4/8
and one q-head per tile against the unsplit packed run).
"""
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
    assert G.gqa_attn_device_status(reset=True) == 0


def run_sampled(seed, shp, causal, pack=-1, splits=0, n_rows=96, inputs=None):
    import gqa_exact_attention_b200 as G
    B, Sq, Sk, Hq, Hk, d = shp
    q, k, v = inputs if inputs is not None else P.device_inputs(seed, *shp, on_device_gen=True)
    out, lse = G.gqa_attn_fwd(q, k, v, causal=causal, pack_gqa=pack, num_splits=splits)
    torch.cuda.synchronize()
    rng = np.random.default_rng(seed + 17 * splits + 3 * max(pack, 0))
    rows = P.sample_rows(rng, B, Sq, Hq, Hk, n_rows)
    idx_b = torch.tensor([r[0] for r in rows], device="cuda")
    idx_h = torch.tensor([r[1] for r in rows], device="cuda")
    idx_i = torch.tensor([r[2] for r in rows], device="cuda")
    o_gpu = out[idx_b, idx_i, idx_h].cpu().numpy()
    l_gpu = lse[idx_b, idx_h, idx_i].cpu().numpy()
    o_ref, l_ref = P.oracle_rows(seed, B, Sq, Sk, Hq, Hk, d, P.default_scale(d), causal, rows)
    return P.check(o_gpu, l_gpu, o_ref, l_ref, f"{shp} c{causal} p{pack} s{splits}")


def test_device_generator_matches_host():
    import inputs
    n = 1 << 22
    dev = inputs.device_tensor(1234, inputs.TID_K, (n,)).view(torch.int16).cpu().numpy()
    host = inputs.bits_range(1234, inputs.TID_K, 0, n).view(np.int16)
    assert np.array_equal(dev, host)


def test_prefill_b64_as_benchmarked():
    run_sampled(1001, (64, 2048, 2048, 32, 8, 128), 1, n_rows=160)


@pytest.mark.parametrize("B", [16, 32, 64, 128, 256])
@pytest.mark.parametrize("causal", [0, 1])
def test_batch_sweep_heuristic(B, causal):
    run_sampled(1002 + B, (B, 2048, 2048, 32, 8, 128), causal)


def max_abs_diff(a, b, chunk=16):
    """max |a - b| over whole tensors, a batch slice at a time (no full-size temporary)."""
    m = 0.0
    for i in range(0, a.shape[0], chunk):
        m = max(m, (a[i:i + chunk] - b[i:i + chunk]).abs().max().item())
    return m


def check_variants(seed, shp, causal, base, variants, n_rows):
    """Each scheduling variant against the fp64 oracle on sampled rows, and as whole
    tensors against the base schedule's GPU result: within 1e-3 everywhere (the
    variants differ only in fp32 summation order)."""
    import gqa_exact_attention_b200 as G
    inp = P.device_inputs(seed, *shp, on_device_gen=True)
    q, k, v = inp
    run_sampled(seed, shp, causal, base[0], base[1], n_rows=n_rows, inputs=inp)
    o_base, l_base = G.gqa_attn_fwd(q, k, v, causal=causal, pack_gqa=base[0], num_splits=base[1])
    torch.cuda.synchronize()
    worst = 0.0
    for pack, splits in variants:
        run_sampled(seed, shp, causal, pack, splits, n_rows=n_rows, inputs=inp)
        o, l = G.gqa_attn_fwd(q, k, v, causal=causal, pack_gqa=pack, num_splits=splits)
        torch.cuda.synchronize()
        do, dl = max_abs_diff(o, o_base), max_abs_diff(l, l_base)
        assert do <= P.VARIANT_MAX and dl <= P.VARIANT_MAX, (pack, splits, do, dl)
        worst = max(worst, do, dl)
        del o, l
    del inp, o_base, l_base
    torch.cuda.empty_cache()
    return worst


# the batch-size sweep: every B, causal and not, all six pack x split variants against
# the unpacked unsplit run
@pytest.mark.parametrize("B", [16, 32, 64, 128, 256])
@pytest.mark.parametrize("causal", [0, 1])
def test_batch_sweep_variants(B, causal):
    shp = (B, 2048, 2048, 32, 8, 128)
    variants = [(pk, sp) for pk in (0, 1) for sp in (1, 2, 4) if (pk, sp) != (0, 1)]
    check_variants(1102 + B + causal, shp, causal, (0, 1), variants, n_rows=48)


# the decode grid: splits 1/2/4/8 with the heuristic's packing, and one q-head per tile,
# each on sampled rows against the oracle; splits 2/4/8 and pack 0 as whole tensors
# against the unsplit packed run
@pytest.mark.parametrize("Sk", [2048, 8192, 32768])
@pytest.mark.parametrize("B", [32, 128, 256])
def test_decode(Sk, B):
    shp = (B, 1, Sk, 32, 8, 128)
    seed = 1003 + Sk + B
    check_variants(seed, shp, 0, (1, 1), [(1, 2), (1, 4), (1, 8), (0, 1)], n_rows=16)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("hk", [32, 8, 4, 1])
def test_long_causal_16k(d, hk):
    run_sampled(1005 + d + hk, (4, 16384, 16384, 32, hk, d), 1, n_rows=48)
