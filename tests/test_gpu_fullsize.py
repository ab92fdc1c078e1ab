"""GPU parity at the benchmark configurations' full sizes, on sampled rows.

Inputs are generated on the device (the same counter-based definition as the host);
the oracle regenerates on the host only the rows a sampled output reads and computes
that row exactly.  Shapes: prefill B=64 (Hq=32, Hk=8, S=2048, d=128, causal, the
scheduler's own choice of pack/splits, as the benchmark runs it); the batch-size sweep
B in {16..256}, causal and not, with pack/split variants; decode Sq=1 against
Sk in {2048, 8192, 32768} for B in {32, 128, 256} and splits in {1, 2, 4, 8}; and the
long causal case Sq=Sk=16384, B=4, for d in {64, 128} and MHA/GQA/MQA head ratios.
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


@pytest.mark.parametrize("B,causal", [(16, 0), (16, 1), (256, 1)])
def test_batch_sweep_variants(B, causal):
    shp = (B, 2048, 2048, 32, 8, 128)
    seed = 1102 + B + causal
    inp = P.device_inputs(seed, *shp, on_device_gen=True)
    for pack in (0, 1):
        for splits in (1, 2, 4):
            run_sampled(seed, shp, causal, pack, splits, n_rows=48, inputs=inp)


@pytest.mark.parametrize("Sk", [2048, 8192, 32768])
@pytest.mark.parametrize("B", [32, 128, 256])
def test_decode(Sk, B):
    shp = (B, 1, Sk, 32, 8, 128)
    seed = 1003 + Sk + B
    inp = P.device_inputs(seed, *shp, on_device_gen=True)
    for splits in (1, 2, 4, 8):
        run_sampled(seed, shp, 0, -1, splits, n_rows=16, inputs=inp)
    run_sampled(seed, shp, 0, 0, 0, n_rows=16, inputs=inp)  # one q-head per tile
    del inp
    torch.cuda.empty_cache()


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("hk", [32, 8, 4, 1])
def test_long_causal_16k(d, hk):
    run_sampled(1005 + d + hk, (4, 16384, 16384, 32, hk, d), 1, n_rows=48)
