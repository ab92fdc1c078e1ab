"""GPU parity of gqa_attn_fwd_kvcache: a KV cache whose sequences have their own lengths
(cache_seqlens), fp32 or bf16 output.

The oracle runs each sequence on its own key count (the cache rows [0, L_b)), so causal
masks are bottom-right aligned to L_b as the entry point defines.  bf16 output must equal
the fp32 output of the same call rounded to nearest even, bit for bit; with no lengths, or
with all lengths = capacity under the same pack/split schedule, the entry point must equal
gqa_attn_fwd bit for bit.
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
    assert G.gqa_attn_device_status(reset=True) == 0, "an in-kernel wait timed out"


def oracle_varlen(seed, shp, lens, causal):
    import oracle
    B, Sq, Sk, Hq, Hk, d = shp
    q, k, v = P.host_inputs_f64(seed, *shp)
    outs, lses = [], []
    for b, L in enumerate(lens):
        o, l = oracle.attn_fwd(q[b:b + 1], k[b:b + 1, :L], v[b:b + 1, :L], P.default_scale(d), causal)
        outs.append(o)
        lses.append(l)
    return np.concatenate(outs), np.concatenate(lses)


def run_kv(q, k, v, lens, causal, pack=-1, splits=0, bf16=False):
    import gqa_exact_attention_b200 as G
    sl = None if lens is None else torch.tensor(lens, dtype=torch.int32, device="cuda")
    out, lse = G.gqa_attn_fwd_kvcache(q, k, v, sl, causal=causal, pack_gqa=pack, num_splits=splits,
                                      out_dtype=torch.bfloat16 if bf16 else torch.float32)
    torch.cuda.synchronize()
    return out, lse


CASES = [
    # (B, Sq, Sk capacity, Hq, Hk, d), lengths per sequence
    ((8, 1, 1000, 32, 8, 128), [1000, 1, 0, 517, 128, 129, 999, 256]),   # decode, ragged, empty
    ((4, 1, 3000, 32, 4, 64), [3000, 2048, 77, 1500]),                   # decode, d=64, g=8
    ((3, 200, 512, 8, 2, 128), [512, 300, 150]),                         # prefill; L < Sq: empty rows
    ((2, 130, 400, 6, 3, 64), [400, 131]),                               # g=3 (packing pads)
]


@pytest.mark.parametrize("case", CASES, ids=[str(c[0]) for c in CASES])
@pytest.mark.parametrize("causal", [0, 1])
@pytest.mark.parametrize("pack,splits", [(-1, 0), (0, 1), (1, 1), (0, 3), (1, 2)])
def test_varlen_against_oracle(case, causal, pack, splits):
    shp, lens = case
    seed = 5000 + sum(shp)
    q, k, v = P.device_inputs(seed, *shp)
    o_ref, l_ref = oracle_varlen(seed, shp, lens, causal)
    out, lse = run_kv(q, k, v, lens, causal, pack, splits)
    P.check(out.cpu().numpy(), lse.cpu().numpy(), o_ref, l_ref, f"{shp} c{causal} p{pack} s{splits}")
    # bf16 output: the same values rounded to nearest even
    ob, lb = run_kv(q, k, v, lens, causal, pack, splits, bf16=True)
    assert ob.dtype == torch.bfloat16
    assert torch.equal(ob, out.to(torch.bfloat16))
    assert torch.equal(lb, lse)


@pytest.mark.parametrize("causal", [0, 1])
def test_no_lengths_equals_fwd(causal):
    import gqa_exact_attention_b200 as G
    shp = (4, 300, 700, 32, 8, 128)
    q, k, v = P.device_inputs(6000 + causal, *shp)
    ref, lref = G.gqa_attn_fwd(q, k, v, causal=causal)
    # no lengths: the same plan as gqa_attn_fwd
    out, lse = run_kv(q, k, v, None, causal)
    assert torch.equal(out, ref) and torch.equal(lse, lref)
    # all lengths = capacity: the same values under the same schedule (with lengths given
    # the automatic split count follows the ragged-length rule, so pin pack and splits)
    pk, ns = G.gqa_attn_choose(*shp, causal)
    ref, lref = G.gqa_attn_fwd(q, k, v, causal=causal, pack_gqa=pk, num_splits=ns)
    out, lse = run_kv(q, k, v, [700] * 4, causal, pk, ns)
    assert torch.equal(out, ref) and torch.equal(lse, lref)


def test_lengths_are_clamped_to_capacity():
    shp = (3, 1, 600, 32, 8, 128)
    seed = 6100
    q, k, v = P.device_inputs(seed, *shp)
    out, lse = run_kv(q, k, v, [-5, 100000, 300], 0)
    o_ref, l_ref = oracle_varlen(seed, shp, [0, 600, 300], 0)
    P.check(out.cpu().numpy(), lse.cpu().numpy(), o_ref, l_ref, "clamped lengths")


def test_prefill_bf16_full_size_sampled():
    """The benchmark's prefill shape with bf16 output through the TMA-store epilogue."""
    import gqa_exact_attention_b200 as G
    shp = (16, 2048, 2048, 32, 8, 128)
    q, k, v = P.device_inputs(1001, *shp, on_device_gen=True)
    for causal in (0, 1):
        ref, lref = G.gqa_attn_fwd(q, k, v, causal=causal)
        ob, lb = run_kv(q, k, v, None, causal, bf16=True)
        assert torch.equal(ob, ref.to(torch.bfloat16)) and torch.equal(lb, lref)
