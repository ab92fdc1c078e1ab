"""Out-of-bounds write check for every entry point: the kernels write their own out and lse
and nothing around them, and they write every element of both.

Each output is a view into the middle of a larger buffer.  Before the call the whole buffer
holds a NaN bit pattern (a canary); after it the margins on both sides must still hold it
bit for bit, and no element of the view may.  This stands in for a memory checker, which is
not available here: a TMA box, a packed-row store or a combine row that strays past its
tensor shows up as a changed margin, a skipped row as a canary left inside.
"""
import math

import numpy as np
import pytest

from tests import parity as P

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")

MARGIN = 4096  # elements on each side; keeps the view 256-byte aligned
FILL = {torch.float32: (torch.int32, 0x7FBADBAD), torch.bfloat16: (torch.int16, 0x7FA1)}


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import gqa_exact_attention_b200 as G
    G.load()
    yield
    assert G.gqa_attn_device_status(reset=True) == 0, "an in-kernel wait timed out"


class Framed:
    """A tensor of `shape` inside a canary-filled buffer."""

    def __init__(self, shape, dtype):
        self.n = math.prod(shape)
        self.dtype = dtype
        self.buf = torch.empty(self.n + 2 * MARGIN, dtype=dtype, device="cuda")
        ity, fill = FILL[dtype]
        self.buf.view(ity).fill_(fill)
        self.t = self.buf[MARGIN:MARGIN + self.n].view(shape)

    def check(self, what):
        ity, fill = FILL[self.dtype]
        bits = self.buf.view(ity)
        assert bool((bits[:MARGIN] == fill).all()), f"{what}: written before the tensor"
        assert bool((bits[MARGIN + self.n:] == fill).all()), f"{what}: written past the tensor"
        left = int((bits[MARGIN:MARGIN + self.n] == fill).sum())
        assert left == 0, f"{what}: {left} elements not written"


def outputs(B, Sq, Hq, d, out_dtype=torch.float32):
    return Framed((B, Sq, Hq, d), out_dtype), Framed((B, Hq, Sq), torch.float32)


DENSE = [
    # B, Sq, Sk, Hq, Hk, d: packed tiles with a short last tile, one-head tiles with a
    # tail, causal rows with no key (Sq > Sk), and a decode-like short query axis
    (2, 130, 700, 6, 2, 64),
    (2, 77, 300, 8, 2, 128),
    (2, 260, 70, 4, 2, 64),
    (3, 1, 900, 32, 8, 128),
]


@pytest.mark.parametrize("shp", DENSE, ids=[str(s) for s in DENSE])
@pytest.mark.parametrize("causal", [0, 1])
@pytest.mark.parametrize("pack,splits", [(0, 1), (1, 1), (1, 3), (-1, 0)])
def test_dense(shp, causal, pack, splits):
    import gqa_exact_attention_b200 as G
    B, Sq, Sk, Hq, Hk, d = shp
    q, k, v = P.device_inputs(8100 + sum(shp), *shp)
    o, l = outputs(B, Sq, Hq, d)
    G.gqa_attn_fwd(q, k, v, out=o.t, lse=l.t, causal=causal, pack_gqa=pack, num_splits=splits)
    torch.cuda.synchronize()
    what = f"{shp} c{causal} p{pack} s{splits}"
    o.check(what + " out")
    l.check(what + " lse")


KV_LENS = [1000, 0, 1, 513]


@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("splits", [0, 3])
def test_kvcache(out_dtype, splits):
    import gqa_exact_attention_b200 as G
    B, Sq, Sk, Hq, Hk, d = 4, 1, 1000, 32, 8, 128
    q, k, v = P.device_inputs(8200 + splits, B, Sq, Sk, Hq, Hk, d)
    sl = torch.tensor(KV_LENS, dtype=torch.int32, device="cuda")
    o, l = outputs(B, Sq, Hq, d, out_dtype)
    G.gqa_attn_fwd_kvcache(q, k, v, sl, out=o.t, lse=l.t, num_splits=splits)
    torch.cuda.synchronize()
    o.check(f"kvcache {out_dtype} s{splits} out")
    l.check(f"kvcache {out_dtype} s{splits} lse")


@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("splits", [0, 2])
def test_paged(out_dtype, splits):
    import gqa_exact_attention_b200 as G
    from tests.test_gpu_paged import make_paged
    B, Sq, Hq, Hk, d = 3, 1, 32, 8, 128
    lens = [300, 0, 129]
    pg = make_paged(8300 + splits, B, Sq, Hq, Hk, d, lens, 64, 8)
    table = torch.from_numpy(pg["table"]).cuda()
    sl = torch.tensor(lens, dtype=torch.int32, device="cuda")
    o, l = outputs(B, Sq, Hq, d, out_dtype)
    G.gqa_attn_fwd_paged(pg["q"], pg["kp"], pg["vp"], table, sl, out=o.t, lse=l.t,
                         num_splits=splits)
    torch.cuda.synchronize()
    o.check(f"paged {out_dtype} s{splits} out")
    l.check(f"paged {out_dtype} s{splits} lse")


@pytest.mark.parametrize("shp,causal,lens", [
    ((4, 1, 1000, 32, 8, 128), 0, KV_LENS),
    ((1, 130, 300, 8, 2, 64), 1, None),
])
@pytest.mark.parametrize("splits", [0, 2])
def test_fp8(shp, causal, lens, splits):
    import gqa_exact_attention_b200 as G
    B, Sq, Sk, Hq, Hk, d = shp
    q, k, v = P.device_inputs(8400 + sum(shp), *shp)
    q8, k8, v8 = ((t.float() * 8).to(torch.float8_e4m3fn) for t in (q, k, v))
    sl = None if lens is None else torch.tensor(lens, dtype=torch.int32, device="cuda")
    o, l = outputs(B, Sq, Hq, d)
    G.gqa_attn_fwd_fp8(q8, k8, v8, 1 / 8, 1 / 8, 1 / 8, cache_seqlens=sl, out=o.t, lse=l.t,
                       causal=causal, num_splits=splits)
    torch.cuda.synchronize()
    o.check(f"fp8 {shp} s{splits} out")
    l.check(f"fp8 {shp} s{splits} lse")


def test_canary_is_not_a_value_the_kernels_write():
    # the fills are NaN bit patterns, which finite inputs never produce
    f32 = np.array([0x7FBADBAD], dtype=np.uint32).view(np.float32)[0]
    b16 = np.array([0x7FA1 << 16], dtype=np.uint32).view(np.float32)[0]
    assert np.isnan(f32) and np.isnan(b16)
