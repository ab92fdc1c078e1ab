"""gqa_attn_fwd_noalloc, the forward for callers that cannot allocate device memory.

Some callers cannot let a library call cudaMalloc: a serving process that reserved its
device memory up front and forbids allocation on the hot path, code that must not make
a call that can block on the device, a host that embeds the library under another
runtime's allocator.  For them the split-KV partials live in the library's fixed scratch
array instead of a cudaMallocAsync buffer.  These tests call the entry point through
the C ABI and check that it gives the results of gqa_attn_fwd, on two calls in a row
that both use the scratch, and that a request too large for the scratch is refused
before anything is launched.  (This file is collected last on purpose.)
"""
import math
import os

import numpy as np
import pytest

from tests import parity as P

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


def _noalloc(L, q, k, v, out, lse, shp, causal, pack, splits):
    B, Sq, Sk, Hq, Hk, d = shp
    stream = torch.cuda.current_stream().cuda_stream
    return L.gqa_attn_fwd_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                                  lse.data_ptr(), B, Sq, Sk, Hq, Hk, d, 1.0 / math.sqrt(d),
                                  causal, pack, splits, stream)


def test_noalloc_matches_fwd_on_two_calls_in_a_row():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import gqa_exact_attention_b200 as G
    L = G.load()
    # two different problems, back to back, both split along the key axis so both
    # use the shared scratch; the second overwrites what the first left there
    cases = [((4, 1, 2048, 32, 8, 128), 0, 1, 4, 5001),
             ((2, 77, 1000, 8, 2, 64), 1, 0, 3, 5002)]
    runs = []
    for shp, causal, pack, splits, seed in cases:
        B, Sq, Sk, Hq, Hk, d = shp
        ws = G.gqa_attn_workspace_bytes(B, Sq, Sk, Hq, Hk, d, causal, pack, splits)
        assert 0 < ws <= G.GQA_NOALLOC_SCRATCH_BYTES
        q, k, v = P.device_inputs(seed, *shp)
        out = torch.full((B, Sq, Hq, d), float("nan"), device="cuda")
        lse = torch.full((B, Hq, Sq), float("nan"), device="cuda")
        assert _noalloc(L, q, k, v, out, lse, shp, causal, pack, splits) == 0
        runs.append((shp, causal, pack, splits, q, k, v, out, lse))
    torch.cuda.synchronize()
    for shp, causal, pack, splits, q, k, v, out, lse in runs:
        ref_out, ref_lse = G.gqa_attn_fwd(q, k, v, causal=causal, pack_gqa=pack,
                                          num_splits=splits)
        torch.cuda.synchronize()
        assert torch.isfinite(out).all()
        assert (out - ref_out).abs().max().item() <= P.VARIANT_MAX
        assert (lse - ref_lse).abs().max().item() <= P.VARIANT_MAX
    assert G.gqa_attn_device_status(reset=True) == 0


def test_noalloc_refuses_partials_larger_than_the_scratch():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import gqa_exact_attention_b200 as G
    L = G.load()
    shp = (8, 128, 2048, 32, 8, 128)
    B, Sq, Sk, Hq, Hk, d = shp
    assert G.gqa_attn_workspace_bytes(B, Sq, Sk, Hq, Hk, d, 0, 0, 16) > G.GQA_NOALLOC_SCRATCH_BYTES
    q, k, v = P.device_inputs(5003, *shp)
    out = torch.full((B, Sq, Hq, d), float("nan"), device="cuda")
    lse = torch.full((B, Hq, Sq), float("nan"), device="cuda")
    assert _noalloc(L, q, k, v, out, lse, shp, 0, 0, 16) == 10  # GQA_ERR_SCRATCH
    torch.cuda.synchronize()
    assert torch.isnan(out).all() and torch.isnan(lse).all()  # nothing was written
    # the same problem without a split needs no scratch and runs
    assert _noalloc(L, q, k, v, out, lse, shp, 0, 0, 1) == 0
    torch.cuda.synchronize()
    ref_out, ref_lse = G.gqa_attn_fwd(q, k, v, causal=0, pack_gqa=0, num_splits=1)
    torch.cuda.synchronize()
    assert (out - ref_out).abs().max().item() <= P.VARIANT_MAX
    assert np.isfinite(lse.cpu().numpy()).all()


def test_noalloc_shrinks_an_automatic_split_to_fit_the_scratch():
    """An automatic split count whose partials would not fit the fixed scratch is lowered
    (down to no split) instead of failing: a caller that cannot allocate cannot predict
    the split the library will choose either."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import gqa_exact_attention_b200 as G
    L = G.load()
    shp = (1, 1024, 65536, 8, 8, 128)
    B, Sq, Sk, Hq, Hk, d = shp
    pk, ns = G.gqa_attn_choose(B, Sq, Sk, Hq, Hk, d, 0)
    assert ns >= 2
    assert G.gqa_attn_workspace_bytes(B, Sq, Sk, Hq, Hk, d, 0) > G.GQA_NOALLOC_SCRATCH_BYTES
    q, k, v = P.device_inputs(5004, *shp, on_device_gen=True)
    out = torch.full((B, Sq, Hq, d), float("nan"), device="cuda")
    lse = torch.full((B, Hq, Sq), float("nan"), device="cuda")
    assert _noalloc(L, q, k, v, out, lse, shp, 0, -1, 0) == 0
    torch.cuda.synchronize()
    ref_out, ref_lse = G.gqa_attn_fwd(q, k, v, causal=0)
    torch.cuda.synchronize()
    assert (out - ref_out).abs().max().item() <= P.VARIANT_MAX
    assert (lse - ref_lse).abs().max().item() <= P.VARIANT_MAX


def test_noalloc_runs_split_calls_while_allocation_fails():
    """With the library's allocation failure switch on (GQA_FAULT_INJECT_ALLOC, which
    makes gqa_attn_fwd's split-KV allocation fail as on an exhausted device), a split
    call of gqa_attn_fwd returns GQA_ERR_ALLOC while the allocation-free entry point runs
    the same split and matches the unsplit result: it makes no allocation."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import gqa_exact_attention_b200 as G
    L = G.load()
    shp = (4, 1, 4096, 32, 8, 128)
    B, Sq, Sk, Hq, Hk, d = shp
    q, k, v = P.device_inputs(5005, *shp)
    ref_out, ref_lse = G.gqa_attn_fwd(q, k, v, causal=0, num_splits=1)
    torch.cuda.synchronize()
    out = torch.full((B, Sq, Hq, d), float("nan"), device="cuda")
    lse = torch.full((B, Hq, Sq), float("nan"), device="cuda")
    os.environ["GQA_FAULT_INJECT_ALLOC"] = "1"
    try:
        with pytest.raises(G.GqaError) as e:
            G.gqa_attn_fwd(q, k, v, out=out, lse=lse, causal=0, num_splits=4)
        assert e.value.status == 7  # GQA_ERR_ALLOC
        assert _noalloc(L, q, k, v, out, lse, shp, 0, -1, 4) == 0
        torch.cuda.synchronize()
    finally:
        del os.environ["GQA_FAULT_INJECT_ALLOC"]
    assert (out - ref_out).abs().max().item() <= P.VARIANT_MAX
    assert (lse - ref_lse).abs().max().item() <= P.VARIANT_MAX
