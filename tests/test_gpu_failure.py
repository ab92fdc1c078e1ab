"""Failure detection on the GPU, exercised without faulting the GPU.

Two paths, each driven by the library's own host-side switches:

* Allocation failure.  GQA_FAULT_INJECT_ALLOC makes the split-KV partials' allocation
  fail as it would on an exhausted device.  The call must return GQA_ERR_ALLOC before
  launching anything (out and lse keep their NaN fill); calls that need no allocation
  still run.
* Bounded waits.  Every wait inside the forward kernel is bounded.  GQA_FAULT_INJECT_STALL
  makes each CTA first wait on a barrier that nothing arrives on (a flag that nothing
  sets), with the limit at 20 ms (GQA_WAIT_TIMEOUT_MS).  The call must still return
  (asynchronously, GQA_OK), the device status word must read GQA_ERR_TIMEOUT after
  synchronising, every other warp must notice the abort and exit, and a normal call
  afterwards must match the oracle.  This runs in a child process under a time limit,
  once for the one-tile kernel (decode-like shape, the softmax warpgroup writes the
  output) and once for the two-tile kernel (prefill-like shape, epilogue warpgroup with
  TMA stores).
"""
import json
import os
import subprocess
import sys

import numpy as np
import pytest

from tests import parity as P

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import gqa_exact_attention_b200 as G
    G.load()
    yield
    assert G.gqa_attn_device_status(reset=True) == 0


def test_allocation_failure_is_reported_before_any_launch():
    import gqa_exact_attention_b200 as G
    shp = (2, 64, 2048, 8, 2, 128)
    B, Sq, Sk, Hq, Hk, d = shp
    q, k, v = P.device_inputs(7100, *shp)
    ref, lref = G.gqa_attn_fwd(q, k, v, num_splits=1)
    torch.cuda.synchronize()
    out = torch.full((B, Sq, Hq, d), float("nan"), device="cuda")
    lse = torch.full((B, Hq, Sq), float("nan"), device="cuda")
    os.environ["GQA_FAULT_INJECT_ALLOC"] = "1"
    try:
        with pytest.raises(G.GqaError) as e:
            G.gqa_attn_fwd(q, k, v, out=out, lse=lse, num_splits=4)
        assert e.value.status == 7  # GQA_ERR_ALLOC
        with pytest.raises(G.GqaError) as e:
            G.gqa_attn_fwd_kvcache(q, k, v, None, out=out, lse=lse, num_splits=3)
        assert e.value.status == 7
        torch.cuda.synchronize()
        assert torch.isnan(out).all() and torch.isnan(lse).all()  # nothing was launched
        # a call that needs no allocation is unaffected
        G.gqa_attn_fwd(q, k, v, out=out, lse=lse, num_splits=1)
        torch.cuda.synchronize()
    finally:
        del os.environ["GQA_FAULT_INJECT_ALLOC"]
    assert torch.equal(out, ref) and torch.equal(lse, lref)
    # and once the switch is off, the split call allocates and runs
    o2, l2 = G.gqa_attn_fwd(q, k, v, num_splits=4)
    torch.cuda.synchronize()
    assert (o2 - ref).abs().max().item() <= P.VARIANT_MAX
    assert (l2 - lref).abs().max().item() <= P.VARIANT_MAX


_CHILD = r"""
import json, os, sys, time
sys.path.insert(0, os.getcwd())
import numpy as np
import torch
import gqa_exact_attention_b200 as G
from tests import parity as P

torch.cuda.set_device(0)
G.load()
shp = tuple(json.loads(sys.argv[1]))
pack, splits = int(sys.argv[2]), int(sys.argv[3])
B, Sq, Sk, Hq, Hk, d = shp
seed = 7200 + Sq
q, k, v = P.device_inputs(seed, *shp)
res = {}
assert G.gqa_attn_device_status(reset=True) == 0
os.environ["GQA_WAIT_TIMEOUT_MS"] = "20"
os.environ["GQA_FAULT_INJECT_STALL"] = "1"
t0 = time.time()
out, lse = G.gqa_attn_fwd(q, k, v, pack_gqa=pack, num_splits=splits)  # returns: async
res["returned"] = True
torch.cuda.synchronize()
res["sync_s"] = time.time() - t0
res["status_after_short_limit"] = G.gqa_attn_device_status(reset=True)
del os.environ["GQA_FAULT_INJECT_STALL"]
del os.environ["GQA_WAIT_TIMEOUT_MS"]
out, lse = G.gqa_attn_fwd(q, k, v, pack_gqa=pack, num_splits=splits)
torch.cuda.synchronize()
res["status_after_normal_call"] = G.gqa_attn_device_status(reset=True)
o_ref, l_ref = P.oracle_full(seed, *shp, P.default_scale(d), False)
res["parity"] = P.check(out.cpu().numpy(), lse.cpu().numpy(), o_ref, l_ref, "after timeout")
print("RESULT " + json.dumps(res), flush=True)
"""


@pytest.mark.parametrize("shp,pack,splits", [
    ((1, 128, 1024, 8, 2, 128), 0, 2),   # one tile per unit: softmax warpgroup writes rows
    ((1, 256, 1024, 8, 2, 128), 0, 2),   # two tiles per unit: epilogue warpgroup, TMA stores
], ids=["one_tile", "two_tiles"])
def test_bounded_wait_timeout_is_reported_and_recoverable(shp, pack, splits):
    env = dict(os.environ)
    for name in ("GQA_WAIT_TIMEOUT_NS", "GQA_WAIT_TIMEOUT_MS", "GQA_FAULT_INJECT_STALL"):
        env.pop(name, None)
    r = subprocess.run([sys.executable, "-c", _CHILD, json.dumps(list(shp)), str(pack), str(splits)],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-4000:]
    line = [ln for ln in r.stdout.splitlines() if ln.startswith("RESULT ")][-1]
    res = json.loads(line[len("RESULT "):])
    assert res["returned"]
    assert res["status_after_short_limit"] == 9  # GQA_ERR_TIMEOUT
    assert res["status_after_normal_call"] == 0
    # every CTA gave up and drained promptly (the drain waits are bounded at >= 1 s each)
    assert res["sync_s"] < 60.0
    assert np.isfinite(res["parity"]["out_max"])
