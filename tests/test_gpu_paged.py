"""GPU parity of gqa_attn_fwd_paged: a KV cache held in fixed-size pages of a shared pool,
found through a block table, with per-sequence lengths.

Pages are handed to the sequences in a shuffled, non-contiguous order; table entries past a
sequence's last page hold garbage (they must never be used).  The oracle runs each sequence
on its own keys, gathered from its pages.  The paged result must also equal the dense
KV-cache entry point on the same keys bit for bit (same schedule; keys past a sequence's
length are masked, so what those rows hold does not matter as long as it is finite).
"""
import math

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


def make_paged(seed, B, Sq, Hq, Hk, d, lens, ps, max_pages, extra=5, device_gen=False):
    """Page pools, a shuffled block table, lengths, q; plus the gathered dense view."""
    import inputs
    rng = np.random.default_rng(seed)
    need = [(L + ps - 1) // ps for L in lens]
    assert max(need) <= max_pages
    num_pages = sum(need) + extra
    perm = rng.permutation(num_pages)
    table = np.empty((B, max_pages), dtype=np.int32)
    garbage = np.array([-1, num_pages, 10 ** 9, -(10 ** 6), num_pages + 7], dtype=np.int32)
    used = 0
    for b in range(B):
        table[b, :need[b]] = perm[used:used + need[b]]
        used += need[b]
        table[b, need[b]:] = garbage[rng.integers(len(garbage), size=max_pages - need[b])]
    shape = (num_pages, ps, Hk, d)
    if device_gen:
        kp = inputs.device_tensor(seed, inputs.TID_K, shape)
        vp = inputs.device_tensor(seed, inputs.TID_V, shape)
        q = inputs.device_tensor(seed, inputs.TID_Q, (B, Sq, Hq, d))
    else:
        kp = inputs.host_tensor(seed, inputs.TID_K, shape).cuda()
        vp = inputs.host_tensor(seed, inputs.TID_V, shape).cuda()
        q = inputs.host_tensor(seed, inputs.TID_Q, (B, Sq, Hq, d)).cuda()
    return dict(q=q, kp=kp, vp=vp, table=table, lens=list(lens), need=need, ps=ps,
                max_pages=max_pages, num_pages=num_pages)


def gathered(pg, which):
    """Sequence b's keys (or values) as a dense [cap, Hk, d] tensor, zero past its pages; a
    table entry outside [0, num_pages) gives a page of zeros, as the kernel reads it (the
    entries are checked here on the host: they never index the pool)."""
    pool = pg["kp"] if which == "k" else pg["vp"]
    B, cap = len(pg["lens"]), pg["max_pages"] * pg["ps"]
    ps, Hk, d = pool.shape[1], pool.shape[2], pool.shape[3]
    dense = torch.zeros((B, cap, Hk, d), dtype=pool.dtype, device=pool.device)
    for b in range(B):
        n = pg["need"][b]
        if n == 0:
            continue
        tab = pg["table"][b, :n].astype(np.int64)
        valid = (tab >= 0) & (tab < pg["num_pages"])
        idx = torch.from_numpy(np.where(valid, tab, 0)).to(pool.device)  # in range, checked on the host
        dense[b, :n * ps] = pool[idx].reshape(n * ps, Hk, d)
        for i in np.nonzero(~valid)[0]:
            dense[b, int(i) * ps:(int(i) + 1) * ps] = 0
    return dense


def oracle_paged(pg, scale, causal):
    import oracle
    kd = gathered(pg, "k").cpu().float().double().numpy()
    vd = gathered(pg, "v").cpu().float().double().numpy()
    q = pg["q"].cpu().float().double().numpy()
    outs, lses = [], []
    for b, L in enumerate(pg["lens"]):
        o, l = oracle.attn_fwd(q[b:b + 1], kd[b:b + 1, :L], vd[b:b + 1, :L], scale, causal)
        outs.append(o)
        lses.append(l)
    return np.concatenate(outs), np.concatenate(lses)


def run_paged(pg, causal, pack=-1, splits=0, bf16=False):
    import gqa_exact_attention_b200 as G
    table = torch.from_numpy(pg["table"]).cuda()
    sl = torch.tensor(pg["lens"], dtype=torch.int32, device="cuda")
    out, lse = G.gqa_attn_fwd_paged(pg["q"], pg["kp"], pg["vp"], table, sl, causal=causal,
                                    pack_gqa=pack, num_splits=splits,
                                    out_dtype=torch.bfloat16 if bf16 else torch.float32)
    torch.cuda.synchronize()
    return out, lse


CASES = [
    # (B, Sq, Hq, Hk, d), page size, pages per sequence, lengths
    ((8, 1, 32, 8, 128), 16, 40, [640, 1, 0, 15, 16, 17, 333, 511]),      # decode, 8 pages per block
    ((6, 1, 32, 8, 128), 64, 12, [768, 64, 65, 0, 700, 129]),             # 2 pages per block
    ((5, 1, 32, 4, 64), 128, 6, [768, 1, 127, 128, 500]),                 # one page per block
    ((4, 1, 32, 8, 128), 256, 4, [1024, 255, 257, 600]),                  # a block inside a page
    ((3, 200, 8, 2, 128), 32, 20, [512, 300, 150]),                       # prefill; L < Sq: empty rows
    ((2, 130, 6, 2, 64), 16, 30, [400, 131]),                             # g = 3, d = 64
]


@pytest.mark.parametrize("case", CASES, ids=[f"{c[0]}-ps{c[1]}" for c in CASES])
@pytest.mark.parametrize("causal", [0, 1])
@pytest.mark.parametrize("pack,splits", [(-1, 0), (0, 1), (1, 2), (0, 3)])
def test_paged_against_oracle_and_dense(case, causal, pack, splits):
    import gqa_exact_attention_b200 as G
    (B, Sq, Hq, Hk, d), ps, max_pages, lens = case
    pg = make_paged(7000 + sum(case[0]) + ps, B, Sq, Hq, Hk, d, lens, ps, max_pages)
    scale = P.default_scale(d)
    o_ref, l_ref = oracle_paged(pg, scale, causal)
    out, lse = run_paged(pg, causal, pack, splits)
    P.check(out.cpu().numpy(), lse.cpu().numpy(), o_ref, l_ref, f"{case} c{causal} p{pack} s{splits}")
    # the dense KV-cache entry on the gathered keys: the same result, bit for bit
    sl = torch.tensor(lens, dtype=torch.int32, device="cuda")
    od, ld = G.gqa_attn_fwd_kvcache(pg["q"], gathered(pg, "k"), gathered(pg, "v"), sl,
                                    causal=causal, pack_gqa=pack, num_splits=splits)
    torch.cuda.synchronize()
    assert torch.equal(out, od) and torch.equal(lse, ld)
    # bf16 output: the fp32 result rounded to nearest even
    ob, lb = run_paged(pg, causal, pack, splits, bf16=True)
    assert torch.equal(ob, out.to(torch.bfloat16)) and torch.equal(lb, lse)


def test_entry_outside_the_pool_reads_zeros():
    """A table entry outside [0, num_pages) within a sequence reads as a page of zeros: no
    fault, and the result is the oracle's on those zero keys."""
    (B, Sq, Hq, Hk, d), ps, max_pages, lens = (2, 1, 32, 8, 128), 64, 8, [300, 200]
    pg = make_paged(7300, B, Sq, Hq, Hk, d, lens, ps, max_pages)
    pg["table"][0, 1] = pg["num_pages"] + 3
    pg["table"][1, 2] = -7
    out, lse = run_paged(pg, 0)
    # the oracle on the same keys with those two pages zero (gathered() reads them so)
    import oracle
    kd = gathered(pg, "k")
    vd = gathered(pg, "v")
    for b, i in ((0, 1), (1, 2)):
        assert not kd[b, i * ps:(i + 1) * ps].any()
    q = pg["q"].cpu().double().numpy()
    kd, vd = kd.cpu().double().numpy(), vd.cpu().double().numpy()
    refs = [oracle.attn_fwd(q[b:b + 1], kd[b:b + 1, :L], vd[b:b + 1, :L], P.default_scale(d), False)
            for b, L in enumerate(lens)]
    P.check(out.cpu().numpy(), lse.cpu().numpy(), np.concatenate([r[0] for r in refs]),
            np.concatenate([r[1] for r in refs]), "out-of-pool entries")


@pytest.mark.parametrize("ps", [16, 256])
def test_paged_decode_full_size_equals_dense(ps):
    """Decode at the benchmark's size (B=128, capacity 8192, Hq=32, Hk=8, d=128), ragged
    lengths: the paged entry equals the dense KV-cache entry bit for bit, under the
    automatic schedule and a forced split."""
    import gqa_exact_attention_b200 as G
    B, Sq, Hq, Hk, d, cap = 128, 1, 32, 8, 128, 8192
    rng = np.random.default_rng(7400 + ps)
    lens = [int(x) for x in rng.integers(1, cap + 1, size=B)]
    pg = make_paged(7400 + ps, B, Sq, Hq, Hk, d, lens, ps, cap // ps, extra=17, device_gen=True)
    kd, vd = gathered(pg, "k"), gathered(pg, "v")
    sl = torch.tensor(lens, dtype=torch.int32, device="cuda")
    for splits in (0, 4):
        out, lse = run_paged(pg, 0, -1, splits)
        od, ld = G.gqa_attn_fwd_kvcache(pg["q"], kd, vd, sl, causal=0, num_splits=splits)
        torch.cuda.synchronize()
        assert torch.equal(out, od) and torch.equal(lse, ld)
    # and a sample of rows against the oracle
    import oracle
    for b in (0, int(np.argmax(lens)), B - 1):
        L = lens[b]
        o, l = oracle.attn_fwd(pg["q"][b:b + 1].cpu().double().numpy(),
                               kd[b:b + 1, :L].cpu().double().numpy(),
                               vd[b:b + 1, :L].cpu().double().numpy(), P.default_scale(d), False)
        P.check(out[b:b + 1].cpu().numpy(), lse[b:b + 1].cpu().numpy(), o, l, f"row b={b}")
    del kd, vd
    torch.cuda.empty_cache()
