"""Per-shape tuning of the forward's schedule (pack_gqa, num_splits).

The pages choose PackGQA and the split count from batch-size tables tuned on H100 that
contradict one another ("优化GQA在Flash-Attention中的批量敏感性", strategy 2 and "参数组合";
"為什么 GQA 推理吞吐先升后降…", "修復" table).  This module measures the choice instead: for a
shape it times every valid (pack_gqa, num_splits) on the current GPU with CUDA events and
records the fastest in a plain-text table.  The library reads that table once per process
from the file named by the GQA_TUNE_TABLE environment variable, or, when the variable is
unset, from tune_b200.txt beside the library (the table shipped with the package, measured
on B200 with --preset workloads); GQA_TUNE_TABLE set to the empty string turns tuning off.
A fully automatic call (pack_gqa = -1, num_splits = 0, no per-sequence KV lengths) whose
shape falls in a tuned bucket then uses the tuned schedule instead of the heuristic, and
gqa_attn_choose reports it.  A schedule other than the heuristic's is recorded only when it
is at least 3 % faster than the heuristic's own, so timing noise does not flip entries.

Table lines (whitespace separated; '#' starts a comment line):

    d causal Hq Hk bucket(B) bucket(Sq) bucket(Sk) pack_gqa num_splits ms

bucket(x) is the smallest e with 2**e >= x, so one entry covers, e.g., B in 33..64.

    python -m gqa_exact_attention_b200.autotune --out tune.txt \
        --shape 64,2048,2048,32,8,128,1 --shape 32,1,8192,32,8,128,0
    GQA_TUNE_TABLE= python -m gqa_exact_attention_b200.autotune \
        --out gqa_exact_attention_b200/tune_b200.txt --preset workloads
"""
from __future__ import annotations

import argparse
import math
import os

KEY_FIELDS = 7  # d causal Hq Hk bB bSq bSk
MARGIN = 0.97   # another schedule replaces the heuristic's only below this fraction of its time


def preset_workloads():
    """(B, Sq, Sk, Hq, Hk, d, causal) of the benchmark workloads: the tiny GQA case, the
    prefill batch sweep (B 16..256, S=2048, causal and not, which includes the prefill
    benchmark B=64), the decode grid (Sk 2K/8K/32K, B 32/128/256), and the odd shapes
    (Sq=77 against Sk=4096, Sq=Sk=16384 causal; d 64 and 128; Hk 32/8/4/1 of Hq=32)."""
    shapes = [(1, 128, 128, 6, 2, 64, c) for c in (0, 1)]
    shapes += [(B, 2048, 2048, 32, 8, 128, c) for B in (16, 32, 64, 128, 256) for c in (1, 0)]
    shapes += [(B, 1, Sk, 32, 8, 128, 0) for Sk in (2048, 8192, 32768) for B in (32, 128, 256)]
    shapes += [(4, 77, 4096, 32, hk, d, 0) for d in (64, 128) for hk in (32, 8, 4, 1)]
    shapes += [(4, 16384, 16384, 32, hk, d, 1) for d in (64, 128) for hk in (32, 8, 4, 1)]
    return shapes


def bucket(x: int) -> int:
    """Smallest e with 2**e >= x (the library's shape bucket)."""
    e = 0
    while e < 31 and (1 << e) < x:
        e += 1
    return e


def key(B, Sq, Sk, Hq, Hk, d, causal):
    return (d, int(bool(causal)), Hq, Hk, bucket(B), bucket(Sq), bucket(Sk))


def candidates(B, Sq, Sk, Hq, Hk, d):
    """The schedules worth timing: pack 0, pack 1 when a group fits a tile (1 < g <= 128),
    and splits 1, 2, 4, 8, 16 up to the number of 128-key blocks."""
    g = Hq // Hk
    packs = [0] + ([1] if 1 < g <= 128 else [])
    blocks = math.ceil(Sk / 128)
    splits = [s for s in (1, 2, 4, 8, 16) if s <= blocks]
    return [(p, s) for p in packs for s in splits]


def read_table(path: str) -> dict:
    """{key: (pack, splits, ms)}; later lines win, unparsable lines are skipped."""
    table = {}
    if not os.path.exists(path):
        return table
    with open(path) as f:
        for line in f:
            if line.startswith("#"):
                continue
            parts = line.split()
            if len(parts) < KEY_FIELDS + 2:
                continue
            try:
                vals = [int(x) for x in parts[:KEY_FIELDS + 2]]
                ms = float(parts[KEY_FIELDS + 2]) if len(parts) > KEY_FIELDS + 2 else float("nan")
            except ValueError:
                continue
            table[tuple(vals[:KEY_FIELDS])] = (vals[KEY_FIELDS], vals[KEY_FIELDS + 1], ms)
    return table


def write_table(path: str, table: dict) -> None:
    lines = ["# d causal Hq Hk bucket(B) bucket(Sq) bucket(Sk) pack_gqa num_splits ms\n"]
    for k in sorted(table):
        pack, splits, ms = table[k]
        lines.append(" ".join(str(x) for x in k) + f" {pack} {splits} {ms:.4f}\n")
    tmp = path + ".tmp"
    with open(tmp, "w") as f:
        f.writelines(lines)
    os.replace(tmp, path)


def tune_shape(B, Sq, Sk, Hq, Hk, d, causal, steps=10, warmup=3, seed=0):
    """Time every candidate schedule on the current CUDA device; returns
    (best_pack, best_splits, best_ms, {(pack, splits): ms})."""
    import torch

    from . import gqa_attn_fwd, gqa_attn_device_status

    gen = torch.Generator(device="cuda").manual_seed(seed)
    q = torch.randn((B, Sq, Hq, d), generator=gen, device="cuda").to(torch.bfloat16)
    k = torch.randn((B, Sk, Hk, d), generator=gen, device="cuda").to(torch.bfloat16)
    v = torch.randn((B, Sk, Hk, d), generator=gen, device="cuda").to(torch.bfloat16)
    out = torch.empty((B, Sq, Hq, d), dtype=torch.float32, device="cuda")
    lse = torch.empty((B, Hq, Sq), dtype=torch.float32, device="cuda")
    stream = torch.cuda.current_stream()
    # the library's current choice for the shape (the heuristic's, when the process runs
    # with GQA_TUNE_TABLE set to the empty string) is timed with the candidates
    from . import gqa_attn_choose
    current = tuple(gqa_attn_choose(B, Sq, Sk, Hq, Hk, d, causal))
    cands = candidates(B, Sq, Sk, Hq, Hk, d)
    if current not in cands:
        cands.append(current)
    results = {}
    for pack, splits in cands:
        def step():
            gqa_attn_fwd(q, k, v, out=out, lse=lse, causal=causal, pack_gqa=pack,
                         num_splits=splits, stream=stream)
        for _ in range(warmup):
            step()
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(steps):
            step()
        e1.record(stream)
        torch.cuda.synchronize()
        results[(pack, splits)] = e0.elapsed_time(e1) / steps
    if gqa_attn_device_status(reset=True) != 0:
        raise RuntimeError("an in-kernel bounded wait timed out while tuning")
    (bp, bs), bms = min(results.items(), key=lambda kv: kv[1])
    # the current choice stays unless another schedule is clearly faster
    if bms > MARGIN * results[current]:
        (bp, bs), bms = current, results[current]
    return bp, bs, bms, results


def tune(shapes, path, steps=10, warmup=3):
    """Tune each (B, Sq, Sk, Hq, Hk, d, causal) and merge the results into the table at
    path (replacing entries of the same bucket)."""
    table = read_table(path)
    report = []
    for shp in shapes:
        B, Sq, Sk, Hq, Hk, d, causal = shp
        bp, bs, bms, res = tune_shape(B, Sq, Sk, Hq, Hk, d, causal, steps, warmup)
        table[key(*shp)] = (bp, bs, bms)
        report.append((shp, bp, bs, bms, res))
    write_table(path, table)
    return report


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--out", required=True, help="table file (merged if it exists)")
    ap.add_argument("--shape", action="append", default=[],
                    help="B,Sq,Sk,Hq,Hk,d,causal (repeatable)")
    ap.add_argument("--preset", choices=["workloads"], default=None,
                    help="add the benchmark workloads' shapes")
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    args = ap.parse_args()
    shapes = [tuple(int(x) for x in s.split(",")) for s in args.shape]
    if args.preset == "workloads":
        shapes += preset_workloads()
    if not shapes:
        ap.error("give --shape or --preset")
    for shp, bp, bs, bms, res in tune(shapes, args.out, args.steps, args.warmup):
        detail = " ".join(f"p{p}s{s}:{ms:.3f}" for (p, s), ms in sorted(res.items()))
        print(f"{shp}: pack {bp} splits {bs} ({bms:.3f} ms)  [{detail}]")


if __name__ == "__main__":
    main()
