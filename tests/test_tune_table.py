"""The tuned-schedule table: the library reads GQA_TUNE_TABLE once per process, and a
fully automatic call whose shape bucket is in the table uses the tuned (pack, splits)
instead of the heuristic (checked through gqa_attn_choose, host only); the tuner's table
format round-trips."""
import json
import os
import subprocess
import sys

from gqa_exact_attention_b200 import autotune as T

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

PROBE = r"""
import json, sys
import gqa_exact_attention_b200 as G
shapes = json.loads(sys.argv[1])
print(json.dumps([list(G.gqa_attn_choose(*s)) for s in shapes]))
"""


def choose_with_table(table_text, shapes, tmp_path):
    """gqa_attn_choose for each shape in a fresh process reading this table (None: no
    table, the heuristic; "shipped": GQA_TUNE_TABLE unset, the table beside the library)."""
    env = dict(os.environ)
    if table_text is None:
        env["GQA_TUNE_TABLE"] = ""
    elif table_text == "shipped":
        env.pop("GQA_TUNE_TABLE", None)
    else:
        path = tmp_path / "tune.txt"
        path.write_text(table_text)
        env["GQA_TUNE_TABLE"] = str(path)
    r = subprocess.run([sys.executable, "-c", PROBE, json.dumps(shapes)], cwd=ROOT, env=env,
                       capture_output=True, text=True, check=True)
    return [tuple(x) for x in json.loads(r.stdout.strip().splitlines()[-1])]


def line(B, Sq, Sk, Hq, Hk, d, causal, pack, splits):
    return " ".join(str(x) for x in T.key(B, Sq, Sk, Hq, Hk, d, causal)) + f" {pack} {splits} 0.1\n"


def test_bucket():
    assert [T.bucket(x) for x in (1, 2, 3, 4, 5, 33, 64, 65, 2048, 2049)] == [0, 1, 2, 2, 3, 6, 6, 7, 11, 12]


def test_table_replaces_the_heuristic_within_its_bucket(tmp_path):
    dec = (32, 1, 8192, 32, 8, 128, 0)
    heur = choose_with_table(None, [dec], tmp_path)[0]
    assert heur != (0, 3)
    txt = "# comment\n" + line(*dec, 0, 3)
    same_bucket = (17, 1, 5000, 32, 8, 128, 0)    # B 17..32, Sk 4097..8192
    other_bucket = (33, 1, 8192, 32, 8, 128, 0)
    other_causal = (32, 1, 8192, 32, 8, 128, 1)
    got = choose_with_table(txt, [dec, same_bucket, other_bucket, other_causal], tmp_path)
    assert got[0] == (0, 3) and got[1] == (0, 3)
    base = choose_with_table(None, [other_bucket, other_causal], tmp_path)
    assert got[2] == base[0] and got[3] == base[1]


def test_later_lines_win_and_bad_lines_are_skipped(tmp_path):
    shp = (64, 2048, 2048, 32, 8, 128, 1)
    txt = line(*shp, 0, 2) + "not a line\n1 2 3\n" + line(*shp, 1, 4) + "128 1 32 8 6 11 11 2 1\n"
    assert choose_with_table(txt, [shp], tmp_path)[0] == (1, 4)


def test_entries_are_validated_against_the_shape(tmp_path):
    mqa256 = (1, 64, 4096, 256, 1, 64, 0)   # g = 256: packing is impossible
    short = (4, 1, 256, 32, 8, 128, 0)      # 2 key blocks: splits clamp to 2
    txt = line(*mqa256, 1, 1) + line(*short, 1, 16)
    base = choose_with_table(None, [mqa256], tmp_path)[0]
    got = choose_with_table(txt, [mqa256, short], tmp_path)
    assert got[0] == base
    assert got[1] == (1, 2)


def test_missing_file_keeps_the_heuristic(tmp_path):
    shp = (64, 2048, 2048, 32, 8, 128, 1)
    env_missing = choose_with_table(None, [shp], tmp_path)
    assert choose_with_table("", [shp], tmp_path) == env_missing


def test_candidates():
    assert T.candidates(4, 1, 256, 32, 8, 128) == [(0, 1), (0, 2), (1, 1), (1, 2)]
    assert T.candidates(4, 1, 4096, 32, 32, 128) == [(0, 1), (0, 2), (0, 4), (0, 8), (0, 16)]
    assert all(p == 0 for p, _ in T.candidates(1, 64, 512, 256, 1, 64))


def test_table_round_trip(tmp_path):
    path = str(tmp_path / "t.txt")
    tab = {T.key(64, 2048, 2048, 32, 8, 128, 1): (1, 1, 2.5),
           T.key(32, 1, 8192, 32, 8, 128, 0): (1, 2, 0.17)}
    T.write_table(path, tab)
    assert T.read_table(path) == tab


SHIPPED = os.path.join(ROOT, "gqa_exact_attention_b200", "tune_b200.txt")


def test_shipped_table_is_read_by_default(tmp_path):
    """With GQA_TUNE_TABLE unset the library reads the table shipped beside it; set to the
    empty string, no table at all (the heuristic)."""
    table = T.read_table(SHIPPED)
    assert table, "the package ships a tuned table"
    shapes = T.preset_workloads()
    shipped = choose_with_table("shipped", shapes, tmp_path)
    heur = choose_with_table(None, shapes, tmp_path)
    for shp, got, h in zip(shapes, shipped, heur):
        k = T.key(*shp)
        assert k in table, f"{shp} is not in the shipped table"
        blocks = -(-shp[2] // 128)
        want = (table[k][0], min(table[k][1], blocks, 16))
        assert got == want, (shp, got, want)
    # the same table named explicitly gives the same answers
    assert choose_with_table(open(SHIPPED).read(), shapes, tmp_path) == shipped
    assert len(heur) == len(shipped)


def test_shipped_table_entries_are_valid():
    for k, (pack, splits, ms) in T.read_table(SHIPPED).items():
        d, causal, Hq, Hk = k[:4]
        assert d in (64, 128) and causal in (0, 1) and Hq % Hk == 0
        assert pack in (0, 1) and 1 <= splits <= 16 and ms > 0
        assert pack == 0 or 1 < Hq // Hk <= 128
