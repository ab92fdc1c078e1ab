"""The tuner on the GPU: it times every candidate schedule of a shape, records the fastest,
and a process reading that table makes the tuned schedule the automatic one."""
import json
import os
import subprocess
import sys

import pytest

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


def test_tune_and_use(tmp_path):
    from gqa_exact_attention_b200 import autotune as T
    shp = (4, 1, 4096, 32, 8, 128, 0)
    path = str(tmp_path / "tune.txt")
    import gqa_exact_attention_b200 as G
    current = tuple(G.gqa_attn_choose(*shp))
    (got,) = T.tune([shp], path, steps=3, warmup=1)
    _, bp, bs, bms, res = got
    assert set(res) == set(T.candidates(*shp[:6])) | {current}
    fastest = min(res.values())
    # the fastest schedule, unless the current choice is within the margin of it
    assert res[(bp, bs)] == bms
    assert bms == fastest or ((bp, bs) == current and fastest > T.MARGIN * bms)
    assert T.read_table(path)[T.key(*shp)][:2] == (bp, bs)
    env = dict(os.environ, GQA_TUNE_TABLE=path)
    probe = ("import json, gqa_exact_attention_b200 as G; "
             f"print(json.dumps(list(G.gqa_attn_choose(*{list(shp)}))))")
    r = subprocess.run([sys.executable, "-c", probe], cwd=ROOT, env=env, capture_output=True,
                       text=True, check=True)
    assert tuple(json.loads(r.stdout.strip().splitlines()[-1])) == (bp, bs)
