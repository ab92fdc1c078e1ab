"""Host logic of bench.py: the work accounting its metrics rest on, and the rule that
reports committed DRAM counters only for the kernel source and schedule they were taken
on."""
import importlib.util
import json
import os

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def brute_pairs(Sq, Sk):
    """Allowed (query, key) pairs under the bottom-right causal mask, by enumeration."""
    return sum(1 for i in range(Sq) for j in range(Sk) if j <= i + Sk - Sq)


@pytest.mark.parametrize("Sq,Sk", [(1, 1), (5, 5), (7, 3), (3, 7), (1, 9), (9, 1), (16, 16),
                                   (130, 257), (257, 130), (64, 64), (100, 1)])
def test_causal_pairs_brute_force(bench, Sq, Sk):
    assert bench.causal_pairs(Sq, Sk) == brute_pairs(Sq, Sk)


def test_flops_conventions(bench):
    # non-causal: 2 flops per multiply-add in QK^T and in PV
    assert bench.flops(2, 3, 5, 4, 8, 0) == 4.0 * 2 * 4 * 8 * 3 * 5
    # causal with Sq == Sk: halved (the pages' convention), not the exact pair count
    assert bench.flops(1, 64, 64, 1, 1, 1) == 4.0 * 64 * 64 / 2
    # causal with Sq != Sk: the exact allowed pairs
    assert bench.flops(1, 7, 3, 1, 1, 1) == 4.0 * brute_pairs(7, 3)
    # the benchmark's prefill workload: 2.199 TFLOP per launch
    assert abs(bench.flops(64, 2048, 2048, 32, 128, 1) - 2.199e12) < 1e9


def test_hbm_bytes(bench):
    B, Sq, Sk, Hq, Hk, d = 3, 5, 7, 8, 2, 64
    q = B * Sq * Hq * d * 2
    kv = 2 * B * Sk * Hk * d * 2
    o = B * Sq * Hq * d * 4
    lse = B * Hq * Sq * 4
    assert bench.hbm_bytes(B, Sq, Sk, Hq, Hk, d) == q + kv + o + lse
    # the decode configuration's algorithmic bytes as the profiles state them
    assert bench.hbm_bytes(256, 1, 8192, 32, 8, 128) == 8596258816


def test_job_throughput_is_weak_scaling(bench):
    # every rank processes the same work per step; the slowest rank's time sets the rate
    assert bench.job_throughput(10.0, 4, total_ms=20.0, steps=10) == 4 * 10.0 / 0.002


def test_traffic_only_for_matching_source_and_schedule(bench, tmp_path, monkeypatch):
    key = "w"
    entry = {"dram_bytes_per_launch": 123, "pack_gqa": 1, "num_splits": 1}
    path = tmp_path / "traffic.json"
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(path))
    assert bench.traffic_for(key, 1, 1) is None  # no file
    path.write_text(json.dumps({"kernel_sha256_16": bench.kernel_hash(), "workloads": {key: entry}}))
    assert bench.traffic_for(key, 1, 1) == 123
    assert bench.traffic_for(key, 0, 1) is None  # other pack
    assert bench.traffic_for(key, 1, 2) is None  # other split
    assert bench.traffic_for("other", 1, 1) is None
    path.write_text(json.dumps({"kernel_sha256_16": "0" * 16, "workloads": {key: entry}}))
    assert bench.traffic_for(key, 1, 1) is None  # other kernel source


def test_committed_traffic_matches_the_current_kernel(bench):
    """The committed counters are for this kernel source; their algorithmic bytes agree
    with the accounting above."""
    t = json.load(open(os.path.join(ROOT, "profiles", "traffic.json")))
    if t["kernel_sha256_16"] != bench.kernel_hash():
        pytest.skip("the counters are for an earlier kernel source: the bench reports null")
    w = t["workloads"]["prefill B=64 Hq=32 Hk=8 Sq=Sk=2048 d=128 causal"]
    assert w["algorithmic_bytes"] == bench.hbm_bytes(64, 2048, 2048, 32, 8, 128)
    assert w["dram_bytes_per_launch"] == w["dram_bytes_read"] + w["dram_bytes_write"]


def test_committed_traffic_covers_both_objects_of_the_default_line(bench):
    """The default line reports roofline.traffic for the prefill workload and for its
    decode object; the committed counters must be found under both names (and agree with
    the algorithmic accounting), or a matching source hash would still print null."""
    t = json.load(open(os.path.join(ROOT, "profiles", "traffic.json")))
    if t["kernel_sha256_16"] != bench.kernel_hash():
        pytest.skip("the counters are for an earlier kernel source: the bench reports null")
    c = bench.DECODE_CFG
    for name, shape in (("prefill B=64 Hq=32 Hk=8 Sq=Sk=2048 d=128 causal", (64, 2048, 2048, 32, 8, 128)),
                        (c["name"], (c["B"], c["Sq"], c["Sk"], c["Hq"], c["Hk"], c["d"]))):
        assert bench.traffic_for(name, 1, 1) is not None, name
        w = t["workloads"][name]
        assert w["algorithmic_bytes"] == bench.hbm_bytes(*shape)
        assert 0.9 < w["dram_bytes_per_launch"] / w["algorithmic_bytes"] < 1.3


def test_every_fraction_is_also_given_against_the_nominal_peaks():
    import bench
    t = bench.with_spec({"bound": "tensor", "achieved": 1125.0})
    h = bench.with_spec({"bound": "hbm", "achieved": 6000.0})
    assert t["spec_peak"] == 2250.0 and t["frac_of_spec"] == 0.5
    assert h["spec_peak"] == 8000.0 and h["frac_of_spec"] == 0.75
