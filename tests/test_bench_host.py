"""bench.py host logic (CPU only): the sources each profiled kernel is built
from, the rule that a committed ncu traffic record counts only while those
sources hash the same, and the verification fields of the config."""
import json
import os

import bench
from kv_cache_bandwidth_b200.workloads import WORKLOADS, make_inputs

CSRC = os.path.join(bench.ROOT, "kv_cache_bandwidth_b200", "csrc")


def test_kernel_sources_exist():
    for kernel, files in bench.KERNEL_SOURCES.items():
        for f in files:
            assert os.path.isfile(os.path.join(CSRC, f)), (kernel, f)


def test_every_record_names_its_kernel_and_summary():
    with open(os.path.join(bench.ROOT, "profiles", "ncu_traffic.json")) as f:
        records = json.load(f)
    for key, e in records.items():
        assert e["kernel_name"] in bench.KERNEL_SOURCES, key
        assert list(e["sources"]) == list(bench.KERNEL_SOURCES[e["kernel_name"]]), key
        assert os.path.isfile(os.path.join(bench.ROOT, e["summary"])), key
        assert e["dram_bytes_per_launch"] > 0


def test_traffic_record_follows_its_sources(tmp_path, monkeypatch):
    pkg = tmp_path / "kv_cache_bandwidth_b200"
    pkg.mkdir()
    os.symlink(CSRC, pkg / "csrc")
    (tmp_path / "profiles").mkdir()
    files = bench.KERNEL_SOURCES["gqa_decode_kernel"]
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    good = bench.kernel_source_hash(files)
    records = {"w_ok": {"kernel_name": "gqa_decode_kernel", "kernel_hash": good, "dram_bytes_per_launch": 123.0},
               "w_stale": {"kernel_name": "gqa_decode_kernel", "kernel_hash": "0" * 16,
                           "dram_bytes_per_launch": 456.0}}
    (tmp_path / "profiles" / "ncu_traffic.json").write_text(json.dumps(records))
    assert bench.recorded_traffic("w_ok") == 123.0
    assert bench.recorded_traffic("w_stale") is None
    assert bench.recorded_traffic("absent") is None
    # the hash covers exactly the named files: another kernel's sources give another hash
    assert bench.kernel_source_hash(bench.KERNEL_SOURCES["gqa_verify_tc_kernel"]) != good


def test_traffic_keys_and_verification_config():
    assert bench.traffic_key("llama70b") == "llama70b"
    assert bench.traffic_key("llama70b", 8) == "llama70b_verify8"
    w = WORKLOADS["tiny"]
    inp = make_inputs(w)
    c1 = bench.config_dict(w, inp)
    assert "query_tokens" not in c1 and c1["workload"] == w.name
    c4 = bench.config_dict(w, inp, 4)
    assert c4["query_tokens"] == 4 and c4["rows_per_kv_group"] == 4 * w.r
    assert c4["kv_bytes_per_step"] == c1["kv_bytes_per_step"]
    # the config names the workload only: the library's split plan is reported apart
    assert "split_tokens" not in c1 and "decomposition" not in c1
    p = bench.plan_dict(4096, 131072)
    assert p["split_tokens"] == 4096 and "32 per sequence" in p["decomposition"]
    assert "equal-work" in bench.plan_dict(0, 32768)["decomposition"]


def test_l2_plan_keeps_steps_out_of_l2():
    L2 = bench.L2_BYTES
    assert bench.l2_plan(4 * L2) == ("resident", 1)
    for kv in (L2 // 4, L2 // 2, L2, 2 * L2, 3 * L2):
        how, n = bench.l2_plan(kv)
        assert how == "rotate" and 2 <= n <= bench.MAX_ROTATE_COPIES
        # between two reads of one copy, the other copies' bytes exceed twice the L2
        assert (n - 1) * kv > 2 * L2
        assert (n - 2) * kv <= 2 * L2  # and no more copies than that needs
    assert bench.l2_plan(256 * 1024) == ("flush", 1)
    assert bench.l2_plan(0) == ("flush", 1)
    assert "flushed" in bench.l2_desc(1000) and "copies" in bench.l2_desc(L2)


def test_sweep_fit_recovers_a_line():
    """Points on t = 5 us + bytes / 7 TB/s give back the line; a small point
    that takes longer than the line reports its ratio."""
    per = {}
    for g, kv in ((1, 67108864), (4, 268435456), (8, 536870912), (32, 2147483648)):
        per["sweep_g%d" % g] = {"kv_bytes": kv, "us_per_step": 5.0 + kv / 7e6}
    per["sweep_g1"]["us_per_step"] *= 1.5
    per["llama70b"] = {"kv_bytes": 536870912, "us_per_step": 1e9}  # not a sweep point
    fit = bench.sweep_fit(per)
    assert fit["fit_points"] == 3
    assert abs(fit["fixed_us"] - 5.0) < 1e-6
    assert abs(fit["marginal_gbs"] - 7000.0) < 1e-6
    assert abs(fit["time_over_fit"]["sweep_g1"] - 1.5) < 1e-9
    assert abs(fit["time_over_fit"]["sweep_g8"] - 1.0) < 1e-9
    assert "llama70b" not in fit["time_over_fit"]
    assert bench.sweep_fit({"sweep_g1": per["sweep_g1"]}) is None
