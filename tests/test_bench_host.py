"""Host logic of bench.py that needs no GPU: the clock summary that decides
which throttle reasons a bench line reports, and the rule that ncu traffic
counters are used only while they were taken on the current kernel sources
and the same workload."""
import json
import os

import bench


def _summary_of(tmp_path, lines):
    path = tmp_path / "clocks.csv"
    path.write_text("".join(l + "\n" for l in lines))
    cs = bench.ClockSampler(0)
    cs.proc = object()                      # as if nvidia-smi had been started
    cs.path = str(path)
    return cs.summary()


def test_clock_summary_median_max_and_reasons(tmp_path):
    na, act = "Not Active", "Active"
    rows = [f"0, {mhz}, 1965, 700.0, 0x0, {na}, {na}, {na}, {cap}"
            for mhz, cap in ((1965, na), (1950, act), (1800, na), (1965, na), (1900, act))]
    s = _summary_of(tmp_path, rows + ["garbage line"])
    assert s["samples"] == 5
    assert s["sm_mhz"] == 1950 and s["sm_max_mhz"] == 1965
    assert s["reasons"] == ["sw_power_cap"]


def test_clock_summary_reports_thermal_and_hw_slowdowns(tmp_path):
    na, act = "Not Active", "Active"
    rows = [f"0, 1500, 1965, 900.0, 0x0, {act}, {na}, {na}, {na}",
            f"0, 1400, 1965, 950.0, 0x0, {na}, {act}, {act}, {na}"]
    s = _summary_of(tmp_path, rows)
    assert s["reasons"] == ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"]
    assert s["sm_mhz"] == 1450


def test_clock_summary_without_samples_is_none(tmp_path):
    assert _summary_of(tmp_path, []) is None
    assert bench.ClockSampler(0).summary() is None          # nvidia-smi never started


def test_traffic_record_only_for_current_sources_and_workload(monkeypatch):
    """Records are keyed kernel@workload: each workload gets its own kernel's
    record, and only while the device-code hash matches."""
    with open(os.path.join(bench.ROOT, "profiles", "ncu_traffic.json")) as f:
        rec = json.load(f)
    recs = {k: v for k, v in rec.items() if isinstance(v, dict) and "source_sha" in v}
    assert recs and all(k == f"{v['kernel']}@{v['workload']}" for k, v in recs.items())
    r = next(iter(recs.values()))
    monkeypatch.setattr(bench, "kernel_source_sha", lambda: r["source_sha"])
    for v in recs.values():
        assert bench.kernel_traffic_record(v["kernel"], v["workload"]) == v
    name = r["kernel"]
    assert bench.kernel_traffic_record(name, r["workload"] + "_other") is None
    assert bench.kernel_traffic_record(name, r["workload"], coef="state") is None
    assert bench.kernel_traffic_record("no_such_kernel", r["workload"]) is None
    # the same kernel on two workloads: two different records
    by_kernel = {}
    for v in recs.values():
        by_kernel.setdefault(v["kernel"], []).append(v)
    for vs in by_kernel.values():
        if len(vs) > 1:
            a, b = vs[0], vs[1]
            assert bench.kernel_traffic_record(a["kernel"], a["workload"])["dram_bytes_per_launch"] != \
                bench.kernel_traffic_record(b["kernel"], b["workload"])["dram_bytes_per_launch"]
    monkeypatch.setattr(bench, "kernel_source_sha", lambda: "0" * 16)
    assert bench.kernel_traffic_record(name, r["workload"]) is None


def test_kernel_source_sha_ignores_the_host_api_file(tmp_path, monkeypatch):
    csrc = tmp_path / "ssm_decode_b200" / "csrc"
    csrc.mkdir(parents=True)
    (csrc / "k.cu").write_text("kernel")
    (csrc / "ss_api.cu").write_text("host v1")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    a = bench.kernel_source_sha()
    (csrc / "ss_api.cu").write_text("host v2")
    assert bench.kernel_source_sha() == a
    (csrc / "k.cu").write_text("kernel changed")
    assert bench.kernel_source_sha() != a


def test_cpu_baseline_all_cores_leg_and_its_fallback():
    """The oracle baseline: a 1-thread figure, then single-threaded spawned
    processes whose rates add up; a parallel leg that fails or runs out of
    time leaves the 1-thread figure and says why."""
    import argparse
    a = argparse.Namespace(workload="mamba2_b4")
    r = bench.cpu_baseline(a, one_s=0.3, each_s=0.3, max_workers=2)
    assert r["kind"] == "oracle" and r["one_thread"]["value"] > 0
    if bench.host_cores() > 1:
        assert r["cores"] == 2 and "parallel_error" not in r
        assert r["value"] > r["one_thread"]["value"]
    f = bench.cpu_baseline(a, one_s=0.3, each_s=30.0, max_workers=2, timeout_s=0.5)
    if bench.host_cores() > 1:
        assert f["cores"] == 1 and f["value"] == f["one_thread"]["value"]
        assert f["parallel_error"].startswith("TimeoutError")
