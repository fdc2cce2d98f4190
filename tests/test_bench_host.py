"""Host logic of bench.py (no GPU): the reference arm's JSON line, the
roofline arithmetic, the clock record and the traffic lookup."""
import json
import os
import subprocess
import sys
import types

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def test_reference_arm_prints_one_json_line():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--workload", "tiny", "--steps", "1", "--warmup", "3",
                          "--cpu-seconds", "1"],
                         capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["higher_is_better"] is True
    assert d["unit"] == "blocks/s" and d["value"] > 0 and d["steps"] == 1 and d["warmup"] >= 3
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"] and cb["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": "blocks/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}
    assert d["config"]["workload"] == "tiny"


def test_reference_arm_other_ranks_exit_quietly():
    """Under torchrun only rank 0 runs and prints the reference arm; the
    other ranks exit 0 without output or work."""
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--workload", "tiny", "--steps", "1", "--warmup", "3"],
                         capture_output=True, text=True, timeout=600, cwd=ROOT, env=env)
    assert out.returncode == 0, out.stderr[-2000:]
    assert out.stdout.strip() == ""


def _run(R, C, blocks):
    L = types.SimpleNamespace(R=R, C=C)
    return types.SimpleNamespace(layers=[L], blocks=lambda: blocks)


def test_roofline_local_hessian_without_counters_is_labelled_definition_equivalent(
        tmp_path, monkeypatch):
    import bench
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(tmp_path / "missing.json"))
    pk = {"sm_max_mhz": 1965.0, "hbm_gbs": 6555.5}
    run = _run(4096, 4096, 1 << 20)
    evals = 30.0 * (1 << 20)
    r = bench.make_roofline(run, {"search_lh": {"ms": 0.5}}, pk, "measured", "dense", evals)
    peak = 148 * 128 * 2 * 1965e6 / 1e12
    assert r["bound"] == "alu" and r["unit"] == "TFLOP/s" and "not a utilisation" in r["basis"]
    assert abs(r["peak"] - round(peak, 2)) < 1e-9
    assert abs(r["achieved"] - round(544 * evals / 0.5e-3 / 1e12, 2)) < 1e-9
    assert abs(r["frac"] - round(r["achieved"] / r["peak"], 4)) < 2e-4
    assert r["evaluated_per_block"] == 30.0
    d = r["definition_equivalent"]
    assert abs(d["TFLOP/s_all_126_equivalent"] - round(544 * 126 * (1 << 20) / 0.5e-3 / 1e12, 2)) < 1e-9


def test_roofline_local_hessian_is_issue_slots_from_recorded_instructions(tmp_path, monkeypatch):
    """With an ncu instruction count taken on the current sources, the
    search's roofline is warp instructions per call over the live call time
    against 148 SMs x 4 issue slots at the sampled SM clock."""
    import bench
    f = tmp_path / "traffic.json"
    f.write_text(json.dumps({"search_lh": {"moe": {
        "source_hash": bench.kernel_source_hash("search_lh"),
        "dram_bytes_per_launch": 4.5e8, "warp_inst_per_launch": 2.0e9}}}))
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(f))
    run = _run(768, 2048, 12582912)
    r = bench.make_roofline(run, {"search_lh": {"ms": 2.5}}, {"sm_max_mhz": 1965.0}, "measured",
                            "moe", 18.0 * 12582912, sm_mhz_live=1900.0)
    peak = 148 * 4 * 1900e6 / 1e12
    assert r["bound"] == "alu" and r["unit"] == "Twarp-instructions/s"
    assert abs(r["peak"] - round(peak, 4)) < 1e-12
    assert abs(r["achieved"] - round(2.0e9 / 2.5e-3 / 1e12, 4)) < 1e-12
    assert abs(r["frac"] - round(r["achieved"] / r["peak"], 4)) < 2e-4
    assert r["traffic"] == 4.5e8 and r["warp_inst_per_call"] == 2.0e9
    assert bench.search_blocks_per_s(run, {"search_lh": {"ms": 2.5}}) == round(12582912 / 2.5e-3, 1)


def test_roofline_gptq_is_fp64_definition_flops():
    import bench
    pk = {"sm_max_mhz": 1965.0}
    run = _run(4096, 4096, 1 << 20)
    r = bench.make_roofline(run, {"gptq": {"ms": 10.0}, "search_lh": {"ms": 0.4}}, pk, "measured",
                            "lh_gptq", 1.0)
    peak = 148 * 64 * 2 * 1965e6 / 1e12
    flop = 4096 * 4096 ** 2 + 4096 ** 3 / 3
    assert r["bound"] == "alu" and abs(r["peak"] - round(peak, 2)) < 1e-9
    assert abs(r["achieved"] - round(flop / 10e-3 / 1e12, 2)) < 1e-9
    assert r["traffic"] is None


def test_gptq_launch_count_follows_the_panel_schedule():
    import bench
    # C = 128: lambda, copy, one diagonal block, one row kernel
    # C = 256: + panel solve and next-panel update, a second block, one product
    # C = 384: + one update beyond the next panel, a third panel and block
    assert [bench.gptq_launches(n) for n in (1, 2, 3)] == [4, 9, 15]


class _Done:
    def terminate(self):
        pass

    def wait(self, timeout=None):
        return 0

    def join(self, timeout=None):
        pass


def test_clock_sampler_reads_nvidia_smi_lines():
    """The clocks key: median SM clock under load, the largest max clock,
    and every throttle reason seen Active; short or unparsable lines are
    skipped."""
    import bench
    s = bench.ClockSampler(0)
    s.proc, s.thread = _Done(), _Done()
    na = "Not Active"
    s.lines = [
        "0, 1965, 1965, 812.3, 0x0, %s, %s, %s, %s" % (na, na, na, na),
        "0, 1800, 1965, 990.1, 0x4, %s, %s, %s, Active" % (na, na, na),
        "0, 1890, 1965, 950.0, 0x4, %s, %s, %s, Active" % (na, na, na),
        "0, [N/A], 1965, 950.0, 0x0, %s, %s, %s, %s" % (na, na, na, na),
        "garbage",
        "",
    ]
    c = s.stop()
    assert c == {"sm_mhz": 1890.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"],
                 "samples": 3}
    s.lines = ["0, 1200, 1965, 400, 0x8, Active, %s, Active, %s" % (na, na)]
    assert s.stop()["reasons"] == ["hw_slowdown", "sw_thermal_slowdown"]
    s.lines = ["nothing usable"]
    assert s.stop() is None


def test_recorded_traffic_needs_the_current_sources(tmp_path, monkeypatch):
    """ncu traffic is reported only while the kernel's sources hash to the
    value recorded with it; otherwise (or with no file) it reads null."""
    import bench
    f = tmp_path / "traffic.json"
    f.write_text(json.dumps({
        "gram": {"dense": {"source_hash": bench.kernel_source_hash("gram"),
                           "dram_bytes_per_launch": 123456}},
        "fake_quant": {"w4a4": {"source_hash": "0000000000000000",
                                "dram_bytes_per_launch": 7}},
    }))
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(f))
    assert bench.recorded_traffic("gram", "dense") == 123456
    assert bench.recorded_traffic("gram", "moe") is None
    assert bench.recorded_traffic("fake_quant", "w4a4") is None
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(tmp_path / "missing.json"))
    assert bench.recorded_traffic("gram", "dense") is None
