"""Host logic of bench.py (no GPU): the reference arm's JSON line and the
roofline arithmetic."""
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


def _run(R, C, blocks):
    L = types.SimpleNamespace(R=R, C=C)
    return types.SimpleNamespace(layers=[L], blocks=lambda: blocks)


def test_roofline_local_hessian_counts_the_evaluations_made():
    import bench
    pk = {"sm_max_mhz": 1965.0, "hbm_gbs": 6555.5}
    run = _run(4096, 4096, 1 << 20)
    evals = 30.0 * (1 << 20)
    r = bench.make_roofline(run, {"search_lh": {"ms": 0.5}}, pk, "measured", "dense", evals)
    peak = 148 * 128 * 2 * 1965e6 / 1e12
    assert r["bound"] == "alu" and r["unit"] == "TFLOP/s"
    assert abs(r["peak"] - round(peak, 2)) < 1e-9
    assert abs(r["achieved"] - round(544 * evals / 0.5e-3 / 1e12, 2)) < 1e-9
    assert abs(r["frac"] - round(r["achieved"] / r["peak"], 4)) < 2e-4
    assert r["evaluated_per_block"] == 30.0


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
