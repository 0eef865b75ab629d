"""The bench's reference arm runs on the host (the oracle, no GPU): its JSON
line carries the keys the benchmark contract asks for."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _line(args):
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py")] + args, capture_output=True, text=True,
                         timeout=600, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, out.stdout[-2000:]
    return json.loads(lines[0])


def test_reference_arm_line():
    d = _line(["--impl", "reference", "--steps", "1", "--warmup", "0"])
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
              "vs_baseline", "dtype", "data", "config", "impl", "cpu_baseline", "e2e", "gpu_launches"):
        assert k in d, k
    assert d["impl"] == "reference" and d["unit"] == "TFLOP/s" and d["value"] > 0
    assert d["config"]["workload"] == "prefill_2k"
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"] and cb["sample"]
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0



def test_traffic_records_follow_code_not_comments():
    """Recorded DRAM traffic is reported only while the kernel's code is the
    one it was measured on: the source hash ignores comments and blank lines
    but not code, string literals included."""
    sys.path.insert(0, ROOT)
    import bench
    base = 'int a = 1; // note\n/* block\n comment */\nconst char *s = "x//y";\n\n'
    assert bench._code_only(base) == bench._code_only(base.replace("// note", "// other note") + "\n\n// tail")
    assert bench._code_only(base) != bench._code_only(base.replace("a = 1", "a = 2"))
    assert bench._code_only(base) != bench._code_only(base.replace('"x//y"', '"x//z"'))
    assert '"x//y"' in bench._code_only(base)
    # a record is reported only while its hash is the kernel's current one
    with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
        records = json.load(f)
    for key, rec in records.items():
        kernel, workload = key.split(":")
        current = rec["sources"] == bench.kernel_sources_hash(kernel)
        assert bench.recorded_traffic(kernel, workload) == (rec["bytes_per_launch"] if current else None), key


class _FakeWorkload:
    name, kernel, unit, scale_unit, launches_per_step = "prefill_2k", "prefill_bf16_kernel", "TFLOP/s", 1e12, 1
    work = 4.0 * 4 * 16 * 128 * (2048 * 2049 // 2)


def test_roofline_fraction_uses_the_burst_peak_whatever_the_clocks():
    """frac is always against one fixed denominator (the measured burst bf16
    peak for tensor-bound kernels); the sustained-peak ratio is an extra
    field, even when the region's clocks show the power cap."""
    sys.path.insert(0, ROOT)
    import bench
    pk = {"bf16_tflops": 1635.2, "bf16_tflops_sustained": 1399.6, "hbm_gbs": 6535.7}
    capped = {"sm_mhz": 1300.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"]}
    for clocks in (None, capped):
        r = bench.roofline(_FakeWorkload(), 0.08594, pk, "measured", "tensor", clocks)
        assert r["peak"] == 1635.2
        assert abs(r["achieved"] - _FakeWorkload.work / 0.08594e-3 / 1e12) < 0.01
        assert abs(r["frac"] - r["achieved"] / 1635.2) < 1e-4
        assert abs(r["frac_of_sustained"] - r["achieved"] / 1399.6) < 1e-4
    # 68.75 GFLOP in 0.08594 ms: 800 TFLOP/s, 0.489 of the burst peak
    assert abs(r["achieved"] - 800.0) < 0.2 and abs(r["frac"] - 0.4892) < 2e-4


def test_timing_stats_median_and_spread():
    sys.path.insert(0, ROOT)
    import bench
    rep = [2.0, 2.2, 1.8, 2.0, 2.1, 1.9, 2.0, 5.0, 2.0, 2.0, 2.0]  # ms per replay of 4 steps, one outlier
    tm = {"rep_ms": rep, "total_ms": sum(rep), "span": (10.0, 11.5), "replays": len(rep), "steps": 4,
          "timing": "graph"}
    st = bench.timing_stats(tm)
    assert st["steps_timed"] == 44 and st["replays"] == 11 and st["region_s"] == 1.5
    ps = st["per_step_ms"]
    assert ps["median"] == 0.5 and ps["min"] == 0.45 and ps["max"] == 1.25
    assert abs(ps["mean"] - sum(rep) / 44) < 1e-5
    assert ps["p10"] <= ps["median"] <= ps["p90"]
