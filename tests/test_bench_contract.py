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
