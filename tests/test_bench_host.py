"""bench.py's entry points exist and its CLI parses (no GPU needed)."""
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_bench_defines_every_measurement():
    sys.path.insert(0, ROOT)
    import bench
    for name in ("main", "e2e", "decode_bench", "run_reference", "oracle_sample", "Layer"):
        assert callable(getattr(bench, name)), name


def test_bench_help():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--help"],
                       capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stderr
    for flag in ("--gpus", "--steps", "--warmup", "--impl", "--no-e2e", "--no-decode"):
        assert flag in r.stdout


def test_reference_arm_prints_its_line_on_cpu():
    """--impl reference times the fp64 oracle on the host cores: one JSON line
    with the reference keys (here on the small bf16 layer, one step)."""
    import json
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--config", "2", "--steps", "1", "--warmup", "3"],
                       capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["value"] > 0 and line["dtype"] == "f64"
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["value"] == line["value"]
    assert line["e2e"] == {"value": line["value"], "unit": line["unit"], "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}
    assert line["config"]["L"] == 2048


def test_bench_rejects_the_parity_only_config():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--config", "1"],
                       capture_output=True, text=True, timeout=120)
    assert r.returncode != 0 and "invalid choice" in r.stderr
