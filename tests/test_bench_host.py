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
