"""Device index checks of the debug build (the library compiled with
-DSSM_DEBUG, selected through SSM_LIBRARY).

The GPU parity tests run once more in a child process against the debug
library with SSM_DEBUG_CHECKS=1; conftest then asserts after every test that
no kernel access left the range its shapes give it. The selftest shows that
a failing check is recorded and its access redirected, without a fault."""
import os
import re
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

# every GPU test file but the whole-config sizes (slow under the debug build)
DEBUG_SUITE = ["tests/test_parity_gpu.py", "tests/test_fast16_gpu.py", "tests/test_deterministic_gpu.py",
               "tests/test_recurrent_gpu.py", "tests/test_fused_gpu.py", "tests/test_zoh_gpu.py",
               "tests/test_complex_gpu.py", "tests/test_cp_gpu.py", "tests/test_ssd_gpu.py",
               "tests/test_debug_gpu.py::test_selftest_is_recorded"]


def _inside_debug_run() -> bool:
    return os.environ.get("SSM_DEBUG_CHECKS") == "1"


@pytest.mark.gpu
def test_gpu_suite_passes_the_index_checks():
    if _inside_debug_run():
        pytest.skip("the child process itself")
    from selective_state_space_35_b200 import build
    env = dict(os.environ, SSM_LIBRARY=build.build_debug(), SSM_DEBUG_CHECKS="1")
    r = subprocess.run([sys.executable, "-m", "pytest", *DEBUG_SUITE, "-m", "gpu", "-x", "-q",
                        "-k", "not full_size", "-p", "no:cacheprovider"],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=1800)
    assert r.returncode == 0, r.stdout[-4000:] + r.stderr[-2000:]
    summary = r.stdout.strip().splitlines()[-1]
    print("debug-build run:", summary)
    m = re.search(r"(\d+) passed", summary)
    assert m and int(m.group(1)) >= 100, summary  # the parity files ran, not an empty selection


@pytest.mark.gpu
def test_selftest_is_recorded():
    if not _inside_debug_run():
        pytest.skip("runs in the debug-library child process")
    import torch

    import selective_state_space_35_b200 as ssm
    ssm.debug_report(reset=True)
    buf = torch.zeros(7, dtype=torch.float32, device="cuda")
    ssm.debug_selftest(buf)
    rep = ssm.debug_report(reset=True)
    assert rep == dict(failures=1, site=1, site_name="debug selftest", offset=7, count=1, extent=7)
    assert buf[0].item() == 1.0 and int(torch.count_nonzero(buf[1:])) == 0
    assert ssm.debug_report()["failures"] == 0
