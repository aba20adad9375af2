"""The boundary is a plain C ABI: a C99 program (and the same source as
C++17) includes include/ssmscan.h with warnings as errors, links
libssmscan.so directly and exercises calls that need no GPU (version,
workspace size, argument errors and their message)."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "selective_state_space_35_b200")

SRC = r"""
#include <stdio.h>
#include <string.h>
#include "ssmscan.h"
int main(void) {
    if (ssm_abi_version() != SSM_ABI_VERSION) { printf("version\n"); return 1; }
    ssm_scan_params p;
    memset(&p, 0, sizeof p);
    p.struct_size = sizeof p;
    p.B = 2; p.D = 8; p.L = 1000; p.N = 16; p.dtype = SSM_DTYPE_BF16; p.delta_softplus = 1;
    size_t bytes = 0;
    if (ssm_scan_workspace_size(&p, &bytes) != SSM_OK || bytes == 0) { printf("size\n"); return 2; }
    p.struct_size = 3;
    if (ssm_scan_workspace_size(&p, &bytes) != SSM_ERR_INVALID_ARG) { printf("struct\n"); return 3; }
    if (strlen(ssm_last_error()) == 0) { printf("message\n"); return 4; }
    if (ssm_state_carry(NULL, NULL, 1, 0, 0, NULL, NULL, NULL, 0, NULL, 1, 1, 1, NULL)
        != SSM_ERR_INVALID_ARG) { printf("carry\n"); return 5; }
    printf("ok\n");
    return 0;
}
"""


@pytest.mark.parametrize("compiler,std", [("gcc", "-std=c99"), ("g++", "-std=c++17")])
def test_header_compiles_and_links_from_c(tmp_path, compiler, std):
    if shutil.which(compiler) is None:
        pytest.skip(f"{compiler} not available")
    from selective_state_space_35_b200 import _lib, build
    try:
        build.nvcc()
        have_nvcc = True
    except RuntimeError:
        have_nvcc = False
    if have_nvcc:
        build.build()
    elif not os.path.exists(_lib.LIB_PATH):
        pytest.skip("neither nvcc nor a prebuilt libssmscan.so is available")
    src = tmp_path / ("t.c" if compiler == "gcc" else "t.cpp")
    src.write_text(SRC)
    exe = tmp_path / "t"
    subprocess.run([compiler, std, "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"),
                    str(src), "-o", str(exe), "-L", PKG, "-lssmscan", f"-Wl,-rpath,{PKG}"],
                   check=True, capture_output=True, text=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True)
    assert r.returncode == 0 and r.stdout.strip() == "ok", (r.returncode, r.stdout, r.stderr)
