"""Host-side checks of the C ABI: the library loads, exports every function
include/ssmscan.h declares, and rejects bad arguments before any launch.
No GPU is needed: every call here returns before touching the device."""
import ctypes
import os
import re
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "ssmscan.h")


@pytest.fixture(scope="module")
def ssm():
    from selective_state_space_35_b200 import build
    build.build()
    import selective_state_space_35_b200 as m
    m.load()
    return m


def _declared():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(ssm_[a-z0-9_]+)\s*\(", src)))


def test_header_declares_expected_entry_points():
    names = _declared()
    for n in ("ssm_conv1d_fwd", "ssm_conv1d_bwd", "ssm_conv1d_bwd_workspace_size",
              "ssm_scan_workspace_size", "ssm_scan_fwd", "ssm_scan_bwd", "ssm_last_error",
              "ssm_abi_version", "ssm_decode_step", "ssm_scan_status"):
        assert n in names


def test_library_exports_every_declared_symbol(ssm):
    from selective_state_space_35_b200 import _lib
    out = subprocess.run(["nm", "-D", "--defined-only", _lib.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\bT (ssm_\w+)", out))
    missing = [n for n in _declared() if n not in exported]
    assert not missing, missing
    lib = ctypes.CDLL(_lib.LIB_PATH)
    for n in _declared():
        assert hasattr(lib, n), n


def test_abi_version(ssm):
    src = open(HEADER).read()
    v = int(re.search(r"#define SSM_ABI_VERSION (\d+)", src).group(1))
    assert ssm.ssm_abi_version() == v


def _params(ssm, **kw):
    p = ssm.ssm_scan_params()
    p.struct_size = ctypes.sizeof(ssm.ssm_scan_params)
    p.B, p.D, p.L, p.N = 2, 8, 1000, 16
    p.dtype = 1
    p.delta_softplus = 1
    for k, v in kw.items():
        setattr(p, k, v)
    return p


def test_workspace_size_layout(ssm):
    nchunks = (1000 + 255) // 256
    # N = 16, one range per row, L % 8 == 0: the state entering every 8-token
    # segment (8 bytes per token and row) and B / C packed per chunk (32 KB)
    p = _params(ssm, n_splits=1)
    n1 = ssm.ssm_scan_workspace_size(p)
    assert n1 >= 2 * 8 * nchunks * 256 * 8 + 2 * nchunks * 32768
    # with a gate, y before the gate is kept for the backward (bf16 here)
    assert ssm.ssm_scan_workspace_size(_params(ssm, n_splits=1, z=1 << 20)) >= n1 + 2 * 8 * 1000 * 2
    # other cases: the state entering every 16-token block, and split carries
    p8 = _params(ssm, n_splits=1, N=8)
    n8 = ssm.ssm_scan_workspace_size(p8)
    assert n8 >= 2 * 8 * nchunks * 16 * 16 * 4
    assert ssm.ssm_scan_workspace_size(_params(ssm, n_splits=3, N=8)) > n8
    # a length that is not a multiple of 8 takes the general kernels too
    assert ssm.ssm_scan_workspace_size(_params(ssm, n_splits=1, L=1001)) < n1 + 2 * 8 * 8
    assert ssm.ssm_conv1d_bwd_workspace_size(2, 8, 1000, 4) >= 2 * 8 * 5 * 4


@pytest.mark.parametrize("field,value,status", [
    ("struct_size", 3, 1), ("B", 0, 1), ("N", 17, 2), ("N", 0, 1), ("dtype", 7, 1),
    ("n_splits", -1, 1), ("discretization", 2, 1), ("state_complex", 2, 1),
])
def test_scan_param_validation(ssm, field, value, status):
    from selective_state_space_35_b200 import _lib
    p = _params(ssm, **{field: value})
    n = ctypes.c_size_t(0)
    st = _lib.load().ssm_scan_workspace_size(ctypes.byref(p), ctypes.byref(n))
    assert st == status
    assert ssm.ssm_last_error()


def test_scan_fwd_rejects_null_and_small_workspace(ssm):
    from selective_state_space_35_b200 import _lib
    p = _params(ssm)
    assert ssm.ssm_scan_fwd(p, None) == _lib.SSM_ERR_INVALID_ARG  # null inputs
    fake = 1 << 20  # never dereferenced: validation fails first
    p = _params(ssm, u=fake, delta=fake, A=fake, Bm=fake, Cm=fake, out=fake, workspace=fake,
                workspace_bytes=16)
    assert ssm.ssm_scan_fwd(p, None) == _lib.SSM_ERR_INVALID_ARG
    assert "workspace" in ssm.ssm_last_error()
    p = _params(ssm, u=fake, delta=fake, A=fake, Bm=fake, Cm=fake, out=fake, workspace=fake + 8,
                workspace_bytes=1 << 30)
    assert ssm.ssm_scan_fwd(p, None) == _lib.SSM_ERR_INVALID_ARG
    assert "aligned" in ssm.ssm_last_error()


def test_cu_seqlens_rules(ssm):
    from selective_state_space_35_b200 import _lib
    fake = 1 << 20
    p = _params(ssm, seq_idx=fake, cu_seqlens=fake, n_docs=2)
    n = ctypes.c_size_t(0)
    assert _lib.load().ssm_scan_workspace_size(ctypes.byref(p), ctypes.byref(n)) == 1
    p = _params(ssm, cu_seqlens=fake, n_docs=2)  # B=2
    assert _lib.load().ssm_scan_workspace_size(ctypes.byref(p), ctypes.byref(n)) == 1
    p = _params(ssm, B=1, cu_seqlens=fake, n_docs=0)
    assert _lib.load().ssm_scan_workspace_size(ctypes.byref(p), ctypes.byref(n)) == 1


def test_conv_validation(ssm):
    fake = ctypes.c_void_p(1 << 20)
    assert ssm.ssm_conv1d_fwd(None, fake, None, None, fake, 1, 1, 8, 4, 1, 1, None) == 1
    assert ssm.ssm_conv1d_fwd(fake, fake, None, None, fake, 1, 1, 8, 4, 1, 1, None) == 1  # u aliases x
    other = ctypes.c_void_p((1 << 20) + 4096)
    assert ssm.ssm_conv1d_fwd(fake, fake, None, None, other, 1, 1, 8, 3, 1, 1, None) == 2  # W=3
    assert ssm.ssm_conv1d_fwd(fake, fake, None, None, other, 1, 0, 8, 4, 1, 1, None) == 1
    assert ssm.ssm_conv1d_bwd(fake, fake, None, None, fake, other, fake, None, 1, 1, 8, 4, 1, 1,
                              None, 0, None) == 1  # workspace missing


def test_fault_injection_is_host_only():
    code = r"""
import ctypes, os, sys
sys.path.insert(0, %r)
os.environ["SSM_INJECT_FAIL"] = "ssm_scan_fwd,ssm_conv1d_fwd"
import selective_state_space_35_b200 as ssm
p = ssm.ssm_scan_params()
p.struct_size = ctypes.sizeof(p)
assert ssm.ssm_scan_fwd(p, None) == 5, ssm.ssm_last_error()
assert "injected" in ssm.ssm_last_error()
assert ssm.ssm_conv1d_fwd(None, None, None, None, None, 1, 1, 1, 4, 1, 1, None) == 5
# not named: normal validation
assert ssm.ssm_scan_bwd(p, None, None) == 1
""" % ROOT
    r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr


def test_binding_rejects_cpu_tensors(ssm):
    torch = pytest.importorskip("torch")
    x = torch.zeros(1, 2, 8, dtype=torch.bfloat16)
    w = torch.zeros(2, 4)
    with pytest.raises(ValueError):
        ssm.conv1d_fwd(x, w)


def _decode_params(ssm, **kw):
    fake = 1 << 20
    p = ssm.ssm_decode_params()
    p.struct_size = ctypes.sizeof(ssm.ssm_decode_params)
    p.B, p.D, p.N, p.W = 2, 8, 16, 4
    p.dtype = 1
    p.delta_softplus = 1
    p.x, p.conv_state, p.conv_w, p.delta = fake, fake + 4096, fake + 8192, fake + 12288
    p.Bm, p.Cm, p.A, p.state = fake + 16384, fake + 20480, fake + 24576, fake + 28672
    p.out = fake + 32768
    for k, v in kw.items():
        setattr(p, k, v)
    return p


@pytest.mark.parametrize("field,value,status", [
    ("struct_size", 3, 1), ("B", 0, 1), ("D", 0, 1), ("N", 0, 1), ("N", 17, 2), ("W", 3, 2),
    ("dtype", 7, 1), ("x", None, 1), ("state", None, 1), ("out", None, 1),
    ("out", 1 << 20, 1),            # aliases x
    ("state", (1 << 20) + 2, 1),    # fp32 state misaligned
    ("x", (1 << 20) + 1, 1),        # bf16 activation misaligned
])
def test_decode_param_validation(ssm, field, value, status):
    """Every check fails before a launch (the fake pointers are never touched)."""
    p = _decode_params(ssm, **{field: value})
    assert ssm.ssm_decode_step(p, None) == status
    assert ssm.ssm_last_error()


def test_decode_null_params(ssm):
    assert ssm.ssm_decode_step(None, None) == 1


def test_grads_struct_has_initial_state_gradient(ssm):
    names = [f[0] for f in ssm.ssm_scan_grads._fields_]
    assert names[-4:] == ["dinitial_state", "dfinal_state", "workspace", "workspace_bytes"]
    assert [f[0] for f in ssm.ssm_scan_params._fields_][-3:] == ["initial_state", "discretization",
                                                                 "state_complex"]


def test_fused_forward_validation(ssm):
    from selective_state_space_35_b200 import _lib
    fake = 1 << 20
    p = _params(ssm, u=fake, delta=fake + 4096, A=fake + 8192, Bm=fake + 12288, Cm=fake + 16384,
                out=fake + 20480, workspace=fake + 65536, workspace_bytes=1 << 30)
    L = _lib.load()
    assert L.ssm_conv1d_scan_fwd(ctypes.byref(p), None, fake, None, None) == 1     # no x
    assert L.ssm_conv1d_scan_fwd(ctypes.byref(p), fake + 40960, None, None, None) == 1  # no w
    assert L.ssm_conv1d_scan_fwd(ctypes.byref(p), fake, fake + 40960, None, None) == 1  # x == u
    assert "alias" in ssm.ssm_last_error()
    assert L.ssm_conv1d_scan_fwd(ctypes.byref(p), fake + 40961, fake + 44000, None, None) == 1


def test_complex_a_rules(ssm):
    """Complex A: dt B discretisation and one CTA per row only, doubled
    checkpoints, 8-byte aligned A / states, not fused with the conv."""
    from selective_state_space_35_b200 import _lib
    L = _lib.load()
    n = ctypes.c_size_t(0)
    for kw, status in [(dict(discretization=1), 2), (dict(n_splits=2), 2),
                       (dict(n_splits=1), 0), (dict(n_splits=0), 0)]:
        p = _params(ssm, state_complex=1, **kw)
        assert L.ssm_scan_workspace_size(ctypes.byref(p), ctypes.byref(n)) == status, kw
    real = ssm.ssm_scan_workspace_size(_params(ssm, n_splits=1, N=8))
    cplx = ssm.ssm_scan_workspace_size(_params(ssm, state_complex=1, N=8))
    nchunks = (1000 + 255) // 256
    assert cplx >= real + 2 * 8 * nchunks * 16 * 16 * 4  # (re, im) checkpoints
    fake = 1 << 20
    good = dict(u=fake, delta=fake + 4096, A=fake + 8192, Bm=fake + 12288, Cm=fake + 16384,
                out=fake + 20480, workspace=fake + 65536, workspace_bytes=1 << 30, state_complex=1)
    p = _params(ssm, **dict(good, A=fake + 8196))   # 4-byte but not 8-byte aligned
    assert L.ssm_scan_fwd(ctypes.byref(p), None) == 1
    assert "8-byte" in ssm.ssm_last_error()
    p = _params(ssm, **good)
    assert L.ssm_conv1d_scan_fwd(ctypes.byref(p), fake + (1 << 24), fake, None, None) == 2


def test_piece_calls_validation(ssm):
    """Summaries, carry and conv halos reject bad arguments before any launch."""
    from selective_state_space_35_b200 import _lib
    L = _lib.load()
    fake = 1 << 20
    good = dict(u=fake, delta=fake + 4096, A=fake + 8192, Bm=fake + 12288, Cm=fake + 16384,
                out=fake + 20480, workspace=fake + 65536, workspace_bytes=1 << 30)
    dec, val = fake + (1 << 22), fake + (1 << 23)
    p = _params(ssm, **dict(good, state_complex=1))
    assert L.ssm_scan_fwd_summary(ctypes.byref(p), None, dec, val, None) == 2
    p = _params(ssm, **good)
    assert L.ssm_scan_fwd_summary(ctypes.byref(p), None, None, val, None) == 1
    assert L.ssm_scan_bwd_summary(ctypes.byref(p), None, None, dec, val, None) == 1   # no dout
    p = _params(ssm, **dict(good, workspace_bytes=16))
    assert L.ssm_scan_fwd_summary(ctypes.byref(p), None, dec, val, None) == 1
    assert "workspace" in ssm.ssm_last_error()
    # carry: r outside [0, R), bad direction, aliasing
    assert L.ssm_state_carry(dec, val, 2, 2, 0, None, None, None, 0, fake, 2, 8, 16, None) == 1
    assert L.ssm_state_carry(dec, val, 2, 1, 3, None, None, None, 0, fake, 2, 8, 16, None) == 1
    assert L.ssm_state_carry(dec, val, 2, 1, 0, None, None, None, 0, dec, 2, 8, 16, None) == 1
    # conv halos: ids needed with a segmented row, x_next and du_next together
    x, w, u = fake, fake + 4096, fake + 8192
    assert L.ssm_conv1d_fwd_ctx(x, w, None, fake + 12288, fake + 16384, None, u, 2, 8, 64, 4, 1, 1,
                                None) == 1
    assert L.ssm_conv1d_bwd_ctx(x, w, None, None, None, None, fake + 16384, None, None, fake, u,
                                fake + 20480, None, 2, 8, 64, 4, 1, 1, fake + 65536, 1 << 20,
                                None) == 1
    assert L.ssm_conv1d_bwd_ctx(x, w, None, fake + 12288, None, None, fake + 16384, fake + 24576,
                                None, fake, u, fake + 20480, None, 2, 8, 64, 4, 1, 1,
                                fake + 65536, 1 << 20, None) == 1


def _grads(ssm, **kw):
    g = ssm.ssm_scan_grads()
    g.struct_size = ctypes.sizeof(ssm.ssm_scan_grads)
    for k, v in kw.items():
        setattr(g, k, v)
    return g


def test_deterministic_backward_workspace(ssm):
    """deterministic = 1 needs (channel groups) x (dB, dC) x B x N x L fp32
    partial sums: groups of 12 rows on the N = 16 kernels, 8 on the others,
    both planes for a complex A; 0 bytes otherwise; other values rejected."""
    from selective_state_space_35_b200 import _lib
    L = _lib.load()
    up = lambda x: (x + 255) // 256 * 256
    assert ssm.ssm_scan_bwd_workspace_size(_params(ssm, n_splits=1), _grads(ssm)) == 0
    for kw, groups, planes in [(dict(n_splits=1, D=30), 3, 1),
                               (dict(n_splits=1, D=30, N=8), 4, 1),
                               (dict(n_splits=2, D=30), 4, 1),
                               (dict(n_splits=1, D=30, L=1001), 4, 1),
                               (dict(n_splits=1, D=30, N=8, state_complex=1), 4, 2)]:
        p = _params(ssm, **kw)
        want = up(groups * 2 * p.B * p.N * planes * p.L * 4)
        assert ssm.ssm_scan_bwd_workspace_size(p, _grads(ssm, deterministic=1)) == want, kw
    n = ctypes.c_size_t(0)
    p = _params(ssm, n_splits=1)
    g = _grads(ssm, deterministic=2)
    assert L.ssm_scan_bwd_workspace_size(ctypes.byref(p), ctypes.byref(g), ctypes.byref(n)) == 1
    fake = 1 << 20
    p = _params(ssm, u=fake, delta=fake + 4096, A=fake + 8192, Bm=fake + 12288, Cm=fake + 16384,
                out=fake + 20480, workspace=fake + 65536, workspace_bytes=1 << 30, n_splits=1)
    g = _grads(ssm, dout=fake, du=fake, ddelta=fake, dA=fake, dB=fake, dC=fake, deterministic=1)
    assert L.ssm_scan_bwd(ctypes.byref(p), ctypes.byref(g), None) == 1  # no scratch given
    assert "grads.workspace" in ssm.ssm_last_error()
    g.workspace, g.workspace_bytes = fake + (1 << 24), 1000
    assert L.ssm_scan_bwd(ctypes.byref(p), ctypes.byref(g), None) == 1  # too small
    g.workspace, g.workspace_bytes = fake + (1 << 24) + 16, 1 << 30
    assert L.ssm_scan_bwd(ctypes.byref(p), ctypes.byref(g), None) == 1  # misaligned
    assert "aligned" in ssm.ssm_last_error()


def test_ssd_param_validation(ssm):
    """ssm_ssd_fwd rejects bad arguments before any launch: struct size, sizes,
    groups that do not divide the heads, fp32 storage, P / N other than 64 /
    128, NULL and misaligned pointers."""
    from selective_state_space_35_b200 import _lib
    L = _lib.load()
    fake = 1 << 20

    def params(**kw):
        p = ssm.ssm_ssd_params()
        p.struct_size = ctypes.sizeof(ssm.ssm_ssd_params)
        p.B, p.L, p.H, p.P, p.G, p.N = 1, 256, 4, 64, 2, 128
        p.dtype = 1
        p.x, p.dt_raw, p.A, p.Bm, p.Cm, p.y = fake, fake + 4096, fake + 8192, fake + 12288, \
            fake + 16384, fake + 20480
        p.dt_softplus = 1
        for k, v in kw.items():
            setattr(p, k, v)
        return p

    for kw, status in [(dict(struct_size=3), 1), (dict(B=0), 1), (dict(G=3), 1), (dict(dtype=0), 2),
                       (dict(P=32), 2), (dict(N=64), 2), (dict(x=None), 1), (dict(y=fake + 8), 1),
                       (dict(A=fake + 2), 1)]:
        p = params(**kw)
        assert L.ssm_ssd_fwd(ctypes.byref(p), None) == status, kw
        assert ssm.ssm_last_error()


def test_ssd_bwd_param_validation(ssm):
    """ssm_ssd_bwd rejects bad arguments before any launch: the forward's
    checks, a missing chunk_states, grads struct size, NULL and misaligned
    gradient pointers; and a misaligned chunk_states in the forward."""
    from selective_state_space_35_b200 import _lib
    L = _lib.load()
    fake = 1 << 20

    def params(**kw):
        p = ssm.ssm_ssd_params()
        p.struct_size = ctypes.sizeof(ssm.ssm_ssd_params)
        p.B, p.L, p.H, p.P, p.G, p.N = 1, 256, 4, 64, 2, 128
        p.dtype = 1
        p.x, p.dt_raw, p.A, p.Bm, p.Cm = fake, fake + 4096, fake + 8192, fake + 12288, fake + 16384
        p.chunk_states = fake + 65536
        p.dt_softplus = 1
        for k, v in kw.items():
            setattr(p, k, v)
        return p

    def grads(**kw):
        g = ssm.ssm_ssd_grads()
        g.struct_size = ctypes.sizeof(ssm.ssm_ssd_grads)
        g.dy, g.dx, g.ddt_raw, g.dA, g.dB, g.dC = (fake + 1024 * i for i in range(40, 46))
        for k, v in kw.items():
            setattr(g, k, v)
        return g

    cases = [(dict(), dict(struct_size=5), 1), (dict(), dict(dy=None), 1), (dict(), dict(dB=fake + 4), 1),
             (dict(), dict(ddt_raw=fake + 2), 1), (dict(chunk_states=None), dict(), 1),
             (dict(chunk_states=fake + 8), dict(), 1), (dict(P=32), dict(), 2), (dict(G=3), dict(), 1)]
    for pkw, gkw, status in cases:
        p, g = params(**pkw), grads(**gkw)
        assert L.ssm_ssd_bwd(ctypes.byref(p), ctypes.byref(g), None) == status, (pkw, gkw)
        assert ssm.ssm_last_error()
    assert L.ssm_ssd_bwd(ctypes.byref(params()), None, None) == 1
    p = params(y=fake + 20480, chunk_states=fake + 8)
    assert L.ssm_ssd_fwd(ctypes.byref(p), None) == 1
    assert "aligned" in ssm.ssm_last_error()


def test_release_build_has_no_debug_checks(ssm):
    # the release library answers both debug calls before touching the device
    with pytest.raises(ssm.SsmError) as e:
        ssm.debug_report()
    assert e.value.status == 2  # SSM_ERR_UNSUPPORTED
    assert ssm.ssm_debug_selftest(None, 1, None) == 2


def test_debug_library_builds_with_every_symbol():
    """The -DSSM_DEBUG build compiles, exports what the header declares and
    carries the checks (its report asks the device instead of refusing)."""
    from selective_state_space_35_b200 import build
    try:
        lib_path = build.build_debug()
    except RuntimeError as err:  # no nvcc on this machine
        pytest.skip(str(err))
    lib = ctypes.CDLL(lib_path)
    for n in _declared():
        assert hasattr(lib, n), n
    from selective_state_space_35_b200 import _lib
    info = _lib.ssm_debug_info()
    info.struct_size = ctypes.sizeof(_lib.ssm_debug_info)
    lib.ssm_debug_report.restype = ctypes.c_int
    lib.ssm_debug_report.argtypes = [ctypes.POINTER(_lib.ssm_debug_info), ctypes.c_int]
    st = lib.ssm_debug_report(ctypes.byref(info), 0)
    assert st in (0, 3), st  # 0 with a device, SSM_ERR_CUDA without one; never unsupported
    bad = _lib.ssm_debug_info()
    bad.struct_size = 1
    assert lib.ssm_debug_report(ctypes.byref(bad), 0) == 1
