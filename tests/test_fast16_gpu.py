"""The N = 16 kernels (one CTA range per row, dt B discretisation, real A,
L a multiple of 8) against the fp64 oracle on shapes that cut their tiles
every way: a single row, an odd number of rows (a row pair with one live
row), one and several backward CTAs of 12 rows with a partial last one, L
shorter than one 256-token chunk, one 8-token segment past a chunk, and
document starts at chunk and segment edges. n_splits=1 selects them (the
automatic choice splits rows this short)."""
import numpy as np
import pytest

import oracle
import synth
from pipeline import device_inputs, gpu_layer, host64, rel_l2
from test_parity_gpu import _compare_all, _oracle_layer, _small

pytestmark = pytest.mark.gpu

FAST_CASES = [
    # B, D, L, document starts, dtype
    (1, 1, 8, 0, "f32"),
    (1, 2, 16, 1, "f32"),
    (2, 3, 264, 3, "f32"),
    (1, 12, 512, 4, "f32"),
    (2, 13, 1000, 5, "f32"),
    (1, 25, 2056, 9, "f32"),
    (2, 8, 776, 6, "bf16"),
    (1, 17, 1536, 0, "bf16"),
    (2, 24, 2048, 7, "bf16"),
]


@pytest.mark.parametrize("B,D,L,nb,dtype", FAST_CASES)
def test_fast16_layer_parity(B, D, L, nb, dtype):
    inp = _small(B, D, 16, L, 3000 + L + D, dtype=dtype, nbound=nb)
    res = gpu_layer(device_inputs(inp), n_splits=1)
    fp32 = dtype == "f32"
    want = _oracle_layer(inp, bf16_points=not fp32)
    _compare_all(res, want, fp32=fp32)


@pytest.mark.parametrize("use_z,softplus,noD", [(False, True, False), (True, False, False),
                                                 (False, False, True)])
def test_fast16_optional_inputs(use_z, softplus, noD):
    inp = _small(2, 7, 16, 520, 5550, nbound=3)
    if not softplus:  # the step is used as given: keep it positive
        inp.delta.f32 = np.abs(inp.delta.f32) * np.float32(0.2)
        inp.delta.f64 = inp.delta.f32.astype(np.float64)
        inp.delta_bias = np.zeros_like(inp.delta_bias)
    if noD:
        inp.Dskip = np.zeros_like(inp.Dskip)
    res = gpu_layer(device_inputs(inp), n_splits=1, use_z=use_z, softplus=softplus)
    want = _oracle_layer(inp, bf16_points=False, use_z=use_z, softplus=softplus)
    _compare_all(res, want, fp32=True, use_z=use_z)


def test_fast16_document_edges():
    B, D, N, L = 1, 5, 16, 520
    inp = _small(B, D, N, L, 77)
    seq = np.zeros((B, L), dtype=np.int32)
    doc = 0
    for t in range(L):  # 1-token documents at the start, at segment and chunk edges, and at the end
        if t in (1, 2, 3, 7, 8, 9, 15, 16, 255, 256, 257, 263, 264, 511, 512, 518, 519) or t % 41 == 0:
            doc += 1
        seq[0, t] = doc
    inp.seq_idx = seq
    res = gpu_layer(device_inputs(inp), n_splits=1)
    want = _oracle_layer(inp, bf16_points=False)
    _compare_all(res, want, fp32=True)


def test_fast16_matches_general_kernels():
    """The N = 16 kernels and the general ones (forced by n_splits=2) agree."""
    inp = _small(2, 10, 16, 1024, 4141, dtype="bf16", nbound=4)
    dv = device_inputs(inp)
    r1 = gpu_layer(dv, n_splits=1)
    r2 = gpu_layer(dv, n_splits=2)
    for k in ("out", "final_state", "du", "ddelta", "dz", "dA", "dB", "dC", "dD", "ddelta_bias",
              "dx"):
        assert rel_l2(host64(r1[k]), host64(r2[k])) <= 2e-3, k


def test_fast16_unaligned_gradient_buffers():
    import torch
    import selective_state_space_35_b200 as ssm
    B, D, N, L = 1, 5, 16, 512
    inp = _small(B, D, N, L, 808, dtype="bf16", nbound=2)
    dv = device_inputs(inp)
    u = ssm.conv1d_fwd(dv["x"], dv["conv_w"], dv["conv_b"], dv["seq_idx"])
    kw = dict(z=dv["z"], Dskip=dv["Dskip"], delta_bias=dv["delta_bias"], seq_idx=dv["seq_idx"],
              n_splits=1)
    _, _, ws = ssm.scan_fwd(u, dv["delta"], dv["A"], dv["Bm"], dv["Cm"], **kw)
    ref = ssm.scan_bwd(u, dv["delta"], dv["A"], dv["Bm"], dv["Cm"], dv["dout"], ws, **kw)
    n = B * N * L
    bufB = torch.empty(n + 1, dtype=torch.float32, device="cuda")
    bufC = torch.empty(n + 1, dtype=torch.float32, device="cuda")
    m = B * D * L
    bu = torch.empty(m + 1, dtype=torch.bfloat16, device="cuda")
    g = ssm.scan_bwd(u, dv["delta"], dv["A"], dv["Bm"], dv["Cm"], dv["dout"], ws,
                     grads={"dB": bufB[1:].view(B, N, L), "dC": bufC[1:].view(B, N, L),
                            "du": bu[1:].view(B, D, L)}, **kw)
    for k in ("dB", "dC", "du", "ddelta", "dz"):
        assert rel_l2(host64(g[k]), host64(ref[k])) <= 1e-6, k


def test_fast16_cu_seqlens_equals_seq_idx():
    import torch
    import selective_state_space_35_b200 as ssm
    B, D, N, L = 1, 6, 16, 776
    inp = _small(B, D, N, L, 91)
    cuts = [0, 1, 100, 256, 257, 600, 775, L]
    seq = np.zeros((1, L), dtype=np.int32)
    for i in range(len(cuts) - 1):
        seq[0, cuts[i]:cuts[i + 1]] = i
    inp.seq_idx = seq
    dv = device_inputs(inp)
    cu = torch.tensor(cuts, dtype=torch.int32, device="cuda")
    u = ssm.conv1d_fwd(dv["x"], dv["conv_w"], dv["conv_b"], dv["seq_idx"])
    kw = dict(z=dv["z"], Dskip=dv["Dskip"], delta_bias=dv["delta_bias"], n_splits=1)
    o1, f1, w1 = ssm.scan_fwd(u, dv["delta"], dv["A"], dv["Bm"], dv["Cm"], seq_idx=dv["seq_idx"],
                              return_final_state=True, **kw)
    o2, f2, w2 = ssm.scan_fwd(u, dv["delta"], dv["A"], dv["Bm"], dv["Cm"], cu_seqlens=cu,
                              return_final_state=True, **kw)
    assert torch.equal(o1, o2) and torch.equal(f1, f2)
    g1 = ssm.scan_bwd(u, dv["delta"], dv["A"], dv["Bm"], dv["Cm"], dv["dout"], w1,
                      seq_idx=dv["seq_idx"], **kw)
    g2 = ssm.scan_bwd(u, dv["delta"], dv["A"], dv["Bm"], dv["Cm"], dv["dout"], w2, cu_seqlens=cu,
                      **kw)
    for k in ("du", "ddelta", "dz", "dA", "dD", "ddelta_bias"):
        assert torch.equal(g1[k], g2[k]), k
    for k in ("dB", "dC"):
        assert rel_l2(host64(g2[k]), host64(g1[k])) <= 1e-6, k


def test_fast16_run_twice_bitwise():
    import torch
    inp = _small(2, 9, 16, 1200, 5, dtype="bf16", nbound=3)
    dv = device_inputs(inp)
    r1 = gpu_layer(dv, n_splits=1)
    r2 = gpu_layer(dv, n_splits=1)
    for k in ("u", "out", "final_state", "du", "ddelta", "dz", "dA", "dD", "ddelta_bias", "dx",
              "dconv_w", "dconv_b"):
        assert torch.equal(r1[k], r2[k]), k
