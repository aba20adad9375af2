"""Deterministic backward (grads.deterministic = 1): dB and dC are summed over
channel groups in a fixed order instead of with atomic adds, so two runs on the
same inputs give the same bits in every gradient. Checked on each backward
kernel (N = 16 kernels, the general ones with one and two time ranges per row,
the complex-A kernels) and against the fp64 oracle."""
import numpy as np
import pytest

import oracle
import synth
from pipeline import TOL_F32, f32_dev, host64, rel_l2, to_dev
from test_parity_gpu import _small

pytestmark = pytest.mark.gpu

KEYS = ("du", "ddelta", "dz", "dA", "dB", "dC", "dD", "ddelta_bias", "dinitial_state")


def _run(dv, *, n_splits, deterministic, complex_a=False):
    import selective_state_space_35_b200 as ssm
    kw = dict(z=dv["z"], Dskip=dv["Dskip"], delta_bias=dv["delta_bias"], seq_idx=dv["seq_idx"],
              n_splits=n_splits)
    _, _, ws = ssm.scan_fwd(dv["u"], dv["delta"], dv["A"], dv["Bm"], dv["Cm"], **kw)
    return ssm.scan_bwd(dv["u"], dv["delta"], dv["A"], dv["Bm"], dv["Cm"], dv["dout"], ws,
                        deterministic=deterministic, **kw)


def _real_inputs(B, D, N, L, seed, dtype):
    import torch
    inp = _small(B, D, N, L, seed, dtype=dtype, nbound=4)
    dev = "cuda"
    dv = {"u": to_dev(inp.x, dev), "delta": to_dev(inp.delta, dev), "z": to_dev(inp.z, dev),
          "Bm": to_dev(inp.Bm, dev), "Cm": to_dev(inp.Cm, dev), "dout": to_dev(inp.dout, dev),
          "A": f32_dev(inp.A, dev), "Dskip": f32_dev(inp.Dskip, dev),
          "delta_bias": f32_dev(inp.delta_bias, dev),
          "seq_idx": torch.from_numpy(np.ascontiguousarray(inp.seq_idx)).to(dev)}
    return inp, dv


def _bitwise_equal(r1, r2):
    import torch
    for k in KEYS:
        if r1.get(k) is None:
            continue
        assert torch.equal(r1[k], r2[k]), k


@pytest.mark.parametrize("B,D,N,L,n_splits,dtype", [
    (2, 30, 16, 1000, 1, "f32"),    # N = 16 kernels: 3 groups of 12 rows, the last partial
    (2, 30, 16, 1000, 2, "f32"),    # general kernels, two time ranges per row
    (1, 21, 5, 777, 1, "f32"),      # general kernels, N < 16, ragged L
    (2, 40, 16, 2048, 1, "bf16"),
])
def test_deterministic_real_a(B, D, N, L, n_splits, dtype):
    import torch
    inp, dv = _real_inputs(B, D, N, L, 6100 + D + L, dtype)
    r1 = _run(dv, n_splits=n_splits, deterministic=True)
    r2 = _run(dv, n_splits=n_splits, deterministic=True)
    ra = _run(dv, n_splits=n_splits, deterministic=False)
    torch.cuda.synchronize()
    _bitwise_equal(r1, r2)
    for k in ("dB", "dC"):  # the atomic order only moves the last bits
        assert rel_l2(host64(r1[k]), host64(ra[k])) <= 1e-6, k
    for k in ("du", "ddelta", "dz", "dA", "dD", "ddelta_bias"):
        assert torch.equal(r1[k], ra[k]), k
    if dtype == "f32":
        kw = dict(z=inp.z.f64, Dskip=inp.Dskip, delta_bias=inp.delta_bias, softplus=True,
                  seq_idx=inp.seq_idx, nthreads=8)
        g = oracle.scan_bwd(inp.x.f64, inp.delta.f64, inp.A, inp.Bm.f64, inp.Cm.f64,
                            inp.dout.f64, **kw)
        for k in ("dB", "dC", "dA"):
            assert rel_l2(host64(r1[k]), g[k]) <= TOL_F32, k


def test_deterministic_complex_a():
    import torch
    import selective_state_space_35_b200 as ssm
    B, D, N, L = 2, 19, 8, 600
    seed = 6301
    seq = synth.random_segments(np.random.Generator(np.random.PCG64(seed)), B, L, 3)
    ci = synth.complex_inputs(B, D, N, L, "f32", seed, seq_idx=seq, with_h0=False)
    dev = "cuda"
    u, dl, dout, z = (to_dev(ci.u, dev), to_dev(ci.delta, dev), to_dev(ci.dout, dev),
                      to_dev(ci.z, dev))
    Bm, Cm, A = to_dev(ci.Bm, dev), to_dev(ci.Cm, dev), f32_dev(ci.A, dev)
    kw = dict(z=z, Dskip=f32_dev(ci.Dskip, dev), delta_bias=f32_dev(ci.delta_bias, dev),
              seq_idx=torch.from_numpy(ci.seq_idx).to(dev))
    _, _, ws = ssm.scan_fwd(u, dl, A, Bm, Cm, **kw)
    r1 = ssm.scan_bwd(u, dl, A, Bm, Cm, dout, ws, deterministic=True, **kw)
    r2 = ssm.scan_bwd(u, dl, A, Bm, Cm, dout, ws, deterministic=True, **kw)
    ra = ssm.scan_bwd(u, dl, A, Bm, Cm, dout, ws, **kw)
    torch.cuda.synchronize()
    _bitwise_equal(r1, r2)
    for k in ("dB", "dC"):
        assert rel_l2(host64(r1[k]), host64(ra[k])) <= 1e-6, k
    Ac = ci.A[..., 0] + 1j * ci.A[..., 1]
    Bc = ci.Bm.f64[:, :, 0] + 1j * ci.Bm.f64[:, :, 1]
    Cc = ci.Cm.f64[:, :, 0] + 1j * ci.Cm.f64[:, :, 1]
    g = oracle.cscan_bwd(ci.u.f64, ci.delta.f64, Ac, Bc, Cc, ci.dout.f64, z=ci.z.f64,
                         Dskip=ci.Dskip, delta_bias=ci.delta_bias, seq_idx=ci.seq_idx)
    for k in ("dB", "dC"):
        assert rel_l2(host64(r1[k]), np.stack([g[k].real, g[k].imag], axis=2)) <= TOL_F32, k


def test_deterministic_repeat_many():
    """Ten runs of the N = 16 backward at several CTAs per row group give one
    result, bit for bit."""
    import torch
    _, dv = _real_inputs(1, 64, 16, 4096, 6402, "bf16")
    ref = _run(dv, n_splits=1, deterministic=True)
    for _ in range(9):
        _bitwise_equal(ref, _run(dv, n_splits=1, deterministic=True))
    torch.cuda.synchronize()
