"""Complex diagonal A (S4D form) on the GPU against the fp64 oracle on the
same seeded inputs: forward (out, final state) and every gradient (dA, dB,
dC and the initial-state gradient as (re, im) pairs). Cases span several
16-token blocks with a ragged tail, N < 16, channel counts that leave part of
a CTA idle, document resets, with and without the gate."""
import numpy as np
import pytest

import oracle
import synth
from pipeline import (TOL_BF16_OUT, TOL_BF16_OUT_MAX, TOL_F32, TOL_GRAD, bf16_out_max_abs_ok, f32_dev, host64,
                      rel_l2, to_dev)

pytestmark = pytest.mark.gpu

# fp32 inputs: the same bound as the real scan. The kernels compute e^{i theta}
# to about 1 ulp (quadrant reduction + Taylor series) and dt with the accurate
# library softplus, since the phase dt Im A magnifies dt's error by |Im A|.
TOL_C32 = TOL_F32


def _cplx_planes(a):
    a = np.asarray(a, dtype=np.float64)
    return a[:, :, 0] + 1j * a[:, :, 1]


def _cplx_pairs(a):
    a = np.asarray(a, dtype=np.float64)
    return a[..., 0] + 1j * a[..., 1]


def _pairs(c):
    return np.stack([c.real, c.imag], axis=-1)


def _planes(c):
    return np.stack([c.real, c.imag], axis=2)


def _run_gpu(ci, *, with_z, with_h0):
    import torch
    import selective_state_space_35_b200 as ssm
    dev = "cuda"
    u, dl, dout = to_dev(ci.u, dev), to_dev(ci.delta, dev), to_dev(ci.dout, dev)
    z = to_dev(ci.z, dev) if with_z else None
    Bm, Cm = to_dev(ci.Bm, dev), to_dev(ci.Cm, dev)
    sq = torch.from_numpy(ci.seq_idx).to(dev) if ci.seq_idx is not None else None
    h0 = f32_dev(ci.h0, dev) if with_h0 else None
    kw = dict(z=z, Dskip=f32_dev(ci.Dskip, dev), delta_bias=f32_dev(ci.delta_bias, dev),
              seq_idx=sq, initial_state=h0)
    A = f32_dev(ci.A, dev)
    out, fs, ws = ssm.scan_fwd(u, dl, A, Bm, Cm, return_final_state=True, **kw)
    assert ssm.scan_status(u, A, ws) == 0
    g = ssm.scan_bwd(u, dl, A, Bm, Cm, dout, ws, **kw)
    torch.cuda.synchronize()
    return out, fs, g


def _run_oracle(ci, *, with_z, with_h0):
    kw = dict(z=ci.z.f64 if with_z else None, Dskip=ci.Dskip, delta_bias=ci.delta_bias,
              seq_idx=ci.seq_idx, h0=_cplx_pairs(ci.h0) if with_h0 else None)
    A, Bm, Cm = _cplx_pairs(ci.A), _cplx_planes(ci.Bm.f64), _cplx_planes(ci.Cm.f64)
    f = oracle.cscan_fwd(ci.u.f64, ci.delta.f64, A, Bm, Cm, **kw)
    g = oracle.cscan_bwd(ci.u.f64, ci.delta.f64, A, Bm, Cm, ci.dout.f64, **kw)
    return f, g


def _compare(ci, out, fs, gr, f, g, *, fp32, with_z, with_h0):
    errs = {}
    want_out = f["out"] if fp32 else oracle.round_bf16(f["out"])
    errs["out"] = rel_l2(host64(out), want_out)
    assert errs["out"] <= (TOL_C32 if fp32 else TOL_BF16_OUT), errs
    if not fp32:  # one bf16 step allowed where |want| >= 4 (the same reading as the real scan's)
        ok, worst = bf16_out_max_abs_ok(host64(out), want_out, TOL_BF16_OUT_MAX)
        assert ok, worst
    errs["final_state"] = rel_l2(host64(fs), _pairs(f["final_state"]))
    assert errs["final_state"] <= (TOL_C32 if fp32 else TOL_GRAD), errs
    pairs = [("du", g["du"]), ("ddelta", g["ddelta"]), ("dA", _pairs(g["dA"])),
             ("dB", _planes(g["dB"])), ("dC", _planes(g["dC"])), ("dD", g["dD"]),
             ("ddelta_bias", g["ddelta_bias"]), ("dinitial_state", _pairs(g["dh0"]))]
    if with_z:
        pairs.append(("dz", g["dz"]))
    for k, w in pairs:
        if k in ("du", "ddelta", "dz") and not fp32:
            w = oracle.round_bf16(w)
        errs[k] = rel_l2(host64(gr[k]), w)
        assert errs[k] <= (TOL_C32 if fp32 else TOL_GRAD), (k, errs)
    return errs


@pytest.mark.parametrize("dtype,B,D,N,L,packed,with_z,with_h0", [
    ("f32", 2, 16, 16, 700, False, True, True),
    ("f32", 2, 13, 5, 333, True, True, True),
    ("f32", 1, 8, 16, 17, True, False, False),
    ("f32", 1, 3, 3, 1, False, True, True),
    ("bf16", 2, 24, 16, 2048, True, True, True),
    ("bf16", 1, 9, 7, 999, False, True, False),
])
def test_complex_parity(dtype, B, D, N, L, packed, with_z, with_h0):
    seed = 9100 + D + N + L + (7 if dtype == "bf16" else 0)
    seq = None
    if packed:
        seq = synth.random_segments(np.random.Generator(np.random.PCG64(seed)), B, L, 5)
    ci = synth.complex_inputs(B, D, N, L, dtype, seed, seq_idx=seq, with_h0=with_h0)
    out, fs, gr = _run_gpu(ci, with_z=with_z, with_h0=with_h0)
    f, g = _run_oracle(ci, with_z=with_z, with_h0=with_h0)
    _compare(ci, out, fs, gr, f, g, fp32=dtype == "f32", with_z=with_z, with_h0=with_h0)


def test_complex_with_zero_imaginary_parts_equals_real_scan():
    """Im A = Im B = Im C = 0: the complex kernels give the real kernels'
    results with C doubled (a check between the two CUDA paths)."""
    import torch
    import selective_state_space_35_b200 as ssm
    B, D, N, L = 2, 16, 16, 600
    inp = synth.make_inputs(synth.Shape("c-real", B, D, N, L, "f32"), 9301, dskip_random=True)
    inp.seq_idx = synth.random_segments(np.random.Generator(np.random.PCG64(9302)), B, L, 4)
    dev = "cuda"
    u, dl, z = to_dev(inp.x, dev), to_dev(inp.delta, dev), to_dev(inp.z, dev)
    dout = to_dev(inp.dout, dev)
    Bm, Cm = to_dev(inp.Bm, dev), to_dev(inp.Cm, dev)
    zeros = torch.zeros_like(Bm)
    Bc = torch.stack([Bm, zeros], dim=2).contiguous()
    Cc = torch.stack([Cm, zeros], dim=2).contiguous()
    A = f32_dev(inp.A, dev)
    Ac = torch.stack([A, torch.zeros_like(A)], dim=2).contiguous()
    sq = torch.from_numpy(inp.seq_idx).to(dev)
    kw = dict(z=z, Dskip=f32_dev(inp.Dskip, dev), delta_bias=f32_dev(inp.delta_bias, dev),
              seq_idx=sq)
    o_r, fs_r, ws_r = ssm.scan_fwd(u, dl, A, Bm, 2 * Cm, return_final_state=True, n_splits=1, **kw)
    g_r = ssm.scan_bwd(u, dl, A, Bm, 2 * Cm, dout, ws_r, n_splits=1, **kw)
    o_c, fs_c, ws_c = ssm.scan_fwd(u, dl, Ac, Bc, Cc, return_final_state=True, **kw)
    g_c = ssm.scan_bwd(u, dl, Ac, Bc, Cc, dout, ws_c, **kw)
    torch.cuda.synchronize()
    assert rel_l2(host64(o_c), host64(o_r)) <= 1e-5
    assert rel_l2(host64(fs_c[..., 0]), host64(fs_r)) <= 1e-5
    assert float(fs_c[..., 1].abs().max()) == 0.0
    for k in ("du", "ddelta", "dz", "dD", "ddelta_bias"):
        assert rel_l2(host64(g_c[k]), host64(g_r[k])) <= 1e-5, k
    assert rel_l2(host64(g_c["dA"][..., 0]), host64(g_r["dA"])) <= 1e-5
    assert rel_l2(host64(g_c["dB"][:, :, 0]), host64(g_r["dB"])) <= 1e-5
    assert rel_l2(host64(g_c["dC"][:, :, 0]), 2 * host64(g_r["dC"])) <= 1e-5


def test_complex_state_continues_across_calls():
    """Running [0, L1) and then [L1, L) from the first call's final state gives
    the single call's outputs and final state."""
    import torch
    import selective_state_space_35_b200 as ssm
    B, D, N, L, L1 = 1, 8, 16, 512, 200
    ci = synth.complex_inputs(B, D, N, L, "f32", 9401)
    dev = "cuda"
    u, dl, z = to_dev(ci.u, dev), to_dev(ci.delta, dev), to_dev(ci.z, dev)
    Bm, Cm, A = to_dev(ci.Bm, dev), to_dev(ci.Cm, dev), f32_dev(ci.A, dev)
    kw = dict(Dskip=f32_dev(ci.Dskip, dev), delta_bias=f32_dev(ci.delta_bias, dev))
    full, fs, _ = ssm.scan_fwd(u, dl, A, Bm, Cm, z=z, return_final_state=True, **kw)

    def part(t0, t1, h0):
        sl = lambda x: x[..., t0:t1].contiguous()
        return ssm.scan_fwd(sl(u), sl(dl), A, sl(Bm), sl(Cm), z=sl(z), return_final_state=True,
                            initial_state=h0, **kw)

    o1, f1, _ = part(0, L1, None)
    o2, f2, _ = part(L1, L, f1)
    torch.cuda.synchronize()
    got = torch.cat([o1, o2], dim=-1)
    assert rel_l2(host64(got), host64(full)) <= 1e-5
    assert rel_l2(host64(f2), host64(fs)) <= 1e-5
