"""Pieces of a longer sequence on the GPU: the final-state gradient, the
forward / backward summaries, the carry fold and the conv halos against the
fp64 oracle, then the context-parallel driver end to end with R ranks
emulated as threads on one device (no kernel waits on another; the host
threads exchange the tensors) against the unsharded oracle and the
unsharded GPU path."""
import numpy as np
import pytest

import oracle
from cp_support import (REDUCED, SHARDED, SHARDED_BC, OracleOps, full_problem, full_reference,
                        run_threads, shard)
from pipeline import TOL_BF16_OUT, TOL_F32, TOL_GRAD, host64, rel_l2

pytestmark = pytest.mark.gpu


def _f32(p):
    """Inputs rounded to fp32 (the oracle then runs on exactly these values)."""
    q = dict(p)
    for k, v in p.items():
        if isinstance(v, np.ndarray) and v.dtype == np.float64:
            q[k] = v.astype(np.float32).astype(np.float64)
    return q


def _bf16(p):
    q = _f32(p)
    for k in ("x", "z", "delta", "Bm", "Cm", "dout"):
        q[k] = oracle.round_bf16(q[k])
    return q


def _dev(a, dtype):
    import torch
    if a is None:
        return None
    if a.dtype == np.int32:
        return torch.from_numpy(np.ascontiguousarray(a)).cuda()
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda().to(dtype)


_ACT = ("x", "z", "delta", "Bm", "Cm", "dout")


def _devs(s, act_dtype):
    import torch
    return {k: (_dev(v, act_dtype) if k in _ACT else _dev(v, torch.float32) if
                isinstance(v, np.ndarray) and v.dtype != np.int32 else _dev(v, None))
            for k, v in s.items()}


@pytest.mark.parametrize("zoh", [False, True])
def test_final_state_gradient_matches_oracle(zoh):
    import torch
    import selective_state_space_35_b200 as ssm
    p = _f32(full_problem(2, 16, 16, 700, seed=801, seq_bounds=(300,)))
    d = _devs(p, torch.float32)
    kw = dict(z=d["z"], Dskip=d["Dskip"], delta_bias=d["delta_bias"], seq_idx=d["seq_idx"],
              initial_state=d["h0"], zoh=zoh)
    for n_splits in (1, 3):
        out, fs, ws = ssm.scan_fwd(d["x"], d["delta"], d["A"], d["Bm"], d["Cm"],
                                   n_splits=n_splits, **kw)
        g = ssm.scan_bwd(d["x"], d["delta"], d["A"], d["Bm"], d["Cm"], d["dout"], ws,
                         n_splits=n_splits, dfinal_state=d["dhL"], **kw)
        torch.cuda.synchronize()
        w = oracle.scan_bwd(p["x"], p["delta"], p["A"], p["Bm"], p["Cm"], p["dout"], z=p["z"],
                            Dskip=p["Dskip"], delta_bias=p["delta_bias"], seq_idx=p["seq_idx"],
                            h0=p["h0"], dhL=p["dhL"], zoh=zoh)
        for k, ok in (("du", "du"), ("ddelta", "ddelta"), ("dA", "dA"), ("dB", "dB"),
                      ("dC", "dC"), ("dinitial_state", "dh0")):
            e = rel_l2(host64(g[k]), w[ok])
            assert e <= TOL_F32, (n_splits, k, e)


def test_complex_final_state_gradient_matches_oracle():
    import torch
    import synth
    import selective_state_space_35_b200 as ssm
    ci = synth.complex_inputs(1, 8, 16, 300, "f32", 802, with_h0=True)
    rng = np.random.Generator(np.random.PCG64(803))
    dhL = rng.standard_normal((1, 8, 16, 2)).astype(np.float32)
    dv = lambda t: torch.from_numpy(np.ascontiguousarray(t.f32)).cuda()  # noqa: E731
    f32 = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda()  # noqa: E731
    kw = dict(z=dv(ci.z), Dskip=f32(ci.Dskip), delta_bias=f32(ci.delta_bias),
              initial_state=f32(ci.h0))
    A = f32(ci.A)
    out, fs, ws = ssm.scan_fwd(dv(ci.u), dv(ci.delta), A, dv(ci.Bm), dv(ci.Cm), **kw)
    g = ssm.scan_bwd(dv(ci.u), dv(ci.delta), A, dv(ci.Bm), dv(ci.Cm), dv(ci.dout), ws,
                     dfinal_state=f32(dhL), **kw)
    torch.cuda.synchronize()
    c = lambda a: a[..., 0].astype(np.float64) + 1j * a[..., 1]  # noqa: E731
    planes = lambda a: a[:, :, 0] + 1j * a[:, :, 1]  # noqa: E731
    w = oracle.cscan_bwd(ci.u.f64, ci.delta.f64, c(ci.A), planes(ci.Bm.f64), planes(ci.Cm.f64),
                         ci.dout.f64, z=ci.z.f64, Dskip=ci.Dskip, delta_bias=ci.delta_bias,
                         h0=c(ci.h0), dhL=c(dhL))
    pairs = lambda z: np.stack([z.real, z.imag], axis=-1)  # noqa: E731
    assert rel_l2(host64(g["du"]), w["du"]) <= TOL_F32
    assert rel_l2(host64(g["dA"]), pairs(w["dA"])) <= TOL_F32
    assert rel_l2(host64(g["dinitial_state"]), pairs(w["dh0"])) <= TOL_F32


@pytest.mark.parametrize("L,bounds,cut,n_splits", [(333, (100, 250), False, 0), (333, (100, 250), True, 0),
                                                   (40, (), False, 0), (40, (), True, 0),
                                                   (40, (), False, 1), (528, (100, 300), True, 1),
                                                   (528, (), False, 1)])
def test_summaries_and_carry_match_oracle(L, bounds, cut, n_splits):
    """Summaries against oracle runs; rows with a document start inside have
    decay 0, and a start at token 0 (seq_prev differs) zeroes decay and the
    backward summary. n_splits=1 with L a multiple of 8 takes the N = 16
    summary kernels (the automatic choice splits rows this short)."""
    import torch
    import selective_state_space_35_b200 as ssm
    p = _f32(full_problem(2, 12, 16, L, seed=804 + L + int(cut), seq_bounds=bounds))
    d = _devs(p, torch.float32)
    seq_prev = torch.tensor([p["seq_idx"][0, 0] - (1 if cut else 0), p["seq_idx"][1, 0]],
                            dtype=torch.int32, device="cuda")
    dec, end = ssm.scan_fwd_summary(d["x"], d["delta"], d["A"], d["Bm"],
                                    delta_bias=d["delta_bias"], seq_idx=d["seq_idx"],
                                    seq_prev=seq_prev, n_splits=n_splits)
    bdec, adj = ssm.scan_bwd_summary(d["delta"], d["A"], d["Cm"], d["dout"], z=d["z"],
                                     delta_bias=d["delta_bias"], seq_idx=d["seq_idx"],
                                     seq_prev=seq_prev, n_splits=n_splits)
    torch.cuda.synchronize()
    ops = OracleOps()
    T = lambda a: torch.from_numpy(a)  # noqa: E731
    sp = seq_prev.cpu()
    wdec, wend = ops.scan_fwd_summary(T(p["x"]), T(p["delta"]), T(p["A"]), T(p["Bm"]),
                                      T(p["seq_idx"]), sp, T(p["delta_bias"]), True)
    _, wadj = ops.scan_bwd_summary(T(p["delta"]), T(p["A"]), T(p["Cm"]), T(p["dout"]), T(p["z"]),
                                   T(p["seq_idx"]), sp, T(p["delta_bias"]), True)
    assert rel_l2(host64(end), wend.numpy()) <= TOL_F32
    assert rel_l2(host64(adj), wadj.numpy()) <= TOL_F32
    wd = wdec.numpy()
    if np.abs(wd).max() > 0:
        assert rel_l2(host64(dec), wd) <= TOL_F32
        assert rel_l2(host64(bdec), wd) <= TOL_F32
    else:
        assert float(dec.abs().max()) == 0.0 and float(bdec.abs().max()) == 0.0
    if cut:
        assert float(dec[0].abs().max()) == 0.0 and float(adj[0].abs().max()) == 0.0
    # carry fold over 4 stacked random summaries, both directions
    rng = np.random.Generator(np.random.PCG64(805))
    R = 4
    decs = rng.uniform(0, 1, size=(R, 2, 12, 16)).astype(np.float32)
    vals = rng.standard_normal((R, 2, 12, 16)).astype(np.float32)
    init = rng.standard_normal((2, 12, 16)).astype(np.float32)
    for r in range(R):
        for rev in (False, True):
            got = ssm.state_carry(torch.from_numpy(decs).cuda(), torch.from_numpy(vals).cuda(), r,
                                  reverse=rev, init=torch.from_numpy(init).cuda())
            want = ops.state_carry(T(decs.astype(np.float64)), T(vals.astype(np.float64)), r, rev,
                                   T(init.astype(np.float64)), None, None)
            assert rel_l2(host64(got), want.numpy()) <= 1e-6, (r, rev)


@pytest.mark.parametrize("L,vec", [(256, True), (203, False)])
def test_conv_halos_match_oracle(L, vec):
    import torch
    import selective_state_space_35_b200 as ssm
    p = _f32(full_problem(2, 8, 4, L + 6, seed=806 + L, seq_bounds=(2, 5, L + 2, L + 4)))
    x, seq, du_all = p["x"], p["seq_idx"], p["dout"]
    mid = slice(3, 3 + L)
    d = lambda a: _dev(np.ascontiguousarray(a), torch.float32 if a.dtype != np.int32 else None)  # noqa: E731
    xs, sq = d(x[..., mid]), d(seq[..., mid])
    x_prev, seq_prev = d(x[..., :3]), d(seq[..., :3])
    x_next, seq_next, du_next = d(x[..., 3 + L:]), d(seq[..., 3 + L:]), d(du_all[..., 3 + L:])
    w, b = d(p["conv_w"]), d(p["conv_b"])
    u = ssm.conv1d_fwd(xs, w, b, sq, x_prev=x_prev, seq_prev=seq_prev)
    du = d(du_all[..., mid])
    dx, dw, db = ssm.conv1d_bwd(xs, w, b, sq, du, x_prev=x_prev, seq_prev=seq_prev, x_next=x_next,
                                du_next=du_next, seq_next=seq_next)
    torch.cuda.synchronize()
    ops = OracleOps()
    T = lambda a: torch.from_numpy(np.ascontiguousarray(a))  # noqa: E731
    wu = ops.conv_fwd(T(x[..., mid]), T(p["conv_w"]), T(p["conv_b"]), T(seq[..., mid]),
                      T(x[..., :3]), T(seq[..., :3]))
    wdx, wdw, wdb = ops.conv_bwd(T(x[..., mid]), T(p["conv_w"]), T(p["conv_b"]), T(seq[..., mid]),
                                 T(du_all[..., mid]), T(x[..., :3]), T(seq[..., :3]),
                                 T(x[..., 3 + L:]), T(du_all[..., 3 + L:]), T(seq[..., 3 + L:]))
    assert rel_l2(host64(u), wu.numpy()) <= TOL_F32
    assert rel_l2(host64(dx), wdx.numpy()) <= TOL_F32
    assert rel_l2(host64(dw), wdw.numpy()) <= TOL_F32
    assert rel_l2(host64(db), wdb.numpy()) <= TOL_F32


def _gpu_rank(p, R, r, comm, act_dtype, zoh=False):
    import torch
    from selective_state_space_35_b200.cp import ContextParallelLayer
    s, lo, hi = shard(p, R, r)
    d = _devs(s, act_dtype)
    layer = ContextParallelLayer(comm, zoh=zoh)
    out, fs, ctx = layer.forward(d["x"], d["delta"], d["z"], d["Bm"], d["Cm"], d["A"], d["Dskip"],
                                 d["delta_bias"], d["conv_w"], d["conv_b"], seq_idx=d["seq_idx"],
                                 initial_state=d["h0"])
    g = layer.backward(ctx, d["dout"], dfinal_state=d["dhL"])
    torch.cuda.synchronize()
    res = {k: (host64(v) if v is not None else None) for k, v in g.items()}
    res["out"] = host64(out)
    res["final_state"] = host64(fs)
    return res, lo, hi


@pytest.mark.parametrize("R,L,bounds,dtype", [
    (1, 300, (100,), "f32"),
    (3, 9, (3, 5), "f32"),
    (2, 1024, (512, 700), "f32"),
    (3, 771, (257, 516, 100), "f32"),
    (4, 1200, (300, 602, 1000), "f32"),
    (4, 4096, (1024, 2050, 3000), "bf16"),
])
def test_cp_gpu_equal_unsharded(R, L, bounds, dtype):
    """Boundaries at a shard start, inside a conv halo and mid-shard; shard
    lengths both multiples of 8 and ragged."""
    import torch
    raw = full_problem(2, 24, 16, L, seed=900 + R + L, seq_bounds=bounds)
    p = _f32(raw) if dtype == "f32" else _bf16(raw)
    act = torch.float32 if dtype == "f32" else torch.bfloat16
    results = run_threads(R, lambda r, comm: _gpu_rank(p, R, r, comm, act))
    fp32 = dtype == "f32"
    want = full_reference(p, bf16_points=not fp32)
    for r, (res, lo, hi) in enumerate(results):
        for k in SHARDED + SHARDED_BC:
            w = want[k][..., lo:hi]
            if not fp32 and k in ("out", "du", "ddelta", "dz", "dx"):
                w = oracle.round_bf16(w)
            tol = TOL_F32 if fp32 else (TOL_BF16_OUT if k == "out" else TOL_GRAD)
            # du and dx pass through the bf16 du between the scan and the conv
            e = rel_l2(res[k], w)
            assert e <= tol, (r, k, e)
        for k in REDUCED:
            e = rel_l2(res[k], want[k])
            assert e <= (TOL_F32 if fp32 else TOL_GRAD), (r, k, e)
    assert rel_l2(results[-1][0]["final_state"], want["final_state"]) <= (TOL_F32 if fp32 else TOL_GRAD)
    assert rel_l2(results[0][0]["dinitial_state"], want["dinitial_state"]) <= (TOL_F32 if fp32 else TOL_GRAD)


def test_cp_gpu_zero_order_hold():
    raw = full_problem(2, 16, 16, 900, seed=990, seq_bounds=(450, 300))
    p = _f32(raw)
    import torch
    results = run_threads(3, lambda r, comm: _gpu_rank(p, 3, r, comm, torch.float32, zoh=True))
    want = full_reference(p, zoh=True)
    for r, (res, lo, hi) in enumerate(results):
        for k in SHARDED + SHARDED_BC:
            assert rel_l2(res[k], want[k][..., lo:hi]) <= TOL_F32, (r, k)
        for k in REDUCED:
            assert rel_l2(res[k], want[k]) <= TOL_F32, (r, k)
    assert rel_l2(results[0][0]["dinitial_state"], want["dinitial_state"]) <= TOL_F32
