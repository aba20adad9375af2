"""Parity of the CUDA path (through the C ABI) with the fp64 CPU oracle.

Same seeded inputs on both sides; the oracle never sees a GPU value. fp32:
rel-L2 <= 1e-5 everywhere. bf16 inputs with fp32 state: out rel-L2 <= 2e-3
and max-abs <= 2e-2 against the oracle rounded to bf16, gradients rel-L2 <=
5e-3. Segment handling is checked exactly where it is exact (packed ==
separate in the oracle) and by parity everywhere else.
"""
import numpy as np
import pytest

import oracle
import synth
from pipeline import (TOL_BF16_OUT, TOL_BF16_OUT_MAX, TOL_F32, TOL_GRAD, bf16_out_max_abs_ok,
                      device_inputs, gpu_layer, host64, max_abs, rel_l2)

pytestmark = pytest.mark.gpu

GRAD_KEYS = ("du", "ddelta", "dz", "dA", "dB", "dC", "dD", "ddelta_bias", "dx", "dconv_w", "dconv_b")


def _torch():
    import torch
    return torch


def _compare_all(res, want, *, fp32, use_z=True, keys_out=("u", "out", "final_state")):
    errs = {}
    for k in keys_out:
        if res.get(k) is None:
            continue
        w = want["u_stored"] if k == "u" else want[k]
        if k in ("u", "out") and not fp32:
            w = oracle.round_bf16(w)
        errs[k] = rel_l2(host64(res[k]), w)
        tol = TOL_F32 if fp32 else TOL_BF16_OUT
        assert errs[k] <= tol, (k, errs[k])
        if not fp32 and k == "out":
            assert max_abs(host64(res[k]), w) <= TOL_BF16_OUT_MAX
    for k in GRAD_KEYS:
        if k == "dz" and not use_z:
            continue
        w = want[k]
        if k in ("du", "ddelta", "dz", "dx") and not fp32:
            w = oracle.round_bf16(w)
        errs[k] = rel_l2(host64(res[k]), w)
        tol = TOL_F32 if fp32 else TOL_GRAD
        assert errs[k] <= tol, (k, errs[k])
    return errs


def _oracle_layer(inp, *, bf16_points, use_z=True, use_seq=True, softplus=True, nthreads=8):
    seq = inp.seq_idx if use_seq else None
    z = inp.z.f64 if use_z else None
    c, u = oracle.conv1d_fwd(inp.x.f64, inp.conv_w, inp.conv_b, seq)
    u_s = oracle.round_bf16(u) if bf16_points else u
    kw = dict(z=z, Dskip=inp.Dskip, delta_bias=inp.delta_bias, softplus=softplus, seq_idx=seq,
              nthreads=nthreads)
    f = oracle.scan_fwd(u_s, inp.delta.f64, inp.A, inp.Bm.f64, inp.Cm.f64, **kw)
    g = oracle.scan_bwd(u_s, inp.delta.f64, inp.A, inp.Bm.f64, inp.Cm.f64, inp.dout.f64, **kw)
    du_s = oracle.round_bf16(g["du"]) if bf16_points else g["du"]
    dx, dw, dcb = oracle.conv1d_bwd(inp.x.f64, inp.conv_w, inp.conv_b, seq, du_s)
    r = {"u_stored": u_s, "dx": dx, "dconv_w": dw, "dconv_b": dcb}
    r.update(f)
    r.update(g)
    return r


def _small(B, D, N, L, seed, *, dtype="f32", nbound=0, packed=False, boundary_at=None):
    sh = synth.Shape("test", B, D, N, L, dtype, packed=packed, boundary_at=boundary_at)
    inp = synth.make_inputs(sh, seed, conv_bias_scale=0.3, dskip_random=True)
    if nbound:
        inp.seq_idx = synth.random_segments(np.random.Generator(np.random.PCG64(seed)), B, L, nbound)
    return inp


def test_tiny_fp32_layer_with_boundary():
    inp = synth.make_inputs(synth.CONFIGS[1], synth.seed_for(1))
    res = gpu_layer(device_inputs(inp))
    want = _oracle_layer(inp, bf16_points=False)
    _compare_all(res, want, fp32=True)


SMALL_CASES = [
    # B, D, N, L, nbound
    (1, 1, 1, 1, 0),
    (1, 3, 4, 7, 0),
    (2, 5, 16, 64, 3),
    (1, 4, 8, 255, 5),
    (1, 4, 16, 256, 4),
    (2, 3, 16, 257, 6),
    (1, 6, 5, 600, 9),
    (2, 13, 16, 33, 2),     # backward: a second CTA with 5 of its 8 rows; one token past a block
    (1, 9, 3, 95, 3),       # L just short of three 32-token blocks
    (2, 9, 16, 1031, 12),
    (1, 4, 16, 2048, 0),
]


@pytest.mark.parametrize("B,D,N,L,nb", SMALL_CASES)
def test_small_fp32_shapes(B, D, N, L, nb):
    inp = _small(B, D, N, L, 1000 + L + D, nbound=nb)
    res = gpu_layer(device_inputs(inp))
    want = _oracle_layer(inp, bf16_points=False)
    _compare_all(res, want, fp32=True)


@pytest.mark.parametrize("B,D,N,L,nb", [(1, 5, 16, 520, 7), (2, 4, 16, 1024, 5), (1, 3, 4, 13, 2)])
def test_small_bf16_shapes(B, D, N, L, nb):
    inp = _small(B, D, N, L, 2000 + L, dtype="bf16", nbound=nb)
    res = gpu_layer(device_inputs(inp))
    want = _oracle_layer(inp, bf16_points=True)
    _compare_all(res, want, fp32=False)


def test_one_token_documents_and_edge_boundaries():
    B, D, N, L = 1, 4, 16, 300
    inp = _small(B, D, N, L, 77)
    seq = np.zeros((B, L), dtype=np.int32)
    doc = 0
    for t in range(L):  # 1-token documents at the start, chunk edge, and end
        if t in (1, 2, 3, 4, 255, 256, 257, 298, 299) or t % 37 == 0:
            doc += 1
        seq[0, t] = doc
    inp.seq_idx = seq
    res = gpu_layer(device_inputs(inp))
    want = _oracle_layer(inp, bf16_points=False)
    _compare_all(res, want, fp32=True)


@pytest.mark.parametrize("use_z,softplus,noD", [(False, True, False), (True, False, False),
                                                 (False, False, True)])
def test_optional_inputs(use_z, softplus, noD):
    inp = _small(2, 5, 8, 333, 555, nbound=3)
    if not softplus:  # the step is used as given: keep it positive
        inp.delta.f32 = np.abs(inp.delta.f32) * np.float32(0.2)
        inp.delta.f64 = inp.delta.f32.astype(np.float64)
        inp.delta_bias = np.zeros_like(inp.delta_bias)
    if noD:
        inp.Dskip = np.zeros_like(inp.Dskip)
    res = gpu_layer(device_inputs(inp), use_z=use_z, softplus=softplus)
    want = _oracle_layer(inp, bf16_points=False, use_z=use_z, softplus=softplus)
    _compare_all(res, want, fp32=True, use_z=use_z)


@pytest.mark.parametrize("P", [2, 3, 5])
def test_forced_splits_fp32(P):
    inp = _small(2, 5, 16, 1500, 31 + P, nbound=4)
    res = gpu_layer(device_inputs(inp), n_splits=P)
    want = _oracle_layer(inp, bf16_points=False)
    _compare_all(res, want, fp32=True)


def test_mamba130m_layer_bf16_full():
    inp = synth.make_inputs(synth.CONFIGS[2], synth.seed_for(2))
    res = gpu_layer(device_inputs(inp))
    want = _oracle_layer(inp, bf16_points=True)
    _compare_all(res, want, fp32=False)


def test_mamba130m_layer_splits_match_unsplit():
    torch = _torch()
    inp = synth.make_inputs(synth.CONFIGS[2], synth.seed_for(2, 1))
    dv = device_inputs(inp)
    r1 = gpu_layer(dv, n_splits=1)
    r4 = gpu_layer(dv, n_splits=4)
    for k in ("out", "final_state", "du", "ddelta", "dz", "dA", "dB", "dC", "dD", "dx"):
        assert rel_l2(host64(r4[k]), host64(r1[k])) <= 1e-3, k
    torch.cuda.synchronize()


def test_cu_seqlens_equals_seq_idx():
    torch = _torch()
    import selective_state_space_35_b200 as ssm
    B, D, N, L = 1, 6, 16, 777
    inp = _small(B, D, N, L, 91)
    cuts = [0, 1, 100, 256, 257, 600, 776, L]
    seq = np.zeros((1, L), dtype=np.int32)
    for i in range(len(cuts) - 1):
        seq[0, cuts[i]:cuts[i + 1]] = i
    inp.seq_idx = seq
    dv = device_inputs(inp)
    cu = torch.tensor(cuts, dtype=torch.int32, device="cuda")
    u = ssm.conv1d_fwd(dv["x"], dv["conv_w"], dv["conv_b"], dv["seq_idx"])
    kw = dict(z=dv["z"], Dskip=dv["Dskip"], delta_bias=dv["delta_bias"])
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


@pytest.mark.parametrize("n_splits", [0, 1])
def test_run_twice_bitwise(n_splits):
    """Two runs give the same bits in every output and gradient, dB and dC
    included with the deterministic backward (n_splits=1: the N = 16
    kernels; 0: the automatic choice, L split in two at this size)."""
    torch = _torch()
    inp = _small(2, 9, 16, 1200, 5, dtype="bf16", nbound=3)
    dv = device_inputs(inp)
    r1 = gpu_layer(dv, n_splits=n_splits, deterministic=True)
    r2 = gpu_layer(dv, n_splits=n_splits, deterministic=True)
    for k in ("u", "out", "final_state", "du", "ddelta", "dz", "dA", "dB", "dC", "dD",
              "ddelta_bias", "dx", "dconv_w", "dconv_b"):
        assert torch.equal(r1[k], r2[k]), k


def test_packed_equals_separate_on_gpu():
    torch = _torch()
    B, D, N, L = 1, 4, 16, 700
    inp = _small(B, D, N, L, 606)
    cuts = [0, 3, 260, 261, 512, L]
    seq = np.zeros((1, L), dtype=np.int32)
    for i in range(len(cuts) - 1):
        seq[0, cuts[i]:cuts[i + 1]] = i
    inp.seq_idx = seq
    full = gpu_layer(device_inputs(inp))
    for s, e in zip(cuts[:-1], cuts[1:]):
        sub = _small(B, D, N, e - s, 606)
        for name in ("x", "z", "delta", "dout"):
            t = getattr(inp, name)
            getattr(sub, name).f32 = np.ascontiguousarray(t.f32[:, :, s:e])
        for name in ("Bm", "Cm"):
            getattr(sub, name).f32 = np.ascontiguousarray(getattr(inp, name).f32[:, :, s:e])
        for name in ("A", "Dskip", "delta_bias", "conv_w", "conv_b"):
            setattr(sub, name, getattr(inp, name))
        sub.seq_idx = None
        part = gpu_layer(device_inputs(sub))
        for k in ("u", "out", "du", "ddelta", "dz", "dx"):
            a = host64(full[k])[:, :, s:e]
            assert rel_l2(a, host64(part[k])) <= 1e-6, k
        for k in ("dB", "dC"):
            assert rel_l2(host64(full[k])[:, :, s:e], host64(part[k])) <= 1e-6, k
    torch.cuda.synchronize()


def test_output_red_zones_untouched():
    torch = _torch()
    import selective_state_space_35_b200 as ssm
    B, D, N, L = 1, 3, 16, 300
    inp = _small(B, D, N, L, 4242, dtype="bf16", nbound=2)
    dv = device_inputs(inp)
    pad = 64
    n = B * D * L

    def guarded():
        buf = torch.full((n + 2 * pad,), float("nan"), dtype=torch.bfloat16, device="cuda")
        return buf, buf[pad:pad + n].view(B, D, L)

    bu, u = guarded()
    ssm.conv1d_fwd(dv["x"], dv["conv_w"], dv["conv_b"], dv["seq_idx"], out=u)
    bo, o = guarded()
    _, _, ws = ssm.scan_fwd(u, dv["delta"], dv["A"], dv["Bm"], dv["Cm"], z=dv["z"],
                            Dskip=dv["Dskip"], delta_bias=dv["delta_bias"], seq_idx=dv["seq_idx"],
                            out=o)
    bufs = {k: guarded() for k in ("du", "ddelta", "dz")}
    ssm.scan_bwd(u, dv["delta"], dv["A"], dv["Bm"], dv["Cm"], dv["dout"], ws, z=dv["z"],
                 Dskip=dv["Dskip"], delta_bias=dv["delta_bias"], seq_idx=dv["seq_idx"],
                 grads={k: v[1] for k, v in bufs.items()})
    bx, dx = guarded()
    ssm.conv1d_bwd(dv["x"], dv["conv_w"], dv["conv_b"], dv["seq_idx"], bufs["du"][1], dx=dx)
    torch.cuda.synchronize()
    for buf in [bu, bo, bx] + [v[0] for v in bufs.values()]:
        assert torch.isnan(buf[:pad]).all() and torch.isnan(buf[-pad:]).all()
        assert not torch.isnan(buf[pad:-pad]).any()


# ---------------------------------------------------------------------------
# Full-size workloads: the GPU runs the whole layer in the benchmark's launch
# configuration (at B = 2, D = 1536 one 22-row CTA per SM; at B = 4, D = 5120
# 12-row CTAs, two per SM); the oracle recomputes every channel of each batch
# row in fp64 and every output and gradient is compared over the whole row:
# all CTAs, every channel position within a CTA and a row pair, and dB / dC
# (sums over all channels) at every token.
# ---------------------------------------------------------------------------
def _nthreads():
    import os
    try:
        return max(1, len(os.sched_getaffinity(0)))
    except Exception:
        return os.cpu_count() or 1


@pytest.mark.parametrize("cfg", [3, 4, 5])
def test_full_size_all_channels(cfg):
    torch = _torch()
    sh = synth.CONFIGS[cfg]
    inp = synth.make_inputs(sh, synth.seed_for(cfg))
    res = gpu_layer(device_inputs(inp))
    torch.cuda.synchronize()
    nt = _nthreads()
    acc = {k: 0.0 for k in ("dA", "dD", "ddelta_bias", "dconv_w", "dconv_b")}
    for b in range(sh.B):
        sl = np.s_[b:b + 1]
        seq = None if inp.seq_idx is None else np.ascontiguousarray(inp.seq_idx[sl])
        x = inp.x.f64[sl]
        _, u = oracle.conv1d_fwd(x, inp.conv_w, inp.conv_b, seq)
        u_s = oracle.round_bf16(u)
        del u
        kw = dict(z=inp.z.f64[sl], Dskip=inp.Dskip, delta_bias=inp.delta_bias, seq_idx=seq,
                  nthreads=nt)
        Bm, Cm = inp.Bm.f64[sl], inp.Cm.f64[sl]
        f = oracle.scan_fwd(u_s, inp.delta.f64[sl], inp.A, Bm, Cm, **kw)
        assert rel_l2(host64(res["u"][sl]), u_s) <= TOL_BF16_OUT
        o, wo = host64(res["out"][sl]), oracle.round_bf16(f["out"])
        assert rel_l2(o, wo) <= TOL_BF16_OUT, b
        ok, worst = bf16_out_max_abs_ok(o, wo, TOL_BF16_OUT_MAX)
        assert ok, (b, worst, max_abs(o, wo))
        del o, wo
        assert rel_l2(host64(res["final_state"][sl]), f["final_state"]) <= TOL_BF16_OUT
        del f
        g = oracle.scan_bwd(u_s, inp.delta.f64[sl], inp.A, Bm, Cm, inp.dout.f64[sl], **kw)
        for k in ("du", "ddelta", "dz"):
            assert rel_l2(host64(res[k][sl]), oracle.round_bf16(g[k])) <= TOL_GRAD, (k, b)
        for k in ("dB", "dC"):
            assert rel_l2(host64(res[k][sl]), g[k]) <= TOL_GRAD, (k, b)
        # a middle window on its own (the sums over all channels)
        mid = np.s_[b:b + 1, :, sh.L // 2 - 192:sh.L // 2 + 192]
        for k in ("dB", "dC"):
            assert rel_l2(host64(res[k][mid]), g[k][(0,) + mid[1:]][None]) <= TOL_GRAD, (k, b)
        for k in ("dA", "dD", "ddelta_bias"):
            acc[k] = acc[k] + g[k]
        dx, dw, db = oracle.conv1d_bwd(x, inp.conv_w, inp.conv_b, seq, oracle.round_bf16(g["du"]))
        del g
        # dx depends on du, which the GPU rounds to bf16 on its own path
        assert rel_l2(host64(res["dx"][sl]), oracle.round_bf16(dx)) <= TOL_GRAD, b
        acc["dconv_w"] = acc["dconv_w"] + dw
        acc["dconv_b"] = acc["dconv_b"] + db
        del dx, u_s
    for k, w in acc.items():
        assert rel_l2(host64(res[k]), w) <= TOL_GRAD, k
        # every channel on its own, against the array's RMS (a channel's sum
        # over B x L terms of both signs may cancel to far below that scale,
        # so its own norm is not the yardstick)
        got = host64(res[k]).reshape(sh.D, -1)
        want = np.asarray(w).reshape(sh.D, -1)
        rms = float(np.sqrt(np.mean(want * want)))
        err = np.sqrt(np.mean((got - want) ** 2, axis=1)) / rms
        assert float(np.max(err)) <= 2 * TOL_GRAD, (k, int(np.argmax(err)), float(np.max(err)))


def test_unaligned_gradient_buffers_take_scalar_path():
    torch = _torch()
    import selective_state_space_35_b200 as ssm
    B, D, N, L = 1, 5, 16, 512
    inp = _small(B, D, N, L, 808, dtype="bf16", nbound=2)
    dv = device_inputs(inp)
    u = ssm.conv1d_fwd(dv["x"], dv["conv_w"], dv["conv_b"], dv["seq_idx"])
    kw = dict(z=dv["z"], Dskip=dv["Dskip"], delta_bias=dv["delta_bias"], seq_idx=dv["seq_idx"])
    _, _, ws = ssm.scan_fwd(u, dv["delta"], dv["A"], dv["Bm"], dv["Cm"], **kw)
    ref = ssm.scan_bwd(u, dv["delta"], dv["A"], dv["Bm"], dv["Cm"], dv["dout"], ws, **kw)
    n = B * N * L
    bufB = torch.empty(n + 1, dtype=torch.float32, device="cuda")
    bufC = torch.empty(n + 1, dtype=torch.float32, device="cuda")
    g = ssm.scan_bwd(u, dv["delta"], dv["A"], dv["Bm"], dv["Cm"], dv["dout"], ws,
                     grads={"dB": bufB[1:].view(B, N, L), "dC": bufC[1:].view(B, N, L)}, **kw)
    for k in ("dB", "dC", "du", "ddelta", "dz"):
        assert rel_l2(host64(g[k]), host64(ref[k])) <= 1e-6, k


def test_device_status_word_clear_after_tma_staged_runs():
    import selective_state_space_35_b200 as ssm
    inp = _small(2, 9, 16, 2048, 909, dtype="bf16", nbound=3)  # bf16, L % 8 == 0: TMA-staged tiles
    dv = device_inputs(inp)
    u = ssm.conv1d_fwd(dv["x"], dv["conv_w"], dv["conv_b"], dv["seq_idx"])
    kw = dict(z=dv["z"], Dskip=dv["Dskip"], delta_bias=dv["delta_bias"], seq_idx=dv["seq_idx"])
    for P in (1, 3):
        _, _, ws = ssm.scan_fwd(u, dv["delta"], dv["A"], dv["Bm"], dv["Cm"], n_splits=P, **kw)
        ssm.scan_bwd(u, dv["delta"], dv["A"], dv["Bm"], dv["Cm"], dv["dout"], ws, n_splits=P, **kw)
        assert ssm.scan_status(u, dv["A"], ws) == 0
