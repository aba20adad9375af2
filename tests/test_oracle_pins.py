"""Pins for the fp64 CPU oracle: checks that do not go through the oracle's
own formulas (closed forms, special cases, brute force, a library conv, the
associative split, packing invariance, finite differences, hand-worked
values). Every check here runs on CPU."""
import json
import math
import os

import numpy as np
import pytest

import oracle
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rng(seed=1234):
    return np.random.Generator(np.random.PCG64(seed))


def _sig(v):
    return 1.0 / (1.0 + np.exp(-v))


def _problem(rng, B=1, D=3, N=4, L=40, seq=None):
    u = rng.standard_normal((B, D, L))
    delta = 0.5 * rng.standard_normal((B, D, L))
    z = rng.standard_normal((B, D, L))
    A = -rng.uniform(0.2, 2.0, size=(D, N))
    Bm = rng.standard_normal((B, N, L))
    Cm = rng.standard_normal((B, N, L))
    Dskip = rng.uniform(0.5, 1.5, size=D)
    dbias = rng.uniform(-3, -1, size=D)
    return dict(u=u, delta=delta, z=z, A=A, Bm=Bm, Cm=Cm, Dskip=Dskip,
                delta_bias=dbias, seq_idx=seq)


# --------------------------------------------------------------------------
# bf16 rounding used at the storage points
# --------------------------------------------------------------------------
def test_round_bf16_hand_values():
    # spacing of bf16 at 1.0 is 2^-7; ties go to the even mantissa
    vals = np.array([1.0 + 2**-8, 1.0 + 3 * 2**-8, 1.0 + 2**-8 + 2**-20, -3.0, 0.0,
                     2**-130])
    want = np.array([1.0, 1.0 + 2**-6, 1.0 + 2**-7, -3.0, 0.0, 2**-130])
    np.testing.assert_array_equal(oracle.round_bf16(vals), want)


def test_round_bf16_matches_fp32_rne_bits():
    x = _rng(7).standard_normal(10000).astype(np.float32) * 37.0
    bits = synth.f32_to_bf16_bits(x)
    np.testing.assert_array_equal(oracle.round_bf16(x.astype(np.float64)),
                                  synth.bf16_bits_to_f32(bits).astype(np.float64))


# --------------------------------------------------------------------------
# conv1d
# --------------------------------------------------------------------------
def test_conv_identity_tap():
    rng = _rng()
    x = rng.standard_normal((2, 3, 50))
    w = np.zeros((3, 4))
    w[:, 3] = 1.0  # the newest tap multiplies x_t
    c, u = oracle.conv1d_fwd(x, w, None, None, silu=False)
    np.testing.assert_array_equal(u, x)
    np.testing.assert_array_equal(c, x)


def test_conv_matches_torch_conv1d():
    torch = pytest.importorskip("torch")
    rng = _rng(3)
    B, D, L = 2, 5, 37
    x = rng.standard_normal((B, D, L))
    w = rng.uniform(-0.5, 0.5, size=(D, 4))
    b = rng.standard_normal(D)
    ref = torch.nn.functional.conv1d(torch.from_numpy(x), torch.from_numpy(w)[:, None, :],
                                     torch.from_numpy(b), padding=3, groups=D)[..., :L].numpy()
    c, u = oracle.conv1d_fwd(x, w, b, None, silu=True)
    np.testing.assert_allclose(c, ref, rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(u, ref * _sig(ref), rtol=1e-13, atol=1e-13)


def test_conv_packed_equals_separate():
    rng = _rng(5)
    D, L = 3, 60
    seq = np.zeros((1, L), dtype=np.int32)
    cuts = [0, 1, 2, 17, 18, 40, L]
    for i in range(len(cuts) - 1):
        seq[0, cuts[i]:cuts[i + 1]] = i
    x = rng.standard_normal((1, D, L))
    w = rng.uniform(-0.5, 0.5, size=(D, 4))
    b = rng.standard_normal(D)
    du = rng.standard_normal((1, D, L))
    _, u = oracle.conv1d_fwd(x, w, b, seq)
    dx, dw, db = oracle.conv1d_bwd(x, w, b, seq, du)
    dw_sum = np.zeros_like(dw)
    db_sum = np.zeros_like(db)
    for i in range(len(cuts) - 1):
        s, e = cuts[i], cuts[i + 1]
        _, ui = oracle.conv1d_fwd(x[:, :, s:e].copy(), w, b, None)
        np.testing.assert_array_equal(u[:, :, s:e], ui)
        dxi, dwi, dbi = oracle.conv1d_bwd(x[:, :, s:e].copy(), w, b, None, du[:, :, s:e].copy())
        np.testing.assert_array_equal(dx[:, :, s:e], dxi)
        dw_sum += dwi
        db_sum += dbi
    np.testing.assert_allclose(dw, dw_sum, rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(db, db_sum, rtol=1e-13, atol=1e-13)


def _fd(f, arr, h_rel=1e-6):
    g = np.zeros_like(arr)
    it = np.nditer(arr, flags=["multi_index"])
    for _ in it:
        i = it.multi_index
        old = arr[i]
        h = h_rel * max(1.0, abs(old))
        arr[i] = old + h
        fp = f()
        arr[i] = old - h
        fm = f()
        arr[i] = old
        g[i] = (fp - fm) / (2 * h)
    return g


def _close(fd, an, tol=1e-6):
    scale = max(1.0, float(np.abs(an).max()))
    err = np.abs(fd - an).max() / scale
    assert err < tol, err


def test_conv_bwd_finite_differences():
    rng = _rng(11)
    B, D, L = 1, 3, 20
    seq = np.zeros((B, L), dtype=np.int32)
    seq[:, 9:] = 1
    x = rng.standard_normal((B, D, L))
    w = rng.uniform(-0.5, 0.5, size=(D, 4))
    b = rng.standard_normal(D)
    gu = rng.standard_normal((B, D, L))

    def loss():
        return float(np.sum(oracle.conv1d_fwd(x, w, b, seq)[1] * gu))

    dx, dw, db = oracle.conv1d_bwd(x, w, b, seq, gu)
    _close(_fd(loss, x), dx)
    _close(_fd(loss, w), dw)
    _close(_fd(loss, b), db)


# --------------------------------------------------------------------------
# scan forward: closed forms and special cases
# --------------------------------------------------------------------------
def test_scan_L1_closed_form():
    rng = _rng(13)
    p = _problem(rng, B=2, D=3, N=5, L=1)
    r = oracle.scan_fwd(p["u"], p["delta"], p["A"], p["Bm"], p["Cm"], z=p["z"],
                        Dskip=p["Dskip"], delta_bias=p["delta_bias"])
    v = p["delta"] + p["delta_bias"][None, :, None]
    dt = np.log1p(np.exp(v))
    # y_0 = sum_n C_n * (delta_0 B_n u_0) + D u_0   (h_{-1} = 0)
    y = np.einsum("bnl,bnl->bl", p["Cm"], p["Bm"])[:, None, :] * dt * p["u"] \
        + p["Dskip"][None, :, None] * p["u"]
    np.testing.assert_allclose(r["y"], y, rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(r["out"], y * p["z"] * _sig(p["z"]), rtol=1e-13, atol=1e-14)


def test_scan_zero_step_gives_skip_only():
    rng = _rng(17)
    p = _problem(rng, L=33)
    zero = np.zeros_like(p["delta"])
    r = oracle.scan_fwd(p["u"], zero, p["A"], p["Bm"], p["Cm"], Dskip=p["Dskip"],
                        softplus=False)
    np.testing.assert_array_equal(r["y"], p["Dskip"][None, :, None] * p["u"])
    np.testing.assert_array_equal(r["final_state"], 0.0)
    # the same limit through softplus: delta_raw -> -inf makes delta underflow to 0
    r2 = oracle.scan_fwd(p["u"], np.full_like(p["delta"], -1000.0), p["A"], p["Bm"],
                         p["Cm"], Dskip=p["Dskip"], softplus=True)
    np.testing.assert_array_equal(r2["y"], p["Dskip"][None, :, None] * p["u"])


def test_scan_A_zero_is_prefix_sum():
    rng = _rng(19)
    p = _problem(rng, B=2, D=2, N=3, L=45)
    A0 = np.zeros_like(p["A"])
    r = oracle.scan_fwd(p["u"], p["delta"], A0, p["Bm"], p["Cm"], Dskip=None,
                        delta_bias=p["delta_bias"])
    dt = np.log1p(np.exp(p["delta"] + p["delta_bias"][None, :, None]))
    contrib = dt[:, :, None, :] * p["Bm"][:, None, :, :] * p["u"][:, :, None, :]  # [B,D,N,L]
    h = np.cumsum(contrib, axis=-1)
    y = np.einsum("bdnl,bnl->bdl", h, p["Cm"])
    np.testing.assert_allclose(r["y"], y, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(r["final_state"], h[..., -1], rtol=1e-12, atol=1e-12)


def _brute_force_y(u, dt, A, Bm, Cm, Dskip, seq):
    """h_t = sum_{s<=t, same doc} exp(A * sum_{s<r<=t} dt_r) dt_s B_s u_s."""
    B_, D, L = u.shape
    N = A.shape[1]
    y = np.zeros_like(u)
    for b in range(B_):
        for d in range(D):
            for t in range(L):
                acc = Dskip[d] * u[b, d, t]
                for s in range(t + 1):
                    if seq is not None and np.any(seq[b, s:t + 1] != seq[b, t]):
                        continue
                    decay = np.exp(A[d] * dt[b, d, s + 1:t + 1].sum())
                    acc += np.sum(Cm[b, :, t] * decay * dt[b, d, s] * Bm[b, :, s]) * u[b, d, s]
                y[b, d, t] = acc
    assert N == Bm.shape[1]
    return y


@pytest.mark.parametrize("packed", [False, True])
def test_scan_unrolled_sum_brute_force(packed):
    rng = _rng(23)
    L = 48
    seq = None
    if packed:
        seq = np.zeros((2, L), dtype=np.int32)
        seq[0, 10:] = 1
        seq[0, 11:] = 2
        seq[0, 30:] = 3
        seq[1, 47:] = 5
    p = _problem(rng, B=2, D=2, N=3, L=L, seq=seq)
    r = oracle.scan_fwd(p["u"], p["delta"], p["A"], p["Bm"], p["Cm"], Dskip=p["Dskip"],
                        delta_bias=p["delta_bias"], seq_idx=seq)
    dt = np.log1p(np.exp(p["delta"] + p["delta_bias"][None, :, None]))
    y = _brute_force_y(p["u"], dt, p["A"], p["Bm"], p["Cm"], p["Dskip"], seq)
    np.testing.assert_allclose(r["y"], y, rtol=1e-11, atol=1e-12)


def test_scan_lti_is_causal_convolution():
    # delta, B, C constant in t: y = u * K + D u with K_k = sum_n C_n e^{k dt A_n} dt B_n
    rng = _rng(29)
    D, N, L = 2, 4, 64
    u = rng.standard_normal((1, D, L))
    A = -rng.uniform(0.1, 1.0, size=(D, N))
    dt = np.array([0.3, 0.07])
    bv = rng.standard_normal(N)
    cv = rng.standard_normal(N)
    Bm = np.repeat(bv[None, :, None], L, axis=2)
    Cm = np.repeat(cv[None, :, None], L, axis=2)
    delta = np.repeat(dt[None, :, None], L, axis=2)
    Dskip = np.array([0.7, -0.2])
    r = oracle.scan_fwd(u, delta, A, Bm, Cm, Dskip=Dskip, softplus=False)
    for d in range(D):
        k = np.arange(L)
        K = (cv[None, :] * np.exp(k[:, None] * dt[d] * A[d][None, :]) * dt[d] * bv[None, :]).sum(1)
        y = np.convolve(u[0, d], K)[:L] + Dskip[d] * u[0, d]
        np.testing.assert_allclose(r["y"][0, d], y, rtol=1e-11, atol=1e-12)


def test_scan_associative_split():
    # (a1,b1) (+) (a2,b2) = (a1 a2, a2 b1 + b2): pieces from zero state, combined.
    rng = _rng(31)
    p = _problem(rng, B=1, D=2, N=3, L=70)
    cuts = [0, 23, 24, 70]
    full = oracle.scan_fwd(p["u"], p["delta"], p["A"], p["Bm"], p["Cm"],
                           delta_bias=p["delta_bias"])["final_state"]
    dt = np.log1p(np.exp(p["delta"] + p["delta_bias"][None, :, None]))
    P = np.ones_like(full)
    H = np.zeros_like(full)
    for s, e in zip(cuts[:-1], cuts[1:]):
        sl = np.s_[:, :, s:e]
        Hi = oracle.scan_fwd(p["u"][sl].copy(), p["delta"][sl].copy(), p["A"],
                             p["Bm"][sl].copy(), p["Cm"][sl].copy(),
                             delta_bias=p["delta_bias"])["final_state"]
        Pi = np.exp(p["A"][None] * dt[sl].sum(-1)[..., None])
        H = Pi * H + Hi
        P = P * Pi
    np.testing.assert_allclose(H, full, rtol=1e-12, atol=1e-13)


def test_scan_linear_in_u():
    rng = _rng(37)
    p = _problem(rng, L=30)
    u2 = rng.standard_normal(p["u"].shape)
    kw = dict(Dskip=p["Dskip"], delta_bias=p["delta_bias"])
    y1 = oracle.scan_fwd(p["u"], p["delta"], p["A"], p["Bm"], p["Cm"], **kw)["out"]
    y2 = oracle.scan_fwd(u2, p["delta"], p["A"], p["Bm"], p["Cm"], **kw)["out"]
    y3 = oracle.scan_fwd(2.5 * p["u"] - 0.5 * u2, p["delta"], p["A"], p["Bm"], p["Cm"], **kw)["out"]
    np.testing.assert_allclose(y3, 2.5 * y1 - 0.5 * y2, rtol=1e-11, atol=1e-12)


def test_scan_hand_worked_golden():
    with open(os.path.join(GOLDEN, "hand_worked_s6.json")) as f:
        g = json.load(f)
    for c in g["cases"]:
        L = len(c["u"])
        u = np.array(c["u"], dtype=np.float64).reshape(1, 1, L)
        dl = np.array(c["delta"], dtype=np.float64).reshape(1, 1, L)
        A = np.array(c["A"], dtype=np.float64).reshape(1, -1)
        Bm = np.array(c["Bm"], dtype=np.float64)[None]
        Cm = np.array(c["Cm"], dtype=np.float64)[None]
        seq = None if c["seq_idx"] is None else np.array(c["seq_idx"], dtype=np.int32)[None]
        r = oracle.scan_fwd(u, dl, A, Bm, Cm, Dskip=np.array([c["D"]]), softplus=False,
                            seq_idx=seq)
        np.testing.assert_allclose(r["y"][0, 0], c["y"], rtol=1e-14, atol=1e-14, err_msg=c["name"])
        np.testing.assert_allclose(r["final_state"][0, 0], c["final_state"], rtol=1e-14,
                                   atol=1e-14, err_msg=c["name"])


# --------------------------------------------------------------------------
# packing: a packed batch equals its documents run separately
# --------------------------------------------------------------------------
def test_scan_packed_equals_separate():
    rng = _rng(41)
    L = 57
    cuts = [0, 1, 2, 20, 21, 50, L]
    seq = np.zeros((1, L), dtype=np.int32)
    for i in range(len(cuts) - 1):
        seq[0, cuts[i]:cuts[i + 1]] = 10 - i  # ids need not increase
    p = _problem(rng, B=1, D=2, N=3, L=L, seq=seq)
    dout = rng.standard_normal(p["u"].shape)
    kw = dict(z=p["z"], Dskip=p["Dskip"], delta_bias=p["delta_bias"])
    f = oracle.scan_fwd(p["u"], p["delta"], p["A"], p["Bm"], p["Cm"], seq_idx=seq, **kw)
    g = oracle.scan_bwd(p["u"], p["delta"], p["A"], p["Bm"], p["Cm"], dout, seq_idx=seq, **kw)
    acc = {k: np.zeros_like(g[k]) for k in ("dA", "dD", "ddelta_bias")}
    for s, e in zip(cuts[:-1], cuts[1:]):
        sl = np.s_[:, :, s:e]
        kw_i = dict(z=p["z"][sl].copy(), Dskip=p["Dskip"], delta_bias=p["delta_bias"])
        fi = oracle.scan_fwd(p["u"][sl].copy(), p["delta"][sl].copy(), p["A"],
                             p["Bm"][sl].copy(), p["Cm"][sl].copy(), **kw_i)
        gi = oracle.scan_bwd(p["u"][sl].copy(), p["delta"][sl].copy(), p["A"],
                             p["Bm"][sl].copy(), p["Cm"][sl].copy(), dout[sl].copy(), **kw_i)
        np.testing.assert_array_equal(f["out"][sl], fi["out"])
        for k in ("du", "ddelta", "dz", "dB", "dC"):
            np.testing.assert_array_equal(g[k][sl], gi[k], err_msg=k)
        for k in acc:
            acc[k] += gi[k]
        if e == L:
            np.testing.assert_array_equal(f["final_state"], fi["final_state"])
    for k in acc:
        np.testing.assert_allclose(g[k], acc[k], rtol=1e-12, atol=1e-13, err_msg=k)


# --------------------------------------------------------------------------
# backward: finite differences and closed forms
# --------------------------------------------------------------------------
@pytest.mark.parametrize("softplus", [True, False])
def test_scan_bwd_finite_differences(softplus):
    inp = synth.make_inputs(synth.CONFIGS[1], synth.seed_for(1), dskip_random=True)
    rng = _rng(43)
    p = dict(u=rng.standard_normal((1, 4, 64)), delta=inp.delta.f64.copy(), z=inp.z.f64.copy(),
             A=inp.A.astype(np.float64), Bm=inp.Bm.f64.copy(), Cm=inp.Cm.f64.copy(),
             Dskip=inp.Dskip.astype(np.float64), delta_bias=inp.delta_bias.astype(np.float64))
    if not softplus:
        p["delta"] = np.abs(p["delta"]) * 0.2
        p["delta_bias"] = np.zeros_like(p["delta_bias"])
    seq = inp.seq_idx
    dout = inp.dout.f64

    def loss():
        r = oracle.scan_fwd(p["u"], p["delta"], p["A"], p["Bm"], p["Cm"], z=p["z"],
                            Dskip=p["Dskip"], delta_bias=p["delta_bias"], softplus=softplus,
                            seq_idx=seq)
        return float(np.sum(r["out"] * dout))

    g = oracle.scan_bwd(p["u"], p["delta"], p["A"], p["Bm"], p["Cm"], dout, z=p["z"],
                        Dskip=p["Dskip"], delta_bias=p["delta_bias"], softplus=softplus,
                        seq_idx=seq)
    pairs = [("u", "du"), ("delta", "ddelta"), ("z", "dz"), ("A", "dA"), ("Bm", "dB"),
             ("Cm", "dC"), ("Dskip", "dD"), ("delta_bias", "ddelta_bias")]
    for name, gname in pairs:
        _close(_fd(loss, p[name]), g[gname])


def test_scan_dD_closed_form():
    rng = _rng(47)
    p = _problem(rng, B=2, D=3, N=2, L=25)
    dout = rng.standard_normal(p["u"].shape)
    g = oracle.scan_bwd(p["u"], p["delta"], p["A"], p["Bm"], p["Cm"], dout, z=p["z"],
                        Dskip=p["Dskip"], delta_bias=p["delta_bias"])
    dy = dout * p["z"] * _sig(p["z"])
    np.testing.assert_allclose(g["dD"], (dy * p["u"]).sum(axis=(0, 2)), rtol=1e-12)


def test_layer_chain_finite_differences():
    """conv -> scan -> gate, end to end, against finite differences in x, w, bias."""
    inp = synth.make_inputs(synth.CONFIGS[1], synth.seed_for(1), conv_bias_scale=0.3)
    x = inp.x.f64.copy()
    w = inp.conv_w.astype(np.float64)
    cb = inp.conv_b.astype(np.float64)
    seq = inp.seq_idx

    def loss():
        _, u = oracle.conv1d_fwd(x, w, cb, seq)
        r = oracle.scan_fwd(u, inp.delta.f64, inp.A, inp.Bm.f64, inp.Cm.f64, z=inp.z.f64,
                            Dskip=inp.Dskip, delta_bias=inp.delta_bias, seq_idx=seq)
        return float(np.sum(r["out"] * inp.dout.f64))

    r = oracle.layer_fwd_bwd(inp, bf16_points=False)
    _close(_fd(loss, x), r["dx"])
    _close(_fd(loss, w), r["dconv_w"])
    _close(_fd(loss, cb), r["dconv_b"])


def test_threaded_driver_matches_single_thread():
    rng = _rng(53)
    p = _problem(rng, B=2, D=5, N=4, L=31)
    dout = rng.standard_normal(p["u"].shape)
    kw = dict(z=p["z"], Dskip=p["Dskip"], delta_bias=p["delta_bias"])
    f1 = oracle.scan_fwd(p["u"], p["delta"], p["A"], p["Bm"], p["Cm"], **kw)
    f4 = oracle.scan_fwd(p["u"], p["delta"], p["A"], p["Bm"], p["Cm"], nthreads=4, **kw)
    np.testing.assert_array_equal(f1["out"], f4["out"])
    g1 = oracle.scan_bwd(p["u"], p["delta"], p["A"], p["Bm"], p["Cm"], dout, **kw)
    g4 = oracle.scan_bwd(p["u"], p["delta"], p["A"], p["Bm"], p["Cm"], dout, nthreads=4, **kw)
    for k in g1:
        np.testing.assert_allclose(g1[k], g4[k], rtol=1e-12, atol=1e-13, err_msg=k)


def test_softplus_reading_is_exact_log1p_exp():
    # delta = log(1 + e^v): check the oracle's step against a direct evaluation
    u = np.ones((1, 1, 5))
    v = np.array([-30.0, -1.0, 0.0, 1.0, 30.0]).reshape(1, 1, 5)
    A = np.zeros((1, 1))
    Bm = np.zeros((1, 1, 5))
    Bm[0, 0, :] = 1.0
    Cm = np.ones((1, 1, 5))
    y = oracle.scan_fwd(u, v, A, Bm, Cm, softplus=True)["y"][0, 0]
    want = np.cumsum([math.log1p(math.exp(t)) for t in v.ravel()])
    np.testing.assert_allclose(y, want, rtol=1e-14)


# --------------------------------------------------------------------------
# initial state and the recurrent (decode) form
# --------------------------------------------------------------------------
def test_scan_h0_continues_a_prefix():
    """A suffix started from the prefix's final state reproduces the full run
    (the recurrence carries nothing else across the cut)."""
    rng = _rng(61)
    p = _problem(rng, B=2, D=3, N=4, L=40)
    full = oracle.scan_fwd(p["u"], p["delta"], p["A"], p["Bm"], p["Cm"], z=p["z"],
                           Dskip=p["Dskip"], delta_bias=p["delta_bias"])
    for s in (1, 17, 39):
        pre = oracle.scan_fwd(p["u"][..., :s], p["delta"][..., :s], p["A"], p["Bm"][..., :s],
                              p["Cm"][..., :s], z=p["z"][..., :s], Dskip=p["Dskip"],
                              delta_bias=p["delta_bias"])
        suf = oracle.scan_fwd(p["u"][..., s:], p["delta"][..., s:], p["A"], p["Bm"][..., s:],
                              p["Cm"][..., s:], z=p["z"][..., s:], Dskip=p["Dskip"],
                              delta_bias=p["delta_bias"], h0=pre["final_state"])
        np.testing.assert_allclose(suf["out"], full["out"][..., s:], rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(suf["final_state"], full["final_state"], rtol=1e-12,
                                   atol=1e-12)


def test_scan_h0_reset_at_document_start():
    """With seq_idx, h0 feeds the first document only."""
    rng = _rng(62)
    seq = np.array([[0] * 12 + [1] * 20], dtype=np.int32)
    p = _problem(rng, B=1, D=2, N=3, L=32, seq=seq)
    h0 = rng.standard_normal((1, 2, 3))
    a = oracle.scan_fwd(p["u"], p["delta"], p["A"], p["Bm"], p["Cm"], seq_idx=seq, h0=h0)
    b = oracle.scan_fwd(p["u"], p["delta"], p["A"], p["Bm"], p["Cm"], seq_idx=seq)
    assert np.abs(a["out"][..., :12] - b["out"][..., :12]).max() > 1e-6
    np.testing.assert_array_equal(a["out"][..., 12:], b["out"][..., 12:])


@pytest.mark.parametrize("softplus", [True, False])
def test_scan_bwd_h0_finite_differences(softplus):
    """dh0, and the h0 term inside dA and d(delta), against finite differences."""
    rng = _rng(63)
    p = _problem(rng, B=2, D=3, N=4, L=24)
    if not softplus:
        p["delta"] = np.abs(p["delta"]) * 0.2
        p["delta_bias"] = np.zeros_like(p["delta_bias"])
    h0 = rng.standard_normal((2, 3, 4))
    dout = rng.standard_normal(p["u"].shape)

    def loss():
        r = oracle.scan_fwd(p["u"], p["delta"], p["A"], p["Bm"], p["Cm"], z=p["z"],
                            Dskip=p["Dskip"], delta_bias=p["delta_bias"], softplus=softplus,
                            h0=h0)
        return float(np.sum(r["out"] * dout))

    g = oracle.scan_bwd(p["u"], p["delta"], p["A"], p["Bm"], p["Cm"], dout, z=p["z"],
                        Dskip=p["Dskip"], delta_bias=p["delta_bias"], softplus=softplus, h0=h0)
    _close(_fd(loss, h0), g["dh0"])
    _close(_fd(loss, p["A"]), g["dA"])
    _close(_fd(loss, p["delta"]), g["ddelta"])


def test_decode_steps_equal_the_sequence_form():
    """Stepping the recurrent form over a sequence from a zero conv window and
    a zero state gives the sequence form's u, out and final state."""
    rng = _rng(64)
    B, D, N, L, W = 2, 3, 4, 30, 4
    p = _problem(rng, B=B, D=D, N=N, L=L)
    x = rng.standard_normal((B, D, L))
    w = rng.uniform(-0.5, 0.5, size=(D, W))
    cb = rng.uniform(-0.2, 0.2, size=D)
    _, u = oracle.conv1d_fwd(x, w, cb, None)
    full = oracle.scan_fwd(u, p["delta"], p["A"], p["Bm"], p["Cm"], z=p["z"],
                           Dskip=p["Dskip"], delta_bias=p["delta_bias"])
    cs = np.zeros((B, D, W - 1))
    h = np.zeros((B, D, N))
    for t in range(L):
        out, ut, cs, h = oracle.decode_step(x[..., t], cs, w, cb, p["delta"][..., t],
                                            p["Bm"][..., t], p["Cm"][..., t], p["A"], h,
                                            z=p["z"][..., t], Dskip=p["Dskip"],
                                            delta_bias=p["delta_bias"])
        np.testing.assert_allclose(ut, u[..., t], rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(out, full["out"][..., t], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(h, full["final_state"], rtol=1e-12, atol=1e-12)
    np.testing.assert_array_equal(cs, x[..., L - W + 1:])


def test_decode_continues_a_prefill():
    """Prefill with the sequence form, then decode: conv window = the last
    W-1 inputs, state = the prefill's final state."""
    rng = _rng(65)
    B, D, N, L, W, s = 1, 2, 3, 20, 4, 13
    p = _problem(rng, B=B, D=D, N=N, L=L)
    x = rng.standard_normal((B, D, L))
    w = rng.uniform(-0.5, 0.5, size=(D, W))
    _, u = oracle.conv1d_fwd(x, w, None, None)
    full = oracle.scan_fwd(u, p["delta"], p["A"], p["Bm"], p["Cm"], Dskip=p["Dskip"],
                           delta_bias=p["delta_bias"])
    pre = oracle.scan_fwd(u[..., :s], p["delta"][..., :s], p["A"], p["Bm"][..., :s],
                          p["Cm"][..., :s], Dskip=p["Dskip"], delta_bias=p["delta_bias"])
    cs, h = x[..., s - W + 1:s].copy(), pre["final_state"]
    for t in range(s, L):
        out, _, cs, h = oracle.decode_step(x[..., t], cs, w, None, p["delta"][..., t],
                                           p["Bm"][..., t], p["Cm"][..., t], p["A"], h,
                                           Dskip=p["Dskip"], delta_bias=p["delta_bias"])
        np.testing.assert_allclose(out, full["out"][..., t], rtol=1e-12, atol=1e-12)


# --------------------------------------------------------------------------
# zero-order-hold discretisation ("Discretization": B_bar = A^-1 (exp(dA) - I) B)
# --------------------------------------------------------------------------
def test_zoh_equals_ode_integration():
    """ZOH is the exact solution of dh/dtau = A h + B u over a step of length
    dt with u and B held constant: integrate that ODE with fine RK4 steps
    from the previous state (zero at a document start) and compare."""
    rng = _rng(71)
    seq = np.array([[0, 0, 0, 1, 1, 1, 1]], dtype=np.int32)
    p = _problem(rng, B=1, D=2, N=3, L=7, seq=seq)
    r = oracle.scan_fwd(p["u"], p["delta"], p["A"], p["Bm"], p["Cm"], z=p["z"], Dskip=p["Dskip"],
                        delta_bias=p["delta_bias"], seq_idx=seq, zoh=True)
    v = p["delta"] + p["delta_bias"][None, :, None]
    dt = np.log1p(np.exp(v))
    out = np.zeros_like(p["u"])
    for d in range(2):
        h = np.zeros(3)
        for t in range(7):
            if t > 0 and seq[0, t] != seq[0, t - 1]:
                h = np.zeros(3)
            A, Bv, u = p["A"][d], p["Bm"][0, :, t], p["u"][0, d, t]
            steps = 2000
            k = dt[0, d, t] / steps
            f = lambda hh: A * hh + Bv * u  # noqa: E731
            for _ in range(steps):
                k1 = f(h)
                k2 = f(h + 0.5 * k * k1)
                k3 = f(h + 0.5 * k * k2)
                k4 = f(h + k * k3)
                h = h + k / 6.0 * (k1 + 2 * k2 + 2 * k3 + k4)
            y = float(p["Cm"][0, :, t] @ h) + p["Dskip"][d] * u
            out[0, d, t] = y * p["z"][0, d, t] * _sig(p["z"][0, d, t])
    np.testing.assert_allclose(r["out"], out, rtol=1e-10, atol=1e-12)


def test_zoh_lti_is_causal_convolution():
    """Constant dt, B, C: y = u * K + D u with K_k = sum_n C_n A_bar^k phi_n B_n,
    phi_n = (exp(dt A_n) - 1) / A_n."""
    rng = _rng(72)
    L, N = 50, 4
    A = -rng.uniform(0.2, 2.0, size=(1, N))
    Bc, Cc = rng.standard_normal(N), rng.standard_normal(N)
    u = rng.standard_normal((1, 1, L))
    dt = 0.3
    r = oracle.scan_fwd(u, np.full((1, 1, L), dt), A, np.tile(Bc[None, :, None], (1, 1, L)),
                        np.tile(Cc[None, :, None], (1, 1, L)), Dskip=np.array([0.7]),
                        softplus=False, zoh=True)
    a = np.exp(dt * A[0])
    phi = np.expm1(dt * A[0]) / A[0]
    K = np.array([np.sum(Cc * a ** k * phi * Bc) for k in range(L)])
    want = np.convolve(u[0, 0], K)[:L] + 0.7 * u[0, 0]
    np.testing.assert_allclose(r["out"][0, 0], want, rtol=1e-12, atol=1e-12)


def test_zoh_small_A_limit_is_dt_B():
    """As A -> 0 the ZOH factor (exp(dt A) - 1) / A tends to dt."""
    rng = _rng(73)
    p = _problem(rng, B=1, D=2, N=3, L=20)
    A = np.full((2, 3), -1e-9)
    a = oracle.scan_fwd(p["u"], p["delta"], A, p["Bm"], p["Cm"], delta_bias=p["delta_bias"], zoh=True)
    b = oracle.scan_fwd(p["u"], p["delta"], A, p["Bm"], p["Cm"], delta_bias=p["delta_bias"])
    np.testing.assert_allclose(a["out"], b["out"], rtol=1e-7, atol=1e-12)


@pytest.mark.parametrize("softplus", [True, False])
def test_zoh_bwd_finite_differences(softplus):
    """Every gradient of the ZOH scan (incl. dA through B_bar and dh0)."""
    rng = _rng(74)
    p = _problem(rng, B=2, D=3, N=4, L=20, seq=np.array([[0] * 8 + [1] * 12, [0] * 20],
                                                        dtype=np.int32))
    if not softplus:
        p["delta"] = np.abs(p["delta"]) * 0.2
        p["delta_bias"] = np.zeros_like(p["delta_bias"])
    p["A"][0, 0] = -1e-5  # exercises the series branch of dB_bar/dA
    h0 = rng.standard_normal((2, 3, 4))
    dout = rng.standard_normal(p["u"].shape)
    kw = dict(z=p["z"], Dskip=p["Dskip"], delta_bias=p["delta_bias"], softplus=softplus,
              seq_idx=p["seq_idx"], h0=h0, zoh=True)

    def loss():
        r = oracle.scan_fwd(p["u"], p["delta"], p["A"], p["Bm"], p["Cm"], **kw)
        return float(np.sum(r["out"] * dout))

    g = oracle.scan_bwd(p["u"], p["delta"], p["A"], p["Bm"], p["Cm"], dout, **kw)
    for name, gname in [("u", "du"), ("delta", "ddelta"), ("z", "dz"), ("A", "dA"),
                        ("Bm", "dB"), ("Cm", "dC"), ("Dskip", "dD"),
                        ("delta_bias", "ddelta_bias")]:
        _close(_fd(loss, p[name]), g[gname])
    _close(_fd(loss, h0), g["dh0"])


# --------------------------------------------------------------------------
# complex diagonal A (S4D form): h_t = exp(dt A) h_{t-1} + dt u B_t,
# y = 2 Re(sum_n C_t h_t) + D u
# --------------------------------------------------------------------------
def _cproblem(rng, B=2, D=3, N=4, L=20, seq=None):
    p = _problem(rng, B=B, D=D, N=N, L=L, seq=seq)
    p["A"] = p["A"] + 1j * np.pi * rng.integers(0, 4, size=(D, N))  # S4D-Lin style phases
    p["Bm"] = p["Bm"] + 1j * rng.standard_normal((B, N, L))
    p["Cm"] = p["Cm"] + 1j * rng.standard_normal((B, N, L))
    return p


def test_cscan_real_case_equals_real_scan():
    """Imaginary parts zero: the complex scan is the real scan with C doubled,
    forward and every gradient (dC picks up the same factor 2)."""
    rng = _rng(81)
    seq = np.array([[0] * 9 + [1] * 11, [0] * 20], dtype=np.int32)
    p = _problem(rng, B=2, D=3, N=4, L=20, seq=seq)
    h0 = rng.standard_normal((2, 3, 4))
    dout = rng.standard_normal(p["u"].shape)
    kw = dict(z=p["z"], Dskip=p["Dskip"], delta_bias=p["delta_bias"], seq_idx=seq, h0=h0)
    c = oracle.cscan_fwd(p["u"], p["delta"], p["A"] + 0j, p["Bm"] + 0j, p["Cm"] + 0j, **kw)
    r = oracle.scan_fwd(p["u"], p["delta"], p["A"], p["Bm"], 2 * p["Cm"], **kw)
    np.testing.assert_allclose(c["out"], r["out"], rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(c["final_state"].real, r["final_state"], rtol=1e-13, atol=1e-13)
    assert np.all(c["final_state"].imag == 0)
    gc = oracle.cscan_bwd(p["u"], p["delta"], p["A"] + 0j, p["Bm"] + 0j, p["Cm"] + 0j, dout, **kw)
    gr = oracle.scan_bwd(p["u"], p["delta"], p["A"], p["Bm"], 2 * p["Cm"], dout, **kw)
    for k in ("du", "ddelta", "dz", "dD", "ddelta_bias"):
        np.testing.assert_allclose(gc[k], gr[k], rtol=1e-12, atol=1e-12)
    for k in ("dA", "dB", "dh0"):
        np.testing.assert_allclose(gc[k].real, gr[k], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(gc["dC"].real, 2 * gr["dC"], rtol=1e-12, atol=1e-12)


def test_cscan_unrolled_sum_brute_force():
    """y_t = 2 Re sum_n C_t,n [ sum_{s<=t, same document} prod_{s<r<=t} a_r dt_s u_s B_s
    + prod_{r<=t} a_r h0 (if t is in the first document) ] + D u_t, by numpy
    complex products, no recurrence."""
    rng = _rng(82)
    B, D, N, L = 2, 2, 3, 17
    seq = np.array([[0] * 6 + [1] * 11, [0] * 17], dtype=np.int32)
    p = _cproblem(rng, B=B, D=D, N=N, L=L, seq=seq)
    p["A"] += 1j * rng.standard_normal((D, N))
    h0 = rng.standard_normal((B, D, N)) + 1j * rng.standard_normal((B, D, N))
    c = oracle.cscan_fwd(p["u"], p["delta"], p["A"], p["Bm"], p["Cm"], z=None,
                         Dskip=p["Dskip"], delta_bias=p["delta_bias"], seq_idx=seq, h0=h0)
    dt = np.log1p(np.exp(p["delta"] + p["delta_bias"][None, :, None]))
    want = np.empty((B, D, L))
    for b in range(B):
        for d in range(D):
            for t in range(L):
                acc = 0j
                for n in range(N):
                    hn = 0j
                    for s in range(t + 1):
                        if seq[b, s] != seq[b, t]:
                            continue
                        decay = np.prod(np.exp(dt[b, d, s + 1:t + 1] * p["A"][d, n]))
                        hn += decay * dt[b, d, s] * p["u"][b, d, s] * p["Bm"][b, n, s]
                    if seq[b, t] == seq[b, 0]:
                        hn += np.prod(np.exp(dt[b, d, :t + 1] * p["A"][d, n])) * h0[b, d, n]
                    acc += p["Cm"][b, n, t] * hn
                want[b, d, t] = 2 * acc.real + p["Dskip"][d] * p["u"][b, d, t]
    np.testing.assert_allclose(c["y"], want, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(c["out"], want, rtol=1e-12, atol=1e-12)


def test_cscan_pure_rotation_keeps_modulus():
    """Re A = 0, no input after t=0: |h_t| = |h_0| and arg h_t advances by
    Im(A) * sum dt (a lossless oscillator)."""
    rng = _rng(83)
    B, D, N, L = 1, 1, 2, 12
    u = np.zeros((B, D, L))
    u[0, 0, 0] = 1.0
    delta = 0.3 * rng.standard_normal((B, D, L))
    A = np.array([[1.7j, -0.4j]])
    Bm = np.ones((B, N, L)) + 0j
    Cm = np.zeros((B, N, L)) + 0j
    c = oracle.cscan_fwd(u, delta, A, Bm, Cm, delta_bias=np.zeros(1))
    dt = np.log1p(np.exp(delta[0, 0]))
    h_end = c["final_state"][0, 0]
    np.testing.assert_allclose(np.abs(h_end), dt[0], rtol=1e-13)
    phase = A[0].imag * dt[1:].sum()
    np.testing.assert_allclose(h_end, dt[0] * np.exp(1j * phase), rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("softplus", [True, False])
def test_cscan_bwd_finite_differences(softplus):
    """Every gradient of the complex scan, each complex input through its real
    and imaginary parts, with a document reset and an initial state."""
    rng = _rng(84)
    seq = np.array([[0] * 8 + [1] * 12, [0] * 20], dtype=np.int32)
    p = _cproblem(rng, seq=seq)
    p["A"] = p["A"] + 1j * rng.standard_normal(p["A"].shape)
    if not softplus:
        p["delta"] = np.abs(p["delta"]) * 0.2
        p["delta_bias"] = np.zeros_like(p["delta_bias"])
    h0 = rng.standard_normal((2, 3, 4)) + 1j * rng.standard_normal((2, 3, 4))
    dout = rng.standard_normal(p["u"].shape)
    parts = {"u": p["u"], "delta": p["delta"], "z": p["z"], "Dskip": p["Dskip"],
             "delta_bias": p["delta_bias"]}
    for k, v in (("A", p["A"]), ("Bm", p["Bm"]), ("Cm", p["Cm"]), ("h0", h0)):
        parts[k + ".re"] = np.ascontiguousarray(v.real)
        parts[k + ".im"] = np.ascontiguousarray(v.imag)

    def cx(k):
        return parts[k + ".re"] + 1j * parts[k + ".im"]

    def loss():
        r = oracle.cscan_fwd(parts["u"], parts["delta"], cx("A"), cx("Bm"), cx("Cm"),
                             z=parts["z"], Dskip=parts["Dskip"], delta_bias=parts["delta_bias"],
                             softplus=softplus, seq_idx=seq, h0=cx("h0"))
        return float(np.sum(r["out"] * dout))

    g = oracle.cscan_bwd(p["u"], p["delta"], p["A"], p["Bm"], p["Cm"], dout, z=p["z"],
                         Dskip=p["Dskip"], delta_bias=p["delta_bias"], softplus=softplus,
                         seq_idx=seq, h0=h0)
    for name, gname in [("u", "du"), ("delta", "ddelta"), ("z", "dz"), ("Dskip", "dD"),
                        ("delta_bias", "ddelta_bias")]:
        _close(_fd(loss, parts[name]), g[gname])
    for name, gname in [("A", "dA"), ("Bm", "dB"), ("Cm", "dC"), ("h0", "dh0")]:
        _close(_fd(loss, parts[name + ".re"]), g[gname].real)
        _close(_fd(loss, parts[name + ".im"]), g[gname].imag)


# --------------------------------------------------------------------------
# a gradient reaching the final state from outside (dhL)
# --------------------------------------------------------------------------
@pytest.mark.parametrize("zoh", [False, True])
def test_scan_bwd_final_state_gradient_fd(zoh):
    """loss = <out, dout> + <final state, dhL>: every gradient against finite
    differences, with a reset (which must stop dhL) and an initial state."""
    rng = _rng(91)
    seq = np.array([[0] * 6 + [1] * 14, [0] * 20], dtype=np.int32)
    p = _problem(rng, B=2, D=3, N=4, L=20, seq=seq)
    h0 = rng.standard_normal((2, 3, 4))
    dout = rng.standard_normal(p["u"].shape)
    dhL = rng.standard_normal((2, 3, 4))
    kw = dict(z=p["z"], Dskip=p["Dskip"], delta_bias=p["delta_bias"], seq_idx=seq, zoh=zoh)

    def loss():
        r = oracle.scan_fwd(p["u"], p["delta"], p["A"], p["Bm"], p["Cm"], h0=h0, **kw)
        return float(np.sum(r["out"] * dout) + np.sum(r["final_state"] * dhL))

    g = oracle.scan_bwd(p["u"], p["delta"], p["A"], p["Bm"], p["Cm"], dout, h0=h0, dhL=dhL, **kw)
    for name, gname in [("u", "du"), ("delta", "ddelta"), ("z", "dz"), ("A", "dA"),
                        ("Bm", "dB"), ("Cm", "dC"), ("Dskip", "dD"),
                        ("delta_bias", "ddelta_bias")]:
        _close(_fd(loss, p[name]), g[gname])
    _close(_fd(loss, h0), g["dh0"])
    # the reset at t=6 of row 0 stops dhL from reaching h0 there
    g0 = oracle.scan_bwd(p["u"], p["delta"], p["A"], p["Bm"], p["Cm"], dout, h0=h0, **kw)
    np.testing.assert_allclose(g["dh0"][0], g0["dh0"][0], rtol=1e-13, atol=1e-13)
    assert np.abs(g["dh0"][1] - g0["dh0"][1]).max() > 1e-6


def test_cscan_bwd_final_state_gradient_fd():
    rng = _rng(92)
    seq = np.array([[0] * 11 + [1] * 9, [0] * 20], dtype=np.int32)
    p = _cproblem(rng, seq=seq)
    p["A"] = p["A"] + 1j * rng.standard_normal(p["A"].shape)
    h0 = rng.standard_normal((2, 3, 4)) + 1j * rng.standard_normal((2, 3, 4))
    dhL = rng.standard_normal((2, 3, 4)) + 1j * rng.standard_normal((2, 3, 4))
    dout = rng.standard_normal(p["u"].shape)
    parts = {"u": p["u"], "delta": p["delta"]}
    for k, v in (("A", p["A"]), ("Bm", p["Bm"]), ("Cm", p["Cm"]), ("h0", h0)):
        parts[k + ".re"] = np.ascontiguousarray(v.real)
        parts[k + ".im"] = np.ascontiguousarray(v.imag)
    kw = dict(z=p["z"], Dskip=p["Dskip"], delta_bias=p["delta_bias"], seq_idx=seq)

    def cx(k):
        return parts[k + ".re"] + 1j * parts[k + ".im"]

    def loss():
        r = oracle.cscan_fwd(parts["u"], parts["delta"], cx("A"), cx("Bm"), cx("Cm"), h0=cx("h0"),
                             **kw)
        fs = r["final_state"]
        return float(np.sum(r["out"] * dout) + np.sum(fs.real * dhL.real + fs.imag * dhL.imag))

    g = oracle.cscan_bwd(p["u"], p["delta"], p["A"], p["Bm"], p["Cm"], dout, h0=h0, dhL=dhL, **kw)
    _close(_fd(loss, parts["u"]), g["du"])
    _close(_fd(loss, parts["delta"]), g["ddelta"])
    for name, gname in [("A", "dA"), ("Bm", "dB"), ("Cm", "dC"), ("h0", "dh0")]:
        _close(_fd(loss, parts[name + ".re"]), g[gname].real)
        _close(_fd(loss, parts[name + ".im"]), g[gname].imag)


# --------------------------------------------------------------------------
# Mamba-2 SSD form (scalar A per head, heads, groups of shared B / C)
# --------------------------------------------------------------------------
def _ssd_problem(rng, B=2, L=14, H=4, P=3, G=2, N=5):
    return dict(x=rng.standard_normal((B, L, H, P)), dt_raw=0.5 * rng.standard_normal((B, L, H)),
                A=-rng.uniform(0.3, 2.0, size=H), Bm=rng.standard_normal((B, L, G, N)),
                Cm=rng.standard_normal((B, L, G, N)), D=rng.uniform(0.5, 1.5, size=H),
                dt_bias=rng.uniform(-2.0, -0.5, size=H))


def test_ssd_equals_its_attention_form():
    """The duality the SSD section states: per head, Y = (M o C B^T)(dt x) +
    D x with M[i][j] = exp(A sum_{j<k<=i} dt_k) for j <= i in the same
    document, 0 otherwise (numpy matrices, no recurrence)."""
    rng = _rng(95)
    p = _ssd_problem(rng)
    B, L, H, P = p["x"].shape
    G = p["Bm"].shape[2]
    seq = np.array([[0] * 6 + [1] * 8, [0] * 14], dtype=np.int32)
    y = oracle.ssd_fwd(p["x"], p["dt_raw"], p["A"], p["Bm"], p["Cm"], D=p["D"],
                       dt_bias=p["dt_bias"], seq_idx=seq)["y"]
    dt = np.log1p(np.exp(p["dt_raw"] + p["dt_bias"][None, None, :]))
    want = np.empty_like(y)
    for b in range(B):
        for h in range(H):
            g = h // (H // G)
            cs = np.cumsum(dt[b, :, h] * p["A"][h])
            M = np.exp(cs[:, None] - cs[None, :])
            M *= np.tril(np.ones((L, L)))
            M *= seq[b][:, None] == seq[b][None, :]
            CB = p["Cm"][b, :, g, :] @ p["Bm"][b, :, g, :].T
            want[b, :, h, :] = (M * CB) @ (dt[b, :, h, None] * p["x"][b, :, h, :]) \
                + p["D"][h] * p["x"][b, :, h, :]
    np.testing.assert_allclose(y, want, rtol=1e-11, atol=1e-11)


def test_ssd_one_group_equals_the_mamba1_scan():
    """With one group, SSD is the Mamba-1 scan over H*P channels whose A is
    the head's scalar for every state, whose step is the head's and whose B
    and C are shared by all channels: both oracles (written separately) agree,
    forward and every gradient."""
    rng = _rng(96)
    p = _ssd_problem(rng, G=1)
    B, L, H, P = p["x"].shape
    N = p["Bm"].shape[3]
    seq = np.array([[0] * 5 + [1] * 9, [0] * 3 + [1] * 11], dtype=np.int32)
    dy = rng.standard_normal(p["x"].shape)
    kw = dict(D=p["D"], dt_bias=p["dt_bias"], seq_idx=seq)
    f = oracle.ssd_fwd(p["x"], p["dt_raw"], p["A"], p["Bm"], p["Cm"], **kw)
    g = oracle.ssd_bwd(p["x"], p["dt_raw"], p["A"], p["Bm"], p["Cm"], dy, **kw)
    # channel d = h P + q; activations [B, D, L]
    u = p["x"].reshape(B, L, H * P).transpose(0, 2, 1)
    delta = np.repeat(p["dt_raw"], P, axis=2).transpose(0, 2, 1)
    A1 = np.repeat(p["A"], P)[:, None] * np.ones((1, N))
    Bm1 = p["Bm"][:, :, 0, :].transpose(0, 2, 1)
    Cm1 = p["Cm"][:, :, 0, :].transpose(0, 2, 1)
    kw1 = dict(Dskip=np.repeat(p["D"], P), delta_bias=np.repeat(p["dt_bias"], P), seq_idx=seq)
    r = oracle.scan_fwd(u, delta, A1, Bm1, Cm1, **kw1)
    gr = oracle.scan_bwd(u, delta, A1, Bm1, Cm1, dy.reshape(B, L, H * P).transpose(0, 2, 1), **kw1)
    np.testing.assert_allclose(f["y"].reshape(B, L, H * P).transpose(0, 2, 1), r["out"],
                               rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(f["final_state"].reshape(B, H * P, N), r["final_state"],
                               rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(g["dx"].reshape(B, L, H * P).transpose(0, 2, 1), gr["du"],
                               rtol=1e-11, atol=1e-11)
    np.testing.assert_allclose(g["ddt_raw"], gr["ddelta"].reshape(B, H, P, L).sum(2).transpose(0, 2, 1),
                               rtol=1e-11, atol=1e-11)
    np.testing.assert_allclose(g["dA"], gr["dA"].reshape(H, P, N).sum((1, 2)), rtol=1e-11, atol=1e-11)
    np.testing.assert_allclose(g["dB"][:, :, 0, :], gr["dB"].transpose(0, 2, 1), rtol=1e-11, atol=1e-11)
    np.testing.assert_allclose(g["dC"][:, :, 0, :], gr["dC"].transpose(0, 2, 1), rtol=1e-11, atol=1e-11)
    np.testing.assert_allclose(g["dD"], gr["dD"].reshape(H, P).sum(1), rtol=1e-11, atol=1e-11)
    np.testing.assert_allclose(g["ddt_bias"], gr["ddelta_bias"].reshape(H, P).sum(1), rtol=1e-11,
                               atol=1e-11)


@pytest.mark.parametrize("softplus", [True, False])
def test_ssd_bwd_finite_differences(softplus):
    """Every SSD gradient against central differences, two groups, a reset."""
    rng = _rng(97)
    p = _ssd_problem(rng, L=10)
    if not softplus:
        p["dt_raw"] = np.abs(p["dt_raw"]) * 0.3
        p["dt_bias"] = np.zeros_like(p["dt_bias"])
    seq = np.array([[0] * 4 + [1] * 6, [0] * 10], dtype=np.int32)
    dy = rng.standard_normal(p["x"].shape)

    def loss():
        r = oracle.ssd_fwd(p["x"], p["dt_raw"], p["A"], p["Bm"], p["Cm"], D=p["D"],
                           dt_bias=p["dt_bias"], softplus=softplus, seq_idx=seq)
        return float(np.sum(r["y"] * dy))

    g = oracle.ssd_bwd(p["x"], p["dt_raw"], p["A"], p["Bm"], p["Cm"], dy, D=p["D"],
                       dt_bias=p["dt_bias"], softplus=softplus, seq_idx=seq)
    for name, gname in [("x", "dx"), ("dt_raw", "ddt_raw"), ("A", "dA"), ("Bm", "dB"),
                        ("Cm", "dC"), ("D", "dD"), ("dt_bias", "ddt_bias")]:
        _close(_fd(loss, p[name]), g[gname])
