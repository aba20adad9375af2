"""Initial state, its gradient, and the recurrent one-token form on the GPU,
against the fp64 oracle on the same seeded inputs (synth).

fp32: rel-L2 <= 1e-5. bf16 activations with fp32 state: outputs rel-L2 <=
2e-3 against the oracle rounded to bf16, gradients and states <= 5e-3.
"""
import numpy as np
import pytest

import oracle
import synth
from pipeline import TOL_BF16_OUT, TOL_F32, TOL_GRAD, f32_dev, host64, rel_l2, to_dev

pytestmark = pytest.mark.gpu


def _ssm():
    import selective_state_space_35_b200 as ssm
    return ssm


# ---------------------------------------------------------------- initial state
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("n_splits", [1, 3])
@pytest.mark.parametrize("packed", [False, True])
def test_scan_initial_state_parity(dtype, n_splits, packed):
    """Forward with h0 (out, final state) and backward (every gradient and
    dh0): D = 24 spans three CTAs of the backward, L = 1000 several 256-token
    chunks, 32-token blocks and a ragged tail."""
    import torch
    ssm = _ssm()
    B, D, N, L = 2, 24, 16, 1000
    seed = 7100 + 10 * n_splits + int(packed) + (5 if dtype == "bf16" else 0)
    inp = synth.make_inputs(synth.Shape("h0", B, D, N, L, dtype), seed, dskip_random=True)
    if packed:
        inp.seq_idx = synth.random_segments(np.random.Generator(np.random.PCG64(seed)), B, L, 6)
    h0 = synth.initial_state(B, D, N, seed + 1)
    seq = inp.seq_idx
    kw_o = dict(z=inp.z.f64, Dskip=inp.Dskip, delta_bias=inp.delta_bias, seq_idx=seq,
                h0=h0.astype(np.float64))
    f = oracle.scan_fwd(inp.x.f64, inp.delta.f64, inp.A, inp.Bm.f64, inp.Cm.f64, **kw_o)
    g = oracle.scan_bwd(inp.x.f64, inp.delta.f64, inp.A, inp.Bm.f64, inp.Cm.f64, inp.dout.f64,
                        **kw_o)

    dev = "cuda"
    u, dl, z = to_dev(inp.x, dev), to_dev(inp.delta, dev), to_dev(inp.z, dev)
    Bm, Cm, dout = to_dev(inp.Bm, dev), to_dev(inp.Cm, dev), to_dev(inp.dout, dev)
    A, Dk, db = f32_dev(inp.A, dev), f32_dev(inp.Dskip, dev), f32_dev(inp.delta_bias, dev)
    sq = torch.from_numpy(seq).to(dev) if seq is not None else None
    h0d = f32_dev(h0, dev)
    kw = dict(z=z, Dskip=Dk, delta_bias=db, seq_idx=sq, n_splits=n_splits, initial_state=h0d)
    out, fs, ws = ssm.scan_fwd(u, dl, A, Bm, Cm, return_final_state=True, **kw)
    assert ssm.scan_status(u, A, ws) == 0
    gr = ssm.scan_bwd(u, dl, A, Bm, Cm, dout, ws, **kw)
    torch.cuda.synchronize()

    fp32 = dtype == "f32"
    want_out = f["out"] if fp32 else oracle.round_bf16(f["out"])
    assert rel_l2(host64(out), want_out) <= (TOL_F32 if fp32 else TOL_BF16_OUT)
    assert rel_l2(host64(fs), f["final_state"]) <= (TOL_F32 if fp32 else TOL_GRAD)
    for k, ok in (("du", "du"), ("ddelta", "ddelta"), ("dz", "dz"), ("dA", "dA"), ("dB", "dB"),
                  ("dC", "dC"), ("dD", "dD"), ("ddelta_bias", "ddelta_bias"),
                  ("dinitial_state", "dh0")):
        w = g[ok]
        if k in ("du", "ddelta", "dz") and not fp32:
            w = oracle.round_bf16(w)
        e = rel_l2(host64(gr[k]), w)
        assert e <= (TOL_F32 if fp32 else TOL_GRAD), (k, e)


def test_scan_initial_state_zero_equals_none():
    """initial_state = 0 gives bitwise the same results as no initial state;
    dinitial_state is still the gradient with respect to the zero state."""
    import torch
    ssm = _ssm()
    B, D, N, L = 1, 16, 16, 512
    inp = synth.make_inputs(synth.Shape("h0-zero", B, D, N, L, "bf16"), 7201)
    dev = "cuda"
    args = [to_dev(inp.x, dev), to_dev(inp.delta, dev), f32_dev(inp.A, dev), to_dev(inp.Bm, dev),
            to_dev(inp.Cm, dev)]
    kw = dict(z=to_dev(inp.z, dev), Dskip=f32_dev(inp.Dskip, dev),
              delta_bias=f32_dev(inp.delta_bias, dev))
    dout = to_dev(inp.dout, dev)
    o1, _, w1 = ssm.scan_fwd(*args, **kw)
    g1 = ssm.scan_bwd(*args, dout, w1, **kw)
    zero = torch.zeros(B, D, N, device=dev)
    o2, _, w2 = ssm.scan_fwd(*args, initial_state=zero, **kw)
    g2 = ssm.scan_bwd(*args, dout, w2, initial_state=zero, **kw)
    assert torch.equal(o1, o2)
    for k in ("du", "ddelta", "dz", "dA", "dinitial_state"):
        assert torch.equal(g1[k], g2[k]), k
    f = oracle.scan_bwd(inp.x.f64, inp.delta.f64, inp.A, inp.Bm.f64, inp.Cm.f64, inp.dout.f64,
                        z=inp.z.f64, Dskip=inp.Dskip, delta_bias=inp.delta_bias)
    assert rel_l2(host64(g1["dinitial_state"]), f["dh0"]) <= TOL_GRAD


# ---------------------------------------------------------------- recurrent form
def _run_decode_gpu(di, B, D, N, steps, *, use_z=True, softplus=True):
    import torch
    ssm = _ssm()
    dev = "cuda"
    x, dl, z = to_dev(di.x, dev), to_dev(di.delta, dev), to_dev(di.z, dev)
    Bm, Cm = to_dev(di.Bm, dev), to_dev(di.Cm, dev)
    cs = to_dev(di.conv_state, dev).contiguous()
    st = f32_dev(di.h0, dev)
    kw = dict(conv_bias=f32_dev(di.conv_b, dev), Dskip=f32_dev(di.Dskip, dev),
              delta_bias=f32_dev(di.delta_bias, dev), softplus=softplus)
    A, w = f32_dev(di.A, dev), f32_dev(di.conv_w, dev)
    outs, us = [], []
    for t in range(steps):
        u = torch.empty_like(x[t])
        o = ssm.decode_step(x[t], cs, w, dl[t], A, Bm[t], Cm[t], st,
                            z=z[t] if use_z else None, u_out=u, **kw)
        outs.append(host64(o))
        us.append(host64(u))
    torch.cuda.synchronize()
    return np.stack(outs), np.stack(us), host64(cs), host64(st)


def _run_decode_oracle(di, steps, *, use_z=True, softplus=True):
    cs = di.conv_state.f64.copy()
    h = di.h0.astype(np.float64)
    outs, us = [], []
    for t in range(steps):
        o, u, cs, h = oracle.decode_step(di.x.f64[t], cs, di.conv_w, di.conv_b, di.delta.f64[t],
                                         di.Bm.f64[t], di.Cm.f64[t], di.A, h,
                                         z=di.z.f64[t] if use_z else None, Dskip=di.Dskip,
                                         delta_bias=di.delta_bias, softplus=softplus)
        outs.append(o)
        us.append(u)
    return np.stack(outs), np.stack(us), cs, h


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("N,use_z,softplus", [(16, True, True), (5, False, True), (16, True, False)])
def test_decode_steps_parity(dtype, N, use_z, softplus):
    """20 steps from a random conv window and state; B * D = 3 * 40 rows
    leaves a partial CTA."""
    B, D, steps = 3, 40, 20
    di = synth.decode_inputs(B, D, N, steps, dtype, 7300 + N + 2 * int(use_z) + int(softplus))
    if not softplus:  # keep dt positive without the softplus
        di.delta_bias[:] = 0.0
        bits = di.delta.bits if di.delta.bits is not None else None
        v = np.abs(di.delta.f64) * 0.2
        if bits is not None:
            di.delta = synth.Tensor(f64=synth.bf16_bits_to_f32(synth.f32_to_bf16_bits(
                v.astype(np.float32))).astype(np.float64),
                bits=synth.f32_to_bf16_bits(v.astype(np.float32)))
        else:
            di.delta = synth.Tensor(f64=v.astype(np.float32).astype(np.float64),
                                    f32=v.astype(np.float32))
    go, gu, gcs, gh = _run_decode_gpu(di, B, D, N, steps, use_z=use_z, softplus=softplus)
    wo, wu, wcs, wh = _run_decode_oracle(di, steps, use_z=use_z, softplus=softplus)
    fp32 = dtype == "f32"
    tol = TOL_F32 if fp32 else TOL_BF16_OUT
    for t in range(steps):
        w_o = wo[t] if fp32 else oracle.round_bf16(wo[t])
        w_u = wu[t] if fp32 else oracle.round_bf16(wu[t])
        assert rel_l2(go[t], w_o) <= tol, (t, rel_l2(go[t], w_o))
        assert rel_l2(gu[t], w_u) <= tol
    assert rel_l2(gh, wh) <= (TOL_F32 if fp32 else TOL_GRAD)
    np.testing.assert_array_equal(gcs, wcs)  # stored input values: moved, never rounded


def test_decode_continues_gpu_prefill():
    """fp32: conv + scan forward over a prefix on the GPU, then decode steps
    from its final state and last three inputs, against the oracle's
    sequence form over the whole sequence."""
    import torch
    ssm = _ssm()
    B, D, N, L, s = 2, 24, 16, 300, 257
    inp = synth.make_inputs(synth.Shape("prefill", B, D, N, L, "f32"), 7400, conv_bias_scale=0.2,
                            dskip_random=True)
    dev = "cuda"
    x = to_dev(inp.x, dev)
    w, cb = f32_dev(inp.conv_w, dev), f32_dev(inp.conv_b, dev)
    dl, z = to_dev(inp.delta, dev), to_dev(inp.z, dev)
    Bm, Cm = to_dev(inp.Bm, dev), to_dev(inp.Cm, dev)
    A, Dk, db = f32_dev(inp.A, dev), f32_dev(inp.Dskip, dev), f32_dev(inp.delta_bias, dev)
    xp = x[..., :s].contiguous()
    up = ssm.conv1d_fwd(xp, w, cb)
    _, fs, _ = ssm.scan_fwd(up, dl[..., :s].contiguous(), A, Bm[..., :s].contiguous(),
                            Cm[..., :s].contiguous(), z=z[..., :s].contiguous(), Dskip=Dk,
                            delta_bias=db, return_final_state=True)
    cs = x[..., s - 3:s].contiguous()
    outs = []
    for t in range(s, L):
        o = ssm.decode_step(x[..., t].contiguous(), cs, w, dl[..., t].contiguous(), A,
                            Bm[..., t].contiguous(), Cm[..., t].contiguous(), fs, conv_bias=cb,
                            z=z[..., t].contiguous(), Dskip=Dk, delta_bias=db)
        outs.append(host64(o))
    torch.cuda.synchronize()
    _, u = oracle.conv1d_fwd(inp.x.f64, inp.conv_w, inp.conv_b, None)
    full = oracle.scan_fwd(u, inp.delta.f64, inp.A, inp.Bm.f64, inp.Cm.f64, z=inp.z.f64,
                           Dskip=inp.Dskip, delta_bias=inp.delta_bias)
    got = np.stack(outs, axis=-1)
    assert rel_l2(got, full["out"][..., s:]) <= TOL_F32
    # the state was advanced in place through the last token
    assert rel_l2(host64(fs), full["final_state"]) <= TOL_F32


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_decode_many_tiles_parity(dtype):
    """B * D = 130 * 1000 rows: 1016 CTAs of 128 rows (the last one half
    full), several waves on 148 SMs. 3 steps against the oracle."""
    B, D, N, steps = 130, 1000, 16, 3
    di = synth.decode_inputs(B, D, N, steps, dtype, 7350 + int(dtype == "bf16"))
    go, gu, gcs, gh = _run_decode_gpu(di, B, D, N, steps)
    wo, wu, wcs, wh = _run_decode_oracle(di, steps)
    fp32 = dtype == "f32"
    tol = TOL_F32 if fp32 else TOL_BF16_OUT
    for t in range(steps):
        w_o = wo[t] if fp32 else oracle.round_bf16(wo[t])
        w_u = wu[t] if fp32 else oracle.round_bf16(wu[t])
        assert rel_l2(go[t], w_o) <= tol, (t, rel_l2(go[t], w_o))
        assert rel_l2(gu[t], w_u) <= tol
    # every row's state, not only the whole-array norm
    err = np.abs(gh - wh).max(axis=-1) / np.maximum(np.abs(wh).max(axis=-1), 1e-3)
    assert err.max() <= (1e-5 if fp32 else 2e-3), err.max()
    np.testing.assert_array_equal(gcs, wcs)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_decode_vector_equals_scalar_access(dtype):
    """N = 16 with the state 16-byte aligned takes the kernel's 16-byte
    state accesses; the same state one float off that alignment takes its
    scalar accesses. Both do the same operations per row in the same order:
    outputs, conv window and state bitwise equal over 4 steps."""
    import torch
    ssm = _ssm()
    B, D, N, steps = 7, 300, 16, 4
    di = synth.decode_inputs(B, D, N, steps, dtype, 7360 + int(dtype == "bf16"))
    dev = "cuda"
    x, dl, z = to_dev(di.x, dev), to_dev(di.delta, dev), to_dev(di.z, dev)
    Bm, Cm = to_dev(di.Bm, dev), to_dev(di.Cm, dev)
    kw = dict(conv_bias=f32_dev(di.conv_b, dev), Dskip=f32_dev(di.Dskip, dev),
              delta_bias=f32_dev(di.delta_bias, dev))
    A, w = f32_dev(di.A, dev), f32_dev(di.conv_w, dev)
    h0 = f32_dev(di.h0, dev)
    runs = []
    for off in (0, 1):
        buf = torch.zeros(B * D * N + 4, dtype=torch.float32, device=dev)
        st = buf[off:off + B * D * N].view(B, D, N)
        st.copy_(h0)
        assert (st.data_ptr() % 16 == 0) == (off == 0)
        cs = to_dev(di.conv_state, dev).contiguous()
        outs = [ssm.decode_step(x[t], cs, w, dl[t], A, Bm[t], Cm[t], st, z=z[t], **kw).clone()
                for t in range(steps)]
        torch.cuda.synchronize()
        runs.append((torch.stack(outs), cs.clone(), st.clone()))
    for a, b in zip(runs[0], runs[1]):
        assert torch.equal(a, b)
