"""fp64 CPU oracle for the Mamba-1 selective-SSM layer core — TEST INFRASTRUCTURE.

Only `tests/`, `__graft_entry__.smoke()` and the benchmark's CPU-baseline leg
may import this package. The product library never does: it shares no code
with the CUDA path, and nothing here ever consumes a value the CUDA path
produced.

The arithmetic lives in `ssm_oracle.c` (plain C, fp64, one row at a time);
this module only marshals numpy arrays to it. Page references for every step
are in that file's header.
"""
from __future__ import annotations

import ctypes

import numpy as np

from . import build as _build

_lib = None
_dp = ctypes.POINTER(ctypes.c_double)
_ip = ctypes.POINTER(ctypes.c_int32)


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        i, dp, ip, sz = ctypes.c_int, _dp, _ip, ctypes.c_size_t
        L.oracle_round_bf16.argtypes = [dp, dp, sz]
        L.oracle_conv1d_fwd.argtypes = [dp, dp, dp, ip, dp, dp, i, i, i, i, i]
        L.oracle_conv1d_bwd.argtypes = [dp, dp, dp, ip, dp, dp, dp, dp, i, i, i, i, i]
        L.oracle_scan_fwd.argtypes = [dp] * 8 + [i, i, ip, dp, dp, dp, dp, i, i, i, i]
        L.oracle_scan_bwd.argtypes = [dp] * 8 + [i, i, ip] + [dp] * 12 + [i, i, i, i]
        L.oracle_scan_fwd_mt.argtypes = [dp] * 8 + [i, i, ip, dp, dp, dp, dp, i, i, i, i, i]
        L.oracle_scan_bwd_mt.argtypes = [dp] * 8 + [i, i, ip] + [dp] * 12 + [i, i, i, i, i]
        L.oracle_decode_step.argtypes = [dp] * 11 + [i] + [dp] * 3 + [i, i, i, i]
        L.oracle_cscan_fwd.argtypes = [dp] * 8 + [i, ip, dp, dp, dp, dp, i, i, i, i]
        L.oracle_cscan_bwd.argtypes = [dp] * 8 + [i, ip] + [dp] * 12 + [i, i, i, i]
        L.oracle_ssd_fwd.argtypes = [dp] * 7 + [i, ip, dp, dp] + [i] * 6
        L.oracle_ssd_bwd.argtypes = [dp] * 7 + [i, ip] + [dp] * 8 + [i] * 6
        for f in ("oracle_round_bf16", "oracle_conv1d_fwd", "oracle_conv1d_bwd",
                  "oracle_scan_fwd", "oracle_scan_bwd", "oracle_scan_fwd_mt",
                  "oracle_scan_bwd_mt", "oracle_decode_step", "oracle_cscan_fwd",
                  "oracle_cscan_bwd", "oracle_ssd_fwd", "oracle_ssd_bwd"):
            getattr(L, f).restype = None
        _lib = L
    return _lib


def _d(a):
    """Pointer to a C-contiguous float64 array (or NULL for None)."""
    if a is None:
        return None
    assert a.dtype == np.float64 and a.flags.c_contiguous, (a.dtype, a.flags)
    return a.ctypes.data_as(_dp)


def _i(a):
    if a is None:
        return None
    assert a.dtype == np.int32 and a.flags.c_contiguous
    return a.ctypes.data_as(_ip)


def _f64(a):
    return None if a is None else np.ascontiguousarray(a, dtype=np.float64)


def _i32(a):
    return None if a is None else np.ascontiguousarray(a, dtype=np.int32)


def round_bf16(x: np.ndarray) -> np.ndarray:
    """Round float64 values to the nearest bfloat16 value (ties to even)."""
    x = _f64(x)
    out = np.empty_like(x)
    lib().oracle_round_bf16(_d(x), _d(out), x.size)
    return out


def conv1d_fwd(x, w, bias, seq_idx, silu=True):
    """Depthwise causal conv (cross-correlation, left pad W-1) + optional SiLU.

    x [B, D, L], w [D, W], bias [D] or None, seq_idx [B, L] or None.
    Returns (c, u): pre-activation and output, both [B, D, L] float64.
    """
    x, w, bias, seq = _f64(x), _f64(w), _f64(bias), _i32(seq_idx)
    B, D, L = x.shape
    W = w.shape[1]
    c = np.empty_like(x)
    u = np.empty_like(x)
    lib().oracle_conv1d_fwd(_d(x), _d(w), _d(bias), _i(seq), _d(c), _d(u),
                            B, D, L, W, int(silu))
    return c, u


def conv1d_bwd(x, w, bias, seq_idx, du, silu=True):
    """Gradients of conv1d_fwd's u: returns (dx [B,D,L], dw [D,W], dbias [D])."""
    x, w, bias, seq, du = _f64(x), _f64(w), _f64(bias), _i32(seq_idx), _f64(du)
    B, D, L = x.shape
    W = w.shape[1]
    dx = np.empty_like(x)
    dw = np.empty((D, W))
    db = np.empty(D)
    lib().oracle_conv1d_bwd(_d(x), _d(w), _d(bias), _i(seq), _d(du), _d(dx),
                            _d(dw), _d(db), B, D, L, W, int(silu))
    return dx, dw, db


def scan_fwd(u, delta, A, Bm, Cm, *, z=None, Dskip=None, delta_bias=None,
             softplus=True, seq_idx=None, h0=None, zoh=False, nthreads=1):
    """Selective scan forward. Returns dict(out, y, final_state).

    u, delta, z: [B, D, L]; A: [D, N]; Bm, Cm: [B, N, L]; Dskip,
    delta_bias: [D] or None; seq_idx: [B, L] or None; h0: [B, D, N] state
    before token 0, or None for zero. zoh: zero-order-hold B_bar
    ((exp(dt A) - 1) / A B) instead of dt B.
    """
    u, delta, z, A = _f64(u), _f64(delta), _f64(z), _f64(A)
    Dskip, delta_bias, Bm, Cm = _f64(Dskip), _f64(delta_bias), _f64(Bm), _f64(Cm)
    seq, h0 = _i32(seq_idx), _f64(h0)
    B, D, L = u.shape
    N = A.shape[1]
    out = np.empty_like(u)
    y = np.empty_like(u)
    fs = np.empty((B, D, N))
    args = [_d(u), _d(delta), _d(z), _d(A), _d(Dskip), _d(delta_bias), _d(Bm),
            _d(Cm), int(softplus), int(zoh), _i(seq), _d(h0), _d(out), _d(y), _d(fs), B, D, L, N]
    if nthreads > 1:
        lib().oracle_scan_fwd_mt(*args, int(nthreads))
    else:
        lib().oracle_scan_fwd(*args)
    return {"out": out, "y": y, "final_state": fs}


def scan_bwd(u, delta, A, Bm, Cm, dout, *, z=None, Dskip=None, delta_bias=None,
             softplus=True, seq_idx=None, h0=None, zoh=False, dhL=None, nthreads=1):
    """Selective scan backward. Returns dict of gradients (fp64):
    du, ddelta (w.r.t. the raw delta), dz, dA, dB, dC, dD, ddelta_bias and
    dh0 (w.r.t. the state before token 0). dhL [B, D, N]: a gradient reaching
    the final state from outside (None: 0)."""
    u, delta, z, A = _f64(u), _f64(delta), _f64(z), _f64(A)
    Dskip, delta_bias, Bm, Cm = _f64(Dskip), _f64(delta_bias), _f64(Bm), _f64(Cm)
    seq, dout, h0, dhL = _i32(seq_idx), _f64(dout), _f64(h0), _f64(dhL)
    B, D, L = u.shape
    N = A.shape[1]
    du = np.empty_like(u)
    ddelta = np.empty_like(u)
    dz = np.zeros_like(u)
    dA = np.empty((D, N))
    dB = np.empty((B, N, L))
    dC = np.empty((B, N, L))
    dD = np.empty(D)
    ddb = np.empty(D)
    dh0 = np.empty((B, D, N))
    args = [_d(u), _d(delta), _d(z), _d(A), _d(Dskip), _d(delta_bias), _d(Bm),
            _d(Cm), int(softplus), int(zoh), _i(seq), _d(h0), _d(dout), _d(du), _d(ddelta), _d(dz),
            _d(dA), _d(dB), _d(dC), _d(dD), _d(ddb), _d(dh0), _d(dhL), B, D, L, N]
    if nthreads > 1:
        lib().oracle_scan_bwd_mt(*args, int(nthreads))
    else:
        lib().oracle_scan_bwd(*args)
    return {"du": du, "ddelta": ddelta, "dz": dz, "dA": dA, "dB": dB, "dC": dC,
            "dD": dD, "ddelta_bias": ddb, "dh0": dh0}


def decode_step(x, conv_state, w, conv_bias, delta, Bt, Ct, A, h, *, z=None,
                Dskip=None, delta_bias=None, softplus=True):
    """One token of the recurrent form for every (b, d).

    x, delta, z: [B, D]; conv_state: [B, D, W-1] (previous inputs, oldest
    first); w: [D, W]; conv_bias, Dskip, delta_bias: [D] or None; Bt, Ct:
    [B, N]; A: [D, N]; h: [B, D, N] state after the previous token.
    Returns (out [B, D], u [B, D], new conv_state, new h); inputs unchanged.
    """
    x, w, cb, delta, z = _f64(x), _f64(w), _f64(conv_bias), _f64(delta), _f64(z)
    Bt, Ct, A, Dskip, delta_bias = _f64(Bt), _f64(Ct), _f64(A), _f64(Dskip), _f64(delta_bias)
    cs = np.array(conv_state, dtype=np.float64, order="C", copy=True)
    hh = np.array(h, dtype=np.float64, order="C", copy=True)
    B, D = x.shape
    N, W = A.shape[1], w.shape[1]
    out = np.empty((B, D))
    u = np.empty((B, D))
    lib().oracle_decode_step(_d(x), _d(cs), _d(w), _d(cb), _d(delta), _d(z), _d(Bt),
                             _d(Ct), _d(A), _d(Dskip), _d(delta_bias), int(softplus),
                             _d(hh), _d(out), _d(u), B, D, N, W)
    return out, u, cs, hh


def cscan_fwd(u, delta, A, Bm, Cm, *, z=None, Dskip=None, delta_bias=None,
              softplus=True, seq_idx=None, h0=None):
    """Selective scan with complex diagonal A. Returns dict(out, y, final_state).

    u, delta, z: [B, D, L]; A: [D, N] complex; Bm, Cm: [B, N, L] complex;
    h0: [B, D, N] complex or None. y = 2 Re(sum_n C h) + D u; final_state is
    complex [B, D, N].
    """
    u, delta, z = _f64(u), _f64(delta), _f64(z)
    Dskip, delta_bias, seq = _f64(Dskip), _f64(delta_bias), _i32(seq_idx)
    B, D, L = u.shape
    N = A.shape[1]
    Ar = _cplx_pairs(A)
    Bp, Cp = _cplx_planes(Bm), _cplx_planes(Cm)
    h0p = None if h0 is None else _cplx_pairs(h0)
    out = np.empty_like(u)
    y = np.empty_like(u)
    fs = np.empty((B, D, N, 2))
    lib().oracle_cscan_fwd(_d(u), _d(delta), _d(z), _d(Ar), _d(Dskip), _d(delta_bias), _d(Bp),
                           _d(Cp), int(softplus), _i(seq), _d(h0p), _d(out), _d(y), _d(fs),
                           B, D, L, N)
    return {"out": out, "y": y, "final_state": fs[..., 0] + 1j * fs[..., 1]}


def cscan_bwd(u, delta, A, Bm, Cm, dout, *, z=None, Dskip=None, delta_bias=None,
              softplus=True, seq_idx=None, h0=None, dhL=None):
    """Backward of cscan_fwd. Real inputs get real gradients; for a complex
    input w the gradient is returned as dL/dRe(w) + i dL/dIm(w) (dA, dB, dC,
    dh0). dhL [B, D, N] complex: dL/dRe h_{L-1} + i dL/dIm h_{L-1} from
    outside (None: 0)."""
    u, delta, z, dout = _f64(u), _f64(delta), _f64(z), _f64(dout)
    Dskip, delta_bias, seq = _f64(Dskip), _f64(delta_bias), _i32(seq_idx)
    B, D, L = u.shape
    N = A.shape[1]
    Ar = _cplx_pairs(A)
    Bp, Cp = _cplx_planes(Bm), _cplx_planes(Cm)
    h0p = None if h0 is None else _cplx_pairs(h0)
    dhLp = None if dhL is None else _cplx_pairs(dhL)
    du = np.empty_like(u)
    ddelta = np.empty_like(u)
    dz = np.zeros_like(u)
    dA = np.empty((D, N, 2))
    dB = np.empty((B, N, 2, L))
    dC = np.empty((B, N, 2, L))
    dD = np.empty(D)
    ddb = np.empty(D)
    dh0 = np.empty((B, D, N, 2))
    lib().oracle_cscan_bwd(_d(u), _d(delta), _d(z), _d(Ar), _d(Dskip), _d(delta_bias), _d(Bp),
                           _d(Cp), int(softplus), _i(seq), _d(h0p), _d(dout), _d(du),
                           _d(ddelta), _d(dz), _d(dA), _d(dB), _d(dC), _d(dD), _d(ddb), _d(dh0),
                           _d(dhLp), B, D, L, N)
    return {"du": du, "ddelta": ddelta, "dz": dz, "dA": dA[..., 0] + 1j * dA[..., 1],
            "dB": dB[:, :, 0] + 1j * dB[:, :, 1], "dC": dC[:, :, 0] + 1j * dC[:, :, 1],
            "dD": dD, "ddelta_bias": ddb, "dh0": dh0[..., 0] + 1j * dh0[..., 1]}


def ssd_fwd(x, dt_raw, A, Bm, Cm, *, D=None, dt_bias=None, softplus=True, seq_idx=None):
    """Mamba-2 SSD forward. x [B, L, H, P]; dt_raw [B, L, H]; A, D, dt_bias
    [H]; Bm, Cm [B, L, G, N] (head h uses group h // (H // G)); seq_idx
    [B, L]. Returns dict(y [B, L, H, P], final_state [B, H, P, N])."""
    x, dt_raw, A, Bm, Cm = _f64(x), _f64(dt_raw), _f64(A), _f64(Bm), _f64(Cm)
    D, dt_bias, seq = _f64(D), _f64(dt_bias), _i32(seq_idx)
    B, L, H, P = x.shape
    G, N = Bm.shape[2], Bm.shape[3]
    assert H % G == 0
    y = np.empty_like(x)
    fs = np.empty((B, H, P, N))
    lib().oracle_ssd_fwd(_d(x), _d(dt_raw), _d(A), _d(Bm), _d(Cm), _d(D), _d(dt_bias),
                         int(softplus), _i(seq), _d(y), _d(fs), B, L, H, P, G, N)
    return {"y": y, "final_state": fs}


def ssd_bwd(x, dt_raw, A, Bm, Cm, dy, *, D=None, dt_bias=None, softplus=True, seq_idx=None):
    """Backward of ssd_fwd: dict(dx, ddt_raw, dA, dB, dC, dD, ddt_bias)."""
    x, dt_raw, A, Bm, Cm, dy = _f64(x), _f64(dt_raw), _f64(A), _f64(Bm), _f64(Cm), _f64(dy)
    D, dt_bias, seq = _f64(D), _f64(dt_bias), _i32(seq_idx)
    B, L, H, P = x.shape
    G, N = Bm.shape[2], Bm.shape[3]
    assert H % G == 0
    dx = np.empty_like(x)
    ddt = np.empty_like(dt_raw)
    dA = np.empty(H)
    dB = np.empty_like(Bm)
    dC = np.empty_like(Cm)
    dD = np.empty(H)
    ddb = np.empty(H)
    lib().oracle_ssd_bwd(_d(x), _d(dt_raw), _d(A), _d(Bm), _d(Cm), _d(D), _d(dt_bias),
                         int(softplus), _i(seq), _d(dy), _d(dx), _d(ddt), _d(dA), _d(dB), _d(dC),
                         _d(dD), _d(ddb), B, L, H, P, G, N)
    return {"dx": dx, "ddt_raw": ddt, "dA": dA, "dB": dB, "dC": dC, "dD": dD, "ddt_bias": ddb}


def _cplx_pairs(a):
    """Complex array [..] -> float64 [.., 2] (re, im interleaved)."""
    a = np.asarray(a, dtype=np.complex128)
    return np.ascontiguousarray(np.stack([a.real, a.imag], axis=-1))


def _cplx_planes(a):
    """Complex [B, N, L] -> float64 [B, N, 2, L] (real plane, imaginary plane)."""
    a = np.asarray(a, dtype=np.complex128)
    return np.ascontiguousarray(np.stack([a.real, a.imag], axis=2))


def layer_fwd_bwd(inp, *, bf16_points: bool, softplus=True, nthreads=1):
    """The whole core on one layer's inputs (a `synth.LayerInputs`).

    conv -> SiLU -> scan (softplus delta, D skip, SiLU(z) gate), then the
    backward from `dout`. With `bf16_points` the oracle rounds the two values
    that the layer stores between its stages in bf16 (u after the conv and
    du after the scan backward) exactly where bf16 storage rounds them.
    Returns a dict with every intermediate and gradient.
    """
    seq = inp.seq_idx
    c, u = conv1d_fwd(inp.x.f64, inp.conv_w, inp.conv_b, seq, silu=True)
    u_s = round_bf16(u) if bf16_points else u
    f = scan_fwd(u_s, inp.delta.f64, inp.A, inp.Bm.f64, inp.Cm.f64, z=inp.z.f64,
                 Dskip=inp.Dskip, delta_bias=inp.delta_bias, softplus=softplus,
                 seq_idx=seq, nthreads=nthreads)
    g = scan_bwd(u_s, inp.delta.f64, inp.A, inp.Bm.f64, inp.Cm.f64, inp.dout.f64,
                 z=inp.z.f64, Dskip=inp.Dskip, delta_bias=inp.delta_bias,
                 softplus=softplus, seq_idx=seq, nthreads=nthreads)
    du_s = round_bf16(g["du"]) if bf16_points else g["du"]
    dx, dw, dcb = conv1d_bwd(inp.x.f64, inp.conv_w, inp.conv_b, seq, du_s, silu=True)
    res = {"c": c, "u": u, "u_stored": u_s, "du_stored": du_s, "dx": dx,
           "dconv_w": dw, "dconv_b": dcb}
    res.update(f)
    res.update(g)
    return res


__all__ = ["round_bf16", "conv1d_fwd", "conv1d_bwd", "scan_fwd", "scan_bwd",
           "decode_step", "layer_fwd_bwd", "lib"]
