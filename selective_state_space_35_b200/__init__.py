"""B200 (sm_100a) Mamba-1 selective-SSM layer core: torch-facing binding.

Each function marshals torch CUDA tensors to the C ABI of libssmscan
(include/ssmscan.h) and returns torch tensors; every step of the layer core
runs in the library's kernels. Tensors must be CUDA and C-contiguous; layouts
are activations [B, D, L], B/C [B, N, L], A [D, N], per-channel vectors [D],
conv weight [D, 4], seq_idx int32 [B, L]. Activations are bf16 or fp32;
parameters and the gradients of parameters, B and C are fp32. A complex
diagonal A is passed as [D, N, 2] (B/C [B, N, 2, L], states [B, D, N, 2]).
Pieces of a longer sequence (summaries, carries, conv halos) serve the
context-parallel driver in `cp.py`.
"""
from __future__ import annotations

import ctypes

from . import _lib
from ._lib import (SsmError, ssm_abi_version, ssm_conv1d_bwd, ssm_conv1d_bwd_noalloc,
                   ssm_conv1d_bwd_workspace_size,
                   ssm_conv1d_fwd, ssm_conv1d_scan_fwd, ssm_decode_params, ssm_decode_step,
                   ssm_last_error,
                   ssm_probe_ex2_rate, ssm_scan_bwd, ssm_scan_status,
                   ssm_scan_fwd, ssm_scan_grads, ssm_scan_params, ssm_scan_workspace_size,
                   ssm_scan_bwd_workspace_size, ssm_ssd_params, ssm_ssd_fwd,
                   ssm_ssd_grads, ssm_ssd_bwd, ssm_scan_fwd_summary, ssm_scan_bwd_summary, ssm_state_carry,
                   ssm_conv1d_fwd_ctx, ssm_conv1d_bwd_ctx, ssm_debug_info, ssm_debug_report,
                   ssm_debug_selftest)

__all__ = [
    "SsmError", "ssm_abi_version", "ssm_last_error", "ssm_conv1d_fwd", "ssm_conv1d_bwd",
    "ssm_conv1d_bwd_workspace_size", "ssm_conv1d_bwd_noalloc", "ssm_scan_workspace_size", "ssm_scan_fwd", "ssm_scan_bwd",
    "ssm_scan_params", "ssm_scan_grads", "ssm_scan_bwd_workspace_size", "ssm_ssd_params",
    "ssm_ssd_fwd", "ssd_fwd", "ssm_ssd_grads", "ssm_ssd_bwd", "ssd_bwd", "ssd_chunk_states_shape",
    "ssm_probe_ex2_rate", "probe_ex2_rate", "ssm_scan_status",
    "scan_status", "conv1d_fwd", "conv1d_bwd", "scan_params",
    "scan_workspace_size", "scan_fwd", "scan_bwd", "load",
    "ssm_decode_params", "ssm_decode_step", "decode_step", "ssm_conv1d_scan_fwd",
    "conv1d_scan_fwd", "ssm_scan_fwd_summary", "ssm_scan_bwd_summary", "ssm_state_carry",
    "ssm_conv1d_fwd_ctx", "ssm_conv1d_bwd_ctx", "scan_fwd_summary", "scan_bwd_summary",
    "state_carry", "ssm_debug_info", "ssm_debug_report", "ssm_debug_selftest", "debug_report",
    "debug_selftest",
]

load = _lib.load


def _torch():
    import torch
    return torch


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _dtype_code(t):
    torch = _torch()
    if t.dtype == torch.bfloat16:
        return _lib.SSM_DTYPE_BF16
    if t.dtype == torch.float32:
        return _lib.SSM_DTYPE_F32
    raise TypeError(f"activations must be bf16 or fp32, got {t.dtype}")


def _need(t, name, dtype=None, shape=None):
    torch = _torch()
    if t is None:
        return
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (no CPU path)")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")


def _stream(stream, device):
    torch = _torch()
    s = stream if stream is not None else torch.cuda.current_stream(device)
    return ctypes.c_void_p(s.cuda_stream)


def probe_ex2_rate(device=None) -> float:
    """Measured ex2.approx.f32 results per second of the current device."""
    torch = _torch()
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else device
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    sink = torch.empty(sms * 2048, dtype=torch.float32, device=dev)
    return ssm_probe_ex2_rate(_ptr(sink), sink.numel(), _stream(None, dev))


def conv1d_fwd(x, w, bias=None, seq_idx=None, *, silu=True, out=None, x_prev=None,
               seq_prev=None, stream=None):
    """u = silu(causal depthwise conv1d(x)) (width 4, segment-masked taps).

    For a piece of a longer sequence, x_prev [B, D, 3] (x dtype) holds the 3
    inputs before token 0 and seq_prev [B, 3] their document ids."""
    torch = _torch()
    B, D, L = x.shape
    _need(x, "x", shape=(B, D, L))
    _need(w, "w", torch.float32, (D, 4))
    _need(bias, "bias", torch.float32, (D,))
    _need(seq_idx, "seq_idx", torch.int32, (B, L))
    _need(x_prev, "x_prev", x.dtype, (B, D, 3))
    _need(seq_prev, "seq_prev", torch.int32, (B, 3))
    if out is None:
        out = torch.empty_like(x)
    _need(out, "out", x.dtype, (B, D, L))
    if x_prev is None and seq_prev is None:
        _lib.check(ssm_conv1d_fwd(_ptr(x), _ptr(w), _ptr(bias), _ptr(seq_idx), _ptr(out), B, D, L,
                                  4, _dtype_code(x), int(silu), _stream(stream, x.device)))
    else:
        _lib.check(ssm_conv1d_fwd_ctx(_ptr(x), _ptr(w), _ptr(bias), _ptr(seq_idx), _ptr(x_prev),
                                      _ptr(seq_prev), _ptr(out), B, D, L, 4, _dtype_code(x),
                                      int(silu), _stream(stream, x.device)))
    return out


def conv1d_bwd(x, w, bias, seq_idx, du, *, silu=True, dx=None, dw=None, dbias=None,
               workspace=None, x_prev=None, seq_prev=None, x_next=None, du_next=None,
               seq_next=None, stream=None):
    """Gradients of conv1d_fwd: returns (dx, dw, dbias).

    For a piece of a longer sequence: x_prev / seq_prev as in conv1d_fwd, and
    x_next, du_next [B, D, 3], seq_next [B, 3] the next piece's first inputs,
    upstream gradients and ids (they reach this piece's last 3 dx); dw and
    dbias then cover this piece's own tokens."""
    torch = _torch()
    B, D, L = x.shape
    _need(x, "x", shape=(B, D, L))
    _need(du, "du", x.dtype, (B, D, L))
    _need(w, "w", torch.float32, (D, 4))
    _need(bias, "bias", torch.float32, (D,))
    _need(seq_idx, "seq_idx", torch.int32, (B, L))
    for t, nm in ((x_prev, "x_prev"), (x_next, "x_next"), (du_next, "du_next")):
        _need(t, nm, x.dtype, (B, D, 3))
    for t, nm in ((seq_prev, "seq_prev"), (seq_next, "seq_next")):
        _need(t, nm, torch.int32, (B, 3))
    dx = torch.empty_like(x) if dx is None else dx
    dw = torch.empty((D, 4), dtype=torch.float32, device=x.device) if dw is None else dw
    if dbias is None:
        dbias = torch.empty((D,), dtype=torch.float32, device=x.device)
    ws_bytes = ssm_conv1d_bwd_workspace_size(B, D, L, 4)
    if workspace is None:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=x.device)
    if all(t is None for t in (x_prev, seq_prev, x_next, du_next, seq_next)):
        _lib.check(ssm_conv1d_bwd(_ptr(x), _ptr(w), _ptr(bias), _ptr(seq_idx), _ptr(du), _ptr(dx),
                                  _ptr(dw), _ptr(dbias), B, D, L, 4, _dtype_code(x), int(silu),
                                  _ptr(workspace), workspace.numel(), _stream(stream, x.device)))
    else:
        _lib.check(ssm_conv1d_bwd_ctx(_ptr(x), _ptr(w), _ptr(bias), _ptr(seq_idx), _ptr(x_prev),
                                      _ptr(seq_prev), _ptr(x_next), _ptr(du_next), _ptr(seq_next),
                                      _ptr(du), _ptr(dx), _ptr(dw), _ptr(dbias), B, D, L, 4,
                                      _dtype_code(x), int(silu), _ptr(workspace),
                                      workspace.numel(), _stream(stream, x.device)))
    return dx, dw, dbias


def scan_params(u, delta, A, Bm, Cm, *, z=None, Dskip=None, delta_bias=None, softplus=True,
                seq_idx=None, cu_seqlens=None, n_splits=0, out=None, final_state=None,
                workspace=None, initial_state=None, zoh=False) -> ssm_scan_params:
    """Fill an ssm_scan_params from tensors (validating shapes and dtypes).

    A of shape [D, N, 2] selects the complex diagonal A ((re, im) pairs); Bm
    and Cm are then [B, N, 2, L] and the states [B, D, N, 2].
    """
    torch = _torch()
    B, D, L = u.shape
    N = A.shape[1]
    cplx = A.dim() == 3
    c2 = (2,) if cplx else ()
    _need(u, "u", shape=(B, D, L))
    _need(delta, "delta", u.dtype, (B, D, L))
    _need(z, "z", u.dtype, (B, D, L))
    _need(A, "A", torch.float32, (D, N) + c2)
    _need(Dskip, "Dskip", torch.float32, (D,))
    _need(delta_bias, "delta_bias", torch.float32, (D,))
    _need(Bm, "Bm", u.dtype, (B, N) + c2 + (L,))
    _need(Cm, "Cm", u.dtype, (B, N) + c2 + (L,))
    _need(seq_idx, "seq_idx", torch.int32, (B, L))
    _need(cu_seqlens, "cu_seqlens", torch.int32)
    _need(out, "out", u.dtype, (B, D, L))
    _need(final_state, "final_state", torch.float32, (B, D, N) + c2)
    _need(initial_state, "initial_state", torch.float32, (B, D, N) + c2)
    p = ssm_scan_params()
    p.struct_size = ctypes.sizeof(ssm_scan_params)
    p.B, p.D, p.L, p.N = B, D, L, N
    p.dtype = _dtype_code(u)
    p.u, p.delta, p.z = u.data_ptr(), delta.data_ptr(), (z.data_ptr() if z is not None else None)
    p.A = A.data_ptr()
    p.Dskip = Dskip.data_ptr() if Dskip is not None else None
    p.delta_bias = delta_bias.data_ptr() if delta_bias is not None else None
    p.Bm, p.Cm = Bm.data_ptr(), Cm.data_ptr()
    p.delta_softplus = int(softplus)
    p.seq_idx = seq_idx.data_ptr() if seq_idx is not None else None
    p.cu_seqlens = cu_seqlens.data_ptr() if cu_seqlens is not None else None
    p.n_docs = (cu_seqlens.numel() - 1) if cu_seqlens is not None else 0
    p.n_splits = int(n_splits)
    p.out = out.data_ptr() if out is not None else None
    p.final_state = final_state.data_ptr() if final_state is not None else None
    p.workspace = workspace.data_ptr() if workspace is not None else None
    p.workspace_bytes = workspace.numel() if workspace is not None else 0
    p.initial_state = initial_state.data_ptr() if initial_state is not None else None
    p.discretization = 1 if zoh else 0
    p.state_complex = int(cplx)
    return p


def scan_workspace_size(p: ssm_scan_params) -> int:
    return ssm_scan_workspace_size(p)


def scan_status(u, A, workspace, stream=None) -> int:
    """Device status word of `workspace` (0 = ok, 4 = a bounded wait timed out);
    synchronises the stream."""
    B, D, L = u.shape
    p = ssm_scan_params()
    p.struct_size = ctypes.sizeof(ssm_scan_params)
    p.B, p.D, p.L, p.N = B, D, L, A.shape[1]
    p.dtype = _dtype_code(u)
    p.workspace, p.workspace_bytes = workspace.data_ptr(), workspace.numel()
    return ssm_scan_status(p, _stream(stream, u.device))


def scan_fwd(u, delta, A, Bm, Cm, *, z=None, Dskip=None, delta_bias=None, softplus=True,
             seq_idx=None, cu_seqlens=None, n_splits=0, return_final_state=False, out=None,
             workspace=None, initial_state=None, zoh=False, final_state=None, stream=None):
    """Selective scan forward.

    Returns (out, final_state or None, workspace). Keep `workspace` (it holds
    the state checkpoints and the pre-gate output) and pass it to scan_bwd
    unchanged. `final_state` is a preallocated output for the final state
    (implies return_final_state). `initial_state` [B, D, N] fp32 is the state before token 0;
    `zoh` selects the zero-order-hold B_bar = (exp(dt A) - 1) / A B. A of
    shape [D, N, 2] selects the complex diagonal A (see scan_params).
    """
    torch = _torch()
    B, D, L = u.shape
    N = A.shape[1]
    c2 = (2,) if A.dim() == 3 else ()
    out = torch.empty_like(u) if out is None else out
    if final_state is not None:
        _need(final_state, "final_state", torch.float32, (B, D, N) + c2)
        fs = final_state
    else:
        fs = (torch.empty((B, D, N) + c2, dtype=torch.float32, device=u.device)
              if return_final_state else None)
    p = scan_params(u, delta, A, Bm, Cm, z=z, Dskip=Dskip, delta_bias=delta_bias, softplus=softplus,
                    seq_idx=seq_idx, cu_seqlens=cu_seqlens, n_splits=n_splits, out=out,
                    final_state=fs, initial_state=initial_state, zoh=zoh)
    need = ssm_scan_workspace_size(p)
    if workspace is None or workspace.numel() < need:
        workspace = torch.empty(need, dtype=torch.uint8, device=u.device)
    p.workspace, p.workspace_bytes = workspace.data_ptr(), workspace.numel()
    _lib.check(ssm_scan_fwd(p, _stream(stream, u.device)))
    return out, fs, workspace


def conv1d_scan_fwd(x, conv_w, conv_bias, delta, A, Bm, Cm, *, z=None, Dskip=None,
                    delta_bias=None, softplus=True, seq_idx=None, cu_seqlens=None, n_splits=0,
                    return_final_state=False, u=None, out=None, workspace=None,
                    initial_state=None, zoh=False, stream=None):
    """Fused depthwise conv (W = 4) + SiLU + selective scan forward.

    x [B, D, L] is the conv input; conv_w [D, 4], conv_bias [D] or None.
    Returns (out, u, final_state or None, workspace): u = silu(conv(x)) is
    written by the kernel (pass it, with `workspace`, to scan_bwd; it is the
    conv output for conv1d_bwd). Bitwise equal to conv1d_fwd + scan_fwd.
    """
    torch = _torch()
    B, D, L = x.shape
    N = A.shape[1]
    _need(x, "x", shape=(B, D, L))
    _need(conv_w, "conv_w", torch.float32, (D, 4))
    _need(conv_bias, "conv_bias", torch.float32, (D,))
    u = torch.empty_like(x) if u is None else u
    _need(u, "u", x.dtype, (B, D, L))
    out = torch.empty_like(x) if out is None else out
    fs = torch.empty((B, D, N), dtype=torch.float32, device=x.device) if return_final_state else None
    p = scan_params(u, delta, A, Bm, Cm, z=z, Dskip=Dskip, delta_bias=delta_bias, softplus=softplus,
                    seq_idx=seq_idx, cu_seqlens=cu_seqlens, n_splits=n_splits, out=out,
                    final_state=fs, initial_state=initial_state, zoh=zoh)
    need = ssm_scan_workspace_size(p)
    if workspace is None or workspace.numel() < need:
        workspace = torch.empty(need, dtype=torch.uint8, device=x.device)
    p.workspace, p.workspace_bytes = workspace.data_ptr(), workspace.numel()
    _lib.check(ssm_conv1d_scan_fwd(p, x.data_ptr(), conv_w.data_ptr(),
                                   conv_bias.data_ptr() if conv_bias is not None else None,
                                   _stream(stream, x.device)))
    return out, u, fs, workspace


def scan_bwd(u, delta, A, Bm, Cm, dout, workspace, *, z=None, Dskip=None, delta_bias=None,
             softplus=True, seq_idx=None, cu_seqlens=None, n_splits=0, grads=None,
             initial_state=None, dfinal_state=None, zoh=False, deterministic=False,
             bwd_workspace=None, stream=None):
    """Selective scan backward; `workspace` must come from the matching scan_fwd
    (called with the same `initial_state`).

    deterministic=True sums dB / dC over channel groups in a fixed order
    (bitwise reproducible) through a scratch buffer of
    ssm_scan_bwd_workspace_size bytes: `bwd_workspace` (uint8 on the device)
    or one allocated here.

    Returns a dict: du, ddelta (w.r.t. the raw delta), dz (or None), dA, dB,
    dC, dD, ddelta_bias, dinitial_state (w.r.t. the state before token 0).
    `dfinal_state` (shaped like the final state) is a gradient reaching the
    final state from outside. Preallocated outputs may be passed in `grads`.
    """
    torch = _torch()
    B, D, L = u.shape
    N = A.shape[1]
    c2 = (2,) if A.dim() == 3 else ()
    _need(dout, "dout", u.dtype, (B, D, L))
    g = dict(grads or {})
    dev = u.device
    g.setdefault("du", torch.empty_like(u))
    g.setdefault("ddelta", torch.empty_like(u))
    g.setdefault("dz", torch.empty_like(u) if z is not None else None)
    g.setdefault("dA", torch.empty((D, N) + c2, dtype=torch.float32, device=dev))
    g.setdefault("dB", torch.empty((B, N) + c2 + (L,), dtype=torch.float32, device=dev))
    g.setdefault("dC", torch.empty((B, N) + c2 + (L,), dtype=torch.float32, device=dev))
    g.setdefault("dD", torch.empty((D,), dtype=torch.float32, device=dev))
    g.setdefault("ddelta_bias", torch.empty((D,), dtype=torch.float32, device=dev))
    g.setdefault("dinitial_state", torch.empty((B, D, N) + c2, dtype=torch.float32, device=dev))
    p = scan_params(u, delta, A, Bm, Cm, z=z, Dskip=Dskip, delta_bias=delta_bias, softplus=softplus,
                    seq_idx=seq_idx, cu_seqlens=cu_seqlens, n_splits=n_splits, out=None,
                    workspace=workspace, initial_state=initial_state, zoh=zoh)
    p.out = dout.data_ptr()  # not written by the backward; any valid activation pointer
    gr = ssm_scan_grads()
    gr.struct_size = ctypes.sizeof(ssm_scan_grads)
    gr.dout = dout.data_ptr()
    gr.du, gr.ddelta = g["du"].data_ptr(), g["ddelta"].data_ptr()
    gr.dz = g["dz"].data_ptr() if g["dz"] is not None else None
    gr.dA, gr.dB, gr.dC = g["dA"].data_ptr(), g["dB"].data_ptr(), g["dC"].data_ptr()
    gr.dD = g["dD"].data_ptr() if g["dD"] is not None else None
    gr.ddelta_bias = g["ddelta_bias"].data_ptr() if g["ddelta_bias"] is not None else None
    gr.dinitial_state = (g["dinitial_state"].data_ptr() if g["dinitial_state"] is not None
                         else None)
    _need(dfinal_state, "dfinal_state", torch.float32, (B, D, N) + c2)
    gr.dfinal_state = dfinal_state.data_ptr() if dfinal_state is not None else None
    gr.deterministic = 1 if deterministic else 0
    need = ssm_scan_bwd_workspace_size(p, gr)
    if need:
        if bwd_workspace is None:
            bwd_workspace = torch.empty(need, dtype=torch.uint8, device=dev)
        gr.workspace, gr.workspace_bytes = bwd_workspace.data_ptr(), bwd_workspace.numel()
    _lib.check(ssm_scan_bwd(p, gr, _stream(stream, u.device)))
    return g


def decode_step(x, conv_state, conv_w, delta, A, Bm, Cm, state, *, conv_bias=None, z=None,
                Dskip=None, delta_bias=None, softplus=True, out=None, u_out=None, stream=None):
    """One token of the recurrent form for every (b, d).

    x, delta, z: [B, D] activations; conv_state: [B, D, 3] activation dtype,
    the previous three conv inputs (updated in place); conv_w [D, 4],
    conv_bias [D]; Bm, Cm: [B, N]; A: [D, N]; state: [B, D, N] fp32 (updated
    in place). Returns out [B, D] (and writes u_out [B, D] if given).
    """
    torch = _torch()
    B, D = x.shape
    N = A.shape[1]
    _need(x, "x", shape=(B, D))
    _need(conv_state, "conv_state", x.dtype, (B, D, 3))
    _need(conv_w, "conv_w", torch.float32, (D, 4))
    _need(conv_bias, "conv_bias", torch.float32, (D,))
    _need(delta, "delta", x.dtype, (B, D))
    _need(z, "z", x.dtype, (B, D))
    _need(Bm, "Bm", x.dtype, (B, N))
    _need(Cm, "Cm", x.dtype, (B, N))
    _need(A, "A", torch.float32, (D, N))
    _need(Dskip, "Dskip", torch.float32, (D,))
    _need(delta_bias, "delta_bias", torch.float32, (D,))
    _need(state, "state", torch.float32, (B, D, N))
    out = torch.empty_like(x) if out is None else out
    _need(out, "out", x.dtype, (B, D))
    _need(u_out, "u_out", x.dtype, (B, D))
    p = ssm_decode_params()
    p.struct_size = ctypes.sizeof(ssm_decode_params)
    p.B, p.D, p.N, p.W = B, D, N, 4
    p.dtype = _dtype_code(x)
    p.x, p.conv_state, p.conv_w = x.data_ptr(), conv_state.data_ptr(), conv_w.data_ptr()
    p.conv_bias = conv_bias.data_ptr() if conv_bias is not None else None
    p.delta = delta.data_ptr()
    p.z = z.data_ptr() if z is not None else None
    p.Bm, p.Cm, p.A = Bm.data_ptr(), Cm.data_ptr(), A.data_ptr()
    p.Dskip = Dskip.data_ptr() if Dskip is not None else None
    p.delta_bias = delta_bias.data_ptr() if delta_bias is not None else None
    p.delta_softplus = int(softplus)
    p.state, p.out = state.data_ptr(), out.data_ptr()
    p.u_out = u_out.data_ptr() if u_out is not None else None
    _lib.check(ssm_decode_step(p, _stream(stream, x.device)))
    return out


def scan_fwd_summary(u, delta, A, Bm, *, delta_bias=None, softplus=True, seq_idx=None,
                     seq_prev=None, zoh=False, workspace=None, n_splits=0, stream=None):
    """Summary of this piece of a longer sequence: (decay, state_end), each
    [B, D, N] fp32, with final state = decay * (state entering) + state_end.
    n_splits as in scan_fwd (1 selects the N = 16 kernels where they apply).
    seq_prev [B] int32: document id of the token before token 0."""
    torch = _torch()
    B, D, L = u.shape
    N = A.shape[1]
    _need(seq_prev, "seq_prev", torch.int32, (B,))
    # the forward summary reads no C: Bm fills that slot of the parameter block
    p = scan_params(u, delta, A, Bm, Bm, delta_bias=delta_bias, softplus=softplus,
                    seq_idx=seq_idx, zoh=zoh, n_splits=n_splits)
    need = ssm_scan_workspace_size(p)
    if workspace is None or workspace.numel() < need:
        workspace = torch.empty(need, dtype=torch.uint8, device=u.device)
    p.workspace, p.workspace_bytes = workspace.data_ptr(), workspace.numel()
    decay = torch.empty((B, D, N), dtype=torch.float32, device=u.device)
    end = torch.empty_like(decay)
    _lib.check(ssm_scan_fwd_summary(p, _ptr(seq_prev), decay.data_ptr(), end.data_ptr(),
                                    _stream(stream, u.device)))
    return decay, end


def scan_bwd_summary(delta, A, Cm, dout, *, z=None, delta_bias=None, softplus=True,
                     seq_idx=None, seq_prev=None, workspace=None, n_splits=0, stream=None):
    """Backward summary of this piece from dout alone: (decay, adj_start),
    each [B, D, N] fp32; the gradient leaving the piece through its start is
    decay * (gradient of its final state) + adj_start."""
    torch = _torch()
    B, D, L = delta.shape
    N = A.shape[1]
    _need(dout, "dout", delta.dtype, (B, D, L))
    _need(seq_prev, "seq_prev", torch.int32, (B,))
    # the backward summary reads no u and no B: delta and Cm fill those slots
    p = scan_params(delta, delta, A, Cm, Cm, z=z, delta_bias=delta_bias, softplus=softplus,
                    seq_idx=seq_idx, n_splits=n_splits)
    need = ssm_scan_workspace_size(p)
    if workspace is None or workspace.numel() < need:
        workspace = torch.empty(need, dtype=torch.uint8, device=delta.device)
    p.workspace, p.workspace_bytes = workspace.data_ptr(), workspace.numel()
    decay = torch.empty((B, D, N), dtype=torch.float32, device=delta.device)
    adj = torch.empty_like(decay)
    _lib.check(ssm_scan_bwd_summary(p, dout.data_ptr(), _ptr(seq_prev), decay.data_ptr(),
                                    adj.data_ptr(), _stream(stream, delta.device)))
    return decay, adj


def state_carry(decay, value, r, *, reverse=False, init=None, seq_prev=None, seq_idx=None,
                out=None, stream=None):
    """Fold stacked piece summaries decay, value [R, B, D, N] fp32: the state
    entering piece r (reverse=False; zero when piece r's token 0 starts a
    document per seq_prev [B] / seq_idx [B, L]) or the gradient reaching
    piece r's final state (reverse=True)."""
    torch = _torch()
    R, B, D, N = decay.shape
    _need(decay, "decay", torch.float32)
    _need(value, "value", torch.float32, (R, B, D, N))
    _need(init, "init", torch.float32, (B, D, N))
    _need(seq_prev, "seq_prev", torch.int32, (B,))
    _need(seq_idx, "seq_idx", torch.int32)
    L = seq_idx.shape[1] if seq_idx is not None else 0
    out = torch.empty((B, D, N), dtype=torch.float32, device=decay.device) if out is None else out
    _need(out, "out", torch.float32, (B, D, N))
    _lib.check(ssm_state_carry(decay.data_ptr(), value.data_ptr(), R, int(r), int(reverse),
                               _ptr(init), _ptr(seq_prev), _ptr(seq_idx), L, out.data_ptr(), B, D,
                               N, _stream(stream, decay.device)))
    return out


SSD_CHUNK = 128  # tokens per chunk of the SSD kernels


def ssd_chunk_states_shape(B, L, H, P=64, N=128):
    """Shape of the per-chunk entering states the SSD forward saves for the
    backward: [B, H, ceil(L / 128), N, P] fp32."""
    return (B, H, (L + SSD_CHUNK - 1) // SSD_CHUNK, N, P)


def _ssd_params(x, dt_raw, A, Bm, Cm, D, dt_bias, softplus, seq_idx, status, chunk_states):
    torch = _torch()
    B, L, H, P = x.shape
    G, N = Bm.shape[2], Bm.shape[3]
    _need(x, "x", torch.bfloat16, (B, L, H, P))
    _need(dt_raw, "dt_raw", torch.bfloat16, (B, L, H))
    _need(Bm, "Bm", torch.bfloat16, (B, L, G, N))
    _need(Cm, "Cm", torch.bfloat16, (B, L, G, N))
    _need(A, "A", torch.float32, (H,))
    _need(D, "D", torch.float32, (H,))
    _need(dt_bias, "dt_bias", torch.float32, (H,))
    _need(seq_idx, "seq_idx", torch.int32, (B, L))
    _need(chunk_states, "chunk_states", torch.float32, ssd_chunk_states_shape(B, L, H, P, N))
    p = ssm_ssd_params()
    p.struct_size = ctypes.sizeof(ssm_ssd_params)
    p.B, p.L, p.H, p.P, p.G, p.N = B, L, H, P, G, N
    p.dtype = 1
    p.x, p.dt_raw, p.A = x.data_ptr(), dt_raw.data_ptr(), A.data_ptr()
    p.Bm, p.Cm = Bm.data_ptr(), Cm.data_ptr()
    p.D = D.data_ptr() if D is not None else None
    p.dt_bias = dt_bias.data_ptr() if dt_bias is not None else None
    p.dt_softplus = 1 if softplus else 0
    p.seq_idx = seq_idx.data_ptr() if seq_idx is not None else None
    p.status = status.data_ptr() if status is not None else None
    p.chunk_states = chunk_states.data_ptr() if chunk_states is not None else None
    return p


def ssd_fwd(x, dt_raw, A, Bm, Cm, *, D=None, dt_bias=None, softplus=True, seq_idx=None,
            return_final_state=False, chunk_states=None, out=None, status=None, stream=None):
    """Mamba-2 SSD forward on the tensor cores.

    x [B, L, H, 64] bf16; dt_raw [B, L, H] bf16; Bm, Cm [B, L, G, 128] bf16;
    A, D, dt_bias [H] fp32; seq_idx [B, L] int32. chunk_states: a tensor of
    ssd_chunk_states_shape(B, L, H) fp32 to receive the state entering each
    chunk (what ssd_bwd needs), or None. Returns (y [B, L, H, 64] bf16,
    final_state [B, H, 64, 128] fp32 or None)."""
    torch = _torch()
    B, L, H, P = x.shape
    N = Bm.shape[3]
    p = _ssd_params(x, dt_raw, A, Bm, Cm, D, dt_bias, softplus, seq_idx, status, chunk_states)
    y = torch.empty_like(x) if out is None else out
    _need(y, "out", torch.bfloat16, (B, L, H, P))
    fs = (torch.empty((B, H, P, N), dtype=torch.float32, device=x.device)
          if return_final_state else None)
    p.y = y.data_ptr()
    p.final_state = fs.data_ptr() if fs is not None else None
    _lib.check(ssm_ssd_fwd(p, _stream(stream, x.device)))
    return y, fs


def ssd_bwd(x, dt_raw, A, Bm, Cm, dy, chunk_states, *, D=None, dt_bias=None, softplus=True,
            seq_idx=None, status=None, stream=None):
    """Backward of ssd_fwd from dy [B, L, H, 64] bf16 and the chunk_states the
    forward saved for the same inputs. Returns dict(dx [B, L, H, 64] bf16,
    ddt_raw [B, L, H] fp32, dA [H], dB, dC [B, L, G, 128] fp32, dD [H] or
    None, ddt_bias [H] or None)."""
    torch = _torch()
    B, L, H, P = x.shape
    G, N = Bm.shape[2], Bm.shape[3]
    if chunk_states is None:
        raise ValueError("ssd_bwd needs the chunk_states written by ssd_fwd")
    p = _ssd_params(x, dt_raw, A, Bm, Cm, D, dt_bias, softplus, seq_idx, status, chunk_states)
    _need(dy, "dy", torch.bfloat16, (B, L, H, P))
    f32 = dict(dtype=torch.float32, device=x.device)
    out = {"dx": torch.empty_like(x), "ddt_raw": torch.empty((B, L, H), **f32),
           "dA": torch.empty((H,), **f32), "dB": torch.empty((B, L, G, N), **f32),
           "dC": torch.empty((B, L, G, N), **f32),
           "dD": torch.empty((H,), **f32) if D is not None else None,
           "ddt_bias": torch.empty((H,), **f32) if dt_bias is not None else None}
    g = ssm_ssd_grads()
    g.struct_size = ctypes.sizeof(ssm_ssd_grads)
    g.dy, g.dx, g.ddt_raw = dy.data_ptr(), out["dx"].data_ptr(), out["ddt_raw"].data_ptr()
    g.dA, g.dB, g.dC = out["dA"].data_ptr(), out["dB"].data_ptr(), out["dC"].data_ptr()
    g.dD = out["dD"].data_ptr() if out["dD"] is not None else None
    g.ddt_bias = out["ddt_bias"].data_ptr() if out["ddt_bias"] is not None else None
    _lib.check(ssm_ssd_bwd(p, g, _stream(stream, x.device)))
    return out


def debug_report(reset: bool = False) -> dict:
    """Failed device index checks of a debug build (SSM_LIBRARY naming the
    library built with -DSSM_DEBUG): synchronises the device and returns
    dict(failures, site, site_name, offset, count, extent) of the first kept
    failure; reset clears the records. A release build raises SsmError
    (SSM_ERR_UNSUPPORTED)."""
    info = ssm_debug_info()
    info.struct_size = ctypes.sizeof(ssm_debug_info)
    _lib.check(ssm_debug_report(ctypes.byref(info), 1 if reset else 0))
    return dict(failures=int(info.failures), site=int(info.site),
                site_name=info.site_name.decode(errors="replace"), offset=int(info.offset),
                count=int(info.count), extent=int(info.extent))


def debug_selftest(buf, stream=None) -> None:
    """Debug build only: one write through offset buf.numel() of the fp32
    device tensor `buf`, which its check turns into a recorded failure and a
    write to buf[0]."""
    torch = _torch()
    _need(buf, "buf", torch.float32)
    _lib.check(ssm_debug_selftest(_ptr(buf), buf.numel(), _stream(stream, buf.device)))
