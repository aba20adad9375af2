"""Test helpers: run the layer core through the CUDA library, and compare.

The GPU side goes through the package's binding (and so the C ABI); the
expected side comes only from `oracle` on the same seeded inputs.
"""
from __future__ import annotations

import numpy as np

import synth


def rel_l2(got, want) -> float:
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    den = np.linalg.norm(want.ravel())
    num = np.linalg.norm((got - want).ravel())
    return float(num / den) if den > 0 else float(num)


def max_abs(got, want) -> float:
    return float(np.max(np.abs(np.asarray(got, np.float64) - np.asarray(want, np.float64))))


def bf16_out_max_abs_ok(got, want, tol) -> tuple[bool, float]:
    """The max-abs bound on a bf16 output against the oracle rounded to bf16.

    Both sides round to bf16, so where the exact value sits near a rounding
    boundary they can land one bf16 step apart; for |y| >= 4 that step
    (2^-5) already exceeds a bound of 2e-2. So: |got - want| <= tol where
    |want| < 4, and at most one bf16 step of `want` elsewhere. Returns
    (ok, worst error in units of the allowed bound)."""
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    err = np.abs(got - want)
    aw = np.abs(want)
    step = np.exp2(np.floor(np.log2(np.maximum(aw, 1e-30))) - 7)
    allowed = np.where(aw < 4.0, tol, np.maximum(tol, step))
    worst = float(np.max(err / allowed))
    return worst <= 1.0, worst


def to_dev(t: synth.Tensor, device):
    import torch
    if t.bits is not None:
        return torch.from_numpy(t.bits.view(np.int16).copy()).view(torch.bfloat16).to(device)
    return torch.from_numpy(np.ascontiguousarray(t.f32)).to(device)


def f32_dev(a, device):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(device)


def host64(t) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def device_inputs(inp: synth.LayerInputs, device="cuda"):
    import torch
    d = {
        "x": to_dev(inp.x, device), "z": to_dev(inp.z, device), "delta": to_dev(inp.delta, device),
        "Bm": to_dev(inp.Bm, device), "Cm": to_dev(inp.Cm, device), "dout": to_dev(inp.dout, device),
        "A": f32_dev(inp.A, device), "Dskip": f32_dev(inp.Dskip, device),
        "delta_bias": f32_dev(inp.delta_bias, device), "conv_w": f32_dev(inp.conv_w, device),
        "conv_b": f32_dev(inp.conv_b, device),
        "seq_idx": (torch.from_numpy(np.ascontiguousarray(inp.seq_idx, dtype=np.int32)).to(device)
                    if inp.seq_idx is not None else None),
    }
    return d


def gpu_layer(dv, *, n_splits=0, use_z=True, use_seq=True, softplus=True, final_state=True,
              deterministic=False):
    """conv fwd -> scan fwd -> scan bwd -> conv bwd on device tensors `dv`."""
    import selective_state_space_35_b200 as ssm
    seq = dv["seq_idx"] if use_seq else None
    z = dv["z"] if use_z else None
    u = ssm.conv1d_fwd(dv["x"], dv["conv_w"], dv["conv_b"], seq)
    out, fs, ws = ssm.scan_fwd(u, dv["delta"], dv["A"], dv["Bm"], dv["Cm"], z=z,
                               Dskip=dv["Dskip"], delta_bias=dv["delta_bias"], softplus=softplus,
                               seq_idx=seq, n_splits=n_splits, return_final_state=final_state)
    # the forward's bounded tile waits record a timeout in the status word
    assert ssm.scan_status(u, dv["A"], ws) == 0
    g = ssm.scan_bwd(u, dv["delta"], dv["A"], dv["Bm"], dv["Cm"], dv["dout"], ws, z=z,
                     Dskip=dv["Dskip"], delta_bias=dv["delta_bias"], softplus=softplus,
                     seq_idx=seq, n_splits=n_splits, deterministic=deterministic)
    dx, dw, dcb = ssm.conv1d_bwd(dv["x"], dv["conv_w"], dv["conv_b"], seq, g["du"])
    res = {"u": u, "out": out, "final_state": fs, "dx": dx, "dconv_w": dw, "dconv_b": dcb}
    res.update(g)
    return res


# Tolerances. fp32: rel-L2 1e-5 on everything. bf16 inputs with fp32 state:
# out rel-L2 2e-3 and max-abs 2e-2 (against the oracle rounded to bf16);
# every gradient rel-L2 5e-3.
TOL_F32 = 1e-5
TOL_BF16_OUT = 2e-3
TOL_BF16_OUT_MAX = 2e-2
TOL_GRAD = 5e-3
