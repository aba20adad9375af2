"""The fused conv + SiLU + scan forward (ssm_conv1d_scan_fwd) against the
separate ssm_conv1d_fwd + ssm_scan_fwd: bitwise equal u, out, final state
and workspace (so an identical backward), including ragged L, packed
documents, forced L-splits (the conv halo at every split start) and N < 16;
and the fused layer against the fp64 oracle."""
import numpy as np
import pytest

import oracle
import synth
from pipeline import (TOL_BF16_OUT, TOL_F32, TOL_GRAD, device_inputs, f32_dev, host64, rel_l2,
                      to_dev)

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dtype,L,N,packed,n_splits,zoh", [
    ("bf16", 2048, 16, False, 1, False),
    ("bf16", 2048, 16, True, 3, False),
    ("bf16", 1001, 16, True, 1, False),     # ragged: scalar path
    ("f32", 777, 5, False, 2, False),
    ("f32", 512, 16, True, 1, False),
    ("bf16", 1024, 16, True, 2, True),      # zero-order hold
])
def test_fused_equals_separate_bitwise(dtype, L, N, packed, n_splits, zoh):
    import torch
    import selective_state_space_35_b200 as ssm
    B, D = 2, 24
    seed = 7500 + L + N + 10 * n_splits + int(packed)
    inp = synth.make_inputs(synth.Shape("fused", B, D, N, L, dtype), seed, conv_bias_scale=0.3,
                            dskip_random=True)
    if packed:
        inp.seq_idx = synth.random_segments(np.random.Generator(np.random.PCG64(seed)), B, L, 9)
    dv = device_inputs(inp)
    kw = dict(z=dv["z"], Dskip=dv["Dskip"], delta_bias=dv["delta_bias"], seq_idx=dv["seq_idx"],
              n_splits=n_splits, zoh=zoh)
    # zero-filled workspaces: the regions the forward does not write compare equal too
    size = ssm.scan_workspace_size(ssm.scan_params(dv["x"], dv["delta"], dv["A"], dv["Bm"],
                                                   dv["Cm"], z=dv["z"], seq_idx=dv["seq_idx"],
                                                   n_splits=n_splits))
    w1 = torch.zeros(size, dtype=torch.uint8, device="cuda")
    w2 = torch.zeros(size, dtype=torch.uint8, device="cuda")
    u1 = ssm.conv1d_fwd(dv["x"], dv["conv_w"], dv["conv_b"], dv["seq_idx"])
    o1, f1, w1 = ssm.scan_fwd(u1, dv["delta"], dv["A"], dv["Bm"], dv["Cm"], return_final_state=True,
                              workspace=w1, **kw)
    o2, u2, f2, w2 = ssm.conv1d_scan_fwd(dv["x"], dv["conv_w"], dv["conv_b"], dv["delta"], dv["A"],
                                         dv["Bm"], dv["Cm"], return_final_state=True, workspace=w2,
                                         **kw)
    assert ssm.scan_status(u2, dv["A"], w2) == 0
    torch.cuda.synchronize()
    assert torch.equal(u1, u2)
    assert torch.equal(o1, o2)
    assert torch.equal(f1, f2)
    assert torch.equal(w1, w2)
    g1 = ssm.scan_bwd(u1, dv["delta"], dv["A"], dv["Bm"], dv["Cm"], dv["dout"], w1, **kw)
    g2 = ssm.scan_bwd(u2, dv["delta"], dv["A"], dv["Bm"], dv["Cm"], dv["dout"], w2, **kw)
    for k in ("du", "ddelta", "dz", "dA", "dD", "ddelta_bias", "dinitial_state"):
        assert torch.equal(g1[k], g2[k]), k


def test_fused_layer_parity_with_oracle():
    """conv+scan fused forward, then the scan and conv backward, against the
    oracle's chained layer (bf16 rounding points as in the separate path)."""
    import torch
    import selective_state_space_35_b200 as ssm
    inp = synth.make_inputs(synth.Shape("fused-parity", 2, 32, 16, 1536, "bf16"), 7601,
                            conv_bias_scale=0.2, dskip_random=True)
    inp.seq_idx = synth.random_segments(np.random.Generator(np.random.PCG64(7601)), 2, 1536, 5)
    dv = device_inputs(inp)
    kw = dict(z=dv["z"], Dskip=dv["Dskip"], delta_bias=dv["delta_bias"], seq_idx=dv["seq_idx"])
    out, u, _, ws = ssm.conv1d_scan_fwd(dv["x"], dv["conv_w"], dv["conv_b"], dv["delta"], dv["A"],
                                        dv["Bm"], dv["Cm"], **kw)
    g = ssm.scan_bwd(u, dv["delta"], dv["A"], dv["Bm"], dv["Cm"], dv["dout"], ws, **kw)
    dx, dw, db = ssm.conv1d_bwd(dv["x"], dv["conv_w"], dv["conv_b"], dv["seq_idx"], g["du"])
    torch.cuda.synchronize()
    want = oracle.layer_fwd_bwd(inp, bf16_points=True, nthreads=8)
    assert rel_l2(host64(u), oracle.round_bf16(want["u_stored"])) <= TOL_BF16_OUT
    assert rel_l2(host64(out), oracle.round_bf16(want["out"])) <= TOL_BF16_OUT
    for k, got in (("dx", dx), ("dconv_w", dw), ("dconv_b", db), ("dA", g["dA"]),
                   ("dB", g["dB"]), ("dC", g["dC"])):
        w = oracle.round_bf16(want[k]) if k == "dx" else want[k]
        assert rel_l2(host64(got), w) <= TOL_GRAD, k
