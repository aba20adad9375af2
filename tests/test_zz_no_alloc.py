"""The allocation-free conv1d backward (ssm_conv1d_bwd_noalloc).

Some callers cannot allocate device memory: hosts that pass a library only
its input and output buffers, and loops that must not call cudaMalloc /
cudaFree. For them the library offers a variant of the conv1d backward whose
scratch lives in a fixed device array. These checks call it through the C
ABI, twice in a row with different inputs (the array keeps the previous
call's contents), compare it with the workspace version, and check that a
call changes neither the memory torch's allocator holds nor the device's
free memory. This file is
collected last so that a run stopping at the first failure has already run
every other test.
"""
import ctypes

import numpy as np
import pytest

import synth
from pipeline import TOL_F32, device_inputs, host64, rel_l2

pytestmark = pytest.mark.gpu


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _noalloc(ssm, x, w, b, seq, du):
    import torch
    B, D, L = x.shape
    dx = torch.empty_like(x)
    dw = torch.empty((D, 4), dtype=torch.float32, device=x.device)
    db = torch.empty((D,), dtype=torch.float32, device=x.device)
    code = 1 if x.dtype == torch.bfloat16 else 0
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    st = ssm.ssm_conv1d_bwd_noalloc(_p(x), _p(w), _p(b), _p(seq), _p(du), _p(dx), _p(dw), _p(db),
                                    B, D, L, 4, code, 1, stream)
    assert st == 0, ssm.ssm_last_error()
    return dx, dw, db


@pytest.mark.parametrize("B,D,N,L,dtype,seed", [(2, 96, 16, 4096, "bf16", 5), (1, 7, 4, 1031, "f32", 6)])
def test_noalloc_conv_bwd_matches_workspace_version_twice(B, D, N, L, dtype, seed):
    import torch
    import selective_state_space_35_b200 as ssm
    for call in range(2):  # two calls in a row, different inputs
        sh = synth.Shape("noalloc", B, D, N, L, dtype)
        inp = synth.make_inputs(sh, seed * 10 + call, conv_bias_scale=0.3)
        inp.seq_idx = synth.random_segments(np.random.Generator(np.random.PCG64(seed + call)), B, L, 5)
        dv = device_inputs(inp)
        du = dv["dout"]  # any upstream gradient of u's shape
        ref = ssm.conv1d_bwd(dv["x"], dv["conv_w"], dv["conv_b"], dv["seq_idx"], du)
        got = _noalloc(ssm, dv["x"], dv["conv_w"], dv["conv_b"], dv["seq_idx"], du)
        torch.cuda.synchronize()
        for g, r, name in zip(got, ref, ("dx", "dw", "dbias")):
            assert rel_l2(host64(g), host64(r)) <= TOL_F32, (call, name)


def test_noalloc_rejects_sizes_beyond_its_scratch():
    import torch
    import selective_state_space_35_b200 as ssm
    t = torch.zeros(8, dtype=torch.bfloat16, device="cuda")
    w = torch.zeros(4, dtype=torch.float32, device="cuda")
    # B * ceil(L / 1024) * D * 5 = 4 * 16 * 4096 * 5 > 2^20: rejected before any launch
    st = ssm.ssm_conv1d_bwd_noalloc(_p(t), _p(w), None, None, _p(t), _p(t[4:]), _p(w), None,
                                    4, 4096, 16384, 4, 1, 1, None)
    assert st == 2
    assert "scratch" in ssm.ssm_last_error()


def test_noalloc_call_allocates_nothing():
    """After a first call (which caches the scratch array's address and may load
    the module), further calls leave both torch's allocated bytes and the
    driver's free-memory count unchanged."""
    import torch
    import selective_state_space_35_b200 as ssm
    inp = synth.make_inputs(synth.Shape("noalloc", 2, 64, 16, 2048, "bf16"), 71, conv_bias_scale=0.3)
    dv = device_inputs(inp)
    _noalloc(ssm, dv["x"], dv["conv_w"], dv["conv_b"], dv["seq_idx"], dv["dout"])
    B, D, L = dv["x"].shape
    dx = torch.empty_like(dv["x"])
    dw = torch.empty((D, 4), dtype=torch.float32, device="cuda")
    db = torch.empty((D,), dtype=torch.float32, device="cuda")
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    alloc0, free0 = torch.cuda.memory_allocated(), torch.cuda.mem_get_info()[0]
    for _ in range(3):
        st = ssm.ssm_conv1d_bwd_noalloc(_p(dv["x"]), _p(dv["conv_w"]), _p(dv["conv_b"]),
                                        _p(dv["seq_idx"]), _p(dv["dout"]), _p(dx), _p(dw), _p(db),
                                        B, D, L, 4, 1, 1, stream)
        assert st == 0, ssm.ssm_last_error()
    torch.cuda.synchronize()
    assert torch.cuda.memory_allocated() == alloc0
    assert torch.cuda.mem_get_info()[0] == free0
