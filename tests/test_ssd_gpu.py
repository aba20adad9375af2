"""Mamba-2 SSD forward and backward on the tensor cores against the fp64
oracle, on the same bf16 inputs: chunks of 128 tokens with a ragged tail,
several heads per B / C group, document starts inside a chunk, at a chunk
start and in consecutive tokens, with and without softplus, D and the dt
bias. Forward: y rel-L2 <= 2e-3 against the oracle rounded to bf16, final
state <= 5e-3. Backward: every gradient rel-L2 <= 5e-3 (dx against the
oracle rounded to bf16)."""
import numpy as np
import pytest

import oracle
import synth
from pipeline import TOL_BF16_OUT, TOL_BF16_OUT_MAX, TOL_GRAD, bf16_out_max_abs_ok, host64, rel_l2

pytestmark = pytest.mark.gpu


def _dev(t):
    import torch
    return torch.from_numpy(t.bits.view(np.int16).copy()).view(torch.bfloat16).cuda()


def _f32(a):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda()


def _run(si, softplus=True, use_D=True):
    import torch
    import selective_state_space_35_b200 as ssm
    seq = torch.from_numpy(si.seq_idx).cuda() if si.seq_idx is not None else None
    y, fs = ssm.ssd_fwd(_dev(si.x), _dev(si.dt_raw), _f32(si.A), _dev(si.Bm), _dev(si.Cm),
                        D=_f32(si.D) if use_D else None, dt_bias=_f32(si.dt_bias),
                        softplus=softplus, seq_idx=seq, return_final_state=True)
    torch.cuda.synchronize()
    want = oracle.ssd_fwd(si.x.f64, si.dt_raw.f64, si.A, si.Bm.f64, si.Cm.f64,
                          D=si.D if use_D else None, dt_bias=si.dt_bias, softplus=softplus,
                          seq_idx=si.seq_idx)
    return y, fs, want


def _check(y, fs, want):
    wy = oracle.round_bf16(want["y"])
    e = rel_l2(host64(y), wy)
    assert e <= TOL_BF16_OUT, e
    ok, worst = bf16_out_max_abs_ok(host64(y), wy, TOL_BF16_OUT_MAX)
    assert ok, worst
    ef = rel_l2(host64(fs), want["final_state"])
    assert ef <= TOL_GRAD, ef


@pytest.mark.parametrize("B,L,H,G,nb", [(1, 128, 1, 1, 0), (1, 256, 2, 1, 0), (2, 300, 4, 2, 3),
                                        (1, 1000, 3, 1, 6), (2, 77, 2, 2, 2), (2, 520, 4, 2, 2)])
def test_ssd_fwd_parity(B, L, H, G, nb):
    seed = 7100 + L + H
    seq = None
    if nb:
        seq = synth.random_segments(np.random.Generator(np.random.PCG64(seed)), B, L, nb)
    si = synth.ssd_inputs(B, L, H, 64, G, 128, seed, seq_idx=seq)
    _check(*_run(si))


def test_ssd_fwd_edges_of_documents():
    B, L, H = 1, 384, 2
    seq = np.zeros((B, L), dtype=np.int32)
    doc = 0
    for t in range(L):  # starts at a chunk start, right after one, in a row, at the end
        if t in (1, 2, 3, 127, 128, 129, 255, 256, 300, 383):
            doc += 1
        seq[0, t] = doc
    si = synth.ssd_inputs(B, L, H, 64, 1, 128, 7301, seq_idx=seq)
    _check(*_run(si))


@pytest.mark.parametrize("softplus,use_D", [(False, True), (True, False)])
def test_ssd_fwd_options(softplus, use_D):
    si = synth.ssd_inputs(1, 256, 2, 64, 1, 128, 7402)
    if not softplus:  # dt used as given: keep it positive
        bits = synth.f32_to_bf16_bits(np.abs(synth.bf16_bits_to_f32(si.dt_raw.bits)) * 0.1)
        si.dt_raw = synth.Tensor(f64=synth.bf16_bits_to_f32(bits).astype(np.float64), bits=bits)
        si.dt_bias = np.zeros_like(si.dt_bias)
    _check(*_run(si, softplus=softplus, use_D=use_D))


# ---------------------------------------------------------------- backward
def _run_bwd(si, seed, softplus=True, use_D=True, use_bias=True):
    import torch
    import selective_state_space_35_b200 as ssm
    B, L, H, P = si.x.f64.shape
    seq = torch.from_numpy(si.seq_idx).cuda() if si.seq_idx is not None else None
    rng = np.random.Generator(np.random.PCG64(seed))
    bits = synth.f32_to_bf16_bits(rng.standard_normal((B, L, H, P)).astype(np.float32))
    dy = synth.Tensor(f64=synth.bf16_bits_to_f32(bits).astype(np.float64), bits=bits)
    kw = dict(D=_f32(si.D) if use_D else None, dt_bias=_f32(si.dt_bias) if use_bias else None,
              softplus=softplus, seq_idx=seq)
    x, dt, A, Bm, Cm = _dev(si.x), _dev(si.dt_raw), _f32(si.A), _dev(si.Bm), _dev(si.Cm)
    cs = torch.full(ssm.ssd_chunk_states_shape(B, L, H), float("nan"), device="cuda")
    ssm.ssd_fwd(x, dt, A, Bm, Cm, chunk_states=cs, **kw)
    got = ssm.ssd_bwd(x, dt, A, Bm, Cm, _dev(dy), cs, **kw)
    torch.cuda.synchronize()
    want = oracle.ssd_bwd(si.x.f64, si.dt_raw.f64, si.A, si.Bm.f64, si.Cm.f64, dy.f64,
                          D=si.D if use_D else None, dt_bias=si.dt_bias if use_bias else None,
                          softplus=softplus, seq_idx=si.seq_idx)
    return got, want


def _check_bwd(got, want):
    errs = {"dx": rel_l2(host64(got["dx"]), oracle.round_bf16(want["dx"]))}
    for k in ("ddt_raw", "dA", "dB", "dC", "dD", "ddt_bias"):
        if got[k] is not None:
            errs[k] = rel_l2(host64(got[k]), want[k])
    bad = {k: e for k, e in errs.items() if not e <= TOL_GRAD}
    assert not bad, errs


@pytest.mark.parametrize("B,L,H,G,nb", [(1, 128, 1, 1, 0), (1, 256, 2, 1, 0), (2, 300, 4, 2, 3),
                                        (1, 1000, 3, 1, 6), (2, 77, 2, 2, 2), (2, 520, 4, 2, 2)])
def test_ssd_bwd_parity(B, L, H, G, nb):
    """Every gradient against the oracle: one chunk, several, a ragged tail,
    two heads per B / C group (dB, dC summed over them), document starts.
    L a multiple of 8 takes the tensor-map copies for whole chunks (with two
    batch entries at L = 520: rows offset by the batch, and the ragged last
    chunk's dB / dC boxes reaching into the next entry's rows with zeros)."""
    seed = 7500 + L + H
    seq = None
    if nb:
        seq = synth.random_segments(np.random.Generator(np.random.PCG64(seed)), B, L, nb)
    si = synth.ssd_inputs(B, L, H, 64, G, 128, seed, seq_idx=seq)
    _check_bwd(*_run_bwd(si, seed + 1))


def test_ssd_bwd_edges_of_documents():
    B, L, H = 1, 384, 2
    seq = np.zeros((B, L), dtype=np.int32)
    doc = 0
    for t in range(L):
        if t in (1, 2, 3, 127, 128, 129, 255, 256, 300, 383):
            doc += 1
        seq[0, t] = doc
    si = synth.ssd_inputs(B, L, H, 64, 1, 128, 7601, seq_idx=seq)
    _check_bwd(*_run_bwd(si, 7602))


@pytest.mark.parametrize("softplus,use_D,use_bias", [(False, True, False), (True, False, True),
                                                     (True, True, False)])
def test_ssd_bwd_options(softplus, use_D, use_bias):
    si = synth.ssd_inputs(1, 256, 2, 64, 1, 128, 7702)
    if not softplus:  # dt used as given: keep it positive
        bits = synth.f32_to_bf16_bits(np.abs(synth.bf16_bits_to_f32(si.dt_raw.bits)) * 0.1)
        si.dt_raw = synth.Tensor(f64=synth.bf16_bits_to_f32(bits).astype(np.float64), bits=bits)
        si.dt_bias = np.zeros_like(si.dt_bias)
    _check_bwd(*_run_bwd(si, 7703, softplus=softplus, use_D=use_D, use_bias=use_bias))
