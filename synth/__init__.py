"""Seeded synthetic inputs for the Mamba-1 selective-SSM layer core.

This module is shared by the tests, the benchmark and the CPU checker. It only
draws random numbers (numpy PCG64, fixed seeds) and rounds them to the storage
format the caller asks for. It computes nothing of the layer itself: no
convolution, no discretisation, no scan.

Value recipes follow the pages' layer set-up ("hung-phan ml-skills mamba",
section "Mamba: Selective State Spaces (S6)" and "Key Training Tips" 1):
  * A[d, n] = -exp(A_log[d, n]) with A_log = log(1..N) repeated over channels,
    i.e. A[d, n] = -(n + 1) (S4D-real);
  * the delta bias is the inverse softplus of U(0.001, 0.1);
  * D (skip) = 1;
  * conv weight ~ U(-0.5, 0.5), x / z / B / C / dout ~ N(0, 1),
    raw delta ~ 0.5 * N(0, 1).
Packed rows follow the Axolotl page ("FLA Mamba and Mamba2", packing
paragraph): documents with bounded right padding, one segment id per document,
pad tokens in a segment of their own (id -1).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

SEED_BASE = 20261202


# ----------------------------------------------------------------------------
# bfloat16 storage format (round-to-nearest-even from float32)
# ----------------------------------------------------------------------------
def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16 (RNE); return the raw uint16 bits."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32)
    bias = (u >> 16) & np.uint32(1)
    bias += np.uint32(0x7FFF)
    # finite inputs cannot wrap: u + 0x8000 overflows only for NaN bit patterns
    bias += u
    bias >>= np.uint32(16)
    return bias.astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Widen raw bfloat16 bits to float32 (exact)."""
    b = np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32)


# ----------------------------------------------------------------------------
# Workload descriptions
# ----------------------------------------------------------------------------
@dataclass(frozen=True)
class Shape:
    name: str
    B: int
    D: int
    N: int
    L: int
    dtype: str  # "f32" or "bf16"
    layers: int = 1
    packed: bool = False
    boundary_at: int | None = None  # single seq_idx boundary (tiny case)
    final_state: bool = False
    conv_bias_zero: bool = True


CONFIGS = {
    1: Shape("tiny-fp32 B1 D4 N4 L64", 1, 4, 4, 64, "f32", boundary_at=30),
    2: Shape("mamba-130m layer B2 D1536 N16 L2048", 2, 1536, 16, 2048, "bf16"),
    3: Shape("long-context 4 layers B2 D1536 N16 L32768", 2, 1536, 16, 32768, "bf16", layers=4),
    4: Shape("packed-64K B2 D1536 N16 L65536", 2, 1536, 16, 65536, "bf16", packed=True),
    5: Shape("mamba-2.8b layer B4 D5120 N16 L8192", 4, 5120, 16, 8192, "bf16", final_state=True),
}


def seed_for(config: int, layer: int = 0) -> int:
    return SEED_BASE + 100 * config + layer


def packed_seq_idx(rng: np.random.Generator, L: int, mean_len: float = 2048.0,
                   sigma: float = 1.0, lo: int = 16, hi: int = 16384,
                   max_pad: int = 64) -> np.ndarray:
    """One packed row: document ids 0, 1, 2, ... and -1 for right padding.

    Lengths ~ lognormal with the given mean (mu = ln(mean) - sigma^2 / 2),
    clipped to [lo, hi]; documents are appended while they fit; the leftover
    R becomes padding when R <= max_pad, else a last document of length
    R - p followed by p ~ U{0..min(max_pad, R - lo)} pad tokens.
    """
    mu = math.log(mean_len) - 0.5 * sigma * sigma
    out = np.empty(L, dtype=np.int32)
    pos, doc = 0, 0
    while True:
        n = int(np.clip(round(rng.lognormal(mu, sigma)), lo, hi))
        rem = L - pos
        if n > rem:
            break
        out[pos:pos + n] = doc
        pos += n
        doc += 1
    rem = L - pos
    if rem > 0:
        if rem <= max_pad:
            out[pos:] = -1
        else:
            p = int(rng.integers(0, min(max_pad, rem - lo) + 1))
            out[pos:L - p] = doc
            out[L - p:] = -1
    return out


@dataclass
class Tensor:
    """One input array: float64 values plus, for bf16 storage, the raw bits."""
    f64: np.ndarray
    bits: np.ndarray | None = None  # uint16 when stored as bf16
    f32: np.ndarray | None = None   # float32 when stored as fp32

    def storage(self) -> np.ndarray:
        return self.bits if self.bits is not None else self.f32


@dataclass
class LayerInputs:
    shape: Shape
    x: Tensor
    z: Tensor
    delta: Tensor
    Bm: Tensor
    Cm: Tensor
    dout: Tensor
    A: np.ndarray          # float32 [D, N]
    Dskip: np.ndarray      # float32 [D]
    delta_bias: np.ndarray  # float32 [D]
    conv_w: np.ndarray     # float32 [D, 4]
    conv_b: np.ndarray     # float32 [D]
    seq_idx: np.ndarray | None  # int32 [B, L]
    extra: dict = field(default_factory=dict)


def _act(rng: np.random.Generator, shape, dtype: str, scale: float = 1.0,
         want_f64: bool = True) -> Tensor:
    v = rng.standard_normal(shape, dtype=np.float32)
    if scale != 1.0:
        v *= np.float32(scale)
    if dtype == "bf16":
        bits = f32_to_bf16_bits(v)
        f64 = bf16_bits_to_f32(bits).astype(np.float64) if want_f64 else None
        return Tensor(f64=f64, bits=bits)
    return Tensor(f64=v.astype(np.float64) if want_f64 else None, f32=v)


def make_inputs(shape: Shape, seed: int, *, want_f64: bool = True,
                conv_bias_scale: float = 0.0, dskip_random: bool = False) -> LayerInputs:
    """Draw one layer's inputs for `shape` from `seed`.

    Arrays use the layout of the layer core: activations [B, D, L] (L
    contiguous), B/C [B, N, L], A [D, N], per-channel vectors [D].
    `conv_bias_scale` > 0 draws a nonzero conv bias ~ U(-s, s) and
    `dskip_random` draws D ~ U(0.5, 1.5); the benchmark workloads use neither.
    """
    rng = np.random.Generator(np.random.PCG64(seed))
    B, D, N, L = shape.B, shape.D, shape.N, shape.L
    conv_w = rng.uniform(-0.5, 0.5, size=(D, 4)).astype(np.float32)
    if conv_bias_scale > 0:
        conv_b = rng.uniform(-conv_bias_scale, conv_bias_scale, size=D).astype(np.float32)
    else:
        conv_b = np.zeros(D, dtype=np.float32)
    A = -np.tile(np.arange(1, N + 1, dtype=np.float32), (D, 1))
    Dskip = (rng.uniform(0.5, 1.5, size=D).astype(np.float32) if dskip_random
             else np.ones(D, dtype=np.float32))
    dt0 = rng.uniform(1e-3, 1e-1, size=D)
    delta_bias = np.log(np.expm1(dt0)).astype(np.float32)  # inverse softplus
    x = _act(rng, (B, D, L), shape.dtype, want_f64=want_f64)
    z = _act(rng, (B, D, L), shape.dtype, want_f64=want_f64)
    delta = _act(rng, (B, D, L), shape.dtype, 0.5, want_f64=want_f64)
    Bm = _act(rng, (B, N, L), shape.dtype, want_f64=want_f64)
    Cm = _act(rng, (B, N, L), shape.dtype, want_f64=want_f64)
    dout = _act(rng, (B, D, L), shape.dtype, want_f64=want_f64)
    seq = None
    if shape.packed:
        seq = np.stack([packed_seq_idx(rng, L) for _ in range(B)])
    elif shape.boundary_at is not None:
        seq = np.zeros((B, L), dtype=np.int32)
        seq[:, shape.boundary_at:] = 1
    return LayerInputs(shape, x, z, delta, Bm, Cm, dout, A, Dskip, delta_bias,
                       conv_w, conv_b, seq)


def random_segments(rng: np.random.Generator, B: int, L: int, n_bound: int,
                    include_edges: bool = True) -> np.ndarray:
    """seq_idx with `n_bound` boundaries per row at random positions.

    With `include_edges` the boundaries include t = 1, t = L-1 and some chunk
    edges (multiples of 8 and 256) so that every tile edge case is hit.
    """
    seq = np.zeros((B, L), dtype=np.int32)
    for b in range(B):
        cand = set(int(v) for v in rng.integers(1, max(2, L), size=n_bound))
        if include_edges and L > 2:
            cand |= {1, L - 1}
            for m in (8, 256):
                if L > m:
                    cand.add(m)
                    cand.add((L // m) * m if (L // m) * m < L else m)
        cand = sorted(c for c in cand if 0 < c < L)
        cur = 0
        prev = 0
        for c in cand:
            seq[b, prev:c] = cur
            cur += 1
            prev = c
        seq[b, prev:] = cur
    return seq


def initial_state(B: int, D: int, N: int, seed: int, scale: float = 0.5) -> np.ndarray:
    """A state before token 0, float32 [B, D, N] ~ scale * N(0, 1)."""
    rng = np.random.Generator(np.random.PCG64(seed))
    return (scale * rng.standard_normal((B, D, N), dtype=np.float32)).astype(np.float32)


@dataclass
class DecodeInputs:
    """Inputs of `steps` consecutive tokens of the recurrent form.

    Per-token activations are [steps, B, D] (x, delta, z) and [steps, B, N]
    (Bm, Cm); the starting conv window is [B, D, 3] (activation dtype) and the
    starting state [B, D, N] float32."""
    x: Tensor
    delta: Tensor
    z: Tensor
    Bm: Tensor
    Cm: Tensor
    conv_state: Tensor
    h0: np.ndarray
    A: np.ndarray
    Dskip: np.ndarray
    delta_bias: np.ndarray
    conv_w: np.ndarray
    conv_b: np.ndarray


def decode_inputs(B: int, D: int, N: int, steps: int, dtype: str, seed: int) -> DecodeInputs:
    """Seeded inputs for a run of decode steps, with the value distributions
    of `make_inputs` (A = -(n+1), softplus-inverse delta bias) plus a nonzero
    conv bias, random D, a random starting conv window and starting state."""
    rng = np.random.Generator(np.random.PCG64(seed))
    conv_w = rng.uniform(-0.5, 0.5, size=(D, 4)).astype(np.float32)
    conv_b = rng.uniform(-0.2, 0.2, size=D).astype(np.float32)
    A = -np.tile(np.arange(1, N + 1, dtype=np.float32), (D, 1))
    Dskip = rng.uniform(0.5, 1.5, size=D).astype(np.float32)
    delta_bias = np.log(np.expm1(rng.uniform(1e-3, 1e-1, size=D))).astype(np.float32)
    x = _act(rng, (steps, B, D), dtype)
    z = _act(rng, (steps, B, D), dtype)
    delta = _act(rng, (steps, B, D), dtype, 0.5)
    Bm = _act(rng, (steps, B, N), dtype)
    Cm = _act(rng, (steps, B, N), dtype)
    conv_state = _act(rng, (B, D, 3), dtype)
    h0 = (0.5 * rng.standard_normal((B, D, N), dtype=np.float32)).astype(np.float32)
    return DecodeInputs(x, delta, z, Bm, Cm, conv_state, h0, A, Dskip, delta_bias, conv_w, conv_b)


@dataclass
class ComplexInputs:
    """Inputs of the scan with a complex diagonal A.

    u, delta, z, dout: [B, D, L]; Bm, Cm: [B, N, 2, L] (per state a real then
    an imaginary row); A: float32 [D, N, 2] (re, im); h0: float32
    [B, D, N, 2] or None."""
    u: Tensor
    delta: Tensor
    z: Tensor
    dout: Tensor
    Bm: Tensor
    Cm: Tensor
    A: np.ndarray
    Dskip: np.ndarray
    delta_bias: np.ndarray
    seq_idx: np.ndarray | None
    h0: np.ndarray | None



def complex_inputs(B: int, D: int, N: int, L: int, dtype: str, seed: int, *,
                   seq_idx: np.ndarray | None = None, with_h0: bool = False) -> ComplexInputs:
    """Seeded inputs for the complex-A scan. A follows S4D-Lin:
    A[d, n] = -1/2 + i pi n; the delta bias, D, u, z, delta and dout follow
    `make_inputs` (u ~ N(0, 1) stands for the conv output); the real and
    imaginary parts of B and C are each ~ N(0, 1)."""
    rng = np.random.Generator(np.random.PCG64(seed))
    A = np.zeros((D, N, 2), dtype=np.float32)
    A[:, :, 0] = -0.5
    A[:, :, 1] = (np.pi * np.arange(N)).astype(np.float32)[None, :]
    Dskip = rng.uniform(0.5, 1.5, size=D).astype(np.float32)
    delta_bias = np.log(np.expm1(rng.uniform(1e-3, 1e-1, size=D))).astype(np.float32)
    u = _act(rng, (B, D, L), dtype)
    z = _act(rng, (B, D, L), dtype)
    delta = _act(rng, (B, D, L), dtype, 0.5)
    Bm = _act(rng, (B, N, 2, L), dtype)
    Cm = _act(rng, (B, N, 2, L), dtype)
    dout = _act(rng, (B, D, L), dtype)
    h0 = (0.5 * rng.standard_normal((B, D, N, 2), dtype=np.float32)).astype(np.float32) \
        if with_h0 else None
    return ComplexInputs(u, delta, z, dout, Bm, Cm, A, Dskip, delta_bias, seq_idx, h0)


@dataclass
class SsdInputs:
    """Inputs of the Mamba-2 SSD forward: x [B, L, H, P], dt_raw [B, L, H],
    Bm, Cm [B, L, G, N] (bf16 storage); A, D, dt_bias float32 [H]; seq_idx
    int32 [B, L] or None."""
    x: Tensor
    dt_raw: Tensor
    Bm: Tensor
    Cm: Tensor
    A: np.ndarray
    D: np.ndarray
    dt_bias: np.ndarray
    seq_idx: np.ndarray | None


def ssd_inputs(B: int, L: int, H: int, P: int, G: int, N: int, seed: int, *,
               seq_idx: np.ndarray | None = None) -> SsdInputs:
    """Seeded SSD inputs, the Mamba-1 recipes with A a scalar per head:
    A[h] = -U(1, 16), the dt bias the inverse softplus of U(0.001, 0.1),
    D ~ U(0.5, 1.5), x / B / C ~ N(0, 1), raw dt ~ 0.5 * N(0, 1); bf16 storage."""
    rng = np.random.Generator(np.random.PCG64(seed))
    A = (-rng.uniform(1.0, 16.0, size=H)).astype(np.float32)
    D = rng.uniform(0.5, 1.5, size=H).astype(np.float32)
    dt_bias = np.log(np.expm1(rng.uniform(1e-3, 1e-1, size=H))).astype(np.float32)
    x = _act(rng, (B, L, H, P), "bf16")
    dt_raw = _act(rng, (B, L, H), "bf16", 0.5)
    Bm = _act(rng, (B, L, G, N), "bf16")
    Cm = _act(rng, (B, L, G, N), "bf16")
    return SsdInputs(x, dt_raw, Bm, Cm, A, D, dt_bias, seq_idx)
