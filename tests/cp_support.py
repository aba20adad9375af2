"""Test helpers for the context-parallel driver.

`OracleOps`: the per-shard steps computed by the fp64 oracle on CPU torch
tensors (float64), so that the driver's exchange logic can run on CPU ranks
(gloo). Conv halos are handled by running the oracle conv on the shard with
its halos attached; summaries come from oracle runs (decay = final state
from a ones initial state minus from zeros; the backward summary is the
oracle's dh0 with nothing reaching the final state).

`ThreadComm`: R ranks as threads of one process exchanging tensors through
shared slots and a barrier (no kernel waits on another; the host threads
synchronise), for running the GPU driver on one device.

`full_problem` / `full_reference`: seeded inputs for a whole sequence and the
unsharded oracle result (conv -> scan -> scan backward -> conv backward).
"""
from __future__ import annotations

import threading

import numpy as np

import oracle

HALO = 3


def _np(t, dtype=np.float64):
    return None if t is None else t.detach().cpu().numpy().astype(dtype)


def _t(a):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a))


def _cat(parts, axis=-1):
    return np.concatenate([p for p in parts if p is not None], axis=axis)


class OracleOps:
    def conv_fwd(self, x, w, b, seq, x_prev, seq_prev):
        xs = _cat([_np(x_prev), _np(x)])
        sq = None if seq is None else _cat([_np(seq_prev, np.int32), _np(seq, np.int32)])
        _, u = oracle.conv1d_fwd(xs, _np(w), _np(b), sq)
        return _t(u[..., HALO:] if x_prev is not None else u)

    def conv_bwd(self, x, w, b, seq, du, x_prev, seq_prev, x_next, du_next, seq_next):
        xn, dun = _np(x), _np(du)
        xs = _cat([_np(x_prev), xn, _np(x_next)])
        sq = None if seq is None else _cat([_np(seq_prev, np.int32), _np(seq, np.int32),
                                            _np(seq_next, np.int32)])
        lo = HALO if x_prev is not None else 0
        zeros = np.zeros(xn.shape[:-1] + (HALO,))
        pre = zeros if x_prev is not None else None
        # dx: this shard's du plus the next shard's first du (through the taps)
        dx, _, _ = oracle.conv1d_bwd(xs, _np(w), _np(b), sq,
                                     _cat([pre, dun, _np(du_next)]))
        # dw, dbias: this shard's own tokens only
        post = zeros if x_next is not None else None
        _, dw, db = oracle.conv1d_bwd(xs, _np(w), _np(b), sq, _cat([pre, dun, post]))
        L = xn.shape[-1]
        return _t(dx[..., lo:lo + L]), _t(dw), _t(db)

    @staticmethod
    def _cut(seq, seq_prev):
        if seq is None or seq_prev is None:
            return None
        return _np(seq_prev, np.int64) != _np(seq, np.int64)[:, 0]

    def scan_fwd_summary(self, u, delta, A, Bm, seq, seq_prev, delta_bias, softplus, zoh=False):
        un, dn, An, Bn = _np(u), _np(delta), _np(A), _np(Bm)
        sq = _np(seq, np.int32)
        kw = dict(delta_bias=_np(delta_bias), softplus=softplus, seq_idx=sq, zoh=zoh)
        f0 = oracle.scan_fwd(un, dn, An, Bn, Bn, **kw)["final_state"]
        f1 = oracle.scan_fwd(un, dn, An, Bn, Bn, h0=np.ones_like(f0), **kw)["final_state"]
        decay = f1 - f0
        cut = self._cut(seq, seq_prev)
        if cut is not None:
            decay[cut] = 0.0
        return _t(decay), _t(f0)

    def scan_bwd_summary(self, delta, A, Cm, dout, z, seq, seq_prev, delta_bias, softplus):
        dn, An, Cn = _np(delta), _np(A), _np(Cm)
        zeros_u = np.zeros_like(dn)
        sq = _np(seq, np.int32)
        kw = dict(z=_np(z), delta_bias=_np(delta_bias), softplus=softplus, seq_idx=sq)
        g = oracle.scan_bwd(zeros_u, dn, An, Cn, Cn, _np(dout), **kw)
        f1 = oracle.scan_fwd(zeros_u, dn, An, Cn, Cn, h0=np.ones(g["dh0"].shape), **kw)
        decay, adj = f1["final_state"], g["dh0"]
        cut = self._cut(seq, seq_prev)
        if cut is not None:
            decay[cut] = 0.0
            adj[cut] = 0.0
        return _t(decay), _t(adj)

    def state_carry(self, decay, value, r, reverse, init, seq_prev, seq):
        dec, val = _np(decay), _np(value)
        h = np.zeros(dec.shape[1:]) if init is None else _np(init).copy()
        R = dec.shape[0]
        order = range(R - 1, r, -1) if reverse else range(r)
        for j in order:
            h = dec[j] * h + val[j]
        if not reverse:
            cut = self._cut(seq, seq_prev)
            if cut is not None:
                h[cut] = 0.0
        return _t(h)

    def scan_forward(self, u, delta, A, Bm, Cm, z, Dskip, delta_bias, softplus, seq, h0,
                     zoh=False):
        f = oracle.scan_fwd(_np(u), _np(delta), _np(A), _np(Bm), _np(Cm), z=_np(z),
                            Dskip=_np(Dskip), delta_bias=_np(delta_bias), softplus=softplus,
                            seq_idx=_np(seq, np.int32), h0=_np(h0), zoh=zoh)
        return _t(f["out"]), _t(f["final_state"]), None

    def scan_backward(self, u, delta, A, Bm, Cm, dout, ws, z, Dskip, delta_bias, softplus, seq,
                      h0, dfinal, zoh=False):
        g = oracle.scan_bwd(_np(u), _np(delta), _np(A), _np(Bm), _np(Cm), _np(dout), z=_np(z),
                            Dskip=_np(Dskip), delta_bias=_np(delta_bias), softplus=softplus,
                            seq_idx=_np(seq, np.int32), h0=_np(h0), dhL=_np(dfinal), zoh=zoh)
        names = {"du": "du", "ddelta": "ddelta", "dz": "dz", "dA": "dA", "dB": "dB", "dC": "dC",
                 "dD": "dD", "ddelta_bias": "ddelta_bias", "dinitial_state": "dh0"}
        return {k: _t(g[v]) for k, v in names.items()}


class ThreadHub:
    def __init__(self, world):
        self.world = world
        self.barrier = threading.Barrier(world, timeout=120)
        self.slots = [None] * world


class ThreadComm:
    def __init__(self, rank, hub):
        self.rank, self.world, self.hub = rank, hub.world, hub

    def _exchange(self, t):
        h = self.hub
        h.slots[self.rank] = t
        h.barrier.wait()
        got = list(h.slots)
        h.barrier.wait()
        return got

    def shift(self, t, step):
        got = self._exchange(t.contiguous())
        src = self.rank - step
        return got[src].clone() if 0 <= src < self.world else None

    def all_gather(self, t):
        import torch
        return torch.stack([g.contiguous() for g in self._exchange(t.contiguous())])

    def all_reduce_(self, t):
        got = self._exchange(t.clone())
        acc = got[0].clone()
        for g in got[1:]:
            acc += g
        t.copy_(acc)
        return t


def run_threads(world, fn):
    """Run fn(rank, comm) on `world` threads; return the per-rank results."""
    hub = ThreadHub(world)
    res, err = [None] * world, []

    def body(r):
        try:
            res[r] = fn(r, ThreadComm(r, hub))
        except BaseException as e:  # noqa: BLE001 - reported below
            err.append(e)
            hub.barrier.abort()

    th = [threading.Thread(target=body, args=(r,)) for r in range(world)]
    for t in th:
        t.start()
    for t in th:
        t.join()
    if err:
        raise err[0]
    return res


def full_problem(B, D, N, L, seed, seq_bounds=None):
    """Seeded fp64 inputs of a whole sequence (values as in `synth`); document
    starts at the positions in `seq_bounds` (None: no document ids; () : ids
    all 0)."""
    rng = np.random.Generator(np.random.PCG64(seed))
    p = dict(
        x=rng.standard_normal((B, D, L)), z=rng.standard_normal((B, D, L)),
        delta=0.5 * rng.standard_normal((B, D, L)), Bm=rng.standard_normal((B, N, L)),
        Cm=rng.standard_normal((B, N, L)), dout=rng.standard_normal((B, D, L)),
        A=-np.tile(np.arange(1, N + 1, dtype=np.float64), (D, 1)),
        Dskip=rng.uniform(0.5, 1.5, size=D),
        delta_bias=np.log(np.expm1(rng.uniform(1e-3, 1e-1, size=D))),
        conv_w=rng.uniform(-0.5, 0.5, size=(D, 4)), conv_b=rng.uniform(-0.2, 0.2, size=D),
        h0=0.5 * rng.standard_normal((B, D, N)), dhL=rng.standard_normal((B, D, N)),
    )
    seq = None
    if seq_bounds is not None:
        seq = np.zeros((B, L), dtype=np.int32)
        for b in range(B):
            for s in seq_bounds:
                seq[b, s + b:] += 1   # the rows' boundaries differ by one token
    p["seq_idx"] = seq
    return p


def full_reference(p, bf16_points=False, zoh=False):
    """Unsharded oracle: conv -> scan (from h0) -> scan backward (with dhL)
    -> conv backward. With `bf16_points`, u and du are rounded to bf16 where
    bf16 storage rounds them between the stages."""
    seq = p["seq_idx"]
    _, u = oracle.conv1d_fwd(p["x"], p["conv_w"], p["conv_b"], seq)
    if bf16_points:
        u = oracle.round_bf16(u)
    kw = dict(z=p["z"], Dskip=p["Dskip"], delta_bias=p["delta_bias"], seq_idx=seq, h0=p["h0"],
              zoh=zoh)
    f = oracle.scan_fwd(u, p["delta"], p["A"], p["Bm"], p["Cm"], **kw)
    g = oracle.scan_bwd(u, p["delta"], p["A"], p["Bm"], p["Cm"], p["dout"], dhL=p["dhL"], **kw)
    du = oracle.round_bf16(g["du"]) if bf16_points else g["du"]
    dx, dw, db = oracle.conv1d_bwd(p["x"], p["conv_w"], p["conv_b"], seq, du)
    r = dict(u=u, out=f["out"], final_state=f["final_state"], dx=dx, dconv_w=dw, dconv_b=db)
    r.update(du=g["du"], ddelta=g["ddelta"], dz=g["dz"], dA=g["dA"], dB=g["dB"], dC=g["dC"],
             dD=g["dD"], ddelta_bias=g["ddelta_bias"], dinitial_state=g["dh0"])
    return r


SHARDED = ("out", "du", "ddelta", "dz", "dx")   # [B, D, Ls] per rank
SHARDED_BC = ("dB", "dC")                        # [B, N, Ls] per rank
REDUCED = ("dA", "dD", "ddelta_bias", "dconv_w", "dconv_b")


def shard(p, R, r):
    """Rank r's piece of the inputs: contiguous, lengths differing by at most 1."""
    L = p["x"].shape[-1]
    bounds = [L * i // R for i in range(R + 1)]
    lo, hi = bounds[r], bounds[r + 1]
    s = {k: (v[..., lo:hi] if k in ("x", "z", "delta", "Bm", "Cm", "dout", "seq_idx") and v is not None
             else v) for k, v in p.items()}
    return s, lo, hi
