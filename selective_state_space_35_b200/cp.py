"""Context parallelism: the layer core over a sequence cut along L into
contiguous shards, one per rank.

"FLA Mamba and Mamba2" (the Axolotl page, context-parallel paragraph): the
shards are contiguous, neighbouring ranks exchange convolution halos and
recurrent states, and packed-document boundaries stay active across shard
boundaries. The state exchange here uses the affine form of the recurrence
("hung-phan ml-skills mamba", "Hardware-Aware Parallel Scan": pieces compose
with (a1, b1) + (a2, b2) = (a1 a2, a2 b1 + b2)), so no rank waits for the
previous one to finish its scan:

forward, rank r of R (tokens [r Ls, (r+1) Ls) of every row):
  1. the last 3 inputs (and document ids) go to rank r+1: its conv halo;
  2. conv1d + SiLU with the halo from rank r-1 -> u;
  3. the shard's summary (prod a, end state from 0), all-gathered;
  4. the state entering the shard = fold of the earlier summaries (from the
     initial state), then the shard's scan from it.
backward:
  5. the shard's backward summary (gradient leaving its start from its own
     dout), all-gathered; the gradient reaching the shard's final state =
     fold of the later summaries (from the final-state gradient);
  6. the shard's scan backward from it;
  7. the first 3 inputs, their du and ids go to rank r-1: its conv halo;
  8. conv1d backward with both halos;
  9. parameter gradients (A, D, delta bias, conv weight and bias) are summed
     over ranks. dB, dC, du, ddelta, dz and dx stay sharded.

Every step of the compute runs in the library's kernels (`GpuOps`); this
module only orders the calls and the exchanges. The exchanges are a 3-token
halo per neighbour and 2 [B, D, N] fp32 summaries per rank per direction
(0.4 MB each at B 2, D 1536, N 16), plus the all-reduce of the parameter
gradients.
"""
from __future__ import annotations

HALO = 3  # conv width - 1


class TorchComm:
    """Exchanges between the ranks of a torch.distributed process group
    (NCCL for CUDA tensors, gloo for CPU tensors)."""

    def __init__(self, group=None):
        import torch.distributed as dist
        self.dist = dist
        self.group = group
        self.rank = dist.get_rank(group)
        self.world = dist.get_world_size(group)

    def _global(self, r):
        return r if self.group is None else self.dist.get_global_rank(self.group, r)

    def shift(self, t, step):
        """Send `t` to rank + step and return what rank - step sent (None at an
        edge of the rank range)."""
        import torch
        dist = self.dist
        dst, src = self.rank + step, self.rank - step
        ops, recv = [], None
        if 0 <= dst < self.world:
            ops.append(dist.P2POp(dist.isend, t.contiguous(), self._global(dst), self.group))
        if 0 <= src < self.world:
            recv = torch.empty_like(t.contiguous())
            ops.append(dist.P2POp(dist.irecv, recv, self._global(src), self.group))
        if ops:
            for req in dist.batch_isend_irecv(ops):
                req.wait()
        return recv

    def all_gather(self, t):
        """[world, *t.shape]: every rank's `t`, in rank order."""
        import torch
        parts = [torch.empty_like(t.contiguous()) for _ in range(self.world)]
        self.dist.all_gather(parts, t.contiguous(), group=self.group)
        return torch.stack(parts)

    def all_reduce_(self, t):
        self.dist.all_reduce(t, group=self.group)
        return t


class GpuOps:
    """The library's kernels for the per-shard steps (no other compute path)."""

    def __init__(self):
        from . import (conv1d_bwd, conv1d_fwd, scan_bwd, scan_bwd_summary, scan_fwd,
                       scan_fwd_summary, state_carry)
        self.conv1d_fwd, self.conv1d_bwd = conv1d_fwd, conv1d_bwd
        self.scan_fwd, self.scan_bwd = scan_fwd, scan_bwd
        self.fwd_summary, self.bwd_summary = scan_fwd_summary, scan_bwd_summary
        self.carry = state_carry

    def conv_fwd(self, x, w, b, seq, x_prev, seq_prev):
        return self.conv1d_fwd(x, w, b, seq, x_prev=x_prev, seq_prev=seq_prev)

    def conv_bwd(self, x, w, b, seq, du, x_prev, seq_prev, x_next, du_next, seq_next):
        return self.conv1d_bwd(x, w, b, seq, du, x_prev=x_prev, seq_prev=seq_prev, x_next=x_next,
                               du_next=du_next, seq_next=seq_next)

    def scan_fwd_summary(self, u, delta, A, Bm, seq, seq_prev, delta_bias, softplus, zoh):
        return self.fwd_summary(u, delta, A, Bm, delta_bias=delta_bias, softplus=softplus,
                                seq_idx=seq, seq_prev=seq_prev, zoh=zoh)

    def scan_bwd_summary(self, delta, A, Cm, dout, z, seq, seq_prev, delta_bias, softplus):
        return self.bwd_summary(delta, A, Cm, dout, z=z, delta_bias=delta_bias, softplus=softplus,
                                seq_idx=seq, seq_prev=seq_prev)

    def state_carry(self, decay, value, r, reverse, init, seq_prev, seq):
        return self.carry(decay, value, r, reverse=reverse, init=init, seq_prev=seq_prev,
                          seq_idx=seq)

    def scan_forward(self, u, delta, A, Bm, Cm, z, Dskip, delta_bias, softplus, seq, h0, zoh):
        return self.scan_fwd(u, delta, A, Bm, Cm, z=z, Dskip=Dskip, delta_bias=delta_bias,
                             softplus=softplus, seq_idx=seq, return_final_state=True,
                             initial_state=h0, zoh=zoh)

    def scan_backward(self, u, delta, A, Bm, Cm, dout, ws, z, Dskip, delta_bias, softplus, seq,
                      h0, dfinal, zoh):
        return self.scan_bwd(u, delta, A, Bm, Cm, dout, ws, z=z, Dskip=Dskip,
                             delta_bias=delta_bias, softplus=softplus, seq_idx=seq,
                             initial_state=h0, dfinal_state=dfinal, zoh=zoh)


class ContextParallelLayer:
    """conv1d + SiLU -> selective scan (softplus step, D skip, SiLU(z) gate),
    forward and backward, over this rank's shard of the sequence.

    Parameters (A [D, N] real, Dskip, delta_bias [D], conv_w [D, 4], conv_b
    [D]) are replicated; activations are this rank's shard ([B, D, Ls]; B, C
    [B, N, Ls]; seq_idx [B, Ls] int32 or None), Ls >= 3. `zoh` selects the
    zero-order-hold discretisation (the summaries are the same: the carry
    passes through prod a either way).
    """

    def __init__(self, comm, ops=None, softplus=True, zoh=False):
        self.comm = comm
        self.ops = ops if ops is not None else GpuOps()
        self.softplus = softplus
        self.zoh = zoh

    def forward(self, x, delta, z, Bm, Cm, A, Dskip, delta_bias, conv_w, conv_b, seq_idx=None,
                initial_state=None):
        """Returns (out, final_state of this shard, ctx). `initial_state`
        [B, D, N] is the state before the whole sequence (the same on every
        rank, or None)."""
        c, ops = self.comm, self.ops
        if x.shape[-1] < HALO:
            raise ValueError(f"shard length {x.shape[-1]} < {HALO} (the conv halo)")
        x_prev = c.shift(x[..., -HALO:], +1)
        seq_prev3 = c.shift(seq_idx[..., -HALO:], +1) if seq_idx is not None else None
        seq_prev = seq_prev3[:, -1].contiguous() if seq_prev3 is not None else None
        u = ops.conv_fwd(x, conv_w, conv_b, seq_idx, x_prev, seq_prev3)
        decay, end = ops.scan_fwd_summary(u, delta, A, Bm, seq_idx, seq_prev, delta_bias,
                                          self.softplus, self.zoh)
        summ = c.all_gather(_stack2(decay, end))
        decay_all, end_all = summ[:, 0].contiguous(), summ[:, 1].contiguous()
        h_in = ops.state_carry(decay_all, end_all, c.rank, False, initial_state, seq_prev, seq_idx)
        out, fs, ws = ops.scan_forward(u, delta, A, Bm, Cm, z, Dskip, delta_bias, self.softplus,
                                       seq_idx, h_in, self.zoh)
        ctx = dict(x=x, delta=delta, z=z, Bm=Bm, Cm=Cm, A=A, Dskip=Dskip, delta_bias=delta_bias,
                   conv_w=conv_w, conv_b=conv_b, seq_idx=seq_idx, u=u, ws=ws, h_in=h_in,
                   x_prev=x_prev, seq_prev3=seq_prev3, seq_prev=seq_prev, decay_all=decay_all)
        return out, fs, ctx

    def backward(self, ctx, dout, dfinal_state=None):
        """Gradients of this shard (dx, du, ddelta, dz, dB, dC) and of the
        parameters summed over ranks (dA, dD, ddelta_bias, dconv_w, dconv_b),
        plus dinitial_state on rank 0 (w.r.t. the sequence's initial state).
        `dfinal_state`: gradient of the sequence's final state (the last
        rank's), the same tensor on every rank, or None."""
        c, ops, k = self.comm, self.ops, ctx
        seq = k["seq_idx"]
        _, adj = ops.scan_bwd_summary(k["delta"], k["A"], k["Cm"], dout, k["z"], seq,
                                      k["seq_prev"], k["delta_bias"], self.softplus)
        adj_all = c.all_gather(adj)
        dfin = ops.state_carry(k["decay_all"], adj_all, c.rank, True, dfinal_state, None, None)
        g = ops.scan_backward(k["u"], k["delta"], k["A"], k["Bm"], k["Cm"], dout, k["ws"], k["z"],
                              k["Dskip"], k["delta_bias"], self.softplus, seq, k["h_in"], dfin,
                              self.zoh)
        x_next = c.shift(k["x"][..., :HALO], -1)
        du_next = c.shift(g["du"][..., :HALO], -1)
        seq_next = c.shift(seq[..., :HALO], -1) if seq is not None else None
        dx, dw, dcb = ops.conv_bwd(k["x"], k["conv_w"], k["conv_b"], seq, g["du"], k["x_prev"],
                                   k["seq_prev3"], x_next, du_next, seq_next)
        for t in (g["dA"], g["dD"], g["ddelta_bias"], dw, dcb):
            c.all_reduce_(t)
        res = dict(g)
        res.update(dx=dx, dconv_w=dw, dconv_b=dcb)
        if c.rank != 0:
            res["dinitial_state"] = None
        return res


def _stack2(a, b):
    import torch
    return torch.stack([a, b])
