"""The context-parallel driver on CPU: its exchange logic with the per-shard
steps computed by the fp64 oracle, against the unsharded oracle. Ranks run
as threads of this process and as gloo processes (world size 2 and 3). The
shards cut through documents, put a document start exactly at a shard start
and within the conv halo of one, and carry an initial state and a
final-state gradient across every boundary."""
import datetime
import os
import socket

import numpy as np
import pytest

from cp_support import (REDUCED, SHARDED, SHARDED_BC, OracleOps, full_problem, full_reference,
                        run_threads, shard)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_run(p, R, r, comm, zoh=False):
    import torch
    from selective_state_space_35_b200.cp import ContextParallelLayer
    s, lo, hi = shard(p, R, r)
    T = lambda a: None if a is None else torch.from_numpy(np.ascontiguousarray(a))  # noqa: E731
    layer = ContextParallelLayer(comm, ops=OracleOps(), zoh=zoh)
    out, fs, ctx = layer.forward(T(s["x"]), T(s["delta"]), T(s["z"]), T(s["Bm"]), T(s["Cm"]),
                                 T(s["A"]), T(s["Dskip"]), T(s["delta_bias"]), T(s["conv_w"]),
                                 T(s["conv_b"]), seq_idx=T(s["seq_idx"]), initial_state=T(s["h0"]))
    g = layer.backward(ctx, T(s["dout"]), dfinal_state=T(s["dhL"]))
    res = {k: (v.numpy() if v is not None else None) for k, v in g.items()}
    res["out"] = out.numpy()
    res["final_state"] = fs.numpy()
    return res, lo, hi


def _check(p, R, results, tol=1e-10, zoh=False):
    want = full_reference(p, zoh=zoh)
    for r, (res, lo, hi) in enumerate(results):
        for k in SHARDED + SHARDED_BC:
            np.testing.assert_allclose(res[k], want[k][..., lo:hi], rtol=tol, atol=tol,
                                       err_msg=f"rank {r} {k}")
        for k in REDUCED:
            np.testing.assert_allclose(res[k], want[k], rtol=tol, atol=tol,
                                       err_msg=f"rank {r} {k}")
    np.testing.assert_allclose(results[-1][0]["final_state"], want["final_state"], rtol=tol,
                               atol=tol)
    np.testing.assert_allclose(results[0][0]["dinitial_state"], want["dinitial_state"], rtol=tol,
                               atol=tol)
    assert all(res["dinitial_state"] is None for res, _, _ in results[1:])


# boundaries: one at a shard start (L=60, R=3 -> 20, 40), one two tokens
# after a shard start (inside the conv halo), one mid-shard
_CASES = [(2, 60, (20, 42, 7)), (3, 60, (20, 42, 7)), (4, 61, (15, 30, 47)), (2, 40, None),
          (3, 45, ()),
          (1, 30, (11,)),          # one rank: every exchange is empty
          (3, 9, (3, 5)),          # shards of 3 tokens, the conv halo's length
          (4, 13, (3, 4, 9))]      # ragged shards of 3 and 4 tokens


@pytest.mark.parametrize("R,L,bounds", _CASES)
def test_cp_threads_equal_unsharded(R, L, bounds):
    p = full_problem(2, 3, 4, L, seed=500 + R + L, seq_bounds=bounds)
    results = run_threads(R, lambda r, comm: _rank_run(p, R, r, comm))
    _check(p, R, results)


def test_cp_threads_zero_order_hold():
    p = full_problem(2, 3, 4, 50, seed=560, seq_bounds=(25, 17))
    results = run_threads(2, lambda r, comm: _rank_run(p, 2, r, comm, zoh=True))
    _check(p, 2, results, zoh=True)


def _gloo_worker(rank, world, port, L, bounds, q):
    import torch.distributed as dist
    from selective_state_space_35_b200.cp import TorchComm
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        p = full_problem(2, 3, 4, L, seed=700 + world + L, seq_bounds=bounds)
        res = _rank_run(p, world, rank, TorchComm())
        q.put((rank, res))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,L,bounds", [(2, 48, (24, 26, 9)), (3, 60, (20, 41, 33))])
def test_cp_gloo_processes_equal_unsharded(world, L, bounds):
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.SimpleQueue()
    port = _free_port()
    procs = [ctx.Process(target=_gloo_worker, args=(r, world, port, L, bounds, q))
             for r in range(world)]
    for pr in procs:
        pr.start()
    got = {}
    for _ in range(world):
        r, res = q.get()
        got[r] = res
    for pr in procs:
        pr.join(timeout=120)
        assert pr.exitcode == 0
    p = full_problem(2, 3, 4, L, seed=700 + world + L, seq_bounds=bounds)
    _check(p, world, [got[r] for r in range(world)])


def test_cp_rejects_shards_shorter_than_the_halo():
    p = full_problem(1, 2, 4, 5, seed=570)
    with pytest.raises(ValueError, match="halo"):
        run_threads(2, lambda r, comm: _rank_run(p, 2, r, comm))
