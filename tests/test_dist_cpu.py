"""The row-sharded path on two CPU ranks (gloo): each rank runs the backward on its
own rows (here the oracle stands in for the device kernels), the parameter
gradients are summed with the one all-reduce the method needs, and the result
must equal the backward over all rows."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from elementwise_reduction_b200.dist import allreduce_param_grads, shard_rows

WORLD = 2


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _inputs(M, N):
    from synth import workloads
    w = workloads.Workload("dist", M, N, "f32", "f32", alpha=0.8)
    return workloads.make_inputs(w)


def _rank(rank: int, port: int, M: int, N: int, q, world: int = WORLD):
    import oracle
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        inp = _inputs(M, N)
        b, e = shard_rows(M, world, rank)
        r = oracle.backward(inp["x"][b * N:e * N], inp["dy"][b * N:e * N], inp["alpha"], inp["gamma"],
                            e - b, N, "f32", "f32", want_dx=False)
        dg = torch.tensor(r["dgamma"], dtype=torch.float32)
        db = torch.tensor(r["dbeta"], dtype=torch.float32)
        da = torch.tensor([r["dalpha"]], dtype=torch.float32)
        allreduce_param_grads(dg, db, da)
        q.put((rank, dg.numpy(), db.numpy(), float(da.item())))
    finally:
        dist.destroy_process_group()


def test_shard_rows_is_a_balanced_partition():
    for M in (0, 1, 7, 65537):
        for world in (1, 2, 3, 8):
            parts = [shard_rows(M, world, r) for r in range(world)]
            assert parts[0][0] == 0 and parts[-1][1] == M
            assert all(parts[i][1] == parts[i + 1][0] for i in range(world - 1))
            sizes = [e - b for b, e in parts]
            assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        shard_rows(5, 2, 2)


@pytest.mark.parametrize("world,M", [(WORLD, 1001), (3, 1000)])
def test_gloo_ranks_sum_to_the_whole_matrix(world, M):
    import oracle
    N = 24
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, port, M, N, q, world)) for r in range(world)]
    for p in procs:
        p.start()
    got = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    inp = _inputs(M, N)
    full = oracle.backward(inp["x"], inp["dy"], inp["alpha"], inp["gamma"], M, N, "f32", "f32", want_dx=False)
    for rank, dg, db, da in got:  # every rank holds the same sums
        assert np.all(np.abs(dg - full["dgamma"]) <= 2e-6 + 1e-5 * full["mag_dgamma"])
        assert np.all(np.abs(db - full["dbeta"]) <= 2e-6 + 1e-5 * full["mag_dbeta"])
        assert abs(da - full["dalpha"]) <= 1e-5 * full["mag_dalpha"]
    for r in range(1, world):
        assert np.array_equal(got[0][1], got[r][1])


def _single_rank(port: int, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=0, world_size=1)
    try:
        out = []
        for dt in (torch.float32, torch.bfloat16, torch.float16):
            g = torch.linspace(-3, 5, 7).to(dt)
            b = torch.linspace(2, -1, 7).to(dt)
            a = torch.tensor([0.375]).to(dt)
            dg, db, da = g.clone(), b.clone(), a.clone()
            allreduce_param_grads(dg, db, da)  # one rank: the sum is the identity
            out.append((str(dt), torch.equal(dg, g), torch.equal(db, b), torch.equal(da, a),
                        dg.dtype == dt))
        q.put(out)
    finally:
        dist.destroy_process_group()


def test_gradient_exchange_keeps_each_parameter_dtype():
    # The 2N + 1 gradients travel as one binary32 vector; 16-bit parameter
    # gradients come back in their own dtype, unchanged by a one-rank sum.
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    p = ctx.Process(target=_single_rank, args=(_free_port(), q))
    p.start()
    out = q.get(timeout=120)
    p.join(timeout=60)
    assert p.exitcode == 0
    for name, *oks in out:
        assert all(oks), name
