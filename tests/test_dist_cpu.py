"""The row-sharded path on two CPU ranks (gloo): each rank runs the backward on its
own rows (here the oracle stands in for the device kernels), the parameter
gradients are summed with the one all-reduce the method needs, and the result
must equal the backward over all rows."""
import datetime
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


# ---- the fused cross-rank sum: its protocol on CPU ranks ----------------------------------------
#
# FusedGradientSum drives the device through an `ops` object. Here the ops are
# the oracle: stage 1 leaves the shard's binary64 column sums (one partial row
# per rank) in a numpy buffer, the barrier is a gloo all-reduce, and the
# finalize's peer loads are a gloo gather of every rank's buffer of that call,
# summed in rank order like the kernel does. This checks the protocol: layouts
# and handles exchanged once, buffers rotated so no consecutive calls share
# one, every rank adding the ranks' totals in rank order with one rounding.


class _OracleOps:
    def __init__(self, rank, N):
        self.rank, self.N, self.used, self.closed = rank, N, [], []

    def layout(self, x, dy, dx, N):
        return {"bytes": 8 * (2 * N + 1), "off_dgamma": 0, "off_dbeta": 8 * N, "off_dalpha": 16 * N, "rows": 1,
                "dalpha_parts": 1}

    def workspace(self, x, gamma):
        return np.zeros(2 * self.N + 1)

    def pointer(self, buf):
        return ("own", self.rank, id(buf))

    def export(self, buf):
        return (self.rank, id(buf))

    def import_(self, handle):
        return ("peer",) + tuple(handle)

    def close(self, ptr, handle):
        self.closed.append(handle)

    def partials(self, x, dy, alpha, gamma, dx, buf, stream):
        import oracle
        M = x.size // self.N
        r = oracle.backward(x, dy, alpha, gamma, M, self.N, "f32", "f32", want_dx=False)
        buf[:self.N], buf[self.N:2 * self.N], buf[2 * self.N] = r["dgamma"], r["dbeta"], r["dalpha"]
        self.used.append(next(i for i, b in enumerate(self.fgs.buffers) if b is buf))
        return self.layout(x, dy, dx, self.N)

    def barrier(self, group, stream):
        dist.all_reduce(torch.zeros(1), group=group)

    def finalize(self, ptrs, layouts, alpha, gamma, beta, dgamma, dbeta, dalpha, stream):
        mine = next(b for b in self.fgs.buffers if ("own", self.rank, id(b)) == ptrs[self.rank])
        every = [torch.zeros(2 * self.N + 1, dtype=torch.float64) for _ in ptrs]
        dist.all_gather(every, torch.from_numpy(mine.copy()))  # stands in for the peer loads
        total = every[0].clone()
        for t in every[1:]:
            total += t  # the ranks' totals in rank order, binary64
        dgamma.copy_(total[:self.N]), dbeta.copy_(total[self.N:2 * self.N]), dalpha.copy_(total[2 * self.N:])


def _fused_rank(rank: int, port: int, world: int, M: int, N: int, calls: int, q):
    from elementwise_reduction_b200.dist import FusedGradientSum
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        inp = _inputs(M, N)
        b, e = shard_rows(M, world, rank)
        x, dy = inp["x"][b * N:e * N], inp["dy"][b * N:e * N]
        ops = _OracleOps(rank, N)
        fgs = FusedGradientSum.__new__(FusedGradientSum)
        ops.fgs = fgs
        gamma = torch.from_numpy(inp["gamma"])
        fgs.__init__(x, dy, None, gamma, ops=ops)
        outs = []
        for _ in range(calls):
            dg, db, da = torch.empty(N), torch.empty(N), torch.empty(1)
            fgs(x, dy, inp["alpha"], inp["gamma"], None, None, dg, db, da)
            outs.append((dg.numpy().copy(), db.numpy().copy(), float(da.item())))
        fgs.close()
        q.put((rank, outs, ops.used, len(ops.closed)))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,M", [(2, 1001), (3, 1000), (4, 7)])
def test_fused_sum_protocol_on_gloo_ranks(world, M):
    import oracle
    N, calls = 24, 4
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_fused_rank, args=(r, port, world, M, N, calls, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = sorted([q.get(timeout=180) for _ in range(world)])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    inp = _inputs(M, N)
    # the ranks' totals, each the oracle's binary64 sum over that rank's rows,
    # added in rank order and rounded once to binary32
    totals = []
    for r in range(world):
        b, e = shard_rows(M, world, r)
        t = oracle.backward(inp["x"][b * N:e * N], inp["dy"][b * N:e * N], inp["alpha"], inp["gamma"], e - b, N,
                            "f32", "f32", want_dx=False)
        totals.append(np.concatenate([t["dgamma"], t["dbeta"], [t["dalpha"]]]))
    want = totals[0].copy()
    for t in totals[1:]:
        want += t
    want32 = want.astype(np.float32)
    full = oracle.backward(inp["x"], inp["dy"], inp["alpha"], inp["gamma"], M, N, "f32", "f32", want_dx=False)
    for rank, outs, used, closed in got:
        assert used == [0, 1, 2, 0][:calls]          # three buffers in rotation
        assert closed == 3 * (world - 1)             # every imported peer buffer released
        for dg, db, da in outs:                      # same bits on every rank and call
            assert np.array_equal(dg, want32[:N]) and np.array_equal(db, want32[N:2 * N])
            assert da == float(want32[2 * N])
            assert np.all(np.abs(db - full["dbeta"]) <= 2e-6 + 1e-5 * np.abs(full["dbeta"]))
            assert abs(da - full["dalpha"]) <= 1e-5 * full["mag_dalpha"]


class _FailingOps(_OracleOps):
    """_OracleOps whose rank `bad` fails to export (or, with on_import, to import)."""

    def __init__(self, rank, N, bad, on_import):
        super().__init__(rank, N)
        self.bad, self.on_import = bad, on_import

    def export(self, buf):
        if self.rank == self.bad and not self.on_import:
            raise RuntimeError("cannot share this memory")
        return super().export(buf)

    def import_(self, handle):
        if self.rank == self.bad and self.on_import and handle[0] != 0:
            raise RuntimeError("cannot map that peer")
        return super().import_(handle)


def _failing_rank(rank: int, port: int, world: int, bad: int, on_import: bool, q):
    from elementwise_reduction_b200.dist import FusedGradientSum
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        N = 8
        ops = _FailingOps(rank, N, bad, on_import)
        fgs = FusedGradientSum.__new__(FusedGradientSum)
        ops.fgs = fgs
        fgs.__init__(np.zeros(4 * N, dtype=np.float32), None, None, torch.zeros(N), ops=ops)
        # what the bench does next: one collective over every rank's verdict
        ok = torch.tensor([1 if fgs.error is None else 0])
        dist.all_reduce(ok, op=dist.ReduceOp.MIN)
        fgs.close()
        q.put((rank, fgs.error, int(ok.item()), len(fgs._imported)))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("on_import", [False, True])
def test_fused_sum_records_a_failing_rank(on_import):
    # A rank that cannot export (or import) its workspaces records the failure
    # instead of raising between two collectives: every rank finishes the
    # construction, and the ranks agree to fall back.
    world, bad = 3, 1
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_failing_rank, args=(r, port, world, bad, on_import, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = sorted([q.get(timeout=180) for _ in range(world)])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, error, ok, imported in got:
        assert ok == 0 and imported == 0                   # all fall back; imported peers released
        if rank == bad:
            assert "cannot" in error
        elif not on_import:
            assert error == "another rank could not export its workspaces"
        else:
            assert error is None                           # only the bad rank failed to map


def test_replay_schedule_never_reuses_a_buffer_back_to_back():
    from elementwise_reduction_b200.dist import FusedGradientSum
    for k in range(2, 40):
        s = FusedGradientSum.schedule(k)
        assert len(s) == k and set(s) <= {0, 1, 2}
        cyc = s + s  # two replays back to back
        assert all(cyc[i] != cyc[i + 1] for i in range(len(cyc) - 1)), (k, s)
    with pytest.raises(ValueError):
        FusedGradientSum.schedule(1)
