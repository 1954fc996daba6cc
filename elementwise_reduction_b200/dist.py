"""Row-sharded DyT across ranks: the one exchange the method needs.

Rows are independent, so a batch of rows splits across ranks with no
communication in the forward or in dx. The parameter gradients are sums over
ALL rows (dgamma[j] = sum_i dy t, dbeta[j] = sum_i dy, dalpha = sum_ij ...), so
ranks that each ran the backward on their own rows must add their partial sums
once. Two ways to do it:

- FusedGradientSum: each rank runs stage 1 of the backward on its rows, which
  leaves binary64 partial sums in one of its workspaces; a one-element NCCL
  all-reduce on the stream serves as the barrier; then every rank's finalize
  reads ALL ranks' partials through peer pointers (CUDA IPC, plain loads over
  NVLink) in rank order and rounds each gradient once. The exchange is the
  finalize itself: no second rounding, and every rank gets the same bits.
- allreduce_param_grads: the rounded gradients of each rank summed with one
  all-reduce of 2N + 1 binary32 values, for where GPU memory cannot be shared
  between the processes.
"""
from __future__ import annotations

import torch
import torch.distributed as dist


def shard_rows(M: int, world: int, rank: int) -> tuple[int, int]:
    """Rows [begin, end) of `rank` when M rows are split into `world` balanced shards."""
    if world < 1 or not 0 <= rank < world or M < 0:
        raise ValueError("bad shard request")
    q, r = divmod(M, world)
    begin = rank * q + min(rank, r)
    return begin, begin + q + (1 if rank < r else 0)


def pack_param_grads(dgamma: torch.Tensor, dbeta: torch.Tensor, dalpha: torch.Tensor,
                     buf: torch.Tensor | None = None) -> torch.Tensor:
    """[dgamma | dbeta | dalpha] as one binary32 vector of 2N + 1 values."""
    N = dgamma.numel()
    if buf is None:
        buf = torch.empty(2 * N + 1, dtype=torch.float32, device=dgamma.device)
    buf[:N].copy_(dgamma.reshape(-1))
    buf[N:2 * N].copy_(dbeta.reshape(-1))
    buf[2 * N:].copy_(dalpha.reshape(-1))
    return buf


def unpack_param_grads(buf: torch.Tensor, dgamma: torch.Tensor, dbeta: torch.Tensor,
                       dalpha: torch.Tensor) -> None:
    N = dgamma.numel()
    dgamma.reshape(-1).copy_(buf[:N])
    dbeta.reshape(-1).copy_(buf[N:2 * N])
    dalpha.reshape(-1).copy_(buf[2 * N:])


def allreduce_param_grads(dgamma: torch.Tensor, dbeta: torch.Tensor, dalpha: torch.Tensor,
                          group=None, buf: torch.Tensor | None = None) -> None:
    """Sum the rank-local parameter gradients over all ranks, in place (one all-reduce)."""
    buf = pack_param_grads(dgamma, dbeta, dalpha, buf)
    dist.all_reduce(buf, op=dist.ReduceOp.SUM, group=group)
    unpack_param_grads(buf, dgamma, dbeta, dalpha)


class DeviceOps:
    """What FusedGradientSum does on the device: the library's stage 1 and
    finalize, its CUDA IPC helpers, and a one-element NCCL all-reduce as the
    barrier between them."""

    def __init__(self, device):
        self.device = torch.device(device)
        self._flag = torch.zeros(1, dtype=torch.float32, device=self.device)

    def layout(self, x, dy, dx, N: int) -> dict:
        from . import partials_layout
        return partials_layout(x, dy, dx, N)

    def workspace(self, x, gamma):
        from . import workspace
        return workspace(x, gamma)

    def pointer(self, buf) -> int:
        return buf.data_ptr()

    def export(self, buf) -> bytes:
        from . import dyt_ipc_export
        with torch.cuda.device(self.device):
            return dyt_ipc_export(buf.data_ptr())

    def import_(self, handle: bytes) -> int:
        from . import dyt_ipc_import
        with torch.cuda.device(self.device):
            return dyt_ipc_import(handle)

    def close(self, ptr: int, handle: bytes) -> None:
        from . import dyt_ipc_close
        with torch.cuda.device(self.device):
            dyt_ipc_close(ptr, handle)

    def partials(self, x, dy, alpha, gamma, dx, buf, stream) -> dict:
        from . import backward_partials
        return backward_partials(x, dy, alpha, gamma, buf, dx=dx, stream=stream)[1]

    def barrier(self, group, stream) -> None:
        # NCCL runs the all-reduce after this rank's queued work and lets the
        # stream continue only once every rank has joined: on every rank, what
        # follows runs after every rank's stage 1.
        if stream is None:
            dist.all_reduce(self._flag, group=group)
        else:
            with torch.cuda.stream(stream):
                dist.all_reduce(self._flag, group=group)

    def finalize(self, ptrs, layouts, alpha, gamma, beta, dgamma, dbeta, dalpha, stream) -> None:
        from . import finalize_partials
        finalize_partials(ptrs, layouts, alpha, gamma, beta, dgamma, dbeta, dalpha, stream=stream)


class FusedGradientSum:
    """The backward of a row-sharded DyT whose cross-rank gradient sum is the finalize.

    Built once per process group and tensor layout (every rank passes its own
    row shard; N and the dtypes agree). Each call: stage 1 on this rank's rows
    into one of three workspaces, a barrier, then a finalize that reads the same
    workspace of every rank (peer pointers) in rank order. A workspace is never
    used by two consecutive calls: a rank can only overwrite it after every rank
    has passed the next call's barrier, which each reaches only after finishing
    the finalize that read it. Workspaces rotate by call; a caller that replays a
    captured sequence passes `buffer=` itself, keeping consecutive calls (across
    the end of one replay and the start of the next, too) on different buffers.
    """

    NBUF = 3

    def __init__(self, x, dy, dx, gamma, group=None, ops=None):
        self.group = group
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        from . import MAX_RANKS
        if self.world > MAX_RANKS:  # the same on every rank, before any collective
            raise ValueError(f"at most {MAX_RANKS} ranks")
        self.ops = ops if ops is not None else DeviceOps(x.device)
        self.N = gamma.numel()
        # Why this rank cannot take part (None: it can). Every rank runs the same
        # collectives whatever fails locally, so a failure is recorded, not
        # raised between two collectives; callers agree on `error` (one
        # collective over all ranks) before the first call.
        self.error = None
        self.buffers, self._imported, self.ptrs, self.calls = [], [], [], 0
        mine, handles = None, None
        try:
            mine = self.ops.layout(x, dy, dx, self.N)
            self.buffers = [self.ops.workspace(x, gamma) for _ in range(self.NBUF)]
            handles = [self.ops.export(b) for b in self.buffers]
        except Exception as e:  # e.g. memory that CUDA IPC cannot share
            self.error = f"{type(e).__name__}: {e}"
            mine, handles = None, None
        self.layouts = [None] * self.world
        dist.all_gather_object(self.layouts, mine, group=group)
        everyone = [None] * self.world
        dist.all_gather_object(everyone, handles, group=group)
        if self.error is None and any(h is None for h in everyone):
            self.error = "another rank could not export its workspaces"
        if self.error is None:
            try:
                for b in range(self.NBUF):
                    row = []
                    for r in range(self.world):
                        if r == self.rank:
                            row.append(self.ops.pointer(self.buffers[b]))
                        else:
                            p = self.ops.import_(everyone[r][b])
                            self._imported.append((p, everyone[r][b]))
                            row.append(p)
                    self.ptrs.append(row)
            except Exception as e:
                self.error = f"{type(e).__name__}: {e}"
                self.close()
                self.ptrs = []

    def __call__(self, x, dy, alpha, gamma, beta, dx, dgamma, dbeta, dalpha, stream=None, buffer=None):
        if self.error is not None:
            raise RuntimeError(f"the fused gradient sum cannot run on this rank: {self.error}")
        b = self.calls % self.NBUF if buffer is None else buffer
        layout = self.ops.partials(x, dy, alpha, gamma, dx, self.buffers[b], stream)
        if layout != self.layouts[self.rank]:
            raise ValueError("the tensors' layout changed since the ranks exchanged their partials' layouts")
        self.ops.barrier(self.group, stream)
        self.ops.finalize(self.ptrs[b], self.layouts, alpha, gamma, beta, dgamma, dbeta, dalpha, stream)
        self.calls += 1
        return b

    @staticmethod
    def schedule(k: int) -> list[int]:
        """Buffers for k calls replayed back to back: no two consecutive calls, the
        last of one replay and the first of the next included, share a buffer."""
        if k == 1:
            raise ValueError("a replayed single call would reuse its buffer; capture at least two calls")
        s = [i % FusedGradientSum.NBUF for i in range(k)]
        if k >= 2 and s[-1] == s[0]:
            s[-1] = next(b for b in range(FusedGradientSum.NBUF) if b not in (s[-2], s[0]))
        return s

    def close(self) -> None:
        for p, h in self._imported:
            self.ops.close(p, h)
        self._imported = []
