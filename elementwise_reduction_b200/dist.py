"""Row-sharded DyT across ranks: the one exchange the method needs.

Rows are independent, so a batch of rows splits across ranks with no
communication in the forward or in dx. The parameter gradients are sums over
ALL rows (dgamma[j] = sum_i dy t, dbeta[j] = sum_i dy, dalpha = sum_ij ...),
so ranks that each ran the backward on their own rows add their partial
gradients with one all-reduce of 2N + 1 values per step. This module is that
exchange (torch.distributed: NCCL between GPUs, gloo on CPU); the sums are in
binary32.
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
