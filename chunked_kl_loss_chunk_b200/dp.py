"""Data-parallel sharding of the fused chunked KL loss along the positions.

The loss is a mean over the T_total positions of a batch and every position's
terms (its logsumexp, its KL, its row of dz and of dH) depend on that position
alone; only dW = dz^T h sums over positions.  So a batch splits along T over
ranks with no exchange inside the loss: each rank runs the fused forward and
backward on its own contiguous block of rows, normalised by the batch's
T_total (``kd_fused_kl_fwd_shard`` / ``kd_fused_kl_bwd_shard``), and then one
all-reduce (sum) of the scalar loss and of dW [V, d] fp32 over the ranks gives
the batch's loss and dW.  dH needs no exchange: each rank holds exactly the
batch gradient's rows of its shard.

The pages run the method on a single GPU; they describe the multi-node
sharding it made unnecessary (goaixin.org, "Breaking the Memory Barrier ...",
section "Detailed Chronology and Technical Evolution"; andresseo.expert,
section "What a Single H200 GPU Can Now Do That Once Required Four Nodes").
This module is the plain data-parallel form of the same loss.

Host logic only: the per-shard work runs in libkd's kernels, the exchange in
``torch.distributed`` (NCCL on GPUs, gloo on CPU).  ``shard_step`` takes the
per-shard computation as an argument so that the partitioning, the
normalisation and the reduction can be exercised on CPU ranks.
"""

from __future__ import annotations

from typing import Callable, NamedTuple

import torch
import torch.distributed as dist


class Shard(NamedTuple):
    row0: int      # first position of this rank's block
    rows: int      # positions in the block (0 when T_total < world)


def shard_rows(T_total: int, world: int, rank: int) -> Shard:
    """Contiguous, balanced split of T_total positions over `world` ranks: the
    first T_total % world ranks get one position more.  Blocks tile
    [0, T_total) in rank order."""
    if T_total < 0 or world < 1 or not (0 <= rank < world):
        raise ValueError("need T_total >= 0, world >= 1 and 0 <= rank < world")
    base, extra = divmod(T_total, world)
    rows = base + (1 if rank < extra else 0)
    row0 = rank * base + min(rank, extra)
    return Shard(row0, rows)


def kd_shard_compute(h, W, t_vals, t_idx, T_total: int, chunk: int, temperature: float = 1.0,
                     cache: str = "logits", tau_squared: bool = False, grad_loss=None):
    """One rank's shard on the GPU: (loss part [] f32, dH [rows, d], dW part
    [V, d] f32), all from libkd's kernels."""
    from chunked_kl_loss_chunk_b200 import kd
    loss, lse, _, ws = kd.fused_kl_fwd(h, W, t_vals, t_idx, chunk, temperature, cache=cache,
                                       tau_squared=tau_squared, T_total=T_total)
    dH, dW, _ = kd.fused_kl_bwd(h, W, t_vals, t_idx, lse, chunk, temperature, grad_loss=grad_loss,
                                ws=ws, cache=cache, tau_squared=tau_squared, T_total=T_total)
    return loss, dH, dW


def shard_step(h, W, t_vals, t_idx, T_total: int, chunk: int, temperature: float = 1.0, *,
               compute: Callable = kd_shard_compute, group=None, dtype=torch.float32, **kw):
    """Loss and gradients of a batch of T_total positions of which this rank
    holds the rows in `h`, `t_vals`, `t_idx` (its ``shard_rows`` block).

    Returns (loss, dH, dW): the batch's loss and dW, identical on every rank
    after the all-reduce, and dH for this rank's rows.  A rank with no rows
    contributes zeros and still joins both collectives, so every rank takes the
    same collective steps in the same order.  `dtype` is the type of the loss
    and dW that `compute` returns (fp32 for libkd)."""
    rows = h.shape[0]
    V, d = W.shape
    if rows > 0:
        loss, dH, dW = compute(h, W, t_vals, t_idx, T_total, chunk, temperature, **kw)
        loss = loss.reshape(1)
    else:
        loss = torch.zeros(1, dtype=dtype, device=W.device)
        dH = torch.empty((0, d), dtype=h.dtype, device=W.device)
        dW = torch.zeros((V, d), dtype=dtype, device=W.device)
    world = dist.get_world_size(group) if dist.is_available() and dist.is_initialized() else 1
    if world > 1:
        dist.all_reduce(dW, op=dist.ReduceOp.SUM, group=group)
        dist.all_reduce(loss, op=dist.ReduceOp.SUM, group=group)
    return loss.reshape(()), dH, dW
