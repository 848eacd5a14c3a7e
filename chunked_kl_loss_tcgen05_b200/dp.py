"""Row-sharded data parallelism over torch.distributed.

Rows are independent except for three sums (see the per-row form of the loss):
the valid-row count N_v, the loss sum, and dW = sum over rows of dlogits^T h.
So each rank passes its own shard of rows (hidden, teacher cache, mask) and the
replicated W; the ranks all-reduce N_v first, each computes its rows with the
global N_v (loss contribution, final dH of its rows, partial dW) in one fused
call, and the partial dW and loss are all-reduced.  Works with any
torch.distributed backend (NCCL for GPUs; the host logic is tested with gloo).
"""
from __future__ import annotations

import torch
import torch.distributed as dist

__all__ = ["shard_rows", "fused_kl_fwd_bwd_dp"]


def shard_rows(N: int, rank: int, world: int) -> tuple:
    """Contiguous row range [lo, hi) of `rank` among `world` ranks."""
    return rank * N // world, (rank + 1) * N // world


def fused_kl_fwd_bwd_dp(hidden, W, topk_idx, topk_logit, row_mask=None, T=1.0, chunk=0,
                        teacher=0, group=None, compute=None, workspace=None):
    """Full-batch loss and dW (identical on every rank) and the dH rows of this
    rank's shard.  ``compute`` defaults to the library's fused call; it receives
    ``n_valid_total`` (the global N_v) and returns (loss[1], row_loss, dH, dW)."""
    if compute is None:
        from .torch_api import fused_kl_fwd_bwd

        def compute(h, w, i, l, m, **kw):
            return fused_kl_fwd_bwd(h, w, i, l, m, workspace=workspace, **kw)
    dev = hidden.device
    local = (row_mask != 0).sum() if row_mask is not None else torch.tensor(hidden.shape[0])
    count = local.to(device=dev, dtype=torch.int64).reshape(1)
    dist.all_reduce(count, group=group)
    n_total = int(count.item())
    loss, _, dH, dW = compute(hidden, W, topk_idx, topk_logit, row_mask, T=T, chunk=chunk,
                              teacher=teacher, n_valid_total=n_total)
    dist.all_reduce(dW, group=group)
    dist.all_reduce(loss, group=group)
    return loss, dH, dW
