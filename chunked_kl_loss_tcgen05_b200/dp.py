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
                        teacher=0, group=None, compute=None, workspace=None, n_slices=4,
                        out=None, dw_rows=0):
    """Full-batch loss and dW (identical on every rank) and the dH rows of this
    rank's shard.

    With the library's fused call (``compute`` None, CUDA tensors) the last dW
    GEMM runs in ``n_slices`` vocabulary slices and each finished slice of dW
    is all-reduced on a side stream while the next slice is computed, so only
    the last slice's all-reduce follows the GEMM.  ``compute`` replaces the
    fused call (host-logic tests): it receives ``n_valid_total`` (the global
    N_v) and returns (loss[1], dH, dW, slices) with slices a list of (row0,
    row1, event or None) covering dW's rows in order.  ``out`` (loss, dH, dW)
    and ``dw_rows`` are passed to the fused call."""
    if compute is None:
        from .torch_api import fused_kl_fwd_bwd_sliced

        def compute(h, w, i, l, m, **kw):
            return fused_kl_fwd_bwd_sliced(h, w, i, l, m, workspace=workspace,
                                           n_slices=n_slices, out=out, dw_rows=dw_rows, **kw)
    dev = hidden.device
    local = (row_mask != 0).sum() if row_mask is not None else torch.tensor(hidden.shape[0])
    count = local.to(device=dev, dtype=torch.int64).reshape(1)
    dist.all_reduce(count, group=group)
    n_total = int(count.item())
    loss, dH, dW, slices = compute(hidden, W, topk_idx, topk_logit, row_mask, T=T, chunk=chunk,
                                   teacher=teacher, n_valid_total=n_total)
    _all_reduce_slices(dW, slices, group)
    dist.all_reduce(loss, group=group)
    return loss, dH, dW


def _all_reduce_slices(dW, slices, group):
    """All-reduce dW slice by slice as each slice becomes final."""
    rows = [0]
    for r0, r1, _ in slices:
        if r0 != rows[-1] or r1 < r0:
            raise ValueError("dW slices must cover the rows in order")
        rows.append(r1)
    if rows[-1] != dW.shape[0]:
        raise ValueError("dW slices must cover every row")
    if not dW.is_cuda:
        for r0, r1, _ in slices:
            if r1 > r0:
                dist.all_reduce(dW[r0:r1], group=group)
        return
    main = torch.cuda.current_stream(dW.device)
    side = _side_stream(dW.device)
    works = []
    for r0, r1, ev in slices:
        if r1 <= r0:
            continue
        if ev is not None:
            side.wait_event(ev)
        else:
            side.wait_stream(main)
        with torch.cuda.stream(side):
            works.append(dist.all_reduce(dW[r0:r1], group=group, async_op=True))
    for w in works:
        w.wait()  # the current stream waits for the collective
    main.wait_stream(side)


_SIDE = {}


def _side_stream(device):
    key = torch.device(device).index
    if key not in _SIDE:
        _SIDE[key] = torch.cuda.Stream(device)
    return _SIDE[key]
