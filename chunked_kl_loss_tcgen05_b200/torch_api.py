"""Tensor-level helpers over the C ABI (PyTorch supplies memory and streams only).

``fused_kl_fwd_bwd`` / ``fused_kl_fwd`` allocate outputs and the workspace
with PyTorch on the inputs' device and call the library on the current
stream.  ``FusedChunkedKL`` is an autograd Function that computes the
gradients inside its forward (one fused library call) and scales them by the
upstream gradient in backward.
"""
from __future__ import annotations

import torch

from . import (FcklError, FcklProblem, FCKL_OK, fckl_check, fckl_fwd, fckl_fwd_bwd,
               fckl_fwd_bwd_host, fckl_fwd_bwd_sliced, fckl_host_workspace_bytes,
               fckl_workspace_bytes)

__all__ = ["make_problem", "alloc_workspace", "fused_kl_fwd", "fused_kl_fwd_bwd", "student_entropy",
           "select_top_rows", "fused_kl_rows", "arrays_to_device",
           "fused_kl_from_host", "alloc_host_workspace", "fused_kl_fwd_bwd_host",
           "fused_kl_fwd_bwd_sliced",
           "FusedChunkedKL", "fused_chunked_kl_loss"]


def _bits(t: torch.Tensor) -> torch.Tensor:
    if t.dtype == torch.bfloat16:
        return t
    if t.dtype in (torch.int16, torch.uint16):
        return t.view(torch.bfloat16)
    raise TypeError(f"expected bfloat16 (or its uint16 bits), got {t.dtype}")


def make_problem(hidden, W, topk_idx, T=1.0, chunk=0, teacher=0, n_valid_total=0,
                 dw_rows=0) -> FcklProblem:
    N, H = hidden.shape
    V = W.shape[0]
    K = topk_idx.shape[1]
    return FcklProblem(N, H, V, K, T, chunk, teacher, n_valid_total, dw_rows)


def alloc_workspace(prob: FcklProblem, device) -> torch.Tensor:
    nbytes = fckl_workspace_bytes(prob)
    if nbytes == 0:
        raise FcklError(1, "fckl_workspace_bytes")
    return torch.empty(nbytes, dtype=torch.uint8, device=device)


def _check_shapes(hidden, W, topk_idx=None, topk_logit=None, row_mask=None):
    """Shapes and dtypes the library reads without further checks: hidden [N,H],
    W [V,H], topk_idx int32 and topk_logit float32 [N,K], row_mask uint8 [N]."""
    if hidden.dim() != 2 or W.dim() != 2 or W.shape[1] != hidden.shape[1]:
        raise ValueError(f"hidden must be [N,H] and W [V,H]; got {tuple(hidden.shape)} "
                         f"and {tuple(W.shape)}")
    N = hidden.shape[0]
    if topk_idx is not None:
        if (topk_idx.dim() != 2 or tuple(topk_logit.shape) != tuple(topk_idx.shape)
                or topk_idx.shape[0] != N):
            raise ValueError(f"topk_idx and topk_logit must both be [N={N},K]; got "
                             f"{tuple(topk_idx.shape)} and {tuple(topk_logit.shape)}")
        if topk_idx.dtype != torch.int32 or topk_logit.dtype != torch.float32:
            raise TypeError("topk_idx must be int32 and topk_logit float32")
    if row_mask is not None:
        if row_mask.dtype != torch.uint8 or row_mask.numel() != N:
            raise TypeError(f"row_mask must be a uint8 tensor of N={N} entries")


def _check_placement(cuda, tensors):
    """Every named tensor contiguous and on one CUDA device (cuda=True) or on
    the host (cuda=False)."""
    devices = set()
    for name, t in tensors:
        if t is None:
            continue
        where = "CUDA" if cuda else "CPU"
        if t.is_cuda != cuda or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous {where} tensor")
        devices.add(t.device)
    if cuda and len(devices) > 1:
        raise ValueError(f"all tensors must be on one device; got {sorted(map(str, devices))}")


def _workspace(workspace, prob, device, host_inputs=False):
    """The caller's workspace (a contiguous uint8 tensor on ``device``; the
    library checks its size), or a new one of the size the problem needs."""
    if workspace is None:
        return (alloc_host_workspace if host_inputs else alloc_workspace)(prob, device)
    if workspace.dtype != torch.uint8 or not workspace.is_contiguous() or workspace.device != device:
        raise ValueError(f"workspace must be a contiguous uint8 tensor on {device}")
    return workspace


def _check_out(out, prob, device, with_loss=True):
    """Caller-supplied outputs: (loss[>=1],) dH [N,H], dW [V,H], contiguous float32
    tensors on the inputs' device."""
    names = ("loss", "dH", "dW") if with_loss else ("dH", "dW")
    if len(out) != len(names):
        raise ValueError("out must be (" + ", ".join(names) + ")")
    want = {"loss": None, "dH": (prob.N, prob.H), "dW": (prob.V, prob.H)}
    for name, t in zip(names, out):
        shape_ok = t.numel() >= 1 if want[name] is None else tuple(t.shape) == want[name]
        if (not shape_ok or t.dtype != torch.float32 or not t.is_contiguous()
                or t.device != device):
            raise ValueError(f"out {name} must be a contiguous float32 tensor on {device}"
                             + ("" if want[name] is None else f" of shape {want[name]}"))


def _check_inputs(hidden, W, topk_idx, topk_logit, row_mask):
    _check_shapes(hidden, W, topk_idx, topk_logit, row_mask)
    _check_placement(True, (("hidden", hidden), ("W", W), ("topk_idx", topk_idx),
                            ("topk_logit", topk_logit), ("row_mask", row_mask)))


def fused_kl_fwd_bwd(hidden, W, topk_idx, topk_logit, row_mask=None, T=1.0, chunk=0,
                     workspace=None, want_row_loss=False, check=True, out=None, teacher=0,
                     n_valid_total=0, dw_rows=0):
    """Returns (loss[1], row_loss[N] or None, dH[N,H] fp32, dW[V,H] fp32).

    ``out``: optional (loss, dH, dW) tensors to write into instead of allocating.
    ``n_valid_total``: N_v for the mean and gradient scale when these rows are one
    shard of a larger batch (0 = the valid rows of this call).
    ``dw_rows``: group chunks so that each dW GEMM covers at least this many
    rows (0 = one dW GEMM per chunk)."""
    hidden, W = _bits(hidden), _bits(W)
    _check_inputs(hidden, W, topk_idx, topk_logit, row_mask)
    prob = make_problem(hidden, W, topk_idx, T, chunk, teacher, n_valid_total, dw_rows)
    dev = hidden.device
    workspace = _workspace(workspace, prob, dev)
    if out is not None:
        _check_out(out, prob, dev)
        loss, dH, dW = out
    else:
        loss = torch.empty(1, dtype=torch.float32, device=dev)
        dH = torch.empty(prob.N, prob.H, dtype=torch.float32, device=dev)
        dW = torch.empty(prob.V, prob.H, dtype=torch.float32, device=dev)
    row_loss = torch.empty(prob.N, dtype=torch.float32, device=dev) if want_row_loss else None
    stream = torch.cuda.current_stream(dev).cuda_stream
    st = fckl_fwd_bwd(prob, hidden.data_ptr(), W.data_ptr(), topk_idx.data_ptr(),
                      topk_logit.data_ptr(), None if row_mask is None else row_mask.data_ptr(),
                      loss.data_ptr(), None if row_loss is None else row_loss.data_ptr(),
                      dH.data_ptr(), dW.data_ptr(), workspace.data_ptr(), workspace.numel(),
                      stream)
    if st != FCKL_OK:
        raise FcklError(st, "fckl_fwd_bwd")
    if check:
        st = fckl_check(workspace.data_ptr(), stream)
        if st != FCKL_OK:
            raise FcklError(st, "fckl_check")
    return loss, row_loss, dH, dW


def fused_kl_fwd_bwd_sliced(hidden, W, topk_idx, topk_logit, row_mask=None, T=1.0, chunk=0,
                            workspace=None, n_slices=4, teacher=0, n_valid_total=0, out=None,
                            dw_rows=0):
    """fused_kl_fwd_bwd whose last dW launch is split into ``n_slices``
    vocabulary slices.  Returns (loss[1], dH, dW, slices) with slices a list of
    (row0, row1, event): dW[row0:row1] is final once ``event`` (a
    torch.cuda.Event recorded on the current stream) has completed."""
    hidden, W = _bits(hidden), _bits(W)
    _check_inputs(hidden, W, topk_idx, topk_logit, row_mask)
    prob = make_problem(hidden, W, topk_idx, T, chunk, teacher, n_valid_total, dw_rows)
    dev = hidden.device
    workspace = _workspace(workspace, prob, dev)
    if out is None:
        out = (torch.empty(1, dtype=torch.float32, device=dev),
               torch.empty(prob.N, prob.H, dtype=torch.float32, device=dev),
               torch.empty(prob.V, prob.H, dtype=torch.float32, device=dev))
    _check_out(out, prob, dev)
    loss, dH, dW = out
    stream = torch.cuda.current_stream(dev)
    events = [torch.cuda.Event() for _ in range(n_slices)]
    for e in events:
        e.record(stream)  # creates the CUDA event; the call records it again
    st, rows = fckl_fwd_bwd_sliced(prob, hidden.data_ptr(), W.data_ptr(), topk_idx.data_ptr(),
                                   topk_logit.data_ptr(),
                                   None if row_mask is None else row_mask.data_ptr(),
                                   loss.data_ptr(), None, dH.data_ptr(), dW.data_ptr(),
                                   workspace.data_ptr(), workspace.numel(), stream.cuda_stream,
                                   [e.cuda_event for e in events])
    if st != FCKL_OK:
        raise FcklError(st, "fckl_fwd_bwd_sliced")
    slices = [(rows[i], rows[i + 1], events[i]) for i in range(n_slices)]
    return loss, dH, dW, slices


def fused_kl_fwd(hidden, W, topk_idx, topk_logit, row_mask=None, T=1.0, chunk=0,
                 workspace=None, want_row_loss=False, check=True, teacher=0):
    """Returns (loss[1], row_loss[N] or None)."""
    hidden, W = _bits(hidden), _bits(W)
    _check_inputs(hidden, W, topk_idx, topk_logit, row_mask)
    prob = make_problem(hidden, W, topk_idx, T, chunk, teacher)
    dev = hidden.device
    workspace = _workspace(workspace, prob, dev)
    loss = torch.empty(1, dtype=torch.float32, device=dev)
    row_loss = torch.empty(prob.N, dtype=torch.float32, device=dev) if want_row_loss else None
    stream = torch.cuda.current_stream(dev).cuda_stream
    st = fckl_fwd(prob, hidden.data_ptr(), W.data_ptr(), topk_idx.data_ptr(),
                  topk_logit.data_ptr(), None if row_mask is None else row_mask.data_ptr(),
                  loss.data_ptr(), None if row_loss is None else row_loss.data_ptr(),
                  workspace.data_ptr(), workspace.numel(), stream)
    if st != FCKL_OK:
        raise FcklError(st, "fckl_fwd")
    if check:
        st = fckl_check(workspace.data_ptr(), stream)
        if st != FCKL_OK:
            raise FcklError(st, "fckl_check")
    return loss, row_loss


def alloc_host_workspace(prob: FcklProblem, device) -> torch.Tensor:
    nbytes = fckl_host_workspace_bytes(prob)
    if nbytes == 0:
        raise FcklError(1, "fckl_host_workspace_bytes")
    return torch.empty(nbytes, dtype=torch.uint8, device=device)


def fused_kl_fwd_bwd_host(hidden, W, topk_idx, topk_logit, row_mask=None, T=1.0, chunk=0,
                          workspace=None, out=None, loss_host=None, check=True, dw_rows=0):
    """Forward + backward from HOST inputs (contiguous CPU tensors; pinned for
    overlapped copies): hidden bf16 [N,H], topk_idx int32 [N,K], topk_logit
    float32 [N,K], row_mask uint8 [N] or None.  W is a CUDA bf16 tensor.  The
    library streams the inputs to the device chunk by chunk, overlapped with
    the kernels.  Returns (loss as a Python float, dH, dW); the loss read
    synchronises the stream."""
    hidden, W = _bits(hidden), _bits(W)
    _check_shapes(hidden, W, topk_idx, topk_logit, row_mask)
    _check_placement(False, (("hidden", hidden), ("topk_idx", topk_idx),
                             ("topk_logit", topk_logit), ("row_mask", row_mask)))
    _check_placement(True, (("W", W),))
    prob = make_problem(hidden, W, topk_idx, T, chunk, dw_rows=dw_rows)
    dev = W.device
    workspace = _workspace(workspace, prob, dev, host_inputs=True)
    if out is None:
        out = (torch.empty(prob.N, prob.H, dtype=torch.float32, device=dev),
               torch.empty(prob.V, prob.H, dtype=torch.float32, device=dev))
    _check_out(out, prob, dev, with_loss=False)
    dH, dW = out
    if loss_host is None:
        loss_host = torch.empty(1, dtype=torch.float32, pin_memory=True)
    stream = torch.cuda.current_stream(dev)
    st = fckl_fwd_bwd_host(prob, hidden.data_ptr(), W.data_ptr(), topk_idx.data_ptr(),
                           topk_logit.data_ptr(),
                           None if row_mask is None else row_mask.data_ptr(),
                           loss_host.data_ptr(), dH.data_ptr(), dW.data_ptr(),
                           workspace.data_ptr(), workspace.numel(), stream.cuda_stream)
    if st != FCKL_OK:
        raise FcklError(st, "fckl_fwd_bwd_host")
    if check:
        st = fckl_check(workspace.data_ptr(), stream.cuda_stream)
        if st != FCKL_OK:
            raise FcklError(st, "fckl_check")
    else:
        stream.synchronize()
    return float(loss_host[0]), dH, dW


def fused_kl_from_host(dev_bufs: dict, host: dict, T=1.0, chunk=0, workspace=None, out=None):
    """End-to-end call from pinned host arrays: copies the inputs host->device on
    the current stream, runs fused forward+backward, and reads the loss back.
    ``dev_bufs`` holds preallocated device tensors with the same keys as
    ``host`` (hidden, W, topk_idx, topk_logit, row_mask).  Returns (loss as a
    Python float, dH, dW)."""
    for k, h in host.items():
        dev_bufs[k].copy_(h, non_blocking=True)
    loss, _, dH, dW = fused_kl_fwd_bwd(dev_bufs["hidden"], dev_bufs["W"], dev_bufs["topk_idx"],
                                       dev_bufs["topk_logit"], dev_bufs.get("row_mask"), T=T,
                                       chunk=chunk, workspace=workspace, check=False, out=out)
    return float(loss.item()), dH, dW


class FusedChunkedKL(torch.autograd.Function):
    """loss = FusedChunkedKL.apply(hidden_bf16, W_bf16, topk_idx, topk_logit, row_mask, T, chunk)

    Gradients flow to hidden and W (returned as fp32 tensors cast to the input
    dtype); the fused call computes them in forward."""

    @staticmethod
    def forward(ctx, hidden, W, topk_idx, topk_logit, row_mask, T, chunk):
        loss, _, dH, dW = fused_kl_fwd_bwd(hidden, W, topk_idx, topk_logit, row_mask, T, chunk)
        ctx.save_for_backward(dH, dW)
        ctx.dtypes = (hidden.dtype, W.dtype)
        return loss[0]

    @staticmethod
    def backward(ctx, grad_out):
        dH, dW = ctx.saved_tensors
        return ((dH * grad_out).to(ctx.dtypes[0]), (dW * grad_out).to(ctx.dtypes[1]),
                None, None, None, None, None)


def fused_chunked_kl_loss(hidden, W, topk_idx, topk_logit, row_mask=None, T=1.0, chunk=0):
    return FusedChunkedKL.apply(hidden, W, topk_idx, topk_logit, row_mask, T, chunk)


def arrays_to_device(hidden_bits, W_bits, topk_idx, topk_logit, row_mask, device="cuda"):
    """numpy arrays (bf16 bit patterns as uint16, int32 ids, float32 logits,
    uint8 mask or None) -> contiguous device tensors, in that order."""
    import numpy as np

    def t(a, dt):
        return torch.from_numpy(np.ascontiguousarray(a).view(dt))

    out = [t(hidden_bits, np.int16).to(device).view(torch.bfloat16),
           t(W_bits, np.int16).to(device).view(torch.bfloat16),
           t(topk_idx, np.int32).to(device),
           t(topk_logit, np.float32).to(device),
           None if row_mask is None else t(row_mask, np.uint8).to(device)]
    return tuple(out)


def student_entropy(hidden, W, row_mask=None, T=1.0, chunk=0, workspace=None, check=True):
    """Per-row student entropy H(softmax(W h / T)) in nats, [N] fp32 (0 for masked rows)."""
    from . import fckl_student_entropy
    hidden, W = _bits(hidden), _bits(W)
    _check_shapes(hidden, W, row_mask=row_mask)
    _check_placement(True, (("hidden", hidden), ("W", W), ("row_mask", row_mask)))
    N, H = hidden.shape
    prob = FcklProblem(N, H, W.shape[0], 1, T, chunk)
    dev = hidden.device
    workspace = _workspace(workspace, prob, dev)
    ent = torch.empty(N, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev).cuda_stream
    st = fckl_student_entropy(prob, hidden.data_ptr(), W.data_ptr(),
                              None if row_mask is None else row_mask.data_ptr(), ent.data_ptr(),
                              workspace.data_ptr(), workspace.numel(), stream)
    if st != FCKL_OK:
        raise FcklError(st, "fckl_student_entropy")
    if check:
        st = fckl_check(workspace.data_ptr(), stream)
        if st != FCKL_OK:
            raise FcklError(st, "fckl_check")
    return ent


def select_top_rows(score, n_select, row_mask=None):
    """(rows int32 [n_select] ascending, padded with -1; count int32 [1]) on device."""
    from . import fckl_select_top_rows
    if score.dtype != torch.float32 or score.dim() != 1:
        raise TypeError("score must be a 1-D float32 tensor")
    if row_mask is not None and (row_mask.dtype != torch.uint8 or row_mask.numel() != score.numel()):
        raise TypeError("row_mask must be a uint8 tensor with one entry per score")
    _check_placement(True, (("score", score), ("row_mask", row_mask)))
    N = score.numel()
    rows = torch.empty(n_select, dtype=torch.int32, device=score.device)
    count = torch.empty(1, dtype=torch.int32, device=score.device)
    st = fckl_select_top_rows(score.data_ptr(), None if row_mask is None else row_mask.data_ptr(),
                              N, n_select, rows.data_ptr(), count.data_ptr(),
                              torch.cuda.current_stream(score.device).cuda_stream)
    if st != FCKL_OK:
        raise FcklError(st, "fckl_select_top_rows")
    return rows, count


def fused_kl_rows(hidden, W, topk_idx, topk_logit, rows, T=1.0, chunk=0, workspace=None,
                  grads=True, want_row_loss=False, check=True, teacher=0, dw_rows=0):
    """Loss (and dH, dW) over the listed rows only.  Returns (loss, row_loss, dH, dW)."""
    from . import fckl_fwd_bwd_rows
    hidden, W = _bits(hidden), _bits(W)
    if rows.dtype != torch.int32 or rows.dim() != 1:
        raise TypeError("rows must be a 1-D int32 tensor")
    _check_inputs(hidden, W, topk_idx, topk_logit, None)
    _check_placement(True, (("hidden", hidden), ("rows", rows)))
    prob = make_problem(hidden, W, topk_idx, T, chunk, teacher, dw_rows=dw_rows)
    dev = hidden.device
    workspace = _workspace(workspace, prob, dev)
    loss = torch.empty(1, dtype=torch.float32, device=dev)
    row_loss = torch.empty(prob.N, dtype=torch.float32, device=dev) if want_row_loss else None
    dH = torch.empty(prob.N, prob.H, dtype=torch.float32, device=dev) if grads else None
    dW = torch.empty(prob.V, prob.H, dtype=torch.float32, device=dev) if grads else None
    stream = torch.cuda.current_stream(dev).cuda_stream
    st = fckl_fwd_bwd_rows(prob, hidden.data_ptr(), W.data_ptr(), topk_idx.data_ptr(),
                           topk_logit.data_ptr(), rows.data_ptr(), rows.numel(), loss.data_ptr(),
                           None if row_loss is None else row_loss.data_ptr(),
                           None if dH is None else dH.data_ptr(),
                           None if dW is None else dW.data_ptr(), workspace.data_ptr(),
                           workspace.numel(), stream)
    if st != FCKL_OK:
        raise FcklError(st, "fckl_fwd_bwd_rows")
    if check:
        st = fckl_check(workspace.data_ptr(), stream)
        if st != FCKL_OK:
            raise FcklError(st, "fckl_check")
    return loss, row_loss, dH, dW
