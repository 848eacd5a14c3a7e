"""Fused chunked forward-KL distillation loss on B200 (sm_100a).

Thin ctypes binding over the C ABI in ``include/fckl.h`` (``libfckl.so``, built
in-tree by ``chunked_kl_loss_tcgen05_b200.build``).  The functions below keep
the C names and only marshal arguments; every step of the loss runs in the
library's CUDA kernels.  There is no CPU fallback: if the library is missing,
``load()`` raises.

``torch_api`` adds tensor-level helpers (allocation of outputs and workspace
with PyTorch, an autograd Function) on top of these calls.
"""
from __future__ import annotations

import ctypes
import os

__all__ = [
    "FCKL_OK", "FCKL_ERR_INVALID_ARG", "FCKL_ERR_UNSUPPORTED", "FCKL_ERR_WORKSPACE",
    "FCKL_ERR_BAD_INDEX", "FCKL_ERR_BAD_TEACHER", "FCKL_ERR_TIMEOUT", "FCKL_ERR_CUDA",
    "FCKL_K_MAX", "FCKL_TEACHER_LOGITS", "FCKL_TEACHER_PROBS", "FcklProblem", "FcklError", "load", "lib_path", "exported_symbols",
    "fckl_workspace_bytes", "fckl_resolved_chunk", "fckl_fwd", "fckl_fwd_bwd", "fckl_check",
    "fckl_status_string", "FcklKernelStat", "fckl_profile_begin", "fckl_profile_end",
    "fckl_fwd_noalloc", "fckl_student_entropy", "fckl_select_top_rows", "fckl_fwd_bwd_rows",
    "fckl_host_workspace_bytes", "fckl_fwd_bwd_host", "fckl_fwd_bwd_sliced",
]

FCKL_OK = 0
FCKL_ERR_INVALID_ARG = 1
FCKL_ERR_UNSUPPORTED = 2
FCKL_ERR_WORKSPACE = 3
FCKL_ERR_BAD_INDEX = 4
FCKL_ERR_BAD_TEACHER = 5
FCKL_ERR_TIMEOUT = 6
FCKL_ERR_CUDA = 7
FCKL_K_MAX = 256

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB = None

exported_symbols = ("fckl_workspace_bytes", "fckl_resolved_chunk", "fckl_fwd", "fckl_fwd_bwd",
                    "fckl_check", "fckl_status_string", "fckl_profile_begin", "fckl_profile_end",
                    "fckl_fwd_noalloc", "fckl_student_entropy", "fckl_select_top_rows",
                    "fckl_fwd_bwd_rows", "fckl_host_workspace_bytes", "fckl_fwd_bwd_host",
                    "fckl_fwd_bwd_sliced")


FCKL_TEACHER_LOGITS = 0
FCKL_TEACHER_PROBS = 1


class FcklProblem(ctypes.Structure):
    """Mirror of ``fckl_problem``."""
    _fields_ = [("N", ctypes.c_int64), ("H", ctypes.c_int64), ("V", ctypes.c_int64),
                ("K", ctypes.c_int32), ("T", ctypes.c_float), ("chunk", ctypes.c_int64),
                ("teacher", ctypes.c_int32), ("n_valid_total", ctypes.c_int64),
                ("dw_rows", ctypes.c_int64)]

    def __init__(self, N, H, V, K, T=1.0, chunk=0, teacher=FCKL_TEACHER_LOGITS, n_valid_total=0,
                 dw_rows=0):
        super().__init__(int(N), int(H), int(V), int(K), float(T), int(chunk), int(teacher),
                         int(n_valid_total), int(dw_rows))


class FcklKernelStat(ctypes.Structure):
    """Mirror of ``fckl_kernel_stat``."""
    _fields_ = [("name", ctypes.c_char * 32), ("launches", ctypes.c_int64),
                ("total_ms", ctypes.c_double), ("flops", ctypes.c_double),
                ("bytes", ctypes.c_double)]


class FcklError(RuntimeError):
    def __init__(self, status: int, where: str = ""):
        self.status = int(status)
        super().__init__(f"{where}: {fckl_status_string(status)} ({status})")


def lib_path() -> str:
    return os.environ.get("FCKL_LIB", os.path.join(_HERE, "libfckl.so"))


def load() -> ctypes.CDLL:
    """Load libfckl.so (raises if it has not been built)."""
    global _LIB
    if _LIB is not None:
        return _LIB
    path = lib_path()
    if not os.path.exists(path):
        raise FileNotFoundError(
            f"{path} is missing; build it with `python -m chunked_kl_loss_tcgen05_b200.build`")
    lib = ctypes.CDLL(path)
    P = ctypes.POINTER(FcklProblem)
    vp, sz = ctypes.c_void_p, ctypes.c_size_t
    lib.fckl_workspace_bytes.argtypes = [P]
    lib.fckl_workspace_bytes.restype = sz
    lib.fckl_resolved_chunk.argtypes = [P]
    lib.fckl_resolved_chunk.restype = ctypes.c_int64
    lib.fckl_fwd.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.fckl_fwd.restype = ctypes.c_int
    lib.fckl_fwd_bwd.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.fckl_fwd_bwd.restype = ctypes.c_int
    lib.fckl_fwd_bwd_sliced.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp,
                                         ctypes.c_int32, ctypes.POINTER(vp),
                                         ctypes.POINTER(ctypes.c_int64)]
    lib.fckl_fwd_bwd_sliced.restype = ctypes.c_int
    lib.fckl_host_workspace_bytes.argtypes = [P]
    lib.fckl_host_workspace_bytes.restype = sz
    lib.fckl_fwd_bwd_host.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.fckl_fwd_bwd_host.restype = ctypes.c_int
    lib.fckl_check.argtypes = [vp, vp]
    lib.fckl_check.restype = ctypes.c_int
    lib.fckl_status_string.argtypes = [ctypes.c_int]
    lib.fckl_status_string.restype = ctypes.c_char_p
    lib.fckl_student_entropy.argtypes = [P, vp, vp, vp, vp, vp, sz, vp]
    lib.fckl_student_entropy.restype = ctypes.c_int
    lib.fckl_select_top_rows.argtypes = [vp, vp, ctypes.c_int64, ctypes.c_int64, vp, vp, vp]
    lib.fckl_select_top_rows.restype = ctypes.c_int
    lib.fckl_fwd_bwd_rows.argtypes = [P, vp, vp, vp, vp, vp, ctypes.c_int64, vp, vp, vp, vp, vp,
                                      sz, vp]
    lib.fckl_fwd_bwd_rows.restype = ctypes.c_int
    lib.fckl_fwd_noalloc.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, vp, vp]
    lib.fckl_fwd_noalloc.restype = ctypes.c_int
    lib.fckl_profile_begin.argtypes = [ctypes.c_uint32]
    lib.fckl_profile_begin.restype = None
    lib.fckl_profile_end.argtypes = [ctypes.POINTER(FcklKernelStat), ctypes.c_int]
    lib.fckl_profile_end.restype = ctypes.c_int
    _LIB = lib
    return lib


def _ptr(x):
    return None if x is None or x == 0 else ctypes.c_void_p(int(x))


def fckl_workspace_bytes(prob: FcklProblem) -> int:
    return int(load().fckl_workspace_bytes(ctypes.byref(prob)))


def fckl_host_workspace_bytes(prob: FcklProblem) -> int:
    return int(load().fckl_host_workspace_bytes(ctypes.byref(prob)))


def fckl_resolved_chunk(prob: FcklProblem) -> int:
    return int(load().fckl_resolved_chunk(ctypes.byref(prob)))


def fckl_fwd(prob, hidden, W, topk_idx, topk_logit, row_mask, loss, row_loss,
             workspace, workspace_bytes, stream) -> int:
    """All array arguments are device addresses (ints) or None; returns the status."""
    return int(load().fckl_fwd(ctypes.byref(prob), _ptr(hidden), _ptr(W), _ptr(topk_idx),
                               _ptr(topk_logit), _ptr(row_mask), _ptr(loss), _ptr(row_loss),
                               _ptr(workspace), ctypes.c_size_t(int(workspace_bytes)),
                               _ptr(stream)))


def fckl_fwd_bwd(prob, hidden, W, topk_idx, topk_logit, row_mask, loss, row_loss, dH, dW,
                 workspace, workspace_bytes, stream) -> int:
    """All array arguments are device addresses (ints) or None; returns the status."""
    return int(load().fckl_fwd_bwd(ctypes.byref(prob), _ptr(hidden), _ptr(W), _ptr(topk_idx),
                                   _ptr(topk_logit), _ptr(row_mask), _ptr(loss),
                                   _ptr(row_loss), _ptr(dH), _ptr(dW), _ptr(workspace),
                                   ctypes.c_size_t(int(workspace_bytes)), _ptr(stream)))


def fckl_fwd_bwd_host(prob, hidden_host, W, topk_idx_host, topk_logit_host, row_mask_host,
                      loss_host, dH, dW, workspace, workspace_bytes, stream) -> int:
    """Inputs and the loss are HOST addresses (ints; row_mask may be None); W, dH,
    dW and the workspace are device addresses.  Returns the status."""
    return int(load().fckl_fwd_bwd_host(ctypes.byref(prob), _ptr(hidden_host), _ptr(W),
                                        _ptr(topk_idx_host), _ptr(topk_logit_host),
                                        _ptr(row_mask_host), _ptr(loss_host), _ptr(dH), _ptr(dW),
                                        _ptr(workspace), ctypes.c_size_t(int(workspace_bytes)),
                                        _ptr(stream)))


def fckl_fwd_bwd_sliced(prob, hidden, W, topk_idx, topk_logit, row_mask, loss, row_loss, dH, dW,
                        workspace, workspace_bytes, stream, events) -> tuple:
    """fckl_fwd_bwd with the last dW launch split into len(events) vocabulary
    slices; events are cudaEvent_t handles (ints).  Returns (status, row
    boundaries of the slices as a list of len(events) + 1 ints)."""
    n = len(events)
    ev = (ctypes.c_void_p * max(n, 1))(*[ctypes.c_void_p(int(e)) if e else None for e in events])
    rows = (ctypes.c_int64 * (n + 1))()
    st = load().fckl_fwd_bwd_sliced(ctypes.byref(prob), _ptr(hidden), _ptr(W), _ptr(topk_idx),
                                    _ptr(topk_logit), _ptr(row_mask), _ptr(loss), _ptr(row_loss),
                                    _ptr(dH), _ptr(dW), _ptr(workspace),
                                    ctypes.c_size_t(int(workspace_bytes)), _ptr(stream),
                                    ctypes.c_int32(n), ev, rows)
    return int(st), list(rows)


def fckl_fwd_noalloc(prob, hidden, W, topk_idx, topk_logit, row_mask, loss, row_loss,
                     device_status, stream) -> int:
    """Forward loss with the library's own static scratch (no workspace, no
    allocation).  Array arguments are device addresses (ints) or None."""
    return int(load().fckl_fwd_noalloc(ctypes.byref(prob), _ptr(hidden), _ptr(W), _ptr(topk_idx),
                                       _ptr(topk_logit), _ptr(row_mask), _ptr(loss),
                                       _ptr(row_loss), _ptr(device_status), _ptr(stream)))


def fckl_student_entropy(prob, hidden, W, row_mask, row_entropy, workspace, workspace_bytes,
                         stream) -> int:
    return int(load().fckl_student_entropy(ctypes.byref(prob), _ptr(hidden), _ptr(W),
                                           _ptr(row_mask), _ptr(row_entropy), _ptr(workspace),
                                           ctypes.c_size_t(int(workspace_bytes)), _ptr(stream)))


def fckl_select_top_rows(score, row_mask, N, n_select, rows_out, count_out, stream) -> int:
    return int(load().fckl_select_top_rows(_ptr(score), _ptr(row_mask), ctypes.c_int64(int(N)),
                                           ctypes.c_int64(int(n_select)), _ptr(rows_out),
                                           _ptr(count_out), _ptr(stream)))


def fckl_fwd_bwd_rows(prob, hidden, W, topk_idx, topk_logit, rows, n_rows, loss, row_loss, dH, dW,
                      workspace, workspace_bytes, stream) -> int:
    return int(load().fckl_fwd_bwd_rows(ctypes.byref(prob), _ptr(hidden), _ptr(W), _ptr(topk_idx),
                                        _ptr(topk_logit), _ptr(rows), ctypes.c_int64(int(n_rows)),
                                        _ptr(loss), _ptr(row_loss), _ptr(dH), _ptr(dW),
                                        _ptr(workspace), ctypes.c_size_t(int(workspace_bytes)),
                                        _ptr(stream)))


def fckl_check(workspace, stream) -> int:
    return int(load().fckl_check(_ptr(workspace), _ptr(stream)))


def fckl_status_string(status: int) -> str:
    return load().fckl_status_string(int(status)).decode()


KERNEL_KINDS = ("count_valid", "prep_teacher", "fwd_logits_lse", "merge_loss", "bwd_dlogits",
                "dH_gemm", "dW_gemm", "finalize", "entropy_gemm", "merge_entropy", "gather_rows",
                "scatter_rows", "select_rows", "zero_dw")


def fckl_profile_begin(kinds=None) -> None:
    """Start per-kernel event timing for the named kinds (None = all)."""
    mask = 0
    for k in (kinds or ()):
        mask |= 1 << KERNEL_KINDS.index(k)
    load().fckl_profile_begin(mask)


def fckl_profile_end(max_stats: int = 16) -> list:
    """Returns a list of dicts (name, launches, total_ms, flops, bytes)."""
    arr = (FcklKernelStat * max_stats)()
    n = int(load().fckl_profile_end(arr, max_stats))
    if n < 0:
        raise FcklError(FCKL_ERR_CUDA, "fckl_profile_end")
    return [dict(name=a.name.decode(), launches=int(a.launches), total_ms=float(a.total_ms),
                 flops=float(a.flops), bytes=float(a.bytes)) for a in arr[:min(n, max_stats)]]
