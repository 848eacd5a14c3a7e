"""fp64 reference of the selective-distillation helpers (student entropy and
top-k% position selection).

TEST INFRASTRUCTURE ONLY -- see the package docstring.

Passages: "기술 요약: 선택적 지식 증류(Selective Knowledge Distillation)의 재고",
section 방법론 -- SE-KD uses the student entropy H(q_t) as the position-importance
signal and supervises the top-k% positions; section 효율성 최적화 -- entropy is
computed chunk by chunk and logits/gradients only at the selected positions
(the loss over selected rows is the plain loss with the other rows masked out,
so it needs no oracle of its own: ``fused_chunked_kl`` with that mask).

Readings: the entropy is that of the temperature-T student softmax (the same q
as the loss), in nats; ties at the selection threshold go to the lower row
index; masked rows are never selected and get entropy 0.
"""
from __future__ import annotations

import numpy as np

from .kl import student_log_probs, widen_bf16

__all__ = ["student_entropy", "select_top_rows"]


def student_entropy(hidden, W, T: float, row_mask=None, *, rows=None, row_block: int = 256):
    """H(q_r) = -sum_v q_v log q_v for each row (0 for masked rows).

    hidden [N, H], W [V, H] as float arrays or bf16 bit patterns.  ``rows``:
    optional subset to evaluate; returns (rows, entropies) then, else [N]."""
    W = widen_bf16(W) if np.asarray(W).dtype == np.uint16 else np.asarray(W, dtype=np.float64)
    bits = np.asarray(hidden).dtype == np.uint16
    N = hidden.shape[0]
    mask = np.ones(N, bool) if row_mask is None else (np.asarray(row_mask) != 0)
    todo = np.arange(N) if rows is None else np.asarray(rows, dtype=np.int64)
    out = np.zeros(todo.size)
    for b0 in range(0, todo.size, row_block):
        rb = todo[b0:b0 + row_block]
        Hb = widen_bf16(hidden[rb]) if bits else np.asarray(hidden[rb], dtype=np.float64)
        logq = student_log_probs(Hb @ W.T, T)
        q = np.exp(logq)
        with np.errstate(invalid="ignore"):
            ent = -np.where(q > 0, q * logq, 0.0).sum(axis=1)
        out[b0:b0 + rb.size] = np.where(mask[rb], ent, 0.0)
    if rows is None:
        return out
    return todo, out


def select_top_rows(score, row_mask, n_select: int):
    """The n_select valid rows with the largest score, ascending; ties go to the
    lower row index.  Returns (rows padded with -1 to n_select, count)."""
    score = np.asarray(score)
    N = score.size
    valid = np.ones(N, bool) if row_mask is None else (np.asarray(row_mask) != 0)
    idx = np.nonzero(valid)[0]
    order = np.lexsort((idx, -score[idx].astype(np.float64)))  # score desc, then row asc
    take = np.sort(idx[order[:n_select]])
    out = np.full(n_select, -1, dtype=np.int64)
    out[:take.size] = take
    return out, int(take.size)
