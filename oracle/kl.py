"""fp64 reference of the fused chunked KL loss (forward and gradients).

TEST INFRASTRUCTURE ONLY -- see the package docstring.

What is computed (the pages' method, stated in the oracle's own notation):

  rows r = 0..N-1 (the flattened batch x sequence positions), valid when
  row_mask[r] != 0; N_v = number of valid rows.
  z_r = W h_r                      student logits over the whole vocabulary V
  a   = z_r / T                    temperature-softened student logits
  log q = a - logsumexp(a)         student log-probabilities over all V
  t_k = topk_logit[r, k] / T       softened cached teacher logits, k = 0..K-1
  log p = t - logsumexp(t)         teacher distribution over the K cached ids
                                   only (zero probability elsewhere)
  l_r = sum_k p_k (log p_k - log q[id_k])          forward KL(p || q)
  L   = (1/N_v) sum_{valid r} l_r
  dlogits_r = (q - p~) / (T N_v),  p~_v = sum_{k: id_k = v} p_k
  dH_r = dlogits_r W               dW = sum_r dlogits_r^T h_r

Passages this follows:
  * forward KL between temperature-softened teacher and student outputs:
    LLM Primer ch.6 "프루닝과 지식 증류", section 6.2 (the distillation loss is the
    KL divergence between softened teacher and student outputs; MiniLLM's
    reverse KL is named as the alternative, so the default is forward KL);
  * teacher reduced to a top-K cache (top-100 per position), student compared
    against it without a dense teacher grid: aibase.it write-up
    "Knowledge Distillation 비용 줄이기", sections "offline top-K logits 방식" and
    "chunked KL loss가 하는 일";
  * dense KL as the correctness baseline, output projection fused into the loss
    and chunked over positions: same write-up, section "chunked KL loss가 하는 일";
    "[논문리뷰] Efficient Knowledge Distillation for LLMs: Offline Top-K Logits and
    a Fused Chunked KL Loss", section 1 (Fused Chunked KL Loss definition);
  * losses identical across the dense / chunked / fused variants ("lossless"):
    AI Trends summary of the paper, evidence list.

Readings taken where the pages are silent:
  * no T^2 factor on the gradients; the loss is exactly L above;
  * p is renormalised over the K cached logits; q is normalised over all V;
  * the reduction is the mean over valid rows of the flattened batch;
  * N_v = 0 gives L = 0 and zero gradients;
  * a teacher logit of -inf is allowed and gives p_k = 0 with 0 * log 0 := 0;
  * repeated ids in one row add into one cell of the dense teacher p~ (the
    dense-KL baseline expands the cache into the dense teacher grid), so the
    loss is KL(p~ || q) over the distinct ids;
  * teacher format "probs" (random-sampled sparse targets, "기술 요약: 선택적 지식
    증류의 재고", section 방법론, RS-KD): the cache holds non-negative class
    weights, p = w / sum(w), and the temperature applies to the student only.

The oracle materialises each block's full [rows, V] fp64 softmax (the dense
formulation); blocking over rows only regroups independent rows.
"""
from __future__ import annotations

import numpy as np

__all__ = ["log_softmax", "teacher_distribution", "student_log_probs", "dense_teacher",
           "fused_chunked_kl", "widen_bf16", "oracle_from_inputs"]


def widen_bf16(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) -> exact float64 values."""
    u = np.ascontiguousarray(bits, dtype=np.uint16)
    return (u.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def log_softmax(x: np.ndarray, axis: int = -1) -> np.ndarray:
    """log(exp(x) / sum exp(x)) along ``axis`` with the usual max shift.

    Entries equal to -inf give -inf (probability 0)."""
    x = np.asarray(x, dtype=np.float64)
    m = np.max(x, axis=axis, keepdims=True)
    m = np.where(np.isfinite(m), m, 0.0)
    with np.errstate(divide="ignore"):
        lse = m + np.log(np.sum(np.exp(x - m), axis=axis, keepdims=True))
    return x - lse


def teacher_distribution(topk_logit: np.ndarray, T: float, teacher: str = "logits"):
    """Teacher probabilities over the K cache entries of each row.

    "logits": p = softmax(topk_logit / T) -- aibase.it write-up, section
    "offline top-K logits 방식" (only the top-K logits per position are kept);
    LLM Primer ch.6, section 6.2 (temperature).
    "probs": p = w / sum(w) with w = topk_logit >= 0 -- sampled sparse targets
    (RS-KD, "기술 요약: 선택적 지식 증류의 재고", section 방법론).
    Returns (p, log p), both [rows, K] float64 (log p = -inf where p = 0)."""
    x = np.asarray(topk_logit, dtype=np.float64)
    if teacher == "probs":
        tot = x.sum(axis=1, keepdims=True)
        p = x / tot
        with np.errstate(divide="ignore"):
            return p, np.log(p)
    logp = log_softmax(x / float(T), axis=1)
    return np.exp(logp), logp


def student_log_probs(Z: np.ndarray, T: float) -> np.ndarray:
    """log q = log_softmax(Z / T) over the full vocabulary (LLM Primer ch.6, 6.2)."""
    return log_softmax(np.asarray(Z, dtype=np.float64) / float(T), axis=1)


def dense_teacher(p: np.ndarray, ids: np.ndarray, V: int) -> np.ndarray:
    """Expand the sparse teacher into the dense [rows, V] grid p~ (entry-wise
    sum over repeated ids): the dense-KL correctness baseline of the aibase.it
    write-up, section "chunked KL loss가 하는 일"."""
    rows = p.shape[0]
    out = np.zeros((rows, V), dtype=np.float64)
    r = np.repeat(np.arange(rows), ids.shape[1])
    np.add.at(out, (r, ids.reshape(-1).astype(np.int64)), p.reshape(-1))
    return out


def fused_chunked_kl(hidden: np.ndarray, W: np.ndarray, topk_idx: np.ndarray,
                     topk_logit: np.ndarray, row_mask: np.ndarray | None, T: float,
                     *, rows: np.ndarray | None = None, row_block: int = 256,
                     grads: bool = True, return_dlogits: bool = False,
                     teacher: str = "logits", n_valid: int | None = None) -> dict:
    """Loss and gradients of the fused chunked forward KL, in fp64.

    hidden [N, H] and W [V, H]: float arrays, or uint16 bf16 bit patterns
    (widened exactly; hidden one block of rows at a time).  topk_idx int
    [N, K] in [0, V), topk_logit [N, K], row_mask [N] (nonzero = row included;
    None = all rows), temperature T > 0, teacher format "logits" or "probs"
    (see teacher_distribution).  ``n_valid``: the N_v of the mean and of the
    gradient scale when these rows are one shard of a larger batch (default:
    the valid rows of ``row_mask``).

    ``rows``: optional subset of rows to evaluate (masked ones are dropped;
    N_v still counts every valid row of the mask).  Without it every valid row
    is evaluated.  ``row_block``: how many rows share one materialised [rows, V]
    grid.

    Returns a dict:
      n_valid, rows (evaluated rows, ascending), row_loss_rows [len(rows)],
      loss (mean over valid rows; only when ``rows`` is None),
      row_loss [N] (only when ``rows`` is None; 0 for masked rows),
      when ``grads``: dH_rows [len(rows), H], dW [V, H] (the evaluated rows'
      contribution), and dH [N, H] when ``rows`` is None;
      when ``return_dlogits``: dlogits_rows [len(rows), V].
    """
    W = widen_bf16(W) if np.asarray(W).dtype == np.uint16 else np.asarray(W, dtype=np.float64)
    hidden_bits = np.asarray(hidden).dtype == np.uint16
    N, H = hidden.shape
    V = W.shape[0]
    mask = np.ones(N, dtype=bool) if row_mask is None else (np.asarray(row_mask) != 0)
    n_valid = int(mask.sum()) if n_valid is None else int(n_valid)
    if rows is None:
        todo = np.nonzero(mask)[0]
    else:
        todo = np.unique(np.asarray(rows, dtype=np.int64))
        todo = todo[mask[todo]]
    n = todo.size
    out = {"n_valid": n_valid, "rows": todo, "row_loss_rows": np.zeros(n)}
    if grads:
        out["dH_rows"] = np.zeros((n, H))
        out["dW"] = np.zeros((V, H))
    if return_dlogits:
        out["dlogits_rows"] = np.zeros((n, V))
    if n_valid > 0 and n > 0:
        grad_scale = 1.0 / (float(T) * n_valid)
        step = max(1, int(row_block))
        for b0 in range(0, n, step):
            sel = slice(b0, min(n, b0 + step))
            rb = todo[sel]
            Hb = widen_bf16(hidden[rb]) if hidden_bits else np.asarray(hidden[rb], dtype=np.float64)
            Z = Hb @ W.T                                  # student logits [b, V]
            logq = student_log_probs(Z, T)                # normalised over all V
            p, logp = teacher_distribution(topk_logit[rb], T, teacher)
            ids = np.asarray(topk_idx[rb], dtype=np.int64)
            P = dense_teacher(p, ids, V)            # [b, V]: repeated ids add up
            with np.errstate(divide="ignore", invalid="ignore"):
                terms = np.where(P > 0.0, P * (np.log(P) - logq), 0.0)
            out["row_loss_rows"][sel] = terms.sum(axis=1)
            if grads or return_dlogits:
                G = (np.exp(logq) - P) * grad_scale
                if return_dlogits:
                    out["dlogits_rows"][sel] = G
                if grads:
                    out["dH_rows"][sel] = G @ W
                    out["dW"] += G.T @ Hb
    if rows is None:
        row_loss = np.zeros(N)
        row_loss[todo] = out["row_loss_rows"]
        out["row_loss"] = row_loss
        out["loss"] = float(row_loss.sum() / n_valid) if n_valid > 0 else 0.0
        if grads:
            dH = np.zeros((N, H))
            dH[todo] = out["dH_rows"]
            out["dH"] = dH
    return out


def oracle_from_inputs(inp, *, rows=None, row_block: int = 256, grads: bool = True,
                       teacher: str = "logits") -> dict:
    """Run ``fused_chunked_kl`` on a ``synth.Inputs`` bundle (bf16 widened exactly)."""
    return fused_chunked_kl(inp.hidden, inp.W, inp.topk_idx, inp.topk_logit, inp.row_mask,
                            inp.cfg.T, rows=rows, row_block=row_block, grads=grads,
                            teacher=teacher)
