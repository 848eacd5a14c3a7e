"""Pins of the selective-distillation oracle functions (CPU)."""
import numpy as np
import scipy.special
import scipy.stats

import oracle


def _case(seed, N=30, H=12, V=70, wscale=0.5):
    rng = np.random.default_rng(seed)
    return rng.standard_normal((N, H)), rng.standard_normal((V, H)) * wscale


def test_entropy_matches_scipy():
    for seed, T in [(1, 1.0), (2, 0.5), (3, 2.5)]:
        h, W = _case(seed)
        mask = (np.arange(h.shape[0]) % 7 != 3).astype(np.uint8)
        e = oracle.student_entropy(h, W, T, mask)
        q = scipy.special.softmax((h @ W.T) / T, axis=1)
        ref = scipy.stats.entropy(q, axis=1)
        np.testing.assert_allclose(e[mask != 0], ref[mask != 0], rtol=1e-12, atol=1e-13)
        assert (e[mask == 0] == 0).all()


def test_entropy_closed_forms():
    h, W = _case(4)
    # all logits equal -> uniform q -> entropy log V
    np.testing.assert_allclose(oracle.student_entropy(h, np.zeros_like(W), 1.0), np.log(W.shape[0]),
                               rtol=1e-14)
    # adding a row-constant to every row of W shifts all logits of a row equally
    c = np.random.default_rng(5).standard_normal(h.shape[1])
    np.testing.assert_allclose(oracle.student_entropy(h, W + c[None, :], 1.3),
                               oracle.student_entropy(h, W, 1.3), rtol=1e-10)
    # bounds 0 <= H <= log V, and low temperature concentrates q
    e = oracle.student_entropy(h, W * 4, 1.0)
    assert (e >= 0).all() and (e <= np.log(W.shape[0]) + 1e-12).all()
    assert oracle.student_entropy(h, W, 0.05).mean() < oracle.student_entropy(h, W, 5.0).mean()


def test_entropy_row_subset():
    h, W = _case(6)
    full = oracle.student_entropy(h, W, 1.0)
    rows, sub = oracle.student_entropy(h, W, 1.0, rows=[3, 0, 17])
    np.testing.assert_array_equal(rows, [3, 0, 17])
    np.testing.assert_allclose(sub, full[[3, 0, 17]], rtol=1e-14)


def _brute_select(score, mask, n):
    """Pure-Python rank count: row i is taken iff fewer than n valid rows beat it."""
    N = len(score)
    valid = [mask is None or mask[i] != 0 for i in range(N)]
    take = []
    for i in range(N):
        if not valid[i]:
            continue
        rank = sum(1 for j in range(N) if valid[j] and (score[j] > score[i] or (score[j] == score[i] and j < i)))
        if rank < n:
            take.append(i)
    return take


def test_select_matches_brute_force_with_ties_and_mask():
    rng = np.random.default_rng(7)
    for trial in range(20):
        N = int(rng.integers(1, 60))
        score = rng.integers(0, 6, N).astype(np.float32) * 0.5 - 1.0  # many ties, negatives
        mask = (rng.random(N) < 0.8).astype(np.uint8)
        n = int(rng.integers(1, N + 1))
        rows, count = oracle.select_top_rows(score, mask, n)
        ref = _brute_select(score.tolist(), mask.tolist(), n)
        assert count == len(ref)
        assert rows[:count].tolist() == ref
        assert (rows[count:] == -1).all()


def test_select_without_mask_takes_exactly_n():
    score = np.random.default_rng(8).standard_normal(1000).astype(np.float32)
    rows, count = oracle.select_top_rows(score, None, 200)
    assert count == 200 and (np.diff(rows) > 0).all()
    assert score[rows].min() >= np.sort(score)[-200]
