"""Pins of the fp64 oracle to things other than itself.

Each check below is either a library routine (scipy's KL / entropy, torch's
cross-entropy, torch autograd of a dense kl_div formulation), a closed form, an
invariant of the mathematics, or finite differences.  ``test_mutants_are_caught``
plants mistakes in the oracle (on the CPU) and checks that the pins notice.
"""
import numpy as np
import pytest
import scipy.special
import scipy.stats
import torch
import torch.nn.functional as F

import oracle
from oracle import kl as okl


def _rand_case(seed, N=12, H=16, V=50, K=7, T=1.0, sigma=2.0, mask_frac=0.0, wscale=0.3):
    rng = np.random.default_rng(seed)
    h = rng.standard_normal((N, H))
    W = rng.standard_normal((V, H)) * wscale
    ids = np.stack([rng.choice(V, K, replace=False) for _ in range(N)]).astype(np.int32)
    lg = np.sort(rng.standard_normal((N, K)) * sigma, axis=1)[:, ::-1].copy()
    mask = np.ones(N, np.uint8)
    nm = int(round(mask_frac * N))
    if nm:
        mask[rng.choice(N, nm, replace=False)] = 0
    return h, W, ids, lg, mask, T


def _run(f, case, **kw):
    h, W, ids, lg, mask, T = case
    return f(h, W, ids, lg, mask, T, **kw)


# ---------------------------------------------------------------- the pins
# Each pin takes the oracle callable so that planted mutants can be fed in.

def pin_cross_entropy_k1(f):
    """K = 1: p is one-hot, so the row loss is the cross-entropy -log q[id]."""
    h, W, ids, lg, mask, T = _rand_case(1, K=1, T=1.7)
    o = f(h, W, ids, lg, mask, T)
    Z = torch.from_numpy(h @ W.T)
    ce = F.cross_entropy(Z / T, torch.from_numpy(ids[:, 0].astype(np.int64)), reduction="none").numpy()
    np.testing.assert_allclose(o["row_loss"], ce, rtol=1e-12, atol=1e-13)


def pin_scipy_kl(f):
    """Row loss equals scipy's KL(p || q) of the dense teacher against the
    dense student softmax (the dense-KL correctness baseline)."""
    for seed, T in [(2, 1.0), (3, 0.6), (4, 3.0)]:
        h, W, ids, lg, mask, _ = _rand_case(seed, K=9, mask_frac=0.25)
        o = f(h, W, ids, lg, mask, T)
        q = scipy.special.softmax((h @ W.T) / T, axis=1)
        pk = scipy.special.softmax(lg / T, axis=1)
        for r in range(h.shape[0]):
            if not mask[r]:
                assert o["row_loss"][r] == 0.0
                continue
            pd = np.zeros(W.shape[0])
            pd[ids[r]] = pk[r]
            ref = scipy.stats.entropy(pd, q[r])
            ref2 = scipy.special.rel_entr(pd, q[r]).sum()
            np.testing.assert_allclose(o["row_loss"][r], ref, rtol=1e-11, atol=1e-13)
            np.testing.assert_allclose(o["row_loss"][r], ref2, rtol=1e-11, atol=1e-13)
        np.testing.assert_allclose(o["loss"], o["row_loss"][mask != 0].mean(), rtol=1e-13)


def pin_k_equals_v_closed_form(f):
    """K = V: l = LSE_q - LSE_p + sum_v p_v (t_v - a_v), a different
    arithmetic path from the entry-wise sum."""
    N, H, V, T = 6, 10, 23, 1.3
    rng = np.random.default_rng(5)
    h = rng.standard_normal((N, H)); W = rng.standard_normal((V, H)) * 0.5
    ids = np.stack([rng.permutation(V) for _ in range(N)]).astype(np.int32)
    lg = rng.standard_normal((N, V)) * 2
    o = f(h, W, ids, lg, None, T)
    a = (h @ W.T) / T
    for r in range(N):
        t = lg[r] / T
        p = np.exp(t - scipy.special.logsumexp(t))
        ref = scipy.special.logsumexp(a[r]) - scipy.special.logsumexp(t) + np.sum(p * (t - a[r, ids[r]]))
        np.testing.assert_allclose(o["row_loss"][r], ref, rtol=1e-12, atol=1e-12)


def pin_zero_when_equal(f):
    """K = V and teacher logits equal to the student's: loss 0, gradients 0."""
    N, H, V, T = 5, 8, 17, 2.5
    rng = np.random.default_rng(6)
    h = rng.standard_normal((N, H)); W = rng.standard_normal((V, H))
    ids = np.stack([rng.permutation(V) for _ in range(N)]).astype(np.int32)
    Z = h @ W.T
    lg = np.take_along_axis(Z, ids.astype(np.int64), axis=1)
    o = f(h, W, ids, lg, None, T)
    assert abs(o["loss"]) < 1e-13
    assert np.abs(o["dH"]).max() < 1e-13 and np.abs(o["dW"]).max() < 1e-13


def pin_gibbs_bound(f):
    """0 <= -log sum_k q[id_k] <= l_r (Gibbs' inequality on the top-K set)."""
    for seed in range(3):
        h, W, ids, lg, mask, T = _rand_case(10 + seed, K=4, wscale=1.0)
        o = f(h, W, ids, lg, mask, T)
        q = scipy.special.softmax((h @ W.T) / T, axis=1)
        lower = -np.log(np.take_along_axis(q, ids.astype(np.int64), axis=1).sum(axis=1))
        assert (lower >= 0).all()
        assert (o["row_loss"] >= lower - 1e-12).all()


def pin_dlogits_sum_zero(f):
    """sum_v dlogits_r = 0, so the columns of dW sum to 0, and dH does not
    change when one row vector is added to every row of W."""
    case = _rand_case(20, mask_frac=0.2)
    h, W, ids, lg, mask, T = case
    o = f(*case)
    scale = np.abs(o["dW"]).max()
    assert np.abs(o["dW"].sum(axis=0)).max() < 1e-12 * max(1.0, scale) * W.shape[0]
    c = np.random.default_rng(21).standard_normal(W.shape[1])
    o2 = f(h, W + c[None, :], ids, lg, mask, T)
    np.testing.assert_allclose(o2["dH"], o["dH"], rtol=1e-9, atol=1e-12)


def pin_invariances(f):
    """Teacher-logit shift per row; (T, W, logits) == (1, W/T, logits/T);
    randomising masked rows changes nothing."""
    case = _rand_case(30, mask_frac=0.3, T=2.0)
    h, W, ids, lg, mask, T = case
    o = f(*case)
    shift = np.random.default_rng(31).standard_normal((h.shape[0], 1)) * 5
    o_s = f(h, W, ids, lg + shift, mask, T)
    np.testing.assert_allclose(o_s["row_loss"], o["row_loss"], rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(o_s["dW"], o["dW"], rtol=1e-9, atol=1e-14)
    o1 = f(h, W / T, ids, lg / T, mask, 1.0)
    np.testing.assert_allclose(o1["loss"], o["loss"], rtol=1e-12)
    np.testing.assert_allclose(o1["dH"], o["dH"], rtol=1e-10, atol=1e-14)
    np.testing.assert_allclose(o1["dW"] / T, o["dW"], rtol=1e-10, atol=1e-14)
    rng = np.random.default_rng(32)
    h2, ids2, lg2 = h.copy(), ids.copy(), lg.copy()
    m = mask == 0
    h2[m] = rng.standard_normal(h2[m].shape) * 10
    lg2[m] = rng.standard_normal(lg2[m].shape) * 10
    ids2[m] = rng.integers(0, W.shape[0], ids2[m].shape)
    o_m = f(h2, W, ids2, lg2, mask, T)
    np.testing.assert_allclose(o_m["loss"], o["loss"], rtol=1e-13)
    np.testing.assert_allclose(o_m["dW"], o["dW"], rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(o_m["dH"], o["dH"], rtol=1e-12, atol=1e-15)
    assert np.abs(o_m["dH"][m]).max() == 0.0


def pin_uniform_teacher(f):
    """All K teacher logits equal: l = -log K - (1/K) sum_k log q[id_k]."""
    h, W, ids, lg, mask, T = _rand_case(40, K=6, T=0.8)
    lg = np.full_like(lg, 1.234)
    o = f(h, W, ids, lg, mask, T)
    logq = scipy.special.log_softmax((h @ W.T) / T, axis=1)
    ref = -np.log(6) - np.take_along_axis(logq, ids.astype(np.int64), axis=1).mean(axis=1)
    np.testing.assert_allclose(o["row_loss"], ref, rtol=1e-12, atol=1e-13)


def pin_autograd_kl_div(f):
    """Loss and gradients equal torch autograd (fp64, CPU) of the dense
    formulation built from library ops: kl_div(log_softmax(h W^T / T), p~)."""
    for seed, T in [(50, 1.0), (51, 2.0), (52, 0.7)]:
        h, W, ids, lg, mask, _ = _rand_case(seed, N=9, H=11, V=31, K=5, mask_frac=0.3)
        o = f(h, W, ids, lg, mask, T)
        th = torch.tensor(h, requires_grad=True)
        tW = torch.tensor(W, requires_grad=True)
        logq = F.log_softmax(th @ tW.T / T, dim=1)
        pk = torch.softmax(torch.tensor(lg) / T, dim=1)
        pd = torch.zeros(h.shape[0], W.shape[0], dtype=torch.float64)
        pd.scatter_add_(1, torch.tensor(ids.astype(np.int64)), pk)
        keep = torch.tensor(mask != 0)
        loss = F.kl_div(logq[keep], pd[keep], reduction="sum") / keep.sum()
        loss.backward()
        np.testing.assert_allclose(o["loss"], loss.item(), rtol=1e-12)
        np.testing.assert_allclose(o["dH"], th.grad.numpy(), rtol=1e-9, atol=1e-14)
        np.testing.assert_allclose(o["dW"], tW.grad.numpy(), rtol=1e-9, atol=1e-14)


def pin_finite_differences(f):
    """Central finite differences of the loss w.r.t. every entry of h and W."""
    h, W, ids, lg, mask, T = _rand_case(60, N=6, H=8, V=40, K=5, T=1.5, mask_frac=0.17)
    o = f(h, W, ids, lg, mask, T)
    eps = 1e-6

    def L(hh, WW):
        return f(hh, WW, ids, lg, mask, T)["loss"]

    num_h = np.zeros_like(h)
    for i in np.ndindex(*h.shape):
        hp = h.copy(); hp[i] += eps
        hm = h.copy(); hm[i] -= eps
        num_h[i] = (L(hp, W) - L(hm, W)) / (2 * eps)
    num_W = np.zeros_like(W)
    for i in np.ndindex(*W.shape):
        Wp = W.copy(); Wp[i] += eps
        Wm = W.copy(); Wm[i] -= eps
        num_W[i] = (L(h, Wp) - L(h, Wm)) / (2 * eps)
    def rel(a, b):
        return np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300)
    assert rel(o["dH"], num_h) < 1e-6
    assert rel(o["dW"], num_W) < 1e-6


def pin_row_block_invariance(f):
    """Chunking rows differently does not change the result ("lossless")."""
    case = _rand_case(70, N=37, mask_frac=0.1)
    ref = _run(f, case, row_block=1000)
    for rb in (1, 7, 16):
        o = _run(f, case, row_block=rb)
        np.testing.assert_allclose(o["loss"], ref["loss"], rtol=1e-13)
        np.testing.assert_allclose(o["dH"], ref["dH"], rtol=1e-12, atol=1e-16)
        np.testing.assert_allclose(o["dW"], ref["dW"], rtol=1e-12, atol=1e-16)


PINS = [pin_cross_entropy_k1, pin_scipy_kl, pin_k_equals_v_closed_form, pin_zero_when_equal,
        pin_gibbs_bound, pin_dlogits_sum_zero, pin_invariances, pin_uniform_teacher,
        pin_autograd_kl_div, pin_finite_differences, pin_row_block_invariance]


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_pin(pin):
    pin(oracle.fused_chunked_kl)


# ------------------------------------------------------ edge-case readings

def test_neg_inf_teacher_logit_is_zero_probability():
    """A -inf teacher logit gives p = 0: identical to dropping that entry."""
    h, W, ids, lg, mask, T = _rand_case(80, K=6)
    lg2 = lg.copy(); lg2[:, -2:] = -np.inf
    o = oracle.fused_chunked_kl(h, W, ids, lg2, mask, T)
    o_ref = oracle.fused_chunked_kl(h, W, ids[:, :-2].copy(), lg[:, :-2].copy(), mask, T)
    np.testing.assert_allclose(o["row_loss"], o_ref["row_loss"], rtol=1e-13)
    np.testing.assert_allclose(o["dW"], o_ref["dW"], rtol=1e-12, atol=1e-16)


def test_no_valid_rows():
    h, W, ids, lg, mask, T = _rand_case(81)
    o = oracle.fused_chunked_kl(h, W, ids, lg, np.zeros_like(mask), T)
    assert o["loss"] == 0.0 and o["n_valid"] == 0
    assert not o["dH"].any() and not o["dW"].any()


def test_duplicate_ids_add_into_one_dense_cell():
    """Repeated ids: the teacher is the dense grid p~ (entries of one id add up)
    and the loss is KL(p~ || q); checked against scipy's KL of the dense grid and
    autograd of kl_div on it."""
    h, W, ids, lg, mask, T = _rand_case(82, K=5)
    ids[:, 3] = ids[:, 1]
    o = oracle.fused_chunked_kl(h, W, ids, lg, mask, T)
    q = scipy.special.softmax((h @ W.T) / T, axis=1)
    pk = scipy.special.softmax(lg / T, axis=1)
    for r in range(h.shape[0]):
        pd = np.zeros(W.shape[0])
        np.add.at(pd, ids[r], pk[r])
        np.testing.assert_allclose(o["row_loss"][r], scipy.stats.entropy(pd, q[r]), rtol=1e-11)
    th = torch.tensor(h, requires_grad=True); tW = torch.tensor(W, requires_grad=True)
    logq = F.log_softmax(th @ tW.T / T, dim=1)
    pd = torch.zeros(h.shape[0], W.shape[0], dtype=torch.float64)
    pd.scatter_add_(1, torch.tensor(ids.astype(np.int64)), torch.softmax(torch.tensor(lg) / T, 1))
    loss = F.kl_div(logq, pd, reduction="sum") / h.shape[0]
    loss.backward()
    np.testing.assert_allclose(o["loss"], loss.item(), rtol=1e-12)
    np.testing.assert_allclose(o["dW"], tW.grad.numpy(), rtol=1e-9, atol=1e-15)


def test_probs_teacher_matches_scipy_and_autograd():
    """Teacher given as sampled class weights (RS-KD): p = w / sum(w), repeats
    allowed (sampling with replacement), temperature on the student only."""
    rng = np.random.default_rng(90)
    h, W, _, _, mask, _ = _rand_case(91, N=10, V=40, mask_frac=0.2)
    K, T = 12, 1.7
    ids = rng.integers(0, 40, (10, K)).astype(np.int32)          # repeats are likely
    w = rng.random((10, K)) * (rng.random((10, K)) < 0.8)        # some zero weights
    w[:, 0] += 0.1
    o = oracle.fused_chunked_kl(h, W, ids, w, mask, T, teacher="probs")
    q = scipy.special.softmax((h @ W.T) / T, axis=1)
    for r in range(10):
        if not mask[r]:
            continue
        pd = np.zeros(40)
        np.add.at(pd, ids[r], w[r] / w[r].sum())
        np.testing.assert_allclose(o["row_loss"][r], scipy.stats.entropy(pd, q[r]), rtol=1e-11)
    th = torch.tensor(h, requires_grad=True); tW = torch.tensor(W, requires_grad=True)
    logq = F.log_softmax(th @ tW.T / T, dim=1)
    pd = torch.zeros(10, 40, dtype=torch.float64)
    pd.scatter_add_(1, torch.tensor(ids.astype(np.int64)), torch.tensor(w / w.sum(1, keepdims=True)))
    keep = torch.tensor(mask != 0)
    loss = F.kl_div(logq[keep], pd[keep], reduction="sum") / keep.sum()
    loss.backward()
    np.testing.assert_allclose(o["loss"], loss.item(), rtol=1e-12)
    np.testing.assert_allclose(o["dH"], th.grad.numpy(), rtol=1e-9, atol=1e-15)
    np.testing.assert_allclose(o["dW"], tW.grad.numpy(), rtol=1e-9, atol=1e-15)
    # scaling the weights of a row changes nothing
    o2 = oracle.fused_chunked_kl(h, W, ids, w * 3.5, mask, T, teacher="probs")
    np.testing.assert_allclose(o2["row_loss"], o["row_loss"], rtol=1e-12)


def test_row_subset_matches_full():
    """Evaluating a subset of rows gives those rows' values from the full run."""
    case = _rand_case(83, N=20, mask_frac=0.25)
    full = _run(oracle.fused_chunked_kl, case)
    rows = np.array([0, 3, 4, 11, 19])
    sub = _run(oracle.fused_chunked_kl, case, rows=rows)
    np.testing.assert_array_equal(sub["rows"], rows[case[4][rows] != 0])
    np.testing.assert_allclose(sub["row_loss_rows"], full["row_loss"][sub["rows"]], rtol=1e-14)
    np.testing.assert_allclose(sub["dH_rows"], full["dH"][sub["rows"]], rtol=1e-13, atol=1e-18)


def test_bf16_widening_exact():
    from synth import f32_to_bf16_bits, bf16_bits_to_f32
    x = np.array([1.0, -2.5, 3.140625, 1e-3, 65504.0, 1.00390625, 1.01171875], np.float32)
    b = f32_to_bf16_bits(x)
    back = okl.widen_bf16(b)
    assert back.dtype == np.float64
    np.testing.assert_array_equal(back, bf16_bits_to_f32(b).astype(np.float64))
    # round-to-nearest-even at the halfway points 1 + 2^-8 and 1 + 3 * 2^-8
    assert back[5] == 1.0 and back[6] == 1.015625


# ---------------------------------------------------------------- mutants

def _mutant(kind):
    """Return a copy of the oracle with one planted mistake."""
    def f(h, W, ids, lg, mask, T, **kw):
        saved = (okl.student_log_probs, okl.teacher_distribution, okl.dense_teacher)
        try:
            if kind == "student_no_T":
                okl.student_log_probs = lambda Z, T_: saved[0](Z, 1.0)
            elif kind == "teacher_no_T":
                okl.teacher_distribution = lambda lg_, T_, *a: saved[1](lg_, 1.0, *a)
            elif kind == "q_over_topk_only":
                # normalising the student only over a prefix of the vocabulary
                okl.student_log_probs = lambda Z, T_: okl.log_softmax(
                    np.where(np.arange(Z.shape[1])[None, :] < Z.shape[1] - 3, Z / T_, -np.inf), axis=1)
            elif kind == "p_sign":
                okl.dense_teacher = lambda p, i, V: -saved[2](p, i, V)
            elif kind == "id_off_by_one":
                ids = (ids + 1) % W.shape[0]
            elif kind == "reverse_kl_weights":
                okl.teacher_distribution = lambda lg_, T_, *a: (
                    lambda pl: (np.full_like(pl[0], 1.0 / pl[0].shape[1]), pl[1]))(saved[1](lg_, T_, *a))
            return okl.fused_chunked_kl(h, W, ids, lg, mask, T, **kw)
        finally:
            okl.student_log_probs, okl.teacher_distribution, okl.dense_teacher = saved
    return f


@pytest.mark.parametrize("kind", ["student_no_T", "teacher_no_T", "q_over_topk_only", "p_sign",
                                  "id_off_by_one", "reverse_kl_weights"])
def test_mutants_are_caught(kind):
    f = _mutant(kind)
    caught = []
    for pin in PINS:
        if pin is pin_finite_differences:
            continue
        try:
            pin(f)
        except AssertionError:
            caught.append(pin.__name__)
    assert caught, f"planted mistake {kind!r} passed every pin"
