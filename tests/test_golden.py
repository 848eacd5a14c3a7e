"""The oracle reproduces its stored output on the small seeded case."""
import json
import os

import numpy as np

import oracle
import synth

GOLD = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "oracle_small.json")


def test_oracle_matches_stored_small_case():
    with open(GOLD) as fh:
        g = json.load(fh)
    inp = synth.make_custom(**g["case"])
    o = oracle.oracle_from_inputs(inp)
    assert o["n_valid"] == g["n_valid"]
    np.testing.assert_allclose(o["loss"], g["loss"], rtol=1e-13)
    np.testing.assert_allclose(o["row_loss"], np.array(g["row_loss"]), rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(o["dH"], np.array(g["dH"]), rtol=1e-11, atol=1e-17)
    np.testing.assert_allclose(o["dW"], np.array(g["dW"]), rtol=1e-11, atol=1e-17)


def test_synth_recipe_is_stable():
    """The seeded generator is part of the parity contract: same seed, same bits."""
    a = synth.make_custom(N=33, H=24, V=300, K=10, T=1.0, mask_frac=0.1, seed=7)
    b = synth.make_custom(N=33, H=24, V=300, K=10, T=1.0, mask_frac=0.1, seed=7)
    for x, y in [(a.hidden, b.hidden), (a.W, b.W), (a.topk_idx, b.topk_idx),
                 (a.topk_logit, b.topk_logit), (a.row_mask, b.row_mask)]:
        np.testing.assert_array_equal(x, y)
    assert int((a.row_mask == 0).sum()) == 3
    s = np.sort(a.topk_idx, axis=1)
    assert (s[:, 1:] != s[:, :-1]).all() and a.topk_idx.min() >= 0 and a.topk_idx.max() < 300
    assert (np.diff(a.topk_logit, axis=1) <= 0).all()
