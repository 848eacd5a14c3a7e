"""Seeded random small shapes against the fp64 oracle: hidden sizes that take
the 3-D operand maps (H % 64 == 0), the 2-D ones (H % 64 != 0) and the
half-width last tile (H % 256 <= 128); vocabularies with a padded last 64-column
chunk; explicit and automatic chunks; masks from none to most rows;
temperatures from 0.5 to 3; each draw once with one dW GEMM per chunk and once
with chunks grouped into one dW GEMM (dw_rows)."""
import numpy as np
import pytest

import oracle
import synth
from test_gpu_parity import check_full, run_gpu

pytestmark = pytest.mark.gpu


def _cases(n=24, seed=2024):
    rng = np.random.default_rng(seed)
    Hs = [8, 40, 64, 120, 128, 192, 256, 264, 320, 384, 448, 512, 576]
    out = []
    for i in range(n):
        N = int(rng.integers(1, 700))
        H = int(rng.choice(Hs))
        V = int(rng.integers(16, 2600))
        K = int(rng.integers(1, min(64, V) + 1))
        chunk = int(rng.choice([0, 0, 64, 96, 128, 200, 256, 512]))
        mask = float(rng.choice([0.0, 0.0, 0.1, 0.5, 0.9]))
        T = float(rng.choice([0.5, 1.0, 1.0, 2.0, 3.0]))
        out.append((i, N, H, V, K, chunk, mask, T))
    # the same draws again with chunks grouped into one dW GEMM (dw_rows)
    for j, c in enumerate(list(out)):
        out.append((n + j,) + c[1:] + (int(rng.choice([64, 300, 4096])),))
    return [c if len(c) == 9 else c + (0,) for c in out]


@pytest.mark.parametrize("case", _cases(),
                         ids=lambda c: "N%d_H%d_V%d_K%d_c%d_m%.1f" % c[1:7] + "_g%d" % c[8])
def test_random_shape_matches_oracle(case):
    i, N, H, V, K, chunk, mask, T, dw_rows = case
    inp = synth.make_custom(N, H, V, K, T=T, sigma=2.0, mask_frac=mask, seed=500 + i % 24,
                            chunk=chunk)
    o = oracle.oracle_from_inputs(inp)
    g = run_gpu(inp, dw_rows=dw_rows)
    if o["n_valid"] == 0:
        assert g["loss"] == 0.0 and not g["dH"].any().item() and not g["dW"].any().item()
        return
    check_full(inp, g, o)
