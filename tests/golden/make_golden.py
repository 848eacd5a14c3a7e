"""Writes tests/golden/oracle_small.json from the oracle alone.

The pages print no worked example with values, so the stored numbers are the
fp64 oracle's own output on a small seeded case.  They guard the oracle
against unintended changes: any later change to its arithmetic must be
justified by a passage of the pages (or a stated reading of one) and this
file regenerated with:  python tests/golden/make_golden.py
"""
import json
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import synth  # noqa: E402
import oracle  # noqa: E402

CASE = dict(N=6, H=16, V=40, K=4, T=1.5, sigma=2.0, mask_frac=0.34, seed=4242)


def main():
    inp = synth.make_custom(**CASE)
    o = oracle.oracle_from_inputs(inp)
    doc = {
        "what": "fp64 oracle output on synth.make_custom(**case); regression guard",
        "case": CASE,
        "n_valid": o["n_valid"],
        "loss": o["loss"],
        "row_loss": o["row_loss"].tolist(),
        "dH": o["dH"].tolist(),
        "dW": o["dW"].tolist(),
    }
    with open(os.path.join(HERE, "oracle_small.json"), "w") as fh:
        json.dump(doc, fh, indent=1)


if __name__ == "__main__":
    main()
