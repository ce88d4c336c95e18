"""Writes tests/golden/gdn_tiny_exact.json with the exact rational oracle.

Calls only ``oracle.exact_tiny``.  The pages print no worked numeric example of
the gated delta rule, so this fixture is an exact evaluation of the page's
expanded one-step form (page "ARCHITECTURE PREVIEW / FIELD NOTES", section 03)
on hand-picked rational inputs: unit keys and queries with rational entries
(3/5, 4/5), (5/13, 12/13), ... so that L2 normalisation leaves them unchanged.
Run:  python tests/golden/make_golden.py
"""
import json
import os
import sys
from fractions import Fraction as F

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__)))))
from oracle.exact_tiny import one_step_exact  # noqa: E402

CASE = {
    "S0": [[F(1, 2), F(-1, 3), F(0)], [F(1, 4), F(2, 5), F(-1)]],          # dk=2, dv=3
    "k": [[F(3, 5), F(4, 5)], [F(1), F(0)], [F(5, 13), F(12, 13)], [F(-4, 5), F(3, 5)],
          [F(3, 5), F(4, 5)]],
    "v": [[F(1), F(-2), F(1, 2)], [F(0), F(3, 4), F(-1)], [F(2), F(1), F(1)],
          [F(-1, 2), F(1, 3), F(5, 4)], [F(1), F(-2), F(1, 2)]],
    "q": [[F(0), F(1)], [F(8, 17), F(15, 17)], [F(3, 5), F(-4, 5)], [F(1), F(0)],
          [F(3, 5), F(4, 5)]],
    "alpha": [F(1, 2), F(3, 4), F(9, 10), F(1), F(1)],
    "beta": [F(1, 4), F(1, 2), F(1), F(3, 5), F(1)],
}


def _s(x):
    return f"{x.numerator}/{x.denominator}"


def main():
    ys, S = one_step_exact(CASE["S0"], CASE["k"], CASE["v"], CASE["q"], CASE["alpha"],
                           CASE["beta"])
    doc = {
        "source": "exact rational evaluation of the expanded one-step recurrence, page "
                  "'ARCHITECTURE PREVIEW / FIELD NOTES' section 03 (GATED DELTANET)",
        "layout": "S[d_k][d_v]; k,q: T x d_k; v, y: T x d_v",
        "inputs": {key: ([[_s(x) for x in row] for row in val] if isinstance(val[0], list)
                         else [_s(x) for x in val]) for key, val in CASE.items()},
        "y": [[_s(x) for x in row] for row in ys],
        "S_T": [[_s(x) for x in row] for row in S],
    }
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "gdn_tiny_exact.json")
    with open(path, "w") as f:
        json.dump(doc, f, indent=1)
    print("wrote", path)


if __name__ == "__main__":
    main()
