"""Write ema_rounding.json: an EMA trajectory whose exact rounding is fixed.

The predictor's update is e <- alpha*e + beta*[b in S] with beta = 1 - alpha, each
multiply and the add rounded to the nearest double (no fused multiply-add).  This
script derives the trajectory with exact rational arithmetic (fractions.Fraction,
rounded to the nearest double by CPython's correctly rounded int/int division), so the
stored values depend on no floating-point unit and no compiler flag.  It also records
the trajectory a contracted update fma(alpha, e, beta*ind) would give, and the first
step where the two differ, to show the fixture tells them apart.

Run from the repository root:  python tests/golden/make_ema_rounding.py
"""
import json
import os
from fractions import Fraction as F

ALPHA = 0.9
STEPS = 6


def rn(x: F) -> float:
    """Round an exact rational to the nearest double (ties to even)."""
    return x.numerator / x.denominator


def main():
    beta = rn(F(1) - F(ALPHA))
    # block 0 is selected at steps where t % 3 != 2, block 1 never
    sel = [[0] if t % 3 != 2 else [] for t in range(STEPS)]
    sep, fused = [], []
    e_s = e_f = 0.0
    for s in sel:
        ind = 1.0 if 0 in s else 0.0
        added = rn(F(beta) * F(ind))
        e_s = rn(F(rn(F(ALPHA) * F(e_s))) + F(added))   # two roundings
        e_f = rn(F(ALPHA) * F(e_f) + F(added))           # one rounding (contracted)
        sep.append(e_s)
        fused.append(e_f)
    first = next(i for i, (a, b) in enumerate(zip(sep, fused)) if a != b)
    doc = {
        "_about": "EMA predictor update rounding (PRR abstract: an exponential moving average of past "
                  "selections).  Each step rounds alpha*e and beta*ind to the nearest double, then rounds "
                  "their sum; values derived with exact rationals by make_ema_rounding.py.",
        "alpha": ALPHA, "beta_hex": beta.hex(), "nb": 2, "selections": sel,
        "e_block0_hex": [x.hex() for x in sep],
        "contracted_block0_hex": [x.hex() for x in fused],
        "first_step_where_contraction_differs": first,
    }
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "ema_rounding.json")
    with open(path, "w") as fh:
        json.dump(doc, fh, indent=1)
        fh.write("\n")
    print(path, "first difference at step", first)


if __name__ == "__main__":
    main()
