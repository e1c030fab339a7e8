"""Reference for the profiling-guided speculation budget (plain numpy).

TEST INFRASTRUCTURE ONLY, like the rest of this package.  PRR (abstract) sizes its
speculation from profiling so that speculative work stays off the critical path; its
limitations list says overheads at context lengths off the profiled grid (between or
beyond its points) come from polynomial regressions.  Reference definitions:
  fit:    least-squares polynomial of the measured times in x = context / 65536
          (numpy's lstsq on the Vandermonde matrix), coefficients lowest order first;
  choose: the largest profiled budget whose predicted speculation time is at most the
          predicted selection time at the given context, else 0.
"""
from __future__ import annotations

import numpy as np

UNIT = 65536.0


def fit(context_tokens, us, degree: int) -> np.ndarray:
    x = np.asarray(context_tokens, np.float64) / UNIT
    v = np.vander(x, degree + 1, increasing=True)
    coef, *_ = np.linalg.lstsq(v, np.asarray(us, np.float64), rcond=None)
    return coef


def evaluate(coef, context_tokens) -> np.ndarray:
    x = np.asarray(context_tokens, np.float64) / UNIT
    return np.polynomial.polynomial.polyval(x, np.asarray(coef, np.float64))


def choose(sel_coef, spec_coef, p_grid, context_tokens: int) -> int:
    sel = evaluate(sel_coef, context_tokens)
    best = 0
    for p, c in zip(p_grid, spec_coef):
        if evaluate(c, context_tokens) <= sel:
            best = int(p)
    return best
