"""Coefficients of the exp2 polynomial that the attention contract uses.

TEST INFRASTRUCTURE ONLY (part of the CPU oracle; it writes no stored value).

2^f on f in [-1/2, 1/2] is approximated by p(f) = 1 + c1 f + ... + c_d f^d with
c0 fixed at 1 (so that 2^n is exact at integers): a quadratic (d = 2) for
the per-key weights and a quintic (d = 5) for the once-per-tile rescale factor.
c1..c_d minimise the maximum
relative error |p(f) / 2^f - 1| on a dense grid, as a linear program
(minimise t subject to -t <= p(f_i) / 2^f_i - 1 <= t), and are then rounded to
binary32.  Running this file prints the rounded coefficients and the maximum
relative error of the binary32 Horner evaluation (fused multiply-adds), which
the oracle's constants and pins restate.

    python oracle/fit_exp2.py
"""
from __future__ import annotations

import numpy as np
from scipy.optimize import linprog

DEGREES = (2, 5)


def fit(degree: int, points: int = 4001) -> np.ndarray:
    f = np.linspace(-0.5, 0.5, points)
    w = np.exp2(-f)                                   # relative error weight
    # variables: c1..c_degree, t
    A_f = np.stack([f ** k * w for k in range(1, degree + 1)], axis=1)
    base = w - 1.0                                    # the c0 = 1 term, moved right
    ones = np.ones((points, 1))
    A_ub = np.vstack([np.hstack([A_f, -ones]), np.hstack([-A_f, -ones])])
    b_ub = np.concatenate([-base, base])
    cost = np.zeros(degree + 1)
    cost[-1] = 1.0
    res = linprog(cost, A_ub=A_ub, b_ub=b_ub, bounds=[(None, None)] * (degree + 1), method="highs")
    if not res.success:
        raise RuntimeError(res.message)
    return np.concatenate([[1.0], res.x[:degree]]).astype(np.float32)


def main() -> None:
    import os
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    from oracle.numerics import fma32

    for degree in DEGREES:
        c = fit(degree)
        f = np.linspace(-0.5, 0.5, 200001).astype(np.float32)
        p = np.full_like(f, c[-1])
        for k in range(len(c) - 2, -1, -1):
            p = fma32(p, f, np.float32(c[k]))
        err = np.abs(p.astype(np.float64) / np.exp2(f.astype(np.float64)) - 1).max()
        print(f"degree {degree}:")
        for k, v in enumerate(c):
            print(f"  c{k} = {float(v)!r}  ({np.float32(v).view(np.uint32):#010x})")
        print(f"  max relative error of the binary32 evaluation: {err:.3e}")


if __name__ == "__main__":
    main()
