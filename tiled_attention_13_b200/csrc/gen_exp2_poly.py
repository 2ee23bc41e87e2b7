"""Fit the polynomial used for 2^f on the FMA pipe (f in [-1/2, 1/2]).

    python tiled_attention_13_b200/csrc/gen_exp2_poly.py [degree]

Method: Remez exchange for the minimax *relative* error of a degree-n
polynomial p(f) ~= 2^f on [-1/2, 1/2] (Remez, 1934; any numerical-analysis
text).  The kernel reduces x = n + f with n = round(x) (adding and subtracting
1.5 * 2^23 rounds to the nearest integer in fp32), evaluates p(f) by Horner's
rule and adds n to the exponent field.  The coefficients are rounded to fp32
and the error is re-measured in fp32 arithmetic.  The printed constants are
the ones in ptx.cuh (exp2_poly_x2); tests/test_exp2_poly.py re-runs this fit
and checks them and their error bound.
"""

from __future__ import annotations

import sys

import numpy as np

LO, HI = -0.5, 0.5


def _solve(nodes: np.ndarray, deg: int) -> tuple[np.ndarray, float]:
    # p(x_i) + (-1)^i E 2^{x_i} = 2^{x_i}  (relative error equioscillates)
    n = len(nodes)
    A = np.zeros((n, deg + 2))
    for i, x in enumerate(nodes):
        A[i, : deg + 1] = [x ** k for k in range(deg + 1)]
        A[i, deg + 1] = (-1) ** i * 2.0 ** x
    sol = np.linalg.solve(A, 2.0 ** nodes)
    return sol[: deg + 1], sol[deg + 1]


def fit(deg: int = 3, iters: int = 30) -> np.ndarray:
    k = np.arange(deg + 2)
    nodes = 0.5 * (LO + HI) + 0.5 * (HI - LO) * np.cos(np.pi * (deg + 1 - k) / (deg + 1))
    grid = np.linspace(LO, HI, 20001)
    c = None
    for _ in range(iters):
        c, _e = _solve(nodes, deg)
        err = (np.polyval(c[::-1], grid) - 2.0 ** grid) / 2.0 ** grid
        # new nodes: extrema of the error in each sign-alternating segment
        sgn = np.sign(err)
        idx = [0] + [i for i in range(1, len(grid)) if sgn[i] != sgn[i - 1]] + [len(grid)]
        ext = []
        for a, b in zip(idx[:-1], idx[1:]):
            seg = np.abs(err[a:b])
            ext.append(grid[a + int(np.argmax(seg))])
        if len(ext) == deg + 2:
            nodes = np.array(ext)
        else:
            break
    return c


def fp32_error(c: np.ndarray) -> float:
    """Max relative error of Horner evaluation in fp32 on [-1/2, 1/2]."""
    cf = c.astype(np.float32)
    f = np.linspace(LO, HI, 200001).astype(np.float32)
    p = np.full_like(f, cf[-1])
    for a in cf[-2::-1]:
        p = (p * f + a).astype(np.float32)
    ref = 2.0 ** f.astype(np.float64)
    return float(np.max(np.abs(p.astype(np.float64) - ref) / ref))


def main() -> None:
    deg = int(sys.argv[1]) if len(sys.argv) > 1 else 3
    c = fit(deg)
    for i, a in enumerate(c.astype(np.float32)):
        print(f"c{i} = {float(a):.9e}f")
    print(f"max relative error in fp32: {fp32_error(c):.3e}")


if __name__ == "__main__":
    main()
