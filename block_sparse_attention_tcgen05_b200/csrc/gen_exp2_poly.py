"""Fits the polynomial the attention kernel uses for part of its exponentials.

Method: Cody–Waite style range reduction x = j + f with j = round(x) (obtained by
adding 1.5·2^23 in float32) and f in [-1/2, 1/2], then 2^f by a degree-3 polynomial
whose coefficients minimise the maximum relative error on [-1/2, 1/2] (Remez exchange
on the relative error), and 2^j applied by adding j to the float32 exponent field.

Run it to print the coefficients embedded in attention.cu and the error bound of the
float32 evaluation. The tests re-run `fit()` and check the embedded constants.
"""

import numpy as np

DEGREE = 3
LO, HI = -0.5, 0.5


def _solve_levelled(nodes):
    """Coefficients c and level e with (p(x) - 2^x) / 2^x = (-1)^i e at the nodes."""
    n = DEGREE + 2
    A = np.zeros((n, n))
    rhs = np.exp2(nodes)
    for i, x in enumerate(nodes):
        A[i, :DEGREE + 1] = x ** np.arange(DEGREE + 1)
        A[i, DEGREE + 1] = -((-1) ** i) * np.exp2(x)
    sol = np.linalg.solve(A, rhs)
    return sol[:DEGREE + 1], sol[DEGREE + 1]


def _rel_err(c, x):
    return np.polyval(c[::-1], x) / np.exp2(x) - 1.0


def fit(iterations=30):
    """Remez exchange for the minimax relative error; returns (coefficients c0..c3,
    max relative error of the exact-arithmetic polynomial)."""
    k = np.arange(DEGREE + 2)
    nodes = 0.5 * (LO + HI) + 0.5 * (HI - LO) * np.cos(np.pi * k[::-1] / (DEGREE + 1))
    grid = np.linspace(LO, HI, 20001)
    c = None
    for _ in range(iterations):
        c, _ = _solve_levelled(nodes)
        e = _rel_err(c, grid)
        # new reference: the extremum of each sign-alternating run of the error
        sgn = np.sign(e)
        runs = np.split(np.arange(len(grid)), np.nonzero(np.diff(sgn))[0] + 1)
        ext = [r[np.argmax(np.abs(e[r]))] for r in runs if len(r)]
        if len(ext) < DEGREE + 2:
            break
        if len(ext) > DEGREE + 2:  # keep the largest alternating set
            ext = sorted(ext, key=lambda i: -abs(e[i]))[:DEGREE + 2]
            ext.sort()
        nodes = grid[np.array(ext)]
    return c, float(np.abs(_rel_err(c, grid)).max())


def emulate_float32(x, c):
    """The kernel's evaluation in float32: clamp, shifter rounding, Horner, exponent add."""
    x = np.maximum(np.asarray(x, dtype=np.float32), np.float32(-126.0))
    shifter = np.float32(12582912.0)  # 1.5 * 2^23
    t = (x + shifter).astype(np.float32)
    r = (t - shifter).astype(np.float32)
    f = (x - r).astype(np.float32)
    cf = [np.float32(v) for v in c]
    p = np.float32(cf[3])
    for ci in (cf[2], cf[1], cf[0]):
        p = (p * f + ci).astype(np.float32)  # fma rounding differs by at most 1 ulp
    bits = p.view(np.int32) + (t.view(np.int32) << 23)
    return bits.astype(np.int32).view(np.float32)


if __name__ == "__main__":
    c, err = fit()
    print("coefficients c0..c3:", ", ".join(f"{v:.9e}f" for v in np.float32(c)))
    print(f"max relative error on [-1/2, 1/2] (exact arithmetic): {err:.3e}")
    xs = np.linspace(-126.0, 8.0, 200001, dtype=np.float32)
    got = emulate_float32(xs, np.float32(c)).astype(np.float64)
    print(f"max relative error of the float32 evaluation on [-126, 8]: "
          f"{np.abs(got / np.exp2(xs.astype(np.float64)) - 1).max():.3e}")
