"""Fit the polynomial behind the kernels' division-free log1p (build-time helper).

softplus needs log(1 + e) for e = exp(-|v|) in (0, 1]. The kernels evaluate it
as e * Q(e), with Q(e) ~ log(1 + e) / e a polynomial whose maximum RELATIVE
error on [0, 1] is minimised by the Remez exchange algorithm (equioscillation
at deg + 2 points). log(1 + e) is analytic on a disc of radius 1 around 0, so
the minimax error falls geometrically with the degree. The fit runs in float64;
the coefficients are rounded to float32 and the float32 FMA-Horner evaluation
is checked on a dense grid. Run it to regenerate the constants in
ssm_math.cuh:  python fit_log1p_poly.py [DEG]
"""
import sys

import numpy as np

LO, HI = 0.0, 1.0


def target(x):
    out = np.ones_like(x)
    nz = x > 0
    out[nz] = np.log1p(x[nz]) / x[nz]
    return out


def remez(deg, iters=40):
    n = deg + 2
    x = 0.5 * (LO + HI) + 0.5 * (HI - LO) * np.cos(np.pi * np.arange(n)[::-1] / (n - 1))
    grid = np.linspace(LO, HI, 400001)
    for _ in range(iters):
        # p(x_i) - Q(x_i) = (-1)^i E Q(x_i)  (relative error equioscillates)
        A = np.zeros((n, n))
        for k in range(deg + 1):
            A[:, k] = x ** k
        A[:, deg + 1] = -((-1.0) ** np.arange(n)) * target(x)
        sol = np.linalg.solve(A, target(x))
        c = sol[: deg + 1]
        err = np.polyval(c[::-1], grid) / target(grid) - 1.0
        idx = np.where(np.diff(np.sign(err)) != 0)[0]
        bounds = np.concatenate([[0], idx + 1, [len(grid)]])
        ext = [b0 + np.argmax(np.abs(err[b0:b1])) for b0, b1 in zip(bounds[:-1], bounds[1:]) if b1 > b0]
        if len(ext) != n:
            break
        x = grid[ext]
    return c


def fma32(a, b, c):
    """float32 fused multiply-add: the float64 product of two float32 is exact."""
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


def check_f32(c):
    c32 = c.astype(np.float32)
    e = np.linspace(LO, HI, 2000001).astype(np.float32)
    p = np.full_like(e, c32[-1])
    for k in range(len(c32) - 2, -1, -1):
        p = fma32(p, e, np.full_like(e, c32[k]))
    y = (p.astype(np.float64) * e.astype(np.float64)).astype(np.float32)  # e * Q(e), one rounding
    ref = np.log1p(e.astype(np.float64))
    nz = ref > 0
    rel = np.abs(y[nz].astype(np.float64) / ref[nz] - 1.0)
    return c32, rel.max()


if __name__ == "__main__":
    degs = [int(a) for a in sys.argv[1:]] or [8, 9, 10, 11]
    for deg in degs:
        c = remez(deg)
        c32, err = check_f32(c)
        print(f"degree {deg}: max rel error (float32 FMA Horner) {err:.3e}")
        print("  coefficients c0..c%d:" % deg, ", ".join(f"{v:.9e}" for v in c32))
