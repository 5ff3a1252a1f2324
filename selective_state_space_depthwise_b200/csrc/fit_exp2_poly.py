"""Fit the polynomial behind the kernels' FMA-pipe exp2 (build-time helper).

2^x = 2^n * 2^f with n = round(x), f in [-1/2, 1/2]; 2^f is approximated by a
degree-5 polynomial whose maximum RELATIVE error on [-1/2, 1/2] is minimised
by the Remez exchange algorithm (equioscillation at 7 points). The fit runs in
float64; the coefficients are then rounded to float32 and the float32 Horner
evaluation is checked on a dense grid. Run it to regenerate the constants in
ssm_math.cuh:  python fit_exp2_poly.py
"""
import numpy as np

DEG = 5
LO, HI = -0.5, 0.5


def remez(deg=DEG, iters=30):
    n = deg + 2
    x = 0.5 * (LO + HI) + 0.5 * (HI - LO) * np.cos(np.pi * np.arange(n)[::-1] / (n - 1))
    grid = np.linspace(LO, HI, 200001)
    for _ in range(iters):
        # p(x_i) - 2^x_i = (-1)^i E 2^x_i  ->  sum_k c_k x_i^k - (-1)^i E 2^x_i = 2^x_i
        A = np.zeros((n, n))
        for k in range(deg + 1):
            A[:, k] = x ** k
        A[:, deg + 1] = -((-1.0) ** np.arange(n)) * 2.0 ** x
        sol = np.linalg.solve(A, 2.0 ** x)
        c = sol[: deg + 1]
        err = np.polyval(c[::-1], grid) / 2.0 ** grid - 1.0
        # new reference: extrema of err between sign changes
        idx = np.where(np.diff(np.sign(err)) != 0)[0]
        bounds = np.concatenate([[0], idx + 1, [len(grid)]])
        ext = [b0 + np.argmax(np.abs(err[b0:b1])) for b0, b1 in zip(bounds[:-1], bounds[1:]) if b1 > b0]
        if len(ext) != n:
            break
        x = grid[ext]
    return c


def check_f32(c):
    c32 = c.astype(np.float32)
    f = np.linspace(LO, HI, 2000001).astype(np.float32)
    p = np.full_like(f, c32[-1])
    for k in range(DEG - 1, -1, -1):
        p = (p * f + c32[k]).astype(np.float32)  # fp32 Horner (fma-free bound)
    rel = np.abs(p.astype(np.float64) / 2.0 ** f.astype(np.float64) - 1.0)
    return c32, rel.max()


if __name__ == "__main__":
    c = remez()
    c32, e = check_f32(c)
    print("coefficients c0..c5 (float32):")
    for k, v in enumerate(c32):
        print(f"  c{k} = {float(v):.9e}f  ({np.float32(v).view(np.uint32):#010x})")
    print(f"max relative error of the float32 evaluation on [-1/2, 1/2]: {e:.3e}")
