"""Fit the polynomial behind the kernels' FMA-pipe 2^x (``exp2_fma`` in
sm100_ptx.cuh) and print its coefficients and error.

Method: Cody-Waite style range reduction -- write x = j + f with j the
integer nearest x and f in [-1/2, 1/2], so that 2^x = 2^j * 2^f; 2^j is
formed by adding j to the exponent field, and 2^f is approximated by a
degree-3 polynomial c0 + c1 f + c2 f^2 + c3 f^3 chosen to minimise the
maximum *relative* error on [-1/2, 1/2] (Remez exchange on the relative error,
started from a least-squares fit on Chebyshev nodes).

The kernels round every weight to bf16 (8 significant bits, relative step
2^-8) before it enters a tensor-core product, so a relative error a few
hundred times smaller than that is invisible in the results.

Usage: python gen_exp2_poly.py
"""

import numpy as np

DEG = 3


def _fit_remez(deg: int, iters: int = 30):
    # initial reference: Chebyshev extrema on [-1/2, 1/2], deg + 2 points
    k = np.arange(deg + 2)
    xs = 0.5 * np.cos(np.pi * k / (deg + 1))[::-1]
    grid = np.linspace(-0.5, 0.5, 200001)
    coef = None
    for _ in range(iters):
        # solve p(x_i) - 2^x_i = (-1)^i E 2^x_i  (equioscillating relative error)
        A = np.zeros((deg + 2, deg + 2))
        for i, x in enumerate(xs):
            A[i, : deg + 1] = x ** np.arange(deg + 1)
            A[i, deg + 1] = -((-1) ** i) * 2.0 ** x
        sol = np.linalg.solve(A, 2.0 ** xs)
        coef = sol[: deg + 1]
        err = (np.polyval(coef[::-1], grid) - 2.0 ** grid) / 2.0 ** grid
        # new reference: extrema of the error between sign changes
        sign = np.sign(err)
        idx = np.concatenate(([0], np.nonzero(np.diff(sign))[0] + 1, [len(grid)]))
        ext = [seg_start + np.argmax(np.abs(err[seg_start:seg_end]))
               for seg_start, seg_end in zip(idx[:-1], idx[1:])]
        if len(ext) != deg + 2:
            break
        xs = grid[np.array(ext)]
    return coef


def max_rel_error_f32(coef) -> float:
    """Relative error of the float32 evaluation (Horner, fused multiply-add)."""
    c = [np.float32(v) for v in coef]
    f = np.linspace(-0.5, 0.5, 400001, dtype=np.float32)
    p = c[3]
    for ci in (c[2], c[1], c[0]):
        p = np.float32(p * f + ci)
    ref = 2.0 ** f.astype(np.float64)
    return float(np.max(np.abs(p.astype(np.float64) - ref) / ref))


if __name__ == "__main__":
    coef = _fit_remez(DEG)
    for i, v in enumerate(coef):
        print(f"c{i} = {np.float32(v)!r}  ({float(np.float32(v)).hex()})")
    print("max relative error (float32 Horner):", max_rel_error_f32(coef))
