"""Coefficients of the polynomial 2^f ~ c0 + c1 f + c2 f^2 + c3 f^3 on f in [-1/2, 1/2]
used by the tensor-core prefill kernels to compute part of their exponentials on the FMA
pipe (apd_prefill_tc.cuh, exp2_fma): x = j + f with j = round(x), 2^x = 2^j * 2^f, the
integer j added to the exponent field of the polynomial's value.

The fit minimises the maximum relative error (Remez-style iteration on the weighted
least-squares fit over Chebyshev nodes, with c0 pinned to 1 so that 2^0 = 1 exactly).
Run it to print the coefficients and the error bound; the values in the kernel are the
printed ones rounded to fp32.
"""
import numpy as np


def fit(deg=3, iters=60):
    f = np.cos(np.linspace(0, np.pi, 4001)) * 0.5  # Chebyshev-spaced points of [-1/2, 1/2]
    y = np.exp2(f)
    w = np.ones_like(f)
    for _ in range(iters):
        # minimise sum w (p(f)/2^f - 1)^2 with p(0) = 1: unknowns c1..c_deg
        A = np.stack([f ** k / y for k in range(1, deg + 1)], 1) * w[:, None]
        b = (1.0 - 1.0 / y) * w
        c = np.linalg.lstsq(A, b, rcond=None)[0]
        err = np.abs((1.0 + sum(c[k - 1] * f ** k for k in range(1, deg + 1))) / y - 1.0)
        w = w * (1.0 + err / err.max()) ** 2  # push weight towards the worst points
        w /= w.mean()
    return np.concatenate([[1.0], c]), err.max()


if __name__ == "__main__":
    c, e = fit()
    c32 = c.astype(np.float32)
    f = np.linspace(-0.5, 0.5, 200001)
    p = np.polyval(c32[::-1].astype(np.float64), f)
    print("coefficients (fp32):", ", ".join(f"{v:.9g}f" for v in c32))
    print(f"max relative error on [-1/2, 1/2]: {np.max(np.abs(p / np.exp2(f) - 1)):.3e} (bf16 half-ulp: {2**-9:.3e})")
