"""Fit the polynomial used for part of the exp2 evaluations in the prefill kernel.

    python block_sparse_streaming_ssa_b200/csrc/fit_exp2_poly.py

Method (Cody–Waite range reduction + minimax polynomial):
    2^x = 2^j * 2^f,  j = rint(x),  f = x - j in [-1/2, 1/2]
2^j is built by adding j to the exponent field; 2^f is approximated by
    p(f) = c0 + f (c1 + f (c2 + f c3))
whose coefficients minimise the maximum RELATIVE error over [-1/2, 1/2].
The fit is a linear program on a dense grid: minimise e subject to
|p(f_i) - 2^f_i| <= e * 2^f_i for every grid point.  The coefficients are then
rounded to fp32 and the error is re-measured with fp32 Horner evaluation.

Degree 3 gives ~9e-5 relative error; the kernel rounds the result to bf16
(relative step 2^-8 = 3.9e-3), so this is far below the rounding it feeds.
"""
import numpy as np
from scipy.optimize import linprog


def fit(degree=3, n=4001):
    f = np.linspace(-0.5, 0.5, n)
    y = np.exp2(f)
    V = np.vander(f, degree + 1, increasing=True)          # [n, degree+1]
    # variables: c_0..c_d, e ; minimise e
    c = np.zeros(degree + 2)
    c[-1] = 1.0
    A_ub = np.block([[V, -y[:, None]], [-V, -y[:, None]]])
    b_ub = np.concatenate([y, -y])
    res = linprog(c, A_ub=A_ub, b_ub=b_ub, bounds=[(None, None)] * (degree + 1) + [(0, None)],
                  method="highs")
    assert res.success, res.message
    return res.x[:-1], res.x[-1]


def fp32_rel_error(coefs):
    c = np.asarray(coefs, np.float32)
    f = np.linspace(-0.5, 0.5, 200001).astype(np.float32)
    p = np.full_like(f, c[-1])
    for k in range(len(c) - 2, -1, -1):
        p = (p * f + c[k]).astype(np.float32)
    return float(np.max(np.abs(p.astype(np.float64) / np.exp2(f.astype(np.float64)) - 1.0)))


if __name__ == "__main__":
    coefs, err = fit()
    c32 = [float(np.float32(x)) for x in coefs]
    print("minimax relative error (exact coefficients): %.3e" % err)
    print("fp32 coefficients:", ", ".join("%.9ef" % x for x in c32))
    print("fp32 Horner relative error: %.3e" % fp32_rel_error(c32))
