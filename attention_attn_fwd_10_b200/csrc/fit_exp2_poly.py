"""Fit the cubic used by the kernels' software 2^x (build-time constant generator).

The kernels evaluate 2^f on f in [0, 1) as c0 + f*(c1 + f*(c2 + f*c3)) on the
FMA pipe after splitting x = n + f (FlashAttention-4's software exponential:
Cody-Waite range reduction plus a cubic, as described in "AI Infra series
ch. 6, GPU performance engineering (II)", section 7, item 1).  The pages do
not give coefficients.  This script picks them to minimise the maximum
relative error on a dense grid, posed as a linear program

    minimise e  subject to  |p(f_i) - 2^f_i| <= e * 2^f_i  for every grid f_i,

solved with scipy's HiGHS backend, then rounds them to fp32.  Run it to
regenerate the constants in ``sm100_common.cuh`` (kExp2C0..kExp2C3):

    python attention_attn_fwd_10_b200/csrc/fit_exp2_poly.py
"""
import numpy as np
from scipy.optimize import linprog


def fit(n_grid: int = 4001):
    f = np.linspace(0.0, 1.0, n_grid)
    t = np.exp2(f)
    V = np.stack([np.ones_like(f), f, f * f, f ** 3], axis=1)
    # variables: c0..c3, e ; minimise e
    cost = np.array([0, 0, 0, 0, 1.0])
    A_ub = np.vstack([np.hstack([V, -t[:, None]]), np.hstack([-V, -t[:, None]])])
    b_ub = np.concatenate([t, -t])
    res = linprog(cost, A_ub=A_ub, b_ub=b_ub, bounds=[(None, None)] * 4 + [(0, None)], method="highs")
    assert res.success, res.message
    return res.x[:4], res.x[4]


if __name__ == "__main__":
    c, e = fit()
    c32 = c.astype(np.float32)
    print(f"max relative error on the grid: {e:.6e}")
    for i, ci in enumerate(c32):
        print(f"constexpr float kExp2C{i} = {float(ci):.9e}f;  // 0x{ci.view(np.uint32):08x}")
