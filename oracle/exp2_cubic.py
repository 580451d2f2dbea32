"""Software 2^x: Cody-Waite range reduction + minimax cubic -- TEST INFRASTRUCTURE ONLY.

Follows the software exponential of FlashAttention-4 as the pages describe it
(AI Infra series ch. 6, "GPU performance engineering (II)", section 7, item 1:
a polynomial approximation, Cody-Waite reduction plus a cubic, evaluated on
the FMA units for a minority of the exponentials; and "NVIDIA's strongest
B200 wastes 60%", section "three moves", first move: the polynomial is mixed
with the hardware unit to keep accuracy).  The pages give neither the
coefficients nor the reduction's details.  Reading used here:

1. the input is already in base-2 units (x = s*scale*log2(e) - m), so the
   Cody-Waite split of x into n*C + f needs the constant C = 1, whose
   "high part" is exact: n = floor(x), f = x - n in [0, 1), both exact in fp32;
2. 2^f on [0, 1) is a cubic c0 + f(c1 + f(c2 + f c3)) whose coefficients
   minimise the maximum RELATIVE error (Remez exchange, below, in fp64);
3. 2^n is applied by adding n to the fp32 exponent field (an integer add);
4. inputs below -126 are clamped to -126 first.  Since c0 < 1, the
   exponent add can then reach the subnormal range (exponent field 0) but
   never wraps into the sign bit; results for x < -125 are therefore only
   guaranteed to lie in [0, 2^-124), negligible next to the row sum (>= 1).

``remez_cubic()`` fits the coefficients; ``exp2_cubic_f32()`` evaluates the
scheme with fp32 rounding after every fused multiply-add (emulated in fp64:
the fp32 product is exact in fp64, so only the add can double-round).
"""
from __future__ import annotations

import numpy as np


def remez_cubic(iters: int = 30, grid: int = 200001):
    """Minimax-relative-error cubic for 2^f on [0, 1] by the Remez exchange.

    Returns (coeffs c0..c3 as fp64, E = the levelled max relative error).
    Reference set: 5 = degree + 2 points with alternating errors.
    """
    xs = 0.5 - 0.5 * np.cos(np.pi * np.arange(5) / 4)  # Chebyshev extrema on [0, 1]
    fine = np.linspace(0.0, 1.0, grid)
    c, E = None, None
    for _ in range(iters):
        # Solve p(x_i) - 2^x_i = (-1)^i E 2^x_i  for c0..c3, E.
        A = np.zeros((5, 5))
        rhs = np.exp2(xs)
        for i, x in enumerate(xs):
            A[i, :4] = [1.0, x, x * x, x ** 3]
            A[i, 4] = -((-1.0) ** i) * np.exp2(x)
        sol = np.linalg.solve(A, rhs)
        c, E = sol[:4], sol[4]
        err = (np.polyval(c[::-1], fine) - np.exp2(fine)) / np.exp2(fine)
        # New reference: the extremum of each sign-run of the error curve.
        sign = np.sign(err)
        runs = np.flatnonzero(np.diff(sign) != 0) + 1
        bounds = np.concatenate([[0], runs, [len(fine)]])
        new = []
        for a, bnd in zip(bounds[:-1], bounds[1:]):
            seg = np.abs(err[a:bnd])
            new.append(fine[a + int(np.argmax(seg))])
        if len(new) != 5:
            break
        new = np.array(new)
        if np.max(np.abs(new - xs)) < 1e-12:
            xs = new
            break
        xs = new
    return c, abs(E)


def _fma_f32(a, b, c):
    """fp32 fused multiply-add emulated in fp64 (a*b exact; one final fp32 rounding)."""
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


def exp2_cubic_f32(x, coeffs) -> np.ndarray:
    """2^x by the scheme above, with fp32 arithmetic; x array-like of float32."""
    x = np.maximum(np.asarray(x, dtype=np.float32), np.float32(-126.0))
    n = np.floor(x)                          # exact
    f = (x - n).astype(np.float32)           # exact for |x| < 2^23
    c = [np.float32(ci) for ci in coeffs]
    p = np.full_like(f, c[3])
    p = _fma_f32(p, f, np.full_like(f, c[2]))
    p = _fma_f32(p, f, np.full_like(f, c[1]))
    p = _fma_f32(p, f, np.full_like(f, c[0]))
    bits = p.view(np.int32) + (n.astype(np.int32) << 23)
    return bits.view(np.float32)
