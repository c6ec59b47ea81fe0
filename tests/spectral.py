"""Closed forms for the quintic Newton-Schulz iteration (test helpers).

The iteration X <- a X + b (X X^T) X + c (X X^T)^2 X acts on the singular
values of X alone: if X = U diag(s) V^T then one iteration gives
U diag(p(s)) V^T with p(s) = a s + b s^3 + c s^5, and the singular vectors do
not move.  These helpers evaluate that scalar map, by a route that shares
nothing with the matrix iteration of the oracle (no matrix products, an SVD
from LAPACK instead), so that the two can pin each other.
"""
from __future__ import annotations

from fractions import Fraction

import numpy as np

DEFAULT_COEFFS = (3.4445, -4.7750, 2.0315)


def f32(v: float) -> float:
    return float(np.float32(v))


def poly_scalar(s, coeffs=DEFAULT_COEFFS, steps=5):
    """p applied ``steps`` times to s (fp32-valued coefficients, fp64 math)."""
    a, b, c = (f32(v) for v in coeffs)
    s = np.asarray(s, dtype=np.float64)
    for _ in range(steps):
        s2 = s * s
        s = s * (a + s2 * (b + c * s2))
    return s


def poly_sequence_exact(s0, coeffs=DEFAULT_COEFFS, steps=5):
    """Exact rational values of p^k(s0), k = 1..steps (fp32 coefficients)."""
    a, b, c = (Fraction(f32(v)) for v in coeffs)
    s = Fraction(s0)
    out = []
    for _ in range(steps):
        s = a * s + b * s ** 3 + c * s ** 5
        out.append(s)
    return out


def closed_form_ns(x0, coeffs=DEFAULT_COEFFS, steps=5):
    """U diag(p^steps(s)) V^T from the SVD of x0 (any orientation)."""
    u, s, vt = np.linalg.svd(np.asarray(x0, dtype=np.float64), full_matrices=False)
    return (u * poly_scalar(s, coeffs, steps)[None, :]) @ vt


def rel_fro(x, ref) -> float:
    x = np.asarray(x, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    den = np.linalg.norm(ref)
    return float(np.linalg.norm(x - ref) / (den if den > 0 else 1.0))


# Smallest normalised singular value that 5 default iterations lift to >= 0.6
# (solved by bisection on poly_scalar; p is increasing on [0, 0.55]).
def lift_threshold(target=0.6, coeffs=DEFAULT_COEFFS, steps=5):
    lo, hi = 0.0, 0.5
    for _ in range(200):
        mid = 0.5 * (lo + hi)
        if poly_scalar(mid, coeffs, steps) >= target:
            hi = mid
        else:
            lo = mid
    return hi


def band_report(x_out, u, coeffs=DEFAULT_COEFFS, steps=5, low=0.6, high=1.3, slack=0.02):
    """The singular-value band of one orthogonalised update, read as stated
    for the literal [0.6, 1.3] band (which low-rank gradients cannot meet):

    * every singular value of the output is at most ``high``;
    * at least as many output singular values reach ``low - slack`` as the
      normalised input u/||u|| has singular values at or above the lift
      threshold (the smallest s0 that ``steps`` iterations of p carry to
      ``low``): every direction the iteration can lift is lifted.

    Returns (max_sigma, lifted_out, liftable_in, literal_fraction), the last
    being the fraction of output singular values inside [low, high]."""
    x = np.asarray(x_out, dtype=np.float64)
    sv = np.linalg.svd(x, compute_uv=False)
    u = np.asarray(u, dtype=np.float64)
    s0 = np.linalg.svd(u / np.linalg.norm(u), compute_uv=False)
    thr = lift_threshold(low, coeffs, steps)
    lifted = int(np.sum(sv >= low - slack))
    liftable = int(np.sum(s0 >= thr))
    literal = float(np.mean((sv >= low) & (sv <= high))) if sv.size else 1.0
    return float(sv.max()) if sv.size else 0.0, lifted, liftable, literal
