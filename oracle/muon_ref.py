"""Plain, slow, fp64 oracle of the Muon optimizer step.

TEST INFRASTRUCTURE ONLY: imported by tests/, __graft_entry__.smoke() and the
CPU-baseline leg of bench.py, never by the product path.

Sources (page titles as printed at the head of each page):

* "New training speed record for @karpathy's 124M-parameter NanoGPT setup"
  (X thread, tweets 2/8, 5/8, 6/8): the update is the SGD-Nesterov-momentum
  update, orthogonalised per parameter *after* momentum, by a quintic
  Newton-Schulz iteration run in bfloat16 whose coefficients are chosen for a
  large slope at zero, at the cost of some non-convergence.
* "07. Training neural networks", section "Momentum": the PyTorch convention
  buf <- beta*buf + g, without the (1 - beta) factor.
* The quantitative form of the step (a plain reading; the pages give it only
  in words): u = g + beta*buf (Nesterov), X0 = u / ||u||_F, transpose so that
  rows <= cols, five iterations of  A = X X^T,  B = b A + c A^2,
  X <- a X + B X  with (a, b, c) = (3.4445, -4.7750, 2.0315), then
  p <- p - lr * sqrt(max(1, rows/cols)) * X.

Rounding model (the storage points of the GPU path, made explicit so the
oracle is bit-comparable where the GPU's fp32 accumulation allows):

* momentum buffer, Nesterov vector u and parameters: fp32 (one rounding of
  the fp64 value);
* X0, each Gram matrix A, each polynomial matrix B and each iterate X_k:
  bfloat16, round-to-nearest-even, from the fp64 value;
* everything else (sums, norms, coefficients applied to fp32-rounded
  coefficient values) in fp64.

``exact=True`` switches every rounding off (pure fp64), for closed-form pins.

parity pins: see tests/test_oracle_pins.py (scalar recurrences, spectral
closed form, diagonal inputs, brute force on 2x2/4x4, invariances).
"""
from __future__ import annotations

import math
from typing import Sequence, Tuple

import numpy as np

# Added to the Frobenius norm before dividing, so that a zero update gives
# X0 = 0 (and leaves the parameter unchanged) instead of NaN.
EPS = 1e-7

# Largest finite bfloat16: (2 - 2^-7) * 2^127.
BF16_MAX = (2.0 - 2.0 ** -7) * 2.0 ** 127
_BF16_MIN_NORMAL = 2.0 ** -126
_BF16_SUBNORMAL_STEP = 2.0 ** -133


def bf16_round(x) -> np.ndarray:
    """Round float64 values to the nearest bfloat16 value, ties to even.

    bfloat16 = 1 sign bit, 8 exponent bits (fp32's range), 7 stored mantissa
    bits.  Written from the IEEE-754 definition of round-to-nearest-even:

    * normal range: keep 8 significant bits of the fp64 significand; the 45
      dropped bits decide the direction, exact halves go to the even neighbour;
    * below 2^-126: the grid is the fixed subnormal step 2^-133;
    * results above the largest finite bfloat16 become +-inf;
    * NaN stays NaN, +-inf and +-0 are kept.

    Returns float64 values that are exactly representable in bfloat16.
    """
    x = np.asarray(x, dtype=np.float64)
    bits = x.view(np.uint64).copy()
    drop = np.uint64(45)                       # 52 - 7 mantissa bits dropped
    lsb = (bits >> drop) & np.uint64(1)
    bias = np.uint64((1 << 44) - 1) + lsb      # half-ulp minus one, plus the tie-to-even bit
    rounded = ((bits + bias) >> drop) << drop
    out = rounded.view(np.float64)
    ax = np.abs(x)
    small = ax < _BF16_MIN_NORMAL
    if np.any(small):
        # np.round is round-half-to-even; scaling by 2^133 is exact.
        out = np.where(small, np.round(x / _BF16_SUBNORMAL_STEP) * _BF16_SUBNORMAL_STEP, out)
    # Anything that rounded past the largest finite value overflows.
    over = np.isfinite(x) & (np.abs(out) > BF16_MAX)
    if np.any(over):
        out = np.where(over, np.copysign(np.inf, x), out)
    nan = np.isnan(x)
    if np.any(nan):
        out = np.where(nan, np.nan, out)
    return out


def f32_round(x) -> np.ndarray:
    """Round float64 values to fp32 (IEEE round-to-nearest-even), as float64."""
    return np.asarray(x, dtype=np.float64).astype(np.float32).astype(np.float64)


def coeffs_f32(coeffs: Sequence[float]) -> Tuple[float, float, float]:
    """The (a, b, c) triple as the fp32 values the C interface carries."""
    a, b, c = (float(np.float32(v)) for v in coeffs)
    return a, b, c


def momentum_ref(g, buf, beta: float, nesterov: bool):
    """SGD momentum in the PyTorch convention, then the Nesterov look-ahead.

    "07. Training neural networks", section "Momentum": buf <- beta*buf + g
    (no (1 - beta) factor).  X thread tweet 5/8: the update that gets
    orthogonalised is the one *after* Nesterov momentum, u = g + beta*buf_new;
    with nesterov off, u = buf_new.

    Inputs are fp32 arrays; returns (buf_new, u) as fp32-valued float64 arrays.
    """
    beta = float(np.float32(beta))
    g = np.asarray(g, dtype=np.float64)
    buf = np.asarray(buf, dtype=np.float64)
    buf_new = f32_round(beta * buf + g)
    u = f32_round(g + beta * buf_new) if nesterov else buf_new
    return buf_new, u


def orient(x: np.ndarray) -> Tuple[np.ndarray, bool]:
    """Transpose a tall matrix so that rows <= cols; square stays as is."""
    r, c = x.shape
    if r > c:
        return x.T, True
    return x, False


def normalize_ref(u, exact: bool = False) -> np.ndarray:
    """X0 = u / (||u||_F + EPS), rounded to bfloat16 (unless ``exact``).

    The norm is the Frobenius norm of the fp32 vector u, summed in fp64.
    Returns X0 in the stored orientation of u (orientation is a separate step).
    """
    u = np.asarray(u, dtype=np.float64)
    nu = math.sqrt(float(np.sum(u * u)))
    x0 = u / (nu + EPS)
    return x0 if exact else bf16_round(x0)


def newton_schulz_ref(x0, steps: int, coeffs: Sequence[float], exact: bool = False,
                      trace: bool = False):
    """Quintic Newton-Schulz iteration on an already oriented X0 (rows <= cols).

    X thread tweets 5/8 and 6/8: a quintic Newton-Schulz iteration, run in
    bfloat16, with aggressive coefficients.  One iteration is

        A = X X^T            (m x m, rounded to bf16)
        B = b A + c (A A)    (m x m, rounded to bf16)
        X = a X + B X        (m x n, rounded to bf16)

    i.e. X <- a X + b (X X^T) X + c (X X^T)^2 X, the odd quintic p(s) =
    a s + b s^3 + c s^5 applied to every singular value of X.  Sums are fp64;
    the coefficients are the fp32 values the interface carries.

    Returns X (float64 holding bf16 values unless ``exact``); with ``trace``
    also the list of (A, B, X) after every iteration.
    """
    a, b, c = coeffs_f32(coeffs)
    rnd = (lambda t: t) if exact else bf16_round
    x = np.asarray(x0, dtype=np.float64)
    if x.shape[0] > x.shape[1]:
        raise ValueError("newton_schulz_ref expects rows <= cols (orient first)")
    hist = []
    for _ in range(int(steps)):
        A = rnd(x @ x.T)
        B = rnd(b * A + c * (A @ A))
        x = rnd(a * x + B @ x)
        if trace:
            hist.append((A, B, x))
    return (x, hist) if trace else x


def update_scale(rows: int, cols: int, lr: float) -> float:
    """fp32 value of lr * sqrt(max(1, rows/cols)), rows x cols as stored."""
    return float(np.float32(float(np.float32(lr)) * math.sqrt(max(1.0, rows / cols))))


def orthogonalize_ref(u, steps: int, coeffs: Sequence[float], exact: bool = False):
    """Normalise, orient, iterate, and orient back: the orthogonalised update."""
    x0 = normalize_ref(u, exact=exact)
    xo, t = orient(x0)
    x = newton_schulz_ref(xo, steps, coeffs, exact=exact)
    return x.T if t else x


def muon_step_ref(params: Sequence[np.ndarray], grads: Sequence[np.ndarray],
                  bufs: Sequence[np.ndarray], lr: float, beta: float = 0.95,
                  nesterov: bool = True, ns_steps: int = 5,
                  coeffs: Sequence[float] = (3.4445, -4.7750, 2.0315),
                  return_x: bool = False):
    """One Muon step over a list of 2-D fp32 parameters.

    For each matrix independently: momentum + Nesterov (fp32), Frobenius
    normalisation, orientation, ``ns_steps`` Newton-Schulz iterations in bf16,
    orientation back, then p <- p - lr*sqrt(max(1, rows/cols)) * X as one fp32
    rounding of the fp64 value.

    Returns (new_params, new_bufs[, xs]) as float32 arrays (xs: float64 bf16
    values in the stored orientation).
    """
    new_p, new_b, xs = [], [], []
    for p, g, buf in zip(params, grads, bufs):
        if p.ndim != 2:
            raise ValueError("Muon applies to 2-D parameters only")
        r, c = p.shape
        buf_new, u = momentum_ref(g, buf, beta, nesterov)
        x = orthogonalize_ref(u, ns_steps, coeffs)
        s = update_scale(r, c, lr)
        p_new = f32_round(np.asarray(p, dtype=np.float64) - s * x)
        new_p.append(p_new.astype(np.float32))
        new_b.append(buf_new.astype(np.float32))
        xs.append(x)
    if return_x:
        return new_p, new_b, xs
    return new_p, new_b
