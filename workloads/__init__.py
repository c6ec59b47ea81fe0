"""Seeded synthetic inputs for the Muon optimizer step.

This module draws the random tensors that both the CUDA path and the oracle
consume.  It holds no arithmetic of the method itself: no momentum, no
normalisation, no Newton-Schulz and no update.  Everything here is shape
bookkeeping and random draws from NumPy's PCG64 generator.

Workloads (all matrices fp32, row-major, shapes as stored r x c):

* ``single_256``   one 256x256 parameter, N(0,1) gradients, zero momentum.
* ``gpt2_block``   the four hidden matrices of one GPT-2 block at d=768
                   (c_attn 768x2304, attn c_proj 768x768, mlp c_fc 768x3072,
                   mlp c_proj 3072x768); gradients rank-16 + 0.1 noise.
* ``gpt2_124m``    12 such blocks (48 matrices); rank-32 + 0.1 noise;
                   momentum warm-started with N(0, 1e-2) (std 0.1).
* ``gpt2_medium``  24 blocks at d=1024 (96 matrices).
* ``gpt2_xl``      48 blocks at d=1600 (192 matrices).
* ``square``       one n x n matrix U diag(sigma) V^T with log-uniform sigma
                   on [1e-3, 1] (condition number 1e3), for the NS-only sweep.

AdamW workloads (the parameters Muon leaves out; fp32 tensors of any rank):

* ``adamw_ragged``     a handful of tensors with ragged sizes (1, 3, 5, 768,
                       4097, 3x5x7, 50000), some in the no-decay group.
* ``gpt2_124m_adamw``  the non-hidden parameters of GPT-2 124M: token
                       embedding 50257x768 and position embedding 1024x768
                       (decayed), and per block the LayerNorm gains/biases and
                       the linear biases, plus the final LayerNorm (no decay):
                       100 tensors, 39,505,152 elements.

GPT-2 dimensions follow "Let's reproduce GPT-2 (124M)" (12 layers, 768
channels, init std 0.02); the Conv1D weights of GPT-2 are stored transposed
relative to a linear layer, which is why mlp c_proj is listed 3072x768.

Draw order (fixed so that a seed names one exact input):
  init   for each matrix in listing order: p, then buf (if warm-started);
  step   for each matrix in listing order: the gradient's factors, then noise.
  AdamW  init: for each tensor in listing order, p (when drawn), then the
         gradient average, then the squared-gradient average; step: for each
         tensor, its gradient.
"""
from __future__ import annotations

import dataclasses
from typing import List, Sequence, Tuple

import numpy as np

# The default quintic coefficient triple (a, b, c).
DEFAULT_COEFFS = (3.4445, -4.7750, 2.0315)


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    shapes: Tuple[Tuple[int, int], ...]
    grad_rank: int          # 0 = dense N(0,1) gradient; k>0 = rank-k A B^T + noise
    grad_noise: float       # std of the additive Gaussian noise for low-rank grads
    buf_std: float          # 0 = zero-initialised momentum
    param_std: float = 0.02
    lr: float = 0.02
    beta: float = 0.95
    nesterov: bool = True
    ns_steps: int = 5
    coeffs: Tuple[float, float, float] = DEFAULT_COEFFS
    steps: int = 1          # consecutive optimizer steps the workload specifies

    @property
    def n_matrices(self) -> int:
        return len(self.shapes)

    @property
    def n_elements(self) -> int:
        return sum(r * c for r, c in self.shapes)

    def ns_flops(self, dense: bool = False) -> float:
        """Newton-Schulz FLOPs of one optimizer step on this workload.

        Per iteration on an oriented m x n matrix (m <= n): the Gram product
        needs m^2 n (upper triangle only; 2 m^2 n dense), the symmetric square
        m^3 (2 m^3 dense), the X update 2 m^2 n.
        """
        tot = 0.0
        for r, c in self.shapes:
            m, n = min(r, c), max(r, c)
            per = (4 * m * m * n + 2 * m ** 3) if dense else (3 * m * m * n + m ** 3)
            tot += per * self.ns_steps
        return float(tot)


def _gpt2_shapes(layers: int, d: int) -> Tuple[Tuple[int, int], ...]:
    block = ((d, 3 * d), (d, d), (d, 4 * d), (4 * d, d))
    return tuple(s for _ in range(layers) for s in block)


WORKLOADS = {
    "single_256": Workload("single_256", ((256, 256),), grad_rank=0, grad_noise=0.0,
                           buf_std=0.0, steps=3),
    "gpt2_block": Workload("gpt2_block", _gpt2_shapes(1, 768), grad_rank=16,
                           grad_noise=0.1, buf_std=0.0, steps=10),
    "gpt2_124m": Workload("gpt2_124m", _gpt2_shapes(12, 768), grad_rank=32,
                          grad_noise=0.1, buf_std=0.1, steps=100),
    "gpt2_medium": Workload("gpt2_medium", _gpt2_shapes(24, 1024), grad_rank=32,
                            grad_noise=0.1, buf_std=0.1, steps=50),
    "gpt2_xl": Workload("gpt2_xl", _gpt2_shapes(48, 1600), grad_rank=32,
                        grad_noise=0.1, buf_std=0.1, steps=20),
}

SQUARE_SWEEP = (1024, 2048, 4096, 8192)


def _normal32(rng: np.random.Generator, shape, std: float = 1.0) -> np.ndarray:
    x = rng.standard_normal(shape, dtype=np.float32)
    if std != 1.0:
        x *= np.float32(std)
    return x


class WorkloadStream:
    """Seeded state + gradient stream of one workload.

    ``init()`` returns fp32 (params, bufs); every ``next_grads()`` returns the
    next step's fp32 gradients.  ``subset`` restricts to some matrix indices
    while still consuming the random stream of every matrix, so that matrix i
    gets the same values whichever subset is drawn.
    """

    def __init__(self, wl: Workload, seed: int = 0, subset: Sequence[int] | None = None):
        self.wl = wl
        self.rng = np.random.default_rng(seed)
        self.subset = None if subset is None else set(int(i) for i in subset)
        self._initialised = False

    def _want(self, i: int) -> bool:
        return self.subset is None or i in self.subset

    def init_iter(self):
        """Yield (i, p, buf) for every matrix in listing order (the subset is
        ignored), so that a caller can move each matrix elsewhere before the
        next is drawn.  Draws exactly what ``init()`` draws."""
        assert not self._initialised
        self._initialised = True
        for i, (r, c) in enumerate(self.wl.shapes):
            p = _normal32(self.rng, (r, c), self.wl.param_std)
            if self.wl.buf_std > 0:
                b = _normal32(self.rng, (r, c), self.wl.buf_std)
            else:
                b = np.zeros((r, c), np.float32)
            yield i, p, b

    def init(self) -> Tuple[List[np.ndarray], List[np.ndarray]]:
        params, bufs = [], []
        for i, p, b in self.init_iter():
            if self._want(i):
                params.append(p)
                bufs.append(b)
        return params, bufs

    def grads_iter(self, want=None):
        """Yield (i, g) for the next step's gradient of every matrix i with
        ``want(i)`` true (default: every matrix), drawing the random stream of
        all of them in listing order.  Draws exactly what ``next_grads()``
        draws."""
        k = self.wl.grad_rank
        for i, (r, c) in enumerate(self.wl.shapes):
            keep = want is None or want(i)
            if k == 0:
                g = _normal32(self.rng, (r, c))
            else:
                A = _normal32(self.rng, (r, k))
                B = _normal32(self.rng, (c, k))
                noise = _normal32(self.rng, (r, c), self.wl.grad_noise)
                if not keep:
                    continue
                # fp64 product then one rounding: independent of BLAS blocking.
                g = (A.astype(np.float64) @ B.astype(np.float64).T).astype(np.float32)
                g += noise
            if keep:
                yield i, g

    def next_grads(self) -> List[np.ndarray]:
        return [g for _, g in self.grads_iter(self._want)]


def haar_orthogonal(rng: np.random.Generator, n: int) -> np.ndarray:
    """Haar-distributed n x n orthogonal matrix (QR of a Gaussian, sign-fixed)."""
    z = rng.standard_normal((n, n))
    q, r = np.linalg.qr(z)
    q *= np.sign(np.diag(r))[None, :]
    return q


def fwht_rows(x: np.ndarray) -> np.ndarray:
    """Unnormalised Walsh-Hadamard transform applied to every row (length 2^k)."""
    y = np.array(x, dtype=np.float64, copy=True)
    n = y.shape[-1]
    assert n & (n - 1) == 0
    h = 1
    while h < n:
        y = y.reshape(*y.shape[:-1], n // (2 * h), 2, h)
        a = y[..., 0, :].copy()
        b = y[..., 1, :]
        y[..., 0, :] += b
        y[..., 1, :] = a - b
        y = y.reshape(*y.shape[:-3], n)
        h *= 2
    return y


@dataclasses.dataclass
class SquareCase:
    """G = U diag(sigma) V^T with known factors (for closed-form checks)."""
    n: int
    sigma: np.ndarray               # float64, length n
    g: np.ndarray                   # float32 n x n
    kind: str                       # "haar" or "hadamard"
    u: np.ndarray | None = None     # float64 factors (haar only)
    v: np.ndarray | None = None
    d1: np.ndarray | None = None    # +-1 diagonals (hadamard only): U = H D1/sqrt(n)
    d2: np.ndarray | None = None    # V = H D2 / sqrt(n)

    def project(self, x: np.ndarray) -> np.ndarray:
        """Return U^T x V (float64)."""
        x = np.asarray(x, dtype=np.float64)
        if self.kind == "haar":
            return self.u.T @ x @ self.v
        n = self.n
        # U^T x V = D1 H x H D2 / n  (H symmetric)
        t = fwht_rows(x)                  # x H   (row transform = right-multiply by H)
        t = fwht_rows(t.T).T              # H x H
        return (self.d1[:, None] * t * self.d2[None, :]) / n


def square_case(n: int, seed: int = 0, cond: float = 1e3) -> SquareCase:
    """Square NS input with log-uniform singular values on [1/cond, 1]."""
    rng = np.random.default_rng(seed)
    sigma = np.exp(rng.uniform(np.log(1.0 / cond), 0.0, size=n))
    sigma[0] = 1.0
    sigma[-1] = 1.0 / cond
    if n <= 2048:
        u = haar_orthogonal(rng, n)
        v = haar_orthogonal(rng, n)
        g = ((u * sigma[None, :]) @ v.T).astype(np.float32)
        return SquareCase(n, sigma, g, "haar", u=u, v=v)
    d1 = rng.choice(np.array([-1.0, 1.0]), size=n)
    d2 = rng.choice(np.array([-1.0, 1.0]), size=n)
    # G = U diag(s) V^T = H D1 diag(s) D2 H / n
    w = d1 * sigma * d2
    t = fwht_rows(np.diag(w))             # diag(w) H
    g = fwht_rows(t.T).T / n              # H diag(w) H / n
    return SquareCase(n, sigma, g.astype(np.float32), "hadamard", d1=d1, d2=d2)


# ---------------------------------------------------------------- AdamW inputs

@dataclasses.dataclass(frozen=True)
class AdamWTensor:
    name: str
    shape: Tuple[int, ...]
    decay: bool             # False: the no-decay group (biases, 1-D tensors)
    init: str               # "normal" (std 0.02), "ones" or "zeros"

    @property
    def numel(self) -> int:
        return int(np.prod(self.shape)) if self.shape else 1


@dataclasses.dataclass(frozen=True)
class AdamWWorkload:
    name: str
    tensors: Tuple[AdamWTensor, ...]
    lr: float = 6e-4
    beta1: float = 0.9
    beta2: float = 0.999
    eps: float = 1e-8
    weight_decay: float = 0.1
    step: int = 10          # the step number t of the (first) step drawn
    grad_std: float = 1e-2

    @property
    def n_tensors(self) -> int:
        return len(self.tensors)

    @property
    def n_elements(self) -> int:
        return sum(t.numel for t in self.tensors)


def _gpt2_adamw_tensors(layers: int, d: int, vocab: int = 50257, ctx: int = 1024):
    ts = [AdamWTensor("wte", (vocab, d), True, "normal"),
          AdamWTensor("wpe", (ctx, d), True, "normal")]
    for l in range(layers):
        ts += [AdamWTensor(f"h{l}.ln_1.weight", (d,), False, "ones"),
               AdamWTensor(f"h{l}.ln_1.bias", (d,), False, "zeros"),
               AdamWTensor(f"h{l}.attn.c_attn.bias", (3 * d,), False, "zeros"),
               AdamWTensor(f"h{l}.attn.c_proj.bias", (d,), False, "zeros"),
               AdamWTensor(f"h{l}.ln_2.weight", (d,), False, "ones"),
               AdamWTensor(f"h{l}.ln_2.bias", (d,), False, "zeros"),
               AdamWTensor(f"h{l}.mlp.c_fc.bias", (4 * d,), False, "zeros"),
               AdamWTensor(f"h{l}.mlp.c_proj.bias", (d,), False, "zeros")]
    ts += [AdamWTensor("ln_f.weight", (d,), False, "ones"),
           AdamWTensor("ln_f.bias", (d,), False, "zeros")]
    return tuple(ts)


ADAMW_WORKLOADS = {
    "adamw_ragged": AdamWWorkload("adamw_ragged", (
        AdamWTensor("a", (1,), True, "normal"),
        AdamWTensor("b", (3,), False, "normal"),
        AdamWTensor("c", (5,), True, "normal"),
        AdamWTensor("d", (768,), False, "ones"),
        AdamWTensor("e", (4097,), True, "normal"),
        AdamWTensor("f", (3, 5, 7), True, "normal"),
        AdamWTensor("g", (50000,), False, "normal"),
    ), lr=1e-2, step=3),
    "gpt2_124m_adamw": AdamWWorkload("gpt2_124m_adamw", _gpt2_adamw_tensors(12, 768)),
}


class AdamWStream:
    """Seeded AdamW state + gradient stream.

    ``init()`` returns fp32 (params, exp_avgs, exp_avg_sqs) as they stand
    after ``wl.step - 1`` steps: parameters at their GPT-2 initial values
    (normal std 0.02, LayerNorm gains 1, biases 0), gradient averages
    N(0, (0.1 grad_std)^2) and squared-gradient averages (grad_std z)^2 with
    z ~ N(0,1) (non-negative, as a running mean of squares is).  With
    ``wl.step == 1`` both averages start at zero.  Every ``next_grads()``
    returns one step's N(0, grad_std^2) gradients.
    """

    def __init__(self, wl: AdamWWorkload, seed: int = 0):
        self.wl = wl
        self.rng = np.random.default_rng(seed)

    def init(self):
        params, us, vs = [], [], []
        for t in self.wl.tensors:
            if t.init == "normal":
                p = _normal32(self.rng, t.shape, 0.02)
            elif t.init == "ones":
                p = np.ones(t.shape, np.float32)
            else:
                p = np.zeros(t.shape, np.float32)
            if self.wl.step > 1:
                u = _normal32(self.rng, t.shape, 0.1 * self.wl.grad_std)
                z = _normal32(self.rng, t.shape, self.wl.grad_std)
                v = z * z
            else:
                u = np.zeros(t.shape, np.float32)
                v = np.zeros(t.shape, np.float32)
            params.append(p)
            us.append(u)
            vs.append(v)
        return params, us, vs

    def next_grads(self):
        return [_normal32(self.rng, t.shape, self.wl.grad_std) for t in self.wl.tensors]
