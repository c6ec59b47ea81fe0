"""Plain, slow, fp64 oracle of one AdamW step over a list of tensors.

TEST INFRASTRUCTURE ONLY: imported by tests/ and the CPU-baseline leg of
bench.py, never by the product path.

Muon updates the 2-D hidden matrices only; the remaining parameters of the
GPT-2 model (embeddings, biases, LayerNorm gains) take AdamW.  The X-thread
replies of "New training speed record for @karpathy's 124M-parameter NanoGPT
setup" describe that split (2-D tensors to Muon, the rest to AdamW).

Sources (page titles as printed at the head of each page):

* "07. Training neural networks", section "Adam, weight decay and AdamW"
  and its deeper block on bias correction and decoupling:
  - two running averages per entry, of the gradient and of its square, each
    starting at zero with memory constants beta1 and beta2;
  - bias correction: divide them by (1 - beta1^t) and (1 - beta2^t), t the
    step number counted from 1;
  - the step moves each entry by lr * u_hat / (sqrt(v_hat) + eps);
  - decoupled weight decay: the parameter is first multiplied by
    (1 - lr * lambda), and the Adam step is computed from the loss gradient
    alone (the gradient is the one taken before the decay).
* "Let's reproduce GPT-2 (124M)", section "Initialization and Training
  Details": weight decay 0.1, not applied to biases and 1-D tensors.

Rounding model: the caller's parameters and both averages are fp32 tensors.
The oracle computes every entry's new (p, u, v) in fp64 from the fp32 inputs
and the exact (double) hyper-parameters, then rounds each result once to fp32
(``store_f32=True``, the default).  ``store_f32=False`` keeps fp64 throughout,
for the closed-form pins.

parity pins: tests/test_adamw_pins.py (the worked example's printed iterates
and losses, the first-step and constant-gradient closed forms, the decay
factors and halving counts, torch.optim.AdamW in fp64 as an independent
implementation).
"""
from __future__ import annotations

from typing import List, Optional, Sequence, Tuple

import numpy as np


def _f32(x: np.ndarray) -> np.ndarray:
    return np.asarray(x, dtype=np.float64).astype(np.float32)


def adamw_tensor_ref(p, g, u, v, step: int, lr: float, beta1: float = 0.9, beta2: float = 0.999,
                     eps: float = 1e-8, weight_decay: float = 0.0, store_f32: bool = True
                     ) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """One AdamW step on one tensor; returns the new (p, u, v).

    ``u`` and ``v`` are the running averages of the gradient and of its square
    after step - 1 steps (zero before the first step); ``step`` is t >= 1.
    """
    if step < 1:
        raise ValueError("the step number t counts from 1")
    p = np.asarray(p, np.float64)
    g = np.asarray(g, np.float64)
    u = np.asarray(u, np.float64)
    v = np.asarray(v, np.float64)
    # decoupled decay, applied to the parameter before the Adam step
    theta = p * (1.0 - lr * weight_decay)
    # the two running averages
    u_new = beta1 * u + (1.0 - beta1) * g
    v_new = beta2 * v + (1.0 - beta2) * (g * g)
    # bias correction
    u_hat = u_new / (1.0 - beta1 ** step)
    v_hat = v_new / (1.0 - beta2 ** step)
    theta = theta - lr * u_hat / (np.sqrt(v_hat) + eps)
    if store_f32:
        return _f32(theta), _f32(u_new), _f32(v_new)
    return theta, u_new, v_new


def adamw_update_term(g, u, v, step: int, lr: float, beta1: float = 0.9, beta2: float = 0.999,
                      eps: float = 1e-8) -> np.ndarray:
    """|lr * u_hat / (sqrt(v_hat) + eps)| in fp64: the size of the Adam move of
    each entry, which sets the rounding budget of the fp32 update."""
    g = np.asarray(g, np.float64)
    u_new = beta1 * np.asarray(u, np.float64) + (1.0 - beta1) * g
    v_new = beta2 * np.asarray(v, np.float64) + (1.0 - beta2) * (g * g)
    u_hat = u_new / (1.0 - beta1 ** step)
    v_hat = v_new / (1.0 - beta2 ** step)
    return np.abs(lr * u_hat / (np.sqrt(v_hat) + eps))


def adamw_step_ref(params: Sequence[np.ndarray], grads: Sequence[np.ndarray],
                   exp_avgs: Sequence[np.ndarray], exp_avg_sqs: Sequence[np.ndarray], step: int,
                   lr: float, beta1: float = 0.9, beta2: float = 0.999, eps: float = 1e-8,
                   weight_decay: float = 0.0, decay: Optional[Sequence[bool]] = None,
                   store_f32: bool = True) -> Tuple[List[np.ndarray], List[np.ndarray], List[np.ndarray]]:
    """One AdamW step over a list of tensors (any shapes).

    ``decay[i]`` false puts tensor i in the no-decay group (weight decay 0);
    ``decay=None`` decays every tensor.
    """
    n = len(params)
    if not (len(grads) == len(exp_avgs) == len(exp_avg_sqs) == n):
        raise ValueError("params, grads and both averages must have the same length")
    if decay is None:
        decay = [True] * n
    out_p, out_u, out_v = [], [], []
    for i in range(n):
        wd = weight_decay if decay[i] else 0.0
        p, u, v = adamw_tensor_ref(params[i], grads[i], exp_avgs[i], exp_avg_sqs[i], step, lr, beta1,
                                   beta2, eps, wd, store_f32)
        out_p.append(p)
        out_u.append(u)
        out_v.append(v)
    return out_p, out_u, out_v


def adamw_trajectory(theta0, grad_fn, steps: int, lr: float, beta1: float = 0.9,
                     beta2: float = 0.999, eps: float = 1e-8, weight_decay: float = 0.0) -> np.ndarray:
    """fp64 iterates theta_0 .. theta_steps of AdamW on a loss whose gradient
    is ``grad_fn(theta)``, evaluated at the current parameter before decay."""
    theta = np.array(theta0, dtype=np.float64)
    u = np.zeros_like(theta)
    v = np.zeros_like(theta)
    path = [theta.copy()]
    for t in range(1, steps + 1):
        g = grad_fn(theta)
        theta, u, v = adamw_tensor_ref(theta, g, u, v, t, lr, beta1, beta2, eps, weight_decay,
                                       store_f32=False)
        path.append(theta.copy())
    return np.array(path)
