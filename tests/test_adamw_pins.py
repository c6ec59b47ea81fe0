"""Pins of the AdamW oracle (oracle/adamw_ref.py) to facts outside itself.

* the worked example's printed iterates and losses ("07. Training neural
  networks", section "Adam, weight decay and AdamW", output [4]);
* closed forms: the first step (u_hat = g, v_hat = g^2 at t = 1) and a
  constant gradient (u_hat = g, v_hat = g^2 at every t);
* the printed decay factors and halving counts for zero gradient;
* torch.optim.AdamW in fp64 as an independent implementation (the page
  itself reports agreement with it);
* each of a few plausible mistakes, planted in a copy of the oracle's step,
  fails at least one of the checks above.
"""
from __future__ import annotations

import math
import os

import numpy as np
import pytest
import torch

from oracle import adamw_step_ref, adamw_tensor_ref, adamw_trajectory

Q = np.array([1.0, 10.0])
C = np.array([3.0, -1.0])


def bowl_grad(theta):
    # L = (t1 - 3)^2 + 10 (t2 + 1)^2  ->  dL/dt = 2 q (t - c)
    return 2.0 * Q * (np.asarray(theta) - C)


def bowl_loss(theta):
    return float(np.sum(Q * (np.asarray(theta) - C) ** 2))


def _rows(golden_dir, name):
    rows = []
    with open(os.path.join(golden_dir, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append(line.split())
    return rows


def _worked_example_ok(step_fn, golden_dir) -> bool:
    """The printed iterates (6 decimals) and losses (4 significant digits)."""
    theta = np.zeros(2)
    u = np.zeros(2)
    v = np.zeros(2)
    path = [theta]
    for t in range(1, 301):
        theta, u, v = step_fn(theta, bowl_grad(theta), u, v, t, 0.1, 0.9, 0.999, 1e-8, 0.0)
        path.append(theta)
    ok = True
    for row in _rows(golden_dir, "adam_bowl.txt"):
        if row[0] == "loss":
            want = float(row[2])
            got = bowl_loss(path[int(row[1])])
            ok &= float(f"{got:.4g}") == want
        else:
            t = int(row[0])
            ok &= round(path[t][0], 6) == float(row[1]) and round(path[t][1], 6) == float(row[2])
    return bool(ok)


def _oracle_step(p, g, u, v, t, lr, b1, b2, eps, wd):
    return adamw_tensor_ref(p, g, u, v, t, lr, b1, b2, eps, wd, store_f32=False)


def test_worked_example_iterates_and_losses(golden_dir):
    assert _worked_example_ok(_oracle_step, golden_dir)
    path = adamw_trajectory([0.0, 0.0], bowl_grad, 3, 0.1)
    np.testing.assert_allclose(path[1], [0.1, -0.1], rtol=0, atol=1e-8)   # lr * sign(g)


def test_first_step_closed_form():
    """t = 1: u_hat = g and v_hat = g^2, so each entry moves by
    -lr * g / (|g| + eps) after the decay factor."""
    rng = np.random.default_rng(3)
    p = rng.standard_normal(1000)
    g = rng.standard_normal(1000) * np.exp(rng.uniform(-8, 3, 1000))
    lr, wd = 0.05, 0.1
    for eps in (1e-8, 0.3):          # a large eps separates eps placements
        out, u, v = adamw_tensor_ref(p, g, np.zeros(1000), np.zeros(1000), 1, lr, 0.9, 0.999, eps, wd,
                                     store_f32=False)
        want = p * (1 - lr * wd) - lr * g / (np.abs(g) + eps)
        np.testing.assert_allclose(out, want, rtol=1e-14, atol=1e-16)
        np.testing.assert_allclose(u, 0.1 * g, rtol=1e-15)
        np.testing.assert_allclose(v, 0.001 * g * g, rtol=1e-12)


def test_constant_gradient_every_step_moves_lr():
    """With the same gradient every step the corrected averages equal g and
    g^2 exactly, so every step is -lr * g / (|g| + eps)."""
    rng = np.random.default_rng(4)
    g = rng.standard_normal(64)
    theta = rng.standard_normal(64)
    u = np.zeros(64)
    v = np.zeros(64)
    lr, eps = 1e-3, 1e-8
    for t in range(1, 61):
        new, u, v = adamw_tensor_ref(theta, g, u, v, t, lr, 0.9, 0.999, eps, 0.0, store_f32=False)
        np.testing.assert_allclose(new - theta, -lr * g / (np.abs(g) + eps), rtol=1e-9, atol=1e-18)
        theta = new


def test_zero_gradient_decay_factors_and_halving(golden_dir):
    for lr_s, factor_s, half_s in _rows(golden_dir, "adamw_decay.txt"):
        lr = float(lr_s)
        p1, _, _ = adamw_tensor_ref(np.ones(1), np.zeros(1), np.zeros(1), np.zeros(1), 1, lr,
                                    eps=1e-6, weight_decay=1e-2, store_f32=False)
        f = float(p1[0])
        assert f"{f:.7f}" == factor_s
        assert round(math.log(2) / -math.log(f)) == int(half_s)


def test_zero_gradient_halves_at_the_printed_step():
    """lr 5e-3, lambda 1e-2: iterate the oracle itself; the weight first
    drops to one half at the 13,863rd step."""
    theta = np.ones(1)
    z = np.zeros(1)
    t_half = None
    for t in range(1, 14000):
        theta, _, _ = adamw_tensor_ref(theta, z, z, z, t, 5e-3, eps=1e-6, weight_decay=1e-2,
                                       store_f32=False)
        if theta[0] <= 0.5:
            t_half = t
            break
    assert t_half == 13863


def _torch_adamw(tensors, grads_seq, lr, betas, eps, wd, decay):
    ps = [torch.tensor(t, dtype=torch.float64, requires_grad=True) for t in tensors]
    groups = [{"params": [p], "weight_decay": wd if d else 0.0} for p, d in zip(ps, decay)]
    opt = torch.optim.AdamW(groups, lr=lr, betas=betas, eps=eps)
    for grads in grads_seq:
        for p, g in zip(ps, grads):
            p.grad = torch.tensor(g, dtype=torch.float64)
        opt.step()
    return [p.detach().numpy() for p in ps], opt


def _oracle_multi(tensors, grads_seq, lr, betas, eps, wd, decay, step_fn=None):
    ps = [np.array(t, np.float64) for t in tensors]
    us = [np.zeros_like(p) for p in ps]
    vs = [np.zeros_like(p) for p in ps]
    for t, grads in enumerate(grads_seq, start=1):
        if step_fn is None:
            ps, us, vs = adamw_step_ref(ps, grads, us, vs, t, lr, betas[0], betas[1], eps, wd, decay,
                                        store_f32=False)
        else:
            out = [step_fn(p, g, u, v, t, lr, betas[0], betas[1], eps, wd if d else 0.0)
                   for p, g, u, v, d in zip(ps, grads, us, vs, decay)]
            ps, us, vs = [o[0] for o in out], [o[1] for o in out], [o[2] for o in out]
    return ps, us, vs


def _torch_case():
    rng = np.random.default_rng(5)
    shapes = [(7,), (3, 5), (2, 3, 4), (1,)]
    tensors = [rng.standard_normal(s) for s in shapes]
    grads_seq = [[rng.standard_normal(s) * 0.1 for s in shapes] for _ in range(25)]
    return tensors, grads_seq, [True, True, False, False]


def test_matches_torch_adamw_fp64():
    tensors, grads_seq, decay = _torch_case()
    for lr, betas, eps, wd in ((1e-2, (0.9, 0.999), 1e-8, 0.1), (6e-4, (0.9, 0.95), 1e-6, 1e-2)):
        want, opt = _torch_adamw(tensors, grads_seq, lr, betas, eps, wd, decay)
        got, us, vs = _oracle_multi(tensors, grads_seq, lr, betas, eps, wd, decay)
        for w, g in zip(want, got):
            np.testing.assert_allclose(g, w, rtol=1e-13, atol=1e-15)
        # the running averages are torch's exp_avg / exp_avg_sq
        for grp, u, v in zip(opt.param_groups, us, vs):
            st = opt.state[grp["params"][0]]
            np.testing.assert_allclose(u, st["exp_avg"].numpy(), rtol=1e-13, atol=1e-18)
            np.testing.assert_allclose(v, st["exp_avg_sq"].numpy(), rtol=1e-13, atol=1e-20)


def test_no_decay_group_ignores_lambda():
    rng = np.random.default_rng(6)
    p = [rng.standard_normal(10) for _ in range(2)]
    g = [rng.standard_normal(10) for _ in range(2)]
    z = [np.zeros(10)] * 2
    a, _, _ = adamw_step_ref(p, g, z, z, 1, 1e-2, weight_decay=0.5, decay=[False, True])
    b, _, _ = adamw_step_ref(p, g, z, z, 1, 1e-2, weight_decay=0.0)
    np.testing.assert_array_equal(a[0], b[0])
    assert not np.array_equal(a[1], b[1])


def test_store_f32_is_one_rounding_of_fp64():
    rng = np.random.default_rng(7)
    p, g, u = (rng.standard_normal(100).astype(np.float32) for _ in range(3))
    v = (rng.standard_normal(100).astype(np.float32)) ** 2
    e = adamw_tensor_ref(p, g, u, v, 7, 1e-3, weight_decay=0.1, store_f32=False)
    r = adamw_tensor_ref(p, g, u, v, 7, 1e-3, weight_decay=0.1)
    for x, y in zip(e, r):
        assert y.dtype == np.float32
        np.testing.assert_array_equal(y, x.astype(np.float32))


# ---------------------------------------------------------------- planted mistakes

def _no_bias_correction(p, g, u, v, t, lr, b1, b2, eps, wd):
    th = p * (1 - lr * wd)
    u = b1 * u + (1 - b1) * g
    v = b2 * v + (1 - b2) * g * g
    return th - lr * u / (np.sqrt(v) + eps), u, v


def _decay_after_step(p, g, u, v, t, lr, b1, b2, eps, wd):
    th, u, v = adamw_tensor_ref(p, g, u, v, t, lr, b1, b2, eps, 0.0, store_f32=False)
    return th * (1 - lr * wd), u, v


def _eps_inside_sqrt(p, g, u, v, t, lr, b1, b2, eps, wd):
    th = p * (1 - lr * wd)
    u = b1 * u + (1 - b1) * g
    v = b2 * v + (1 - b2) * g * g
    return th - lr * (u / (1 - b1 ** t)) / np.sqrt(v / (1 - b2 ** t) + eps), u, v


def _pytorch_sgd_style_average(p, g, u, v, t, lr, b1, b2, eps, wd):
    th = p * (1 - lr * wd)
    u = b1 * u + g                       # (1 - beta1) dropped
    v = b2 * v + (1 - b2) * g * g
    return th - lr * (u / (1 - b1 ** t)) / (np.sqrt(v / (1 - b2 ** t)) + eps), u, v


def _bias_correction_off_by_one(p, g, u, v, t, lr, b1, b2, eps, wd):
    return adamw_tensor_ref(p, g, u, v, t + 1, lr, b1, b2, eps, wd, store_f32=False)


@pytest.mark.parametrize("mutant", [_no_bias_correction, _decay_after_step, _eps_inside_sqrt,
                                    _pytorch_sgd_style_average, _bias_correction_off_by_one])
def test_planted_mistakes_fail_a_pin(mutant, golden_dir):
    tensors, grads_seq, decay = _torch_case()
    want, _ = _torch_adamw(tensors, grads_seq, 1e-2, (0.9, 0.999), 1e-8, 0.1, decay)
    got, _, _ = _oracle_multi(tensors, grads_seq, 1e-2, (0.9, 0.999), 1e-8, 0.1, decay, step_fn=mutant)
    torch_ok = all(np.allclose(g, w, rtol=1e-13, atol=1e-15) for g, w in zip(got, want))
    assert not (torch_ok and _worked_example_ok(mutant, golden_dir))
