"""Pins of the CPU oracle against facts that do not come from the oracle.

Each test checks the oracle against something fixed independently of it:
hand-worked values (tests/golden/), a library routine (torch's bfloat16 cast,
LAPACK's SVD), the spectral closed form of the iteration (tests/spectral.py),
exact rational arithmetic, brute force on tiny inputs, or an invariant of the
mathematics.  A dropped term, a wrong sign, a swapped coefficient or a
transposed operand anywhere in the oracle fails at least one of them.
"""
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

from oracle import (EPS, BF16_MAX, bf16_round, coeffs_f32, f32_round, momentum_ref,
                    muon_step_ref, newton_schulz_ref, normalize_ref, orient,
                    orthogonalize_ref, update_scale)
from tests.spectral import (closed_form_ns, lift_threshold, poly_scalar,
                            poly_sequence_exact, rel_fro)

COEFFS = (3.4445, -4.7750, 2.0315)


def _golden(golden_dir, name):
    rows = []
    with open(os.path.join(golden_dir, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append([float(t) for t in line.split()])
    return np.array(rows)


# ---------------------------------------------------------------- bf16 rounding

def test_bf16_round_matches_torch_on_fp32_values():
    rng = np.random.default_rng(1)
    x = np.concatenate([
        rng.standard_normal(200000).astype(np.float32),
        (rng.standard_normal(20000) * 1e-38).astype(np.float32),   # bf16 subnormal range
        (rng.standard_normal(20000) * 1e30).astype(np.float32),
        np.array([0.0, -0.0, np.inf, -np.inf, 3.389e38, 3.3961e38, -3.4e38,
                  1e-45, -1e-45, 2.0 ** -126, 2.0 ** -133, 1.5 * 2.0 ** -133], np.float32),
    ])
    # exact ties: 1 + (2k+1) * 2^-8 and their negatives
    k = np.arange(0, 128)
    ties = (1.0 + (2 * k + 1) * 2.0 ** -8).astype(np.float32)
    x = np.concatenate([x, ties, -ties])
    ours = bf16_round(x.astype(np.float64))
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    same = (ours == ref) | (np.isnan(ours) & np.isnan(ref))
    assert same.all(), x[~same][:10]


def test_bf16_round_nan_and_ties_by_hand():
    assert np.isnan(bf16_round(np.array([np.nan]))[0])
    # ties to even: 1 + 2^-8 sits halfway between 1 and 1 + 2^-7 -> 1 (even)
    assert bf16_round(np.array([1.0 + 2.0 ** -8]))[0] == 1.0
    # 1 + 3*2^-8 sits halfway between 1+2^-7 and 1+2^-6 -> 1 + 2^-6 (even)
    assert bf16_round(np.array([1.0 + 3 * 2.0 ** -8]))[0] == 1.0 + 2.0 ** -6
    # rounding straight from fp64: just above the tie must round up, which a
    # detour through fp32 would lose (fp32 drops the 2^-40 and lands on the tie)
    assert bf16_round(np.array([1.0 + 2.0 ** -8 + 2.0 ** -40]))[0] == 1.0 + 2.0 ** -7
    # largest finite value and overflow at the halfway point to 2^128
    assert bf16_round(np.array([BF16_MAX]))[0] == BF16_MAX
    assert np.isinf(bf16_round(np.array([(2.0 - 2.0 ** -8) * 2.0 ** 127]))[0])
    assert bf16_round(np.array([(2.0 - 2.0 ** -8) * 2.0 ** 127 * (1 - 1e-12)]))[0] == BF16_MAX


def test_f32_round_is_ieee():
    x = np.array([1.0 + 2.0 ** -24, 1.0 + 3 * 2.0 ** -24, 0.1])
    assert f32_round(x)[0] == 1.0
    assert f32_round(x)[1] == 1.0 + 2.0 ** -22
    assert f32_round(x)[2] == float(np.float32(0.1))


# ---------------------------------------------------------------- momentum

def test_momentum_hand_worked(golden_dir):
    tab = _golden(golden_dir, "momentum_scalar.txt")
    g = np.ones((2, 3), np.float32)
    buf = np.zeros((2, 3), np.float32)
    for step, buf_exp, u_exp in tab:
        buf_new, u = momentum_ref(g, buf, 0.95, nesterov=True)
        np.testing.assert_allclose(buf_new, buf_exp, rtol=1e-6)
        np.testing.assert_allclose(u, u_exp, rtol=1e-6)
        _, u_plain = momentum_ref(g, buf, 0.95, nesterov=False)
        np.testing.assert_array_equal(u_plain, buf_new)
        buf = buf_new.astype(np.float32)


def test_momentum_is_one_fp32_rounding():
    # beta*buf + g with values whose exact result is representable: no error
    g = np.array([0.5, -0.25], np.float32)
    buf = np.array([2.0, 4.0], np.float32)
    buf_new, u = momentum_ref(g, buf, 0.5, nesterov=True)
    np.testing.assert_array_equal(buf_new, [1.5, 1.75])
    np.testing.assert_array_equal(u, [0.5 + 0.75, -0.25 + 0.875])


# ---------------------------------------------------------------- normalisation

def test_normalize_hand_worked(golden_dir):
    tab = _golden(golden_dir, "normalize_3_4.txt")
    x0 = normalize_ref(np.array([[3.0, 4.0]]))
    np.testing.assert_array_equal(x0, tab)


def test_normalize_unit_norm_and_zero():
    rng = np.random.default_rng(2)
    u = rng.standard_normal((64, 200)) * 37.0
    x0 = normalize_ref(u)
    assert abs(np.linalg.norm(x0) - 1.0) < 2.0 ** -8
    assert np.all(x0 == bf16_round(x0))
    z = normalize_ref(np.zeros((4, 8)))
    assert np.all(z == 0) and not np.any(np.isnan(z))


def test_orient():
    x = np.arange(6.0).reshape(3, 2)
    y, t = orient(x)
    assert t and y.shape == (2, 3) and np.all(y == x.T)
    y, t = orient(x.T)
    assert not t and y.shape == (2, 3)
    y, t = orient(np.eye(3))
    assert not t


# ---------------------------------------------------------------- Newton-Schulz

def test_scalar_sequences_exact_rational():
    """Closed-form factor sequences of p from exact rational arithmetic."""
    # rank-1 input: the one singular value is 1 after normalisation
    seq = [float(v) for v in poly_sequence_exact(1)]
    np.testing.assert_allclose(seq, [0.701000, 1.113620, 0.720706, 1.089974, 0.696436], atol=5e-7)
    # 256x256 orthogonal input: all singular values 1/16 after normalisation
    seq = [float(v) for v in poly_sequence_exact(Fraction(1, 16))]
    np.testing.assert_allclose(seq, [0.214117, 0.691568, 1.124117, 0.735722, 1.070524], atol=5e-7)
    # 2x2 orthogonal input: singular values 2^-1/2
    seq = [float(v) for v in poly_sequence_exact(2 ** -0.5)]
    np.testing.assert_allclose(seq, [1.106534, 0.712085, 1.100594, 0.705764, 1.108111], atol=5e-7)


def test_ns_rank1_exact():
    rng = np.random.default_rng(3)
    u = rng.standard_normal(5)
    v = rng.standard_normal(9)
    x0 = np.outer(u, v)
    x0 /= np.linalg.norm(x0)
    x = newton_schulz_ref(x0, 5, COEFFS, exact=True)
    p5 = float(poly_sequence_exact(1)[-1])
    np.testing.assert_allclose(x, p5 * x0, rtol=1e-12, atol=1e-14)


def test_ns_orthogonal_input_exact():
    rng = np.random.default_rng(4)
    q, _ = np.linalg.qr(rng.standard_normal((16, 16)))
    x = newton_schulz_ref(q / 4.0, 5, COEFFS, exact=True)   # ||q||_F = 4
    np.testing.assert_allclose(x, float(poly_sequence_exact(Fraction(1, 4))[-1]) * q, atol=1e-12)


@pytest.mark.parametrize("m,n", [(2, 2), (4, 4), (3, 7), (8, 20), (33, 47)])
def test_ns_matches_svd_closed_form_exact(m, n):
    """fp64 iteration vs U p^5(S) V^T from LAPACK's SVD (independent route)."""
    rng = np.random.default_rng(100 + m * n)
    g = rng.standard_normal((m, n))
    x0 = g / np.linalg.norm(g)
    for steps in (1, 2, 5):
        x = newton_schulz_ref(x0, steps, COEFFS, exact=True)
        np.testing.assert_allclose(x, closed_form_ns(x0, COEFFS, steps), atol=1e-12)


def test_ns_other_coefficients_exact():
    """The coefficients enter in their own places: a on X, b on A, c on A^2."""
    rng = np.random.default_rng(5)
    g = rng.standard_normal((6, 10))
    x0 = g / np.linalg.norm(g)
    for co in [(1.0, 0.0, 0.0), (0.0, 1.0, 0.0), (0.0, 0.0, 1.0), (1.875, -1.25, 0.375),
               (2.0, -1.5, 0.5)]:
        x = newton_schulz_ref(x0, 3, co, exact=True)
        np.testing.assert_allclose(x, closed_form_ns(x0, co, 3), atol=1e-12)


def test_ns_diagonal_input_follows_scalar_map_bf16():
    """A diagonal X stays diagonal; entry i follows p with bf16 storage points."""
    d = np.array([0.9, 0.3, 0.05, 0.01, 0.002, 0.0])
    x0 = bf16_round(np.diag(d / np.linalg.norm(d)))
    x = newton_schulz_ref(x0, 5, COEFFS)
    off = x - np.diag(np.diag(x))
    assert np.all(off == 0)
    a, b, c = coeffs_f32(COEFFS)
    s = np.diag(x0).copy()
    for _ in range(5):       # scalar emulation: A = s^2, B = b A + c A^2, s = a s + B s
        A = bf16_round(s * s)
        B = bf16_round(b * A + c * A * A)
        s = bf16_round(a * s + B * s)
    np.testing.assert_array_equal(np.diag(x), s)


def test_ns_bf16_close_to_closed_form():
    rng = np.random.default_rng(6)
    g = rng.standard_normal((48, 128))
    x0 = bf16_round(g / np.linalg.norm(g))
    x = newton_schulz_ref(x0, 5, COEFFS)
    assert rel_fro(x, closed_form_ns(x0, COEFFS, 5)) < 3e-2
    assert np.all(x == bf16_round(x))


def test_ns_trace_storage_points_are_bf16():
    rng = np.random.default_rng(7)
    g = rng.standard_normal((16, 40))
    x0 = bf16_round(g / np.linalg.norm(g))
    x, hist = newton_schulz_ref(x0, 3, COEFFS, trace=True)
    assert len(hist) == 3 and np.all(hist[-1][2] == x)
    for A, B, X in hist:
        assert A.shape == (16, 16) and B.shape == (16, 16) and X.shape == (16, 40)
        for t in (A, B, X):
            assert np.all(t == bf16_round(t))
        assert np.all(A == A.T) and np.all(B == B.T)


def test_ns_rejects_tall():
    with pytest.raises(ValueError):
        newton_schulz_ref(np.zeros((5, 3)), 1, COEFFS)


def test_ns_zero_steps_identity():
    x0 = bf16_round(np.random.default_rng(8).standard_normal((4, 6)) / 5)
    assert np.all(newton_schulz_ref(x0, 0, COEFFS) == x0)


# ---------------------------------------------------------------- invariances

def test_transpose_invariance_bitwise():
    rng = np.random.default_rng(9)
    u = rng.standard_normal((24, 56))
    x_wide = orthogonalize_ref(u, 5, COEFFS)
    x_tall = orthogonalize_ref(u.T, 5, COEFFS)
    assert np.array_equal(x_tall, x_wide.T)


def test_sign_invariance_bitwise():
    rng = np.random.default_rng(10)
    u = rng.standard_normal((20, 30))
    assert np.array_equal(orthogonalize_ref(-u, 5, COEFFS), -orthogonalize_ref(u, 5, COEFFS))


def test_orthogonal_equivariance_exact():
    rng = np.random.default_rng(11)
    g = rng.standard_normal((6, 9))
    q1, _ = np.linalg.qr(rng.standard_normal((6, 6)))
    q2, _ = np.linalg.qr(rng.standard_normal((9, 9)))
    a = orthogonalize_ref(q1 @ g @ q2.T, 5, COEFFS, exact=True)
    b = q1 @ orthogonalize_ref(g, 5, COEFFS, exact=True) @ q2.T
    np.testing.assert_allclose(a, b, atol=1e-10)


# ---------------------------------------------------------------- singular-value band

def test_singular_value_band_closed_form():
    s = np.linspace(1e-6, 1.0, 200001)
    y = poly_scalar(s, COEFFS, 5)
    assert y.max() <= 1.2025
    thr = lift_threshold(0.6)
    assert 1.29e-3 < thr < 1.31e-3
    assert np.all(y[s >= thr] >= 0.6 - 1e-12)
    assert np.all(y[s < thr * 0.999] < 0.6)
    # max of p on [0, 1] is at s* solving p'(s) = a + 3 b s^2 + 5 c s^4 = 0
    a, b, c = coeffs_f32(COEFFS)
    s2 = (-3 * b - math.sqrt(9 * b * b - 20 * a * c)) / (10 * c)
    smax = math.sqrt(s2)
    assert abs(smax - 0.5545) < 1e-3 and abs(poly_scalar(smax, COEFFS, 1) - 1.2024) < 1e-3


def test_oracle_output_band_bf16():
    rng = np.random.default_rng(12)
    g = rng.standard_normal((64, 160))
    x = orthogonalize_ref(g, 5, COEFFS)
    sv_in = np.linalg.svd(g / np.linalg.norm(g), compute_uv=False)
    sv = np.linalg.svd(x, compute_uv=False)
    assert sv.max() <= 1.2024 + 0.02
    thr = lift_threshold(0.6)
    # directions lifted above 0.6 by the closed form stay there in bf16
    assert np.sum(sv >= 0.6 - 0.02) >= np.sum(sv_in >= thr)


# ---------------------------------------------------------------- full step

def test_update_scale():
    assert update_scale(3072, 768, 0.02) == float(np.float32(0.04))
    assert update_scale(768, 3072, 0.02) == float(np.float32(0.02))
    assert update_scale(256, 256, 0.02) == float(np.float32(0.02))
    assert update_scale(300, 100, 1.0) == float(np.float32(math.sqrt(3.0)))


def test_zero_gradient_leaves_params():
    p = [np.random.default_rng(13).standard_normal((8, 12)).astype(np.float32)]
    z = [np.zeros((8, 12), np.float32)]
    newp, newb = muon_step_ref(p, z, [z[0].copy()], lr=0.02)
    assert np.array_equal(newp[0], p[0]) and np.all(newb[0] == 0)


@pytest.mark.parametrize("shape", [(12, 40), (40, 12), (16, 16)])
def test_step_matches_spectral_closed_form(shape):
    """First step from zero momentum: u = (1+beta) g, so the applied update is
    -lr*s * U p^5(S/||S||) V^T of g itself (bf16-level agreement)."""
    r, c = shape
    rng = np.random.default_rng(14 + r)
    p = (rng.standard_normal(shape) * 0.02).astype(np.float32)
    g = rng.standard_normal(shape).astype(np.float32)
    buf = np.zeros(shape, np.float32)
    newp, newb, xs = muon_step_ref([p], [g], [buf], lr=0.02, return_x=True)
    np.testing.assert_array_equal(newb[0], g)
    s = math.sqrt(max(1.0, r / c))
    expected_dp = -0.02 * s * closed_form_ns(g / np.linalg.norm(g), COEFFS, 5)
    dp = newp[0].astype(np.float64) - p
    assert rel_fro(dp, expected_dp) < 3e-2
    # the stored update is exactly the bf16 X times the fp32 scale, one fp32 rounding
    np.testing.assert_array_equal(newp[0], f32_round(p - update_scale(r, c, 0.02) * xs[0]))


def test_step_nan_stays_in_its_matrix():
    rng = np.random.default_rng(15)
    ps = [rng.standard_normal((4, 6)).astype(np.float32) for _ in range(2)]
    gs = [rng.standard_normal((4, 6)).astype(np.float32) for _ in range(2)]
    gs[0][1, 2] = np.nan
    bs = [np.zeros((4, 6), np.float32) for _ in range(2)]
    newp, _ = muon_step_ref(ps, gs, bs, lr=0.02)
    assert np.isnan(newp[0]).any() and np.isfinite(newp[1]).all()


def test_step_rejects_1d():
    with pytest.raises(ValueError):
        muon_step_ref([np.zeros(4, np.float32)], [np.zeros(4, np.float32)],
                      [np.zeros(4, np.float32)], lr=0.1)


def test_eps_value():
    assert EPS == 1e-7
