"""The tensor-core accumulation model (tests/tc_model.py), pinned, and what it
says about the 1e-2 bar on momentum trajectories.  CPU only.

The bar: the X thread ("New training speed record for @karpathy's
124M-parameter NanoGPT setup", tweets 5/8-6/8) runs the quintic iteration in
bfloat16, and the oracle rounds each stored matrix from the exact product.
Any fp32-accumulating implementation differs from that in rare bf16
roundings, which the chaotic iteration amplifies.  These tests show, on the
GPT-2 block trajectory, that at step 8 both the tensor core's truncating
accumulation and even round-to-nearest fp32 accumulation (with or without
split-K) land more than 1e-2 from the oracle, so the GPU parity tests hold
momentum-trajectory steps to 2e-2 and check separately (on the GPU) that
the GPU tracks this model step by step.
"""
from fractions import Fraction

import numpy as np
import pytest

from oracle import bf16_round, momentum_ref, orthogonalize_ref
from tests.gpu_util import rel_fro
from tests.tc_model import accumulate, orthogonalize_tc, round_toward_zero_f32
from workloads import WORKLOADS, WorkloadStream

COEFFS = (3.4445, -4.7750, 2.0315)


def _rz_by_nextafter(x):
    """Independent route to truncation: round to nearest fp32, then step one
    fp32 value toward zero where that went past x."""
    y = np.asarray(x, np.float64).astype(np.float32)
    over = np.abs(y.astype(np.float64)) > np.abs(x)
    y[over] = np.nextafter(y[over], np.float32(0))
    return y.astype(np.float64)


def test_round_toward_zero_matches_definition():
    rng = np.random.default_rng(0)
    x = rng.standard_normal(100000) * np.exp(rng.uniform(-40, 40, 100000))
    got = round_toward_zero_f32(x)
    assert np.array_equal(got, _rz_by_nextafter(x))
    assert np.all(np.abs(got) <= np.abs(x))
    assert np.array_equal(got.astype(np.float32).astype(np.float64), got)   # fp32 values
    f = x.astype(np.float32).astype(np.float64)
    assert np.array_equal(round_toward_zero_f32(f), f)                       # fixed points
    assert np.array_equal(round_toward_zero_f32(-x), -got)                   # odd


def _exact_dot(p, q):
    return sum(Fraction(float(a)) * Fraction(float(b)) for a, b in zip(p, q))


def test_one_group_is_the_truncated_exact_sum():
    """K <= 16: one MMA group, one addition into a zero accumulator, so the
    model's result is the exact dot product truncated (or rounded) once."""
    rng = np.random.default_rng(1)
    P = bf16_round(rng.standard_normal((5, 16)))
    Q = bf16_round(rng.standard_normal((16, 7)))
    got_t = accumulate(P, Q, "trunc")
    got_n = accumulate(P, Q, "rn")
    for i in range(5):
        for j in range(7):
            e = _exact_dot(P[i], Q[:, j])
            assert got_t[i, j] == float(round_toward_zero_f32(np.array([float(e)]))[0])
            assert abs(Fraction(got_t[i, j])) <= abs(e)
            assert got_n[i, j] == float(np.float32(float(e)))


def test_groups_add_in_k_order_with_one_rounding_each():
    """K = 48: three groups added in order, each addition truncated: checked
    against the same recurrence in exact rationals."""
    rng = np.random.default_rng(2)
    P = bf16_round(rng.standard_normal((3, 48)))
    Q = bf16_round(rng.standard_normal((48, 4)))
    got = accumulate(P, Q, "trunc")
    for i in range(3):
        for j in range(4):
            acc = Fraction(0)
            for k0 in range(0, 48, 16):
                t = acc + _exact_dot(P[i, k0:k0 + 16], Q[k0:k0 + 16, j])
                acc = Fraction(float(round_toward_zero_f32(np.array([float(t)]))[0]))
            assert got[i, j] == float(acc)


def test_split_k_partials_cover_consecutive_ranges():
    """splits = 2 over K = 128 (two 64-wide stages): partial 0 takes the first
    stage, partial 1 the second, and the two are added once in fp32."""
    rng = np.random.default_rng(3)
    P = bf16_round(rng.standard_normal((4, 128)))
    Q = bf16_round(rng.standard_normal((128, 4)))
    a0 = accumulate(P[:, :64], Q[:64], "trunc")
    a1 = accumulate(P[:, 64:], Q[64:], "trunc")
    want = (a0 + a1).astype(np.float32).astype(np.float64)
    assert np.array_equal(accumulate(P, Q, "trunc", splits=2), want)


def test_model_rounds_like_the_oracle_when_nothing_is_inexact():
    """A diagonal input with power-of-two entries: every product and sum is
    exact in fp32, so the model's iteration equals the oracle's exactly."""
    x = np.zeros((8, 12))
    for i in range(8):
        x[i, i] = 2.0 ** -(i + 1)
    u = x * 3.0
    a = orthogonalize_tc(u, 5, COEFFS)
    b = orthogonalize_ref(u, 5, COEFFS)
    assert rel_fro(a, b) < 2e-3            # only the fp32 epilogue roundings differ


def _block_u(i, step):
    """u of matrix i at the given step (from 1) of the GPT-2 block trajectory."""
    wl = WORKLOADS["gpt2_block"]
    st = WorkloadStream(wl, seed=0)
    _, bufs = st.init()
    for k in range(step):
        grads = st.next_grads()
        if k < step - 1:
            for j in range(len(bufs)):
                bufs[j] = momentum_ref(grads[j], bufs[j], wl.beta, wl.nesterov)[0].astype(np.float32)
    _, u = momentum_ref(grads[i], bufs[i], wl.beta, wl.nesterov)
    return u


@pytest.mark.slow
def test_fp32_accumulation_misses_one_percent_at_trajectory_step_8():
    """GPT-2 block, c_attn (768 x 2304), step 8 of the momentum trajectory:
    truncating accumulation (the tensor core), split-K over four partial
    accumulators, and round-to-nearest fp32 accumulation all land more than
    1e-2 from the oracle (1.34%, 1.18% and 1.05% when written), while a
    zero-momentum step stays inside it."""
    u = _block_u(0, 8)
    ref = orthogonalize_ref(u, 5, COEFFS)
    e_trunc = rel_fro(orthogonalize_tc(u, 5, COEFFS, "trunc"), ref)
    e_split = rel_fro(orthogonalize_tc(u, 5, COEFFS, "trunc", splits=4), ref)
    e_rn = rel_fro(orthogonalize_tc(u, 5, COEFFS, "rn"), ref)
    print(f"step 8: truncating {e_trunc:.4%}, split-K x4 {e_split:.4%}, nearest {e_rn:.4%}")
    assert e_trunc > e_split > e_rn > 1e-2
    assert e_trunc < 2e-2
    u1 = _block_u(0, 1)                      # zero momentum: the first step
    e1 = rel_fro(orthogonalize_tc(u1, 5, COEFFS, "trunc"), orthogonalize_ref(u1, 5, COEFFS))
    print(f"step 1: truncating {e1:.4%}")
    assert e1 < 1e-2
