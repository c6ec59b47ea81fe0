"""GPU parity: every kernel of the Muon step, through the C-ABI, against the
CPU oracle on the same seeded inputs.

Tolerances (from the arithmetic, stated per check):
* momentum buffers: both sides do one fp32 rounding of beta*buf + g, so the
  relative error is at most one fp32 ulp (<= 1.2e-7); the bar is 1e-6.
* X0: both sides divide the same fp32 u by the norm in (at least) double
  precision before one bf16 rounding: at most 1 bf16 ulp apart.
* bf16 GEMM stage outputs (A, B, X1): the GPU accumulates in fp32, the oracle
  in fp64.  Each difference must stay within 1 bf16 ulp plus the rigorous
  fp32 accumulation bound 2 K 2^-24 (|P||Q|)_ij of the product P Q (which
  matters only for entries that cancel to near zero), and differ on at most
  1% of entries.
* orthogonalised update (Delta p = -lr*s*X5) and new parameters: relative
  Frobenius error <= 1e-2 (X_TOL) for a single orthogonalisation and for a
  step from zero momentum (measured <= 0.82%).
* steps taken after momentum has accumulated (every GPT-2 124M, medium and XL
  step, steps 2-10 of the GPT-2 block): <= 2e-2 (X_TOL_TRAJ), because 1e-2
  is out of reach of the tensor core's arithmetic, not of the kernels.
  The bf16 iteration is chaotic: directions with small singular values grow
  up to a = 3.44-fold per iteration, so any difference in an accumulation
  that flips a bf16 rounding grows with every iteration.  The tensor core
  adds each exact 16-product sum into an fp32 accumulator truncated toward
  zero; tests/tc_model.py models that, and its distance from the oracle
  matches the GPU's step by step (checked below, on the GPU, on every step
  of the GPT-2 block trajectory).  At step 8 of that trajectory (768 x 2304)
  the model lands 1.34% from the oracle (the GPU 1.30%); split-K
  accumulation over four partial accumulators would still land 1.18% away,
  and round-to-nearest fp32 accumulation, which this hardware does not offer,
  1.05% (tests/test_tc_model.py pins both of the latter above 1e-2).  Over
  the first three steps of the GPT-2 124M workload (48 matrices each) the
  model lands 1.20%, 1.34% and 1.45% from the oracle on average and 1.53%
  at most (the GPU 1.50% at most), growing with the momentum: 2e-2 leaves
  room for that tail.  Local errors that a whole-step bar cannot see are
  the per-stage tests' job: each kernel's own output is held to one bf16 ulp
  plus the accumulation bound above.
"""
import math

import numpy as np
import pytest
import torch

from oracle import (coeffs_f32, momentum_ref, muon_step_ref, newton_schulz_ref, normalize_ref,
                    orient, orthogonalize_ref)
from tests.gpu_util import (bf16_agreement, bf16_close, fp32_gemm_bound, rel_fro, to_bf16, to_f32,
                            to_np)
from tests.spectral import band_report, lift_threshold, poly_scalar
from tests.tc_model import orthogonalize_tc
from workloads import WORKLOADS, WorkloadStream, square_case

pytestmark = pytest.mark.gpu

COEFFS = (3.4445, -4.7750, 2.0315)
X_TOL = 1e-2          # one orthogonalisation / a step from zero momentum
X_TOL_TRAJ = 2e-2     # steps after momentum has accumulated (see module docstring)
BUF_TOL = 1e-6


@pytest.fixture(scope="module")
def muon():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from newton_schulz_norm_b200 import build
    build.build()
    import newton_schulz_norm_b200 as m
    m.set_wait_limit_ns(2_000_000_000)
    yield m
    assert m.status() == 0


def _rng(seed):
    return np.random.default_rng(seed)


# ---------------------------------------------------------------- first kernel

SHAPES_K1 = [(256, 256), (64, 200), (200, 64), (7, 13), (13, 7), (1, 1), (1, 100), (100, 1),
             (129, 257), (257, 129), (768, 2304), (3072, 768), (65, 66)]


@pytest.mark.parametrize("nesterov", [True, False])
def test_momentum_normalize_stage(muon, nesterov):
    rng = _rng(1)
    gs = [rng.standard_normal(s).astype(np.float32) for s in SHAPES_K1]
    bs = [(rng.standard_normal(s) * 0.1).astype(np.float32) for s in SHAPES_K1]
    g_d = [to_f32(g) for g in gs]
    b_d = [to_f32(b) for b in bs]
    x0_d = muon.momentum_normalize(g_d, b_d, beta=0.95, nesterov=nesterov)
    torch.cuda.synchronize()
    assert muon.status() == 0
    for g, b, bd, xd in zip(gs, bs, b_d, x0_d):
        buf_ref, u = momentum_ref(g, b, 0.95, nesterov)
        got = to_np(bd)
        assert np.max(np.abs(got - buf_ref)) <= BUF_TOL * max(np.max(np.abs(buf_ref)), 1e-30)
        x0_ref, _ = orient(normalize_ref(u))
        x0 = to_np(xd)
        assert x0.shape == x0_ref.shape
        mism, ulps = bf16_agreement(x0, x0_ref)
        assert ulps <= 1.0 and mism <= 1e-3, (g.shape, mism, ulps)


def test_momentum_three_steps_exact_match(muon):
    """Hand-worked recurrence (g = 1, beta = 0.95) through the GPU kernel."""
    g = torch.ones((16, 24), device="cuda")
    b = torch.zeros((16, 24), device="cuda")
    expect_buf = [1.0, 1.95, 2.8525]
    for e in expect_buf:
        muon.momentum_normalize([g], [b], beta=0.95, nesterov=True)
        torch.cuda.synchronize()
        np.testing.assert_allclose(to_np(b), e, rtol=1e-6)


# ---------------------------------------------------------------- NS stages

NS_SHAPES = [(7, 20), (64, 64), (128, 256), (200, 333), (256, 1024), (768, 768), (768, 3072),
             (130, 300), (1, 9), (600, 1000)]


def _trace_inputs(m, n, seed):
    rng = _rng(seed)
    g = rng.standard_normal((m, n))
    x0 = normalize_ref(g)
    x1, hist = newton_schulz_ref(x0, 1, COEFFS, trace=True)
    A, B, X1 = hist[0]
    return x0, A, B, X1


@pytest.mark.parametrize("m,n", NS_SHAPES)
def test_gram_stage(muon, m, n):
    x0, A, _, _ = _trace_inputs(m, n, 10 + m)
    a = to_np(muon.gram(to_bf16(x0)))
    torch.cuda.synchronize()
    mism, _ = bf16_agreement(a, A)
    ratio = bf16_close(a, A, fp32_gemm_bound(x0, x0.T, n))
    assert ratio <= 1.0 and mism <= 1e-2, (mism, ratio)
    assert np.array_equal(a, a.T)


@pytest.mark.parametrize("m,n", NS_SHAPES)
def test_poly_stage(muon, m, n):
    _, A, B, _ = _trace_inputs(m, n, 20 + m)
    a, b, c = coeffs_f32(COEFFS)
    out = to_np(muon.poly(to_bf16(A), b, c))
    torch.cuda.synchronize()
    mism, _ = bf16_agreement(out, B)
    # fp32 product A A (m terms) scaled by |c|, plus the fp32 epilogue b*A + c*acc
    bound = abs(c) * fp32_gemm_bound(A, A, m) + 2.0 ** -22 * (abs(b) * np.abs(A) + abs(c) * (np.abs(A) @ np.abs(A)))
    ratio = bf16_close(out, B, bound)
    assert ratio <= 1.0 and mism <= 1e-2, (mism, ratio)
    assert np.array_equal(out, out.T)


@pytest.mark.parametrize("m,n", NS_SHAPES)
def test_xupdate_stage(muon, m, n):
    x0, _, B, X1 = _trace_inputs(m, n, 30 + m)
    a, _, _ = coeffs_f32(COEFFS)
    out = to_np(muon.xupdate(to_bf16(B), to_bf16(x0), a))
    torch.cuda.synchronize()
    mism, _ = bf16_agreement(out, X1)
    bound = fp32_gemm_bound(B, x0, m) + 2.0 ** -22 * (abs(a) * np.abs(x0) + np.abs(B) @ np.abs(x0))
    ratio = bf16_close(out, X1, bound)
    assert ratio <= 1.0 and mism <= 1e-2, (mism, ratio)


# ---------------------------------------------------------------- orthogonalize

@pytest.mark.parametrize("shape", [(256, 256), (64, 200), (200, 64), (300, 1000), (1000, 300),
                                   (5, 5), (1, 33), (33, 1), (768, 3072)])
@pytest.mark.parametrize("steps", [1, 5])
def test_orthogonalize_vs_oracle(muon, shape, steps):
    rng = _rng(40 + shape[0])
    x = rng.standard_normal(shape).astype(np.float32)
    ref = orthogonalize_ref(x, steps, COEFFS)
    out = to_np(muon.orthogonalize(to_f32(x), ns_steps=steps))
    torch.cuda.synchronize()
    assert rel_fro(out, ref) <= X_TOL
    outb = to_np(muon.orthogonalize(to_f32(x), ns_steps=steps, out_dtype=torch.bfloat16))
    np.testing.assert_array_equal(outb, out)   # fp32 output holds the bf16 values


def test_orthogonalize_zero_steps_is_x0(muon):
    rng = _rng(50)
    x = rng.standard_normal((40, 96)).astype(np.float32)
    out = to_np(muon.orthogonalize(to_f32(x), ns_steps=0))
    mism, ulps = bf16_agreement(out, normalize_ref(x))
    assert ulps <= 1.0 and mism <= 1e-3


def test_orthogonalize_singular_values(muon):
    """Output singular values: <= 1.2024 + slack always; >= 0.6 for every
    direction whose normalised input value the closed form lifts above 0.6."""
    rng = _rng(51)
    x = rng.standard_normal((256, 256)).astype(np.float32)
    out = to_np(muon.orthogonalize(to_f32(x), ns_steps=5))
    sv = np.linalg.svd(out, compute_uv=False)
    s0 = np.linalg.svd(x / np.linalg.norm(x), compute_uv=False)
    assert sv.max() <= 1.3
    thr = lift_threshold(0.6)
    assert np.sum(sv >= 0.6 - 0.02) >= np.sum(s0 >= thr)
    # the literal band, reported: most of a Gaussian's spectrum lies in it
    assert np.mean((sv >= 0.6) & (sv <= 1.3)) > 0.9


@pytest.mark.parametrize("n", [1024, 2048])
def test_square_sweep_vs_oracle(muon, n):
    case = square_case(n, seed=0)
    ref = orthogonalize_ref(case.g, 5, COEFFS)
    out = to_np(muon.orthogonalize(to_f32(case.g), ns_steps=5))
    assert rel_fro(out, ref) <= X_TOL
    # closed form through the known factors: U^T X V ~ diag(p^5(sigma/||sigma||))
    d = case.project(out)
    target = poly_scalar(case.sigma / np.linalg.norm(case.sigma), COEFFS, 5)
    assert rel_fro(np.diag(d), target) < 3e-2
    off = d - np.diag(np.diag(d))
    assert np.linalg.norm(off) / np.linalg.norm(target) < 5e-2


def test_square_4096_vs_oracle(muon):
    """The 4096 square of the sweep (randomised-Hadamard factors) against the
    oracle at the 1e-2 bar, and through its known factors."""
    case = square_case(4096, seed=0)
    out = to_np(muon.orthogonalize(to_f32(case.g), ns_steps=5))
    ref = orthogonalize_ref(case.g, 5, COEFFS)
    err = rel_fro(out, ref)
    print(f"n = 4096: GPU vs oracle {err:.4%}")
    assert err <= X_TOL
    d = case.project(out)
    target = poly_scalar(case.sigma / np.linalg.norm(case.sigma), COEFFS, 5)
    assert rel_fro(np.diag(d), target) < 3e-2


# ---------------------------------------------------------------- full step

def _run_step(muon, params, grads, bufs, **kw):
    p_d = [to_f32(p) for p in params]
    g_d = [to_f32(g) for g in grads]
    b_d = [to_f32(b) for b in bufs]
    muon.step(p_d, g_d, b_d, **kw)
    torch.cuda.synchronize()
    return p_d, b_d


def _check_step(p_old, p_gpu, b_gpu, p_ref, b_ref, tol=X_TOL):
    """Momentum buffers to 1e-6; new parameters and each matrix's update to
    tol; the step's update over all matrices together to tol as well."""
    num = den = 0.0
    errs = []
    for po, pg, bg, pr, br in zip(p_old, p_gpu, b_gpu, p_ref, b_ref):
        pg = to_np(pg)
        bg = to_np(bg)
        assert np.max(np.abs(bg - br)) <= BUF_TOL * max(np.max(np.abs(br)), 1e-30)
        assert rel_fro(pg, pr) <= tol
        dp_g = pg - po
        dp_r = np.asarray(pr, np.float64) - po
        num += float(np.sum((dp_g - dp_r) ** 2))
        den += float(np.sum(dp_r ** 2))
        errs.append((po.shape, rel_fro(dp_g, dp_r)))
        assert errs[-1][1] <= tol, errs[-1]
    if den > 0:
        assert math.sqrt(num / den) <= tol, errs


def _step_x(p_old, p_new, lr):
    """The orthogonalised update X5 a step applied, recovered from the
    parameters: p_new = fp32(p_old - s X5), s = fp32(lr sqrt(max(1, r/c)))."""
    r, c = p_old.shape
    s = float(np.float32(float(np.float32(lr)) * math.sqrt(max(1.0, r / c))))
    new = to_np(p_new) if isinstance(p_new, torch.Tensor) else np.asarray(p_new, np.float64)
    return (np.asarray(p_old, np.float64) - new) / s


def _check_band(x5, u, what):
    """The singular-value band of one step's update (see tests/spectral.py):
    max sigma <= 1.3 and every liftable direction lifted to >= 0.6 (- 0.02)."""
    smax, lifted, liftable, literal = band_report(x5, u)
    assert smax <= 1.3, (what, smax)
    assert lifted >= liftable, (what, lifted, liftable)
    return literal


EDGE_SHAPES = [(1, 1), (1, 100), (100, 1), (7, 13), (13, 7), (64, 64), (129, 257), (257, 129),
               (300, 1000), (1000, 300)]


@pytest.mark.parametrize("steps", [0, 1, 2, 5])
def test_step_edge_shapes(muon, steps):
    rng = _rng(60 + steps)
    ps = [(rng.standard_normal(s) * 0.02).astype(np.float32) for s in EDGE_SHAPES]
    gs = [rng.standard_normal(s).astype(np.float32) for s in EDGE_SHAPES]
    bs = [(rng.standard_normal(s) * 0.1).astype(np.float32) for s in EDGE_SHAPES]
    p_d, b_d = _run_step(muon, ps, gs, bs, lr=0.02, ns_steps=steps)
    p_ref, b_ref = muon_step_ref(ps, gs, bs, lr=0.02, ns_steps=steps)
    _check_step(ps, p_d, b_d, p_ref, b_ref)


def test_step_options(muon):
    """nesterov off, another coefficient triple, another lr and beta."""
    rng = _rng(70)
    shapes = [(96, 160), (160, 96), (128, 128)]
    ps = [(rng.standard_normal(s) * 0.02).astype(np.float32) for s in shapes]
    gs = [rng.standard_normal(s).astype(np.float32) for s in shapes]
    bs = [(rng.standard_normal(s) * 0.1).astype(np.float32) for s in shapes]
    co = (1.875, -1.25, 0.375)
    p_d, b_d = _run_step(muon, ps, gs, bs, lr=0.1, beta=0.9, nesterov=False, ns_steps=4, coeffs=co)
    p_ref, b_ref = muon_step_ref(ps, gs, bs, lr=0.1, beta=0.9, nesterov=False, ns_steps=4, coeffs=co)
    _check_step(ps, p_d, b_d, p_ref, b_ref)


def test_step_zero_grad_and_nan_isolation(muon):
    shapes = [(32, 48), (48, 32), (40, 40)]
    rng = _rng(71)
    ps = [(rng.standard_normal(s) * 0.02).astype(np.float32) for s in shapes]
    gs = [np.zeros(shapes[0], np.float32), rng.standard_normal(shapes[1]).astype(np.float32),
          rng.standard_normal(shapes[2]).astype(np.float32)]
    gs[1][3, 5] = np.nan
    bs = [np.zeros(s, np.float32) for s in shapes]
    p_d, b_d = _run_step(muon, ps, gs, bs, lr=0.02)
    assert np.array_equal(to_np(p_d[0]), ps[0])        # zero update leaves p
    assert np.isnan(to_np(p_d[1])).any()               # NaN stays in its matrix
    assert np.isfinite(to_np(p_d[2])).all()
    p_ref, b_ref = muon_step_ref(ps[2:], gs[2:], bs[2:], lr=0.02)
    _check_step(ps[2:], p_d[2:], b_d[2:], p_ref, b_ref)


@pytest.mark.parametrize("name", ["single_256", "gpt2_block"])
def test_step_workloads_consecutive(muon, name):
    """Every step the workload specifies (3 for the single matrix, 10 for the
    GPT-2 block), each compared with the oracle from identical inputs: the two
    trajectories are put back on the oracle's state after every step.  Every
    step's update also passes the singular-value band.

    For the GPT-2 block, every step of the 768 x 768 matrix (attn c_proj) is
    also compared with the tensor-core accumulation model (tests/tc_model.py)
    on the same input: the GPU must land as far from the oracle as the model
    of its truncating fp32 accumulation predicts (within 15% + 0.1%), which
    is what carries these steps past the 1e-2 bar (module docstring)."""
    wl = WORKLOADS[name]
    st = WorkloadStream(wl, seed=0)
    params, bufs = st.init()
    p_d = [to_f32(p) for p in params]
    b_d = [to_f32(b) for b in bufs]
    p_ref = [p.copy() for p in params]
    b_ref = [b.copy() for b in bufs]
    model_rows = []
    for k in range(wl.steps):
        grads = st.next_grads()
        p_old = [p.copy() for p in p_ref]
        b_old = [b.copy() for b in b_ref]
        muon.step(p_d, [to_f32(g) for g in grads], b_d, lr=wl.lr, beta=wl.beta,
                  nesterov=wl.nesterov, ns_steps=wl.ns_steps, coeffs=wl.coeffs)
        torch.cuda.synchronize()
        p_ref, b_ref = muon_step_ref(p_ref, grads, b_ref, lr=wl.lr, beta=wl.beta,
                                     nesterov=wl.nesterov, ns_steps=wl.ns_steps, coeffs=wl.coeffs)
        zero_momentum = k == 0 and wl.buf_std == 0
        _check_step(p_old, p_d, b_d, p_ref, b_ref, tol=X_TOL if zero_momentum else X_TOL_TRAJ)
        for i in range(len(p_d)):
            _, u = momentum_ref(grads[i], b_old[i], wl.beta, wl.nesterov)
            _check_band(_step_x(p_old[i], p_d[i], wl.lr), u, (name, k, i))
        if name == "gpt2_block":
            i = 1
            _, u = momentum_ref(grads[i], b_old[i], wl.beta, wl.nesterov)
            x_ref = orthogonalize_ref(u, wl.ns_steps, wl.coeffs)
            e_gpu = rel_fro(_step_x(p_old[i], p_d[i], wl.lr), x_ref)
            e_model = rel_fro(orthogonalize_tc(u, wl.ns_steps, wl.coeffs), x_ref)
            model_rows.append((k + 1, e_gpu, e_model))
        # keep the two trajectories on the same state, so that each step is
        # compared from identical inputs
        for i in range(len(p_d)):
            p_d[i].copy_(to_f32(p_ref[i]))
            b_d[i].copy_(to_f32(b_ref[i]))
    for k, e_gpu, e_model in model_rows:
        print(f"step {k}: GPU vs oracle {e_gpu:.4%}, tensor-core model vs oracle {e_model:.4%}")
        assert abs(e_gpu - e_model) <= 0.15 * e_model + 1e-3, (k, e_gpu, e_model)
    assert muon.status() == 0


def test_step_gpt2_124m_all_48_first_3_steps(muon):
    """All 48 matrices in one call (the benchmarked launch configuration),
    the first three steps of the workload, every matrix against the oracle
    (momentum is warm-started, so every step is a trajectory step); one
    matrix of each shape per step passes the singular-value band."""
    wl = WORKLOADS["gpt2_124m"]
    st = WorkloadStream(wl, seed=0)
    params, bufs = st.init()
    p_d = [to_f32(p) for p in params]
    b_d = [to_f32(b) for b in bufs]
    p_ref, b_ref = params, bufs
    for k in range(3):
        grads = st.next_grads()
        p_old, b_old = p_ref, b_ref
        muon.step(p_d, [to_f32(g) for g in grads], b_d, lr=wl.lr, beta=wl.beta,
                  nesterov=wl.nesterov, ns_steps=wl.ns_steps, coeffs=wl.coeffs)
        torch.cuda.synchronize()
        assert muon.status() == 0
        p_ref, b_ref = muon_step_ref(p_old, grads, b_old, lr=wl.lr, beta=wl.beta,
                                     nesterov=wl.nesterov, ns_steps=wl.ns_steps, coeffs=wl.coeffs)
        _check_step(p_old, p_d, b_d, p_ref, b_ref, tol=X_TOL_TRAJ)
        for i in (0, 1, 2, 3):
            _, u = momentum_ref(grads[i], b_old[i], wl.beta, wl.nesterov)
            _check_band(_step_x(p_old[i], p_d[i], wl.lr), u, (k, i))
        for i in range(48):
            p_d[i].copy_(to_f32(p_ref[i]))
            b_d[i].copy_(to_f32(b_ref[i]))


def test_update_scale_on_transposed(muon):
    """c_proj-shaped (tall) matrices get sqrt(rows/cols) = 2 times the step."""
    rng = _rng(80)
    g = rng.standard_normal((256, 64)).astype(np.float32)
    p = np.zeros((256, 64), np.float32)
    b = np.zeros((256, 64), np.float32)
    p_d, _ = _run_step(muon, [p], [g], [b], lr=0.5)
    x = orthogonalize_ref((1 + np.float32(0.95)) * g.astype(np.float64), 5, COEFFS)
    dp = to_np(p_d[0])
    assert rel_fro(dp, -1.0 * x) <= X_TOL      # lr * sqrt(256/64) = 0.5 * 2


def test_timeout_reports_status_and_context_survives(muon):
    """A wait limit of 0 makes device-side waits give up: the kernels record
    MUON_ERR_TIMEOUT and return; the next call with the normal limit works."""
    wl = WORKLOADS["gpt2_block"]
    st = WorkloadStream(wl, seed=3)
    params, bufs = st.init()
    grads = st.next_grads()
    seen = 0
    try:
        for _ in range(3):
            muon.set_wait_limit_ns(0)
            _run_step(muon, params, grads, bufs, lr=0.02)
            seen = muon.status()
            if seen != 0:
                break
    finally:
        muon.set_wait_limit_ns(2_000_000_000)
    assert seen == -5
    p_d, b_d = _run_step(muon, params, grads, bufs, lr=0.02)
    assert muon.status() == 0
    p_ref, b_ref = muon_step_ref(params[1:2], grads[1:2], bufs[1:2], lr=0.02)
    _check_step(params[1:2], p_d[1:2], b_d[1:2], p_ref, b_ref)


def test_rejects_bad_args_before_launch(muon):
    p = torch.zeros((8, 8), device="cuda")
    g = torch.ones((8, 8), device="cuda")
    b = torch.zeros((8, 8), device="cuda")
    with pytest.raises(muon.MuonError):
        muon.step([p], [g], [b], lr=float("nan"))
    assert torch.all(p == 0) and torch.all(b == 0)
    with pytest.raises(muon.MuonError):
        muon.step([p], [g], [b], lr=0.1, ns_steps=-1)
    assert torch.all(b == 0)


def _first_step_sampled(muon, wl, sample, band=()):
    """One step on every matrix of the workload in one call; the oracle on
    the matrices in ``sample``.  Inputs are drawn matrix by matrix and moved
    to the GPU at once, so the host keeps only the sampled ones."""
    st = WorkloadStream(wl, seed=0)
    keep = set(sample)
    p_d, b_d, g_d, host = [], [], [], {}
    for i, p, b in st.init_iter():
        p_d.append(to_f32(p))
        b_d.append(to_f32(b))
        if i in keep:
            host[i] = [p, b, None]
    for i, g in st.grads_iter():
        g_d.append(to_f32(g))
        if i in keep:
            host[i][2] = g
    muon.step(p_d, g_d, b_d, lr=wl.lr, beta=wl.beta, nesterov=wl.nesterov,
              ns_steps=wl.ns_steps, coeffs=wl.coeffs)
    torch.cuda.synchronize()
    assert muon.status() == 0
    del g_d
    params = [host[i][0] for i in sample]
    bufs = [host[i][1] for i in sample]
    grads = [host[i][2] for i in sample]
    p_ref, b_ref = muon_step_ref(params, grads, bufs, lr=wl.lr, beta=wl.beta,
                                 nesterov=wl.nesterov, ns_steps=wl.ns_steps, coeffs=wl.coeffs)
    # warm-started momentum: a trajectory step
    _check_step(params, [p_d[i] for i in sample], [b_d[i] for i in sample], p_ref, b_ref,
                tol=X_TOL_TRAJ)
    for k, i in enumerate(sample):
        if i in band:
            _, u = momentum_ref(grads[k], bufs[k], wl.beta, wl.nesterov)
            _check_band(_step_x(params[k], p_d[i], wl.lr), u, i)


def test_step_gpt2_medium_all_96_sampled(muon):
    """GPT-2 medium shapes (d = 1024): all 96 matrices in one call; the
    oracle on the first and the last layer."""
    _first_step_sampled(muon, WORKLOADS["gpt2_medium"], sample=[0, 1, 2, 3, 92, 93, 94, 95],
                        band=(0, 1, 2, 3))


def test_step_gpt2_xl_all_192_sampled(muon):
    """GPT-2 XL shapes (d = 1600, not a multiple of the 256-wide tiles): all
    192 matrices (1.47e9 elements) in one call, the largest workload; the
    oracle on every shape of the first and the last layer."""
    _first_step_sampled(muon, WORKLOADS["gpt2_xl"], sample=[0, 1, 2, 3, 188, 189, 190, 191],
                        band=(1,))


def test_square_8192_closed_form(muon):
    """The largest square of the sweep, against its known factors."""
    case = square_case(8192, seed=0)
    out = to_np(muon.orthogonalize(to_f32(case.g), ns_steps=5))
    d = case.project(out)
    target = poly_scalar(case.sigma / np.linalg.norm(case.sigma), COEFFS, 5)
    assert rel_fro(np.diag(d), target) < 3e-2


def test_step_nd_weights_viewed_as_2d(muon):
    """A conv weight (out, in, kh, kw) is updated as its (out, in*kh*kw) matrix
    (the im2col view a reply on the X thread asks about)."""
    rng = _rng(90)
    shape = (64, 32, 3, 3)
    p = (rng.standard_normal(shape) * 0.02).astype(np.float32)
    g = rng.standard_normal(shape).astype(np.float32)
    b = np.zeros(shape, np.float32)
    p_d, g_d, b_d = to_f32(p), to_f32(g), to_f32(b)
    muon.step([p_d], [g_d], [b_d], lr=0.02, reshape_nd=True)
    torch.cuda.synchronize()
    p2 = p.reshape(64, -1)
    p_ref, b_ref = muon_step_ref([p2], [g.reshape(64, -1)], [b.reshape(64, -1)], lr=0.02)
    _check_step([p2], [p_d.reshape(64, -1)], [b_d.reshape(64, -1)], p_ref, b_ref)
    with pytest.raises(ValueError):
        muon.step([p_d], [g_d], [b_d], lr=0.02)           # N-D needs the explicit view
    one = torch.zeros(16, device="cuda")
    with pytest.raises(ValueError):
        muon.step([one], [one], [one], lr=0.02, reshape_nd=True)   # 1-D stays excluded


def test_orthogonalize_max_size_rank1_closed_form(muon):
    """A 16384 x 65536 input (2^30 elements, 4 GB fp32) of rank one, u v^T:
    along (u^, v^) the iterate is f_k u^ v^T with the scalar sequence of the
    rank-1 pin (normalised singular value 1: 0.701000, 1.113620, 0.720706,
    1.089974, 0.696436), so u^T X v^ = 0.696436.  (Entry by entry the output
    is not rank one: bf16 rounding puts ~1e-5 into each of the other 16383
    singular directions and five steps multiply such values by up to
    a^5 = 485, so the check is the projection, which that noise leaves alone.)"""
    m, n = 16384, 65536
    rng = _rng(99)
    u = rng.standard_normal(m)
    v = rng.standard_normal(n)
    u /= np.linalg.norm(u)
    v /= np.linalg.norm(v)
    ud = torch.from_numpy(u.astype(np.float32)).cuda()
    vd = torch.from_numpy(v.astype(np.float32)).cuda()
    g = torch.outer(ud, vd) * 3.0            # any positive scale: the iteration normalises
    out = muon.orthogonalize(g, ns_steps=5, out_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    del g
    assert muon.status() == 0
    xv = torch.empty(m, dtype=torch.float64, device="cuda")
    for i in range(0, m, 1024):
        xv[i:i + 1024] = (out[i:i + 1024].float() @ vd).double()
    f_est = float(ud.double() @ xv)
    assert abs(f_est - 0.696436) < 1e-2 * 0.696436
    assert bool(torch.isfinite(out).all())


@pytest.mark.parametrize("co,steps", [((3.4445, -4.7750, 2.0315), 1), ((3.4445, -4.7750, 2.0315), 3),
                                      ((3.4445, -4.7750, 2.0315), 10),
                                      ((1.5, -0.5, 0.0), 8),            # cubic Newton-Schulz (c = 0)
                                      ((1.875, -1.25, 0.375), 6)])      # convergent quintic
def test_ns_steps_and_coefficient_sweep(muon, co, steps):
    """The coefficient/step trade-off space: other triples and step counts
    through the orthogonalisation entry point, against the oracle.

    Up to five iterations the 1e-2 bar holds as for the default step.  Past
    five, the singular values sit in the band the map oscillates in, where it
    contracts them on average (its Lyapunov exponent along an orbit is -0.49
    for the default triple), so the sorted singular values must still agree
    to 1e-2; the singular vectors are not contracted (divided differences of
    p between band values are near 1 in size) and every further iteration
    adds a fresh set of accumulation-order roundings, about 0.25% of the
    Frobenius norm, so the entry-wise bar grows by 2.5e-3 per step past five."""
    rng = _rng(120 + steps)
    g = rng.standard_normal((300, 500)).astype(np.float32)
    ref = orthogonalize_ref(g, steps, co)
    out = to_np(muon.orthogonalize(to_f32(g), ns_steps=steps, coeffs=co))
    err = rel_fro(out, ref)
    sv_out = np.linalg.svd(out.astype(np.float64), compute_uv=False)
    sv_ref = np.linalg.svd(np.asarray(ref, np.float64), compute_uv=False)
    sv_err = rel_fro(sv_out, sv_ref)
    print(f"coeffs {co} steps {steps}: entry-wise {err:.4f}, singular values {sv_err:.4f}")
    assert err <= X_TOL + 2.5e-3 * max(0, steps - 5)
    assert sv_err <= 1e-2


def test_step_more_matrices_than_one_group(muon):
    """600 matrices in one call: more than one launch group holds (512), so
    the call runs as consecutive groups; every matrix is checked."""
    rng = _rng(130)
    shapes = [(int(rng.integers(1, 97)), int(rng.integers(1, 97))) for _ in range(600)]
    ps = [(rng.standard_normal(s) * 0.02).astype(np.float32) for s in shapes]
    gs = [rng.standard_normal(s).astype(np.float32) for s in shapes]
    bs = [(rng.standard_normal(s) * 0.1).astype(np.float32) for s in shapes]
    p_d, b_d = _run_step(muon, ps, gs, bs, lr=0.02)
    assert muon.status() == 0
    p_ref, b_ref = muon_step_ref(ps, gs, bs, lr=0.02)
    _check_step(ps, p_d, b_d, p_ref, b_ref, tol=X_TOL_TRAJ)


@pytest.mark.parametrize("n_mats", [4, 520])
def test_step_mirrored_writes_every_destination(muon, n_mats):
    """muon_step_mirrored: the parameters come out exactly as from muon_step,
    and every mirror holds them too (520 matrices: two launch groups)."""
    rng = _rng(140 + n_mats)
    if n_mats == 4:
        shapes = [(256, 768), (768, 256), (300, 200), (129, 260)]
    else:
        shapes = [(int(rng.integers(1, 97)), 4 * int(rng.integers(1, 25))) for _ in range(n_mats)]
    ps = [(rng.standard_normal(s) * 0.02).astype(np.float32) for s in shapes]
    gs = [rng.standard_normal(s).astype(np.float32) for s in shapes]
    bs = [(rng.standard_normal(s) * 0.1).astype(np.float32) for s in shapes]
    p_ref, b_ref = _run_step(muon, ps, gs, bs, lr=0.02)
    p_d = [to_f32(p) for p in ps]
    b_d = [to_f32(b) for b in bs]
    mirrors = [[torch.full(s, float("nan"), device="cuda") for s in shapes] for _ in range(2)]
    muon.step(p_d, [to_f32(g) for g in gs], b_d, lr=0.02, mirrors=mirrors)
    torch.cuda.synchronize()
    assert muon.status() == 0
    for i in range(n_mats):
        assert torch.equal(p_d[i], p_ref[i]) and torch.equal(b_d[i], b_ref[i])
        for dests in mirrors:
            assert torch.equal(dests[i], p_d[i])
    # and the mirrored step against the oracle itself (a sample of the large case)
    sample = list(range(n_mats)) if n_mats <= 4 else list(range(0, n_mats, 37))
    po, bo = muon_step_ref([ps[i] for i in sample], [gs[i] for i in sample],
                           [bs[i] for i in sample], lr=0.02)
    _check_step([ps[i] for i in sample], [mirrors[1][i] for i in sample],
                [b_d[i] for i in sample], po, bo, tol=X_TOL_TRAJ)
