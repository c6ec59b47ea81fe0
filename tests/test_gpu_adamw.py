"""AdamW kernel (muon_adamw_step) against the fp64 oracle, element by element.

Tolerance, derived from the kernel's fp32 arithmetic (u = 2^-24, every fp32
operation and every host constant rounded once to nearest):

* m' = fma(beta1, m, (1-beta1) g): within 4u (beta1|m| + (1-beta1)|g|) of the
  oracle's fp32 value (three roundings plus the oracle's own);
* v' = fma(beta2, v, (1-beta2) g g): within 6u (beta2 v + (1-beta2) g^2);
* p' = fma(p, fp32(1 - lr lambda), -step * m' / den): the decay term carries
  3u |p| (constant, fma, oracle rounding), the Adam move U = step m'/den
  carries 9u |U| from its own roundings (step constant, product, division,
  and 5.5u of den = sqrt(v')/sqrt(bc2) + eps, whose terms are all positive),
  plus step/den times the error of m'.

The bound is evaluated per element from the oracle's fp64 intermediates.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

from oracle import adamw_step_ref
from workloads import ADAMW_WORKLOADS, AdamWStream

pytestmark = pytest.mark.gpu

U = 2.0 ** -24
TINY = 2.0 ** -126


@pytest.fixture(scope="module")
def muon():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from newton_schulz_norm_b200 import build
    build.build()
    import newton_schulz_norm_b200 as m
    yield m
    assert m.status() == 0


def _dev(xs):
    return [torch.from_numpy(np.ascontiguousarray(x)).cuda() for x in xs]


def _host(ts):
    return [t.cpu().numpy() for t in ts]


def _bounds(p, g, m, v, step, lr, b1, b2, eps, wd):
    """Per-element error bounds of (p', m', v') (module docstring)."""
    p, g, m, v = (np.asarray(x, np.float64) for x in (p, g, m, v))
    s_m = b1 * np.abs(m) + (1 - b1) * np.abs(g)
    s_v = b2 * v + (1 - b2) * g * g
    m_new = b1 * m + (1 - b1) * g
    bc1 = 1 - b1 ** step
    bc2 = 1 - b2 ** step
    den = np.sqrt(s_v / bc2) + eps
    step_size = lr / bc1
    upd = np.abs(step_size * m_new / den)
    p_new = np.abs(p * (1 - lr * wd)) + upd
    bp = 3 * U * (np.abs(p) + p_new) + 9 * U * upd + (step_size / den) * 4 * U * s_m + TINY
    return bp, 4 * U * s_m + TINY, 6 * U * s_v + TINY


def _run(muon, params, grads, us, vs, step, lr, b1, b2, eps, wd, decay=None):
    P, G, M, V = _dev(params), _dev(grads), _dev(us), _dev(vs)
    muon.adamw_step(P, G, M, V, step, lr, betas=(b1, b2), eps=eps, weight_decay=wd, decay=decay)
    torch.cuda.synchronize()
    return _host(P), _host(M), _host(V)


def _check(params, grads, us, vs, got, step, lr, b1, b2, eps, wd, decay=None):
    want = adamw_step_ref(params, grads, us, vs, step, lr, b1, b2, eps, wd, decay)
    n = len(params)
    decay = [True] * n if decay is None else decay
    exact = total = 0
    for i in range(n):
        wdi = wd if decay[i] else 0.0
        bp, bm, bv = _bounds(params[i], grads[i], us[i], vs[i], step, lr, b1, b2, eps, wdi)
        for k, (b, name) in enumerate(((bp, "p"), (bm, "m"), (bv, "v"))):
            g_ = np.asarray(got[k][i], np.float64)
            w_ = np.asarray(want[k][i], np.float64)
            err = np.abs(g_ - w_)
            assert np.all(err <= b), (i, name, float(np.max(err / b)))
        exact += int(np.sum(got[0][i] == want[0][i]))
        total += got[0][i].size
    return exact / max(total, 1)


def test_ragged_tensors_warm_state(muon):
    wl = ADAMW_WORKLOADS["adamw_ragged"]
    st = AdamWStream(wl, seed=0)
    params, us, vs = st.init()
    grads = st.next_grads()
    decay = [t.decay for t in wl.tensors]
    got = _run(muon, params, grads, us, vs, wl.step, wl.lr, wl.beta1, wl.beta2, wl.eps,
               wl.weight_decay, decay)
    frac = _check(params, grads, us, vs, got, wl.step, wl.lr, wl.beta1, wl.beta2, wl.eps,
                  wl.weight_decay, decay)
    assert frac > 0.5      # most parameters come out bit-identical to the oracle


@pytest.mark.parametrize("betas,eps,wd", [((0.9, 0.999), 1e-8, 0.1), ((0.9, 0.95), 1e-6, 1e-2),
                                          ((0.0, 0.5), 0.0, 0.0)])
def test_first_step_from_zero_state(muon, betas, eps, wd):
    rng = np.random.default_rng(11)
    sizes = [1, 2, 3, 4, 7, 2047, 2048, 2049, 6145, 100003]
    params = [rng.standard_normal(s).astype(np.float32) for s in sizes]
    grads = [(rng.standard_normal(s) * np.exp(rng.uniform(-6, 2, s))).astype(np.float32) for s in sizes]
    zs = [np.zeros(s, np.float32) for s in sizes]
    got = _run(muon, params, grads, zs, zs, 1, 1e-2, betas[0], betas[1], eps, wd)
    _check(params, grads, zs, zs, got, 1, 1e-2, betas[0], betas[1], eps, wd)
    # closed form of the first step: p (1 - lr wd) - lr g / (|g| + eps)
    for p, g, pg in zip(params, grads, got[0]):
        p64, g64 = p.astype(np.float64), g.astype(np.float64)
        want = p64 * (1 - 1e-2 * wd) - 1e-2 * g64 / (np.abs(g64) + eps)
        assert np.max(np.abs(pg - want) / (np.abs(want) + 1e-2)) < 1e-6


def test_misaligned_views_take_the_scalar_path(muon):
    """Tensors that start 4 or 8 bytes past a 16-byte boundary (still
    contiguous) use scalar accesses; mixed with aligned ones in one call."""
    rng = np.random.default_rng(12)
    sizes = [5, 4096, 3001, 33]
    offs = [1, 0, 2, 3]
    host = [[rng.standard_normal(s).astype(np.float32) for s in sizes] for _ in range(4)]
    host[3] = [np.abs(x) * 1e-4 for x in host[3]]          # v >= 0
    dev = []
    for k in range(4):
        row = []
        for x, o in zip(host[k], offs):
            base = torch.zeros(x.size + 8, dtype=torch.float32, device="cuda")
            view = base[o:o + x.size]
            view.copy_(torch.from_numpy(x))
            row.append(view)
        dev.append(row)
    assert dev[0][0].data_ptr() % 16 == 4 and dev[0][1].data_ptr() % 16 == 0
    muon.adamw_step(dev[0], dev[1], dev[2], dev[3], 7, 3e-3, betas=(0.9, 0.99), eps=1e-8,
                    weight_decay=0.05)
    torch.cuda.synchronize()
    got = (_host(dev[0]), _host(dev[2]), _host(dev[3]))
    _check(host[0], host[1], host[2], host[3], got, 7, 3e-3, 0.9, 0.99, 1e-8, 0.05)


def test_more_tensors_than_one_launch_holds(muon):
    """300 tensors (launches hold 128): split into three launches, one result."""
    rng = np.random.default_rng(13)
    sizes = rng.integers(1, 5000, 300)
    params = [rng.standard_normal(s).astype(np.float32) for s in sizes]
    grads = [rng.standard_normal(s).astype(np.float32) for s in sizes]
    us = [(rng.standard_normal(s) * 0.1).astype(np.float32) for s in sizes]
    vs = [(rng.standard_normal(s) ** 2 * 0.1).astype(np.float32) for s in sizes]
    decay = [bool(i % 3) for i in range(300)]
    muon.profile_begin()
    got = _run(muon, params, grads, us, vs, 50, 1e-3, 0.9, 0.999, 1e-8, 0.1, decay)
    prof = muon.profile_end()
    assert prof["adamw"][1] == 3
    _check(params, grads, us, vs, got, 50, 1e-3, 0.9, 0.999, 1e-8, 0.1, decay)


def test_consecutive_steps_track_the_oracle(muon):
    wl = ADAMW_WORKLOADS["adamw_ragged"]
    st = AdamWStream(wl, seed=1)
    params, us, vs = st.init()
    decay = [t.decay for t in wl.tensors]
    P, M, V = _dev(params), _dev(us), _dev(vs)
    for k in range(6):
        grads = st.next_grads()
        t = wl.step + k
        muon.adamw_step(P, _dev(grads), M, V, t, wl.lr, betas=(wl.beta1, wl.beta2), eps=wl.eps,
                        weight_decay=wl.weight_decay, decay=decay)
        torch.cuda.synchronize()
        got = (_host(P), _host(M), _host(V))
        _check(params, grads, us, vs, got, t, wl.lr, wl.beta1, wl.beta2, wl.eps, wl.weight_decay,
               decay)
        # continue both from the oracle's state, so each step is checked from
        # identical inputs
        params, us, vs = adamw_step_ref(params, grads, us, vs, t, wl.lr, wl.beta1, wl.beta2, wl.eps,
                                        wl.weight_decay, decay)
        for d, h in zip(P + M + V, params + us + vs):
            d.copy_(torch.from_numpy(h))


def test_gpt2_124m_non_hidden_parameters_full_size(muon):
    """All 100 tensors (39.5M elements) in one call, every element checked."""
    wl = ADAMW_WORKLOADS["gpt2_124m_adamw"]
    st = AdamWStream(wl, seed=0)
    params, us, vs = st.init()
    grads = st.next_grads()
    decay = [t.decay for t in wl.tensors]
    got = _run(muon, params, grads, us, vs, wl.step, wl.lr, wl.beta1, wl.beta2, wl.eps,
               wl.weight_decay, decay)
    _check(params, grads, us, vs, got, wl.step, wl.lr, wl.beta1, wl.beta2, wl.eps,
           wl.weight_decay, decay)


def test_zero_gradient_is_pure_decay_and_nan_stays_put(muon):
    n = 4099
    rng = np.random.default_rng(14)
    p = rng.standard_normal(n).astype(np.float32)
    z = np.zeros(n, np.float32)
    got = _run(muon, [p, p], [z, z], [z, z], [z, z], 1, 5e-3, 0.9, 0.999, 1e-6, 1e-2, [True, False])
    np.testing.assert_array_equal(got[0][1], p)                      # no-decay group untouched
    f = np.float32(1 - 5e-3 * 1e-2)
    np.testing.assert_array_equal(got[0][0], p * f)                  # one fp32 multiply
    assert np.all(got[1][0] == 0) and np.all(got[2][0] == 0)
    g = rng.standard_normal(n).astype(np.float32)
    g[100] = np.nan
    got = _run(muon, [p, p], [g, np.nan_to_num(g)], [z, z], [z, z], 1, 1e-3, 0.9, 0.999, 1e-8, 0.0)
    bad = ~np.isfinite(got[0][0])
    assert bad[100] and bad.sum() == 1 and np.isnan(got[1][0][100]) and np.isnan(got[2][0][100])
    assert np.all(np.isfinite(got[0][1]))


def test_binding_rejects_bad_tensors(muon):
    a = torch.zeros(8, device="cuda")
    with pytest.raises(ValueError):
        muon.adamw_step([a], [torch.zeros(9, device="cuda")], [a], [a], 1, 1e-3)
    with pytest.raises(ValueError):
        muon.adamw_step([a], [a], [a], [torch.zeros(16, device="cuda")[::2]], 1, 1e-3)
    with pytest.raises(ValueError):
        muon.adamw_step([a], [a], [a], [a.double()], 1, 1e-3)
    with pytest.raises(muon.MuonError):
        muon.adamw_step([a], [a], [a], [a], 0, 1e-3)                # t counts from 1


def test_prepared_group_equals_adamw_step(muon):
    """AdamWGroup (arguments packed once) gives exactly adamw_step's result."""
    wl = ADAMW_WORKLOADS["adamw_ragged"]
    st = AdamWStream(wl, seed=5)
    params, us, vs = st.init()
    grads = [st.next_grads() for _ in range(3)]
    decay = [t.decay for t in wl.tensors]
    kw = dict(lr=wl.lr, betas=(wl.beta1, wl.beta2), eps=wl.eps, weight_decay=wl.weight_decay,
              decay=decay)
    a = [_dev(params), _dev(us), _dev(vs)]
    b = [_dev(params), _dev(us), _dev(vs)]
    gb = _dev(grads[0])
    group = muon.AdamWGroup(b[0], gb, b[1], b[2], **kw)
    for k, gs in enumerate(grads):
        muon.adamw_step(a[0], _dev(gs), a[1], a[2], wl.step + k, **kw)
        for d, h in zip(gb, gs):
            d.copy_(torch.from_numpy(h))
        group.step(wl.step + k)
    torch.cuda.synchronize()
    for x, y in zip(a[0] + a[1] + a[2], b[0] + b[1] + b[2]):
        assert torch.equal(x, y)
