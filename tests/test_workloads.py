"""The seeded input generators: shapes, determinism and subset consistency."""
import numpy as np

from workloads import WORKLOADS, WorkloadStream, square_case


def test_shapes_and_counts():
    wl = WORKLOADS["gpt2_124m"]
    assert wl.n_matrices == 48
    assert wl.n_elements == 84934656
    assert set(wl.shapes) == {(768, 2304), (768, 768), (768, 3072), (3072, 768)}
    assert abs(wl.ns_flops() - 1.087e12) / 1.087e12 < 1e-3
    assert WORKLOADS["gpt2_medium"].n_matrices == 96
    assert WORKLOADS["gpt2_xl"].n_matrices == 192
    assert WORKLOADS["single_256"].steps == 3


def test_stream_deterministic_and_subset_consistent():
    wl = WORKLOADS["gpt2_block"]
    s1 = WorkloadStream(wl, seed=0)
    p1, b1 = s1.init()
    g1 = s1.next_grads()
    s2 = WorkloadStream(wl, seed=0, subset=[1, 3])
    p2, b2 = s2.init()
    g2 = s2.next_grads()
    assert len(p2) == 2 and len(g2) == 2
    assert np.array_equal(p1[1], p2[0]) and np.array_equal(p1[3], p2[1])
    assert np.array_equal(g1[3], g2[1])
    assert all(x.dtype == np.float32 for x in p1 + b1 + g1)
    assert all(np.all(b == 0) for b in b1)
    assert abs(float(np.std(p1[0])) - 0.02) < 1e-3


def test_square_case_factors():
    c = square_case(256, seed=0)
    d = c.project(c.g)
    np.testing.assert_allclose(np.diag(d), c.sigma, atol=1e-6)
    assert np.abs(d - np.diag(np.diag(d))).max() < 1e-6
    assert abs(c.sigma.max() / c.sigma.min() - 1e3) < 1e-6


def test_square_case_hadamard_factors():
    import workloads
    # exercise the Hadamard construction at a small power of two
    rng = np.random.default_rng(0)
    n = 64
    d1 = rng.choice([-1.0, 1.0], n)
    d2 = rng.choice([-1.0, 1.0], n)
    sigma = np.linspace(1, 0.01, n)
    w = d1 * sigma * d2
    t = workloads.fwht_rows(np.diag(w))
    g = workloads.fwht_rows(t.T).T / n
    case = workloads.SquareCase(n, sigma, g.astype(np.float32), "hadamard", d1=d1, d2=d2)
    d = case.project(g)
    np.testing.assert_allclose(d, np.diag(sigma), atol=1e-12)
    # H/sqrt(n) is orthogonal
    h = workloads.fwht_rows(np.eye(n)) / np.sqrt(n)
    np.testing.assert_allclose(h @ h.T, np.eye(n), atol=1e-12)


def test_adamw_workloads_sizes_and_determinism():
    from workloads import ADAMW_WORKLOADS, AdamWStream
    wl = ADAMW_WORKLOADS["gpt2_124m_adamw"]
    assert wl.n_tensors == 2 + 12 * 8 + 2
    assert wl.n_elements == 50257 * 768 + 1024 * 768 + 12 * (6 * 768 + 3 * 768 + 4 * 768) + 2 * 768
    # decay only on the two embeddings (weight decay skips biases and 1-D tensors)
    assert [t.name for t in wl.tensors if t.decay] == ["wte", "wpe"]
    small = ADAMW_WORKLOADS["adamw_ragged"]
    a = AdamWStream(small, seed=3)
    b = AdamWStream(small, seed=3)
    for x, y in zip(a.init() + (a.next_grads(),), b.init() + (b.next_grads(),)):
        for s, t in zip(x, y):
            assert s.dtype == np.float32
            np.testing.assert_array_equal(s, t)
    _, _, vs = AdamWStream(small, seed=0).init()
    assert all(np.all(v >= 0) for v in vs)
