"""One shape set, several parameter copies: the cached tensor maps of the last
X update are per pointer set (the 8 most recent), so alternating copies must
give every copy exactly what a run on that copy alone gives, including once
more sets than the cache holds have been used (eviction)."""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

SHAPES = [(256, 768), (768, 256), (128, 128)]


@pytest.fixture(scope="module")
def muon():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from newton_schulz_norm_b200 import build
    build.build()
    import newton_schulz_norm_b200 as m
    yield m
    assert m.status() == 0


def _copies(rng, k):
    p = [(rng.standard_normal(s) * 0.02).astype(np.float32) for s in SHAPES]
    return [[torch.from_numpy(a).cuda() for a in p] for _ in range(k)]


@pytest.mark.parametrize("nsets", [3, 11])
def test_alternating_parameter_sets(muon, nsets):
    rng = np.random.default_rng(200 + nsets)
    sets = _copies(rng, nsets)
    bufs = [[torch.zeros(s, device="cuda") for s in SHAPES] for _ in range(nsets)]
    solo_p = [[t.clone() for t in sets[k]] for k in range(nsets)]
    solo_b = [[t.clone() for t in bufs[k]] for k in range(nsets)]
    grads = [[torch.from_numpy(rng.standard_normal(s).astype(np.float32)).cuda() for s in SHAPES]
             for _ in range(3)]
    # interleaved: every step visits every set in turn
    for g in grads:
        for k in range(nsets):
            muon.step(sets[k], g, bufs[k], lr=0.02)
    torch.cuda.synchronize()
    # reference: each set alone, its three steps back to back
    for k in range(nsets):
        for g in grads:
            muon.step(solo_p[k], g, solo_b[k], lr=0.02)
    torch.cuda.synchronize()
    assert muon.status() == 0
    for k in range(nsets):
        for a, b in zip(sets[k], solo_p[k]):
            assert torch.equal(a, b), k
        for a, b in zip(bufs[k], solo_b[k]):
            assert torch.equal(a, b), k
