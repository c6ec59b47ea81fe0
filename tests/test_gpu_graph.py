"""One Muon step captured in a CUDA graph (capture_step) replays exactly the
eager step: same kernels, same pointers, bit-identical results."""
import pytest
import torch

from workloads import WORKLOADS, WorkloadStream

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def muon():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from newton_schulz_norm_b200 import build
    build.build()
    import newton_schulz_norm_b200 as m
    yield m
    assert m.status() == 0


@pytest.mark.parametrize("name", ["single_256", "gpt2_block"])
def test_graph_replay_is_bitwise_the_eager_step(muon, name):
    wl = WORKLOADS[name]
    st = WorkloadStream(wl, seed=3)
    params, bufs = st.init()
    grad_steps = [st.next_grads() for _ in range(4)]
    kw = dict(lr=wl.lr, beta=wl.beta, nesterov=wl.nesterov, ns_steps=wl.ns_steps, coeffs=wl.coeffs)

    pe = [torch.from_numpy(p).cuda() for p in params]
    be = [torch.from_numpy(b).cuda() for b in bufs]
    for gs in grad_steps:
        muon.step(pe, [torch.from_numpy(g).cuda() for g in gs], be, **kw)
    torch.cuda.synchronize()

    pg = [torch.from_numpy(p).cuda() for p in params]
    bg = [torch.from_numpy(b).cuda() for b in bufs]
    gg = [torch.from_numpy(g).cuda() for g in grad_steps[0]]
    graph = muon.capture_step(pg, gg, bg, **kw)          # runs step 1 eagerly
    for gs in grad_steps[1:]:
        for d, h in zip(gg, gs):
            d.copy_(torch.from_numpy(h))
        graph.replay()                                   # steps 2, 3, 4
    torch.cuda.synchronize()
    assert muon.status() == 0
    for a, b in zip(pe + be, pg + bg):
        assert torch.equal(a, b)
    del graph
