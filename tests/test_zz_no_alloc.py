"""The allocation-free entry point of the fused first kernel.

Some callers cannot allocate device memory while the optimizer runs (a host
that has given all device memory to its own pool allocator, or a process
that must not grow after start-up).  For them the library offers
muon_momentum_normalize_noalloc, whose scratch is a fixed array compiled into
the library.  Its results must equal those of the regular
muon_momentum_normalize on the same inputs, call after call.  This file is
collected last, so a run that stops at the first failure has already run
every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

from oracle import momentum_ref, normalize_ref, orient
from workloads import WORKLOADS, WorkloadStream

pytestmark = pytest.mark.gpu

BUF_TOL = 1e-6
SHAPES = [(256, 256), (200, 64), (7, 13), (13, 7), (768, 2304), (3072, 768), (129, 257)]


@pytest.fixture(scope="module")
def muon():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from newton_schulz_norm_b200 import build
    build.build()
    import newton_schulz_norm_b200 as m
    return m


def _x0_buffers(shapes):
    out = []
    for r, c in shapes:
        m, n = min(r, c), max(r, c)
        out.append(torch.zeros((m, (n + 7) // 8 * 8), dtype=torch.bfloat16, device="cuda"))
    return out


def test_noalloc_matches_allocating_entry_point_two_calls(muon):
    rng = np.random.default_rng(7)
    bufs0 = [(rng.standard_normal(s) * 0.1).astype(np.float32) for s in SHAPES]
    b_ref = [torch.from_numpy(b).cuda() for b in bufs0]
    b_na = [torch.from_numpy(b).cuda() for b in bufs0]
    x_na = _x0_buffers(SHAPES)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    for call in range(2):
        grads = [torch.from_numpy(rng.standard_normal(s).astype(np.float32)).cuda() for s in SHAPES]
        x_ref = muon.momentum_normalize(grads, b_ref, beta=0.95, nesterov=True)
        code = muon.momentum_normalize_noalloc(grads, b_na, x_na, beta=0.95, nesterov=True,
                                               dev_status=status)
        assert code == 0
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        for (r, c), br, bn, xr, xn in zip(SHAPES, b_ref, b_na, x_ref, x_na):
            br_np = br.cpu().numpy()
            diff = np.max(np.abs(bn.cpu().numpy() - br_np))
            assert diff <= BUF_TOL * max(np.max(np.abs(br_np)), 1e-30), (call, (r, c))
            n = max(r, c)
            a = xr.float().cpu().numpy()
            b = xn[:, :n].float().cpu().numpy()
            # same kernel arithmetic: within one bf16 ulp, in practice identical
            ulp = 2.0 ** (np.floor(np.log2(np.maximum(np.abs(a), 2.0 ** -126))) - 7)
            assert np.all(np.abs(a - b) <= ulp), (call, (r, c))
            assert np.mean(a != b) <= 1e-3, (call, (r, c))


def test_noalloc_gpt2_124m_queue_order_and_oracle(muon):
    """All 48 GPT-2 124M matrices: 5184 first-pass work items, far more than
    the queue slack (half the resident CTAs), so the set-up kernel splits
    first-pass runs to queue each matrix's second pass in between (the order
    the allocating entry point builds on the host).  Two calls in a row must
    match the allocating entry point and report no timeout; a sample of the
    outputs is also checked against the oracle (one bf16 rounding of the same
    fp32 u over its norm: within one bf16 ulp)."""
    wl = WORKLOADS["gpt2_124m"]
    st = WorkloadStream(wl, seed=5)
    _, bufs0 = st.init()
    b_ref = [torch.from_numpy(b).cuda() for b in bufs0]
    b_na = [torch.from_numpy(b).cuda() for b in bufs0]
    x_na = _x0_buffers(wl.shapes)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    sample = [0, 3, 46]
    for call in range(2):
        grads_np = st.next_grads()
        grads = [torch.from_numpy(g).cuda() for g in grads_np]
        b_before = [bufs0[i] if call == 0 else b_na[i].cpu().numpy() for i in sample]
        x_ref = muon.momentum_normalize(grads, b_ref, beta=wl.beta, nesterov=wl.nesterov)
        code = muon.momentum_normalize_noalloc(grads, b_na, x_na, beta=wl.beta,
                                               nesterov=wl.nesterov, dev_status=status)
        assert code == 0
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        for (r, c), br, bn, xr, xn in zip(wl.shapes, b_ref, b_na, x_ref, x_na):
            assert torch.equal(br, bn), (call, (r, c))
            assert torch.equal(xr, xn[:, :max(r, c)]), (call, (r, c))
        for k, i in enumerate(sample):
            _, u = momentum_ref(grads_np[i], b_before[k], wl.beta, wl.nesterov)
            want, _ = orient(normalize_ref(u))
            got = x_na[i][:, :want.shape[1]].float().cpu().numpy().astype(np.float64)
            ulp = 2.0 ** (np.floor(np.log2(np.maximum(np.abs(want), 2.0 ** -126))) - 7)
            assert np.all(np.abs(got - want) <= ulp), (call, i)


def test_noalloc_rejects_sizes_beyond_its_scratch(muon):
    lib = muon.library()
    P = ctypes.c_void_p
    g = torch.zeros((4, 4), device="cuda")
    b = torch.ones((4, 4), device="cuda")
    x = torch.zeros((4, 8), dtype=torch.bfloat16, device="cuda")
    n = 65                                                   # one more than the limit
    arr = lambda t: (P * n)(*([t.data_ptr()] * n))           # noqa: E731
    sh = (ctypes.c_int64 * (2 * n))(*([4, 4] * n))
    ld = (ctypes.c_int64 * n)(*([8] * n))
    assert lib.muon_momentum_normalize_noalloc(arr(g), arr(b), arr(x), ld, sh, n, 0.9, 1, None,
                                               None) == -2
    # one matrix with more work items than the fixed queue holds
    sh1 = (ctypes.c_int64 * 2)(20000, 20000)
    ld1 = (ctypes.c_int64 * 1)(20000)
    one = lambda t: (P * 1)(t.data_ptr())                    # noqa: E731
    assert lib.muon_momentum_normalize_noalloc(one(g), one(b), one(x), ld1, sh1, 1, 0.9, 1, None,
                                               None) == -2
    torch.cuda.synchronize()
    assert torch.all(b == 1)                                 # nothing ran
