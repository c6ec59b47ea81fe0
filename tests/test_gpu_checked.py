"""The memory-safety checks that stand in for a GPU memory checker:

* guard bands around every scratch region of a plan, read back by
  muon_guard_check() after real steps (0 bytes changed);
* the bounds-checked build (libmuon_checked.so, include/muon_debug.h), whose
  kernels validate every table entry before using it: on valid input it
  gives exactly what the regular build gives, and a planted invalid tile
  becomes MUON_ERR_INVALID_ARG instead of an access out of bounds.  (The
  planted tile names rows past the end of its matrix, an entry that even the
  unchecked kernels would only read as zeros and never store, so the test
  cannot fault a GPU whichever build runs it.)"""
import ctypes

import numpy as np
import pytest
import torch

from workloads import WORKLOADS, WorkloadStream

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def libs():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from newton_schulz_norm_b200 import build
    build.build()
    path = build.build(checked=True)
    import newton_schulz_norm_b200 as m
    chk = ctypes.CDLL(path)
    P, PP, I64P = ctypes.c_void_p, ctypes.POINTER(ctypes.c_void_p), ctypes.POINTER(ctypes.c_int64)
    i, f = ctypes.c_int, ctypes.c_float
    chk.muon_step.restype = i
    chk.muon_step.argtypes = [PP, PP, PP, I64P, i, f, f, i, i, ctypes.POINTER(f), P]
    chk.muon_status.restype = i
    chk.muon_status.argtypes = [P]
    chk.muon_guard_check.restype = ctypes.c_int64
    chk.muon_guard_check.argtypes = []
    chk.muon_debug_set_tile_row.restype = i
    chk.muon_debug_set_tile_row.argtypes = [I64P, i, i, i, i]
    chk.muon_version.restype = ctypes.c_char_p
    yield m, chk
    chk.muon_release()


def _step(lib, P, G, B, shapes, wl):
    arr = lambda ts: (ctypes.c_void_p * len(ts))(*[t.data_ptr() for t in ts])  # noqa: E731
    flat = [v for s in shapes for v in s]
    sh = (ctypes.c_int64 * len(flat))(*flat)
    return lib.muon_step(arr(P), arr(G), arr(B), sh, len(shapes), wl.lr, wl.beta, 1, wl.ns_steps,
                         None, torch.cuda.current_stream().cuda_stream)


def _inputs(wl, seed):
    st = WorkloadStream(wl, seed=seed)
    params, bufs = st.init()
    grads = st.next_grads()
    on = lambda xs: [torch.from_numpy(x).cuda() for x in xs]  # noqa: E731
    return on(params), on(grads), on(bufs)


def test_checked_build_equals_regular_build_and_guards_hold(libs):
    m, chk = libs
    assert b"bounds-checked" in chk.muon_version()
    wl = WORKLOADS["gpt2_block"]
    P1, G, B1 = _inputs(wl, 11)
    P2, B2 = [t.clone() for t in P1], [t.clone() for t in B1]
    for _ in range(2):
        m.step(P1, G, B1, lr=wl.lr, beta=wl.beta, ns_steps=wl.ns_steps)
        assert _step(chk, P2, G, B2, wl.shapes, wl) == 0
    torch.cuda.synchronize()
    assert m.status() == 0 and chk.muon_status(None) == 0
    for a, b in zip(P1 + B1, P2 + B2):
        assert torch.equal(a, b)
    assert m.guard_check() == 0
    assert chk.muon_guard_check() == 0


def test_checked_build_turns_a_planted_tile_into_an_error(libs):
    _, chk = libs
    wl = WORKLOADS["gpt2_block"]
    P, G, B = _inputs(wl, 12)
    assert _step(chk, P, G, B, wl.shapes, wl) == 0          # builds the plan
    torch.cuda.synchronize()
    assert chk.muon_status(None) == 0
    flat = [v for s in wl.shapes for v in s]
    sh = (ctypes.c_int64 * len(flat))(*flat)
    # tile 0 of the chain (a Gram tile of a 768-row matrix): rows from 1024 on
    assert chk.muon_debug_set_tile_row(sh, len(wl.shapes), wl.ns_steps, 0, 1024) == 0
    assert _step(chk, P, G, B, wl.shapes, wl) == 0
    torch.cuda.synchronize()
    assert chk.muon_status(None) == -1                      # MUON_ERR_INVALID_ARG
    assert chk.muon_guard_check() == 0
    assert bool(torch.isfinite(torch.cat([b.flatten() for b in B])).all())
    chk.muon_release()                                     # drop the corrupted plan
    assert chk.muon_debug_set_tile_row(sh, len(wl.shapes), wl.ns_steps, 0, 0) == -1   # no plan


def test_guards_hold_after_the_largest_plans(libs):
    """GPT-2 124M and an odd-shaped mix through the regular build, then the
    guard bands of every cached plan."""
    m, _ = libs
    wl = WORKLOADS["gpt2_124m"]
    P, G, B = _inputs(wl, 13)
    m.step(P, G, B, lr=wl.lr)
    rng = np.random.default_rng(14)
    shapes = [(1, 1), (7, 300), (300, 7), (129, 257), (1000, 999)]
    on = lambda xs: [torch.from_numpy(x.astype(np.float32)).cuda() for x in xs]  # noqa: E731
    p2 = on([rng.standard_normal(s) for s in shapes])
    g2 = on([rng.standard_normal(s) for s in shapes])
    b2 = on([np.zeros(s) for s in shapes])
    m.step(p2, g2, b2, lr=0.02, ns_steps=3)
    torch.cuda.synchronize()
    assert m.status() == 0
    assert m.guard_check() == 0
