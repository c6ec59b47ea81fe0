"""The C-ABI library builds, loads and exports every declared symbol; host-side
argument checks reject bad input before any GPU work (no GPU needed)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "muon.h")


def _declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"MUON_API\s+[\w\s\*]*?\b(muon_\w+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    from newton_schulz_norm_b200 import build
    build.build()
    import newton_schulz_norm_b200 as m
    return m.library()


def test_header_declares_expected_entry_points():
    syms = _declared_symbols()
    for s in ("muon_step", "muon_orthogonalize", "muon_status", "muon_error_string",
              "muon_release", "muon_momentum_normalize", "muon_gram", "muon_poly", "muon_xupdate"):
        assert s in syms


def test_library_exports_every_declared_symbol(lib):
    import newton_schulz_norm_b200 as m
    syms = _declared_symbols()
    assert sorted(m.EXPORTS) == syms
    for s in syms:
        assert hasattr(lib, s), s


def test_checked_build_exports_debug_symbols():
    """The bounds-checked variant exports every muon.h symbol and the
    muon_debug.h ones; the regular library does not export the latter."""
    from newton_schulz_norm_b200 import build
    import newton_schulz_norm_b200 as m
    chk = ctypes.CDLL(build.build(checked=True))
    text = open(os.path.join(ROOT, "include", "muon_debug.h")).read()
    dbg = sorted(set(re.findall(r"MUON_API\s+[\w\s\*]*?\b(muon_\w+)\s*\(", text)))
    assert dbg == ["muon_debug_set_tile_row"]
    for s in _declared_symbols() + dbg:
        assert hasattr(chk, s), s
    assert not hasattr(m.library(), dbg[0])


def test_no_cpu_fallback_symbols(lib):
    # The library is CUDA-only: its entry points are the declared ones, and the
    # package carries no oracle import.
    import newton_schulz_norm_b200 as m
    src = open(m.__file__).read()
    assert "oracle" not in src.replace("# ", "")


def test_version_and_errors(lib):
    assert b"sm_100a" in lib.muon_version()
    assert lib.muon_error_string(0) == b"success"
    assert lib.muon_error_string(-5) == b"device-side wait timed out"
    assert lib.muon_error_string(12345) == b"unknown status"


def test_argument_checks_without_gpu(lib):
    P = ctypes.c_void_p
    arr = (P * 1)(P(16))
    sh = (ctypes.c_int64 * 2)(4, 4)
    # n = 0 is a no-op
    assert lib.muon_step(None, None, None, None, 0, 0.1, 0.9, 1, 5, None, None) == 0
    # negative n, null pointer arrays, bad shapes, bad steps, non-finite scalars
    assert lib.muon_step(arr, arr, arr, sh, -1, 0.1, 0.9, 1, 5, None, None) == -1
    assert lib.muon_step(None, arr, arr, sh, 1, 0.1, 0.9, 1, 5, None, None) == -1
    bad = (ctypes.c_int64 * 2)(0, 4)
    assert lib.muon_step(arr, arr, arr, bad, 1, 0.1, 0.9, 1, 5, None, None) == -1
    assert lib.muon_step(arr, arr, arr, sh, 1, 0.1, 0.9, 1, -1, None, None) == -1
    assert lib.muon_step(arr, arr, arr, sh, 1, 0.1, 0.9, 1, 101, None, None) == -1
    assert lib.muon_step(arr, arr, arr, sh, 1, float("nan"), 0.9, 1, 5, None, None) == -1
    nanco = (ctypes.c_float * 3)(1.0, float("inf"), 0.0)
    assert lib.muon_step(arr, arr, arr, sh, 1, 0.1, 0.9, 1, 5, nanco, None) == -1
    # misaligned device pointer
    mis = (P * 1)(P(18))
    assert lib.muon_step(mis, arr, arr, sh, 1, 0.1, 0.9, 1, 5, None, None) == -2
    # oversized matrix
    big = (ctypes.c_int64 * 2)(1 << 16, 1 << 16)
    assert lib.muon_step(arr, arr, arr, big, 1, 0.1, 0.9, 1, 5, None, None) == -2
    # stage entry points
    assert lib.muon_gram(None, 8, None, 8, 4, 4, None) == -1
    assert lib.muon_gram(P(16), 6, P(16), 8, 4, 4, None) == -1      # ld not a multiple of 8
    assert lib.muon_xupdate(P(16), 8, P(32), 8, P(32), 8, 4, 4, 3.0, None) == -1   # aliasing
    assert lib.muon_orthogonalize(None, None, 0, 4, 4, 5, None, None) == -1


def test_workspace_bytes_host_only(lib):
    import newton_schulz_norm_b200 as m
    from workloads import WORKLOADS
    b = m.workspace_bytes(WORKLOADS["gpt2_124m"].shapes)
    # two bf16 iterates (85M elements each) + A and B (48 x 768^2 each) + small tables
    lower = 2 * 2 * 84934656 + 2 * 2 * 48 * 768 * 768
    assert lower <= b <= lower * 1.05
    assert m.workspace_bytes([(0, 3)]) == -1


def test_nd_matrix_view_is_a_view_and_rejects_1d():
    import torch
    from newton_schulz_norm_b200 import _as_matrix
    w = torch.zeros(8, 4, 3, 3)
    m = _as_matrix(w)
    assert m.shape == (8, 36) and m.data_ptr() == w.data_ptr()
    m[2, 5] = 1.0
    assert w[2, 0, 1, 2] == 1.0          # row-major: 5 = 0*9 + 1*3 + 2
    assert _as_matrix(torch.zeros(3, 5)).shape == (3, 5)
    with pytest.raises(ValueError):
        _as_matrix(torch.zeros(7))
    with pytest.raises(ValueError):
        _as_matrix(torch.zeros(4, 8, 3, 3).transpose(0, 1))


def test_adamw_argument_checks_without_gpu(lib):
    P = ctypes.c_void_p
    arr = (P * 1)(P(16))
    ne = (ctypes.c_int64 * 1)(10)
    call = lambda n=1, a=arr, numels=ne, step=1, lr=1e-3, b1=0.9, b2=0.999, eps=1e-8, wd=0.0: \
        lib.muon_adamw_step(a, a, a, a, numels, None, n, step, lr, b1, b2, eps, wd, None)  # noqa: E731
    assert lib.muon_adamw_step(None, None, None, None, None, None, 0, 1, 1e-3, 0.9, 0.999, 1e-8, 0.0,
                               None) == 0
    assert call(n=-1) == -1
    assert lib.muon_adamw_step(None, arr, arr, arr, ne, None, 1, 1, 1e-3, 0.9, 0.999, 1e-8, 0.0,
                               None) == -1
    assert call(step=0) == -1
    assert call(lr=float("nan")) == -1
    assert call(lr=-1e-3) == -1
    assert call(b1=1.0) == -1
    assert call(b2=-0.1) == -1
    assert call(eps=float("inf")) == -1
    assert call(wd=-0.1) == -1
    assert call(numels=(ctypes.c_int64 * 1)(-5)) == -1
    assert call(a=(P * 1)(P(None))) == -1                            # null tensor pointer
    assert call(a=(P * 1)(P(18))) == -2                              # not even float-aligned
    # empty tensors are skipped before any device work, even with null pointers
    assert call(a=(P * 1)(P(None)), numels=(ctypes.c_int64 * 1)(0)) == 0


def test_mirrored_step_argument_checks_without_gpu(lib):
    P = ctypes.c_void_p
    arr = (P * 1)(P(16))
    sh = (ctypes.c_int64 * 2)(4, 8)
    mir = (P * 1)(P(32))
    f = lib.muon_step_mirrored
    assert f(arr, arr, arr, sh, 1, 0.1, 0.9, 1, 5, None, mir, 8, None) == -1      # > MUON_MAX_MIRRORS
    assert f(arr, arr, arr, sh, 1, 0.1, 0.9, 1, 5, None, None, 1, None) == -1     # no table
    assert f(arr, arr, arr, sh, 1, 0.1, 0.9, 1, 5, None, (P * 1)(P(None)), 1, None) == -1
    assert f(arr, arr, arr, sh, 1, 0.1, 0.9, 1, 5, None, (P * 1)(P(40)), 1, None) == -2   # misaligned
    assert f(arr, arr, arr, sh, 1, 0.1, 0.9, 1, 0, None, mir, 1, None) == -2      # needs an iteration
    odd = (ctypes.c_int64 * 2)(4, 6)
    assert f(arr, arr, arr, odd, 1, 0.1, 0.9, 1, 5, None, mir, 1, None) == -2     # c % 4 != 0
    assert f(None, None, None, None, 0, 0.1, 0.9, 1, 5, None, None, 0, None) == 0  # n = 0
