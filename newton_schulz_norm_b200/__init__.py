"""Muon optimizer step for NVIDIA B200 (sm_100a).

Python binding of the C interface in include/muon.h.  This module only
marshals arguments: every step of the computation runs in libmuon.so's CUDA
kernels.  PyTorch provides device memory and streams.  There is no CPU
fallback: if libmuon.so is missing or no sm_100 device is present, the calls
raise.

    import newton_schulz_norm_b200 as muon
    muon.step(params, grads, bufs, lr=0.02)      # lists of 2-D fp32 CUDA tensors
"""
from __future__ import annotations

import ctypes
import os
from typing import Sequence

import torch

__all__ = [
    "DEFAULT_COEFFS", "MuonError", "library", "step", "orthogonalize", "momentum_normalize",
    "gram", "poly", "xupdate", "status", "release", "workspace_bytes", "set_wait_limit_ns",
    "adamw_step", "AdamWGroup", "capture_step", "EXPORTS", "guard_check",
]

DEFAULT_COEFFS = (3.4445, -4.7750, 2.0315)
LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libmuon.so")

# Every symbol include/muon.h declares.
EXPORTS = ("muon_step", "muon_orthogonalize", "muon_momentum_normalize", "muon_gram", "muon_poly",
           "muon_xupdate", "muon_status", "muon_error_string", "muon_set_wait_limit_ns",
           "muon_workspace_bytes", "muon_release", "muon_version", "muon_profile_begin",
           "muon_profile_end", "muon_momentum_normalize_noalloc", "muon_adamw_step",
           "muon_step_mirrored", "muon_guard_check")

PROFILE_KINDS = ("momentum_norm_cast", "gram", "poly", "xupdate", "xupdate_final", "apply", "adamw",
                 "ns_chain")

_STATUS = {0: "MUON_OK", -1: "MUON_ERR_INVALID_ARG", -2: "MUON_ERR_UNSUPPORTED",
           -3: "MUON_ERR_CUDA", -4: "MUON_ERR_NOMEM", -5: "MUON_ERR_TIMEOUT"}


class MuonError(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        super().__init__(f"{what}: {_STATUS.get(code, code)} ({code})")


_lib = None

_P = ctypes.c_void_p
_PP = ctypes.POINTER(ctypes.c_void_p)
_I64P = ctypes.POINTER(ctypes.c_int64)
_FP = ctypes.POINTER(ctypes.c_float)


def library() -> ctypes.CDLL:
    """Load libmuon.so (built in-tree by newton_schulz_norm_b200.build)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: run `python -m newton_schulz_norm_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    i, i64, f, u64, d = ctypes.c_int, ctypes.c_int64, ctypes.c_float, ctypes.c_uint64, ctypes.c_double
    sig = {
        "muon_step": (i, [_PP, _PP, _PP, _I64P, i, f, f, i, i, _FP, _P]),
        "muon_orthogonalize": (i, [_P, _P, i, i64, i64, i, _FP, _P]),
        "muon_momentum_normalize": (i, [_PP, _PP, _PP, _I64P, _I64P, i, f, i, _P]),
        "muon_gram": (i, [_P, i64, _P, i64, i64, i64, _P]),
        "muon_poly": (i, [_P, i64, _P, i64, i64, f, f, _P]),
        "muon_xupdate": (i, [_P, i64, _P, i64, _P, i64, i64, i64, f, _P]),
        "muon_status": (i, [_P]),
        "muon_error_string": (ctypes.c_char_p, [i]),
        "muon_set_wait_limit_ns": (None, [u64]),
        "muon_workspace_bytes": (i64, [_I64P, i]),
        "muon_release": (None, []),
        "muon_version": (ctypes.c_char_p, []),
        "muon_profile_begin": (None, []),
        "muon_profile_end": (i, [ctypes.POINTER(ctypes.c_double), _I64P, i]),
        "muon_momentum_normalize_noalloc": (i, [_PP, _PP, _PP, _I64P, _I64P, i, f, i, _P, _P]),
        "muon_adamw_step": (i, [_PP, _PP, _PP, _PP, _I64P, _P, i, i64, d, d, d, d, d, _P]),
        "muon_step_mirrored": (i, [_PP, _PP, _PP, _I64P, i, f, f, i, i, _FP, _PP, i, _P]),
        "muon_guard_check": (i64, []),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def _check(code: int, what: str):
    if code != 0:
        raise MuonError(code, what)


def _stream_ptr(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return int(stream.cuda_stream) if hasattr(stream, "cuda_stream") else int(stream)


def _ptr_array(tensors) -> ctypes.Array:
    return (ctypes.c_void_p * len(tensors))(*[t.data_ptr() for t in tensors])


def _coeffs(coeffs):
    if coeffs is None:
        return None
    return (ctypes.c_float * 3)(*[float(c) for c in coeffs])


def _check_mat(t: torch.Tensor, name: str, dtype=torch.float32):
    if not isinstance(t, torch.Tensor) or t.dim() != 2:
        raise ValueError(f"{name}: expected a 2-D tensor")
    if not t.is_cuda or t.dtype != dtype or not t.is_contiguous():
        raise ValueError(f"{name}: expected a contiguous {dtype} CUDA tensor")


def _as_matrix(t: torch.Tensor) -> torch.Tensor:
    """View an N-D (N >= 3) tensor as (shape[0], prod(shape[1:])) -- a conv
    weight as its im2col matrix.  1-D tensors are not Muon parameters."""
    if t.dim() < 2:
        raise ValueError("Muon updates matrices; 1-D parameters belong to another optimizer")
    if t.dim() == 2:
        return t
    if not t.is_contiguous():
        raise ValueError("an N-D tensor must be contiguous to be updated through its matrix view")
    return t.view(t.shape[0], -1)   # a view: the in-place update reaches t


def step(params: Sequence[torch.Tensor], grads: Sequence[torch.Tensor],
         bufs: Sequence[torch.Tensor], lr: float, beta: float = 0.95, nesterov: bool = True,
         ns_steps: int = 5, coeffs=DEFAULT_COEFFS, stream=None, reshape_nd: bool = False,
         mirrors=None) -> None:
    """One Muon step, in place on params and bufs (see include/muon.h).

    With reshape_nd, tensors of rank >= 3 (conv weights) are updated as their
    (shape[0], prod(shape[1:])) matrix view; they must be contiguous.

    mirrors: optional list of destinations, each a list with one entry per
    parameter (a tensor of the same shape, or a raw device address, e.g. of
    another GPU's copy); the last kernel writes every updated matrix to each
    of them as well (muon_step_mirrored).
    """
    n = len(params)
    if len(grads) != n or len(bufs) != n:
        raise ValueError("params, grads and bufs must have the same length")
    if reshape_nd:
        params = [_as_matrix(t) for t in params]
        grads = [_as_matrix(t) for t in grads]
        bufs = [_as_matrix(t) for t in bufs]
    shapes = []
    for p, g, b in zip(params, grads, bufs):
        for t, nm in ((p, "param"), (g, "grad"), (b, "buf")):
            _check_mat(t, nm)
        if g.shape != p.shape or b.shape != p.shape:
            raise ValueError("param, grad and buf shapes differ")
        shapes += [p.shape[0], p.shape[1]]
    sh = (ctypes.c_int64 * len(shapes))(*shapes)
    if mirrors:
        flat = []
        for dests in mirrors:
            if len(dests) != n:
                raise ValueError("every mirror needs one destination per parameter")
            for t, p in zip(dests, params):
                if isinstance(t, torch.Tensor):
                    if t.shape != p.shape or t.dtype != torch.float32 or not t.is_contiguous():
                        raise ValueError("a mirror tensor must match its parameter (contiguous fp32)")
                    flat.append(t.data_ptr())
                else:
                    flat.append(int(t))
        mir = (ctypes.c_void_p * len(flat))(*flat)
        code = library().muon_step_mirrored(
            _ptr_array(params), _ptr_array(grads), _ptr_array(bufs), sh, n, float(lr), float(beta),
            int(bool(nesterov)), int(ns_steps), _coeffs(coeffs), mir, len(mirrors),
            _stream_ptr(stream))
        _check(code, "muon_step_mirrored")
        return
    code = library().muon_step(_ptr_array(params), _ptr_array(grads), _ptr_array(bufs), sh, n,
                               float(lr), float(beta), int(bool(nesterov)), int(ns_steps),
                               _coeffs(coeffs), _stream_ptr(stream))
    _check(code, "muon_step")


def capture_step(params: Sequence[torch.Tensor], grads: Sequence[torch.Tensor],
                 bufs: Sequence[torch.Tensor], lr: float, beta: float = 0.95,
                 nesterov: bool = True, ns_steps: int = 5, coeffs=DEFAULT_COEFFS,
                 reshape_nd: bool = False) -> "torch.cuda.CUDAGraph":
    """Run one Muon step eagerly, then capture the next one in a CUDA graph.

    The first call for a set of shapes and parameter pointers builds the
    library's plan and tensor maps (allocation and host copies, which a
    capture cannot hold); that is why this function performs one real step
    before capturing.  Every ``replay()`` of the returned graph is one more
    step on the same tensors: write each step's gradients into ``grads`` in
    place before replaying.  The graph keeps the hyper-parameters it was
    captured with.  Launching nothing but kernels and one memset, a replay
    saves the host work and launch gaps of the eager call.
    """
    kw = dict(lr=lr, beta=beta, nesterov=nesterov, ns_steps=ns_steps, coeffs=coeffs,
              reshape_nd=reshape_nd)
    step(params, grads, bufs, **kw)
    torch.cuda.synchronize()
    _check(status(), "muon_step (before capture)")
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step(params, grads, bufs, **kw)
    return graph


def step_raw(param_ptrs, grad_ptrs, buf_ptrs, shapes, lr, beta=0.95, nesterov=True, ns_steps=5,
             coeffs=DEFAULT_COEFFS, stream=0) -> int:
    """muon_step on raw device pointers; returns the status code unchanged."""
    n = len(param_ptrs)
    arr = lambda xs: (ctypes.c_void_p * max(n, 1))(*xs)  # noqa: E731
    flat = [int(v) for s in shapes for v in s]
    sh = (ctypes.c_int64 * max(len(flat), 1))(*flat)
    return library().muon_step(arr(param_ptrs), arr(grad_ptrs), arr(buf_ptrs), sh, n, float(lr),
                               float(beta), int(bool(nesterov)), int(ns_steps), _coeffs(coeffs),
                               int(stream) if stream is not None else None)


def adamw_step(params: Sequence[torch.Tensor], grads: Sequence[torch.Tensor],
               exp_avgs: Sequence[torch.Tensor], exp_avg_sqs: Sequence[torch.Tensor], step: int,
               lr: float, betas=(0.9, 0.999), eps: float = 1e-8, weight_decay: float = 1e-2,
               decay: Sequence[bool] | None = None, stream=None) -> None:
    """One AdamW step, in place on params and both running averages (see
    include/muon.h).  Tensors: fp32, contiguous, on the GPU, any shape; the
    four lists match element by element.  ``decay[i]`` false puts tensor i in
    the no-decay group; ``decay=None`` decays all.  ``step`` counts from 1."""
    n = len(params)
    if not (len(grads) == len(exp_avgs) == len(exp_avg_sqs) == n):
        raise ValueError("params, grads, exp_avgs and exp_avg_sqs must have the same length")
    if decay is not None and len(decay) != n:
        raise ValueError("decay must have one entry per tensor")
    numels = []
    for p, g, m, v in zip(params, grads, exp_avgs, exp_avg_sqs):
        for t, nm in ((p, "param"), (g, "grad"), (m, "exp_avg"), (v, "exp_avg_sq")):
            if not isinstance(t, torch.Tensor) or not t.is_cuda or t.dtype != torch.float32 \
                    or not t.is_contiguous():
                raise ValueError(f"{nm}: expected a contiguous float32 CUDA tensor")
        if g.shape != p.shape or m.shape != p.shape or v.shape != p.shape:
            raise ValueError("param, grad and average shapes differ")
        numels.append(p.numel())
    code = adamw_step_raw([t.data_ptr() for t in params], [t.data_ptr() for t in grads],
                          [t.data_ptr() for t in exp_avgs], [t.data_ptr() for t in exp_avg_sqs],
                          numels, step, lr, betas, eps, weight_decay, decay, _stream_ptr(stream))
    _check(code, "muon_adamw_step")


class AdamWGroup:
    """A fixed set of AdamW tensors, checked and marshalled once.

    ``adamw_step`` validates and packs every tensor on every call (tens of
    microseconds of host time for a hundred tensors); a training loop that
    steps the same tensors each time can build the argument arrays once and
    then call ``step(t)``, which only passes them on.  The tensors must stay
    allocated (and at the same addresses) for the group's lifetime.
    """

    def __init__(self, params: Sequence[torch.Tensor], grads: Sequence[torch.Tensor],
                 exp_avgs: Sequence[torch.Tensor], exp_avg_sqs: Sequence[torch.Tensor],
                 lr: float, betas=(0.9, 0.999), eps: float = 1e-8, weight_decay: float = 1e-2,
                 decay: Sequence[bool] | None = None):
        n = len(params)
        if not (len(grads) == len(exp_avgs) == len(exp_avg_sqs) == n):
            raise ValueError("params, grads, exp_avgs and exp_avg_sqs must have the same length")
        if decay is not None and len(decay) != n:
            raise ValueError("decay must have one entry per tensor")
        for p, g, m, v in zip(params, grads, exp_avgs, exp_avg_sqs):
            for t, nm in ((p, "param"), (g, "grad"), (m, "exp_avg"), (v, "exp_avg_sq")):
                if not isinstance(t, torch.Tensor) or not t.is_cuda or t.dtype != torch.float32 \
                        or not t.is_contiguous():
                    raise ValueError(f"{nm}: expected a contiguous float32 CUDA tensor")
            if g.shape != p.shape or m.shape != p.shape or v.shape != p.shape:
                raise ValueError("param, grad and average shapes differ")
        self._keep = (list(params), list(grads), list(exp_avgs), list(exp_avg_sqs))
        self._n = n
        arr = lambda ts: (ctypes.c_void_p * max(n, 1))(*[t.data_ptr() for t in ts])  # noqa: E731
        self._p, self._g, self._m, self._v = (arr(ts) for ts in self._keep)
        self._numels = (ctypes.c_int64 * max(n, 1))(*[p.numel() for p in params])
        self._decay = None if decay is None else \
            (ctypes.c_ubyte * max(n, 1))(*[1 if d else 0 for d in decay])
        self.lr, self.betas, self.eps, self.weight_decay = float(lr), tuple(betas), float(eps), \
            float(weight_decay)

    def step(self, step: int, lr: float | None = None, stream=None) -> None:
        """One AdamW step (t = ``step``, from 1) on the group's tensors."""
        code = library().muon_adamw_step(
            self._p, self._g, self._m, self._v, self._numels,
            ctypes.cast(self._decay, ctypes.c_void_p) if self._decay is not None else None,
            self._n, int(step), self.lr if lr is None else float(lr), float(self.betas[0]),
            float(self.betas[1]), self.eps, self.weight_decay, _stream_ptr(stream))
        _check(code, "muon_adamw_step")


def adamw_step_raw(param_ptrs, grad_ptrs, avg_ptrs, sq_ptrs, numels, step, lr, betas=(0.9, 0.999),
                   eps=1e-8, weight_decay=1e-2, decay=None, stream=0) -> int:
    """muon_adamw_step on raw device pointers; returns the status code unchanged."""
    n = len(param_ptrs)
    arr = lambda xs: (ctypes.c_void_p * max(n, 1))(*xs)  # noqa: E731
    ne = (ctypes.c_int64 * max(n, 1))(*[int(x) for x in numels])
    dm = None if decay is None else (ctypes.c_ubyte * max(n, 1))(*[1 if d else 0 for d in decay])
    return library().muon_adamw_step(arr(param_ptrs), arr(grad_ptrs), arr(avg_ptrs), arr(sq_ptrs), ne,
                                     ctypes.cast(dm, ctypes.c_void_p) if dm is not None else None, n,
                                     int(step), float(lr), float(betas[0]), float(betas[1]),
                                     float(eps), float(weight_decay),
                                     int(stream) if stream is not None else None)


def orthogonalize(x: torch.Tensor, ns_steps: int = 5, coeffs=DEFAULT_COEFFS,
                  out_dtype=torch.float32, out: torch.Tensor | None = None, stream=None):
    """Newton-Schulz orthogonalisation of one fp32 matrix (normalised first)."""
    _check_mat(x, "x")
    if out is None:
        out = torch.empty(x.shape, dtype=out_dtype, device=x.device)
    _check_mat(out, "out", out.dtype)
    if out.dtype not in (torch.float32, torch.bfloat16) or out.shape != x.shape:
        raise ValueError("out must be fp32 or bf16 with the shape of x")
    code = library().muon_orthogonalize(x.data_ptr(), out.data_ptr(), int(out.dtype == torch.bfloat16),
                                        x.shape[0], x.shape[1], int(ns_steps), _coeffs(coeffs),
                                        _stream_ptr(stream))
    _check(code, "muon_orthogonalize")
    return out


def _ld8(n: int) -> int:
    return (n + 7) // 8 * 8


def momentum_normalize(grads, bufs, beta=0.95, nesterov=True, stream=None):
    """The fused first kernel alone; returns oriented bf16 X0 views (m x n)."""
    n = len(grads)
    x0s, lds, shapes, outs = [], [], [], []
    for g, b in zip(grads, bufs):
        _check_mat(g, "grad")
        _check_mat(b, "buf")
        r, c = g.shape
        m, nn = min(r, c), max(r, c)
        ld = _ld8(nn)
        x = torch.empty((m, ld), dtype=torch.bfloat16, device=g.device)
        x0s.append(x)
        outs.append(x[:, :nn])
        lds.append(ld)
        shapes += [r, c]
    code = library().muon_momentum_normalize(
        _ptr_array(grads), _ptr_array(bufs), _ptr_array(x0s), (ctypes.c_int64 * n)(*lds),
        (ctypes.c_int64 * len(shapes))(*shapes), n, float(beta), int(bool(nesterov)),
        _stream_ptr(stream))
    _check(code, "muon_momentum_normalize")
    return outs


def _bf16_padded(x: torch.Tensor) -> torch.Tensor:
    """Copy into a bf16 buffer whose row pitch is a multiple of 8 elements."""
    m, n = x.shape
    buf = torch.zeros((m, _ld8(n)), dtype=torch.bfloat16, device=x.device)
    buf[:, :n] = x
    return buf


def gram(x: torch.Tensor) -> torch.Tensor:
    """A = bf16(X X^T) for a bf16 m x n X (on the current stream)."""
    stream = None
    m, n = x.shape
    xp = _bf16_padded(x)
    a = torch.empty((m, _ld8(m)), dtype=torch.bfloat16, device=x.device)
    code = library().muon_gram(xp.data_ptr(), xp.shape[1], a.data_ptr(), a.shape[1], m, n,
                               _stream_ptr(stream))
    _check(code, "muon_gram")
    return a[:, :m]


def poly(a: torch.Tensor, cb: float, cc: float) -> torch.Tensor:
    """B = bf16(cb*A + cc*A A) for a symmetric bf16 m x m A (current stream)."""
    stream = None
    m = a.shape[0]
    ap = _bf16_padded(a)
    b = torch.empty((m, _ld8(m)), dtype=torch.bfloat16, device=a.device)
    code = library().muon_poly(ap.data_ptr(), ap.shape[1], b.data_ptr(), b.shape[1], m, float(cb),
                               float(cc), _stream_ptr(stream))
    _check(code, "muon_poly")
    return b[:, :m]


def xupdate(b: torch.Tensor, x: torch.Tensor, ca: float) -> torch.Tensor:
    """X' = bf16(ca*X + B X) for bf16 B (m x m) and X (m x n) (current stream)."""
    stream = None
    m, n = x.shape
    bp = _bf16_padded(b)
    xp = _bf16_padded(x)
    out = torch.empty((m, _ld8(n)), dtype=torch.bfloat16, device=x.device)
    code = library().muon_xupdate(bp.data_ptr(), bp.shape[1], xp.data_ptr(), xp.shape[1],
                                  out.data_ptr(), out.shape[1], m, n, float(ca), _stream_ptr(stream))
    _check(code, "muon_xupdate")
    return out[:, :n]


def status(stream=None) -> int:
    """Synchronise and return (and clear) the device-side status code."""
    return library().muon_status(_stream_ptr(stream))


def guard_check() -> int:
    """Synchronise and return how many guard-band bytes around the library's
    scratch regions were overwritten (0: no kernel wrote out of bounds)."""
    return int(library().muon_guard_check())


def release() -> None:
    library().muon_release()


def set_wait_limit_ns(ns: int) -> None:
    library().muon_set_wait_limit_ns(int(ns))


def workspace_bytes(shapes) -> int:
    flat = [int(v) for s in shapes for v in s]
    return int(library().muon_workspace_bytes((ctypes.c_int64 * max(len(flat), 1))(*flat), len(shapes)))


def version() -> str:
    return library().muon_version().decode()


def profile_begin() -> None:
    """Start bracketing every launch of the library with CUDA events."""
    library().muon_profile_begin()


def profile_end() -> dict:
    """Stop, synchronise, and return {kind: (total_ms, launches)}."""
    k = len(PROFILE_KINDS)
    ms = (ctypes.c_double * k)()
    n = (ctypes.c_int64 * k)()
    code = library().muon_profile_end(ms, n, k)
    if code < 0:
        raise MuonError(code, "muon_profile_end")
    return {PROFILE_KINDS[i]: (float(ms[i]), int(n[i])) for i in range(k)}


def momentum_normalize_noalloc(grads, bufs, x0s, beta=0.95, nesterov=True, dev_status=None,
                               stream=None) -> int:
    """The fused first kernel through the allocation-free entry point.

    For callers that must not allocate device memory while stepping: the
    library's scratch is a fixed array compiled into it.  ``x0s`` are
    caller-allocated bf16 buffers (min(r,c) x ld, ld % 8 == 0, ld >= max(r,c));
    ``dev_status`` an optional int32 CUDA tensor of one element that receives
    a device-side timeout.  Returns the status code (0 on success).
    """
    n = len(grads)
    shapes = [v for g in grads for v in g.shape]
    lds = [x.shape[1] for x in x0s]
    return library().muon_momentum_normalize_noalloc(
        _ptr_array(grads), _ptr_array(bufs), _ptr_array(x0s), (ctypes.c_int64 * max(n, 1))(*lds),
        (ctypes.c_int64 * max(len(shapes), 1))(*shapes), n, float(beta), int(bool(nesterov)),
        None if dev_status is None else dev_status.data_ptr(), _stream_ptr(stream))
