"""Muon over several GPUs: matrices partitioned across ranks, one all-gather.

Every matrix's step is independent of the others (momentum, norm and the
Newton-Schulz iteration are all per matrix), so N ranks that hold the same
gradients (after the data-parallel gradient all-reduce) can split the
matrices between them instead of each repeating the whole step:

* ``partition`` assigns each matrix to one rank, balancing an estimate of its
  cost (tensor-core time of the iteration plus HBM time of the elementwise
  passes) with the longest-first greedy rule;
* every rank runs the Muon step on the matrices it owns only, and keeps
  momentum buffers and scratch for those only (1/N of the state);
* one all-gather then gives every rank every updated matrix.

The parameters live in one flat fp32 buffer laid out by owner: rank k's
matrices are contiguous in segment k, and all segments have the same length,
so the all-gather writes the buffer in place (NCCL all-gather into a tensor
whose k-th slice is rank k's input).

With ``fused=True`` (several GPUs) the flat buffer is symmetric memory: every
rank can address every other rank's copy.  The last kernel of each rank's
step then writes its updated matrices straight into all the other copies
(muon_step_mirrored: peer stores from the epilogue, overlapping the last
GEMM), and a device-side barrier replaces the all-gather.
"""
from __future__ import annotations

from typing import Callable, List, Optional, Sequence, Tuple

import torch

# Rates used only to weigh one matrix against another when partitioning.
_TENSOR_RATE = 1.0e15      # FLOP/s of the Newton-Schulz GEMMs
_HBM_RATE = 5.0e12         # B/s of the elementwise passes
_ALIGN = 64                # elements: every matrix starts 256-byte aligned


def matrix_cost(shape: Tuple[int, int], ns_steps: int = 5) -> float:
    """Estimated seconds of one Muon step on an r x c matrix."""
    r, c = int(shape[0]), int(shape[1])
    m, n = min(r, c), max(r, c)
    flops = (3.0 * m * m * n + float(m) ** 3) * ns_steps   # Gram (triangle), square, update
    hbm = 22.0 * r * c                                      # first kernel 14 B + update 8 B
    return flops / _TENSOR_RATE + hbm / _HBM_RATE


def partition(shapes: Sequence[Tuple[int, int]], world: int, ns_steps: int = 5) -> List[int]:
    """Owner rank of every matrix: longest-first greedy (each matrix, most
    expensive first, goes to the least-loaded rank; ties to the lower rank)."""
    if world < 1:
        raise ValueError("world must be >= 1")
    order = sorted(range(len(shapes)), key=lambda i: (-matrix_cost(shapes[i], ns_steps), i))
    load = [0.0] * world
    owner = [0] * len(shapes)
    for i in order:
        k = min(range(world), key=lambda j: (load[j], j))
        owner[i] = k
        load[k] += matrix_cost(shapes[i], ns_steps)
    return owner


def _round_up(v: int, m: int) -> int:
    return (v + m - 1) // m * m


def mirror_pointers(owned: Sequence[int], byte_offsets: Sequence[int], bases: Sequence[int],
                    rank: int) -> List[List[int]]:
    """Destinations of this rank's matrices in every other rank's buffer:
    one list per other rank (in rank order), one address per owned matrix."""
    return [[int(bases[k]) + int(byte_offsets[i]) for i in owned]
            for k in range(len(bases)) if k != rank]


class ShardedMuon:
    """Muon step partitioned over the ranks of a process group.

    ``params`` (a list of 2-D fp32 views into one flat buffer, the same on
    every rank) are the parameters; initialise them through these views.
    ``step(grads, ...)`` takes the full list of gradients (identical on every
    rank), updates the owned matrices with ``step_fn`` (by default the CUDA
    Muon step of this package) and all-gathers the flat buffer.
    """

    def __init__(self, shapes: Sequence[Tuple[int, int]], group=None, ns_steps: int = 5,
                 device=None, step_fn: Optional[Callable] = None, fused: bool = False):
        import torch.distributed as dist

        self.shapes = [(int(r), int(c)) for r, c in shapes]
        self.group = group
        if dist.is_available() and dist.is_initialized():
            self.world = dist.get_world_size(group)
            self.rank = dist.get_rank(group)
        else:
            self.world, self.rank = 1, 0
        self.ns_steps = ns_steps
        self.owner = partition(self.shapes, self.world, ns_steps)
        if step_fn is None:
            from . import step as muon_step
            step_fn = muon_step
        self.step_fn = step_fn
        device = torch.device(device) if device is not None else torch.device("cuda")

        # flat layout by owner; every segment padded to the longest one
        offs = [0] * len(self.shapes)
        seg_len = [0] * self.world
        for i, (r, c) in enumerate(self.shapes):
            k = self.owner[i]
            offs[i] = seg_len[k]
            seg_len[k] = _round_up(seg_len[k] + r * c, _ALIGN)
        self.seg = max(max(seg_len), _ALIGN)
        self.owned = [i for i in range(len(self.shapes)) if self.owner[i] == self.rank]
        self.fused = bool(fused) and self.world > 1
        self._symm = None
        self._mirrors = None
        if self.fused:
            import torch.distributed._symmetric_memory as symm_mem
            pg = group if group is not None else dist.group.WORLD
            self.flat = symm_mem.empty(self.world * self.seg, dtype=torch.float32, device=device)
            self.flat.zero_()
            self._symm = symm_mem.rendezvous(self.flat, pg)
        else:
            self.flat = torch.zeros(self.world * self.seg, dtype=torch.float32, device=device)
        self.params: List[torch.Tensor] = []
        starts = []
        for i, (r, c) in enumerate(self.shapes):
            base = self.owner[i] * self.seg + offs[i]
            starts.append(base)
            self.params.append(self.flat[base:base + r * c].view(r, c))
        if self.fused:
            self._mirrors = mirror_pointers(self.owned, [4 * b for b in starts],
                                            list(self._symm.buffer_ptrs), self.rank)
        # momentum only for the matrices this rank steps
        self.bufs = {i: torch.zeros(self.shapes[i], dtype=torch.float32, device=device)
                     for i in self.owned}

    def segment(self, rank: Optional[int] = None) -> torch.Tensor:
        k = self.rank if rank is None else rank
        return self.flat[k * self.seg:(k + 1) * self.seg]

    def step(self, grads: Sequence[torch.Tensor], lr: float, beta: float = 0.95,
             nesterov: bool = True, coeffs=None, stream=None) -> None:
        """One step.  ``stream`` (default: torch's current stream) runs the
        owned matrices' kernels, after everything already queued on torch's
        current stream (the previous step's exchange included).  The
        exchange (all-gather, or the device barrier of the fused mode) runs
        on torch's current stream, which is made to wait for ``stream``
        first, so it never reads parameters the kernels have not written
        yet.  In the fused mode every rank's kernels also wait for a device
        barrier at entry: no rank stores into another rank's copy while that
        rank may still be reading its parameters from before this step."""
        if len(grads) != len(self.shapes):
            raise ValueError("one gradient per matrix is required")
        cur = torch.cuda.current_stream() if self.flat.is_cuda else None
        side = stream is not None and cur is not None and stream != cur
        if self.fused:
            self._symm.barrier()     # every rank is done with its parameters of the last step
        if side:
            stream.wait_stream(cur)  # after the entry barrier and the last step's exchange
        if self.owned:
            kw = dict(lr=lr, beta=beta, nesterov=nesterov, ns_steps=self.ns_steps)
            if coeffs is not None:
                kw["coeffs"] = coeffs
            if stream is not None:
                kw["stream"] = stream
            if self.fused:
                kw["mirrors"] = self._mirrors
            self.step_fn([self.params[i] for i in self.owned], [grads[i] for i in self.owned],
                         [self.bufs[i] for i in self.owned], **kw)
        if side:
            cur.wait_stream(stream)  # the exchange below runs after the kernels
        if self.fused:
            self._symm.barrier()     # every rank's peer stores are done and visible
        else:
            self.gather()

    def gather(self) -> None:
        """Every rank's segment to every rank (in place in the flat buffer)."""
        import torch.distributed as dist
        if not (dist.is_available() and dist.is_initialized()):
            return                                   # one process: nothing to exchange
        if dist.get_backend(self.group) == "nccl":
            dist.all_gather_into_tensor(self.flat, self.segment(), group=self.group)
        else:
            outs = [self.segment(k) for k in range(self.world)]
            mine = self.segment().clone()
            dist.all_gather(outs, mine, group=self.group)
