"""Matrix-sharded Muon (newton_schulz_norm_b200.sharded) on CPU: the partition,
and the all-gather path with two and three gloo ranks.

The CUDA step needs a GPU, so each rank steps its matrices with the oracle
(the same per-matrix arithmetic, on the CPU): after the all-gather every rank
must hold exactly what the oracle gives for every matrix stepped in one
process, only owners keep momentum, and every matrix is stepped once.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from newton_schulz_norm_b200.sharded import ShardedMuon, matrix_cost, partition
from workloads import WORKLOADS


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


@pytest.mark.parametrize("world", [1, 2, 3, 4, 8])
def test_partition_covers_and_balances(world):
    shapes = list(WORKLOADS["gpt2_124m"].shapes)
    owner = partition(shapes, world)
    assert len(owner) == len(shapes) and set(owner) <= set(range(world))
    assert owner == partition(shapes, world)                   # deterministic
    load = [0.0] * world
    for s, k in zip(shapes, owner):
        load[k] += matrix_cost(s)
    mean = sum(load) / world
    # longest-first greedy: no rank above the mean by more than one matrix
    assert max(load) <= mean + max(matrix_cost(s) for s in shapes) + 1e-12
    if world <= 8:
        assert max(load) / mean < 1.1                          # 48 matrices spread well


def test_partition_single_rank_and_errors():
    assert partition([(3, 4), (5, 5)], 1) == [0, 0]
    with pytest.raises(ValueError):
        partition([(3, 4)], 0)
    # more ranks than matrices: some ranks own nothing
    assert sorted(partition([(8, 8), (4, 4)], 4)) == [0, 1]


def _fake_step(params, grads, bufs, lr, beta, nesterov, ns_steps, **kw):
    # a plain momentum update, in place (layout tests only)
    for p, g, b in zip(params, grads, bufs):
        b.mul_(beta).add_(g)
        p.sub_(lr * b)


def _oracle_step(params, grads, bufs, lr, beta, nesterov, ns_steps, coeffs=None, **kw):
    """The Muon step of the oracle on CPU tensors, in place: what each rank's
    CUDA step computes for its own matrices."""
    from oracle import muon_step_ref
    extra = {} if coeffs is None else {"coeffs": coeffs}
    p_new, b_new = muon_step_ref([p.numpy() for p in params], [g.numpy() for g in grads],
                                 [b.numpy() for b in bufs], lr=lr, beta=beta, nesterov=nesterov,
                                 ns_steps=ns_steps, **extra)
    for p, b, pn, bn in zip(params, bufs, p_new, b_new):
        p.copy_(torch.from_numpy(pn))
        b.copy_(torch.from_numpy(bn))


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    from oracle import muon_step_ref
    shapes = [(6, 10), (10, 6), (7, 7), (3, 20), (20, 3), (1, 5), (9, 4), (24, 40)]
    sm = ShardedMuon(shapes, device="cpu", step_fn=_oracle_step)
    rng = np.random.default_rng(0)                          # same values on every rank
    p0 = [(rng.standard_normal(s) * 0.02).astype(np.float32) for s in shapes]
    for v, a in zip(sm.params, p0):
        v.copy_(torch.from_numpy(a))
    grads = [[torch.from_numpy(rng.standard_normal(s).astype(np.float32)) for s in shapes]
             for _ in range(2)]
    for g in grads:
        sm.step(g, lr=0.02, beta=0.95)
    # expected: the oracle over every matrix in one process, two steps
    want_p = p0
    want_b = [np.zeros(s, np.float32) for s in shapes]
    for g in grads:
        want_p, want_b = muon_step_ref(want_p, [t.numpy() for t in g], want_b, lr=0.02, beta=0.95)
    ok = True
    for i in range(len(shapes)):
        ok &= np.array_equal(sm.params[i].numpy(), want_p[i])
        if i in sm.bufs:
            ok &= np.array_equal(sm.bufs[i].numpy(), want_b[i])
    ok &= sorted(sm.bufs) == sm.owned                         # momentum only where owned
    ok &= all(sm.owner[i] == rank for i in sm.owned)
    # every rank ends with the same flat buffer
    chk = torch.tensor([float(sm.flat.double().sum()), float(sm.flat.double().abs().sum())])
    allc = [torch.zeros(2) for _ in range(world)]
    dist.all_gather(allc, chk)
    ok &= all(torch.equal(allc[0], c) for c in allc)
    out[rank * 2 + 0] = 1.0 if ok else 0.0
    out[rank * 2 + 1] = float(len(sm.owned))
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.timeout(180)
@pytest.mark.parametrize("world", [2, 3])
def test_gloo_ranks_step_own_matrices_and_gather(world):
    out = torch.zeros(2 * world, dtype=torch.float64).share_memory_()
    mp.start_processes(_worker, args=(world, _free_port(), out), nprocs=world, join=True,
                       start_method="spawn")
    v = out.numpy()
    assert all(v[2 * r] == 1.0 for r in range(world)), v
    assert sum(v[2 * r + 1] for r in range(world)) == 8      # every matrix owned once


def test_single_process_layout_without_group():
    shapes = [(4, 6), (6, 4), (5, 5)]
    sm = ShardedMuon(shapes, device="cpu", step_fn=_fake_step)
    assert sm.world == 1 and sm.owned == [0, 1, 2]
    for v, (r, c) in zip(sm.params, shapes):
        assert v.shape == (r, c) and v.is_contiguous()
        assert v.data_ptr() % 256 == sm.flat.data_ptr() % 256    # 64-element aligned starts
    g = [torch.ones(s) for s in shapes]
    sm.step(g, lr=1.0, beta=0.0)
    assert all(float(p.sum()) == -p.numel() for p in sm.params)


def test_mirror_pointers_address_every_other_rank():
    from newton_schulz_norm_b200.sharded import mirror_pointers
    bases = [1 << 40, 2 << 40, 3 << 40]
    offs = [0, 256, 4096, 8192]
    got = mirror_pointers([1, 3], offs, bases, rank=1)
    assert got == [[bases[0] + 256, bases[0] + 8192], [bases[2] + 256, bases[2] + 8192]]
    assert mirror_pointers([0], offs, bases[:1], rank=0) == []
