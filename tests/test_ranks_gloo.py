"""The multi-rank path of bench.py on CPU with gloo, world_size 2: every rank
draws its own problem, the reported time is the max over ranks, and the
reference arm runs on rank 0 only."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    os.environ["RANK"] = str(rank)
    os.environ["WORLD_SIZE"] = str(world)
    import bench
    from workloads import WORKLOADS, WorkloadStream
    ranks = bench.Ranks(world, backend="gloo", timeout_s=60)
    ranks.barrier()
    local_ms = 1.0 + rank * 2.5                    # rank 1 is slower
    out[rank * 3 + 0] = ranks.max(local_ms)
    st = WorkloadStream(WORKLOADS["single_256"], seed=bench.rank_seed(rank))
    params, _ = st.init()
    out[rank * 3 + 1] = float(params[0][0, 0])
    ranks.barrier()
    ranks.close()
    out[rank * 3 + 2] = 1.0


@pytest.mark.timeout(180)
def test_two_gloo_ranks_max_and_independent_problems():
    world = 2
    out = torch.zeros(3 * world, dtype=torch.float64).share_memory_()
    mp.start_processes(_worker, args=(world, _free_port(), out), nprocs=world, join=True,
                       start_method="spawn")
    v = out.numpy()
    assert v[0] == v[3] == 3.5                     # both ranks report the max
    assert v[1] != v[4]                            # seed = rank: different problems
    assert v[2] == v[5] == 1.0                     # both closed cleanly


def test_reference_arm_runs_on_rank_zero_only(capsys):
    import bench
    from workloads import WORKLOADS

    class A:
        steps, warmup, gpus = 1, 0, 2
    assert bench.run_reference(A, WORKLOADS["gpt2_124m"], rank=1) == 0
    assert capsys.readouterr().out == ""           # no line, no work on rank 1


def test_single_rank_needs_no_process_group():
    import bench
    r = bench.Ranks(1)
    r.barrier()
    assert r.max(2.0) == 2.0
    r.close()
