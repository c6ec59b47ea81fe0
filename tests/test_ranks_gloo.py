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
    assert bench.run_reference(A, WORKLOADS["gpt2_124m"], rank=1, world=2) == 0
    assert capsys.readouterr().out == ""           # no line, no work on rank 1


def test_reference_arm_line_is_self_consistent(capsys):
    """Rank 0's line: steps x ms_per_step is the time actually spent in the
    timed oracle calls, value scales one call to the whole workload, and the
    config is the one the GPU arm prints."""
    import json
    import bench
    from workloads import WORKLOADS

    class A:
        steps, warmup, gpus = 2, 0, 1
    wl = WORKLOADS["gpt2_124m"]
    assert bench.run_reference(A, wl, rank=0, world=1) == 0
    d = json.loads(capsys.readouterr().out.strip())
    assert d["impl"] == "reference" and d["steps"] == 2
    sc = d["sampled_calls"]
    assert sc["calls"] == 2 and sc["matrices_per_call"] == 4
    assert abs(d["steps"] * d["ms_per_step"] - 1e3 * sc["seconds_timed"]) < 1e-6 * d["ms_per_step"] + 1e-3
    assert abs(d["value"] - d["ms_per_step"] * wl.n_matrices / 4) < 1e-9 * d["value"]
    assert d["config"] == dict(bench.workload_config(wl), parallelism=bench.parallelism(1))
    assert d["cpu_baseline"]["value"] == d["value"] and d["e2e"]["value"] == d["value"]


def test_single_rank_needs_no_process_group():
    import bench
    r = bench.Ranks(1)
    r.barrier()
    assert r.max(2.0) == 2.0
    r.close()
