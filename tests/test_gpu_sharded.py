"""Matrix-sharded Muon on one GPU through a one-rank NCCL process group,
against the oracle: the owned-matrix step and the in-place all-gather,
driven once on torch's current stream and once on a side stream (the
exchange must then wait for the side stream's kernels)."""
import os
import socket

import numpy as np
import pytest
import torch

from oracle import muon_step_ref
from tests.gpu_util import rel_fro
from workloads import WORKLOADS, WorkloadStream

pytestmark = pytest.mark.gpu

X_TOL = 1e-2          # a step from zero momentum
X_TOL_TRAJ = 2e-2     # later steps (see tests/test_gpu_parity.py)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


@pytest.fixture(scope="module")
def muon():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from newton_schulz_norm_b200 import build
    build.build()
    import newton_schulz_norm_b200 as m
    yield m
    assert m.status() == 0


@pytest.mark.parametrize("side_stream", [False, True])
def test_sharded_one_rank_nccl_against_oracle(muon, side_stream):
    import datetime
    import torch.distributed as dist
    from newton_schulz_norm_b200.sharded import ShardedMuon

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(_free_port())
    dist.init_process_group("nccl", rank=0, world_size=1, timeout=datetime.timedelta(seconds=60),
                            device_id=torch.device("cuda", torch.cuda.current_device()))
    try:
        wl = WORKLOADS["gpt2_block"]
        st = WorkloadStream(wl, seed=0)
        params, bufs = st.init()
        sm = ShardedMuon(wl.shapes, ns_steps=wl.ns_steps)
        for v, a in zip(sm.params, params):
            v.copy_(torch.from_numpy(a))
        p_ref, b_ref = params, bufs
        stream = torch.cuda.Stream() if side_stream else None
        for k in range(3):
            grads = st.next_grads()
            G = [torch.from_numpy(g).cuda() for g in grads]
            sm.step(G, lr=wl.lr, beta=wl.beta, nesterov=wl.nesterov, stream=stream)
            p_old = p_ref
            p_ref, b_ref = muon_step_ref(p_old, grads, b_ref, lr=wl.lr, beta=wl.beta,
                                         nesterov=wl.nesterov, ns_steps=wl.ns_steps)
            # read on torch's current stream: ordered after the exchange
            got = [v.cpu().numpy() for v in sm.params]
            tol = X_TOL if k == 0 else X_TOL_TRAJ
            for i in range(len(got)):
                assert rel_fro(got[i] - p_old[i], p_ref[i].astype(np.float64) - p_old[i]) <= tol
                assert np.max(np.abs(sm.bufs[i].cpu().numpy() - b_ref[i])) <= \
                    1e-6 * np.max(np.abs(b_ref[i]))
            # back onto the oracle's state, so that every step starts from identical inputs
            for i in range(len(got)):
                sm.params[i].copy_(torch.from_numpy(p_ref[i]))
                sm.bufs[i].copy_(torch.from_numpy(b_ref[i]))
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
