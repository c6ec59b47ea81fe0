"""Matrix-sharded Muon on one GPU through a one-rank NCCL process group: the
owned-matrix step and the in-place all-gather give exactly what one plain
muon.step over all matrices gives."""
import os
import socket

import pytest
import torch

from workloads import WORKLOADS, WorkloadStream

pytestmark = pytest.mark.gpu


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


def test_sharded_one_rank_nccl_equals_plain_step(muon):
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
        P = [torch.from_numpy(a).cuda() for a in params]
        B = [torch.from_numpy(b).cuda() for b in bufs]
        for _ in range(3):
            G = [torch.from_numpy(g).cuda() for g in st.next_grads()]
            sm.step(G, lr=wl.lr, beta=wl.beta, nesterov=wl.nesterov)
            muon.step(P, G, B, lr=wl.lr, beta=wl.beta, nesterov=wl.nesterov, ns_steps=wl.ns_steps)
        torch.cuda.synchronize()
        for a, b in zip(sm.params, P):
            assert torch.equal(a, b)
        for i in sm.owned:
            assert torch.equal(sm.bufs[i], B[i])
    finally:
        dist.destroy_process_group()
