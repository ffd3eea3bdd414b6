"""Expert parallelism on the GPU through NCCL, as one rank (the pool gives one
GPU per run, and ranks whose kernels wait on one another must not share a
GPU): the all-to-alls then exchange with this rank only, but every step of the
EP path runs (moe_group_of_rows, the second moe_permute, moe_grouped_gemm_fp8_rows,
moe_gather_rows, NCCL all-to-all and all-reduce). Its h', expert outputs and
bias update equal MoELayerFP8's bit for bit. Multi-rank exchange logic is
covered on the CPU by tests/test_ep.py."""
import datetime
import socket

import pytest
import torch

import workloads

pytestmark = pytest.mark.gpu


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.fixture()
def nccl_world1():
    import torch.distributed as dist
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{_free_port()}", rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60), device_id=torch.device("cuda", 0))
    try:
        yield
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("name,T", [("tiny", None), ("mid", None), ("decode", 37)])
def test_ep_single_rank_equals_layer(lib, nccl_world1, name, T):
    from fine_grained_fp8_sigmoid_b200 import MoELayerFP8
    from fine_grained_fp8_sigmoid_b200 import binding as B
    from fine_grained_fp8_sigmoid_b200.ep import ExpertParallelMoE
    cfg = workloads.CONFIGS[name]
    if T is not None:
        cfg = cfg.with_tokens(T)
    dev = torch.device("cuda", 0)
    u = workloads.activations(cfg, device=dev)
    e = workloads.centroids(cfg, device=dev)
    b = workloads.bias(cfg, device=dev)
    plain = MoELayerFP8(cfg.T, cfg.d, cfg.N_r, cfg.K_r, cfg.I, gather=False)
    ep = ExpertParallelMoE(cfg.T, cfg.d, cfg.N_r, cfg.K_r, cfg.I)
    for slot in range(cfg.N_r + 1):
        w = workloads.expert_weights(cfg, slot, device=dev)
        plain.load_expert(slot, *w)
        ep.load_expert(slot, *w)
    b1, b2 = b.clone(), b.clone()
    ref = plain.forward(u, e, b1).clone()
    out = ep.forward(u, e, b2)
    torch.cuda.synchronize()
    assert B.moe_get_error() == 0
    assert torch.equal(out, ref)
    assert torch.equal(ep.last["y_perm"], plain.y_perm)
    assert torch.equal(ep.last["y_shared"], plain.y_shared)
    assert torch.equal(b2, b1)
    assert ep.last["send"] == [cfg.T * cfg.K_r] and ep.last["recv"] == [cfg.T * cfg.K_r]
