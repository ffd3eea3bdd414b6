"""Expert parallelism (fine_grained_fp8_sigmoid_b200/ep.py) on the CPU: 2 and
4 gloo ranks, each with its own tokens and a shard of the routed experts, run
the real exchange logic (counts, then rows and scales, then outputs back;
all-reduce of the counts for the bias update) with a CPU stand-in for the
local kernels built on the oracle. Every rank's h' and the updated bias must
equal, bit for bit, the oracle's single-rank forward over all ranks' tokens.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import workloads
from fine_grained_fp8_sigmoid_b200.ep import split_plan
from oracle import moe as O
from oracle.e4m3 import round_bf16


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


class OracleOps:
    """The local steps of one rank in float64 on the CPU (oracle functions);
    the same interface as ep.GpuOps."""

    def __init__(self, E, weights):
        self.E = E
        self.w = {}              # local slot -> oracle-quantised expert
        self.weights = weights

    def load_expert(self, local_slot, w_gate, w_up, w_down):
        self.w[local_slot] = O.quantise_expert(*[t.double().numpy() for t in (w_gate, w_up, w_down)])

    def route(self, u, e, b, K):
        _, _, idx, gates = O.route(u.double().numpy(), e.double().numpy(), b.double().numpy(), K)
        return torch.from_numpy(idx.astype(np.int32)), torch.from_numpy(gates)

    def quant(self, u):
        q, s = O.quant_1x128(u.double().numpy())
        return torch.from_numpy(q), torch.from_numpy(s)

    def permute(self, idx, N, xq, xs):
        counts, offsets, st, inv = O.permute(idx.numpy().astype(np.int64), N)
        t = lambda a: torch.from_numpy(np.ascontiguousarray(a.astype(np.int32)))
        return t(counts), t(offsets), t(inv), xq[torch.from_numpy(st)], xs[torch.from_numpy(st)]

    def group_of_rows(self, offsets, modulo, n_rows):
        off = offsets.numpy()
        g = np.repeat(np.arange(len(off) - 1), np.diff(off))
        assert g.size == n_rows
        return torch.from_numpy((g % modulo).astype(np.int32))

    def experts(self, xq_perm, xs_perm, offsets, xq, xs):
        off = offsets.numpy()
        y = np.zeros((xq_perm.shape[0], xq.shape[1]))
        for g in range(self.E):
            if off[g + 1] > off[g]:
                y[off[g]:off[g + 1]], _ = O.expert_ffn(xq_perm[off[g]:off[g + 1]].numpy(),
                                                       xs_perm[off[g]:off[g + 1]].numpy(), self.w[g])
        ysh, _ = O.expert_ffn(xq.numpy(), xs.numpy(), self.w[self.E])
        # the expert outputs leave as bf16 values, as the GPU's do
        return torch.from_numpy(round_bf16(y)), torch.from_numpy(round_bf16(ysh))

    def gather_rows(self, src, idx):
        return src[idx.long()].contiguous()

    def combine(self, u, y_perm, y_shared, inv, gates):
        return torch.from_numpy(O.combine(u.double().numpy(), y_perm.numpy(), y_shared.numpy(),
                                          inv.numpy(), gates.numpy()))

    def bias_update(self, b, counts, T, K, gamma=0.001):
        nb, ratio = O.bias_update(b.double().numpy(), counts.numpy(), T, K, gamma)
        b.copy_(torch.from_numpy(nb).to(b.dtype))
        return torch.tensor([ratio])


def _rank(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime

    import torch.distributed as dist

    from fine_grained_fp8_sigmoid_b200.ep import ExpertParallelMoE
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=120))
    try:
        cfg = workloads.CONFIGS["tiny"]
        T = cfg.T // world
        u_all = workloads.activations(cfg)                  # 64 tokens, split over the ranks
        u = u_all[rank * T:(rank + 1) * T]
        e, b = workloads.centroids(cfg), workloads.bias(cfg).double()
        layer = ExpertParallelMoE(T, cfg.d, cfg.N_r, cfg.K_r, cfg.I, ops=OracleOps(cfg.N_r // world, None))
        for slot in range(cfg.N_r + 1):
            if layer.owns(slot):
                layer.load_expert(slot, *workloads.expert_weights(cfg, slot))
        out = layer.forward(u, e, b, update_bias=True)
        q.put((rank, out.numpy(), b.numpy(), layer.last["send"], layer.last["recv"],
               layer.last["local_counts"].numpy()))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_split_plan():
    # 2 ranks, 3 experts each: this rank sends 1+0+2 rows to rank 0 and 4+1+0
    # to rank 1, and receives (2, 0, 1) from rank 0 and (0, 3, 3) from rank 1
    send, recv, off = split_plan(np.array([1, 0, 2, 4, 1, 0]), np.array([[2, 0, 1], [0, 3, 3]]), 2, 3)
    assert send == [3, 5] and recv == [3, 6]
    assert off.tolist() == [0, 2, 2, 3, 3, 6, 9]


def test_split_plan_with_idle_ranks_and_experts():
    # 4 ranks, 2 experts each; this rank routes nothing to ranks 1 and 3, and
    # receives nothing at all from rank 2
    counts = np.array([5, 0, 0, 0, 1, 2, 0, 0])
    recv = np.array([[3, 0], [0, 0], [0, 0], [1, 7]])
    send, rv, off = split_plan(counts, recv, 4, 2)
    assert send == [5, 0, 3, 0] and rv == [3, 0, 0, 8]
    assert off.tolist() == [0, 3, 3, 3, 3, 3, 3, 4, 11]
    # nothing anywhere: all splits zero, offsets all zero
    send, rv, off = split_plan(np.zeros(8, np.int64), np.zeros((4, 2), np.int64), 4, 2)
    assert send == [0] * 4 and rv == [0] * 4 and off.tolist() == [0] * 9


@pytest.mark.parametrize("world", [2, 4])
def test_ep_ranks_match_single_rank_oracle(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted([q.get(timeout=300) for _ in range(world)], key=lambda x: x[0])
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0

    cfg = workloads.CONFIGS["tiny"]
    u = workloads.activations(cfg).double().numpy()
    e, b = workloads.centroids(cfg).double().numpy(), workloads.bias(cfg).double().numpy()
    quant = {s: O.quantise_expert(*[t.double().numpy() for t in workloads.expert_weights(cfg, s)])
             for s in range(cfg.N_r + 1)}
    ref = O.moe_forward(u, e, b, cfg.K_r, quant.__getitem__)
    T = cfg.T // world
    E = cfg.N_r // world
    for rank, out, b_new, send, recv, lcounts in res:
        assert np.array_equal(out, ref["out"][rank * T:(rank + 1) * T]), rank
        assert np.array_equal(b_new, ref["bias_new"]), rank
        # this rank's local experts received exactly the global load of each
        assert np.array_equal(lcounts, ref["counts"][rank * E:(rank + 1) * E]), rank
        assert sum(send) == T * cfg.K_r
    # what rank i sent to rank j is what rank j received from rank i
    for i in range(world):
        for j in range(world):
            assert res[i][3][j] == res[j][4][i]
