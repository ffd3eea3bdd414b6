"""The multi-process path of bench.py (one replica per GPU, no exchange on the
data path): the max-over-ranks timing and the whole-job throughput, run as
two gloo ranks on the CPU."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime

    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        dist.barrier()
        # rank r pretends its timed region took 10 + r ms for 5 steps
        ms = bench.max_over_ranks(10.0 + rank, torch.device("cpu"))
        tps = bench.whole_job_tokens_per_s(8192, world, ms / 5)
        q.put((rank, ms, tps))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2])
def test_max_over_ranks_and_throughput_gloo(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    slowest = 10.0 + (world - 1)
    for rank, ms, tps in res:
        assert ms == slowest
        assert tps == pytest.approx(world * 8192 / (slowest / 5 / 1e3))


def test_single_process_is_identity():
    import bench
    assert bench.max_over_ranks(3.5) == 3.5
    assert bench.whole_job_tokens_per_s(100, 1, 1.0) == pytest.approx(1e5)


def test_bench_gpus_flag_launches_that_many_ranks():
    """`bench.py --gpus 2` without torchrun re-runs itself as 2 ranks (here with
    a CPU stand-in for the GPU arm, gloo instead of NCCL); rank 0 alone prints
    one JSON line, with n_gpus = 2 and the slowest rank's time."""
    import json
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = {k: v for k, v in os.environ.items() if k not in ("RANK", "WORLD_SIZE", "LOCAL_RANK")}
    env["CUDA_VISIBLE_DEVICES"] = ""
    r = subprocess.run([sys.executable, os.path.join(root, "tests", "bench_rank_stub.py"),
                        "--gpus", "2", "--steps", "5", "--warmup", "3"],
                       capture_output=True, text=True, timeout=300, env=env)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout
    res = json.loads(lines[0])
    assert res["n_gpus"] == 2
    assert res["ms_per_step"] == pytest.approx(11.0 / 5)
    assert res["value"] == pytest.approx(2 * 8192 / (11.0 / 5 / 1e3))


def test_bench_rejects_a_world_size_other_than_gpus():
    import bench
    os.environ["WORLD_SIZE"] = "2"
    try:
        with pytest.raises(SystemExit):
            bench.main(["--gpus", "4"])
    finally:
        del os.environ["WORLD_SIZE"]
