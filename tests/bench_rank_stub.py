"""bench.py's rank launcher and rank plumbing with a CPU stand-in for the GPU
arm (run by tests/test_multi_rank.py, not collected by pytest): each rank
pretends its timed region took 10 + rank ms for the requested steps."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def cpu_stand_in(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist
    assert dist.is_initialized() and dist.get_world_size() == world == args.gpus
    ms = bench.max_over_ranks(10.0 + rank, torch.device("cpu"))
    if rank != 0:
        return None
    return {"metric": bench.METRIC, "value": bench.whole_job_tokens_per_s(8192, world, ms / args.steps),
            "unit": "tokens/s", "n_gpus": world, "steps": args.steps, "ms_per_step": ms / args.steps}


if __name__ == "__main__":
    bench.run_ours = cpu_stand_in
    bench.main()
