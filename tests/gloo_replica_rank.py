"""One rank of the replica test in ``test_replicas_gloo.py`` (CPU, gloo).

Launched by ``torch.distributed.run`` the way ``bench.py --gpus N`` is, so
that ``bench.dist_env`` reads RANK / WORLD_SIZE / LOCAL_RANK from the
environment.  Each rank times nothing: it feeds ``bench.max_over_ranks`` a
rank-dependent list of times, computes ``bench.job_rate`` from the result,
draws its replica's inputs, and writes what it saw to ``<out_dir>/rank<r>.json``.
"""
import datetime
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def main(out_dir: str) -> None:
    import torch
    import torch.distributed as dist

    import bench
    from workloads import WORKLOADS, TokenSource

    rank, world, local = bench.dist_env()
    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    try:
        times = [10.0 + rank, 4.0 * (rank + 1), 7.0 - rank]
        dist.barrier()
        reduced = bench.max_over_ranks(times, world, "cpu")
        rate = bench.job_rate(world, 1000, reduced[0])
        # each replica draws its own inputs (the salt is its rank)
        q, _, _ = TokenSource(WORKLOADS["tiny"], "cpu", salt=rank).get(0, 4)
        gathered = [torch.empty_like(q) for _ in range(world)]
        dist.all_gather(gathered, q)
        same_as_rank0 = bool(torch.equal(gathered[0], q))
        redraw = TokenSource(WORKLOADS["tiny"], "cpu", salt=rank).get(0, 4)[0]
        rec = {"rank": rank, "world": world, "local": local, "reduced": reduced,
               "rate": rate, "inputs_equal_rank0": same_as_rank0,
               "inputs_reproducible": bool(torch.equal(redraw, q))}
        with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
            json.dump(rec, f)
        dist.barrier()
    finally:
        dist.destroy_process_group()


if __name__ == "__main__":
    main(sys.argv[1])
