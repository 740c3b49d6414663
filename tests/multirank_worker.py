"""Worker for the two-rank CPU test of bench.py's multi-process path (run under torchrun
with the gloo backend; not a test module itself).  Rank 0 prints one JSON line."""
import datetime
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def main():
    import torch
    import torch.distributed as dist

    import bench
    import synth
    world, rank = int(os.environ["WORLD_SIZE"]), int(os.environ["RANK"])
    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    bench.barrier(world)
    # each rank reports a different time: every rank must see the slowest one
    ms = bench.max_over_ranks(100.0 + 25.0 * rank, world)
    # replicas: each rank draws its own inputs (seed + rank), as bench.py does
    ids = synth.uniform_ids((1, 256), 248320, 0 + rank)
    got = [torch.empty_like(ids) for _ in range(world)]
    dist.all_gather(got, ids)
    distinct = not torch.equal(got[0], got[1])
    value = bench.weak_scaling_value(8192, world, ms)
    # the reference arm: ranks other than 0 return at once, without work or output
    class A:
        steps, warmup, ref_tokens, gpus = 1, 0, 1, world
    if rank != 0:
        bench.run_reference(A, world, rank)
    ok = torch.tensor([1 if distinct else 0])
    dist.all_reduce(ok, op=dist.ReduceOp.MIN)
    if rank == 0:
        print(json.dumps({"world": world, "max_ms": ms, "distinct": bool(ok.item()), "value": value}), flush=True)
    bench.barrier(world)
    dist.destroy_process_group()


if __name__ == "__main__":
    main()
