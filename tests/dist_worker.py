"""One rank of the world_size-2 host test of bench.py's replica plumbing (gloo, CPU).

Launched by tests/test_bench_host.py through torch.distributed.run; reads RANK /
WORLD_SIZE / MASTER_* from the environment exactly as bench.py does under torchrun."""
import json
import os
import sys
import types

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

import bench  # noqa: E402


def main():
    out_dir = sys.argv[1]
    args = types.SimpleNamespace(gpus=2, steps=1, warmup=0, impl="reference",
                                 workload="14b_4x")
    rank, world, local, pg = bench.dist_setup(args)
    assert pg is not None and world == 2
    dev = torch.device("cpu")
    # per-rank times differ; every rank must see the maximum
    t = bench.max_over_ranks(10.0 + 5.0 * rank, pg, dev)
    bench.barrier(pg)
    # the reference arm runs on rank 0 only: other ranks return at once, with no work
    skipped = None
    if rank != 0:
        skipped = bench.run_reference(args, rank, world, local, pg) is None
    bench.barrier(pg)
    with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
        json.dump({"rank": rank, "world": world, "max": t, "skipped": skipped,
                   "backend": pg.get_backend()}, f)
    pg.destroy_process_group()


if __name__ == "__main__":
    main()
