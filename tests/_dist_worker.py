"""Worker for the gloo multi-process tests (spawned, CPU only)."""
import datetime
import io
import os
import sys
from contextlib import redirect_stdout

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def run(rank, world, port, results):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        out = {}
        # the slowest rank's time is what every rank reports
        out["max"] = bench.max_over_ranks(world, 1.5 + rank)
        bench.barrier(world)
        # replicas draw different inputs of the same shape
        out["seed"] = bench.replica_seed(2, rank)
        # the reference arm prints on rank 0 only; other ranks do no work
        if rank != 0:
            buf = io.StringIO()

            class A:  # argparse stand-in
                steps, warmup, gpus = 1, 1, world
            with redirect_stdout(buf):
                bench.run_reference(A, world, rank)
            out["ref_stdout"] = buf.getvalue()
        results[rank] = out
    finally:
        dist.destroy_process_group()
