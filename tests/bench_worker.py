"""Worker for the CPU (gloo) test of bench.py's max-over-ranks timing reduction."""
import os

import torch.distributed as dist


def run(rank, world, port, result_path):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        got = bench.max_over_ranks(1.5 + rank, world)   # rank r reports 1.5 + r ms
        bench.barrier(world)
        if rank == 0:
            with open(result_path, "w") as f:
                f.write(repr(got))
    finally:
        dist.destroy_process_group()
