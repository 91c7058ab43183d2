"""Worker for the CPU (gloo) context-parallel decode test: each rank decodes its shard of
the cache with the oracle and merges the gathered parts with the oracle's merge."""
import os

import numpy as np
import torch
import torch.distributed as dist


def run(rank, world, port, result_path):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import oracle
        from oracle.split_kv import merge_lse
        from exact_io_aware_81_b200 import inputs
        from exact_io_aware_81_b200.context_parallel import decode_context_parallel

        B, Hq, Hkv, Nmax, d = 4, 8, 2, 300, 32
        w = inputs.make_decode(B, Hq, Hkv, Nmax, d, seed=95, len_range=(0, Nmax))
        sl = torch.tensor([0, 40, 300, 151], dtype=torch.int32)
        C = -(-Nmax // world)
        kc = w.kcache[:, :, rank * C:(rank + 1) * C].contiguous()
        vc = w.vcache[:, :, rank * C:(rank + 1) * C].contiguous()

        def local(q, k, v, s, scale):
            o, l = oracle.decode(q, k, v, s, w.scale)
            return o.float(), l.float()

        def merge(op, lp, out_dtype):
            o, l = merge_lse(op.double().numpy(), lp.double().numpy())
            return torch.from_numpy(o), torch.from_numpy(l)

        o, lse = decode_context_parallel(w.q, kc, vc, sl, scale=w.scale, local_decode=local, merge=merge)
        if rank == 0:
            ro, rl = oracle.decode(w.q, w.kcache, w.vcache, sl, w.scale)
            np.savez(result_path, o=o.numpy(), lse=lse.numpy(), ro=ro.numpy(), rl=rl.numpy())
    finally:
        dist.destroy_process_group()
