"""Context-parallel decode on CPU ranks (gloo, world size 2 and 3): each rank holds a
contiguous slab of every sequence's keys, decodes it, the (o, lse) parts are all-gathered
and merged; the result must equal the decode over the whole cache.  The kernels are
replaced by the oracle here (they are covered on the GPU); what runs is the sharding of
the lengths and the exchange."""
import os
import socket
import tempfile

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from exact_io_aware_81_b200.context_parallel import shard_seqlens

HERE = os.path.dirname(os.path.abspath(__file__))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_shard_seqlens():
    sl = torch.tensor([0, 1, 99, 100, 101, 250, 300], dtype=torch.int32)
    parts = [shard_seqlens(sl, r, 100) for r in range(3)]
    assert torch.equal(sum(p.to(torch.int64) for p in parts), sl.to(torch.int64))
    assert parts[1].tolist() == [0, 0, 0, 0, 1, 100, 100]
    assert parts[2].tolist() == [0, 0, 0, 0, 0, 50, 100]


@pytest.mark.parametrize("world", [2, 3])
def test_context_parallel_matches_whole_cache(world):
    import sys
    if HERE not in sys.path:
        sys.path.insert(0, HERE)
    import cp_worker
    with tempfile.TemporaryDirectory() as td:
        path = os.path.join(td, "res.npz")
        mp.start_processes(cp_worker.run, args=(world, _free_port(), path), nprocs=world,
                           start_method="spawn", join=True)
        r = np.load(path)
        assert np.allclose(r["o"], r["ro"], atol=1e-6, rtol=0)
        fin = np.isfinite(r["rl"])
        assert np.allclose(r["lse"][fin], r["rl"][fin], atol=1e-5, rtol=0)
        assert np.isneginf(r["lse"][~fin]).all() and (r["o"][0] == 0).all()
