"""fa_decode_noalloc: the decode entry point for callers that cannot allocate device memory.

Plugins that only receive device pointers, serving loops that must not call cudaMalloc
(it can synchronise the device), and fully pre-reserved memory pools cannot hand the
library a workspace.  This entry point keeps the split-KV partials in a fixed scratch
array inside libfa.so instead.  The GPU test checks, through the C ABI, that two calls in
a row give the same output as fa_decode with a caller workspace, that the small case also
matches the fp64 oracle, and that a call leaves the device's free memory unchanged; the
host test checks that a problem larger than the scratch is refused before anything is
launched.

This file is collected last, so that a run stopping at the first failure has already run
every other test.
"""
import ctypes

import pytest
import torch

import oracle
from exact_io_aware_81_b200 import build, inputs, ops
from parity import O_MAX_ABS, O_MEAN_ABS, LSE_MAX_ABS, compare


def test_noalloc_refuses_problems_larger_than_its_scratch():
    build.build()
    lib = ops.load()
    B, Hq, Hkv, Nmax, d = 64, 64, 8, 8192, 128   # needs about 67 MB of scratch
    assert lib.fa_decode_workspace_size(B, Hq, Nmax, d) > ops.NOALLOC_SCRATCH_BYTES
    fake = 0x10000  # never dereferenced: the size check fails first
    rc = lib.fa_decode_noalloc(fake, fake, fake, fake, fake, None, B, Hq, Hkv, Nmax, d, 0.1, None)
    assert rc == ops.FA_ERR_WORKSPACE
    assert "scratch" in lib.fa_last_error_message().decode()


def _close(a, b, la, lb):
    err = (a.double() - b.double()).abs()
    assert err.max().item() <= O_MAX_ABS and err.mean().item() <= O_MEAN_ABS
    fin = torch.isfinite(lb)
    assert torch.equal(torch.isfinite(la), fin)
    assert (la[fin].double() - lb[fin].double()).abs().max().item() <= LSE_MAX_ABS


@pytest.mark.gpu
def test_noalloc_matches_workspace_decode_on_two_calls_in_a_row():
    dev = "cuda"
    lib = ops.load()
    # the full-size GQA decode workload, then a different, smaller one: the second call
    # must not be disturbed by what the first left in the shared scratch
    small = inputs.make_decode(3, 8, 2, 700, 64, seed=21, len_range=(0, 700))
    for w in (inputs.workload(5), small):
        B, Hq, Hkv, Nmax, d = w.shape
        assert lib.fa_decode_workspace_size(B, Hq, Nmax, d) <= ops.NOALLOC_SCRATCH_BYTES
        q, kc, vc, sl = w.q.to(dev), w.kcache.to(dev), w.vcache.to(dev), w.seqlens.to(dev)
        ref_o, ref_l = ops.decode(q, kc, vc, sl, scale=w.scale)
        stream = torch.cuda.current_stream().cuda_stream
        outs = []
        for call in range(2):
            o = torch.full((B, Hq, d), float("nan"), dtype=torch.bfloat16, device=dev)
            lse = torch.full((B, Hq), float("nan"), dtype=torch.float32, device=dev)
            torch.cuda.synchronize()
            free_before = torch.cuda.mem_get_info()[0]
            rc = lib.fa_decode_noalloc(q.data_ptr(), kc.data_ptr(), vc.data_ptr(), sl.data_ptr(),
                                       o.data_ptr(), lse.data_ptr(), B, Hq, Hkv, Nmax, d,
                                       ctypes.c_float(w.scale), stream)
            assert rc == ops.FA_OK, lib.fa_last_error_message()
            assert ops.get_error() == ops.FA_OK
            if call == 1:
                # the first call of a shape may load its kernels; the second allocates nothing
                assert torch.cuda.mem_get_info()[0] == free_before
            _close(o.cpu(), ref_o.cpu(), lse.cpu(), ref_l.cpu())
            outs.append((o.cpu(), lse.cpu()))
        assert torch.equal(outs[0][0], outs[1][0]) and torch.equal(outs[0][1], outs[1][1])
    ro, rl = oracle.decode(small.q, small.kcache, small.vcache, small.seqlens, small.scale)
    compare(outs[1][0], outs[1][1], ro, rl, "noalloc decode, small case")
