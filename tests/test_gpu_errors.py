"""Device-side error reporting, without faulting, trapping or hanging the GPU.

The time-limit test withholds one internal signal (the score-ready arrive of the MMA
warp), so the softmax warps' bounded wait runs out after a short limit; the kernel must
record FA_ERR_TIMEOUT, stop every role at its next wait, free its tensor memory and
return, leaving the context usable for the normal call that follows.
"""
import pytest
import torch

import oracle
from exact_io_aware_81_b200 import inputs, ops
from parity import compare

pytestmark = pytest.mark.gpu


def test_wait_limit_expires_cleanly():
    w = inputs.make_prefill(1, 4, 4, 512, 512, 128, seed=12, causal=True)
    q, k, v = w.q.cuda(), w.k.cuda(), w.v.cuda()
    ops.set_wait_limit_ns(20_000_000)  # 20 ms
    try:
        ops.fwd_selftest_timeout(q, k, v, causal=True)
        assert ops.get_error() == ops.FA_ERR_TIMEOUT
        assert ops.get_error() == ops.FA_OK  # cleared
    finally:
        ops.set_wait_limit_ns(0)
    # the context still works
    o, lse = ops.fwd(q, k, v, causal=True, scale=w.scale)
    assert ops.get_error() == ops.FA_OK
    ro, rl = oracle.attn_fwd(w.q, w.k, w.v, w.scale, True)
    compare(o, lse, ro, rl, "after timeout")
